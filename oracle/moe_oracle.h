/*
 * moe_oracle.h -- plain, slow CPU oracle of the routed MoE FFN forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this library.  It shares no code with the
 * CUDA path and the CUDA path never calls it.
 *
 * What it follows (page = the web pages this layer is defined by):
 *   - LightMoE README, "MoE inference": one call does dispatch, input
 *     quantisation, gate/up projection, gated activation, requantisation of
 *     the hidden, down projection, routing-weight application, deterministic
 *     combine.  "Grouped GEMM": expert-major rows, m_indptr of length E+1,
 *     zero-size experts valid.  "Standalone GEMM": NVFP4 = packed E2M1 values,
 *     E4M3 block scales, one fp32 per-tensor scale.
 *   - pure-Triton fused MoE article: gate and up share one input row, SiLU of
 *     the gate times up; block-id -> (expert, row offset) schedule.
 *   - Alpha-MoE article: FP8 W8A8 (e4m3 weights and activations).
 *   - RaMP abstract: the schedule is a grid of tiles over the runtime expert
 *     histogram.
 * Where the pages leave a step open, the reading taken is stated beside the
 * function that implements it.
 *
 * Floating point: dequantised operands are exact in fp64, dot products and the
 * SwiGLU are fp64; the router logits and every quantiser are fp32 with the
 * rounding written out below, because their results decide integers.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_SCORE_SOFTMAX = 0, ORC_SCORE_SIGMOID = 1 };
enum { ORC_FMT_FP8_ROW = 0, ORC_FMT_FP8_BLOCK128 = 1, ORC_FMT_NVFP4 = 2, ORC_FMT_MX32 = 3 };
enum { ORC_TILE_M = 128 };

/* ---- codecs (OCP FP8 E4M3 "fn" and FP4 E2M1, round to nearest even, saturating) ---- */
double  orc_e4m3_value(uint8_t code);      /* NaN for 0x7F/0xFF */
uint8_t orc_e4m3_encode(float x);          /* nearest value, ties to even code, |x|>=448 -> 448 */
double  orc_e2m1_value(uint8_t code);      /* low 4 bits used */
uint8_t orc_e2m1_encode(float x);          /* nearest of +-{0,.5,1,1.5,2,3,4,6}, ties to even */
void    orc_e4m3_encode_n(const float* x, int64_t n, uint8_t* out);
void    orc_e2m1_encode_n(const float* x, int64_t n, uint8_t* out);

/* ---- router ----
 * logits[t*E+e] = canonical fp32 dot of X row t (bf16 bits) with Wr row e, then
 * + bias[e] (fp32) when bias != NULL.  Canonical order: H = 256*n; lane l in
 * [0,32) owns h = 256*i + 8*l + j (i ascending, then j = 0..7) and runs one
 * fmaf chain from +0.0f; the 32 lane sums are added as a balanced pairwise
 * tree ((p0+p1)+(p2+p3))+... */
void orc_router_logits(const uint16_t* x, int T, int H, const float* wr,
                       const float* bias, int E, float* logits);
/* fp64 dot products, for the error bound check of the canonical order */
void orc_router_logits_f64(const uint16_t* x, int T, int H, const float* wr,
                           const float* bias, int E, double* logits);
/* top-k: the k largest logits, larger first, equal logits -> lower expert id;
 * w = softmax over the selected logits, or sigmoid of each normalised to sum 1. */
void orc_topk(const float* logits, int T, int E, int k, int score,
              int32_t* ids, double* w);

/* ---- dispatch ----
 * counts[e] = #assignments to e; offsets = exclusive prefix sum (E+1, the
 * m_indptr); slot of (t,j) = offsets[e] + #{(t',j') before (t,j) in row-major
 * order with the same expert}; perm[slot] = t*k+j, inv[t*k+j] = slot.
 * tiles: per expert ceil(count/128) row tiles in expert order, entry =
 * (expert, first row); returns the number of tiles. */
void orc_dispatch(const int32_t* ids, int T, int k, int E, int32_t* counts,
                  int32_t* offsets, int32_t* perm, int32_t* inv);
int  orc_schedule(const int32_t* offsets, int E, int32_t* tile_expert, int32_t* tile_row);

/* ---- down GEMM tile choice (wave cost model over the expert histogram) ----
 * RaMP abstract: the configuration is picked from the expert histogram seen at
 * run time by a cost model of CTA waves with four fitted parameters, which
 * looks at nothing but the geometry of the CTA grid.
 * Candidates c = 0, 1, 2 have BN = 256, 128, 64 output columns per tile.  With
 * m_tiles = sum_e ceil(counts[e]/128) and touched = #{e : counts[e] > 0}:
 *   tiles  = m_tiles * (H / BN)
 *   t_mma  = ceil(tiles / num_sms) * (I / 128) * (alpha + beta * BN)
 *   t_load = touched * H * I * 1e6 / (min(tiles, num_sms) * bw)   (0 if no tiles)
 *   cost   = gamma + max(t_mma, t_load)           (all integer; / truncates)
 * Returns the c of the lowest cost, the lower c on equal costs. */
int orc_pick_down_tile(const int32_t* counts, int E, int H, int I, int num_sms,
                       int64_t alpha, int64_t beta, int64_t bw, int64_t gamma, int64_t* costs);
/* K split of the FP8_ROW down GEMM (1 = none) from the expert histogram. */
int orc_pick_split(const int32_t* counts, int E, int split_nb, int split_kb, int64_t o_rows, int num_sms);
/* Mode of the gated FP8_ROW gate/up GEMM from the expert histogram (RaMP
 * abstract: the configuration comes from the runtime histogram through a
 * cost model of CTA waves): 0 single CTAs on 256-wide tiles, 1 CTA pairs, 2
 * single CTAs on 128-wide tiles.  mt_e = ceil(counts[e] / 128) m-tiles per
 * expert, m_tiles their sum, n_odd the number of experts with an odd mt_e.
 * Mode 0 has m_tiles nb units, num_sms at once; mode 1 (m_tiles + n_odd) / 2 nb
 * units (pairs of an expert's m-tiles), num_sms / 2 at once; mode 2
 * 2 m_tiles nb units, num_sms at once.  cost_m = ceil(units_m / at_once_m)
 * (kb ps[2m] + ps[2m+1]) in integers.  The cheapest mode whose bit is set in
 * allow wins, ties to the lower mode; 0 when nb <= 0, the histogram is empty
 * or no mode is allowed. */
int orc_pick_gu_mode(const int32_t* counts, int E, int nb, int kb, int num_sms, int allow, const int64_t* ps);

/* ---- activation quantisation of token rows (X or the hidden) ----
 * FP8_ROW:      one fp32 scale per row: s = fp32(amax/448), q = e4m3(fp32(x/s)),
 *               q = 0 when s == 0.  scales: [rows]
 * FP8_BLOCK128: the same per 128-column block.  scales: [rows, K/128] fp32
 * MX32:         e4m3 codes with a power-of-two scale 2^e per 32-column block (OCP MX
 *               style, UE8M0 code e + 127): e is the smallest integer with
 *               amax_b <= 448 * 2^e (e = -127 when amax_b == 0, clamped to [-127, 127]);
 *               q = e4m3(x * 2^-e).  scales: [rows, K/32] uint8 codes.
 * NVFP4:        g given (fp32, > 0); per 16-column block b: sb = e4m3(fp32(fp32(amax_b/6)/g)),
 *               d = fp32(value(sb)*g), q = e2m1(fp32(x/d)) (q = 0 when d == 0).
 *               codes packed two per byte, element 2i in the low nibble;
 *               scales: [rows, K/16] e4m3 codes (uint8).
 * x is fp32 [rows, K]. */
void orc_quant_rows(int fmt, const float* x, int rows, int K, float g,
                    uint8_t* codes, void* scales);
/* NVFP4 global scale of a tensor: fp32(amax/2688) */
float orc_nvfp4_global(const float* x, int64_t n);

/* ---- expert weights in the plain layout ---- */
typedef struct {
    const uint8_t* q;  /* codes [E_w, N, K] (fp8) or [E_w, N, K/2] (e2m1) */
    const void*    s;  /* FP8_ROW [E_w, N] fp32; BLOCK128 [E_w, N/128, K/128] fp32; NVFP4 [E_w, N, K/16] e4m3 */
    const float*   g;  /* NVFP4 global [E_w] fp32, else NULL */
} orc_proj;

typedef struct {
    int H, I, E, k, score, fmt;
    float hidden_global;   /* NVFP4 static hidden scale */
    orc_proj gate, up, down;   /* gate/up: N=I, K=H.  down: N=H, K=I */
    const int32_t* expert_slot; /* [E] -> index into the weight arrays, -1 = not provided; NULL = identity */
    int act;               /* gated activation, ORC_ACT_* */
    double act_alpha, act_limit;
    int hidden_rule;       /* ORC_HIDDEN_*: how the hidden is requantised */
} orc_layer;

/* Requantisation rule of the hidden (the SwiGLU output).  The workloads ask
 * for activations "dynamically quantised per token"; a GEMM epilogue that sees
 * one block of hidden columns at a time cannot take a row's amax, so the layer
 * uses block scales (ORC_HIDDEN_LAYER: MX32 for FP8_ROW, 1x128 fp32 for
 * FP8_BLOCK128, NVFP4 16-blocks for NVFP4).  ORC_HIDDEN_PER_TOKEN is the
 * literal reading, for comparison only (FP8 formats): one fp32 scale per
 * hidden row, s = fp32(amax/448), q = e4m3(fp32(h/s)), the FP8_ROW rule of X. */
enum { ORC_HIDDEN_LAYER = 0, ORC_HIDDEN_PER_TOKEN = 1 };

/* Gated activations h = act(g, u) of the expert MLP, in fp64 (LightMoE README,
 * "Compatibility": SwiGLU, bounded SwiGLU, SwiGLU-OAI, GeGLU, ReGLU).
 *   SWIGLU          silu(g) u,  silu(g) = g / (1 + exp(-g))
 *   SWIGLU_BOUNDED  silu(min(g, L)) clamp(u, -L, L)
 *   SWIGLU_OAI      g' / (1 + exp(-alpha g')) (u' + 1),  g' = min(g, L), u' = clamp(u, -L, L)
 *   GEGLU           g Phi(g) u,  Phi(g) = (1 + erf(g / sqrt 2)) / 2
 *   REGLU           max(g, 0) u
 *   RELU2           max(u, 0)^2; the expert has no gate projection (two weights,
 *                   LightMoE README "MoE inference": ReLU^2 experts load up and down) */
enum { ORC_ACT_SWIGLU = 0, ORC_ACT_SWIGLU_BOUNDED = 1, ORC_ACT_SWIGLU_OAI = 2, ORC_ACT_GEGLU = 3, ORC_ACT_REGLU = 4,
       ORC_ACT_RELU2 = 5 };
double orc_glu(int act, double alpha, double limit, double g, double u);

/* dequantised weight row (fp64, exact) */
void orc_weight_row(const orc_layer* L, const orc_proj* P, int N, int K, int e, int n, double* out);

/* One expert on quantised input rows.
 *   a_codes/a_scales: rows of the quantised input in the layer's format (K = H)
 *   x_global: NVFP4 global scale of the input (ignored otherwise)
 *   The hidden is requantised with the MX32 rule (power-of-two scale per 32
 *   columns) for FP8_ROW, per (row, 128-column block) with fp32 scales for
 *   FP8_BLOCK128, and with the NVFP4 rule and the static hidden_global scale
 *   for NVFP4; with hidden_rule = ORC_HIDDEN_PER_TOKEN (FP8 formats) by the
 *   FP8_ROW rule over the whole row (hq_scales then [rows] fp32).
 *   outputs: h (fp64 SwiGLU output before requantisation, [rows, I]) may be NULL;
 *            hq codes/scales (requantised hidden) may be NULL;
 *            o [rows, H] fp64 down projection of the dequantised hidden. */
void orc_expert_rows(const orc_layer* L, int e, int rows, const uint8_t* a_codes,
                     const void* a_scales, float x_global, double* h,
                     uint8_t* hq_codes, void* hq_scales, double* o);

/* Down projection alone of quantised hidden rows (hidden format) -> o [rows, H] fp64 */
void orc_down_rows(const orc_layer* L, int e, int rows, const uint8_t* h_codes,
                   const void* h_scales, double* o);

/* Whole layer for a subset of tokens.
 *   x [T, H] bf16 bits, wr [E, H], bias [E] or NULL.
 *   routing for all T tokens is computed and written to ids [T*k], w [T*k];
 *   y_sel [n_sel, H] fp64 = sum_j w_j * o_j for the tokens sel[0..n_sel).
 *   For NVFP4 the input global scale is taken over all T tokens.
 *   Returns 0, or -1 when a selected token needs an expert whose weights were
 *   not provided. */
int orc_moe_forward(const orc_layer* L, const uint16_t* x, int T, const float* wr,
                    const float* bias, int n_sel, const int32_t* sel,
                    int32_t* ids, double* w, double* y_sel);

/* threads the oracle uses (OpenMP), for the baseline report */
int orc_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
