/*
 * moe_b200.h -- C ABI of the routed Mixture-of-Experts FFN forward pass on one
 * NVIDIA B200 (sm_100a).
 *
 * The layer (LightMoE README, "MoE inference"; Alpha-MoE article, "How the
 * megakernel works"): given tokens X[T,H], router weights Wr[E,H] (+ optional
 * per-expert bias), and per expert quantised W_gate, W_up [I,H] and W_down [H,I]
 * with their scales, return
 *     Y[t] = sum_{j<k} w[t,j] * W_down[e_j] q( SiLU(W_gate[e_j] q(x_t)) * (W_up[e_j] q(x_t)) )
 * where e_j are the k experts with the largest router logits (ties -> lower
 * expert id), w the softmax (or sigmoid) of those k logits normalised to sum 1,
 * and q() the activation quantiser of the layer's format.
 *
 * Conventions for every entry point:
 *   - All pointers named *device* are device addresses owned by the caller; the
 *     library never allocates device memory.  A warmed call does not allocate
 *     (LightMoE README, "Standalone GEMM": the caller owns the output).
 *   - Device pointers must be 256-byte aligned (torch allocations are).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Argument errors return at once and launch nothing.  Errors seen
 *     by a kernel (a bounded wait that ran out, an index out of range) go to a
 *     status word inside the workspace; moe_get_status() reports them.
 *   - One workspace per concurrent stream (LightMoE README, "MoE inference":
 *     one plan per concurrent CUDA stream, its workspaces are reused).
 *   - Shape limits (LightMoE README, "Limits", caps the experts of a layer at
 *     256 and its token-expert pairs at 131,072, with K aligned): H a multiple of 256,
 *     I a multiple of 128, 1 <= k <= 8, k <= E <= 256, max_T * k <= 131072.
 *     Otherwise MOE_ERR_UNSUPPORTED_SHAPE.
 *   - moe_last_error() returns a thread-local message for the last failure.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t;   /* same type as cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,
    MOE_ERR_UNSUPPORTED_SHAPE = 2,
    MOE_ERR_WORKSPACE_TOO_SMALL = 3,
    MOE_ERR_CUDA = 4,
    MOE_ERR_DEVICE_TIMEOUT = 5,
    MOE_ERR_DEVICE_BOUNDS = 6
} moe_status;

/* score function of the router (LightMoE README, "MoE inference": top_k_weights) */
enum { MOE_SCORE_SOFTMAX = 0,    /* softmax over the selected k logits */
       MOE_SCORE_SIGMOID = 1 };  /* sigmoid of each selected logit, normalised to sum 1 */

/* quantisation format of weights, activations and hidden (Alpha-MoE article:
 * FP8 W8A8; LightMoE README, "Standalone GEMM": NVFP4 = E2M1 values, E4M3
 * block scales, one fp32 per-tensor scale) */
enum { MOE_FMT_FP8_ROW = 0,      /* e4m3; fp32 scale per weight row and per token; the hidden with a
                                    power-of-two (UE8M0) scale per 32 columns (MX) */
       MOE_FMT_FP8_BLOCK128 = 1, /* e4m3; fp32 scale per 128x128 weight block, per (token, 128 cols) of X
                                    and of the hidden */
       MOE_FMT_NVFP4 = 2 };      /* e2m1; e4m3 scale per 16 along K; fp32 global per tensor (the hidden's
                                    is the static hidden_global_scale) */

typedef struct {
    int H, I, E, k;
    int score;                    /* MOE_SCORE_* */
    int fmt;                      /* MOE_FMT_* */
    int has_bias;                 /* router logits get + bias[e] */
    int max_T;                    /* largest T a workspace must hold */
    float hidden_global_scale;    /* NVFP4 only: static fp32 scale of the hidden (a checkpoint
                                     scale, LightMoE README "set_activation_scales") */
    int act;                      /* MOE_ACT_*, the gated activation h = act(gate, up) */
    float act_alpha;              /* SWIGLU_OAI: sigmoid slope alpha */
    float act_limit;              /* SWIGLU_BOUNDED, SWIGLU_OAI: clamp limit L > 0 */
} moe_config;

/* Gated activations of the expert MLP (LightMoE README, "Compatibility": complete
 * inference supports bounded SwiGLU, SwiGLU-OAI, GeGLU and ReGLU besides SwiGLU;
 * "MoE inference": activation_clamp for bounded SwiGLU).  The pages name them
 * without formulas; the forms computed are, with silu(g) = g / (1 + e^-g):
 *   SWIGLU          silu(g) * u
 *   SWIGLU_BOUNDED  silu(min(g, L)) * clamp(u, -L, L)
 *   SWIGLU_OAI      g' / (1 + e^(-alpha g')) * (u' + 1),  g' = min(g, L), u' = clamp(u, -L, L)
 *   GEGLU           0.5 g (1 + erf(g / sqrt 2)) * u
 *   REGLU           max(g, 0) * u
 *   RELU2           max(u, 0)^2 with no gate projection: two weights per expert
 *                   (README "MoE inference": ReLU^2 experts load up and down);
 *                   moe_weights.gate_* may be NULL; needs I % 256 == 0
 * moe_init returns MOE_ERR_INVALID_ARG for an unknown act, L <= 0 where a
 * limit is used, or alpha <= 0 for SWIGLU_OAI; MOE_ERR_UNSUPPORTED_SHAPE for
 * RELU2 with I not a multiple of 256. */
enum {
    MOE_ACT_SWIGLU = 0,
    MOE_ACT_SWIGLU_BOUNDED = 1,
    MOE_ACT_SWIGLU_OAI = 2,
    MOE_ACT_GEGLU = 3,
    MOE_ACT_REGLU = 4,
    MOE_ACT_RELU2 = 5
};

typedef struct moe_handle moe_handle;

/* Quantised expert weights in the plain layout (device pointers), per projection:
 *   q: codes, [E, N, K] uint8 e4m3, or [E, N, K/2] uint8 e2m1 (element 2i in the low nibble)
 *   s: FP8_ROW [E, N] fp32; FP8_BLOCK128 [E, N/128, K/128] fp32; NVFP4 [E, N, K/16] e4m3 codes
 *   g: NVFP4 [E] fp32 global scales, else NULL
 * gate and up have N = I, K = H; down has N = H, K = I. */
typedef struct {
    const void* gate_q; const void* gate_s; const float* gate_g;
    const void* up_q;   const void* up_s;   const float* up_g;
    const void* down_q; const void* down_s; const float* down_g;
} moe_weights;

/* Device addresses of the intermediates inside a workspace (for inspection and
 * for feeding one step alone).  Row counts use A = max_T * k.
 *
 * Row layouts of xq/xs and hq/hs.  "Slot order": row = slot (the dispatch's
 * expert-major position of an assignment), with 128 spare rows at the end.
 * "Padded": every expert's rows start on a 128-row boundary, so that a row tile
 * owns whole scale chunks: row = 128 * tile_ptr[e] + (slot - offsets[e]), with
 * A + 128 E rows in all.  "Chunked" scale bytes: the scale of (row r, column
 * block c) sits at byte ((r / 128) * (cols / 4) + c / 4) * 512
 * + (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4, cols = scale columns per row
 * (the layout the block-scaled tensor-core MMAs read).
 *   format        xq / xs                                hq / hs
 *   FP8_ROW       slot order: [A+128, H] e4m3,            padded: [A+128E, I] e4m3,
 *                 [A+128] fp32 per row                   chunked UE8M0 codes, I/32 per row
 *                                                        (value = code * 2^(scale - 127))
 *   FP8_BLOCK128  slot order: [A+128, H] e4m3,            slot order: [A+128, I] e4m3,
 *                 [A+128, H/128] fp32                    [A+128, I/128] fp32
 *   NVFP4         padded: [A+128E, H/2] e2m1 (2 per      padded: [A+128E, I/2] e2m1,
 *                 byte, low nibble first), chunked e4m3  chunked e4m3 codes, I/16 per row
 *                 codes, H/16 per row                    (x hidden_global_scale)
 *                 (x the global scale amax|X| / 2688)
 */
typedef struct {
    int32_t* status;     /* [64] status[0] = first device error (moe_status), status[1] = where */
    int32_t* ids;        /* [A] router top-k expert ids, token-major [T, k] */
    float*   w;          /* [A] routing weights [T, k] */
    int32_t* counts;     /* [E] assignments per expert */
    int32_t* offsets;    /* [E+1] exclusive prefix sum of counts (m_indptr) */
    int32_t* num_tiles;  /* [1] row tiles of 128 over all experts */
    int32_t* tile_ptr;   /* [E+1] index of each expert's first row tile */
    int32_t* pick;       /* [3] choices from the histogram: [0] down GEMM tile (0 -> 256, 1 -> 128, 2 -> 64
                          * columns, FP8_BLOCK128); [1] S, the K split of the FP8_ROW down GEMM (1 = none);
                          * [2] the gated FP8_ROW gate/up GEMM's mode: 0 single CTAs, 256-wide
                          * tiles; 1 CTA pairs; 2 single CTAs, 128-wide tiles */
    int32_t* tiles;      /* [A/128 + E + 1][2] (expert, first row) per row tile */
    int32_t* perm;       /* [A] slot -> t*k + j */
    int32_t* inv;        /* [A] t*k + j -> slot */
    float*   x_global;   /* [1] NVFP4: amax |X| over the batch (fp32); X's global scale is amax / 2688 */
    uint8_t* xq;         /* quantised X rows, one per assignment (layout above) */
    void*    xs;         /* scales of xq (layout above) */
    uint8_t* hq;         /* requantised hidden, one row per assignment (layout above) */
    void*    hs;         /* scales of hq (layout above) */
    uint16_t* o;         /* [S][T*k, H] fp16 down projection times routing weight, slot order, each
                          * 32-column block scaled by 2^(15 - o_exp): value = fp16 * 2^(o_exp - 15).
                          * With a K split (pick[1] = S > 1) copy s holds split s's partial sums.
                          * FP8_ROW workspaces hold A + 7 min(A, 256) rows so small batches can split. */
    float*   logits;     /* [max_T, E] fp32 router logits (bias included) of the last moe_route: the
                          * canonical logit for every expert that could be among a token's top k (all
                          * experts up to 128 tokens or with at most 8 experts); above that, the
                          * integer tensor-core approximation for the others (router_tc.cuh) */
    int8_t*  o_exp;      /* [S][T*k, H/32] the block exponents of o */
} moe_workspace_view;

const char* moe_last_error(void);

/* Validate cfg and create a handle (host memory only; queries the current device). */
moe_status moe_init(const moe_config* cfg, moe_handle** out);
moe_status moe_destroy(moe_handle* h);

/* Bytes of the packed expert weights / of one workspace (sized by cfg.max_T). */
moe_status moe_weights_size(const moe_handle* h, size_t* bytes);
moe_status moe_workspace_size(const moe_handle* h, size_t* bytes);
/* Fill `view` with the addresses of the regions of workspace `ws` (no device work). */
moe_status moe_workspace_view_get(const moe_handle* h, void* ws, moe_workspace_view* view);

/* Rearrange plain-layout weights into the packed device layout the GEMMs read
 * (gate and up interleaved in row blocks, 128 + 128 rows for the FP8 formats
 * and 64 + 64 for NVFP4, so one tile holds both).  Not on
 * the timed path (LightMoE README, "Installation": packing outside latency). */
moe_status moe_pack_weights(const moe_handle* h, const moe_weights* src, void* packed,
                            moe_stream_t stream);

/* Router + top-k (Alpha-MoE article: routing is one of the fused stages;
 * LightMoE README "MoE inference": int32 ids, fp32 weights).
 *   x [T, H] bf16, wr [E, H] fp32, bias [E] fp32 (NULL unless has_bias)
 *   -> ids [T, k] int32 (larger logit first, ties -> lower id), w [T, k] fp32.
 * Logits are fp32 in one fixed order: lane l of 32 owns h = 256 i + 8 l + j and
 * runs one fused multiply-add chain over i then j; the 32 lane sums are added as
 * a balanced pairwise tree; then + bias[e].  So ids are reproducible bit for bit. */
moe_status moe_route(const moe_handle* h, const void* x, int T, const float* wr,
                     const float* bias, int32_t* ids, float* w, void* ws, moe_stream_t stream);

/* Deterministic expert-major dispatch (LightMoE README, "Grouped GEMM" m_indptr
 * and "MoE training" MoEDispatch; pure-Triton article: block-id -> (expert,
 * offset) map): counts, offsets, the row-tile schedule, the stable slot of each
 * (t, j) in row-major order, and the quantised X rows written to their slots
 * (LightMoE README: BF16 input quantisation).  ids may be caller-provided. */
moe_status moe_dispatch(const moe_handle* h, const void* x, const int32_t* ids, int T,
                        void* ws, moe_stream_t stream);

/* moe_dispatch without a workspace.  The pages have no counterpart of this
 * entry point; it exists for callers that cannot allocate device memory at
 * all, e.g. a layer running inside a host framework that owns every device
 * allocation and passes it only input and output buffers.  The dispatch's
 * only scratch (per-chunk expert counts) lives in a 128 KB array inside this
 * library that every GPU loading the library holds until the process exits.
 *   Outputs, all device memory owned by the caller, with A = T*k:
 *     counts [E], offsets [E+1], num_tiles [1], tiles [A/128 + E + 1][2],
 *     perm [A], inv [A], xq [A, H] e4m3, xs [A] (FP8_ROW) or [A, H/128]
 *     (FP8_BLOCK128) fp32, status [2] (zeroed by the call, then status[0] =
 *     MOE_ERR_DEVICE_BOUNDS if an id was out of range).
 *   Same results as moe_dispatch.  T*k may not exceed 131072, whatever E and
 *   max_T are, and the format must be FP8 (else MOE_ERR_UNSUPPORTED_SHAPE).
 *   Every call made outside stream capture looks up the array's device
 *   address on the current device (so a cudaDeviceReset between calls is
 *   harmless); a call under capture reuses the address of the last uncaptured
 *   call on that device, so make the first call on a device before any stream
 *   capture (a first call under capture returns MOE_ERR_INVALID_ARG).  The
 *   array is shared by every call on the device and
 *   keeps the last call's contents, so calls whose kernels overlap on the GPU
 *   (other streams, other threads) race: serialise them.  No allocation. */
moe_status moe_dispatch_noalloc(const moe_handle* h, const void* x, const int32_t* ids, int T,
                                int32_t* counts, int32_t* offsets, int32_t* num_tiles, int32_t* tiles,
                                int32_t* perm, int32_t* inv, uint8_t* xq, void* xs, int32_t* status,
                                moe_stream_t stream);

/* Grouped gate+up GEMM over the dispatched rows with SiLU(gate)*up and the
 * requantisation of the hidden fused into its epilogue (pure-Triton article:
 * gate and up share one input tile, SiLU in registers; LightMoE README: gated
 * activation + requantisation).  Reads xq/xs/tiles from ws, writes hq/hs. */
moe_status moe_gate_up(const moe_handle* h, const void* packed, int T, void* ws,
                       moe_stream_t stream);

/* Grouped down GEMM over the hidden, times the routing weight of each row
 * (LightMoE README: down projection, routing-weight application).
 * w [T, k] fp32 (may be view.w).  Reads hq/hs, writes o. */
moe_status moe_down(const moe_handle* h, const void* packed, const float* w, int T,
                    void* ws, moe_stream_t stream);

/* Explicit tile choice of the down GEMM (LightMoE README, "Grouped GEMM",
 * leaves the tile configuration to the caller, since the best one varies with
 * the matrix sizes and with how the assignments spread over experts).  down_bn: 0 = chosen per call, or 64,
 * 128, 256 output columns per tile.  FP8_BLOCK128 takes all three; FP8_ROW
 * takes 128 (128-wide tiles with two accumulators in TMEM, so a tile's MMAs
 * run while the previous tile's epilogue drains; single CTAs) and otherwise
 * runs 256-wide tiles; NVFP4 ignores it.  Host state only. */
moe_status moe_set_tile_config(moe_handle* h, int down_bn);

/* Launch option of every kernel the layer calls (no counterpart in the pages:
 * a property of how the kernels are issued, not of what they compute).
 * pdl = 1 (the default) launches each kernel with programmatic dependent
 * launch allowed: it may be scheduled while the previous kernel in the stream
 * finishes, and orders its memory accesses after that kernel's on the device,
 * so results are identical with either setting.  pdl = 0 launches them in
 * plain stream order.  Host state only; MOE_ERR_INVALID_ARG for other values. */
moe_status moe_set_launch_options(moe_handle* h, int pdl);

/* GEMM options.  cta_pairs = 1 (the default): a gated FP8_ROW layer runs the
 * gate/up GEMM on CTA pairs where the dispatch's cost model picks them from
 * the expert histogram (moe_set_gate_up_model): 2-CTA clusters whose
 * tcgen05.mma.cta_group::2 covers two row tiles of one expert (M = 256), each
 * CTA loading its own 128 rows of X and half of the 256 weight rows (no
 * multicast), so a 32 KB stage feeds what a 48 KB stage feeds alone.  With
 * I > 2048 (FP8_ROW, any activation), where the output rows leave no room for
 * a K split of the down GEMM and the batch holds at least 4 row tiles per
 * expert on average (T*k >= 512 E, a host-side rule), the down GEMM runs on
 * CTA pairs the same way (each CTA loading its hidden rows, their scale chunk
 * and 128 of the 256 rows of W_down).  An expert with an odd row-tile count
 * runs its last pair half empty.  The
 * results are those of the single-CTA kernel up to the fp32 summation order
 * inside the tensor core.  cta_pairs = 0 keeps single CTAs; cta_pairs = 2
 * runs these GEMMs on CTA pairs at every batch size (the down GEMM still only
 * where K > 2048 and no K split is chosen).  Errors: MOE_ERR_INVALID_ARG for a
 * null handle, another value, or 2 while moe_set_gate_up_tile forces 128. */
moe_status moe_set_gemm_options(moe_handle* h, int cta_pairs);

/* Gate/up tile width of a gated FP8_ROW layer.  bn = 0 (the default): picked
 * on the device with the mode (moe_set_gate_up_model); 128 forces 128-wide
 * tiles (64 gate + 64 up accumulator columns, 64 hidden columns, 8 of the 16
 * epilogue warps working), 256 forbids them.  Narrow tiles double the units
 * and halve each unit's weight bytes, so a small batch's weight stream can end
 * in a shorter last wave.  Per element the same products and roundings as the
 * 256-wide tile.  Host state only.  MOE_ERR_INVALID_ARG for another value or
 * for 128 while CTA pairs are forced on; MOE_ERR_UNSUPPORTED_SHAPE for 128 on
 * an NVFP4, FP8_BLOCK128 or ReLU^2 layer. */
moe_status moe_set_gate_up_tile(moe_handle* h, int bn);

/* Limit, in SM clock cycles, of every wait of the GEMM kernels on another
 * role or CTA (stage, accumulator and exchange barriers); default 2e9 (about
 * 1 s).  A wait that runs out records MOE_ERR_DEVICE_TIMEOUT and the role in
 * the status word, and the kernel leaves its loops; it still waits (with a
 * fixed limit) for its own copies and MMAs in flight and frees its TMEM, so
 * the context stays usable (read the status with moe_get_status).  A small
 * value makes the waits run out on purpose (failure-detection tests).  No
 * counterpart in the pages.  Host state only; MOE_ERR_INVALID_ARG for
 * cycles <= 0. */
moe_status moe_set_wait_limit(moe_handle* h, long long cycles);

/* Parameters of the wave cost model that picks the down GEMM's tile width
 * from the runtime expert histogram (RaMP abstract: four-parameter wave cost
 * model fitted from a one-time profiling sweep).  The dispatch's scan kernel
 * evaluates, for BN in {256, 128, 64}, with m_tiles = sum_e ceil(count_e/128):
 *   t_mma  = ceil(m_tiles*(H/BN) / num_sms) * (I/128) * (alpha + beta*BN)
 *   t_load = touched_experts*H*I*1e6 / (min(m_tiles*(H/BN), num_sms) * bw)
 *   cost   = gamma + max(t_mma, t_load)     (integers: picoseconds, bytes/us)
 * and writes the cheapest (the wider on ties) to view.pick[0].
 * For FP8_ROW it also writes view.pick[1] = S, the K split of the down GEMM
 * (no parameters): with units = m_tiles * (H/256), A = T*k and
 * s_max = min(8, o_rows / A, (I/128) / 4) and
 * cost(s) = ceil(units*s / num_sms) * 840/s, S is the s <= s_max of lowest
 * cost (the smaller on ties) when that cost is at most 4/5 of cost(1), else 1
 * (o_rows = A_max + 7 min(A_max, 256)).
 * params = {alpha, beta, bw, gamma}; get also returns num_sms in params[4]. */
moe_status moe_set_picker_params(moe_handle* h, const long long* params);
moe_status moe_get_picker_params(const moe_handle* h, long long* params);

/* Parameters of the model that picks, from the runtime expert histogram, the
 * mode of a gated FP8_ROW layer's gate/up GEMM (RaMP abstract: a cost model
 * of CTA waves over the histogram, fitted once to a profiling sweep):
 *   0  single CTAs on 256-wide tiles (128 gate + 128 up accumulator columns),
 *   1  CTA pairs: tcgen05.mma.cta_group::2 with M = 256 over two row tiles of
 *      one expert, each CTA loading half of the 256 weight rows,
 *   2  single CTAs on 128-wide tiles (64 gate + 64 up columns).
 * The dispatch evaluates, with mt_e = ceil(count_e / 128), m_tiles = sum_e mt_e,
 * n_odd = #{e : mt_e odd}, nb = 2I / 256 and kb = H / 128 (integers, ps):
 *   c0 = ceil(m_tiles nb / num_sms) (kb a_0 + b_0)
 *   c1 = ceil((m_tiles + n_odd) / 2 nb / (num_sms / 2)) (kb a_1 + b_1)
 *   c2 = ceil(2 m_tiles nb / num_sms) (kb a_2 + b_2)
 * and writes view.pick[2] = the cheapest allowed mode (ties to the lower);
 * the gate/up kernel, launched as 2-CTA clusters, reads it.  The allowed modes
 * follow moe_set_gemm_options and moe_set_gate_up_tile.
 * params = {a_0, b_0, a_1, b_1, a_2, b_2}; get also returns nb, kb, num_sms
 * and the allowed-mode mask (bit m: mode m) in params[6..9] (nb = 0: the
 * layer has no choice, mode 0).  Host state only; MOE_ERR_INVALID_ARG for a
 * negative cost. */
moe_status moe_set_gate_up_model(moe_handle* h, const long long* params);
moe_status moe_get_gate_up_model(const moe_handle* h, long long* params);

/* Deterministic combine (LightMoE README, "Highlights": deterministic
 * combine): y[t] = bf16( sum_{j=0..k-1} o[inv[t k + j]] ) in fixed j order,
 * fp32 rows and accumulation, one final rounding, no atomics.  y [T, H] bf16. */
moe_status moe_combine(const moe_handle* h, int T, void* y, void* ws, moe_stream_t stream);

/* The whole layer: route -> dispatch -> gate/up -> down -> combine.  Routing
 * results stay in the workspace (view.ids, view.w).  y [T, H] bf16. */
moe_status moe_forward(const moe_handle* h, const void* x, int T, const float* wr,
                       const float* bias, const void* packed, void* y, void* ws,
                       moe_stream_t stream);

/* The layer with routing given by the caller (LightMoE README, "MoE inference":
 * __call__(x, top_k_ids, top_k_weights)).  ids [T, k] int32 distinct per token,
 * w [T, k] fp32. */
moe_status moe_forward_routed(const moe_handle* h, const void* x, int T, const int32_t* ids,
                              const float* w, const void* packed, void* y, void* ws,
                              moe_stream_t stream);

/* Zero the status words of a freshly allocated workspace; call once before
 * the workspace's first use. */
moe_status moe_workspace_init(const moe_handle* h, void* ws, moe_stream_t stream);

/* Synchronise `stream`, return the first device error recorded in ws since the
 * last call (MOE_OK if none) and clear it. */
moe_status moe_get_status(const moe_handle* h, void* ws, moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif
