/*
 * moe_oracle.c -- plain CPU oracle of the routed MoE FFN forward pass.
 * TEST INFRASTRUCTURE ONLY (see moe_oracle.h for what each function follows).
 *
 * Build: gcc -O2 -fopenmp -mfma -ffp-contract=off -fno-fast-math -shared -fPIC
 * -ffp-contract=off keeps every fp32 expression rounded exactly as written;
 * fused multiply-adds appear only where fmaf() is called on purpose.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

/* ------------------------------------------------------------------ codecs */

/* E4M3 "fn": sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is
 * subnormal (m * 2^-9); 0x7F/0xFF are NaN; no infinities; largest 448. */
double orc_e4m3_value(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp((double)(8 + m), e - 10);   /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

uint8_t orc_e4m3_encode(float x)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;          /* saturate to the largest finite */
    /* largest magnitude code c (0..126; codes are ordered by value) with value <= a */
    int lo = 0, hi = 126;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (orc_e4m3_value((uint8_t)mid) <= a) lo = mid; else hi = mid - 1;
    }
    int c = lo;
    if (c < 126) {
        double d0 = a - orc_e4m3_value((uint8_t)c);
        double d1 = orc_e4m3_value((uint8_t)(c + 1)) - a;
        if (d1 < d0 || (d1 == d0 && ((c + 1) & 1) == 0)) c = c + 1;   /* tie -> even mantissa */
    }
    return sign | (uint8_t)c;
}

/* E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 subnormal. */
double orc_e2m1_value(uint8_t code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

uint8_t orc_e2m1_encode(float x)
{
    uint8_t sign = signbit(x) ? 0x8 : 0x0;
    double a = fabs((double)x);
    if (isnan(x)) return 0x7;                    /* not expected: inputs are finite */
    if (a >= 6.0) return sign | 0x7;
    int c = 0;
    while (c < 7 && orc_e2m1_value((uint8_t)(c + 1)) <= a) c++;
    if (c < 7) {
        double d0 = a - orc_e2m1_value((uint8_t)c);
        double d1 = orc_e2m1_value((uint8_t)(c + 1)) - a;
        if (d1 < d0 || (d1 == d0 && ((c + 1) & 1) == 0)) c = c + 1;
    }
    return sign | (uint8_t)c;
}

void orc_e4m3_encode_n(const float* x, int64_t n, uint8_t* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) out[i] = orc_e4m3_encode(x[i]);
}

void orc_e2m1_encode_n(const float* x, int64_t n, uint8_t* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) out[i] = orc_e2m1_encode(x[i]);
}

static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ------------------------------------------------------------------ router */

static float canonical_dot(const uint16_t* x, const float* w, int H)
{
    float p[32];
    int n = H / 256;
    for (int l = 0; l < 32; l++) {
        float acc = 0.0f;
        for (int i = 0; i < n; i++)
            for (int j = 0; j < 8; j++) {
                int h = 256 * i + 8 * l + j;
                acc = fmaf(bf16_to_f32(x[h]), w[h], acc);
            }
        p[l] = acc;
    }
    /* balanced pairwise tree over lanes: 32 -> 16 -> 8 -> 4 -> 2 -> 1 */
    for (int width = 32; width > 1; width /= 2)
        for (int m = 0; m < width / 2; m++) p[m] = p[2 * m] + p[2 * m + 1];
    return p[0];
}

void orc_router_logits(const uint16_t* x, int T, int H, const float* wr,
                       const float* bias, int E, float* logits)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; t++)
        for (int e = 0; e < E; e++) {
            float v = canonical_dot(x + (int64_t)t * H, wr + (int64_t)e * H, H);
            if (bias) v = v + bias[e];
            logits[(int64_t)t * E + e] = v;
        }
}

void orc_router_logits_f64(const uint16_t* x, int T, int H, const float* wr,
                           const float* bias, int E, double* logits)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; t++)
        for (int e = 0; e < E; e++) {
            double acc = 0.0;
            for (int h = 0; h < H; h++)
                acc += (double)bf16_to_f32(x[(int64_t)t * H + h]) * (double)wr[(int64_t)e * H + h];
            if (bias) acc += (double)bias[e];
            logits[(int64_t)t * E + e] = acc;
        }
}

/* a ranks before b: larger logit first, equal logits -> lower id first */
static int ranks_before(float la, int a, float lb, int b)
{
    return (la > lb) || (la == lb && a < b);
}

void orc_topk(const float* logits, int T, int E, int k, int score, int32_t* ids, double* w)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; t++) {
        const float* l = logits + (int64_t)t * E;
        char taken[1024];
        memset(taken, 0, sizeof(taken));
        for (int j = 0; j < k; j++) {
            int best = -1;
            for (int e = 0; e < E; e++)
                if (!taken[e] && (best < 0 || ranks_before(l[e], e, l[best], best))) best = e;
            taken[best] = 1;
            ids[(int64_t)t * k + j] = best;
        }
        double* wt = w + (int64_t)t * k;
        double sum = 0.0;
        if (score == ORC_SCORE_SOFTMAX) {
            double m = (double)l[ids[(int64_t)t * k]];   /* first slot holds the largest */
            for (int j = 0; j < k; j++) {
                wt[j] = exp((double)l[ids[(int64_t)t * k + j]] - m);
                sum += wt[j];
            }
        } else {
            for (int j = 0; j < k; j++) {
                wt[j] = 1.0 / (1.0 + exp(-(double)l[ids[(int64_t)t * k + j]]));
                sum += wt[j];
            }
        }
        for (int j = 0; j < k; j++) wt[j] /= sum;
    }
}

/* ---------------------------------------------------------------- dispatch */

void orc_dispatch(const int32_t* ids, int T, int k, int E, int32_t* counts,
                  int32_t* offsets, int32_t* perm, int32_t* inv)
{
    int64_t A = (int64_t)T * k;
    for (int e = 0; e < E; e++) counts[e] = 0;
    for (int64_t a = 0; a < A; a++) counts[ids[a]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; e++) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* next = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; e++) next[e] = offsets[e];
    for (int64_t a = 0; a < A; a++) {          /* row-major (t, j) order */
        int32_t slot = next[ids[a]]++;
        perm[slot] = (int32_t)a;
        inv[a] = slot;
    }
    free(next);
}

int orc_schedule(const int32_t* offsets, int E, int32_t* tile_expert, int32_t* tile_row)
{
    int n = 0;
    for (int e = 0; e < E; e++)
        for (int32_t r = offsets[e]; r < offsets[e + 1]; r += ORC_TILE_M) {
            tile_expert[n] = e;
            tile_row[n] = r;
            n++;
        }
    return n;
}

/* ------------------------------------------------------- down tile choice */

int orc_pick_down_tile(const int32_t* counts, int E, int H, int I, int num_sms,
                       int64_t alpha, int64_t beta, int64_t bw, int64_t gamma, int64_t* costs)
{
    int64_t m_tiles = 0, touched = 0;
    for (int e = 0; e < E; e++) {
        m_tiles += (counts[e] + ORC_TILE_M - 1) / ORC_TILE_M;
        touched += counts[e] > 0;
    }
    const int64_t bn_of[3] = {256, 128, 64};
    int best = 0;
    for (int c = 0; c < 3; c++) {
        int64_t bn = bn_of[c];
        int64_t tiles = m_tiles * (H / bn);
        int64_t waves = (tiles + num_sms - 1) / num_sms;
        int64_t t_mma = waves * (I / 128) * (alpha + beta * bn);
        int64_t active = tiles < num_sms ? tiles : num_sms;
        int64_t t_load = active > 0 ? touched * H * I * 1000000LL / (active * bw) : 0;
        costs[c] = gamma + (t_mma > t_load ? t_mma : t_load);
        if (costs[c] < costs[best]) best = c;
    }
    return best;
}

/* K split of the down GEMM for small batches: S copies of the output rows, one
 * per near-equal range of K-blocks.  units = m_tiles * split_nb; the split is
 * bounded by s_max = min(8, o_rows / A, split_kb / 4) (the copies the output
 * buffer holds, at least four K-blocks per range).  With
 * cost(s) = ceil(units * s / num_sms) * (840 / s), the time in rounds of 1/s
 * of a unit, S is the s <= s_max of lowest cost (the smaller s on equal
 * costs), taken only when that cost is at most 4/5 of cost(1); otherwise, and
 * when split_nb is 0 or the batch is empty, S = 1. */
int orc_pick_split(const int32_t* counts, int E, int split_nb, int split_kb, int64_t o_rows, int num_sms)
{
    int64_t m_tiles = 0, A = 0;
    for (int e = 0; e < E; e++) {
        m_tiles += (counts[e] + ORC_TILE_M - 1) / ORC_TILE_M;
        A += counts[e];
    }
    if (split_nb <= 0 || A == 0) return 1;
    int64_t smax = 8;
    if (o_rows / A < smax) smax = o_rows / A;
    if (split_kb / 4 < smax) smax = split_kb / 4;
    /* cost(s) = ceil(units s / num_sms) 840 / s: rounds of 1/s of a unit, in
       840ths (840 is a multiple of 1..8); the cheapest s wins (the smaller on
       ties), if it is at least 20% cheaper than no split */
    const int64_t units = m_tiles * split_nb;
    const int64_t c1 = (units + num_sms - 1) / num_sms * 840;
    int best = 1;
    int64_t best_cost = c1;
    for (int64_t s = 2; s <= smax; s++) {
        const int64_t c = (units * s + num_sms - 1) / num_sms * (840 / s);
        if (c < best_cost && 5 * c <= 4 * c1) {
            best = (int)s;
            best_cost = c;
        }
    }
    return best;
}

int orc_pick_gu_mode(const int32_t* counts, int E, int nb, int kb, int num_sms, int allow, const int64_t* ps)
{
    int64_t m_tiles = 0, n_odd = 0;
    for (int e = 0; e < E; e++) {
        int64_t mt = (counts[e] + ORC_TILE_M - 1) / ORC_TILE_M;
        m_tiles += mt;
        n_odd += mt & 1;
    }
    if (nb <= 0 || m_tiles == 0) return 0;
    /* units and the CTAs (or pairs) that run at once, per mode */
    int64_t units[3], slots[3];
    units[0] = m_tiles * nb;                  /* 256-wide tiles on single CTAs */
    slots[0] = num_sms;
    units[1] = (m_tiles + n_odd) / 2 * nb;    /* pairs of an expert's m-tiles */
    slots[1] = num_sms / 2;
    units[2] = m_tiles * 2 * nb;              /* 128-wide tiles on single CTAs */
    slots[2] = num_sms;
    int best = -1;
    int64_t best_cost = 0;
    for (int m = 0; m < 3; m++) {
        if (!((allow >> m) & 1)) continue;
        int64_t waves = (units[m] + slots[m] - 1) / slots[m];
        int64_t cost = waves * (kb * ps[2 * m] + ps[2 * m + 1]);
        if (best < 0 || cost < best_cost) {
            best = m;
            best_cost = cost;
        }
    }
    return best < 0 ? 0 : best;
}

/* ------------------------------------------------ activation quantisation */

float orc_nvfp4_global(const float* x, int64_t n)
{
    float a = 0.0f;
    for (int64_t i = 0; i < n; i++) a = fmaxf(a, fabsf(x[i]));
    return a / 2688.0f;                          /* 2688 = 448 * 6 */
}

static int64_t row_code_bytes(int fmt, int K) { return fmt == ORC_FMT_NVFP4 ? K / 2 : K; }

/* smallest e with amax <= 448 * 2^e (amax > 0): amax = m 2^x, m in [0.5, 1),
 * 448 = 0.875 2^9, so e = x - 9 when m <= 0.875, else x - 8 */
static int mx_exponent(float amax)
{
    if (amax == 0.0f) return -127;
    int x;
    float m = frexpf(amax, &x);
    int e = (m <= 0.875f) ? x - 9 : x - 8;
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

void orc_quant_rows(int fmt, const float* x, int rows, int K, float g,
                    uint8_t* codes, void* scales)
{
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; r++) {
        const float* xr = x + (int64_t)r * K;
        uint8_t* qr = codes + (int64_t)r * row_code_bytes(fmt, K);
        if (fmt == ORC_FMT_FP8_ROW || fmt == ORC_FMT_FP8_BLOCK128) {
            int bw = (fmt == ORC_FMT_FP8_ROW) ? K : 128;
            for (int b = 0; b < K / bw; b++) {
                float amax = 0.0f;
                for (int c = b * bw; c < (b + 1) * bw; c++) amax = fmaxf(amax, fabsf(xr[c]));
                float s = amax / 448.0f;
                ((float*)scales)[(int64_t)r * (K / bw) + b] = s;
                for (int c = b * bw; c < (b + 1) * bw; c++)
                    qr[c] = (s == 0.0f) ? 0 : orc_e4m3_encode(xr[c] / s);
            }
        } else if (fmt == ORC_FMT_MX32) {
            uint8_t* sr = (uint8_t*)scales + (int64_t)r * (K / 32);
            for (int b = 0; b < K / 32; b++) {
                float amax = 0.0f;
                for (int c = 32 * b; c < 32 * b + 32; c++) amax = fmaxf(amax, fabsf(xr[c]));
                int e = mx_exponent(amax);
                sr[b] = (uint8_t)(e + 127);
                for (int c = 32 * b; c < 32 * b + 32; c++) qr[c] = orc_e4m3_encode(ldexpf(xr[c], -e));
            }
        } else {
            uint8_t* sr = (uint8_t*)scales + (int64_t)r * (K / 16);
            for (int b = 0; b < K / 16; b++) {
                float amax = 0.0f;
                for (int c = 16 * b; c < 16 * b + 16; c++) amax = fmaxf(amax, fabsf(xr[c]));
                uint8_t sb = 0;
                float d = 0.0f;
                if (g > 0.0f) {
                    float u = (amax / 6.0f) / g;
                    sb = orc_e4m3_encode(u);
                    d = (float)orc_e4m3_value(sb) * g;
                }
                sr[b] = sb;
                for (int c = 16 * b; c < 16 * b + 16; c += 2) {
                    uint8_t lo = (d == 0.0f) ? 0 : orc_e2m1_encode(xr[c] / d);
                    uint8_t hi = (d == 0.0f) ? 0 : orc_e2m1_encode(xr[c + 1] / d);
                    qr[c / 2] = (uint8_t)(lo | (hi << 4));
                }
            }
        }
    }
}

/* exact fp64 value of element c of a quantised activation row */
static void dequant_act_row(int fmt, const uint8_t* q, const void* s, float g, int K, double* out)
{
    for (int c = 0; c < K; c++) {
        if (fmt == ORC_FMT_FP8_ROW)
            out[c] = orc_e4m3_value(q[c]) * (double)((const float*)s)[0];
        else if (fmt == ORC_FMT_FP8_BLOCK128)
            out[c] = orc_e4m3_value(q[c]) * (double)((const float*)s)[c / 128];
        else if (fmt == ORC_FMT_MX32)
            out[c] = ldexp(orc_e4m3_value(q[c]), (int)((const uint8_t*)s)[c / 32] - 127);
        else {
            uint8_t nib = (c & 1) ? (q[c / 2] >> 4) : (q[c / 2] & 15);
            out[c] = orc_e2m1_value(nib) * orc_e4m3_value(((const uint8_t*)s)[c / 16]) * (double)g;
        }
    }
}

static int64_t act_scale_bytes(int fmt, int K)
{
    if (fmt == ORC_FMT_FP8_ROW) return 4;
    if (fmt == ORC_FMT_FP8_BLOCK128) return 4 * (K / 128);
    if (fmt == ORC_FMT_MX32) return K / 32;
    return K / 16;
}

/* ------------------------------------------------------------ expert FFN */

/* Format of the requantised hidden.  The gate/up epilogue of a tile sees a
 * block of hidden columns of a row, never the whole row, so the hidden gets
 * block scales: power-of-two scales per 32 columns (MX32, applied by the
 * tensor cores in the down projection) for FP8_ROW, fp32 scales per 128
 * columns (the 1x128 activation rule, like its X) for FP8_BLOCK128, and the
 * NVFP4 16-blocks with the static global scale for NVFP4.  The per-token
 * reading (one fp32 scale per row, the FP8_ROW rule) is kept for comparison. */
static int hidden_fmt(const orc_layer* L)
{
    if (L->hidden_rule == ORC_HIDDEN_PER_TOKEN && L->fmt != ORC_FMT_NVFP4) return ORC_FMT_FP8_ROW;
    if (L->fmt == ORC_FMT_FP8_ROW) return ORC_FMT_MX32;
    return L->fmt;
}

void orc_weight_row(const orc_layer* L, const orc_proj* P, int N, int K, int e, int n, double* out)
{
    int slot = L->expert_slot ? L->expert_slot[e] : e;
    if (L->fmt == ORC_FMT_NVFP4) {
        const uint8_t* q = P->q + ((int64_t)slot * N + n) * (K / 2);
        const uint8_t* sb = (const uint8_t*)P->s + ((int64_t)slot * N + n) * (K / 16);
        double g = (double)P->g[slot];
        for (int c = 0; c < K; c++) {
            uint8_t nib = (c & 1) ? (q[c / 2] >> 4) : (q[c / 2] & 15);
            out[c] = orc_e2m1_value(nib) * orc_e4m3_value(sb[c / 16]) * g;
        }
        return;
    }
    const uint8_t* q = P->q + ((int64_t)slot * N + n) * K;
    for (int c = 0; c < K; c++) {
        double s;
        if (L->fmt == ORC_FMT_FP8_ROW)
            s = ((const float*)P->s)[(int64_t)slot * N + n];
        else
            s = ((const float*)P->s)[((int64_t)slot * (N / 128) + n / 128) * (K / 128) + c / 128];
        out[c] = orc_e4m3_value(q[c]) * s;
    }
}

static double dot64(const double* a, const double* b, int n)
{
    double acc = 0.0;
    for (int i = 0; i < n; i++) acc += a[i] * b[i];
    return acc;
}

static void down_dequantised(const orc_layer* L, int e, int rows, const double* hd, double* o)
{
    int H = L->H, I = L->I;
#pragma omp parallel
    {
        double* wrow = (double*)malloc(sizeof(double) * (size_t)I);
#pragma omp for schedule(static)
        for (int m = 0; m < H; m++) {
            orc_weight_row(L, &L->down, H, I, e, m, wrow);
            for (int r = 0; r < rows; r++) o[(int64_t)r * H + m] = dot64(hd + (int64_t)r * I, wrow, I);
        }
        free(wrow);
    }
}

static void dequant_rows(int fmt, int rows, int K, const uint8_t* codes,
                         const void* scales, float g, double* out)
{
    int64_t cb = row_code_bytes(fmt, K), sb = act_scale_bytes(fmt, K);
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; r++)
        dequant_act_row(fmt, codes + r * cb, (const uint8_t*)scales + r * sb, g, K, out + (int64_t)r * K);
}

double orc_glu(int act, double alpha, double limit, double g, double u)
{
    switch (act) {
    case ORC_ACT_SWIGLU_BOUNDED: {
        double gc = g < limit ? g : limit;
        double uc = u < -limit ? -limit : (u > limit ? limit : u);
        return gc / (1.0 + exp(-gc)) * uc;
    }
    case ORC_ACT_SWIGLU_OAI: {
        double gc = g < limit ? g : limit;
        double uc = u < -limit ? -limit : (u > limit ? limit : u);
        return gc / (1.0 + exp(-alpha * gc)) * (uc + 1.0);
    }
    case ORC_ACT_GEGLU:
        return 0.5 * g * (1.0 + erf(g / sqrt(2.0))) * u;
    case ORC_ACT_REGLU:
        return (g > 0.0 ? g : 0.0) * u;
    case ORC_ACT_RELU2:
        return u > 0.0 ? u * u : 0.0;
    default:
        return g / (1.0 + exp(-g)) * u;
    }
}

void orc_expert_rows(const orc_layer* L, int e, int rows, const uint8_t* a_codes,
                     const void* a_scales, float x_global, double* h,
                     uint8_t* hq_codes, void* hq_scales, double* o)
{
    int H = L->H, I = L->I;
    double* a = (double*)malloc(sizeof(double) * (size_t)rows * H);
    double* hh = (double*)malloc(sizeof(double) * (size_t)rows * I);
    dequant_rows(L->fmt, rows, H, a_codes, a_scales, x_global, a);
#pragma omp parallel
    {
        double* wg = (double*)malloc(sizeof(double) * (size_t)H);
        double* wu = (double*)malloc(sizeof(double) * (size_t)H);
        const int gated = L->act != ORC_ACT_RELU2;   /* ReLU^2 experts have no gate */
#pragma omp for schedule(static)
        for (int n = 0; n < I; n++) {
            if (gated) orc_weight_row(L, &L->gate, I, H, e, n, wg);
            orc_weight_row(L, &L->up, I, H, e, n, wu);
            for (int r = 0; r < rows; r++) {
                double g = gated ? dot64(a + (int64_t)r * H, wg, H) : 0.0;
                double u = dot64(a + (int64_t)r * H, wu, H);
                hh[(int64_t)r * I + n] = orc_glu(L->act, L->act_alpha, L->act_limit, g, u);
            }
        }
        free(wg);
        free(wu);
    }
    if (h) memcpy(h, hh, sizeof(double) * (size_t)rows * I);
    /* requantise the hidden: round to fp32, then the hidden's rule */
    int hf_fmt = hidden_fmt(L);
    float* hf = (float*)malloc(sizeof(float) * (size_t)rows * I);
    for (int64_t i = 0; i < (int64_t)rows * I; i++) hf[i] = (float)hh[i];
    uint8_t* qc = hq_codes ? hq_codes : (uint8_t*)malloc((size_t)(rows * row_code_bytes(hf_fmt, I)));
    void* qs = hq_scales ? hq_scales : malloc((size_t)(rows * act_scale_bytes(hf_fmt, I)));
    orc_quant_rows(hf_fmt, hf, rows, I, L->hidden_global, qc, qs);
    double* hd = (double*)malloc(sizeof(double) * (size_t)rows * I);
    dequant_rows(hf_fmt, rows, I, qc, qs, L->hidden_global, hd);
    down_dequantised(L, e, rows, hd, o);
    if (!hq_codes) free(qc);
    if (!hq_scales) free(qs);
    free(hd);
    free(hf);
    free(hh);
    free(a);
}

void orc_down_rows(const orc_layer* L, int e, int rows, const uint8_t* h_codes,
                   const void* h_scales, double* o)
{
    double* hd = (double*)malloc(sizeof(double) * (size_t)rows * L->I);
    dequant_rows(hidden_fmt(L), rows, L->I, h_codes, h_scales, L->hidden_global, hd);
    down_dequantised(L, e, rows, hd, o);
    free(hd);
}

/* ----------------------------------------------------------- whole layer */

int orc_moe_forward(const orc_layer* L, const uint16_t* x, int T, const float* wr,
                    const float* bias, int n_sel, const int32_t* sel,
                    int32_t* ids, double* w, double* y_sel)
{
    int H = L->H, E = L->E, k = L->k, fmt = L->fmt;
    float* logits = (float*)malloc(sizeof(float) * (size_t)T * E);
    orc_router_logits(x, T, H, wr, bias, E, logits);
    orc_topk(logits, T, E, k, L->score, ids, w);
    free(logits);

    float xg = 0.0f;
    if (fmt == ORC_FMT_NVFP4) {
        float amax = 0.0f;
        for (int64_t i = 0; i < (int64_t)T * H; i++) amax = fmaxf(amax, fabsf(bf16_to_f32(x[i])));
        xg = amax / 2688.0f;
    }
    int64_t cb = row_code_bytes(fmt, H), sbytes = act_scale_bytes(fmt, H);
    float* xf = (float*)malloc(sizeof(float) * (size_t)n_sel * H);
    for (int s = 0; s < n_sel; s++)
        for (int c = 0; c < H; c++) xf[(int64_t)s * H + c] = bf16_to_f32(x[(int64_t)sel[s] * H + c]);
    uint8_t* xq = (uint8_t*)malloc((size_t)(n_sel * cb));
    uint8_t* xs = (uint8_t*)malloc((size_t)(n_sel * sbytes));
    orc_quant_rows(fmt, xf, n_sel, H, xg, xq, xs);
    free(xf);

    double* o_all = (double*)calloc((size_t)n_sel * k * H, sizeof(double));
    uint8_t* aq = (uint8_t*)malloc((size_t)(n_sel * k * cb));
    uint8_t* as = (uint8_t*)malloc((size_t)(n_sel * k * sbytes));
    int* which = (int*)malloc(sizeof(int) * (size_t)n_sel * k);
    int rc = 0;
    for (int e = 0; e < E && rc == 0; e++) {
        int rows = 0;
        for (int s = 0; s < n_sel; s++)
            for (int j = 0; j < k; j++)
                if (ids[(int64_t)sel[s] * k + j] == e) {
                    memcpy(aq + rows * cb, xq + s * cb, (size_t)cb);
                    memcpy(as + rows * sbytes, xs + s * sbytes, (size_t)sbytes);
                    which[rows++] = s * k + j;
                }
        if (rows == 0) continue;
        if (L->expert_slot && L->expert_slot[e] < 0) { rc = -1; break; }
        double* o = (double*)malloc(sizeof(double) * (size_t)rows * H);
        orc_expert_rows(L, e, rows, aq, as, xg, NULL, NULL, NULL, o);
        for (int r = 0; r < rows; r++)
            memcpy(o_all + (int64_t)which[r] * H, o + (int64_t)r * H, sizeof(double) * (size_t)H);
        free(o);
    }
    if (rc == 0)
        for (int s = 0; s < n_sel; s++)
            for (int m = 0; m < H; m++) {
                double y = 0.0;
                for (int j = 0; j < k; j++)            /* fixed slot order */
                    y += w[(int64_t)sel[s] * k + j] * o_all[((int64_t)s * k + j) * H + m];
                y_sel[(int64_t)s * H + m] = y;
            }
    free(which);
    free(as);
    free(aq);
    free(o_all);
    free(xs);
    free(xq);
    return rc;
}

int orc_num_threads(void) { return omp_get_max_threads(); }
