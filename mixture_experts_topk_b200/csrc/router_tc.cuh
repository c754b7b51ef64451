// router_tc.cuh -- router top-k for large batches: an exact integer
// tensor-core pass bounds every logit, and only the experts that could still
// be among a token's k largest get the canonical fp32 logit.
//
// Alpha-MoE article ("How the megakernel works"): routing is the first fused
// stage of the layer; at prefill sizes with 256 experts it is a [T, H] x [H, E]
// product that a SIMT fp32 kernel runs at a fraction of the tensor cores'
// rate.  The selected ids must still be those of the canonical fp32 logits
// (fixed chain order, see router.cuh), bit for bit, ties to the lower id.
//
// 1. Fixed point (router_fixpoint_kernel).  Each X row and each Wr row is
//    scaled by a power of two 2^(14 - e), e the smallest integer with
//    max|row| <= 2^e, and rounded to an integer q with |q| <= 2^14; q is kept
//    as two signed bytes q = 256 hi + lo, hi in [-64, 64], lo in [-128, 127].
//    Per row: e, sum |v| and max |v| (fp64), and for Wr sum |q|.
// 2. Integer products (router_i8_kernel).  tcgen05.mma kind::i8 (int8 x int8
//    -> int32, exact) gives, per (token, expert), S_hh = sum hi_x hi_w,
//    S_x = sum (hi_x lo_w + lo_x hi_w) and S_ll = sum lo_x lo_w, so
//        L~ = 2^(e_x + e_w - 28) (65536 S_hh + 256 S_x + S_ll) + bias[e]
//    is the exact dot product of the rounded rows (+ bias), evaluated in fp64
//    without rounding and stored as fp32.  |int32 sums| <= 2^14 * 2 H * 64, so
//    H <= 65536 cannot overflow.
// 3. Certified filter (router_select_kernel).  With eps = 2^(e - 15) the
//    rounding of one value (half a unit), the exact logit L* = sum x w + b and
//    the canonical fp32 logit C (n = H/32 fused multiply-adds per chain, a
//    5-level tree, one bias add: at most n + 6 roundings on any path),
//        |L~ - L*| <= eps_w sum|x| + eps_x sum|w~|              (fixed point)
//        |C  - L*| <= gamma(n + 6) (sum|x w| + |b|),             gamma(m) = m u / (1 - m u), u = 2^-24
//        |fp32(L~) - L~| <= 2^-24 |L~|,
//    with sum|x w| <= min(sum|x| max|w|, max|x| sum|w|).  So C lies in
//    [l - D, l + D] around the stored l = fp32(L~), D their sum (x (1 + 2^-20)
//    for the fp64 evaluation of D itself).  Let LB_k be the k-th largest
//    l - D of the token.  An expert with l + D < LB_k has k experts whose C
//    is strictly larger, so it is not among the canonical top k whatever the
//    tie rule; every other expert is a candidate.  The candidates get the
//    canonical C (same chains and tree as router.cuh), the top k of the
//    candidates by C (ties to the lower id) is the canonical top k, and the
//    weights are computed from those C exactly as on the SIMT path.
// The logits buffer then holds C for the candidates (a superset of the
// selected experts) and fp32(L~) for the others.
#pragma once
#include "common.cuh"
#include "router.cuh"

namespace moe {

constexpr int RTC_BM = 128;              // tokens per tile (TMEM lanes)
constexpr int RTC_BK = 128;              // K bytes per stage
constexpr int RTC_NT_MAX = 128;          // experts per tile
constexpr int RTC_STAGES = 3;
constexpr int RTC_THREADS = 192;         // producer, MMA, 4 epilogue warps
constexpr int RTC_A_BYTES = RTC_BM * RTC_BK;
constexpr int RTC_B_BYTES = RTC_NT_MAX * RTC_BK;
constexpr int RTC_STAGE_BYTES = 2 * RTC_A_BYTES + 2 * RTC_B_BYTES;     // hi and lo of X and of Wr
constexpr int RTC_BAR_OFF = RTC_STAGES * RTC_STAGE_BYTES;
constexpr int RTC_SMEM = RTC_BAR_OFF + 8 * (2 * RTC_STAGES + 2) + 16 + 1024;   // + alignment slack
constexpr int RTC_MAX_H = 65536;

// per-row scalars of the fixed-point rows
struct RouterFix {
    int8_t* xh;          // [T][H] hi bytes of X rows
    int8_t* xl;          // [T][H] lo bytes
    int8_t* wh;          // [E][H]
    int8_t* wl;
    int32_t* x_exp;      // [T] e of each X row
    double* x_sum;       // [T] sum |x|
    float* x_max;        // [T] max |x|
    int32_t* w_exp;      // [E]
    double* w_sum;       // [E] sum |w|
    double* w_sumq;      // [E] sum |w~| = 2^(e - 14) sum |q|
    float* w_max;        // [E] max |w|
};

// e with max|v| <= 2^e (0 for an all-zero row): amax = m 2^e, m in [0.5, 1)
__device__ __forceinline__ int fix_exponent(float amax) {
    if (amax == 0.0f) return 0;
    int e;
    frexpf(amax, &e);
    return e;
}
// q = rint(v 2^(14 - e)), |q| <= 2^14, split as 256 hi + lo.  The scaling is a
// multiplication by the power of two `scale` when that is a normal float (exact
// unless the product is subnormal, where q = 0 either way), else ldexpf.
__device__ __forceinline__ void fix_split(float v, int e, float scale, int& hi, int& lo, int& q) {
    q = __float2int_rn(scale != 0.0f ? v * scale : ldexpf(v, 14 - e));
    hi = (q + 128) >> 8;
    lo = q - (hi << 8);
}
__device__ __forceinline__ float fix_scale(int e) {
    const int k = 14 - e;
    return (k >= -126 && k <= 127) ? __int_as_float((127 + k) << 23) : 0.0f;
}

// Blocks [0, nbx): 8 X rows each (one warp per row); blocks [nbx, ...): 8 Wr
// rows each.  Lane l takes h = 256 i + 8 l + j (16-byte loads of X).
// Wr rows E .. E_pad - 1 (the padding of the last expert tile) are written as
// zeros, so every tile's TMA box lies inside the tensor.
__global__ void __launch_bounds__(256) router_fixpoint_kernel(const __nv_bfloat16* x, const float* wr, int T, int H,
                                                              int E, int E_pad, int nbx, RouterFix f) {
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool is_x = static_cast<int>(blockIdx.x) < nbx;
    const int row = (is_x ? blockIdx.x : blockIdx.x - nbx) * 8 + warp;
    if (row >= (is_x ? T : E_pad)) return;
    const int nI = H >> 8;
    if (!is_x && row >= E) {
        for (int i = 0; i < nI; i++) {
            *reinterpret_cast<uint2*>(f.wh + static_cast<size_t>(row) * H + 256 * i + 8 * lane) = make_uint2(0u, 0u);
            *reinterpret_cast<uint2*>(f.wl + static_cast<size_t>(row) * H + 256 * i + 8 * lane) = make_uint2(0u, 0u);
        }
        if (lane == 0) {
            f.w_exp[row] = 0;
            f.w_sum[row] = 0.0;
            f.w_sumq[row] = 0.0;
            f.w_max[row] = 0.0f;
        }
        return;
    }
    float amax = 0.0f;
    double sum = 0.0;
#pragma unroll 4
    for (int i = 0; i < nI; i++) {
        const size_t h0 = static_cast<size_t>(row) * H + 256 * i + 8 * lane;
        float v[8];
        if (is_x) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + h0));
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int q = 0; q < 4; q++) {
                v[2 * q] = bf16_lo(w4[q]);
                v[2 * q + 1] = bf16_hi(w4[q]);
            }
        } else {
            const float4 a = __ldg(reinterpret_cast<const float4*>(wr + h0));
            const float4 b = __ldg(reinterpret_cast<const float4*>(wr + h0 + 4));
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        }
#pragma unroll
        for (int j = 0; j < 8; j++) {
            amax = fmaxf(amax, fabsf(v[j]));
            sum += fabs(static_cast<double>(v[j]));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        sum += __shfl_xor_sync(0xffffffffu, sum, off);
    }
    const int e = fix_exponent(amax);
    const float scale = fix_scale(e);
    long long sumq = 0;
    int8_t* dh = (is_x ? f.xh : f.wh) + static_cast<size_t>(row) * H;
    int8_t* dl = (is_x ? f.xl : f.wl) + static_cast<size_t>(row) * H;
#pragma unroll 4
    for (int i = 0; i < nI; i++) {
        const size_t h0 = static_cast<size_t>(row) * H + 256 * i + 8 * lane;
        float v[8];
        if (is_x) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + h0));
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int q = 0; q < 4; q++) {
                v[2 * q] = bf16_lo(w4[q]);
                v[2 * q + 1] = bf16_hi(w4[q]);
            }
        } else {
            const float4 a = __ldg(reinterpret_cast<const float4*>(wr + h0));
            const float4 b = __ldg(reinterpret_cast<const float4*>(wr + h0 + 4));
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        }
        uint32_t ph[2] = {0u, 0u}, pl[2] = {0u, 0u};
#pragma unroll
        for (int j = 0; j < 8; j++) {
            int hi, lo, q;
            fix_split(v[j], e, scale, hi, lo, q);
            sumq += q < 0 ? -q : q;
            ph[j >> 2] |= (static_cast<uint32_t>(hi) & 0xFFu) << (8 * (j & 3));
            pl[j >> 2] |= (static_cast<uint32_t>(lo) & 0xFFu) << (8 * (j & 3));
        }
        *reinterpret_cast<uint2*>(dh + 256 * i + 8 * lane) = make_uint2(ph[0], ph[1]);
        *reinterpret_cast<uint2*>(dl + 256 * i + 8 * lane) = make_uint2(pl[0], pl[1]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sumq += __shfl_xor_sync(0xffffffffu, sumq, off);
    if (lane == 0) {
        if (is_x) {
            f.x_exp[row] = e;
            f.x_sum[row] = sum;
            f.x_max[row] = amax;
        } else {
            f.w_exp[row] = e;
            f.w_sum[row] = sum;
            f.w_sumq[row] = ldexp(static_cast<double>(sumq), e - 14);
            f.w_max[row] = amax;
        }
    }
}

// Instruction descriptor of kind::i8: s32 accumulate [4,6) = 2, A and B signed
// 8-bit [7,10) = [10,13) = 1, both K-major, N >> 3 at [17,23), M >> 4 at [24,29).
__host__ __device__ constexpr uint32_t idesc_s8(int M, int N) {
    return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}
// D[tmem] (+)= A[smem] * B[smem]^T, s8 x s8 -> s32 (exact), one elected thread.
__device__ __forceinline__ void mma_s8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

struct RouterI8Params {
    int T, H, E, NT;
    const int32_t* x_exp;
    const int32_t* w_exp;
    const float* bias;       // nullable
    float* logits;           // [T, E]: fp32(L~)
    int32_t* status;
    long long spin_limit;
};

// One CTA per tile of 128 tokens x NT experts (NT a multiple of 16, <= 128).
// Warp 0: TMA producer of the four 128-byte K slices (X hi/lo rows, Wr hi/lo
// rows) per stage; warp 1: TMEM allocation and the MMA thread (per 32 of K:
// S_hh += hi hi, S_x += hi lo + lo hi, S_ll += lo lo, three accumulators of
// NT columns); warps 2..5: epilogue, one token row per thread.
__global__ void __launch_bounds__(RTC_THREADS, 1)
    router_i8_kernel(const __grid_constant__ CUtensorMap tXh, const __grid_constant__ CUtensorMap tXl,
                     const __grid_constant__ CUtensorMap tWh, const __grid_constant__ CUtensorMap tWl,
                     RouterI8Params p) {
    extern __shared__ uint8_t rtc_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(rtc_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + RTC_BAR_OFF);
    uint64_t* full = bars;
    uint64_t* empty = bars + RTC_STAGES;
    uint64_t* tfull = bars + 2 * RTC_STAGES;
    uint64_t* drain = bars + 2 * RTC_STAGES + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + RTC_BAR_OFF + 8 * (2 * RTC_STAGES + 2));
    volatile int* failed = reinterpret_cast<volatile int*>(tmem_slot + 1);   // set by the MMA thread
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NT = p.NT;
    const int m0 = blockIdx.x * RTC_BM, n0 = blockIdx.y * NT;
    const int num_kb = p.H / RTC_BK;
    const uint32_t stage_tx = 2 * RTC_A_BYTES + 2 * NT * RTC_BK;

    if (threadIdx.x == 0) {
        *failed = 0;
        for (int s = 0; s < RTC_STAGES; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        mbar_init(drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tXh);
        tma_prefetch_desc(&tXl);
        tma_prefetch_desc(&tWh);
        tma_prefetch_desc(&tWl);
    }
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();
    pdl_trigger();
    const long long limit = p.spin_limit;

    if (warp == 0) {
        if (lane == 0) {
            int kb = 0;
            for (; kb < num_kb; kb++) {
                const int s = kb % RTC_STAGES;
                if (!mbar_wait(&empty[s], ((kb / RTC_STAGES) & 1) ^ 1, limit)) {
                    report(p.status, ST_TIMEOUT, WHERE_ROUTER);
                    break;
                }
                uint8_t* st = smem + s * RTC_STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], stage_tx);
                tma_load_2d(st, &tXh, &full[s], kb * RTC_BK, m0);
                tma_load_2d(st + RTC_A_BYTES, &tXl, &full[s], kb * RTC_BK, m0);
                tma_load_2d(st + 2 * RTC_A_BYTES, &tWh, &full[s], kb * RTC_BK, n0);
                tma_load_2d(st + 2 * RTC_A_BYTES + RTC_B_BYTES, &tWl, &full[s], kb * RTC_BK, n0);
            }
            // copies in flight land before the CTA may exit
            const int first = kb > RTC_STAGES ? kb - RTC_STAGES : 0;
            for (int j = first; j < kb; j++) mbar_wait(&full[j % RTC_STAGES], (j / RTC_STAGES) & 1, DRAIN_LIMIT);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_s8(RTC_BM, NT);
            const uint32_t d_hh = tmem_base, d_x = tmem_base + NT, d_ll = tmem_base + 2 * NT;
            for (int kb = 0; kb < num_kb; kb++) {
                const int s = kb % RTC_STAGES;
                if (!mbar_wait(&full[s], (kb / RTC_STAGES) & 1, limit)) {
                    report(p.status, ST_TIMEOUT, WHERE_ROUTER);
                    *failed = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t ah = smem_u32(smem + s * RTC_STAGE_BYTES);
                const uint32_t al = ah + RTC_A_BYTES, bh = ah + 2 * RTC_A_BYTES, bl = bh + RTC_B_BYTES;
#pragma unroll
                for (int kk = 0; kk < RTC_BK / 32; kk++) {
                    const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
                    mma_s8(d_hh, sdesc_sw128(ah + 32 * kk), sdesc_sw128(bh + 32 * kk), idesc, acc);
                    mma_s8(d_x, sdesc_sw128(ah + 32 * kk), sdesc_sw128(bl + 32 * kk), idesc, acc);
                    mma_s8(d_x, sdesc_sw128(al + 32 * kk), sdesc_sw128(bh + 32 * kk), idesc, 1u);
                    mma_s8(d_ll, sdesc_sw128(al + 32 * kk), sdesc_sw128(bl + 32 * kk), idesc, acc);
                }
                mma_commit(&empty[s]);
            }
            __threadfence_block();  // the failure flag is visible before the arrival
            mma_commit(tfull);      // the sums are complete (after a failed wait the
            mma_commit(drain);      // epilogue sees the flag and stores nothing)
            mbar_wait(drain, 0, DRAIN_LIMIT);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const int t = m0 + r;
        const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
        // warp-uniform outcome, so the .sync.aligned TMEM loads run on every lane or none
        const bool got = __all_sync(0xffffffffu, mbar_wait(tfull, 0, limit));
        const bool mma_ok = __all_sync(0xffffffffu, *failed == 0);
        if (!got) {
            if (lane == 0) report(p.status, ST_TIMEOUT, WHERE_ROUTER);
        } else if (mma_ok) {
            tc_fence_after();
            const int ex = t < p.T ? p.x_exp[t] : 0;
            for (int c0 = 0; c0 < NT; c0 += 32) {
                float vh[32], vx[32], vl[32];
                tmem_ld32x2(lane_addr + c0, lane_addr + NT + c0, vh, vx);
                tmem_ld32(lane_addr + 2 * NT + c0, vl);
                if (t < p.T) {
                    float* dst = p.logits + static_cast<size_t>(t) * p.E;
#pragma unroll
                    for (int c = 0; c < 32; c++) {
                        const int e = n0 + c0 + c;
                        if (e >= p.E) continue;
                        const double s = static_cast<double>(__float_as_int(vh[c])) * 65536.0 +
                                         static_cast<double>(__float_as_int(vx[c])) * 256.0 +
                                         static_cast<double>(__float_as_int(vl[c]));
                        double l = ldexp(s, ex + __ldg(p.w_exp + e) - 28);
                        if (p.bias) l += static_cast<double>(__ldg(p.bias + e));
                        dst[e] = static_cast<float>(l);
                    }
                }
            }
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// Bound D of |C - fp32(L~)| for token t and expert e (see the file comment).
__device__ __forceinline__ double router_bound(int ex, double sx, float mx, int ew, double sw, double swq, float mw,
                                               float bias_abs, float l, double gamma) {
    const double eps_x = ldexp(1.0, ex - 15), eps_w = ldexp(1.0, ew - 15);
    const double dfix = eps_w * sx + eps_x * swq;
    const double sxw = fmin(sx * static_cast<double>(mw), static_cast<double>(mx) * sw);
    const double dcan = gamma * (sxw + static_cast<double>(bias_abs));
    const double dst = ldexp(fabs(static_cast<double>(l)), -23);
    return (dfix + dcan + dst) * (1.0 + 0x1p-20);
}

// The canonical fp32 logits of token t for up to RS_BATCH experts es[0..n),
// computed by one warp: lane l runs each expert's chain over h = 256 i + 8 l + j
// (i, then j = 0..7), the chains advancing together so that their loads
// overlap; the xor butterfly over offsets 1..16 forms the pairwise tree on
// every lane, then + bias.  Per expert the same operations as
// router_logits_small_kernel, so the same bits.
constexpr int RS_BATCH = 8;
__device__ __forceinline__ void canonical_logits(const RouterParams& p, int t, const int* es, int n, int lane,
                                                 float* out) {
    const __nv_bfloat16* xrow = p.x + static_cast<size_t>(t) * p.H + 8 * lane;
    float acc[RS_BATCH];
#pragma unroll
    for (int c = 0; c < RS_BATCH; c++) acc[c] = 0.0f;
    const int nI = p.H >> 8;
    for (int i = 0; i < nI; i++) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xrow + 256 * i));
        float4 wa[RS_BATCH], wb[RS_BATCH];
#pragma unroll
        for (int c = 0; c < RS_BATCH; c++) {
            if (c < n) {
                const float* w = p.wr + static_cast<size_t>(es[c]) * p.H + 8 * lane + 256 * i;
                wa[c] = __ldg(reinterpret_cast<const float4*>(w));
                wb[c] = __ldg(reinterpret_cast<const float4*>(w + 4));
            }
        }
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int c = 0; c < RS_BATCH; c++) {
            if (c < n) {
                const float wv[8] = {wa[c].x, wa[c].y, wa[c].z, wa[c].w, wb[c].x, wb[c].y, wb[c].z, wb[c].w};
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const float xj = (j & 1) ? bf16_hi(xw[j >> 1]) : bf16_lo(xw[j >> 1]);
                    acc[c] = __fmaf_rn(xj, wv[j], acc[c]);
                }
            }
        }
    }
#pragma unroll
    for (int c = 0; c < RS_BATCH; c++) {
        if (c < n) {
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) acc[c] = __fadd_rn(acc[c], __shfl_xor_sync(0xffffffffu, acc[c], off));
            if (p.bias) acc[c] = __fadd_rn(acc[c], p.bias[es[c]]);
            out[c] = acc[c];
        }
    }
}

// One warp per token: bounds, the k-th largest lower bound, candidates, their
// canonical logits (written over the approximations), then the top k of the
// candidates and the weights exactly as router_topk_token computes them.
__global__ void __launch_bounds__(256) router_select_kernel(RouterParams p, RouterFix f) {
    __shared__ int s_list[8][256];
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int nm = (p.E + 31) >> 5;
    const double nr = static_cast<double>((p.H >> 5) + 6) * 0x1p-24;
    const double gamma = nr / (1.0 - nr);
    for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < p.T; t += gridDim.x * 8) {
        float* lrow = p.logits + static_cast<size_t>(t) * p.E;
        const int ex = f.x_exp[t];
        const double sx = f.x_sum[t];
        const float mx = f.x_max[t];
        float lv[8];
        double dv[8];
#pragma unroll
        for (int m = 0; m < 8; m++) {
            const int e = 32 * m + lane;
            lv[m] = 0.0f;
            dv[m] = 0.0;
            if (m < nm && e < p.E) {
                lv[m] = lrow[e];
                dv[m] = router_bound(ex, sx, mx, f.w_exp[e], f.w_sum[e], f.w_sumq[e], f.w_max[e],
                                     p.bias ? fabsf(p.bias[e]) : 0.0f, lv[m], gamma);
            }
        }
        // LB_k: the k-th largest lower bound (k rounds of a warp maximum)
        uint32_t taken = 0;
        double lbk = 0.0;
        for (int j = 0; j < p.k; j++) {
            double bv = -INFINITY;
            int bm = -1;
#pragma unroll
            for (int m = 0; m < 8; m++) {
                if (m >= nm || 32 * m + lane >= p.E || ((taken >> m) & 1u)) continue;
                const double lb = static_cast<double>(lv[m]) - dv[m];
                if (bm < 0 || lb > bv) { bv = lb; bm = m; }
            }
            int owner = bm >= 0 ? lane : 32;
            double wv = bv;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const double ov = __shfl_xor_sync(0xffffffffu, wv, off);
                const int oo = __shfl_xor_sync(0xffffffffu, owner, off);
                if (oo < 32 && (owner == 32 || ov > wv || (ov == wv && oo < owner))) { wv = ov; owner = oo; }
            }
            // the winning lane marks its best slot as taken
            if (owner == lane) taken |= 1u << bm;
            lbk = wv;
        }
        // candidates: upper bound reaches LB_k; their canonical logits
        uint32_t cand = 0;
#pragma unroll
        for (int m = 0; m < 8; m++) {
            const int e = 32 * m + lane;
            if (m < nm && e < p.E && static_cast<double>(lv[m]) + dv[m] >= lbk) cand |= 1u << m;
        }
        // the candidates in expert order (a per-warp list in shared memory),
        // RS_BATCH at a time; lane e % 32 keeps expert e's canonical logit
        int* list = s_list[threadIdx.x >> 5];
        int ncand = 0;
#pragma unroll
        for (int m = 0; m < 8; m++) {
            const bool c = m < nm && ((cand >> m) & 1u);
            const uint32_t bal = __ballot_sync(0xffffffffu, c);
            if (c) list[ncand + __popc(bal & ((1u << lane) - 1u))] = 32 * m + lane;
            ncand += __popc(bal);
        }
        __syncwarp();
        float cv[8];
#pragma unroll
        for (int m = 0; m < 8; m++) cv[m] = 0.0f;
        for (int b0 = 0; b0 < ncand; b0 += RS_BATCH) {
            const int n = min(RS_BATCH, ncand - b0);
            int es[RS_BATCH];
#pragma unroll
            for (int q = 0; q < RS_BATCH; q++) es[q] = q < n ? list[b0 + q] : 0;
            float c[RS_BATCH];
            canonical_logits(p, t, es, n, lane, c);
#pragma unroll
            for (int q = 0; q < RS_BATCH; q++) {
                if (q < n && (es[q] & 31) == lane) {
                    const int mq = es[q] >> 5;
#pragma unroll
                    for (int m = 0; m < 8; m++)
                        if (m == mq) cv[m] = c[q];
                    lrow[es[q]] = c[q];
                }
            }
        }
        __syncwarp();   // the list is rewritten for the warp's next token
        router_topk_candidates(p, cv, cand, t, lane);
    }
}

}  // namespace moe
