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
//    is the exact dot product of the rounded rows (+ bias).  The integer sum
//    is exact in 64 bits; it is rounded once to fp32, scaled by an exact power
//    of two and rounded once more by the bias add, and stored.  |int32 sums| <= 2^14 * 2 H * 64, so
//    H <= 65536 cannot overflow.
// 3. Certified filter (router_select_kernel).  With eps = 2^(e - 15) the
//    rounding of one value (half a unit), the exact logit L* = sum x w + b and
//    the canonical fp32 logit C (n = H/32 fused multiply-adds per chain, a
//    5-level tree, one bias add: at most n + 6 roundings on any path),
//        |L~ - L*| <= eps_w sum|x| + eps_x sum|w~|              (fixed point)
//        |C  - L*| <= gamma(n + 6) (sum|x w| + |b|),             gamma(m) = m u / (1 - m u), u = 2^-24
//        |l - L~| <= 2^-23 (|l| + |b|) + 2^-126     (l: L~ evaluated in fp32, stored),
//    with sum|x w| <= min(sum|x| max|w|, max|x| sum|w|).  So C lies in
//    [l - D, l + D] around the stored l, D their sum (x (1 + 2^-20) for the
//    fp64 evaluation of D itself).  Let LB_k be the k-th largest
//    l - D of the token.  An expert with l + D < LB_k has k experts whose C
//    is strictly larger, so it is not among the canonical top k whatever the
//    tie rule; every other expert is a candidate.  The candidates get the
//    canonical C (same chains and tree as router.cuh), the top k of the
//    candidates by C (ties to the lower id) is the canonical top k, and the
//    weights are computed from those C exactly as on the SIMT path.
// The logits buffer then holds C for the candidates (a superset of the
// selected experts) and l for the others.
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

// 2^k as a float; outside the normal range the value is tiny or huge and the
// product is formed by ldexpf (exact scaling either way, up to the final rounding)
__device__ __forceinline__ float pow2_or_ldexp(int k) {
    return (k >= -126 && k <= 127) ? __int_as_float((127 + k) << 23) : ldexpf(1.0f, k);
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
    // the tile's expert exponents and biases, once per CTA
    __shared__ int s_wexp[RTC_NT_MAX];
    __shared__ float s_bias[RTC_NT_MAX];
    for (int c = threadIdx.x; c < NT; c += blockDim.x) {
        const int e = n0 + c;
        s_wexp[c] = e < p.E ? p.w_exp[e] : 0;
        s_bias[c] = (e < p.E && p.bias) ? p.bias[e] : 0.0f;
    }
    __syncthreads();

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
            const bool vec = (p.E & 3) == 0;
            for (int c0 = 0; c0 < NT; c0 += 32) {
                float vh[32], vx[32], vl[32];
                tmem_ld32x2(lane_addr + c0, lane_addr + NT + c0, vh, vx);
                tmem_ld32(lane_addr + 2 * NT + c0, vl);
                if (t < p.T) {
                    float* dst = p.logits + static_cast<size_t>(t) * p.E + n0 + c0;
                    float out[32];
#pragma unroll
                    for (int c = 0; c < 32; c++) {
                        // 65536 S_hh + 256 S_x + S_ll is exact in 64 bits; one rounding to
                        // fp32, an exact power-of-two scale, one rounding of the bias add
                        const long long si = (static_cast<long long>(__float_as_int(vh[c])) << 16) +
                                             (static_cast<long long>(__float_as_int(vx[c])) << 8) +
                                             static_cast<long long>(__float_as_int(vl[c]));
                        const float l = __fmul_rn(__ll2float_rn(si), pow2_or_ldexp(ex + s_wexp[c0 + c] - 28));
                        out[c] = __fadd_rn(l, s_bias[c0 + c]);
                    }
                    if (vec && n0 + c0 + 32 <= p.E) {
#pragma unroll
                        for (int c = 0; c < 32; c += 4)
                            *reinterpret_cast<float4*>(dst + c) = make_float4(out[c], out[c + 1], out[c + 2], out[c + 3]);
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; c++)
                            if (n0 + c0 + c < p.E) dst[c] = out[c];
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

// 2^k as a double (k inside the normal range, as every exponent here is)
__device__ __forceinline__ double pow2d(int k) { return __longlong_as_double(static_cast<long long>(1023 + k) << 52); }

// Bound D of |C - l| for token t and expert e, l the stored approximation (see
// the file comment): the fixed-point term, the canonical chain's term, and
// the fp32 evaluation of l (one rounding of the integer sum, one of the bias
// add: within 2^-23 (|l| + |b|), plus 2^-126 for scales outside the normal
// range).
__device__ __forceinline__ double router_bound(double eps_x, double sx, float mx, double eps_w, double sw, double swq,
                                               float mw, float babs, float l, double gamma) {
    const double dfix = eps_w * sx + eps_x * swq;
    const double sxw = fmin(sx * static_cast<double>(mw), static_cast<double>(mx) * sw);
    const double dcan = gamma * (sxw + static_cast<double>(babs));
    const double dst = (fabs(static_cast<double>(l)) + static_cast<double>(babs)) * 0x1p-23 + 0x1p-126;
    return (dfix + dcan + dst) * (1.0 + 0x1p-20);
}

// The canonical fp32 logits of (token t, experts e0 and e1) computed by one
// warp: lane l runs each expert's chain over h = 256 i + 8 l + j (i, then
// j = 0..7); the two chains share each packed fma (fma.rn.f32x2: two
// independent round-to-nearest fma, the same as two scalar ones).  The xor
// butterfly over offsets 1..16 forms the pairwise tree on every lane, then
// + bias.  Per expert the same operations as router_logits_small_kernel, so
// the same bits.  With two == false only e0 is computed.
__device__ __forceinline__ void canonical_logit2(const RouterParams& p, int t, int e0, int e1, bool two, int lane,
                                                 float& c0, float& c1) {
    const float* w0 = p.wr + static_cast<size_t>(e0) * p.H + 8 * lane;
    const float* w1 = p.wr + static_cast<size_t>(two ? e1 : e0) * p.H + 8 * lane;
    const __nv_bfloat16* xrow = p.x + static_cast<size_t>(t) * p.H + 8 * lane;
    float a0 = 0.0f, a1 = 0.0f;
    const int nI = p.H >> 8;
#pragma unroll 2
    for (int i = 0; i < nI; i++) {
        const float4 pa = __ldg(reinterpret_cast<const float4*>(w0 + 256 * i));
        const float4 pb = __ldg(reinterpret_cast<const float4*>(w0 + 256 * i + 4));
        const float4 qa = __ldg(reinterpret_cast<const float4*>(w1 + 256 * i));
        const float4 qb = __ldg(reinterpret_cast<const float4*>(w1 + 256 * i + 4));
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xrow + 256 * i));
        const float wp[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
        const float wq[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const float xj = (j & 1) ? bf16_hi(xw[j >> 1]) : bf16_lo(xw[j >> 1]);
            // chain 0 += xj * wp[j], chain 1 += xj * wq[j]
            asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %2};\n\tmov.b64 rb, {%3, %4};\n\t"
                "mov.b64 rd, {%0, %1};\n\tfma.rn.f32x2 rd, ra, rb, rd;\n\tmov.b64 {%0, %1}, rd;\n\t}"
                : "+f"(a0), "+f"(a1)
                : "f"(xj), "f"(wp[j]), "f"(wq[j]));
        }
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        a0 = __fadd_rn(a0, __shfl_xor_sync(0xffffffffu, a0, off));
        a1 = __fadd_rn(a1, __shfl_xor_sync(0xffffffffu, a1, off));
    }
    if (p.bias) {
        a0 = __fadd_rn(a0, p.bias[e0]);
        if (two) a1 = __fadd_rn(a1, p.bias[e1]);
    }
    c0 = a0;
    c1 = a1;
}

// (v, id) ranks before (v', id') when v > v', or v == v' and id < id' (the
// selection order: larger logit first, ties to the lower id)
__device__ __forceinline__ bool rank_before(float v, int id, float v2, int id2) {
    return v > v2 || (v == v2 && id < id2);
}

// More candidates than lanes (8-9 per token on the workloads, so rare): k
// rounds of a warp argmax over them, as router_topk_select; lane l reads back
// the canonical logits it wrote (experts l + 32 m).  Out of line, so that its
// registers do not weigh on the common path.
__device__ __noinline__ void select_among_many(const float* lrow, uint32_t cand, int t, int E, int k, int score,
                                               int32_t* ids, float* w, int lane) {
    RouterParams q;
    q.x = nullptr;
    q.wr = nullptr;
    q.bias = nullptr;
    q.logits = nullptr;
    q.ids = ids;
    q.w = w;
    q.T = 0;
    q.H = 0;
    q.E = E;
    q.k = k;
    q.score = score;
    float cv[8];
#pragma unroll
    for (int m = 0; m < 8; m++) cv[m] = ((cand >> m) & 1u) ? lrow[32 * m + lane] : 0.0f;
    router_topk_candidates(q, cv, cand, t, lane);
}

// One warp per token: bounds, the k-th largest lower bound, candidates, their
// canonical logits (written over the approximations), then the top k of the
// candidates and the weights, computed as router_topk_select computes them.
__global__ void __launch_bounds__(256, 4) router_select_kernel(RouterParams p, RouterFix f) {
    __shared__ int s_list[8][256];
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int nm = (p.E + 31) >> 5;
    const double nr = static_cast<double>((p.H >> 5) + 6) * 0x1p-24;
    const double gamma = nr / (1.0 - nr);
    int* list = s_list[threadIdx.x >> 5];
    for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < p.T; t += gridDim.x * 8) {
        float* lrow = p.logits + static_cast<size_t>(t) * p.E;
        const double eps_x = pow2d(f.x_exp[t] - 15);
        const double sx = f.x_sum[t];
        const float mx = f.x_max[t];
        // bounds of the canonical logits, rounded outward to fp32 (only looser)
        float srt[8], ub[8];   // srt: the lower bounds, sorted below
#pragma unroll
        for (int m = 0; m < 8; m++) {
            const int e = 32 * m + lane;
            srt[m] = -INFINITY;
            ub[m] = -INFINITY;
            if (m < nm && e < p.E) {
                const float l = lrow[e];
                const double d = router_bound(eps_x, sx, mx, pow2d(f.w_exp[e] - 15), f.w_sum[e], f.w_sumq[e],
                                              f.w_max[e], p.bias ? fabsf(p.bias[e]) : 0.0f, l, gamma);
                srt[m] = __double2float_rd(static_cast<double>(l) - d);
                ub[m] = __double2float_ru(static_cast<double>(l) + d);
            }
            // four experts' loads at a time in flight (fewer live registers)
            if (m == 3) asm volatile("" ::: "memory");
        }
        // LB_k, the k-th largest lower bound: each lane sorts its eight lower
        // bounds (descending), then k rounds take the warp maximum of the
        // lanes' current heads and advance the winning lane's head
#pragma unroll
        for (int i = 0; i < 8; i++)
#pragma unroll
            for (int j = 7; j > i; j--)
                if (srt[j] > srt[j - 1]) {
                    const float tmp = srt[j];
                    srt[j] = srt[j - 1];
                    srt[j - 1] = tmp;
                }
        float lbk = -INFINITY;
        for (int j = 0; j < p.k; j++) {
            const float head = srt[0];
            float wv = head;
            int owner = lane;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, wv, off);
                const int oo = __shfl_xor_sync(0xffffffffu, owner, off);
                if (ov > wv || (ov == wv && oo < owner)) { wv = ov; owner = oo; }
            }
            lbk = wv;
            if (owner == lane) {
#pragma unroll
                for (int m = 0; m < 7; m++) srt[m] = srt[m + 1];
                srt[7] = -INFINITY;
            }
        }
        // candidates: upper bound reaches LB_k; a per-warp list in expert order
        uint32_t cand = 0;
        int ncand = 0;
#pragma unroll
        for (int m = 0; m < 8; m++) {
            const bool c = m < nm && 32 * m + lane < p.E && ub[m] >= lbk;
            cand |= (c ? 1u : 0u) << m;
            const uint32_t bal = __ballot_sync(0xffffffffu, c);
            if (c) list[ncand + __popc(bal & ((1u << lane) - 1u))] = 32 * m + lane;
            ncand += __popc(bal);
        }
        __syncwarp();
        // their canonical logits, two at a time, written over the
        // approximations in the logits row; lane i < 32 also holds candidate
        // i's (for the sort below)
        float my_v = -INFINITY;
        int my_e = 0x7FFFFFFF;
        for (int i = 0; i < ncand; i += 2) {
            const bool two = i + 1 < ncand;
            const int e0 = list[i], e1 = two ? list[i + 1] : e0;
            float c0, c1;
            canonical_logit2(p, t, e0, e1, two, lane, c0, c1);
#pragma unroll
            for (int h = 0; h < 2; h++) {
                if (h == 1 && !two) break;
                const int e = h ? e1 : e0;
                const float c = h ? c1 : c0;
                if ((e & 31) == lane) lrow[e] = c;
                if (lane == i + h) {
                    my_v = c;
                    my_e = e;
                }
            }
        }
        __syncwarp();   // the list is rewritten for the warp's next token
        if (ncand > 32) {
            select_among_many(lrow, cand, t, p.E, p.k, p.score, p.ids, p.w, lane);
            continue;
        }
        // at most 32 candidates: a bitonic sort over the lanes in selection order
#pragma unroll
        for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, my_v, stride);
                const int oe = __shfl_xor_sync(0xffffffffu, my_e, stride);
                const bool lower = (lane & stride) == 0;           // this lane keeps the earlier rank ...
                const bool up = (lane & size) == 0;                // ... in an ascending-rank block
                const bool other_first = rank_before(ov, oe, my_v, my_e);
                if (lower == up ? other_first : !other_first) {
                    my_v = ov;
                    my_e = oe;
                }
            }
        }
        // lanes 0..k-1 hold the top k in order; weights as router_topk_select
        float sel_v[8];
#pragma unroll
        for (int j = 0; j < 8; j++) sel_v[j] = __shfl_sync(0xffffffffu, my_v, j);
        if (lane == 0) {
            float z[8], sum = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; j++) {
                if (j >= p.k) break;
                z[j] = (p.score == 0) ? expf(sel_v[j] - sel_v[0]) : 1.0f / (1.0f + expf(-sel_v[j]));
                sum += z[j];
            }
#pragma unroll
            for (int j = 0; j < 8; j++) {
                if (j >= p.k) break;
                p.w[static_cast<size_t>(t) * p.k + j] = z[j] / sum;
            }
        }
        if (lane < p.k) p.ids[static_cast<size_t>(t) * p.k + lane] = my_e;
    }
}

}  // namespace moe
