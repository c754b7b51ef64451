// router.cuh -- router logits, top-k and routing weights.
//
// Alpha-MoE article ("How the megakernel works"): routing is the first stage
// of the fused MoE pass.  LightMoE README ("MoE inference"): top_k_ids int32
// with distinct experts per token, top_k_weights fp32.
//
// Logit order (fixed, so that the selected ids are reproducible bit for bit):
// lane l of a warp owns h = 256 i + 8 l + j and runs one fp32 fused
// multiply-add chain over i ascending, then j = 0..7, starting from +0; the 32
// lane sums are combined by an xor butterfly over offsets 1, 2, 4, 8, 16, which
// adds them as the balanced pairwise tree ((p0+p1)+(p2+p3))+...; then + bias[e].
//
// Kernels:
//  router_logits_kernel  a 2-D grid of CTA tiles (TOK tokens x EXP experts; 64 x 16
//                        with 16-token x 8-expert micro-tiles, or 32 x 8 with
//                        4 x 8 micro-tiles when E <= 8).
//                        The 256-wide H chunks of X and Wr go through shared
//                        memory with a 4-stage cp.async pipeline; each warp
//                        owns one micro-tile: per 16 bytes read from
//                        shared memory, 16 x 8 runs 64 fma; two tokens' chains
//                        share each packed fp32 fma (fma.rn.f32x2).
//  router_logits_small_kernel  batches of at most 128 tokens: one warp per
//                        (expert, 4 tokens) reading global memory directly.
//  router_small_fused_kernel   the same for at most 32 experts, with the top-k
//                        of the CTA's 4 tokens in the same launch.
//  router_topk_kernel    one warp per token: k rounds of a warp argmax over
//                        the token's logits, then softmax or sigmoid weights.
#pragma once
#include "common.cuh"

namespace moe {

// A CTA tile of TOK tokens x EXP experts: one warp per micro-tile of MT
// tokens x 8 experts.
template <int TOK, int EXP, int MT>
struct RouterTile {
    static constexpr int NW = (TOK / MT) * (EXP / 8);
    static constexpr int NT = 32 * NW;
    static constexpr int X_BYTES = TOK * 256 * 2;    // 256 bf16 of H per token
    static constexpr int W_BYTES = EXP * 256 * 4;    // 256 fp32 of H per expert
    static constexpr int STAGE = X_BYTES + W_BYTES;
    static constexpr int NSTAGE = 4;                 // 3 chunks in flight hide L2 latency
    static constexpr int SMEM = NSTAGE * STAGE;      // 128 KB (32 x 16) or 160 KB (64 x 8)
};

struct RouterParams {
    const __nv_bfloat16* x;
    const float* wr;
    const float* bias;   // nullable
    float* logits;       // [T, E] fp32 workspace
    int32_t* ids;
    float* w;
    int T, H, E, k, score;
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
    const uint32_t s = smem_u32(smem);
    const int n = valid ? 16 : 0;   // n = 0 writes zeros and reads nothing
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait2() { asm volatile("cp.async.wait_group 2;" ::: "memory"); }
// wait until at most n (0..3, clamped) of this thread's newest groups are pending
__device__ __forceinline__ void cp_async_wait_le(int n) {
    if (n >= 3) asm volatile("cp.async.wait_group 3;" ::: "memory");
    else if (n == 2) asm volatile("cp.async.wait_group 2;" ::: "memory");
    else if (n == 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
    else asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// The 16-byte pieces one of the NT threads copies for every H chunk: X piece
// m is row (tid / 32) + (NT / 32) m, column 8 (tid % 32); Wr piece m is row
// (tid / 64) + (NT / 64) m, column 4 (tid % 64).  Base pointers and validity
// are fixed per thread, so a chunk costs one add and one cp.async per piece.
// Rows past T or E read nothing and are zero-filled.
template <int TOK, int EXP, int NT>
struct RouterLoader {
    static constexpr int XR = NT / 32, WR = NT / 64;   // rows per pass
    static constexpr int XP = TOK / XR;                // X pieces per thread
    static constexpr int WP = EXP / WR;                // Wr pieces per thread
    static_assert(XP * XR == TOK && WP * WR == EXP, "whole passes");
    const __nv_bfloat16* xb;
    const float* wb;
    uint32_t xvalid, wvalid;   // bit m: piece m is inside the tensor
    int H;
    uint32_t xdst, wdst;       // shared-memory byte offsets of piece 0

    __device__ __forceinline__ RouterLoader(const RouterParams& p, int t0, int e0) {
        const int tid = threadIdx.x;
        H = p.H;
        xvalid = wvalid = 0;
        const int xr = tid >> 5, xc = tid & 31;
        const int wr = tid >> 6, wc = tid & 63;
#pragma unroll
        for (int m = 0; m < XP; m++) xvalid |= (t0 + xr + XR * m < p.T ? 1u : 0u) << m;
#pragma unroll
        for (int m = 0; m < WP; m++) wvalid |= (e0 + wr + WR * m < p.E ? 1u : 0u) << m;
        xb = p.x + static_cast<size_t>(xvalid & 1u ? t0 + xr : 0) * p.H + 8 * xc;
        wb = p.wr + static_cast<size_t>(wvalid & 1u ? e0 + wr : 0) * p.H + 4 * wc;
        xdst = xr * 512 + xc * 16;
        // Wr piece c holds h = 4c..4c+3, half (c & 1) of lane (c >> 1)'s eight values;
        // stored at (c & 1) * 512 + (c >> 1) * 16 so each half-read of a warp is
        // 512 contiguous bytes (no bank conflicts)
        wdst = TOK * 512 + wr * 1024 + (wc & 1) * 512 + (wc >> 1) * 16;   // after the X rows
    }
    __device__ __forceinline__ void load(uint8_t* st, int i) const {
#pragma unroll
        for (int m = 0; m < XP; m++) {
            const bool ok = (xvalid >> m) & 1u;
            cp_async16(st + xdst + m * XR * 512, ok ? xb + static_cast<size_t>(XR * m) * H + 256 * i : xb, ok);
        }
#pragma unroll
        for (int m = 0; m < WP; m++) {
            const bool ok = (wvalid >> m) & 1u;
            cp_async16(st + wdst + m * WR * 1024, ok ? wb + static_cast<size_t>(WR * m) * H + 256 * i : wb, ok);
        }
        cp_async_commit();
    }
};

// One step of the lane butterfly: of the 2 HALF values in `in`, a lane keeps
// the upper half if (lane & off), else the lower, and adds the partner lane's
// copy of the kept half.
template <int HALF>
__device__ __forceinline__ void butterfly_halve(const float* in, float* out, int lane, int off) {
    const bool b = lane & off;
#pragma unroll
    for (int v = 0; v < HALF; v++) {
        const float send = b ? in[v] : in[v + HALF], keep = b ? in[v + HALF] : in[v];
        out[v] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, off));
    }
}

// d0 = fma(a0, b, d0), d1 = fma(a1, b, d1), each rounded to nearest (one
// packed sm_100 instruction for two independent chains).
__device__ __forceinline__ void fma2_rn(float& d0, float& d1, float a0, float a1, float b) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\t"
        "mov.b64 rd, {%0, %1};\n\tfma.rn.f32x2 rd, ra, rb, rd;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1), "f"(b));
}

template <int TOK, int EXP, int MT>
__global__ void __launch_bounds__(RouterTile<TOK, EXP, MT>::NT, 1) router_logits_kernel(RouterParams p) {
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_ROUTER);
    using RT = RouterTile<TOK, EXP, MT>;
    extern __shared__ __align__(16) uint8_t rsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * TOK, e0 = blockIdx.y * EXP;
    const int tg = warp % (TOK / MT), eg = warp / (TOK / MT);   // this warp's micro-tile
    const int nI = p.H >> 8;

    float acc[MT][8];
#pragma unroll
    for (int a = 0; a < MT; a++)
#pragma unroll
        for (int b = 0; b < 8; b++) acc[a][b] = 0.0f;

    const RouterLoader<TOK, EXP, RT::NT> ld(p, t0, e0);
    // prologue: chunks 0 .. NSTAGE-2 in flight
    for (int c = 0; c < RT::NSTAGE - 1 && c < nI; c++) ld.load(rsm + c * RT::STAGE, c);
    for (int i = 0; i < nI; i++) {
        uint8_t* st = rsm + (i % RT::NSTAGE) * RT::STAGE;
        // chunk i is complete once at most the groups issued after it (chunks
        // i + 1 .. i + NSTAGE - 2) are pending
        cp_async_wait_le(min(nI - 1 - i, RT::NSTAGE - 2));
        // one barrier per chunk: chunk i is visible to every warp, and every
        // warp is done with chunk i - 1, whose stage the next load refills
        __syncthreads();
        const int ahead = i + RT::NSTAGE - 1;
        if (ahead < nI) ld.load(rsm + (ahead % RT::NSTAGE) * RT::STAGE, ahead);
        const uint8_t* xs = st + (MT * tg) * 512 + lane * 16;
        const uint8_t* ws = st + RT::X_BYTES + (8 * eg) * 1024 + lane * 16;
        // MT tokens x 8 experts: the lane's 8 values per row go in two halves
        // (j = 0..3, then 4..7), so each chain still runs j in order.  Tokens
        // 2 tp and 2 tp + 1 share one packed fma per (expert, j): two
        // independent round-to-nearest fp32 fma, the same as two scalar ones.
        static_assert(MT % 2 == 0, "token pairs");
#pragma unroll
        for (int jh = 0; jh < 2; jh++) {
            float wv[8][4];
#pragma unroll
            for (int ee = 0; ee < 8; ee++) {
                const float4 w4 = *reinterpret_cast<const float4*>(ws + ee * 1024 + jh * 512);
                wv[ee][0] = w4.x; wv[ee][1] = w4.y; wv[ee][2] = w4.z; wv[ee][3] = w4.w;
            }
            uint32_t xw[MT][2];
#pragma unroll
            for (int tt = 0; tt < MT; tt++) {
                const uint2 x2 = *reinterpret_cast<const uint2*>(xs + tt * 512 + jh * 8);
                xw[tt][0] = x2.x; xw[tt][1] = x2.y;
            }
#pragma unroll
            for (int j = 0; j < 4; j++) {
                float xj[MT];
#pragma unroll
                for (int tt = 0; tt < MT; tt++) xj[tt] = (j & 1) ? bf16_hi(xw[tt][j >> 1]) : bf16_lo(xw[tt][j >> 1]);
#pragma unroll
                for (int tp = 0; tp < MT / 2; tp++)
#pragma unroll
                    for (int ee = 0; ee < 8; ee++)
                        fma2_rn(acc[2 * tp][ee], acc[2 * tp + 1][ee], xj[2 * tp], xj[2 * tp + 1], wv[ee][j]);
            }
        }
    }
    // Sum the 32 lane partials of all NV = 8 MT (token, expert) pairs by
    // recursive halving over lane offsets 1, 2, 4, 8, 16: at each step a lane
    // keeps half of its values and adds the partner's copy of that half, so every
    // sum is the pairwise tree ((p0+p1)+(p2+p3))+... of the fixed order.
    // Afterwards lane l holds pairs NV/32 r(l) .. NV/32 r(l) + NV/32 - 1,
    // r = 5-bit reversal of l.
    constexpr int NV = MT * 8;
    float h1[NV / 2], h2[NV / 4], h3[NV / 8], h4[NV / 16], av[NV / 32];
    butterfly_halve<NV / 2>(&acc[0][0], h1, lane, 1);
    butterfly_halve<NV / 4>(h1, h2, lane, 2);
    butterfly_halve<NV / 8>(h2, h3, lane, 4);
    butterfly_halve<NV / 16>(h3, h4, lane, 8);
    butterfly_halve<NV / 32>(h4, av, lane, 16);
    const int rl = ((lane & 1) << 4) | ((lane & 2) << 2) | (lane & 4) | ((lane & 8) >> 2) | ((lane & 16) >> 4);
#pragma unroll
    for (int u = 0; u < NV / 32; u++) {
        const int idx = (NV / 32) * rl + u;
        const int t = t0 + MT * tg + (idx >> 3), e = e0 + 8 * eg + (idx & 7);
        if (t < p.T && e < p.E) {
            float val = av[u];
            if (p.bias) val = __fadd_rn(val, p.bias[e]);
            p.logits[static_cast<size_t>(t) * p.E + e] = val;
        }
    }
}

// Small batches: one warp per (expert, group of RS_TG tokens), straight from
// global memory (X rows stay in L1/L2, each Wr row is read once per token
// group), 4 experts per CTA.  Same chains and tree as the tiled kernel: lane l
// runs the fma chain over h = 256 i + 8 l + j, and the xor butterfly over
// offsets 1, 2, 4, 8, 16 forms the same pairwise sums on every lane.
constexpr int RS_TG = 4;
constexpr int RS_WARPS = 4;
__global__ void __launch_bounds__(RS_WARPS * 32) router_logits_small_kernel(RouterParams p) {
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_ROUTER_SMALL);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.y * RS_WARPS + warp;
    const int t0 = blockIdx.x * RS_TG;
    if (e >= p.E) return;
    const float* wrow = p.wr + static_cast<size_t>(e) * p.H + 8 * lane;
    const __nv_bfloat16* xrow[RS_TG];
#pragma unroll
    for (int tt = 0; tt < RS_TG; tt++)
        xrow[tt] = p.x + static_cast<size_t>(t0 + tt < p.T ? t0 + tt : t0) * p.H + 8 * lane;
    float acc[RS_TG];
#pragma unroll
    for (int tt = 0; tt < RS_TG; tt++) acc[tt] = 0.0f;
    const int nI = p.H >> 8;
#pragma unroll 4
    for (int i = 0; i < nI; i++) {
        const float4 wa = __ldg(reinterpret_cast<const float4*>(wrow + 256 * i));
        const float4 wb = __ldg(reinterpret_cast<const float4*>(wrow + 256 * i + 4));
        const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
        for (int tt = 0; tt < RS_TG; tt++) {
            const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xrow[tt] + 256 * i));
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const float xj = (j & 1) ? bf16_hi(xw[j >> 1]) : bf16_lo(xw[j >> 1]);
                acc[tt] = __fmaf_rn(xj, wv[j], acc[tt]);
            }
        }
    }
#pragma unroll
    for (int tt = 0; tt < RS_TG; tt++)
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) acc[tt] = __fadd_rn(acc[tt], __shfl_xor_sync(0xffffffffu, acc[tt], off));
    if (lane < RS_TG && t0 + lane < p.T) {
        float val = acc[0];
#pragma unroll
        for (int tt = 1; tt < RS_TG; tt++)
            if (lane == tt) val = acc[tt];
        if (p.bias) val = __fadd_rn(val, p.bias[e]);
        p.logits[static_cast<size_t>(t0 + lane) * p.E + e] = val;
    }
}

// top-k of one token by one warp: k rounds of a warp argmax, larger logit
// first, equal logits -> lower expert id; lane l owns experts l + 32 m, with
// logit lv[m], taking part only where bit m of `allowed` is set; then the
// softmax or sigmoid weights of the k selected logits.
__device__ __forceinline__ void router_topk_select(const RouterParams& p, const float* lv, uint32_t allowed, int t,
                                                   int lane) {
    uint32_t taken = 0;
    float sel_v[8];
    int sel_e[8];
#pragma unroll
    for (int j = 0; j < 8; j++) {
        if (j >= p.k) break;
        float bv = 0.0f;
        int be = -1;
#pragma unroll
        for (int m = 0; m < 8; m++) {
            const int e = 32 * m + lane;
            if (e >= p.E || !((allowed >> m) & 1u) || ((taken >> m) & 1u)) continue;
            if (be < 0 || lv[m] > bv) { bv = lv[m]; be = e; }   // e ascending: ties keep the lower id
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (oe >= 0 && (be < 0 || ov > bv || (ov == bv && oe < be))) { bv = ov; be = oe; }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        sel_v[j] = bv;
        sel_e[j] = be;
    }
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
            p.ids[static_cast<size_t>(t) * p.k + j] = sel_e[j];
            p.w[static_cast<size_t>(t) * p.k + j] = z[j] / sum;
        }
    }
}

// top-k of one token over all its E logits `l` (global or shared memory)
__device__ __forceinline__ void router_topk_token(const RouterParams& p, const float* l, int t, int lane) {
    float lv[8];
    uint32_t allowed = 0;
#pragma unroll
    for (int m = 0; m < 8; m++) {
        const bool in = 32 * m + lane < p.E;
        lv[m] = in ? l[32 * m + lane] : 0.0f;
        allowed |= (in ? 1u : 0u) << m;
    }
    router_topk_select(p, lv, allowed, t, lane);
}

// top-k of one token among its candidate experts (bit m of `cand`: expert
// 32 m + lane), whose canonical logits are in cv
__device__ __forceinline__ void router_topk_candidates(const RouterParams& p, const float* cv, uint32_t cand, int t,
                                                       int lane) {
    router_topk_select(p, cv, cand, t, lane);
}

__global__ void __launch_bounds__(256) router_topk_kernel(RouterParams p) {
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_TOPK);
    const int lane = threadIdx.x & 31;
    for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < p.T; t += gridDim.x * 8)
        router_topk_token(p, p.logits + static_cast<size_t>(t) * p.E, t, lane);
}

// Small batches with at most 32 experts: logits and top-k in one launch.  One
// CTA per group of RS_TG tokens, warp e computes expert e's logits exactly as
// router_logits_small_kernel does, they meet in shared memory, and warp tt
// then selects token tt's experts with router_topk_token.
constexpr int RF_MAX_E = 32;
__global__ void __launch_bounds__(RF_MAX_E * 32) router_small_fused_kernel(RouterParams p) {
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_ROUTER_FUSED);
    __shared__ float s_l[RS_TG][RF_MAX_E];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = warp;
    const int t0 = blockIdx.x * RS_TG;
    if (e < p.E) {
        const float* wrow = p.wr + static_cast<size_t>(e) * p.H + 8 * lane;
        const __nv_bfloat16* xrow[RS_TG];
#pragma unroll
        for (int tt = 0; tt < RS_TG; tt++)
            xrow[tt] = p.x + static_cast<size_t>(t0 + tt < p.T ? t0 + tt : t0) * p.H + 8 * lane;
        float acc[RS_TG];
#pragma unroll
        for (int tt = 0; tt < RS_TG; tt++) acc[tt] = 0.0f;
        const int nI = p.H >> 8;
#pragma unroll 4
        for (int i = 0; i < nI; i++) {
            const float4 wa = __ldg(reinterpret_cast<const float4*>(wrow + 256 * i));
            const float4 wb = __ldg(reinterpret_cast<const float4*>(wrow + 256 * i + 4));
            const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int tt = 0; tt < RS_TG; tt++) {
                const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xrow[tt] + 256 * i));
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const float xj = (j & 1) ? bf16_hi(xw[j >> 1]) : bf16_lo(xw[j >> 1]);
                    acc[tt] = __fmaf_rn(xj, wv[j], acc[tt]);
                }
            }
        }
#pragma unroll
        for (int tt = 0; tt < RS_TG; tt++)
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) acc[tt] = __fadd_rn(acc[tt], __shfl_xor_sync(0xffffffffu, acc[tt], off));
        if (lane < RS_TG) {
            float val = acc[0];
#pragma unroll
            for (int tt = 1; tt < RS_TG; tt++)
                if (lane == tt) val = acc[tt];
            if (p.bias) val = __fadd_rn(val, p.bias[e]);
            s_l[lane][e] = val;
            if (t0 + lane < p.T) p.logits[static_cast<size_t>(t0 + lane) * p.E + e] = val;
        }
    }
    __syncthreads();
    if (warp < RS_TG && t0 + warp < p.T) router_topk_token(p, s_l[warp], t0 + warp, lane);
}

}  // namespace moe
