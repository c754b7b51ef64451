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
// Two kernels:
//  router_logits_kernel  a 2-D grid of CTA tiles (TOK tokens x EXP experts; 32 x 16,
//                        or 64 x 8 when E <= 8).
//                        The 256-wide H chunks of X and Wr go through shared
//                        memory with double-buffered cp.async; each of the 8
//                        warps owns one 8-token x 8-expert micro-tile, so one
//                        16-byte X read from shared memory feeds 64 fma.
//  router_topk_kernel    one warp per token: k rounds of a warp argmax over
//                        the token's logits, then softmax or sigmoid weights.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int RT_WARPS = 8;   // (TOK / 8) x (EXP / 8) micro-tiles of 8 x 8

template <int TOK, int EXP>
struct RouterTile {
    static_assert((TOK / 8) * (EXP / 8) == RT_WARPS, "one micro-tile per warp");
    static constexpr int X_BYTES = TOK * 256 * 2;    // 256 bf16 of H per token
    static constexpr int W_BYTES = EXP * 256 * 4;    // 256 fp32 of H per expert
    static constexpr int STAGE = X_BYTES + W_BYTES;
    static constexpr int SMEM = 2 * STAGE;           // 64 KB (32 x 16) or 80 KB (64 x 8)
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

// Load H-chunk i of the tile's X rows and Wr rows into stage buffer `st`.
// Rows past T or E read nothing and are zero-filled.
template <int TOK, int EXP>
__device__ __forceinline__ void router_load_chunk(const RouterParams& p, uint8_t* st, int t0, int e0, int i) {
    // X: TOK rows x 512 B = TOK * 32 pieces of 16 B
    for (int q = threadIdx.x; q < TOK * 32; q += blockDim.x) {
        const int r = q >> 5, c = q & 31;
        const int t = t0 + r;
        const bool ok = t < p.T;
        const __nv_bfloat16* src = p.x + static_cast<size_t>(ok ? t : 0) * p.H + 256 * i + 8 * c;
        cp_async16(st + r * 512 + c * 16, src, ok);
    }
    // Wr: EXP rows x 1024 B = EXP * 64 pieces of 16 B
    for (int q = threadIdx.x; q < EXP * 64; q += blockDim.x) {
        const int r = q >> 6, c = q & 63;
        const int e = e0 + r;
        const bool ok = e < p.E;
        const float* src = p.wr + static_cast<size_t>(ok ? e : 0) * p.H + 256 * i + 4 * c;
        cp_async16(st + RouterTile<TOK, EXP>::X_BYTES + r * 1024 + c * 16, src, ok);
    }
    cp_async_commit();
}

template <int TOK, int EXP>
__global__ void __launch_bounds__(RT_WARPS * 32) router_logits_kernel(RouterParams p) {
    using RT = RouterTile<TOK, EXP>;
    extern __shared__ __align__(16) uint8_t rsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * TOK, e0 = blockIdx.y * EXP;
    const int tg = warp % (TOK / 8), eg = warp / (TOK / 8);   // this warp's micro-tile
    const int nI = p.H >> 8;

    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; a++)
#pragma unroll
        for (int b = 0; b < 8; b++) acc[a][b] = 0.0f;

    router_load_chunk<TOK, EXP>(p, rsm, t0, e0, 0);
    for (int i = 0; i < nI; i++) {
        uint8_t* st = rsm + (i & 1) * RT::STAGE;
        if (i + 1 < nI) {
            router_load_chunk<TOK, EXP>(p, rsm + ((i + 1) & 1) * RT::STAGE, t0, e0, i + 1);
            cp_async_wait1();
        } else {
            cp_async_wait0();
        }
        __syncthreads();
        const uint8_t* xs = st + (8 * tg) * 512 + lane * 16;
        const uint8_t* ws = st + RT::X_BYTES + (8 * eg) * 1024 + lane * 32;
        uint4 xv[8];
#pragma unroll
        for (int tt = 0; tt < 8; tt++) xv[tt] = *reinterpret_cast<const uint4*>(xs + tt * 512);
#pragma unroll
        for (int ee = 0; ee < 8; ee++) {
            const float4 wa = *reinterpret_cast<const float4*>(ws + ee * 1024);
            const float4 wb = *reinterpret_cast<const float4*>(ws + ee * 1024 + 16);
            const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int tt = 0; tt < 8; tt++) {
                const uint32_t u[4] = {xv[tt].x, xv[tt].y, xv[tt].z, xv[tt].w};
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    acc[tt][ee] = __fmaf_rn(bf16_lo(u[q]), wv[2 * q], acc[tt][ee]);
                    acc[tt][ee] = __fmaf_rn(bf16_hi(u[q]), wv[2 * q + 1], acc[tt][ee]);
                }
            }
        }
        __syncthreads();   // the stage is refilled two chunks later
    }
#pragma unroll
    for (int tt = 0; tt < 8; tt++)
#pragma unroll
        for (int ee = 0; ee < 8; ee++)
#pragma unroll
            for (int off = 1; off < 32; off <<= 1)
                acc[tt][ee] = __fadd_rn(acc[tt][ee], __shfl_xor_sync(0xffffffffu, acc[tt][ee], off));
    // lane (tt * 8 + ee) % 32 writes one logit; each lane holds every sum
#pragma unroll
    for (int tt = 0; tt < 8; tt++)
#pragma unroll
        for (int ee = 0; ee < 8; ee++) {
            if (((tt * 8 + ee) & 31) != lane) continue;
            const int t = t0 + 8 * tg + tt, e = e0 + 8 * eg + ee;
            if (t < p.T && e < p.E) {
                float v = acc[tt][ee];
                if (p.bias) v = __fadd_rn(v, p.bias[e]);
                p.logits[static_cast<size_t>(t) * p.E + e] = v;
            }
        }
}

// top-k per token: k rounds of a warp argmax, larger logit first, equal
// logits -> lower expert id.  Lane l owns experts l + 32 m.
__global__ void __launch_bounds__(256) router_topk_kernel(RouterParams p) {
    const int lane = threadIdx.x & 31;
    for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < p.T; t += gridDim.x * 8) {
        const float* l = p.logits + static_cast<size_t>(t) * p.E;
        float lv[8];
#pragma unroll
        for (int m = 0; m < 8; m++) lv[m] = (32 * m + lane < p.E) ? l[32 * m + lane] : 0.0f;
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
                if (e >= p.E || ((taken >> m) & 1u)) continue;
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
}

}  // namespace moe
