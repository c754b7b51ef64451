// router.cuh -- router logits + top-k + routing weights.
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
// A warp computes an 8-token x 8-expert micro-tile so each 16-byte load of X
// feeds 64 fused multiply-adds.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int ROUTER_WARPS = 8;

struct RouterParams {
    const __nv_bfloat16* x;
    const float* wr;
    const float* bias;   // nullable
    int32_t* ids;
    float* w;
    int T, H, E, k, score;
    int token_groups;    // 8-token groups per CTA (more when E is small, so every warp has work)
};

__device__ __forceinline__ void router_load_x(const RouterParams& p, int t0, int h0, uint4* xv) {
#pragma unroll
    for (int tt = 0; tt < 8; tt++) {
        const int t = t0 + tt;
        xv[tt] = (t < p.T) ? __ldg(reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(t) * p.H + h0))
                           : make_uint4(0, 0, 0, 0);
    }
}

__global__ void __launch_bounds__(ROUTER_WARPS * 32) router_topk_kernel(RouterParams p) {
    extern __shared__ float lg[];   // [8 * token_groups][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tokens_per_cta = 8 * p.token_groups;
    const int cta_t0 = blockIdx.x * tokens_per_cta;
    const int nI = p.H >> 8;
    const int ngroups = (p.E + 7) >> 3;

    // work item = (8-token group, 8-expert group): an 8 x 8 micro-tile per warp
    for (int item = warp; item < p.token_groups * ngroups; item += ROUTER_WARPS) {
        const int tg = item / ngroups, grp = item % ngroups;
        const int t0 = cta_t0 + 8 * tg;
        float acc[8][8];
#pragma unroll
        for (int a = 0; a < 8; a++)
#pragma unroll
            for (int b = 0; b < 8; b++) acc[a][b] = 0.0f;

        uint4 xn[8];
        router_load_x(p, t0, 8 * lane, xn);
        for (int i = 0; i < nI; i++) {
            const int h0 = 256 * i + 8 * lane;
            uint4 xv[8];
#pragma unroll
            for (int tt = 0; tt < 8; tt++) xv[tt] = xn[tt];
            if (i + 1 < nI) router_load_x(p, t0, h0 + 256, xn);   // next chunk in flight
#pragma unroll
            for (int ee = 0; ee < 8; ee++) {
                const int e = 8 * grp + ee;
                if (e >= p.E) break;
                const float4* wp = reinterpret_cast<const float4*>(p.wr + static_cast<size_t>(e) * p.H + h0);
                const float4 wa = __ldg(wp), wb = __ldg(wp + 1);
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
        }
#pragma unroll
        for (int tt = 0; tt < 8; tt++)
#pragma unroll
            for (int ee = 0; ee < 8; ee++)
#pragma unroll
                for (int off = 1; off < 32; off <<= 1)
                    acc[tt][ee] = __fadd_rn(acc[tt][ee], __shfl_xor_sync(0xffffffffu, acc[tt][ee], off));
        if (lane == 0) {
#pragma unroll
            for (int tt = 0; tt < 8; tt++)
#pragma unroll
                for (int ee = 0; ee < 8; ee++) {
                    const int e = 8 * grp + ee;
                    if (e < p.E) {
                        float v = acc[tt][ee];
                        if (p.bias) v = __fadd_rn(v, p.bias[e]);
                        lg[(8 * tg + tt) * p.E + e] = v;
                    }
                }
        }
    }
    __syncthreads();

    // top-k per token: k rounds of a warp argmax, larger logit first, equal
    // logits -> lower expert id.  Lane l owns experts l + 32 m.
    for (int tl = warp; tl < tokens_per_cta; tl += ROUTER_WARPS) {
        const int t = cta_t0 + tl;
        if (t >= p.T) break;
        const float* l = lg + tl * p.E;
        uint32_t taken = 0;
        float sel_v[8];
        int sel_e[8];
#pragma unroll
        for (int j = 0; j < 8; j++) {
            if (j >= p.k) break;
            float bv = 0.0f;
            int be = -1;
            for (int m = 0; 32 * m + lane < p.E; m++) {
                const int e = 32 * m + lane;
                if ((taken >> m) & 1u) continue;
                const float v = l[e];
                if (be < 0 || v > bv) { bv = v; be = e; }   // e ascending: equal v keeps the lower id
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
