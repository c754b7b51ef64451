// gemm_fp4.cuh -- persistent grouped NVFP4 GEMM on the 5th-gen tensor cores
// (tcgen05.mma kind::mxf4nvf4, E4M3 scale factor per 16 elements of K applied
// by the hardware) with the two epilogues of the MoE expert MLP.
//
// LightMoE README ("Standalone GEMM", "MoE inference"): NVFP4 operands are
// packed E2M1 values with blocked E4M3 scale factors and one fp32 per-tensor
// scale; one layer call does gate/up, the gated activation, NVFP4
// requantisation of the hidden, the down projection and the routing weight.
// Pure-Triton fused MoE article: gate and up share one input tile.
//
// Tiles of 128 rows (widths below), K stage 256 values = 128 bytes per row.
// The packed gate/up weights hold blocks of 64 gate + 64 up rows, one 64-wide
// hidden block each.  Per stage the producer brings, on one mbarrier: A and B tiles by
// TMA (128-byte swizzle) and the 2 KB of A scale factors and 2 KB per 128 rows
// of B scale factors (4 chunks of 512 B, one per MMA of K = 64) by plain bulk
// copies.  The MMA thread copies the chunks into a TMEM ring (tcgen05.cp, 32
// rows x 16 B repeated over the 4 lane quadrants), then issues the 4
// block-scaled MMAs, which read them in issue order.
//  - Gated gate/up and down: 256-column tiles (gate/up: two consecutive 64
//    gate + 64 up blocks of the packed weights, 128 hidden columns), so each
//    128 x 256 x 256 step needs 54 KB of operands and scales instead of
//    2 x 36 KB, and A is read half as often.  One 256-column accumulator,
//    released as soon as the epilogue holds it in registers; 4 stages (down:
//    3, beside the staging of its fp32 row stores).
//  - ReLU^2 gate/up: 128-column tiles, two 128-column accumulators at
//    [0, 256), 5 stages.
// The scale-factor ring starts at TMEM column 256.
//
// Rows are in the 128-padded expert-major layout (m-tile i = rows 128 i ..),
// so each tile's scale factors are whole chunks.  The epilogue maps a padded
// row back to its assignment slot (offsets) for the outputs indexed by slot.
#pragma once
#include <type_traits>

#include "common.cuh"
#include "gemm.cuh"

namespace moe {

constexpr int F4_A_BYTES = 128 * 128;
constexpr int F4_SF_BYTES = 2048;                 // 4 chunks of 512 B per 128 rows
constexpr int F4_SF_TMEM = 256;                   // first column of the scale-factor ring

// Shared memory and TMEM of one instantiation: BN-column tiles, NBUF
// accumulators, STAGES smem stages, and the float4 row staging of the fp32
// down stores (STG).
template <int BN_, int NBUF_, int STAGES_, bool STG>
struct Fp4Smem {
    static constexpr int BN = BN_;
    static constexpr int NBUF = NBUF_;
    static constexpr int STAGES = STAGES_;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int SFB_BYTES = (BN / 128) * F4_SF_BYTES;
    static constexpr int STAGE_BYTES = F4_A_BYTES + B_BYTES + F4_SF_BYTES + SFB_BYTES;
    static constexpr int SF_COLS = BN == 256 ? 64 : 32;   // TMEM columns per stage: A 16, B 16 per 128 rows
    static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * NBUF + 1;
    static constexpr int TMEM_SLOT_OFF = BAR_OFF + 8 * NUM_BARS;
    static constexpr int TMAP_OFF = TMEM_SLOT_OFF + 16;
    static constexpr int STG_OFF = (TMAP_OFF + TMAP_BYTES + 15) / 16 * 16;
    static constexpr int TOTAL = STG_OFF + (STG ? 8 * STG_WARP_FLOATS * 4 : 0) + 1024;
    static_assert(TOTAL <= 232448, "shared memory of the NVFP4 GEMM exceeds 227 KB");
    static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 128-byte swizzle atoms aligned");
    static_assert(NBUF * BN <= F4_SF_TMEM && F4_SF_TMEM + SF_COLS * STAGES <= 512, "TMEM columns");
};
// Gated gate/up: 256-column tiles (two 64 gate + 64 up blocks), one
// accumulator released as soon as the epilogue holds it in registers, 4
// stages.  Down: 256-column tiles, one accumulator, 3 stages and the row
// staging.  ReLU^2 gate/up: 128-column tiles, two accumulators, 5 stages.
template <int KIND, int ACT>
using Fp4Layout = std::conditional_t<KIND == KIND_DOWN, Fp4Smem<256, 1, 3, true>,
                                     std::conditional_t<ACT == 5, Fp4Smem<128, 2, 5, false>, Fp4Smem<256, 1, 4, false>>>;

struct Fp4Params {
    const int32_t* tiles;
    const int32_t* num_tiles;
    const int32_t* tile_ptr;
    const int32_t* offsets;
    int E;
    int n_blocks;             // N / tile width
    int num_kb;               // K / 256
    int sf_cols;              // K / 16
    int b_rows;               // rows of B per expert (2I for gate/up, H for down)
    const uint8_t* sfa;       // activation scale factors, chunked by padded row tile
    const uint8_t* sfb;       // weight scale factors, chunked per expert
    const int32_t* x_amax;    // gate/up: amax bits of X (global scale = amax / 2688)
    const float* w_global;    // gate/up: [E][2] (gate, up); down: [E]
    float h_global;           // static hidden scale
    int act;                  // gate/up: gated activation (the kernel is instantiated for it)
    float act_alpha, act_limit;
    uint8_t* hq;              // gate/up out: hidden codes [rows][I/2], scale factors hsf
    uint8_t* hsf;
    int I;
    uint16_t* o;              // down out: [A][H] fp16 rows in slot order, block exponents in oe
    int8_t* oe;               //   [A][H / 32]
    int H;
    const int32_t* perm;
    const float* route_w;
    int32_t* status;
    long long spin_limit;
};

template <int KIND, int ACT>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    grouped_gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const Fp4Params p) {
    using L = Fp4Layout<KIND, ACT>;
    constexpr bool WIDE = L::BN == 256;
    constexpr int F4_BN = L::BN, F4_NBUF = L::NBUF, F4_STAGES = L::STAGES;
    constexpr int F4_B_BYTES = L::B_BYTES, F4_STAGE_BYTES = L::STAGE_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* full = bars;
    uint64_t* empty = bars + F4_STAGES;
    uint64_t* tfull = bars + 2 * F4_STAGES;
    uint64_t* tempty = bars + 2 * F4_STAGES + F4_NBUF;
    uint64_t* drain = bars + 2 * F4_STAGES + 2 * F4_NBUF;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::TMEM_SLOT_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < F4_STAGES; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < F4_NBUF; b++) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 8);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();
    pdl_trigger();
    KTRACE(p.o != nullptr ? TR_FP4 + 1 : TR_FP4);
    int32_t* s_tptr = reinterpret_cast<int32_t*>(smem + L::TMAP_OFF);
    const int32_t* s_off = s_tptr + TMAP_STRIDE;
    stage_tile_map(s_tptr, p.tile_ptr, p.offsets, p.E);
    __syncthreads();
    const int ntm = *p.num_tiles;
    const int total = ntm * p.n_blocks;
    const long long limit = p.spin_limit;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                int e, mi, nb;
                decode_tile(t, s_tptr, p.E, p.n_blocks, e, mi, nb);
                const int brow = e * p.b_rows + nb * F4_BN;
                const uint64_t pol = l2_policy(s_tptr[e + 1] - s_tptr[e] == 1);   // weight tile read once?
                const uint8_t* sfa = p.sfa + static_cast<size_t>(mi) * p.sf_cols * 128;
                // scale factors of the tile's 128-row blocks of B (BN / 128 of them)
                const uint8_t* sfb = p.sfb + static_cast<size_t>(e) * p.b_rows * p.sf_cols +
                                     static_cast<size_t>(nb) * (F4_BN / 128) * p.sf_cols * 128;
                for (int kb = 0; kb < p.num_kb; kb++, it++) {
                    const int s = it % F4_STAGES;
                    if (!mbar_wait(&empty[s], ((it / F4_STAGES) & 1) ^ 1, limit)) {
                        report(p.status, ST_TIMEOUT, WHERE_GEMM_PRODUCER);
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + s * F4_STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[s], F4_STAGE_BYTES);
                    tma_load_2d(st, &tmA, &full[s], kb * 128, mi * 128);
                    tma_load_2d_hint(st + F4_A_BYTES, &tmB, &full[s], kb * 128, brow, pol);
                    bulk_load(st + F4_A_BYTES + F4_B_BYTES, sfa + kb * F4_SF_BYTES, F4_SF_BYTES, &full[s]);
#pragma unroll
                    for (int hb = 0; hb < F4_BN / 128; hb++)
                        bulk_load_hint(st + F4_A_BYTES + F4_B_BYTES + F4_SF_BYTES * (1 + hb),
                                       sfb + static_cast<size_t>(hb) * p.sf_cols * 128 + kb * F4_SF_BYTES, F4_SF_BYTES,
                                       &full[s], pol);
                }
            }
            const uint32_t first = it > F4_STAGES ? it - F4_STAGES : 0;
            for (uint32_t j = first; j < it; j++) mbar_wait(&full[j % F4_STAGES], (j / F4_STAGES) & 1, DRAIN_LIMIT);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_nvf4(128, F4_BN);
            uint32_t it = 0, u = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const uint32_t acc = u % F4_NBUF;
                if (!mbar_wait(&tempty[acc], ((u / F4_NBUF) & 1) ^ 1, limit)) { ok = false; break; }
                tc_fence_after();
                for (int kb = 0; kb < p.num_kb; kb++, it++) {
                    const int s = it % F4_STAGES;
                    if (!mbar_wait(&full[s], (it / F4_STAGES) & 1, limit)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * F4_STAGE_BYTES);
                    const uint32_t b_addr = a_addr + F4_A_BYTES;
                    const uint32_t sfa_addr = b_addr + F4_B_BYTES;
                    const uint32_t sfb_addr = sfa_addr + F4_SF_BYTES;
                    // MMA j (K = 64) reads A-scale chunk j (4 columns) and, per
                    // 128-row block hb of B, B-scale chunk j at 4 (BN / 128) j + 4 hb
                    const uint32_t sf_col = tmem_base + F4_SF_TMEM + L::SF_COLS * s;
                    constexpr int NHB = F4_BN / 128;
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        tmem_cp_32x128b_x4(sf_col + 4 * j, sdesc_sf_chunk(sfa_addr + 512 * j));
#pragma unroll
                        for (int hb = 0; hb < NHB; hb++)
                            tmem_cp_32x128b_x4(sf_col + 16 + 4 * NHB * j + 4 * hb,
                                               sdesc_sf_chunk(sfb_addr + F4_SF_BYTES * hb + 512 * j));
                    }
                    const uint32_t d = tmem_base + acc * F4_BN;
#pragma unroll
                    for (int j = 0; j < 4; j++)
                        mma_nvf4(d, sdesc_sw128(a_addr + 32 * j), sdesc_sw128(b_addr + 32 * j), idesc, sf_col + 4 * j,
                                 sf_col + 16 + 4 * NHB * j, (kb > 0 || j > 0));
                    mma_commit(&empty[s]);
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
                u++;
            }
            if (!ok) report(p.status, ST_TIMEOUT, WHERE_GEMM_MMA);
            mma_commit(drain);
            mbar_wait(drain, 0, DRAIN_LIMIT);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int g = (warp - 2) >> 2;           // column group: half of the tile's columns
        const int r = 32 * q + lane;
        const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
        uint32_t u = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            int e, mi, nb;
            decode_tile(t, s_tptr, p.E, p.n_blocks, e, mi, nb);
            const long long prow = static_cast<long long>(mi) * 128 + r;
            const int local = static_cast<int>(prow - static_cast<long long>(s_tptr[e]) * 128);
            const bool valid = local < s_off[e + 1] - s_off[e];
            // loaded while the tile's MMAs run
            const int slot = s_off[e] + local;
            const float gx = __fdiv_rn(__int_as_float(*p.x_amax), 2688.0f);
            const float wg0 = __ldg(p.w_global + (KIND == KIND_GATE_UP ? 2 * e : e));
            const float wg1 = KIND == KIND_GATE_UP ? __ldg(p.w_global + 2 * e + 1) : 0.0f;
            const float rw = (KIND == KIND_DOWN && valid) ? p.route_w[p.perm[slot]] : 0.0f;
            const uint32_t acc = u % F4_NBUF;
            if (!warp_wait(&tfull[acc], (u / F4_NBUF) & 1, limit)) { ok = false; break; }
            tc_fence_after();
            if (!__any_sync(0xffffffffu, valid)) {
                // none of this warp's rows is stored: release the accumulator only
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
                u++;
                continue;
            }
            if (KIND == KIND_GATE_UP) {
                // TMEM columns of a 128-row block of B: gate [0, 64), up [64, 128).
                // Narrow: one block, this warp's 32 columns at 32 g.  Wide: blocks
                // g of the tile (columns 128 g ..), both 32-column runs.
                constexpr int NL = WIDE ? 2 : 1;
                float gv[NL][32], uv[NL][32];
#pragma unroll
                for (int ld = 0; ld < NL; ld++) {
                    const int c0 = WIDE ? 128 * g + 32 * ld : 32 * g;
                    tmem_ld32x2(lane_addr + acc * F4_BN + c0, lane_addr + acc * F4_BN + c0 + 64, gv[ld], uv[ld]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
                u++;
                const float sg = gx * wg0, su = gx * wg1;
                // gated: run l = act(g, u) of load l, at hidden 64 nb + 32 g (narrow)
                // or 128 nb + 64 g + 32 l (wide); ReLU^2 (no gate, 128 up rows per
                // tile): relu(v)^2 of both 32-column halves, at hidden 128 nb + 32 g
                // and 128 nb + 64 + 32 g
                constexpr int NR = (ACT == 5 || WIDE) ? 2 : 1;
                float hv[32 * NR];
#pragma unroll
                for (int c = 0; c < 32; c++) {
                    if constexpr (ACT == 5) {
                        hv[c] = relu_sq(gv[0][c] * sg);
                        hv[32 + c] = relu_sq(uv[0][c] * su);
                    } else {
#pragma unroll
                        for (int ld = 0; ld < NL; ld++)
                            hv[32 * ld + c] = glu<ACT>(gv[ld][c] * sg, uv[ld][c] * su, p.act_alpha, p.act_limit);
                    }
                }
                if (valid) {
#pragma unroll
                    for (int run = 0; run < NR; run++) {
                        // first hidden column of this run
                        const int col0 = ACT == 5 ? nb * 128 + 64 * run + 32 * g
                                                  : (WIDE ? nb * 128 + 64 * g + 32 * run : nb * 64 + 32 * g);
                        uint32_t w[4];
#pragma unroll
                        for (int b = 0; b < 2; b++) {           // two 16-blocks
                            float amax = 0.0f;
#pragma unroll
                            for (int c = 0; c < 16; c++) amax = fmaxf(amax, fabsf(hv[32 * run + 16 * b + c]));
                            const uint8_t sb = f_to_e4m3(__fdiv_rn(__fdiv_rn(amax, 6.0f), p.h_global));
                            const float d = __fmul_rn(e4m3_to_f(sb), p.h_global);
#pragma unroll
                            for (int c = 0; c < 16; c += 8) {
                                uint32_t pk = 0;
                                if (d != 0.0f) {
#pragma unroll
                                    for (int i = 0; i < 4; i++)
                                        pk |= static_cast<uint32_t>(f2_to_e2m1x2(
                                                  __fdiv_rn(hv[32 * run + 16 * b + c + 2 * i], d),
                                                  __fdiv_rn(hv[32 * run + 16 * b + c + 2 * i + 1], d)))
                                              << (8 * i);
                                }
                                w[2 * b + c / 8] = pk;
                            }
                            p.hsf[sf_offset(prow, col0 / 16 + b, p.I / 16)] = sb;
                        }
                        *reinterpret_cast<uint4*>(p.hq + prow * (p.I / 2) + col0 / 2) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            } else {
                // this warp's NC columns of the tile: 64 (narrow) or 128 (wide) at NC g
                constexpr int NC = F4_BN / 2;
                float v[NC];
#pragma unroll
                for (int ch = 0; ch < NC / 64; ch++)
                    tmem_ld32x2(lane_addr + acc * F4_BN + NC * g + 64 * ch, lane_addr + acc * F4_BN + NC * g + 64 * ch + 32,
                                v + 64 * ch, v + 64 * ch + 32);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
                u++;
                store_rows16<NC, false>(
                    v, reinterpret_cast<uint32_t*>(smem + L::STG_OFF) + (warp - 2) * STG_WARP_FLOATS,
                    valid ? p.o + static_cast<size_t>(slot) * p.H + nb * F4_BN + NC * g : nullptr,
                    p.oe + static_cast<size_t>(slot) * (p.H / 32) + (nb * F4_BN + NC * g) / 32, nullptr,
                    p.h_global * wg0 * rw, lane);
            }
        }
        if (!ok) report(p.status, ST_TIMEOUT, WHERE_GEMM_EPILOGUE);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace moe
