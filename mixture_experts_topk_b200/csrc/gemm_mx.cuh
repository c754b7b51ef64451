// gemm_mx.cuh -- persistent grouped down GEMM on MX-scaled FP8 (tcgen05.mma
// kind::mxf8f6f4 with block32 UE8M0 scales applied by the tensor cores).
//
// LightMoE README ("MoE inference"): the requantised hidden feeds the down
// projection and the routing weight is applied; Alpha-MoE article: FP8 W8A8.
// The FP8_ROW hidden carries a power-of-two scale per 32 columns, so the whole
// K reduction stays in TMEM (no per-K-block promotion).  The weights carry one
// fp32 scale per output row, applied with the routing weight in the epilogue;
// their MX scale is the constant 1 (UE8M0 127), copied into TMEM once.
//
// Tile 128 padded rows x 256 columns, K stage 128 (one 512-byte scale chunk of
// A per stage: 4 scales of 32 per row), 3 to 5 stages (see the variants
// below).  For small batches the K
// range of each tile may be split S ways (S read from the dispatch's pick,
// work item t = (tile t / S, split t % S)); split s writes its partial rows to copy s
// of the output rows, o + s * A * H.  MMA j of a stage (K = 32)
// uses byte j of the chunk (scale-factor id j).  TMEM: one 256-column
// accumulator, released as soon as the epilogue has it in registers, then the
// A-scale ring and the constant B-scale chunks.
//
// Large batches with deep K run on CTA pairs (2-CTA clusters): one
// tcgen05.mma.cta_group::2 with M = 256 covers two m-tiles of one expert; each
// CTA loads its 128 hidden rows, its scale chunk and 128 of the 256 B rows,
// completing them on rank 0's barrier (the scale chunk by TMA as two 256-byte
// rows); rank 0 copies both CTAs' scale chunks into their TMEM and issues the
// MMAs; commits reach both CTAs.  An expert with an odd m-tile count runs its
// last pair with rank 1's rows unstored (it loads rank 0's rows).
//
// Output rows (fp16 with a power-of-two scale per 32 columns, see
// store_rows16): a warp whose 32 rows are all stored (rows of one expert are
// consecutive slots) writes them as two 32-row x 64-column fp16 boxes through
// a 128-byte-swizzled shared buffer (two per warp, alternating) with TMA
// tensor stores, so the store runs asynchronously beside the next tile's
// accumulator read; a warp with fewer rows stores its rows directly.
#pragma once
#include "common.cuh"
#include "gemm.cuh"

namespace moe {

constexpr int MX_BN = 256;
constexpr int MX_A_BYTES = 128 * 128;
constexpr int MX_SFA_BYTES = 512;
constexpr int MX_BOX_BYTES = 32 * 128;                           // 32 rows x 64 fp16
// TMEM: the accumulators fill columns [0, 256) (one 256-wide or two 128-wide),
// then the A-scale ring and the constant B-scale chunks
constexpr int MX_SFA_TMEM = 256;                                 // 4 columns per stage
constexpr int MX_SFB_TMEM = 256 + 32;                            // 8 columns (two 128-row chunks)
// Deep K (many K stages per tile): 4 stages, rows stored from registers.
// Shallow K, where a tile's stores outlast its MMAs: 3 stages and the box stores.
constexpr int MX_BOX_MAX_KB = 16;
// CTA pairs (deep K, large batches): 33 KB stages, 5 deep.
constexpr int MX_PAIR_STAGES = 5;
// 128-wide tiles: 33 KB stages, 4 deep beside the box stores, 6 without.
constexpr int MX_NARROW_BOX_STAGES = 4;
constexpr int MX_NARROW_STAGES = 6;

// PAIR: a CTA pair (tcgen05 cta_group::2, M = 256) where each CTA loads its 128
// A rows and 128 of the 256 B rows.
template <int STAGES, bool BOXES, bool PAIR = false, int BN = MX_BN>
struct MxSmem {
    static constexpr int NACC = 256 / BN;                             // accumulators in TMEM
    static constexpr int B_BYTES = (PAIR ? BN / 2 : BN) * 128;
    static constexpr int STAGE_BYTES = MX_A_BYTES + B_BYTES + 1024;   // + 512 B A scales, padded to 1 KB
    static constexpr int SFB_OFF = STAGES * STAGE_BYTES;              // 2 constant chunks (1 KB)
    static constexpr int BAR_OFF = SFB_OFF + 1024;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * NACC + 1;
    static constexpr int TMEM_SLOT_OFF = BAR_OFF + 8 * NUM_BARS;
    static constexpr int TMAP_OFF = TMEM_SLOT_OFF + 16;
    // per epilogue warp: two swizzled boxes, or the float4 row staging
    static constexpr int STG_OFF = BOXES ? (TMAP_OFF + TMAP_BYTES + 1023) / 1024 * 1024
                                         : (TMAP_OFF + TMAP_BYTES + 15) / 16 * 16;
    static constexpr int STG_WARP_BYTES = BOXES ? 2 * MX_BOX_BYTES : STG_WARP_FLOATS * 4;
    static constexpr int PPTR_OFF = STG_OFF + 8 * STG_WARP_BYTES;     // pairs: m-pairs per expert
    static constexpr int TOTAL = PPTR_OFF + (PAIR ? TMAP_STRIDE * 4 : 0) + 1024;
    static_assert(TOTAL <= 232448, "shared memory of the down GEMM exceeds 227 KB");
    static_assert(!(PAIR && BOXES), "pairs store rows from registers");
    static_assert(STG_WARP_FLOATS * 4 <= STG_WARP_BYTES, "row staging fits");
    static_assert(4 * STAGES <= 32, "A-scale ring below the B-scale chunks");
};

// Instruction descriptor of kind::mxf8f6f4 block-scaled: A, B E4M3 (0), K-major,
// N >> 3 at [17,23), UE8M0 scales ([23] = 1), M >> 4 at [24,29), A scale id at
// [29,31), B scale id at [4,6), dense K = 32.
__host__ __device__ constexpr uint32_t idesc_mxf8(int M, int N, int sf_id) {
    return (static_cast<uint32_t>(sf_id) << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
           (static_cast<uint32_t>(M >> 4) << 24) | (static_cast<uint32_t>(sf_id) << 29);
}

__device__ __forceinline__ void mma_mxf8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// cta_group::2 forms: one thread of the pair's first CTA issues them for both
// CTAs (each CTA's own shared memory to its own TMEM; its own A rows).
__device__ __forceinline__ void mma_mxf8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}
__device__ __forceinline__ void tmem_cp_32x128b_x4_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

struct MxDownParams {
    const int32_t* tiles;
    const int32_t* num_tiles;
    const int32_t* tile_ptr;
    const int32_t* offsets;
    int E;
    int n_blocks;              // H / 256
    int num_kb;                // I / 128
    int b_rows;                // H
    const uint8_t* sfa;        // hidden MX scales, chunked by padded row tile (I / 32 per row)
    const float* w_scale;      // [E][H] fp32 per output row of W_down
    uint16_t* o;               // [S][A][H] fp16 rows in slot order (block exponents in oe)
    int8_t* oe;                // [S][A][H / 32]
    int H;
    int A;                     // assignments T * k
    const int32_t* split;      // S, the K split chosen by the dispatch's scan
    int s_max;                 // S is clamped to [1, s_max] (s_max * A rows fit in o)
    const int32_t* gu_done;    // chained after the gate/up GEMM: per-expert finished parts, else null
    int gu_per_mtile;          //   parts per m-tile of an expert (gate/up n-blocks x epilogue warps)
    const int32_t* perm;
    const float* route_w;
    int32_t* status;
    long long spin_limit;
};

// BN: 256-wide tiles with one accumulator, or 128-wide tiles with two, so that
// a tile's MMAs run while the epilogue drains the previous tile's accumulator
template <int STAGES, bool BOXES, bool PAIR = false, int BN = MX_BN>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    grouped_gemm_mx_down_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmS,
                                const MxDownParams p) {
    static_assert(BN == 256 || (BN == 128 && !PAIR), "128-wide down tiles run on single CTAs");
    using L = MxSmem<STAGES, BOXES, PAIR, BN>;
    constexpr int NACC = L::NACC;
    constexpr int NC = BN / 2;                       // output columns per epilogue thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;             // [NACC]
    uint64_t* tempty = bars + 2 * STAGES + NACC;     // [NACC]
    uint64_t* drain = bars + 2 * STAGES + 2 * NACC;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::TMEM_SLOT_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // CTA pairs: rank 0 issues the MMAs; its full and tempty barriers take the
    // arrivals of both CTAs
    const uint32_t rank = PAIR ? cluster_rank() : 0u;

    // constant B scale chunks: 1.0 for every row and block
    for (int i = threadIdx.x; i < 1024 / 4; i += blockDim.x)
        reinterpret_cast<uint32_t*>(smem + L::SFB_OFF)[i] = 0x7F7F7F7Fu;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(&full[s], PAIR ? 2 : 1);   // pairs: one expect_tx arrival per CTA
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < NACC; a++) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], PAIR ? 16 : 8);   // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmO);
        if (PAIR) tma_prefetch_desc(&tmS);
    }
    if (warp == 1) {
        if constexpr (PAIR) tmem_alloc_pair(tmem_slot, 512);
        else tmem_alloc(tmem_slot, 512);
    }
    // the generic-proxy writes of the constant chunks become visible to tcgen05.cp
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();   // both CTAs' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // Chained after the gate/up GEMM, this kernel does not wait for that whole
    // kernel: the schedule it reads was complete before the gate/up GEMM let it
    // launch, and each expert's hidden is waited for below.  Otherwise wait for
    // the preceding kernel.
    if (p.gu_done == nullptr) pdl_wait();
    pdl_trigger();
    KTRACE(TR_MX_DOWN);
    int32_t* s_tptr = reinterpret_cast<int32_t*>(smem + L::TMAP_OFF);
    const int32_t* s_off = s_tptr + TMAP_STRIDE;
    stage_tile_map(s_tptr, p.tile_ptr, p.offsets, p.E);
    int32_t* s_pptr = reinterpret_cast<int32_t*>(smem + L::PPTR_OFF);
    if constexpr (PAIR) {
        __syncthreads();
        if (threadIdx.x == 0) {
            // m-pairs per expert, prefix over experts (E <= 256 steps, once per CTA)
            int acc_p = 0;
            for (int i = 0; i < p.E; i++) {
                s_pptr[i] = acc_p;
                acc_p += (s_tptr[i + 1] - s_tptr[i] + 1) >> 1;
            }
            s_pptr[p.E] = acc_p;
        }
    }
    __syncthreads();
    const int ntm = *p.num_tiles;
    const int units = (PAIR ? s_pptr[p.E] : ntm) * p.n_blocks;
    const int S = min(max(*p.split, 1), p.s_max);
    const int total = units * S;
    const long long limit = p.spin_limit;
    // CTA pairs walk the work items by cluster, single CTAs by block
    const int t_first = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int t_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    // this CTA's m-tile of unit v: (expert, global m-tile, n-block, has rows);
    // a pair's m-pair j holds the expert's m-tiles 2j (rank 0) and 2j + 1
    auto unit_tile = [&](int v, int& e, int& mi, int& nb, bool& has_rows) {
        if constexpr (PAIR) {
            int mp;
            decode_pair(v, s_pptr, p.E, p.n_blocks, e, mp, nb);
            const int local = 2 * mp + static_cast<int>(rank);
            has_rows = local < s_tptr[e + 1] - s_tptr[e];
            mi = s_tptr[e] + local;
        } else {
            decode_tile(v, s_tptr, p.E, p.n_blocks, e, mi, nb);
            has_rows = true;
        }
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            int ready_e = -1;
            for (int t = t_first; t < total && ok; t += t_step) {
                const int sp = t % S;   // unit-major: all splits of a unit together, experts in order
                int e, mi, nb;
                bool has_rows;
                unit_tile(t / S, e, mi, nb, has_rows);
                // a pair's rank 1 without an m-tile (odd count) loads rank 0's rows and
                // scales, so its reads stay inside the buffers; its rows are not stored
                const int mi_ld = has_rows ? mi : mi - 1;
                const int brow = e * p.b_rows + nb * BN + (PAIR ? static_cast<int>(rank) * (BN / 2) : 0);
                const uint64_t pol = l2_policy(s_tptr[e + 1] - s_tptr[e] == 1);   // weight tile read once?
                const uint8_t* sfa = p.sfa + static_cast<size_t>(mi_ld) * p.num_kb * 512;
                // both CTAs of a pair complete their stage bytes on rank 0's barrier
                auto stage_bar = [&](int s) -> uint32_t {
                    return PAIR ? cluster_addr(&full[s], 0) : smem_u32(&full[s]);
                };
                auto expect = [&](int s) {
                    if constexpr (PAIR) mbar_arrive_expect_tx_cluster(stage_bar(s), MX_A_BYTES + L::B_BYTES + MX_SFA_BYTES);
                    else mbar_arrive_expect_tx(&full[s], MX_A_BYTES + L::B_BYTES + MX_SFA_BYTES);
                };
                auto load_b = [&](uint8_t* st, int s, int k) {
                    if constexpr (PAIR) tma_load_2d_pair(st + MX_A_BYTES, &tmB, stage_bar(s), k * 128, brow, pol);
                    else tma_load_2d_hint(st + MX_A_BYTES, &tmB, &full[s], k * 128, brow, pol);
                };
                auto load_a_sfa = [&](uint8_t* st, int s, int k) {
                    if constexpr (PAIR) {
                        tma_load_2d_pair(st, &tmA, stage_bar(s), k * 128, mi_ld * 128, l2_policy(false));
                        // scale chunk (mi_ld, k) = rows 2 (mi_ld num_kb + k) .. + 1 of 256 bytes
                        tma_load_2d_pair(st + MX_A_BYTES + L::B_BYTES, &tmS, stage_bar(s), 0, 2 * (mi_ld * p.num_kb + k),
                                         l2_policy(false));
                    } else {
                        tma_load_2d(st, &tmA, &full[s], k * 128, mi * 128);
                        bulk_load(st + MX_A_BYTES + L::B_BYTES, sfa + k * 512, MX_SFA_BYTES, &full[s]);
                    }
                };
                const int kb0 = sp * p.num_kb / S, kb1 = (sp + 1) * p.num_kb / S;
                int kb = kb0;
                if (p.gu_done != nullptr && e != ready_e) {
                    // The weight tiles do not depend on the gate/up GEMM: the first
                    // stages of the unit take their B tiles now, and their hidden
                    // rows (A) and scales once all gate/up parts of expert e are
                    // stored, so the weight stream overlaps the wait.
                    const int npre = min(kb1 - kb0, STAGES);
                    int armed = 0;
                    for (; armed < npre; armed++) {
                        const uint32_t itj = it + armed;
                        const int s = itj % STAGES;
                        if (!mbar_wait(&empty[s], ((itj / STAGES) & 1) ^ 1, limit)) { ok = false; break; }
                        expect(s);
                        load_b(smem + s * L::STAGE_BYTES, s, kb0 + armed);
                    }
                    if (ok) {
                        const int target = (s_tptr[e + 1] - s_tptr[e]) * p.gu_per_mtile;
                        const long long t0 = clock64();
                        // polled with a pause, so that a hundred CTAs waiting on the few
                        // counters of the first experts do not keep those L2 lines busy
                        // while the gate/up epilogues increment them
                        while (ld_acquire(p.gu_done + e) < target) {
                            if (clock64() - t0 > limit) { ok = false; break; }
                            __nanosleep(500);
                        }
                    }
                    fence_proxy_async_global();
                    // the armed stages get their A and scales even after a timeout, so
                    // that no copy into them is left incomplete
                    for (int j = 0; j < armed; j++) {
                        const uint32_t itj = it + j;
                        load_a_sfa(smem + (itj % STAGES) * L::STAGE_BYTES, itj % STAGES, kb0 + j);
                    }
                    it += armed;
                    kb += armed;
                    if (!ok) {
                        report(p.status, ST_TIMEOUT, WHERE_GEMM_PRODUCER);
                        break;
                    }
                    ready_e = e;
                }
                for (; kb < kb1; kb++, it++) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, limit)) {
                        report(p.status, ST_TIMEOUT, WHERE_GEMM_PRODUCER);
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + s * L::STAGE_BYTES;
                    expect(s);
                    load_a_sfa(st, s, kb);
                    load_b(st, s, kb);
                }
            }
            // loads still in flight land before the CTA may exit (for a pair, rank
            // 0's barriers count both CTAs' loads, and the closing cluster barrier
            // keeps rank 1 until rank 0 is past this)
            if (!PAIR || rank == 0) {
                const uint32_t first = it > STAGES ? it - STAGES : 0;
                for (uint32_t j = first; j < it; j++) mbar_wait(&full[j % STAGES], (j / STAGES) & 1, DRAIN_LIMIT);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && (!PAIR || rank == 0)) {
            // a pair's copies and MMAs (issued here, by rank 0) cover both CTAs
            auto cp_sf = [&](uint32_t taddr, uint64_t sdesc) {
                if constexpr (PAIR) tmem_cp_32x128b_x4_pair(taddr, sdesc);
                else tmem_cp_32x128b_x4(taddr, sdesc);
            };
            const uint32_t sfb = tmem_base + MX_SFB_TMEM;
            cp_sf(sfb, sdesc_sf_chunk(smem_u32(smem + L::SFB_OFF)));
            cp_sf(sfb + 4, sdesc_sf_chunk(smem_u32(smem + L::SFB_OFF + 512)));
            uint32_t it = 0, u = 0;
            bool ok = true;
            for (int t = t_first; t < total && ok; t += t_step) {
                const int sp = t % S;
                const int kb0 = sp * p.num_kb / S, kb1 = (sp + 1) * p.num_kb / S;
                const uint32_t acc = u % NACC;
                if (!mbar_wait(&tempty[acc], ((u / NACC) & 1) ^ 1, limit)) { ok = false; break; }
                tc_fence_after();
                for (int kb = kb0; kb < kb1; kb++, it++) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&full[s], (it / STAGES) & 1, limit)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * L::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + MX_A_BYTES;
                    const uint32_t sfa = tmem_base + MX_SFA_TMEM + 4 * s;
                    cp_sf(sfa, sdesc_sf_chunk(b_addr + L::B_BYTES));
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        if constexpr (PAIR)
                            mma_mxf8_pair(tmem_base, sdesc_sw128(a_addr + 32 * j), sdesc_sw128(b_addr + 32 * j),
                                          idesc_mxf8(256, BN, j), sfa, sfb, (kb > kb0 || j > 0));
                        else
                            mma_mxf8(tmem_base + acc * BN, sdesc_sw128(a_addr + 32 * j), sdesc_sw128(b_addr + 32 * j),
                                     idesc_mxf8(128, BN, j), sfa, sfb, (kb > kb0 || j > 0));
                    }
                    if constexpr (PAIR) mma_commit_pair_both(&empty[s]);   // frees the stage in both CTAs
                    else mma_commit(&empty[s]);
                }
                if (!ok) break;
                if constexpr (PAIR) mma_commit_pair_both(tfull);   // both CTAs' epilogues
                else mma_commit(&tfull[acc]);
                u++;
            }
            if (!ok) report(p.status, ST_TIMEOUT, WHERE_GEMM_MMA);
            if constexpr (PAIR) mma_commit_pair(drain);   // every issued MMA has completed ...
            else mma_commit(drain);
            mbar_wait(drain, 0, DRAIN_LIMIT);             // ... before TMEM can be released
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int g = (warp - 2) >> 2;             // NC columns per column group
        const int r = 32 * q + lane;
        const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
        uint8_t* ostg = smem + L::STG_OFF + (warp - 2) * L::STG_WARP_BYTES;
        uint32_t u = 0, nbox = 0;
        bool ok = true;
        // the accumulator is free again: a pair's MMA thread (rank 0) counts both
        // CTAs' epilogue warps
        auto release_acc = [&](uint32_t acc) {
            if constexpr (PAIR) mbar_arrive_cluster(cluster_addr(tempty, 0));
            else mbar_arrive(&tempty[acc]);
        };
        for (int t = t_first; t < total && ok; t += t_step) {
            const int sp = t % S;
            int e, mi, nb;
            bool has_rows;
            unit_tile(t / S, e, mi, nb, has_rows);
            // none for a pair's absent m-tile (its rows lie past the expert's count)
            const int local = mi * 128 + r - s_tptr[e] * 128;
            const bool valid = local < s_off[e + 1] - s_off[e];
            // the row's routing weight is loaded while the tile's MMAs run
            const int slot = s_off[e] + local;
            const float rw = valid ? p.route_w[p.perm[slot]] : 0.0f;
            const int n0 = nb * BN + NC * g;
            const float* cs = p.w_scale + static_cast<size_t>(e) * p.H + n0;
            const uint32_t acc = u % NACC;
            if (!warp_wait(&tfull[acc], (u / NACC) & 1, limit)) { ok = false; break; }
            tc_fence_after();
            if (!__any_sync(0xffffffffu, valid)) {
                // none of this warp's rows is stored: release the accumulator only
                tc_fence_before();
                __syncwarp();
                if (lane == 0) release_acc(acc);
                u++;
                continue;
            }
            float v[NC];
            const uint32_t col0 = acc * BN + NC * g;
#pragma unroll
            for (int ch = 0; ch < NC / 64; ch++)
                tmem_ld32x2(lane_addr + col0 + 64 * ch, lane_addr + col0 + 64 * ch + 32, v + 64 * ch,
                            v + 64 * ch + 32);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) release_acc(acc);   // the next tile's MMAs may start
            u++;
            const size_t orow = static_cast<size_t>(sp) * p.A + slot;
            if (BOXES && __all_sync(0xffffffffu, valid)) {
                // rows sp A + slot(lane 0) + lane: NC / 64 boxes of 64 fp16 columns
                const int y0 = __shfl_sync(0xffffffffu, static_cast<int>(orow), 0);
                uint32_t ebytes = 0;
#pragma unroll
                for (int b = 0; b < NC / 64; b++, nbox++) {
                    uint8_t* buf = ostg + (nbox & 1) * MX_BOX_BYTES;
                    uint32_t w0[16], w1[16];
                    const int e0 = o16_block<true>(v + 64 * b, cs + 64 * b, rw, w0);
                    const int e1 = o16_block<true>(v + 64 * b + 32, cs + 64 * b + 32, rw, w1);
                    ebytes |= ((static_cast<uint32_t>(e0) & 0xFFu) | ((static_cast<uint32_t>(e1) & 0xFFu) << 8))
                              << (16 * b);
                    // the store issued from this buffer two boxes ago has read it
                    if (lane == 0) bulk_wait_read1();
                    __syncwarp();
#pragma unroll
                    for (int c = 0; c < 8; c++) {
                        // 16-byte chunk c of row `lane` sits at chunk c ^ (lane % 8) (128-byte swizzle)
                        const uint32_t* w = c < 4 ? w0 + 4 * c : w1 + 4 * (c - 4);
                        *reinterpret_cast<uint4*>(buf + lane * 128 + 16 * (c ^ (lane & 7))) =
                            make_uint4(w[0], w[1], w[2], w[3]);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmO, buf, (n0 + 64 * b) * 2, y0);
                        bulk_commit();
                    }
                }
                if constexpr (NC == 128) *reinterpret_cast<uint32_t*>(p.oe + orow * (p.H / 32) + n0 / 32) = ebytes;
                else *reinterpret_cast<uint16_t*>(p.oe + orow * (p.H / 32) + n0 / 32) = static_cast<uint16_t>(ebytes);
            } else {
                if constexpr (BOXES) {
                    // the box buffers serve as the row staging once their stores have read them
                    if (lane == 0) bulk_wait_read0();
                    __syncwarp();
                }
                store_rows16<NC, true>(v, reinterpret_cast<uint32_t*>(ostg), valid ? p.o + orow * p.H + n0 : nullptr,
                                        p.oe + orow * (p.H / 32) + n0 / 32, cs, rw, lane);
                __syncwarp();
            }
        }
        if constexpr (BOXES) {
            // every box store has finished writing global memory and reading shared memory
            if (lane == 0) bulk_wait_all();
            __syncwarp();
        }
        if (!ok) report(p.status, ST_TIMEOUT, WHERE_GEMM_EPILOGUE);
    }

    tc_fence_before();
    __syncthreads();
    // a pair leaves together: no arrival or copy may target a CTA that has exited
    if constexpr (PAIR) cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        if constexpr (PAIR) tmem_dealloc_pair(tmem_base, 512);
        else tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace moe
