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
// A per stage: 4 scales of 32 per row), 3 stages.  For small batches the K
// range of each tile may be split S ways (S read from the dispatch's pick,
// work item t = (tile t / S, split t % S)); split s writes its fp32 partial rows to copy s
// of the output rows, o + s * A * H.  MMA j of a stage (K = 32)
// uses byte j of the chunk (scale-factor id j).  TMEM: one 256-column
// accumulator, released as soon as the epilogue has it in registers, then the
// A-scale ring and the constant B-scale chunks.
//
// Output rows: a warp whose 32 rows are all stored (rows of one expert are
// consecutive slots) writes them as four 32-row x 32-column fp32 boxes through
// a 128-byte-swizzled shared buffer (two per warp, alternating) with TMA
// tensor stores, so the store runs asynchronously beside the next tile's
// accumulator read; a warp with fewer rows stores its rows directly.
#pragma once
#include "common.cuh"
#include "gemm.cuh"

namespace moe {

constexpr int MX_BN = 256;
constexpr int MX_A_BYTES = 128 * 128;
constexpr int MX_B_BYTES = MX_BN * 128;
constexpr int MX_SFA_BYTES = 512;
constexpr int MX_STAGE_BYTES = MX_A_BYTES + MX_B_BYTES + 1024;   // + 512 B A scales, padded to 1 KB
constexpr int MX_BOX_BYTES = 32 * 128;                           // 32 rows x 32 fp32
constexpr int MX_SFA_TMEM = MX_BN;                               // 4 columns per stage
constexpr int MX_SFB_TMEM = MX_BN + 16;                          // 8 columns (two 128-row chunks)
// Deep K (many K stages per tile): 4 stages, rows stored from registers.
// Shallow K, where a tile's stores outlast its MMAs: 3 stages and the box stores.
constexpr int MX_BOX_MAX_KB = 16;

template <int STAGES, bool BOXES>
struct MxSmem {
    static constexpr int SFB_OFF = STAGES * MX_STAGE_BYTES;           // 2 constant chunks (1 KB)
    static constexpr int BAR_OFF = SFB_OFF + 1024;
    static constexpr int NUM_BARS = 2 * STAGES + 3;
    static constexpr int TMEM_SLOT_OFF = BAR_OFF + 8 * NUM_BARS;
    static constexpr int TMAP_OFF = TMEM_SLOT_OFF + 16;
    // per epilogue warp: two swizzled boxes, or the float4 row staging
    static constexpr int STG_OFF = BOXES ? (TMAP_OFF + TMAP_BYTES + 1023) / 1024 * 1024
                                         : (TMAP_OFF + TMAP_BYTES + 15) / 16 * 16;
    static constexpr int STG_WARP_BYTES = BOXES ? 2 * MX_BOX_BYTES : STG_WARP_FLOATS * 4;
    static constexpr int TOTAL = STG_OFF + 8 * STG_WARP_BYTES + 1024;
    static_assert(TOTAL <= 232448, "shared memory of the down GEMM exceeds 227 KB");
    static_assert(STG_WARP_FLOATS * 4 <= STG_WARP_BYTES, "row staging fits");
    static_assert(4 * STAGES <= 16, "A-scale ring below the B-scale chunks");
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
    float* o;                  // [S][A][H] fp32 rows in slot order
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

template <int STAGES, bool BOXES>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    grouped_gemm_mx_down_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                const __grid_constant__ CUtensorMap tmO, const MxDownParams p) {
    using L = MxSmem<STAGES, BOXES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = bars + 2 * STAGES + 1;
    uint64_t* drain = bars + 2 * STAGES + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::TMEM_SLOT_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // constant B scale chunks: 1.0 for every row and block
    for (int i = threadIdx.x; i < 1024 / 4; i += blockDim.x)
        reinterpret_cast<uint32_t*>(smem + L::SFB_OFF)[i] = 0x7F7F7F7Fu;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        mbar_init(tempty, 8);
        mbar_init(drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmO);
    }
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    // the generic-proxy writes of the constant chunks become visible to tcgen05.cp
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
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
    __syncthreads();
    const int ntm = *p.num_tiles;
    const int units = ntm * p.n_blocks;
    const int S = min(max(*p.split, 1), p.s_max);
    const int total = units * S;
    const long long limit = p.spin_limit;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            int ready_e = -1;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const int sp = t % S;   // unit-major: all splits of a unit together, experts in order
                int e, mi, nb;
                decode_tile(t / S, s_tptr, p.E, p.n_blocks, e, mi, nb);
                const int brow = e * p.b_rows + nb * MX_BN;
                const uint64_t pol = l2_policy(s_tptr[e + 1] - s_tptr[e] == 1);   // weight tile read once?
                const uint8_t* sfa = p.sfa + static_cast<size_t>(mi) * p.num_kb * 512;
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
                        mbar_arrive_expect_tx(&full[s], MX_A_BYTES + MX_B_BYTES + MX_SFA_BYTES);
                        tma_load_2d_hint(smem + s * MX_STAGE_BYTES + MX_A_BYTES, &tmB, &full[s], (kb0 + armed) * 128,
                                         brow, pol);
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
                        uint8_t* st = smem + (itj % STAGES) * MX_STAGE_BYTES;
                        tma_load_2d(st, &tmA, &full[itj % STAGES], (kb0 + j) * 128, mi * 128);
                        bulk_load(st + MX_A_BYTES + MX_B_BYTES, sfa + (kb0 + j) * 512, MX_SFA_BYTES,
                                  &full[itj % STAGES]);
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
                    uint8_t* st = smem + s * MX_STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[s], MX_A_BYTES + MX_B_BYTES + MX_SFA_BYTES);
                    tma_load_2d(st, &tmA, &full[s], kb * 128, mi * 128);
                    tma_load_2d_hint(st + MX_A_BYTES, &tmB, &full[s], kb * 128, brow, pol);
                    bulk_load(st + MX_A_BYTES + MX_B_BYTES, sfa + kb * 512, MX_SFA_BYTES, &full[s]);
                }
            }
            const uint32_t first = it > STAGES ? it - STAGES : 0;
            for (uint32_t j = first; j < it; j++) mbar_wait(&full[j % STAGES], (j / STAGES) & 1, DRAIN_LIMIT);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t sfb = tmem_base + MX_SFB_TMEM;
            tmem_cp_32x128b_x4(sfb, sdesc_sf_chunk(smem_u32(smem + L::SFB_OFF)));
            tmem_cp_32x128b_x4(sfb + 4, sdesc_sf_chunk(smem_u32(smem + L::SFB_OFF + 512)));
            uint32_t it = 0, u = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const int sp = t % S;
                const int kb0 = sp * p.num_kb / S, kb1 = (sp + 1) * p.num_kb / S;
                if (!mbar_wait(tempty, (u & 1) ^ 1, limit)) { ok = false; break; }
                tc_fence_after();
                for (int kb = kb0; kb < kb1; kb++, it++) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&full[s], (it / STAGES) & 1, limit)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * MX_STAGE_BYTES);
                    const uint32_t b_addr = a_addr + MX_A_BYTES;
                    const uint32_t sfa = tmem_base + MX_SFA_TMEM + 4 * s;
                    tmem_cp_32x128b_x4(sfa, sdesc_sf_chunk(b_addr + MX_B_BYTES));
#pragma unroll
                    for (int j = 0; j < 4; j++)
                        mma_mxf8(tmem_base, sdesc_sw128(a_addr + 32 * j), sdesc_sw128(b_addr + 32 * j),
                                 idesc_mxf8(128, MX_BN, j), sfa, sfb, (kb > kb0 || j > 0));
                    mma_commit(&empty[s]);
                }
                if (!ok) break;
                mma_commit(tfull);
                u++;
            }
            if (!ok) report(p.status, ST_TIMEOUT, WHERE_GEMM_MMA);
            mma_commit(drain);
            mbar_wait(drain, 0, DRAIN_LIMIT);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int g = (warp - 2) >> 2;             // 128 columns per column group
        const int r = 32 * q + lane;
        const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
        uint8_t* ostg = smem + L::STG_OFF + (warp - 2) * L::STG_WARP_BYTES;
        uint32_t u = 0, nbox = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const int sp = t % S;
            int e, mi, nb;
            decode_tile(t / S, s_tptr, p.E, p.n_blocks, e, mi, nb);
            const int local = mi * 128 + r - s_tptr[e] * 128;
            const bool valid = local < s_off[e + 1] - s_off[e];
            // the row's routing weight is loaded while the tile's MMAs run
            const int slot = s_off[e] + local;
            const float rw = valid ? p.route_w[p.perm[slot]] : 0.0f;
            const int n0 = nb * MX_BN + 128 * g;
            const float* cs = p.w_scale + static_cast<size_t>(e) * p.H + n0;
            if (!warp_wait(tfull, u & 1, limit)) { ok = false; break; }
            tc_fence_after();
            if (!__any_sync(0xffffffffu, valid)) {
                // none of this warp's rows is stored: release the accumulator only
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty);
                u++;
                continue;
            }
            float v[128];
#pragma unroll
            for (int ch = 0; ch < 2; ch++)
                tmem_ld32x2(lane_addr + 128 * g + 64 * ch, lane_addr + 128 * g + 64 * ch + 32, v + 64 * ch,
                            v + 64 * ch + 32);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty);   // the next tile's MMAs may start
            u++;
            if (BOXES && __all_sync(0xffffffffu, valid)) {
                // rows sp A + slot(lane 0) + lane: four boxes of 32 columns
                const int y0 = __shfl_sync(0xffffffffu, sp * p.A + slot, 0);
#pragma unroll
                for (int b = 0; b < 4; b++, nbox++) {
                    uint8_t* buf = ostg + (nbox & 1) * MX_BOX_BYTES;
                    float4 s4[8];
#pragma unroll
                    for (int c = 0; c < 8; c++) s4[c] = __ldg(reinterpret_cast<const float4*>(cs + 32 * b + 4 * c));
                    // the store issued from this buffer two boxes ago has read it
                    if (lane == 0) bulk_wait_read1();
                    __syncwarp();
#pragma unroll
                    for (int c = 0; c < 8; c++) {
                        const float* x = v + 32 * b + 4 * c;
                        // 16-byte chunk c of row `lane` sits at chunk c ^ (lane % 8) (128-byte swizzle)
                        *reinterpret_cast<float4*>(buf + lane * 128 + 16 * (c ^ (lane & 7))) =
                            make_float4(x[0] * s4[c].x * rw, x[1] * s4[c].y * rw, x[2] * s4[c].z * rw,
                                        x[3] * s4[c].w * rw);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmO, buf, (n0 + 32 * b) * 4, y0);
                        bulk_commit();
                    }
                }
            } else {
                if constexpr (BOXES) {
                    // the box buffers serve as the row staging once their stores have read them
                    if (lane == 0) bulk_wait_read0();
                    __syncwarp();
                }
                store_rows_coalesced<128, true>(
                    v, reinterpret_cast<float*>(ostg), valid ? p.o + (static_cast<size_t>(sp) * p.A + slot) * p.H + n0 : nullptr,
                    cs, rw, lane);
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
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace moe
