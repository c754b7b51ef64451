// gemm.cuh -- persistent grouped FP8 GEMM on the 5th-gen tensor cores (tcgen05)
// with the two epilogues of the MoE expert MLP.
//
// Pure-Triton fused MoE article: gate and up projections share one input tile
// load and SiLU runs in registers, so no intermediate buffers; a precomputed
// block-id -> (expert id, offset) map runs variable-size expert groups in one
// launch without padding.  LightMoE README ("MoE inference"): gated
// activation, requantisation of the hidden, down projection and the routing
// weight are part of the one layer call.
//
// Roles (one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: A tile [128 rows x 128 K] + B tile [BN rows x 128 K]
//               per stage into a STAGES-deep shared-memory ring (128-byte swizzle)
//   warp 1      allocates TMEM, one thread issues tcgen05.mma (M=128, N=BN, K=32)
//               into a ring of NBUF fp32 accumulators in TMEM (2 for BN=256,
//               4 for narrower tiles)
//   epilogue    warps 2..9 (320 threads), 2..17 (576 threads, the FP8_ROW gate/up
//               GEMM) or 4..11 (384 threads, the promoted GEMMs, whose warps 2
//               and 3 idle so that warpgroup 0 can hand registers to the two
//               epilogue warpgroups): tcgen05.ld of the accumulator, scales,
//               SwiGLU and requantisation (gate/up) or routing weight and the
//               fp16 row store (down)
// Tiles are visited expert by expert; inside an expert, n-block-major with the
// expert's m-tiles fastest, so all readers of one weight tile run at the same
// time and an expert's rows stay in L2 while its n-blocks go by.
// A tile's rows past the expert's last row belong to the next expert or are
// past the end (TMA zero-fills); the epilogue stores only the expert's rows.
//
// PROMOTE: the A operand (and for 128x128-block weights also B) carries one
// fp32 scale per 128 columns of K, so each 128-deep K block is accumulated
// alone in TMEM and the epilogue adds it into registers times its scales.
// Without PROMOTE the whole K reduction stays in TMEM.
//
// Every wait is bounded (spin_limit clock cycles): on expiry the kernel records
// MOE timeout in the status word and leaves its loops; nothing traps.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 128;                 // K bytes (= e4m3 elements) per stage
constexpr int GEMM_THREADS = 320;            // 8 epilogue warps
constexpr int GEMM_A_BYTES = GEMM_BM * GEMM_BK;

enum { KIND_GATE_UP = 0, KIND_DOWN = 1 };
enum { BSCALE_ROW = 0, BSCALE_BLOCK128 = 1 };

struct GemmParams {
    const int32_t* tiles;       // [ntiles][2] (expert, first row)
    const int32_t* num_tiles;   // number of m-tiles (device scalar)
    const int32_t* tile_ptr;    // [E+1] first m-tile of each expert
    int E;
    const int32_t* offsets;     // [E+1]
    int n_blocks;               // N / BN
    int num_kb;                 // K / 128
    int b_rows;                 // rows of B per expert (2I for gate/up, H for down)
    const float* a_scale;       // X or hidden scales, a_ld floats per row
    int a_ld;
    const float* b_scale;       // BSCALE_ROW: [E][b_rows]; BLOCK128: [E][b_rows/128][num_kb]
    uint8_t* hq;                // gate/up: hidden codes; FP8_ROW: [padded rows][I] + MX scales in hsf,
    float* hs;                  //   BLOCK128: [A][I] + fp32 scales hs [A][I/128]
    uint8_t* hsf;
    int I;
    int act;                    // gate/up: gated activation (the kernel is instantiated for it)
    int32_t* gu_done;           // FP8_ROW gate/up: per-expert count of finished (tile, epilogue warp)
                                //   parts, for a down GEMM that starts before this kernel ends
    float act_alpha, act_limit;
    uint16_t* o;                // down: [A][H] fp16 rows with block exponents oe
    int8_t* oe;                 //   [A][H / 32]
    int H;
    const int32_t* perm;        // down: slot -> t*k + j
    const float* route_w;       // down: [T*k]
    int32_t* status;
    long long spin_limit;
};

constexpr int TMAP_STRIDE = 260;              // shared-memory tile map: 2 x (E + 1) ints, E <= 256
constexpr int TMAP_BYTES = 2 * TMAP_STRIDE * 4;

// Sparse gate/up epilogue (a warp with few stored rows): per epilogue warp a
// [8 rows][32 gate | 32 up] fp32 staging block and the 8 rows' X scales.
constexpr int SPARSE_ROWS_MAX = 16;
constexpr int SPARSE_WARP_FLOATS = 8 * 64 + 8;

// Coalesced fp32 row stores of the down epilogues.  A warp holds 32 rows (one
// per lane) x NC columns; 16-column chunks pass through a per-warp [32][20]
// float block (rows padded to 80 B, so the row-wise float4 writes of 8 lanes
// hit distinct banks), and every store instruction then writes 8 rows x 64
// contiguous bytes (4 lanes per row) instead of 32 rows x 16 bytes.
// dst: this lane's row at its first column, null when the row is not stored.
// Stored value: (v[c] * cs[c]) * rs with column scales, else v[c] * rs.
// Warps with at most 8 stored rows store them directly (fewer steps).
// TMA tensor store of one box from shared memory, and the bulk-group waits.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* tm, const void* src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(tm)),
                 "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// at most one store group of this thread still reading shared memory
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// all store groups of this thread complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

constexpr int STG_STRIDE = 20;
constexpr int STG_WARP_FLOATS = 32 * STG_STRIDE;
template <int NC, bool HAS_CS>
__device__ __forceinline__ void store_rows_coalesced(const float (&v)[NC], float* stg, float* dst, const float* cs,
                                                     float rs, int lane) {
    if (__popc(__ballot_sync(0xffffffffu, dst != nullptr)) <= 8) {
        // few stored rows (small batches): each stores its own row directly
        if (dst != nullptr) {
#pragma unroll
            for (int c = 0; c < NC; c += 4) {
                float4 o;
                if (HAS_CS) {
                    const float4 s4 = __ldg(reinterpret_cast<const float4*>(cs + c));
                    o = make_float4(v[c] * s4.x * rs, v[c + 1] * s4.y * rs, v[c + 2] * s4.z * rs, v[c + 3] * s4.w * rs);
                } else {
                    o = make_float4(v[c] * rs, v[c + 1] * rs, v[c + 2] * rs, v[c + 3] * rs);
                }
                *reinterpret_cast<float4*>(dst + c) = o;
            }
        }
        return;
    }
    const int rsub = lane >> 2, c4 = (lane & 3) * 4;
#pragma unroll
    for (int ch = 0; ch < NC / 16; ch++) {
        float4* w = reinterpret_cast<float4*>(stg + lane * STG_STRIDE);
#pragma unroll
        for (int q4 = 0; q4 < 4; q4++)
            w[q4] = make_float4(v[16 * ch + 4 * q4], v[16 * ch + 4 * q4 + 1], v[16 * ch + 4 * q4 + 2],
                                v[16 * ch + 4 * q4 + 3]);
        __syncwarp();
        float4 s4 = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
        if (HAS_CS) s4 = __ldg(reinterpret_cast<const float4*>(cs + 16 * ch + c4));
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int row = 8 * i + rsub;
            float* d = reinterpret_cast<float*>(__shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(dst), row));
            const float r = __shfl_sync(0xffffffffu, rs, row);
            const float4 x = *reinterpret_cast<const float4*>(stg + row * STG_STRIDE + c4);
            if (d != nullptr) {
                float4 o;
                if (HAS_CS) o = make_float4(x.x * s4.x * r, x.y * s4.y * r, x.z * s4.z * r, x.w * s4.w * r);
                else o = make_float4(x.x * r, x.y * r, x.z * r, x.w * r);
                *reinterpret_cast<float4*>(d + 16 * ch + c4) = o;
            }
        }
        __syncwarp();
    }
}

// ------------------------------------------------------------------ fp16 output rows
// The down GEMMs store each weighted output row (slot order) in fp16 with a
// power-of-two scale per 32 columns: a block's values v are stored as
// fp16(v 2^(15 - e)), e the binary exponent of the block's largest |v|
// (amax < 2^e, clamped to [-110, 127]), and e in one signed byte.  The scaled
// largest value is below 2^15, so nothing overflows, and every value keeps the
// 11 significant bits of fp16 relative to its block's largest (a fifth of a
// bf16 rounding).  The combine reads them back as fp16 2^(e - 15) and adds the
// k rows (and K-split copies) in fixed order in fp32.
__device__ __forceinline__ int o16_exponent(float amax) {
    // amax = 1.m 2^(E - 127) < 2^(E - 126); 0 and subnormals clamp to -110
    const int e = ((__float_as_int(amax) >> 23) & 0xFF) - 126;
    return e < -110 ? -110 : (e > 127 ? 127 : e);
}
__device__ __forceinline__ float pow2f(int k) { return __int_as_float((127 + k) << 23); }   // k in [-126, 127]
__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}
// one 32-column block of this lane's row: (v * cs) * rs (or v * rs) rounded to
// fp32 as before, its exponent, and the 16 words of fp16 pairs
template <bool HAS_CS>
__device__ __forceinline__ int o16_block(const float* v, const float* cs, float rs, uint32_t (&w)[16]) {
    float val[32];
    float amax = 0.0f;
#pragma unroll
    for (int c4 = 0; c4 < 8; c4++) {
        float4 s4 = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
        if (HAS_CS) s4 = __ldg(reinterpret_cast<const float4*>(cs + 4 * c4));
        const float sc[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int c = 4 * c4 + i;
            val[c] = HAS_CS ? v[c] * sc[i] * rs : v[c] * rs;
            amax = fmaxf(amax, fabsf(val[c]));
        }
    }
    const int e = o16_exponent(amax);
    const float up = pow2f(15 - e);
#pragma unroll
    for (int c = 0; c < 16; c++) w[c] = pack_h2(val[2 * c] * up, val[2 * c + 1] * up);
    return e;
}

// Store this lane's NC output columns as fp16 rows with block exponents
// (dst: the row's first fp16, dst_e: its first exponent byte; null when the
// row is not stored).  32-column blocks pass through the per-warp [32][20]-word
// staging so each store instruction writes 8 rows x 64 contiguous bytes; warps
// with at most 8 stored rows store their rows directly.
template <int NC, bool HAS_CS>
__device__ __forceinline__ void store_rows16(const float (&v)[NC], uint32_t* stg, uint16_t* dst, int8_t* dst_e,
                                             const float* cs, float rs, int lane) {
    static_assert(NC % 32 == 0 && NC <= 128, "whole 32-column blocks, at most 4 exponent bytes");
    uint32_t ebytes = 0;
    if (__popc(__ballot_sync(0xffffffffu, dst != nullptr)) <= 8) {
        if (dst != nullptr) {
#pragma unroll
            for (int b = 0; b < NC / 32; b++) {
                uint32_t w[16];
                const int e = o16_block<HAS_CS>(v + 32 * b, HAS_CS ? cs + 32 * b : nullptr, rs, w);
                ebytes |= (static_cast<uint32_t>(e) & 0xFFu) << (8 * b);
                uint4* d = reinterpret_cast<uint4*>(dst + 32 * b);
#pragma unroll
                for (int q4 = 0; q4 < 4; q4++) d[q4] = make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
            }
        }
    } else {
        const int rsub = lane >> 2, c4 = (lane & 3) * 4;
#pragma unroll
        for (int b = 0; b < NC / 32; b++) {
            uint32_t w[16];
            const int e = o16_block<HAS_CS>(v + 32 * b, HAS_CS ? cs + 32 * b : nullptr, rs, w);
            ebytes |= (static_cast<uint32_t>(e) & 0xFFu) << (8 * b);
            uint4* sw = reinterpret_cast<uint4*>(stg + lane * STG_STRIDE);
#pragma unroll
            for (int q4 = 0; q4 < 4; q4++) sw[q4] = make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const int row = 8 * i + rsub;
                uint16_t* d = reinterpret_cast<uint16_t*>(
                    __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(dst), row));
                const uint4 x = *reinterpret_cast<const uint4*>(stg + row * STG_STRIDE + c4);
                if (d != nullptr) *reinterpret_cast<uint4*>(d + 32 * b + 2 * c4) = x;
            }
            __syncwarp();
        }
    }
    if (dst != nullptr) {
        if constexpr (NC == 128) *reinterpret_cast<uint32_t*>(dst_e) = ebytes;
        else if constexpr (NC == 64) *reinterpret_cast<uint16_t*>(dst_e) = static_cast<uint16_t>(ebytes);
        else *dst_e = static_cast<int8_t>(ebytes & 0xFFu);
    }
}

// per epilogue warp: the sparse gate/up staging or the down store staging
constexpr int EPI_WARP_FLOATS = SPARSE_WARP_FLOATS > STG_WARP_FLOATS ? SPARSE_WARP_FLOATS : STG_WARP_FLOATS;

// EPI epilogue warps (8 or 16): 4 TMEM lane quadrants x EPI/4 column groups.
// The promoted (FP8_BLOCK128) GEMMs hold 128 fp32 partial sums per epilogue
// thread across the K loop; they launch a whole warpgroup 0 (producer, MMA
// issuer, two idle warps) so that registers can move from it to the epilogue
// warpgroups (setmaxnreg), and their epilogue warps start at warp 4.
template <int EPI, bool PROMOTE = false>
__host__ __device__ constexpr int gemm_threads() { return (PROMOTE ? 128 : 64) + 32 * EPI; }
template <bool PROMOTE>
__host__ __device__ constexpr int first_epi_warp() { return PROMOTE ? 4 : 2; }
// Register split of the promoted GEMMs: 384 threads launch with 168 registers
// each (65536 / 384, rounded down to the allocation step of 8); warpgroup 0
// drops to 40 and the two epilogue warpgroups rise to 232, which uses exactly
// the launch's 64512 (128 x 40 + 256 x 232), and each sub-partition holds one
// warp of each warpgroup: 32 x (40 + 2 x 232) = 16128 of its 16384.  At 232
// the 128 partial sums, a 64-column TMEM load and the loop state fit without
// spills (at 168 the K loop spilled to local memory, whose traffic competes
// with the MMAs' shared-memory operand reads).
constexpr int PROMOTE_LAUNCH_REGS = 168;
constexpr int PROMOTE_CTRL_REGS = 40;
constexpr int PROMOTE_EPI_REGS = 232;
static_assert(gemm_threads<8, true>() * PROMOTE_LAUNCH_REGS >= 128 * PROMOTE_CTRL_REGS + 256 * PROMOTE_EPI_REGS,
              "the promoted GEMM's register split exceeds its launch allocation");
static_assert(32 * (PROMOTE_CTRL_REGS + 2 * PROMOTE_EPI_REGS) <= 16384,
              "the promoted GEMM's register split exceeds a sub-partition's register file");
// sparse gate/up staging rows per round: 8 with 8 epilogue warps, 4 with 16
template <int EPI>
__host__ __device__ constexpr int sparse_round() { return EPI == 8 ? 8 : 4; }
template <int EPI>
__host__ __device__ constexpr int epi_warp_floats() {
    return EPI == 8 ? EPI_WARP_FLOATS : sparse_round<EPI>() * 64 + sparse_round<EPI>();
}

template <int BN, int STAGES, int EPI = 8, bool PAIR = false>
struct GemmSmem {
    // accumulator buffers in TMEM (512 columns): deeper for narrower tiles, so the
    // MMA can run further ahead of a per-K-block epilogue
    static constexpr int NBUF = (512 / BN) < 4 ? (512 / BN) : 4;
    static constexpr int B_BYTES = (PAIR ? BN / 2 : BN) * GEMM_BK;   // a CTA pair splits B by rows
    static constexpr int STAGE_BYTES = GEMM_A_BYTES + B_BYTES;
    static constexpr int TILES_BYTES = STAGES * STAGE_BYTES;
    // after the tiles: barriers, TMEM address, amax exchange
    static constexpr int BAR_OFF = TILES_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * NBUF + 1;
    static constexpr int TMEM_SLOT_OFF = BAR_OFF + 8 * NUM_BARS;
    static constexpr int XCHG_OFF = (TMEM_SLOT_OFF + 4 + 15) / 16 * 16;
    static constexpr int XCHG_BYTES = 2 * 2 * 128 * 4 * 2;   // [parity][group][row] value + flag
    static constexpr int TMAP_OFF = XCHG_OFF + XCHG_BYTES;
    static constexpr int SPARSE_OFF = TMAP_OFF + TMAP_BYTES;
    static constexpr int PPTR_OFF = SPARSE_OFF + EPI * epi_warp_floats<EPI>() * 4;   // CTA pairs: m-pair map
    static constexpr int TOTAL = PPTR_OFF + (PAIR ? TMAP_STRIDE * 4 : 0) + 1024;       // + alignment slack
    static_assert(SPARSE_OFF % 16 == 0, "staging block must be 16-byte aligned");
};

// The schedule's tile pointers and row offsets, copied into shared memory once
// per CTA (after the dispatch wrote them), so decoding a tile is a few
// shared-memory reads instead of a chain of dependent global loads.
// Layout: tile_ptr[0..E] at s[0..], offsets[0..E] at s[TMAP_STRIDE..].
__device__ __forceinline__ void stage_tile_map(int32_t* s, const int32_t* tile_ptr, const int32_t* offsets, int E) {
    for (int i = threadIdx.x; i <= E; i += blockDim.x) {
        s[i] = tile_ptr[i];
        s[TMAP_STRIDE + i] = offsets[i];
    }
}

// Tile t -> (expert, m-tile index, n-block): expert e owns tiles
// [tile_ptr[e] nb, tile_ptr[e+1] nb), n-block-major with its m-tiles fastest.
__device__ __forceinline__ void decode_tile(int t, const int32_t* s_tptr, int E, int n_blocks, int& e, int& mi,
                                            int& nb) {
    int lo = 0, hi = E;   // tile_ptr[lo] * n_blocks <= t < tile_ptr[hi] * n_blocks
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_tptr[mid] * n_blocks <= t) lo = mid; else hi = mid;
    }
    const int first = s_tptr[lo];
    const int mt = s_tptr[lo + 1] - first;
    const int local = t - first * n_blocks;
    e = lo;
    nb = local / mt;
    mi = first + local % mt;
}

// CTA pairs: unit t -> (expert, m-pair, n-block).  Expert e owns m-pairs
// [pptr[e], pptr[e+1]) (ceil(m-tiles / 2) of them), n-block-major with its
// m-pairs fastest; m-pair j covers the expert's m-tiles 2j (rank 0) and 2j + 1
// (rank 1, absent when the count is odd).
__device__ __forceinline__ void decode_pair(int t, const int32_t* s_pptr, int E, int n_blocks, int& e, int& mp,
                                            int& nb) {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_pptr[mid] * n_blocks <= t) lo = mid; else hi = mid;
    }
    const int first = s_pptr[lo];
    const int np = s_pptr[lo + 1] - first;
    const int local = t - first * n_blocks;
    e = lo;
    nb = local / np;
    mp = local % np;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, long long limit) {
    const bool ok = mbar_wait(bar, parity, limit);
    return __all_sync(0xffffffffu, ok);
}

template <int KIND, int BSCALE, bool PROMOTE, int BN, int STAGES, int EPI = 8, int ACT = 0, bool PAIR = false>
__device__ __forceinline__ void gemm_body(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& p,
                                          const int n_blocks, uint8_t* smem_raw) {
    static_assert(EPI == 8 || (EPI == 16 && KIND == KIND_GATE_UP && BSCALE == BSCALE_ROW && !PROMOTE),
                  "16 epilogue warps are built for the FP8_ROW gate/up GEMM only");
    static_assert(!PAIR || (KIND == KIND_GATE_UP && BSCALE == BSCALE_ROW && !PROMOTE && BN == 256),
                  "CTA pairs are built for the FP8_ROW gate/up GEMM only");
    static_assert(KIND != KIND_GATE_UP || BN == 256 || (BN == 128 && BSCALE == BSCALE_ROW && !PROMOTE && ACT != 5 &&
                                                        !PAIR),
                  "128-wide gate/up tiles are built for gated FP8_ROW activations on single CTAs");
    using S = GemmSmem<BN, STAGES, EPI, PAIR>;
    // column groups with work: a 128-wide gate/up tile launched with 16
    // epilogue warps gives its 64 hidden columns to two groups (32 each, so a
    // 32-column MX block stays in one thread); the other 8 warps idle
    constexpr int CG = (KIND == KIND_GATE_UP && BN == 128 && EPI == 16) ? 2 : EPI / 4;
    constexpr int EPA = 4 * CG;          // epilogue warps with work
    // gate/up: a tile's gate half and up half (128 + 128 accumulator columns, or
    // 64 + 64 in a 128-wide tile), and the hidden columns of each per thread
    constexpr int GU_HALF = KIND == KIND_GATE_UP ? BN / 2 : 128;
    constexpr int GC = GU_HALF / CG;     // 64 or 32
    // first packed weight row of gate/up n-block nb: packed rows come in groups
    // of 128 gate + 128 up rows; a 128-wide tile takes 64 of each, at 64 (nb & 1)
    auto gu_row0 = [&](int nb) { return BN == 256 ? nb * 256 : 256 * (nb >> 1) + 64 * (nb & 1); };
    constexpr int NH = GC / 32;          // 32-column blocks per thread
    constexpr int EPI0 = first_epi_warp<PROMOTE>();
    constexpr int SR = sparse_round<EPI>();
    constexpr int EWF = epi_warp_floats<EPI>();
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    constexpr int NBUF = S::NBUF;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = bars + 2 * STAGES + NBUF;
    uint64_t* drain = bars + 2 * STAGES + 2 * NBUF;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::TMEM_SLOT_OFF);
    float* xval = reinterpret_cast<float*>(smem + S::XCHG_OFF);                 // [2][2][128]
    int* xflag = reinterpret_cast<int*>(smem + S::XCHG_OFF + 2 * 2 * 128 * 4);  // [2][2][128]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr uint32_t TMEM_COLS = NBUF * BN;
    // CTA pairs: rank 0 issues the MMAs; its full and tempty barriers take the
    // arrivals of both CTAs
    const uint32_t rank = PAIR ? cluster_rank() : 0u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(&full[s], PAIR ? 2 : 1);   // pairs: one expect_tx arrival per CTA
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NBUF; b++) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], PAIR ? 2 * EPA : EPA);   // one arrival per working epilogue warp
        }
        mbar_init(drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    for (int i = threadIdx.x; i < 2 * 2 * 128; i += blockDim.x) xflag[i] = 0;
    if (warp == 1) {
        if constexpr (PAIR) tmem_alloc_pair(tmem_slot, TMEM_COLS);
        else tmem_alloc(tmem_slot, TMEM_COLS);
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();   // both CTAs' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    pdl_wait();
    pdl_trigger();
    KTRACE(p.o != nullptr ? TR_GEMM + 3 : TR_GEMM);
    int32_t* s_tptr = reinterpret_cast<int32_t*>(smem + S::TMAP_OFF);
    const int32_t* s_off = s_tptr + TMAP_STRIDE;
    stage_tile_map(s_tptr, p.tile_ptr, p.offsets, p.E);
    int32_t* s_pptr = reinterpret_cast<int32_t*>(smem + S::PPTR_OFF);
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
    const int total = PAIR ? s_pptr[p.E] * n_blocks : ntm * n_blocks;
    const long long limit = p.spin_limit;
    // CTA pairs walk the units by cluster; single CTAs by block
    const int t_first = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int t_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    // this CTA's m-tile of unit t: (expert, global m-tile index, has rows)
    auto unit_tile = [&](int t, int& e, int& mi, int& nb, bool& has_rows) {
        if constexpr (PAIR) {
            int mp;
            decode_pair(t, s_pptr, p.E, n_blocks, e, mp, nb);
            const int local = 2 * mp + static_cast<int>(rank);
            has_rows = local < s_tptr[e + 1] - s_tptr[e];
            mi = s_tptr[e] + local;
        } else {
            decode_tile(t, s_tptr, p.E, n_blocks, e, mi, nb);
            has_rows = true;
        }
    };

    if (warp < EPI0) {
        // control warps: the producer (warp 0), the MMA issuer (warp 1) and, in
        // the promoted GEMMs, two idle warps that complete warpgroup 0, which
        // needs few registers
        if constexpr (PROMOTE) setmaxnreg_dec<PROMOTE_CTRL_REGS>();
        if (warp == 0) {
            // -------------------------------------------------------- producer
            if (lane == 0) {
                uint32_t it = 0;
                bool ok = true;
                for (int t = t_first; t < total && ok; t += t_step) {
                    int e, mi, nb;
                    bool has_rows;
                    unit_tile(t, e, mi, nb, has_rows);
                    // a pair's rank 1 without an m-tile (odd count) loads rank 0's rows,
                    // so its A stays inside the tensor; its accumulator rows are not stored
                    const int row0 = s_off[e] + GEMM_BM * (mi - (has_rows ? 0 : 1) - s_tptr[e]);
                    const int brow = e * p.b_rows + (KIND == KIND_GATE_UP ? gu_row0(nb) : nb * BN) +
                                     (PAIR ? static_cast<int>(rank) * (BN / 2) : 0);
                    // L2 policies: a weight tile read once goes first; in the promoted
                    // GEMMs (slower per K block, so the CTAs sharing a tile drift further
                    // apart) every weight tile goes first and the A tile, which all the
                    // n-blocks of its m-tile read, is kept
                    const uint64_t pol = l2_policy(PROMOTE || s_tptr[e + 1] - s_tptr[e] == 1);
                    for (int kb = 0; kb < p.num_kb; kb++, it++) {
                        const int s = it % STAGES;
                        if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, limit)) {
                            report(p.status, ST_TIMEOUT, WHERE_GEMM_PRODUCER);
                            ok = false;
                            break;
                        }
                        uint8_t* sa = smem + s * S::STAGE_BYTES;
                        if constexpr (PAIR) {
                            // both CTAs' halves complete on rank 0's barrier
                            const uint32_t fb = cluster_addr(&full[s], 0);
                            mbar_arrive_expect_tx_cluster(fb, S::STAGE_BYTES);
                            tma_load_2d_pair(sa, &tmA, fb, kb * GEMM_BK, row0, l2_policy(false));
                            tma_load_2d_pair(sa + GEMM_A_BYTES, &tmB, fb, kb * GEMM_BK, brow, pol);
                        } else {
                            mbar_arrive_expect_tx(&full[s], S::STAGE_BYTES);
                            if constexpr (PROMOTE)
                                tma_load_2d_hint(sa, &tmA, &full[s], kb * GEMM_BK, row0, l2_policy_keep());
                            else
                                tma_load_2d(sa, &tmA, &full[s], kb * GEMM_BK, row0);
                            if (KIND == KIND_GATE_UP && BN == 128) {
                                // 64 gate rows, then the 64 matching up rows 128 further
                                // (the tensor map's box is 64 rows)
                                tma_load_2d_hint(sa + GEMM_A_BYTES, &tmB, &full[s], kb * GEMM_BK, brow, pol);
                                tma_load_2d_hint(sa + GEMM_A_BYTES + 64 * GEMM_BK, &tmB, &full[s], kb * GEMM_BK,
                                                 brow + 128, pol);
                            } else {
                                tma_load_2d_hint(sa + GEMM_A_BYTES, &tmB, &full[s], kb * GEMM_BK, brow, pol);
                            }
                        }
                        if (PROMOTE) KTRACE_BLK(it, 7);
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
                // a pair's MMA covers both CTAs' 128 rows (M = 256)
                constexpr uint32_t idesc = idesc_e4m3(PAIR ? 2 * GEMM_BM : GEMM_BM, BN);
                uint32_t it = 0, u = 0;
                bool ok = true;
                for (int t = t_first; t < total && ok; t += t_step) {
                    uint32_t acc = 0;
                    if (!PROMOTE) {
                        acc = u % NBUF;
                        if (!mbar_wait(&tempty[acc], ((u / NBUF) & 1) ^ 1, limit)) { ok = false; break; }
                        tc_fence_after();
                    }
                    for (int kb = 0; kb < p.num_kb; kb++, it++) {
                        if (PROMOTE) {
                            acc = u % NBUF;
                            if (!mbar_wait(&tempty[acc], ((u / NBUF) & 1) ^ 1, limit)) { ok = false; break; }
                            tc_fence_after();
                            KTRACE_BLK(u, 0);
                        }
                        const int s = it % STAGES;
                        if (!mbar_wait(&full[s], (it / STAGES) & 1, limit)) { ok = false; break; }
                        tc_fence_after();
                        if (PROMOTE) KTRACE_BLK(u, 1);
                        const uint32_t a_addr = smem_u32(smem + s * S::STAGE_BYTES);
                        const uint32_t b_addr = a_addr + GEMM_A_BYTES;
                        const uint32_t d = tmem_base + acc * BN;
                        if constexpr (PAIR) {
#pragma unroll
                            for (int kk = 0; kk < GEMM_BK / 32; kk++)
                                mma_f8_pair(d, sdesc_sw128(a_addr + 32 * kk), sdesc_sw128(b_addr + 32 * kk), idesc,
                                            kb > 0 || kk > 0);
                            mma_commit_pair_both(&empty[s]);   // frees the stage in both CTAs
                        } else {
#pragma unroll
                            for (int kk = 0; kk < GEMM_BK / 32; kk++)
                                mma_f8(d, sdesc_sw128(a_addr + 32 * kk), sdesc_sw128(b_addr + 32 * kk), idesc,
                                       PROMOTE ? (kk > 0) : (kb > 0 || kk > 0));
                            mma_commit(&empty[s]);
                        }
                        if (PROMOTE) {
                            mma_commit(&tfull[acc]);
                            KTRACE_BLK(u, 2);
                            u++;
                        }
                    }
                    if (!ok) break;
                    if (!PROMOTE) {
                        if constexpr (PAIR) mma_commit_pair_both(&tfull[acc]);   // both CTAs' epilogues
                        else mma_commit(&tfull[acc]);
                        u++;
                    }
                }
                if (!ok) report(p.status, ST_TIMEOUT, WHERE_GEMM_MMA);
                if constexpr (PAIR) mma_commit_pair(drain);   // every issued MMA has completed ...
                else mma_commit(drain);
                mbar_wait(drain, 0, DRAIN_LIMIT);        // ... before TMEM can be released
            }
        }
    } else if (warp - EPI0 < EPA) {
        // ------------------------------------------------------------ epilogue
        // (the promoted GEMMs' partial sums take the registers warpgroup 0 gave up)
        if constexpr (PROMOTE) setmaxnreg_inc<PROMOTE_EPI_REGS>();
        const int ew = warp - EPI0;
        const int q = warp & 3;               // TMEM lane quadrant this warp may access
        const int g = ew >> 2;                // column group
        const int r = 32 * q + lane;          // row within the tile
        const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
        uint32_t u = 0, iter = 0;
        bool ok = true;
        // the accumulator is free again: a pair's MMA thread (rank 0) counts both
        // CTAs' epilogue warps
        auto release_acc = [&](uint64_t* bar) {
            if constexpr (PAIR) mbar_arrive_cluster(cluster_addr(bar, 0));
            else mbar_arrive(bar);
        };
        for (int t = t_first; t < total && ok; t += t_step, iter++) {
            int e, mi, nb;
            bool has_rows;
            unit_tile(t, e, mi, nb, has_rows);
            const int row0 = s_off[e] + GEMM_BM * (mi - s_tptr[e]);
            const int row = row0 + r;
            const bool valid = row < s_off[e + 1];   // none for a pair's absent m-tile

            // FP8_ROW gate/up: this warp's part of the tile is stored; publish it
            // (per-lane release, then one count per warp) for the chained down GEMM
            auto publish = [&]() {
                if constexpr (KIND == KIND_GATE_UP && BSCALE == BSCALE_ROW) {
                    if (p.gu_done != nullptr && has_rows) {
                        fence_proxy_async_global();
                        __threadfence();
                        __syncwarp();
                        if (lane == 0) atomicAdd(p.gu_done + e, 1);
                    }
                }
            };
            if (KIND == KIND_GATE_UP) {
                float hv[64];
                float hv2[64];                  // ReLU^2: the up-half columns' outputs (BLOCK128)
                if constexpr (!PROMOTE) {
                    // scales are loaded while the tile's MMAs run: the row's X scale,
                    // and lane c holds the weight scale of column c of each 32-column
                    // half (read back with a shuffle)
                    const float sa = valid ? p.a_scale[static_cast<size_t>(row) * p.a_ld] : 0.0f;
                    const float* bs = p.b_scale + static_cast<size_t>(e) * p.b_rows + gu_row0(nb);
                    float bsg[NH], bsu[NH];
#pragma unroll
                    for (int half = 0; half < NH; half++) {
                        bsg[half] = __ldg(bs + GC * g + 32 * half + lane);
                        bsu[half] = __ldg(bs + 128 + GC * g + 32 * half + lane);
                    }
                    const uint32_t acc = u % NBUF;
                    if (!warp_wait(&tfull[acc], (u / NBUF) & 1, limit)) { ok = false; break; }
                    tc_fence_after();
                    if (!__any_sync(0xffffffffu, valid)) {
                        // none of this warp's rows is stored: release the buffer only
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) release_acc(&tempty[acc]);
                        u++;
                        publish();
                        continue;
                    }
                    const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
                    const int nv = __popc(vmask);
                    if (BSCALE == BSCALE_ROW && nv <= SPARSE_ROWS_MAX) {
                        // Few stored rows (small batches): stage them in shared memory
                        // 8 at a time and let lane c take column c of each, so the work
                        // scales with the stored rows.  Same operations per element as
                        // the row path below, so the same codes and scales.
                        float* sb = reinterpret_cast<float*>(smem + S::SPARSE_OFF) + ew * EWF;
                        const int cidx = __popc(vmask & ((1u << lane) - 1u));
#pragma unroll
                        for (int half = 0; half < NH; half++) {
                            float gv[32], uv[32];
                            const int c0 = GC * g + 32 * half;
                            tmem_ld32x2(lane_addr + acc * BN + c0, lane_addr + acc * BN + GU_HALF + c0, gv, uv);
                            if (half == NH - 1) {
                                tc_fence_before();
                                __syncwarp();
                                if (lane == 0) release_acc(&tempty[acc]);
                            }
                            // first hidden column of this 32-block (ReLU^2: the gate-half
                            // columns are up rows 256 nb + c0, the up half 256 nb + 128 + c0)
                            const int hcol = ACT == 5 ? nb * 256 + c0 : nb * GU_HALF + c0;
                            uint32_t m = vmask;
                            for (int r0 = 0; r0 < nv; r0 += SR) {
                                if (valid && cidx >= r0 && cidx < r0 + SR) {
                                    float4* d = reinterpret_cast<float4*>(sb + (cidx - r0) * 64);
#pragma unroll
                                    for (int q4 = 0; q4 < 8; q4++) {
                                        d[q4] = make_float4(gv[4 * q4], gv[4 * q4 + 1], gv[4 * q4 + 2], gv[4 * q4 + 3]);
                                        d[8 + q4] = make_float4(uv[4 * q4], uv[4 * q4 + 1], uv[4 * q4 + 2], uv[4 * q4 + 3]);
                                    }
                                    sb[SR * 64 + cidx - r0] = sa;
                                }
                                __syncwarp();
                                const int nr = min(SR, nv - r0);
                                for (int i = 0; i < nr; i++) {
                                    const int rl = __ffs(m) - 1;   // lane (tile row 32 q + rl) of stored row r0 + i
                                    m &= m - 1;
                                    const float sa_i = sb[SR * 64 + i];
                                    const float gg = sb[i * 64 + lane] * (sa_i * bsg[half]);
                                    const float uu = sb[i * 64 + 32 + lane] * (sa_i * bsu[half]);
                                    const long long prow = static_cast<long long>(mi) * 128 + 32 * q + rl;
                                    // gated: one block act(gg, uu); ReLU^2: relu(gg)^2 and relu(uu)^2
#pragma unroll
                                    for (int ob = 0; ob < (ACT == 5 ? 2 : 1); ob++) {
                                        const float hvv = ACT == 5 ? relu_sq(ob ? uu : gg)
                                                                   : glu_e4m3<ACT>(gg, uu, p.act_alpha, p.act_limit);
                                        const int col = hcol + 128 * ob;
                                        float amax = fabsf(hvv);
#pragma unroll
                                        for (int off = 16; off > 0; off >>= 1)
                                            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
                                        const int ex = mx_exponent(amax);
                                        p.hq[prow * p.I + col + lane] = f_to_e4m3(__fmul_rn(hvv, mx_inv_scale(ex)));
                                        if (lane == 0) p.hsf[sf_offset(prow, col / 32, p.I / 32)] = static_cast<uint8_t>(ex + 127);
                                    }
                                }
                                __syncwarp();
                            }
                        }
                        u++;
                        publish();
                        continue;
                    }
#pragma unroll
                    for (int half = 0; half < NH; half++) {
                        float gv[32], uv[32];
                        const int c0 = GC * g + 32 * half;
                        tmem_ld32x2(lane_addr + acc * BN + c0, lane_addr + acc * BN + GU_HALF + c0, gv, uv);
#pragma unroll
                        for (int c = 0; c < 32; c++) {
                            const float gg = gv[c] * (sa * __shfl_sync(0xffffffffu, bsg[half], c));
                            const float uu = uv[c] * (sa * __shfl_sync(0xffffffffu, bsu[half], c));
                            if constexpr (ACT == 5) {
                                hv[32 * half + c] = relu_sq(gg);
                                hv[32 * (NH + half) + c] = relu_sq(uu);
                            } else {
                                hv[32 * half + c] = glu_e4m3<ACT>(gg, uu, p.act_alpha, p.act_limit);
                            }
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) release_acc(&tempty[acc]);
                    u++;
                } else {
                    float ag[64], au[64];
#pragma unroll
                    for (int c = 0; c < 64; c++) ag[c] = au[c] = 0.0f;
                    const bool any_valid = __any_sync(0xffffffffu, valid);
                    const float* arow = p.a_scale + static_cast<size_t>(valid ? row : 0) * p.a_ld;
                    const float* bsb = p.b_scale + (static_cast<size_t>(e) * (p.b_rows / 128) + 2 * nb) * p.num_kb;
                    // scales of the next K-block are loaded before waiting on this one
                    float sa_n = valid ? arow[0] : 0.0f, wg_n = __ldg(bsb), wu_n = __ldg(bsb + p.num_kb);
                    for (int kb = 0; kb < p.num_kb; kb++) {
                        const float sa = sa_n, sg = sa * wg_n, su = sa * wu_n;
                        if (kb + 1 < p.num_kb) {
                            sa_n = valid ? arow[kb + 1] : 0.0f;
                            wg_n = __ldg(bsb + kb + 1);
                            wu_n = __ldg(bsb + p.num_kb + kb + 1);
                        }
                        const uint32_t acc = u % NBUF;
                        if (!warp_wait(&tfull[acc], (u / NBUF) & 1, limit)) { ok = false; break; }
                        tc_fence_after();
                        if (ew == 0 && lane == 0) KTRACE_BLK(u, 3);
#pragma unroll
                        for (int half = 0; half < 2; half++) {
                            if (!any_valid) break;   // no stored row: skip the readback
                            float vg[32], vu[32];
                            const int c0 = 64 * g + 32 * half;
                            tmem_ld32x2(lane_addr + acc * BN + c0, lane_addr + acc * BN + GU_HALF + c0, vg, vu);
#pragma unroll
                            for (int c = 0; c < 32; c++) {
                                ag[32 * half + c] = fmaf(vg[c], sg, ag[32 * half + c]);
                                au[32 * half + c] = fmaf(vu[c], su, au[32 * half + c]);
                            }
                        }
                        if (ew == 0 && lane == 0) KTRACE_BLK(u, 4);
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) release_acc(&tempty[acc]);
                        if (ew == 0 && lane == 0) KTRACE_BLK(u, 5);
                        if (ew == EPI - 1 && lane == 0) KTRACE_BLK(u, 6);
                        u++;
                    }
                    if (!ok) break;
                    if constexpr (ACT == 5) {
#pragma unroll
                        for (int c = 0; c < 64; c++) {
                            hv[c] = relu_sq(ag[c]);
                            hv2[c] = relu_sq(au[c]);
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 64; c++) hv[c] = glu_e4m3<ACT>(ag[c], au[c], p.act_alpha, p.act_limit);
                    }
                }
                if constexpr (BSCALE == BSCALE_ROW) {
                    // MX requantisation: power-of-two scale per 32 hidden columns (all
                    // inside this thread), codes to the expert's 128-padded rows and
                    // scales to the chunked layout the down GEMM's tensor cores read
                    if (valid) {
                        const long long prow = static_cast<long long>(mi) * 128 + r;
                        // 32-column blocks of this thread: gated NH blocks at hidden
                        // GU_HALF nb + GC g + 32 b; ReLU^2 2 NH blocks, the gate-half
                        // columns at 256 nb + GC g + 32 b, the up half 128 further
                        constexpr int NB = ACT == 5 ? 2 * NH : NH;
                        static_assert(BSCALE != BSCALE_ROW || 32 * NB <= 64, "hidden values held per thread");
#pragma unroll
                        for (int b = 0; b < NB; b++) {
                            const int col = ACT == 5 ? nb * 256 + (b < NH ? GC * g + 32 * b : 128 + GC * g + 32 * (b - NH))
                                                     : nb * GU_HALF + GC * g + 32 * b;
                            float amax = 0.0f;
#pragma unroll
                            for (int c = 0; c < 32; c++) amax = fmaxf(amax, fabsf(hv[32 * b + c]));
                            const int ex = mx_exponent(amax);
                            const float inv = mx_inv_scale(ex);
                            uint32_t w[8];
#pragma unroll
                            for (int c = 0; c < 32; c += 4) {
                                const uint16_t lo = f2_to_e4m3x2(__fmul_rn(hv[32 * b + c], inv), __fmul_rn(hv[32 * b + c + 1], inv));
                                const uint16_t hi = f2_to_e4m3x2(__fmul_rn(hv[32 * b + c + 2], inv), __fmul_rn(hv[32 * b + c + 3], inv));
                                w[c / 4] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
                            }
                            p.hsf[sf_offset(prow, col / 32, p.I / 32)] = static_cast<uint8_t>(ex + 127);
                            uint4* dst = reinterpret_cast<uint4*>(p.hq + prow * p.I + col);
                            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                        }
                    }
                    publish();
                } else {
                // BLOCK128: requantise the 128-column hidden block of this row; the
                // two column groups exchange their partial amax through shared memory.
                // ReLU^2 tiles hold two hidden blocks (the gate-half columns are up
                // rows 256 nb .. +128, the up half the next 128); each is exchanged
                // under its own tag.
#pragma unroll
                for (int blk = 0; blk < (ACT == 5 ? 2 : 1); blk++) {
                    const float (&hb)[64] = (blk == 1) ? hv2 : hv;
                    const int tag = ACT == 5 ? 2 * static_cast<int>(iter) + blk : static_cast<int>(iter);
                    float amax = 0.0f;
#pragma unroll
                    for (int c = 0; c < 64; c++) amax = fmaxf(amax, fabsf(hb[c]));
                    const int par = tag & 1;
                    volatile float* xv = xval;
                    volatile int* xf = xflag;
                    xv[(par * 2 + g) * 128 + r] = amax;
                    __threadfence_block();
                    xf[(par * 2 + g) * 128 + r] = tag + 1;
                    long long t0 = clock64();
                    while (xf[(par * 2 + (1 - g)) * 128 + r] < tag + 1) {
                        if (clock64() - t0 > limit) { ok = false; break; }
                    }
                    if (!ok) break;
                    __threadfence_block();
                    amax = fmaxf(amax, xv[(par * 2 + (1 - g)) * 128 + r]);
                    const float s = __fdiv_rn(amax, 448.0f);
                    if (valid) {
                        uint32_t w[16];
#pragma unroll
                        for (int c = 0; c < 64; c += 4) {
                            uint16_t lo = 0, hi = 0;
                            if (s != 0.0f) {
                                lo = f2_to_e4m3x2(__fdiv_rn(hb[c], s), __fdiv_rn(hb[c + 1], s));
                                hi = f2_to_e4m3x2(__fdiv_rn(hb[c + 2], s), __fdiv_rn(hb[c + 3], s));
                            }
                            w[c / 4] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
                        }
                        const int hblock = ACT == 5 ? 2 * nb + blk : nb;   // 128-column hidden block
                        uint4* dst = reinterpret_cast<uint4*>(p.hq + static_cast<size_t>(row) * p.I + hblock * 128 + 64 * g);
#pragma unroll
                        for (int v4 = 0; v4 < 4; v4++) dst[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
                        if (g == 0) p.hs[static_cast<size_t>(row) * (p.I / 128) + hblock] = s;
                    }
                }
                if (!ok) break;
                }
            } else {
                // ---------------------------------------------------- down
                constexpr int NC = BN / 2;      // columns per thread
                float acc_r[NC];
#pragma unroll
                for (int c = 0; c < NC; c++) acc_r[c] = 0.0f;
                const int n0 = nb * BN + g * NC;
                const bool any_valid = __any_sync(0xffffffffu, valid);
                const float rw = valid ? p.route_w[p.perm[row]] : 0.0f;   // loaded while the MMAs run
                const float* arow = p.a_scale + static_cast<size_t>(valid ? row : 0) * p.a_ld;
                const float* bsb = p.b_scale + (static_cast<size_t>(e) * (p.b_rows / 128) + n0 / 128) * p.num_kb;
                // the scale of the next K-block is loaded before waiting on this one
                float sa_n = valid ? arow[0] : 0.0f;
                if (BSCALE == BSCALE_BLOCK128) sa_n *= __ldg(bsb);
                for (int kb = 0; kb < p.num_kb; kb++) {
                    const float sa = sa_n;
                    if (kb + 1 < p.num_kb) {
                        sa_n = valid ? arow[kb + 1] : 0.0f;
                        if (BSCALE == BSCALE_BLOCK128) sa_n *= __ldg(bsb + kb + 1);
                    }
                    const uint32_t acc = u % NBUF;
                    if (!warp_wait(&tfull[acc], (u / NBUF) & 1, limit)) { ok = false; break; }
                    tc_fence_after();
                    if (!any_valid) {
                        // no stored row: skip the readback
                    } else if constexpr (NC >= 64) {
#pragma unroll
                        for (int ch = 0; ch < NC / 64; ch++) {
                            float v0[32], v1[32];
                            const uint32_t a = lane_addr + acc * BN + g * NC + 64 * ch;
                            tmem_ld32x2(a, a + 32, v0, v1);
#pragma unroll
                            for (int c = 0; c < 32; c++) {
                                acc_r[64 * ch + c] = fmaf(v0[c], sa, acc_r[64 * ch + c]);
                                acc_r[64 * ch + 32 + c] = fmaf(v1[c], sa, acc_r[64 * ch + 32 + c]);
                            }
                        }
                    } else {
                        float v[32];
                        tmem_ld32(lane_addr + acc * BN + g * NC, v);
#pragma unroll
                        for (int c = 0; c < 32; c++) acc_r[c] = fmaf(v[c], sa, acc_r[c]);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) release_acc(&tempty[acc]);
                    u++;
                }
                if (!ok) break;
                store_rows16<NC, BSCALE == BSCALE_ROW>(
                    acc_r, reinterpret_cast<uint32_t*>(smem + S::SPARSE_OFF) + ew * EWF,
                    valid ? p.o + static_cast<size_t>(row) * p.H + n0 : nullptr,
                    p.oe + static_cast<size_t>(row) * (p.H / 32) + n0 / 32,
                    p.b_scale + static_cast<size_t>(e) * p.b_rows + n0, rw, lane);
            }
        }
        if (!ok) report(p.status, ST_TIMEOUT, WHERE_GEMM_EPILOGUE);
    }

    tc_fence_before();
    __syncthreads();
    // a pair leaves together: no arrival or copy may target a CTA that has exited
    if constexpr (PAIR) cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        if constexpr (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
        else tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <int KIND, int BSCALE, bool PROMOTE, int BN, int STAGES, int EPI, int ACT>
__global__ void __launch_bounds__(gemm_threads<EPI, PROMOTE>(), 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    gemm_body<KIND, BSCALE, PROMOTE, BN, STAGES, EPI, ACT>(tmA, tmB, p, p.n_blocks, smem_raw);
}

// The gated FP8_ROW gate/up GEMM, whose mode the dispatch picks from the
// expert histogram (pick_gu_mode): launched as 2-CTA clusters of 16-epilogue-
// warp CTAs; every CTA reads the mode and runs
//   0: the single-CTA body on 256-wide tiles (128 gate + 128 up columns),
//   1: the pair body (M = 256 over two m-tiles of one expert, each CTA loading
//      half of the 256 weight rows),
//   2: the single-CTA body on 128-wide tiles (64 gate + 64 up columns, twice
//      the n-blocks; 8 of the 16 epilogue warps work).
// No host round trip.  p.n_blocks counts the 256-wide n-blocks.
constexpr int GU_PAIR_STAGES = 6;
constexpr int GU_WIDE_STAGES = 4;
constexpr int GU_NARROW_STAGES = 6;
constexpr int gu_poly_smem() {
    constexpr int a = GemmSmem<256, GU_WIDE_STAGES, 16>::TOTAL;
    constexpr int b = GemmSmem<256, GU_PAIR_STAGES, 16, true>::TOTAL;
    constexpr int c = GemmSmem<128, GU_NARROW_STAGES, 16>::TOTAL;
    return a > b ? (a > c ? a : c) : (b > c ? b : c);
}
constexpr int GU_POLY_SMEM = gu_poly_smem();
template <int ACT>
__global__ void __launch_bounds__(gemm_threads<16>(), 1)
    grouped_gemm_gu_poly_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB256,
                                const __grid_constant__ CUtensorMap tmB128, const __grid_constant__ CUtensorMap tmB64,
                                const GemmParams p, const int32_t* cfg) {
    extern __shared__ uint8_t smem_raw[];
    pdl_wait();   // the mode was picked by the dispatch
    const int mode = *cfg;
    if (mode == 1)
        gemm_body<KIND_GATE_UP, BSCALE_ROW, false, 256, GU_PAIR_STAGES, 16, ACT, true>(tmA, tmB128, p, p.n_blocks,
                                                                                       smem_raw);
    else if (mode == 2)
        gemm_body<KIND_GATE_UP, BSCALE_ROW, false, 128, GU_NARROW_STAGES, 16, ACT>(tmA, tmB64, p, 2 * p.n_blocks,
                                                                                   smem_raw);
    else
        gemm_body<KIND_GATE_UP, BSCALE_ROW, false, 256, GU_WIDE_STAGES, 16, ACT>(tmA, tmB256, p, p.n_blocks,
                                                                                 smem_raw);
}

// Down GEMM whose tile width is chosen on the device: the dispatch's scan
// kernel evaluates the wave cost model on the expert histogram and writes the
// choice (0: BN=256, 1: 128, 2: 64) to *cfg; every CTA reads it and runs that
// tile body with the matching weight tensor map.  No host round trip.
constexpr int POLY_SMEM = GemmSmem<256, 4>::TOTAL > GemmSmem<128, 6>::TOTAL
                              ? (GemmSmem<256, 4>::TOTAL > GemmSmem<64, 8>::TOTAL ? GemmSmem<256, 4>::TOTAL
                                                                                 : GemmSmem<64, 8>::TOTAL)
                              : (GemmSmem<128, 6>::TOTAL > GemmSmem<64, 8>::TOTAL ? GemmSmem<128, 6>::TOTAL
                                                                                 : GemmSmem<64, 8>::TOTAL);

template <int BSCALE>
__global__ void __launch_bounds__(gemm_threads<8, true>(), 1)
    down_gemm_poly_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB256,
                          const __grid_constant__ CUtensorMap tmB128, const __grid_constant__ CUtensorMap tmB64,
                          const GemmParams p, const int32_t* cfg) {
    extern __shared__ uint8_t smem_raw[];
    pdl_wait();   // the tile width was picked by the dispatch scan
    const int c = *cfg;
    if (c == 1)
        gemm_body<KIND_DOWN, BSCALE, true, 128, 6>(tmA, tmB128, p, p.H / 128, smem_raw);
    else if (c == 2)
        gemm_body<KIND_DOWN, BSCALE, true, 64, 8>(tmA, tmB64, p, p.H / 64, smem_raw);
    else
        gemm_body<KIND_DOWN, BSCALE, true, 256, 4>(tmA, tmB256, p, p.H / 256, smem_raw);
}

}  // namespace moe
