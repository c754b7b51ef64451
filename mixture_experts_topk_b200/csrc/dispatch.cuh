// dispatch.cuh -- deterministic expert-major dispatch and X quantisation.
//
// LightMoE README ("Grouped GEMM"): rows are contiguous per expert, m_indptr is
// int32 of length E+1, zero-assignment experts are valid; ("MoE training"):
// MoEDispatch returns gather indices, m_indptr and inverse slots.  Pure-Triton
// article: a precomputed block-id -> (expert id, offset) map lets one launch
// run variable-size groups without padding.
//
// Slot of assignment a = t*k + j (row-major order):
//   offsets[e] + #{a' < a : ids[a'] == e}
// computed without atomics on the result: the assignments are cut into chunks
// of 1024; a per-chunk histogram, one scan over (expert, chunk), and inside a
// chunk a per-warp match + per-expert scan over the 32 warps.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int DISPATCH_CHUNK = 1024;
constexpr int TILE_M = 128;

// Wave cost model of the down GEMM's tile width (RaMP abstract: a
// four-parameter wave cost model picks the configuration from the runtime
// expert histogram and depends only on the CTA grid geometry).  Integer
// picoseconds, so the choice is exact and reproducible.  For candidate c with
// BN_c output columns per tile:
//   tiles  = m_tiles * (H / BN_c)
//   t_mma  = ceil(tiles / num_sms) * (I / 128) * (alpha + beta * BN_c)
//   t_load = touched_experts * H * I / (min(tiles, num_sms) * bw_cta)   (weight bytes)
//   cost   = gamma + max(t_mma, t_load)
// The lowest cost wins; equal costs keep the wider tile.
struct PickerParams {
    long long alpha_ps;        // per K-block fixed cost of a tile
    long long beta_ps;         // per K-block cost per output column
    long long bw_cta;          // weight bytes per microsecond one CTA streams
    long long gamma_ps;        // launch constant
    int num_sms, H, I;
    int split_nb;              // n-blocks of a K-splittable down GEMM (0: no split)
    int split_kb;              // its K-blocks
    int o_rows;                // rows of the fp32 down-output buffer
    // gate/up GEMM mode (pick_gu_mode)
    int gu_nb;                 // n-blocks of its 256-wide tiles (0: no choice, mode 0)
    int gu_kb;                 // its K-blocks
    int gu_allow;              // allowed modes: bit 0 wide single, bit 1 pairs, bit 2 narrow
    long long gu_ps[6];        // per-unit cost kb * a + b of each mode, (a, b) in that order, picoseconds
};

// Mode of the gated FP8_ROW gate/up GEMM, chosen from the expert histogram:
// 0 single CTAs on 256-wide tiles (128 gate + 128 up columns), 1 CTA pairs
// (M = 256 over two m-tiles of one expert, the second absent for the last of
// an odd count; num_sms / 2 pairs run at once), 2 single CTAs on 128-wide
// tiles (twice the units, half the weight rows each).  With
// m_tiles = sum_e mt_e and n_odd = #{e : mt_e odd}:
//   c0 = ceil(m_tiles nb / num_sms) (kb a_0 + b_0)
//   c1 = ceil((m_tiles + n_odd) / 2 nb / (num_sms / 2)) (kb a_1 + b_1)
//   c2 = ceil(m_tiles 2 nb / num_sms) (kb a_2 + b_2)
// The cheapest allowed mode wins; ties go to the lower mode.
__host__ __device__ inline int pick_gu_mode(const PickerParams& q, int m_tiles, int n_odd) {
    if (q.gu_nb <= 0 || m_tiles <= 0) return 0;
    const long long ns = q.num_sms, np = q.num_sms / 2;
    const long long u[3] = {static_cast<long long>(m_tiles) * q.gu_nb,
                            static_cast<long long>((m_tiles + n_odd) / 2) * q.gu_nb,
                            static_cast<long long>(m_tiles) * 2 * q.gu_nb};
    const long long slots[3] = {ns, np, ns};
    int best = -1;
    long long best_c = 0;
    for (int m = 0; m < 3; m++) {
        if (!((q.gu_allow >> m) & 1)) continue;
        const long long c = (u[m] + slots[m] - 1) / slots[m] * (q.gu_kb * q.gu_ps[2 * m] + q.gu_ps[2 * m + 1]);
        if (best < 0 || c < best_c) {
            best = m;
            best_c = c;
        }
    }
    return best < 0 ? 0 : best;
}

// Split of the down GEMM's K for small batches: when the (m-tile, n-block)
// units leave SMs idle, each unit's K-blocks are cut into S near-equal ranges
// run by different CTAs, whose fp32 partial rows go to S copies of the output
// rows that the combine adds in fixed order.  Integer rule:
//   units = m_tiles * split_nb,  s_max = min(8, o_rows / A, split_kb / 4)
//   cost(s) = ceil(units s / num_sms) * 840 / s   (rounds of 1/s of a unit)
//   S = the s <= s_max of lowest cost (the smaller on ties) if that cost is at
//   most 4/5 of cost(1), else 1 (a split also costs copies of the output).
__host__ __device__ inline int split_limit(const PickerParams& q, int A) {
    if (q.split_nb <= 0 || A <= 0) return 1;
    int m = q.o_rows / A;
    if (q.split_kb / 4 < m) m = q.split_kb / 4;
    if (m > 8) m = 8;
    return m < 1 ? 1 : m;
}
__host__ __device__ inline int pick_split(const PickerParams& q, int m_tiles, int A) {
    const int smax = split_limit(q, A);
    const long long units = static_cast<long long>(m_tiles) * q.split_nb;
    const long long c1 = (units + q.num_sms - 1) / q.num_sms * 840;
    int S = 1;
    long long best = c1;
    for (int s = 2; s <= smax; s++) {
        const long long c = (units * s + q.num_sms - 1) / q.num_sms * (840 / s);
        if (c < best && 5 * c <= 4 * c1) {
            S = s;
            best = c;
        }
    }
    return S;
}
constexpr int PICK_NUM = 3;
__host__ __device__ constexpr int pick_bn(int c) { return c == 0 ? 256 : (c == 1 ? 128 : 64); }

__device__ __forceinline__ int pick_down_tile(const PickerParams& q, int m_tiles, int touched) {
    int best = 0;
    long long best_cost = 0;
    for (int c = 0; c < PICK_NUM; c++) {
        const long long bn = pick_bn(c);
        const long long tiles = static_cast<long long>(m_tiles) * (q.H / bn);
        const long long waves = (tiles + q.num_sms - 1) / q.num_sms;
        const long long t_mma = waves * (q.I / 128) * (q.alpha_ps + q.beta_ps * bn);
        const long long active = tiles < q.num_sms ? tiles : q.num_sms;
        const long long bytes = static_cast<long long>(touched) * q.H * q.I;
        const long long t_load = active > 0 ? bytes * 1000000LL / (active * q.bw_cta) : 0;
        const long long cost = q.gamma_ps + (t_mma > t_load ? t_mma : t_load);
        if (c == 0 || cost < best_cost) {
            best = c;
            best_cost = cost;
        }
    }
    return best;
}

__global__ void __launch_bounds__(DISPATCH_CHUNK)
    hist_kernel(const int32_t* ids, int A, int E, int32_t* chunk_counts, int32_t* status) {
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_HIST);
    __shared__ int h[256];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int a = blockIdx.x * DISPATCH_CHUNK + threadIdx.x;
    if (a < A) {
        const int e = ids[a];
        if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) atomicAdd(&h[e], 1);
        else report(status, ST_BOUNDS, WHERE_DISPATCH);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_counts[blockIdx.x * E + e] = h[e];
}

// One CTA: counts, offsets (exclusive scan), per-chunk bases (written over the
// chunk counts), the row-tile table (expert, first row) in expert order, and
// tile_ptr[e] = index of expert e's first row tile (may be null), and the down
// GEMM's tile choice and K split from the histogram (pick_out[0], pick_out[1];
// Copy n 4-byte words with the whole CTA: 16-byte accesses when both ends and
// n allow them, each thread's 8 loads issued before any of its stores, so a
// chain of single-word round trips never forms.
__device__ __forceinline__ void stage_words(int32_t* dst, const int32_t* src, int n) {
    const bool vec = (n % 4 == 0) && ((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) % 16 == 0);
    if (vec) {
        const int n4 = n / 4;
        const int4* s4 = reinterpret_cast<const int4*>(src);
        int4* d4 = reinterpret_cast<int4*>(dst);
        for (int b = threadIdx.x; b < n4; b += 8 * blockDim.x) {
            int4 v[8];
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const int i = b + j * blockDim.x;
                if (i < n4) v[j] = s4[i];
            }
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const int i = b + j * blockDim.x;
                if (i < n4) d4[i] = v[j];
            }
        }
    } else {
        for (int b = threadIdx.x; b < n; b += 8 * blockDim.x) {
            int v[8];
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const int i = b + j * blockDim.x;
                if (i < n) v[j] = src[i];
            }
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const int i = b + j * blockDim.x;
                if (i < n) dst[i] = v[j];
            }
        }
    }
}

// shared memory of scan_kernel: the chunk counts of the largest batch
// (131072 assignments = 128 chunks of 1024, at most 256 experts)
constexpr int SCAN_SMEM_MAX = 128 * 256 * 4;

// may be null).  One exclusive block scan over experts of the packed pair
// (count, row tiles): count < 2^20, so count + (tiles << 20) cannot carry.
// The chunk counts ([nchunks][E], at most 128 KB) are staged in shared memory
// with coalesced loads, summed and scanned there, and written back as bases,
// so no thread walks a chain of dependent global loads.
__global__ void __launch_bounds__(256) scan_kernel(int32_t* chunk_counts, int nchunks, int E, int32_t* counts,
                                                   int32_t* offsets, int32_t* tiles, int32_t* num_tiles,
                                                   int32_t* tile_ptr, int32_t* pick_out, PickerParams pq,
                                                   int32_t* gu_done) {
    extern __shared__ int s_cc[];   // [nchunks][E]
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_SCAN);
    __shared__ int warp_tot[8];
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    const int ncc = nchunks * E;
    stage_words(s_cc, chunk_counts, ncc);
    __syncthreads();
    int c = 0;
    if (e < E) {
        for (int ch = 0; ch < nchunks; ch++) c += s_cc[ch * E + e];
    }
    const int nt_e = (c + TILE_M - 1) / TILE_M;
    const int packed = c + (nt_e << 20);
    int inc = packed;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += n;
    }
    if (lane == 31) warp_tot[warp] = inc;
    const int touched = __syncthreads_count(e < E && c > 0);
    const int n_odd = __syncthreads_count(e < E && (nt_e & 1));
    if (warp == 0) {
        int w = lane < 8 ? warp_tot[lane] : 0;
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += n;
        }
        if (lane < 8) warp_tot[lane] = w;
    }
    __syncthreads();
    const int excl = (warp ? warp_tot[warp - 1] : 0) + inc - packed;
    const int total = warp_tot[7];
    const int off_e = excl & 0xFFFFF, tptr_e = excl >> 20;
    const int A = total & 0xFFFFF, trun = total >> 20;
    if (e == 0) {
        offsets[E] = A;
        *num_tiles = trun;
        if (tile_ptr) tile_ptr[E] = trun;
        if (pick_out) {
            pick_out[0] = pick_down_tile(pq, trun, touched);
            pick_out[1] = pick_split(pq, trun, A);
            pick_out[2] = pick_gu_mode(pq, trun, n_odd);
        }
    }
    if (e < E) {
        counts[e] = c;
        offsets[e] = off_e;
        if (gu_done) gu_done[e] = 0;
        if (tile_ptr) tile_ptr[e] = tptr_e;
        int run = off_e;
        for (int ch = 0; ch < nchunks; ch++) {
            const int v = s_cc[ch * E + e];
            s_cc[ch * E + e] = run;
            run += v;
        }
        for (int i = 0; i < nt_e; i++) {
            tiles[2 * (tptr_e + i)] = e;
            tiles[2 * (tptr_e + i) + 1] = off_e + TILE_M * i;
        }
    }
    __syncthreads();
    stage_words(chunk_counts, s_cc, ncc);
}

__global__ void __launch_bounds__(DISPATCH_CHUNK)
    rank_kernel(const int32_t* ids, int A, int E, const int32_t* chunk_base, int32_t* perm, int32_t* inv) {
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_RANK);
    __shared__ int wc[32][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < 32 * 256; i += blockDim.x) wc[i >> 8][i & 255] = 0;
    __syncthreads();
    const int a = blockIdx.x * DISPATCH_CHUNK + threadIdx.x;
    int e = (a < A) ? ids[a] : -1;
    const bool valid = static_cast<unsigned>(e) < static_cast<unsigned>(E);
    if (!valid) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (valid && rank == 0) wc[warp][e] = __popc(peers);
    __syncthreads();
    if (threadIdx.x < E) {
        int run = chunk_base[blockIdx.x * E + threadIdx.x];
        for (int w = 0; w < 32; w++) {
            const int v = wc[w][threadIdx.x];
            wc[w][threadIdx.x] = run;
            run += v;
        }
    }
    __syncthreads();
    if (a < A) {
        if (valid) {
            const int slot = wc[warp][e] + rank;
            perm[slot] = a;
            inv[a] = slot;
        } else {
            inv[a] = -1;
        }
    }
}

// Small batches (A <= DISPATCH_CHUNK assignments, one chunk): histogram,
// scan, tile table, tile choice and stable ranks in one 1024-thread CTA, with
// the same results as hist_kernel + scan_kernel + rank_kernel on one chunk:
// thread a takes assignment a; a warp match gives its rank among equal ids of
// its warp; per-(warp, expert) counts are summed and scanned over experts
// (count + (row tiles << 20), as in scan_kernel) and then over warps.
__global__ void __launch_bounds__(DISPATCH_CHUNK) dispatch_small_kernel(
    const int32_t* ids, int A, int E, int32_t* counts, int32_t* offsets, int32_t* tiles, int32_t* num_tiles,
    int32_t* tile_ptr, int32_t* pick_out, PickerParams pq, int32_t* perm, int32_t* inv, int32_t* status,
    int32_t* gu_done) {
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_DISPATCH_SMALL);
    __shared__ int wc[32][256];
    __shared__ int warp_tot[8];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < 32 * 256; i += blockDim.x) wc[i >> 8][i & 255] = 0;
    __syncthreads();
    int e = (tid < A) ? ids[tid] : -1;
    const bool valid = static_cast<unsigned>(e) < static_cast<unsigned>(E);
    if (tid < A && !valid) report(status, ST_BOUNDS, WHERE_DISPATCH);
    if (!valid) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (valid && rank == 0) wc[warp][e] = __popc(peers);
    __syncthreads();
    // per-expert totals and the packed exclusive scan (threads 0..255 = warps 0..7)
    int c = 0;
    if (tid < E)
        for (int w = 0; w < 32; w++) c += wc[w][tid];
    const int nt_e = (c + TILE_M - 1) / TILE_M;
    const int packed = c + (nt_e << 20);
    int inc = packed;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += n;
    }
    if (warp < 8 && lane == 31) warp_tot[warp] = inc;
    const int touched = __syncthreads_count(tid < E && c > 0);
    const int n_odd = __syncthreads_count(tid < E && (nt_e & 1));
    if (warp == 0) {
        int w = lane < 8 ? warp_tot[lane] : 0;
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += n;
        }
        if (lane < 8) warp_tot[lane] = w;
    }
    __syncthreads();
    if (tid < 256) {
        const int excl = (warp ? warp_tot[warp - 1] : 0) + inc - packed;
        const int total = warp_tot[7];
        const int off_e = excl & 0xFFFFF, tptr_e = excl >> 20;
        if (tid == 0) {
            offsets[E] = total & 0xFFFFF;
            *num_tiles = total >> 20;
            tile_ptr[E] = total >> 20;
            pick_out[0] = pick_down_tile(pq, total >> 20, touched);
            pick_out[1] = pick_split(pq, total >> 20, total & 0xFFFFF);
            pick_out[2] = pick_gu_mode(pq, total >> 20, n_odd);
        }
        if (tid < E) {
            counts[tid] = c;
            offsets[tid] = off_e;
            gu_done[tid] = 0;
            tile_ptr[tid] = tptr_e;
            for (int i = 0; i < nt_e; i++) {
                tiles[2 * (tptr_e + i)] = tid;
                tiles[2 * (tptr_e + i) + 1] = off_e + TILE_M * i;
            }
            // per-warp bases of this expert's slots, warps in order
            int run = off_e;
            for (int w = 0; w < 32; w++) {
                const int v = wc[w][tid];
                wc[w][tid] = run;
                run += v;
            }
        }
    }
    __syncthreads();
    if (tid < A) {
        if (valid) {
            const int slot = wc[warp][e] + rank;
            perm[slot] = tid;
            inv[tid] = slot;
        } else {
            inv[tid] = -1;
        }
    }
}

// Quantise each token row of X once and write it to the k slots of its
// assignments (LightMoE README: BF16 input quantisation inside the layer).
// FP8_ROW: s = amax/448 over the row; BLOCK128: per 128 columns;
// q = e4m3(x / s) with correctly rounded division, q = 0 when s == 0.
// One warp per token; lane l handles columns 256 i + 8 l .. +8.
template <int FMT>
__global__ void __launch_bounds__(256) quant_scatter_kernel(const __nv_bfloat16* x, int T, int H, int k,
                                                            const int32_t* inv, uint8_t* xq, float* xs) {
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_QUANT);
    const int lane = threadIdx.x & 31;
    const int nI = H >> 8;
    for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < T; t += gridDim.x * 8) {
        int slot[8];
#pragma unroll
        for (int j = 0; j < 8; j++) slot[j] = (j < k) ? inv[static_cast<size_t>(t) * k + j] : -1;
        const __nv_bfloat16* xr = x + static_cast<size_t>(t) * H;
        float s_row = 0.0f;
        if (FMT == 0) {
            float amax = 0.0f;
            for (int i = 0; i < nI; i++) {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(xr + 256 * i + 8 * lane));
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; q++) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(u[q])), fabsf(bf16_hi(u[q]))));
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            s_row = __fdiv_rn(amax, 448.0f);
#pragma unroll
            for (int j = 0; j < 8; j++)
                if (j == lane && slot[j] >= 0) xs[slot[j]] = s_row;
        }
        for (int i = 0; i < nI; i++) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(xr + 256 * i + 8 * lane));
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
            float s = s_row;
            if (FMT == 1) {
                float amax = 0.0f;
#pragma unroll
                for (int q = 0; q < 4; q++) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(u[q])), fabsf(bf16_hi(u[q]))));
#pragma unroll
                for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
                s = __fdiv_rn(amax, 448.0f);
                if ((lane & 15) == 0) {
#pragma unroll
                    for (int j = 0; j < 8; j++)
                        if (slot[j] >= 0) xs[static_cast<size_t>(slot[j]) * (H >> 7) + 2 * i + (lane >> 4)] = s;
                }
            }
            uint32_t packed[2];
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const float a = bf16_lo(u[q]), b = bf16_hi(u[q]);
                const uint16_t c = (s == 0.0f) ? static_cast<uint16_t>(0)
                                               : f2_to_e4m3x2(__fdiv_rn(a, s), __fdiv_rn(b, s));
                if (q & 1) packed[q >> 1] |= static_cast<uint32_t>(c) << 16;
                else packed[q >> 1] = c;
            }
#pragma unroll
            for (int j = 0; j < 8; j++)
                if (slot[j] >= 0)
                    *reinterpret_cast<uint2*>(xq + static_cast<size_t>(slot[j]) * H + 256 * i + 8 * lane) =
                        make_uint2(packed[0], packed[1]);
        }
    }
}

// Quantise token row t with one 256-thread CTA and write it to the slots
// slot[0..k) (-1: none).  Thread i handles columns 8 (i + 256 m); a 128-column
// block is 16 consecutive lanes, the row amax (FP8_ROW) is a warp then CTA
// maximum.  Same operations per element as quant_scatter_kernel.  s_amax: 8
// floats of shared memory.
template <int FMT>
__device__ __forceinline__ void quant_row_to_slots(const __nv_bfloat16* x, int t, int H, int k, const int* slot,
                                                   uint8_t* xq, float* xs, float* s_amax) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const __nv_bfloat16* xr = x + static_cast<size_t>(t) * H;
    float s_row = 0.0f;
    if (FMT == 0) {
        float amax = 0.0f;
        for (int m = 0; 8 * (tid + 256 * m) < H; m++) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(xr + 8 * (tid + 256 * m)));
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; q++) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(u[q])), fabsf(bf16_hi(u[q]))));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (lane == 0) s_amax[warp] = amax;
        __syncthreads();
        amax = s_amax[0];
#pragma unroll
        for (int w = 1; w < 8; w++) amax = fmaxf(amax, s_amax[w]);
        __syncthreads();   // s_amax is rewritten for the next token
        s_row = __fdiv_rn(amax, 448.0f);
#pragma unroll
        for (int j = 0; j < 8; j++)
            if (j < k && j == tid && slot[j] >= 0) xs[slot[j]] = s_row;
    }
    for (int m = 0; 8 * (tid + 256 * m) < H; m++) {
        const int c0 = 8 * (tid + 256 * m);
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(xr + c0));
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
        float s = s_row;
        if (FMT == 1) {
            float amax = 0.0f;
#pragma unroll
            for (int q = 0; q < 4; q++) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(u[q])), fabsf(bf16_hi(u[q]))));
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            s = __fdiv_rn(amax, 448.0f);
            if ((lane & 15) == 0) {
#pragma unroll
                for (int j = 0; j < 8; j++)
                    if (j < k && slot[j] >= 0) xs[static_cast<size_t>(slot[j]) * (H >> 7) + (c0 >> 7)] = s;
            }
        }
        uint32_t packed[2];
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const float a = bf16_lo(u[q]), b = bf16_hi(u[q]);
            const uint16_t c = (s == 0.0f) ? static_cast<uint16_t>(0)
                                           : f2_to_e4m3x2(__fdiv_rn(a, s), __fdiv_rn(b, s));
            if (q & 1) packed[q >> 1] |= static_cast<uint32_t>(c) << 16;
            else packed[q >> 1] = c;
        }
#pragma unroll
        for (int j = 0; j < 8; j++)
            if (j < k && slot[j] >= 0)
                *reinterpret_cast<uint2*>(xq + static_cast<size_t>(slot[j]) * H + c0) = make_uint2(packed[0], packed[1]);
    }
}

// Small batches: the quantisation with one 256-thread CTA per token, so a
// row's loads are spread over 8 warps.
template <int FMT>
__global__ void __launch_bounds__(256) quant_scatter_row_kernel(const __nv_bfloat16* x, int T, int H, int k,
                                                                const int32_t* inv, uint8_t* xq, float* xs) {
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_QUANT_ROW);
    __shared__ float s_amax[8];
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        int slot[8];
#pragma unroll
        for (int j = 0; j < 8; j++) slot[j] = (j < k) ? inv[static_cast<size_t>(t) * k + j] : -1;
        quant_row_to_slots<FMT>(x, t, H, k, slot, xq, xs, s_amax);
    }
}

// Small batches (A <= DISPATCH_CHUNK assignments): the dispatch and the X
// quantisation in one launch, one 256-thread CTA per token.  Every CTA reads
// all A ids and derives the histogram, the offsets and the slots of its own
// token's k assignments itself -- slot of a = offsets[e] + #{a' < a : ids[a'] ==
// e}, the stable order of rank_kernel -- so the CTAs need nothing from one
// another.  CTA 0 also writes the counts, offsets, row-tile table, tile
// pointers and picks (the packed (count, tiles) scan of scan_kernel) and resets
// the per-expert gate/up counters.  Then the CTA quantises its token's row as
// quant_scatter_row_kernel does.  Same results as dispatch_small_kernel +
// quant_scatter_row_kernel.
template <int FMT>
__global__ void __launch_bounds__(256) dispatch_quant_small_kernel(
    const int32_t* ids, int A, int E, int T, int H, int k, const __nv_bfloat16* x, int32_t* counts, int32_t* offsets,
    int32_t* tiles, int32_t* num_tiles, int32_t* tile_ptr, int32_t* pick_out, PickerParams pq, int32_t* perm,
    int32_t* inv, int32_t* status, int32_t* gu_done, uint8_t* xq, float* xs) {
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_DISPATCH_SMALL);
    __shared__ int s_ids[DISPATCH_CHUNK];
    __shared__ int s_cnt[256];
    __shared__ int s_off[256];
    __shared__ int warp_tot[8];
    __shared__ int s_slot[8];
    __shared__ float s_amax[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int a = tid; a < A; a += 256) s_ids[a] = ids[a];
    s_cnt[tid] = 0;
    __syncthreads();
    for (int a = tid; a < A; a += 256) {
        const int e = s_ids[a];
        if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) atomicAdd(&s_cnt[e], 1);
        else if (blockIdx.x == 0) report(status, ST_BOUNDS, WHERE_DISPATCH);
    }
    __syncthreads();
    // exclusive scan over experts of the packed (count, row tiles), as scan_kernel
    const int c = tid < E ? s_cnt[tid] : 0;
    const int nt_e = (c + TILE_M - 1) / TILE_M;
    const int packed = c + (nt_e << 20);
    int inc = packed;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += n;
    }
    if (lane == 31) warp_tot[warp] = inc;
    const int touched = __syncthreads_count(tid < E && c > 0);
    const int n_odd = __syncthreads_count(tid < E && (nt_e & 1));
    if (warp == 0) {
        int w = lane < 8 ? warp_tot[lane] : 0;
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += n;
        }
        if (lane < 8) warp_tot[lane] = w;
    }
    __syncthreads();
    const int excl = (warp ? warp_tot[warp - 1] : 0) + inc - packed;
    const int total = warp_tot[7];
    const int off_e = excl & 0xFFFFF, tptr_e = excl >> 20;
    s_off[tid] = off_e;
    if (blockIdx.x == 0) {
        if (tid == 0) {
            offsets[E] = total & 0xFFFFF;
            *num_tiles = total >> 20;
            tile_ptr[E] = total >> 20;
            pick_out[0] = pick_down_tile(pq, total >> 20, touched);
            pick_out[1] = pick_split(pq, total >> 20, total & 0xFFFFF);
            pick_out[2] = pick_gu_mode(pq, total >> 20, n_odd);
        }
        if (tid < E) {
            counts[tid] = c;
            offsets[tid] = off_e;
            gu_done[tid] = 0;
            tile_ptr[tid] = tptr_e;
            for (int i = 0; i < nt_e; i++) {
                tiles[2 * (tptr_e + i)] = tid;
                tiles[2 * (tptr_e + i) + 1] = off_e + TILE_M * i;
            }
        }
    }
    __syncthreads();
    // the slots of this CTA's token: warp j ranks assignment t k + j among the
    // earlier ones with the same expert
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        if (warp < k) {
            const int a = t * k + warp;
            const int e = s_ids[a];
            const bool valid = static_cast<unsigned>(e) < static_cast<unsigned>(E);
            int cnt = 0;
            if (valid)
                for (int a2 = lane; a2 < a; a2 += 32) cnt += s_ids[a2] == e;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
            if (lane == 0) {
                const int slot = valid ? s_off[e] + cnt : -1;
                s_slot[warp] = slot;
                inv[a] = slot;
                if (valid) perm[slot] = a;
            }
        }
        __syncthreads();
        int slot[8];
#pragma unroll
        for (int j = 0; j < 8; j++) slot[j] = j < k ? s_slot[j] : -1;
        __syncthreads();   // s_slot is rewritten for the next token
        quant_row_to_slots<FMT>(x, t, H, k, slot, xq, xs, s_amax);
    }
}

// y[t] = bf16(sum_j sum_s o[s][inv[t k + j]]) in fixed (j, s) order with fp32
// accumulation.  o holds the down GEMM's weighted rows in fp16 with a power-of-
// two scale per 32 columns (value = fp16 * 2^(oe - 15), exact in fp32), in S
// copies of A rows when the down GEMM split its K (S from the dispatch's pick,
// clamped to [1, s_max]), so the only rounding to bf16 is the final one.
// A thread takes 16 columns (32 bytes of each row, one exponent) of a group of
// G = max(1, 8 / k) consecutive tokens, so that up to 8 rows' loads are in
// flight per thread whatever k is: all loads of the group are issued before
// the first is used (a load followed by its use would keep one row in flight).
constexpr int COMBINE_COLS = 16;
constexpr int COMBINE_THREADS = 128;
__host__ __device__ constexpr int combine_group(int k) { return k >= 8 ? 1 : 8 / k; }
__global__ void __launch_bounds__(COMBINE_THREADS) combine_kernel(const uint16_t* o, const int8_t* oe,
                                                                  const int32_t* inv, int T, int H, int k,
                                                                  const int32_t* split, int s_max, __nv_bfloat16* y) {
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_COMBINE);
    const int S = split ? min(max(*split, 1), s_max) : 1;
    const size_t copy = static_cast<size_t>(T) * k;   // rows per copy
    const int HB = H >> 5;                            // exponent bytes per row
    const int G = combine_group(k);
    constexpr int SPAN = COMBINE_COLS * COMBINE_THREADS;
    // CTA (x, y): token groups x, x + gridDim.x, ..., columns [SPAN y, SPAN y + SPAN)
    const int c_end = min(H, SPAN * (static_cast<int>(blockIdx.y) + 1));
    for (int t0 = blockIdx.x * G; t0 < T; t0 += gridDim.x * G) {
        // row r of the group: token t0 + r / k, its j = r % k
        int slot[8];
#pragma unroll
        for (int r = 0; r < 8; r++) {
            const int g = r / k, j = r - g * k;
            slot[r] = (g < G && t0 + g < T) ? inv[static_cast<size_t>(t0 + g) * k + j] : -1;
        }
        for (int c0 = SPAN * blockIdx.y + COMBINE_COLS * threadIdx.x; c0 < c_end; c0 += SPAN) {
            uint4 q[8][2];
            int8_t ex[8];
            if (S == 1) {
#pragma unroll
                for (int r = 0; r < 8; r++) {
                    if (slot[r] < 0) continue;
                    const size_t row = static_cast<size_t>(slot[r]);
                    const uint4* src = reinterpret_cast<const uint4*>(o + row * H + c0);
                    q[r][0] = src[0];
                    q[r][1] = src[1];
                    ex[r] = oe[row * HB + (c0 >> 5)];
                }
            }
            float acc[16];
            auto add = [&](const uint4& q0, const uint4& q1, int8_t e8) {
                const float sc = __int_as_float((127 - 15 + e8) << 23);
                const uint32_t wq[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wq[i]));
                    acc[2 * i] += f.x * sc;
                    acc[2 * i + 1] += f.y * sc;
                }
            };
#pragma unroll
            for (int r = 0; r < 8; r++) {
                const int g = r / k, j = r - g * k;
                if (g >= G || t0 + g >= T) continue;
                if (j == 0) {
#pragma unroll
                    for (int i = 0; i < 16; i++) acc[i] = 0.0f;
                }
                if (slot[r] >= 0) {
                    if (S == 1) {
                        add(q[r][0], q[r][1], ex[r]);
                    } else {
                        for (int sp = 0; sp < S; sp++) {
                            const size_t row = static_cast<size_t>(sp) * copy + slot[r];
                            const uint4* src = reinterpret_cast<const uint4*>(o + row * H + c0);
                            add(src[0], src[1], oe[row * HB + (c0 >> 5)]);
                        }
                    }
                }
                if (j == k - 1) {
                    uint32_t w[8];
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
                        w[i] = *reinterpret_cast<const uint32_t*>(&b2);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(y + static_cast<size_t>(t0 + g) * H + c0);
                    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
        }
    }
}

// Interleave gate and up rows in groups of G: packed row R of expert e takes
// gate row (R / 2G) G + R % 2G when R % 2G < G, else up row (R / 2G) G + R % 2G - G.
// Rows are row_words 4-byte words long.
__global__ void interleave_rows_kernel(const uint32_t* gate, const uint32_t* up, uint32_t* dst, int E,
                                       int rows_per_proj, int G, int row_words) {
    const long long total_rows = 2LL * E * rows_per_proj;
    for (long long R = blockIdx.x; R < total_rows; R += gridDim.x) {
        const int e = static_cast<int>(R / (2 * rows_per_proj));
        const int r = static_cast<int>(R % (2 * rows_per_proj));
        const int grp = r / (2 * G), within = r % (2 * G);
        const uint32_t* src = (within < G) ? gate : up;
        const long long sr = static_cast<long long>(e) * rows_per_proj + grp * G + (within < G ? within : within - G);
        for (int c = threadIdx.x; c < row_words; c += blockDim.x) dst[R * row_words + c] = src[sr * row_words + c];
    }
}


// ------------------------------------------------------------------ NVFP4
// LightMoE README ("Standalone GEMM", "MoE inference"): NVFP4 = packed E2M1
// values, E4M3 scale factors per 16 elements, one fp32 scale per tensor; the
// layer quantises its BF16 input itself.
//
// Global scale of X: g = amax(|X|) / (448 * 6).  amax as the bit pattern of a
// non-negative float, so an integer max gives the float max (order-free).
__global__ void __launch_bounds__(256) amax_kernel(const __nv_bfloat16* x, long long n8, int32_t* amax_bits) {
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_AMAX);
    float m = 0.0f;
    for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n8; i += 256LL * gridDim.x) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(x) + i);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; q++) m = fmaxf(m, fmaxf(fabsf(bf16_lo(u[q])), fabsf(bf16_hi(u[q]))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_int(m));
}

// NVFP4 quantisation of X rows, scattered to the rows of the assignments in the
// 128-padded expert-major layout: assignment slot s of expert e goes to row
// tile_ptr[e] * 128 + (s - offsets[e]).  Per 16-block: sb = e4m3((amax/6)/g),
// d = value(sb) * g, q = e2m1(x / d) (all correctly rounded fp32; q = 0 when
// d == 0).  One warp per token; lane l holds columns 256 i + 8 l .. +8, so a
// 16-block is lanes (l, l^1).
__global__ void __launch_bounds__(256) quant_scatter_nvfp4_kernel(
    const __nv_bfloat16* x, int T, int H, int k, const int32_t* ids, const int32_t* inv, const int32_t* offsets,
    const int32_t* tile_ptr, const int32_t* amax_bits, uint8_t* xq, uint8_t* xsf) {
    pdl_wait();
    pdl_trigger();
    KTRACE(TR_QUANT_FP4);
    const int lane = threadIdx.x & 31;
    const int nI = H >> 8;
    const float g = __fdiv_rn(__int_as_float(*amax_bits), 2688.0f);
    for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < T; t += gridDim.x * 8) {
        long long prow[8];
#pragma unroll
        for (int j = 0; j < 8; j++) {
            prow[j] = -1;
            if (j < k) {
                const int s = inv[static_cast<size_t>(t) * k + j];
                const int e = ids[static_cast<size_t>(t) * k + j];
                if (s >= 0) prow[j] = static_cast<long long>(tile_ptr[e]) * 128 + (s - offsets[e]);
            }
        }
        const __nv_bfloat16* xr = x + static_cast<size_t>(t) * H;
        for (int i = 0; i < nI; i++) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(xr + 256 * i + 8 * lane));
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
            float f[8];
#pragma unroll
            for (int q = 0; q < 4; q++) {
                f[2 * q] = bf16_lo(u[q]);
                f[2 * q + 1] = bf16_hi(u[q]);
            }
            float amax = 0.0f;
#pragma unroll
            for (int q = 0; q < 8; q++) amax = fmaxf(amax, fabsf(f[q]));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            uint8_t sb = 0;
            float d = 0.0f;
            if (g > 0.0f) {
                sb = f_to_e4m3(__fdiv_rn(__fdiv_rn(amax, 6.0f), g));
                d = __fmul_rn(e4m3_to_f(sb), g);
            }
            uint32_t packed = 0;
            if (d != 0.0f) {
#pragma unroll
                for (int q = 0; q < 4; q++)
                    packed |= static_cast<uint32_t>(f2_to_e2m1x2(__fdiv_rn(f[2 * q], d), __fdiv_rn(f[2 * q + 1], d)))
                              << (8 * q);
            }
            const int c = 16 * i + (lane >> 1);   // scale column of this lane's block
#pragma unroll
            for (int j = 0; j < 8; j++) {
                if (prow[j] < 0) continue;
                *reinterpret_cast<uint32_t*>(xq + prow[j] * (H / 2) + 128 * i + 4 * lane) = packed;
                if ((lane & 1) == 0) xsf[sf_offset(prow[j], c, H / 16)] = sb;
            }
        }
    }
}

// Scale factors of weights [E][rows][K/16] e4m3 -> the chunked layout per
// expert (rows a multiple of 128).  With `interleave` the destination row R of
// expert e takes source row (R / 2G) G + R % 2G of gate (R % 2G < G) or up.
__global__ void pack_sf_kernel(const uint8_t* gate, const uint8_t* up, uint8_t* dst, int E, int rows_per_proj,
                               int G, int sf_cols, int interleave) {
    const int dst_rows = interleave ? 2 * rows_per_proj : rows_per_proj;
    const long long total = static_cast<long long>(E) * dst_rows * sf_cols;
    for (long long i = blockIdx.x * 256LL + threadIdx.x; i < total; i += 256LL * gridDim.x) {
        const int c = static_cast<int>(i % sf_cols);
        const long long er = i / sf_cols;
        const int e = static_cast<int>(er / dst_rows), R = static_cast<int>(er % dst_rows);
        const uint8_t* src = gate;
        int sr = R;
        if (interleave) {
            const int grp = R / (2 * G), within = R % (2 * G);
            src = within < G ? gate : up;
            sr = grp * G + (within < G ? within : within - G);
        }
        const uint8_t v = src[(static_cast<long long>(e) * rows_per_proj + sr) * sf_cols + c];
        dst[static_cast<size_t>(e) * dst_rows * sf_cols + sf_offset(R, c, sf_cols)] = v;
    }
}

}  // namespace moe
