// common.cuh -- device helpers shared by the kernels of the routed MoE layer:
// status reporting, bounded mbarrier waits, TMA loads and tcgen05 (5th-gen
// tensor core) instructions for sm_100a, as inline PTX.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// status[0] holds the first error any kernel recorded, status[1] where.
enum : int { ST_OK = 0, ST_TIMEOUT = 5, ST_BOUNDS = 6 };
enum : int {
    WHERE_GEMM_PRODUCER = 1, WHERE_GEMM_MMA = 2, WHERE_GEMM_EPILOGUE = 3,
    WHERE_DISPATCH = 4, WHERE_ROUTER = 5, WHERE_COMBINE = 6, WHERE_GEMM_SCHEDULE = 7
};

__device__ __forceinline__ void report(int32_t* status, int code, int where) {
    if (atomicCAS(status, 0, code) == 0) status[1] = where;
}

// ------------------------------------------------------------------ programmatic dependent launch
// Every kernel of the layer calls pdl_wait() before its first global-memory
// access: it returns once the preceding kernel in the stream has completed and
// its writes are visible (at once for a launch without the PDL attribute).
// Since each kernel waits for its predecessor before it can complete, the
// chain orders every kernel after all earlier ones.  pdl_trigger() lets the
// next kernel be scheduled now, so its launch and prologue (barrier init, TMEM
// allocation, tensor-map prefetch) overlap this kernel's tail.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ optional timeline trace
// Built only with -DMOE_TRACE (off in the library): KTRACE(id) at the top of a
// kernel body records the global timer of its first CTA's entry and of its
// last warp's exit in slot id, for a per-kernel timeline of one layer step
// as it runs in the stream (PDL overlap included).  moe_trace_clear() and
// moe_trace_read() in the C API of such a build reset and fetch the slots.
#ifdef MOE_TRACE
constexpr int TRACE_SLOTS = 32;
__device__ unsigned long long moe_trace_buf[2 * TRACE_SLOTS];
__device__ __forceinline__ unsigned long long global_timer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
struct TraceScope {
    int id;
    __device__ explicit TraceScope(int i) : id(i) {
        if (threadIdx.x == 0) atomicMin(&moe_trace_buf[2 * id], global_timer());
    }
    __device__ ~TraceScope() {
        if ((threadIdx.x & 31) == 0) atomicMax(&moe_trace_buf[2 * id + 1], global_timer());
    }
};
#define KTRACE(id) ::moe::TraceScope moe_trace_scope_(id)
// Per-K-block events of CTA 0 in the promoted (FP8_BLOCK128) GEMMs, for the
// first TRACE_BLKS accumulation units i: k = 0 MMA thread got a free
// accumulator, 1 it got the filled stage, 2 it committed the MMAs, 3 epilogue
// warp 0 saw the accumulator full, 4 it had read and added it, 5 it released
// it, 6 the last epilogue warp released it, 7 the producer issued the stage.
constexpr int TRACE_BLKS = 96;
__device__ unsigned long long moe_trace_blk[TRACE_BLKS][8];
#define KTRACE_BLK(i, k) \
    do { if (blockIdx.x == 0 && (i) < ::moe::TRACE_BLKS) ::moe::moe_trace_blk[(i)][(k)] = ::moe::global_timer(); } while (0)
#else
#define KTRACE(id) ((void)0)
#define KTRACE_BLK(i, k) ((void)0)
#endif
enum : int {
    TR_ROUTER = 0, TR_ROUTER_SMALL = 1, TR_TOPK = 2, TR_ROUTER_FUSED = 3, TR_HIST = 4, TR_SCAN = 5,
    TR_RANK = 6, TR_DISPATCH_SMALL = 7, TR_QUANT = 8, TR_QUANT_ROW = 9, TR_COMBINE = 10, TR_AMAX = 11,
    TR_QUANT_FP4 = 12, TR_GEMM = 13, TR_MX_DOWN = 14, TR_FP4 = 15
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Limit of the waits for a CTA's own copies and MMAs in flight (the drain
// before it exits or frees TMEM).  Those always finish, so this limit is fixed;
// the configurable limit applies to the waits between roles and CTAs.
constexpr long long DRAIN_LIMIT = 2000000000LL;

// Wait until the phase with the given parity completed; give up after
// `limit` clock cycles (returns false, the caller records ST_TIMEOUT).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) return false;
    }
    return true;
}

// Acquire load of a counter another CTA releases (after its generic-proxy
// stores, a fence.proxy.async and a __threadfence), for a wait that gates this
// CTA's TMA reads of those stores.
__device__ __forceinline__ int ld_acquire(const int32_t* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* tm) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm)) : "memory");
}
// 2D tiled load of box {x .. x+box0, y .. y+box1} into shared memory, completion
// counted in bytes on `bar`.  No multicast.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// L2 eviction priority of a load (createpolicy): expert weight tiles that one
// m-tile alone reads go in as evict_first, so streaming them does not push the
// layer's small buffers and kernels' code out of L2; tiles that several
// m-tiles read keep the normal priority for their reuse.
__device__ __forceinline__ uint64_t l2_policy(bool evict_first) {
    uint64_t pol;
    if (evict_first)
        asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    else
        asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// evict_last: lines that several CTAs read at different times stay in L2
// ahead of normal and evict_first lines
__device__ __forceinline__ uint64_t l2_policy_keep() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// tma_load_2d with an L2 cache policy
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* tm, uint64_t* bar, int x, int y,
                                                 uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(pol)
        : "memory");
}

// Plain (non-tensor) bulk copy global -> shared, completion counted in bytes
// on `bar`.  Both addresses 16-byte aligned, bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// bulk_load with an L2 cache policy
__device__ __forceinline__ void bulk_load_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                               uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}

// ------------------------------------------------------------------ tcgen05
// Per-warpgroup register limits (all four warps of a warpgroup execute the
// same one); an increase waits until the block has that many registers free.
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
    static_assert(N >= 24 && N <= 256 && N % 8 == 0, "setmaxnreg count");
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
    static_assert(N >= 24 && N <= 256 && N % 8 == 0, "setmaxnreg count");
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, e4m3 x e4m3 -> fp32, one elected thread.
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= (A * SFA)[smem] * (B * SFB)[smem]^T with packed e2m1 operands and
// e4m3 scale factors per 16 elements of K (MMA K = 64), scale factors in TMEM.
__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}
// Copy 32 rows x 16 bytes from shared memory (descriptor) into TMEM columns
// taddr..taddr+3 of lanes 0-31, repeated in all four 32-lane quadrants.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Arrive once on `bar` when every tcgen05 op issued so far by this thread completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
// ------------------------------------------------------------------ CTA pairs (cta_group::2)
// Two CTAs of a cluster of 2 (ranks 0 and 1) run one M = 256 MMA: each holds
// 128 rows of A and half of the N rows of B in its own shared memory at the
// same offsets, and receives its 128 rows of the accumulator in its own TMEM.
// Rank 0 issues the MMAs.  No multicast loads are used: each CTA loads its own
// halves, and the copies complete on rank 0's barrier.
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// address of the same shared-memory object in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx_cluster(uint32_t cluster_bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cluster.b64 _, [%0], %1;" ::"r"(cluster_bar), "r"(bytes)
                 : "memory");
}
// 2D tiled load into this CTA's shared memory, completion counted on a barrier
// of either CTA of the pair (a shared::cluster address).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* tm, uint32_t cluster_bar, int x, int y,
                                                 uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(cluster_bar), "r"(x), "r"(y), "l"(pol)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_f8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// the pair's MMAs issued so far arrive on `bar` (same offset) in both CTAs
__device__ __forceinline__ void mma_commit_pair_both(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}
// ... on `bar` in this CTA only
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (32x32b shape); the
// wait sits in the same asm statement, so no use of the registers can be
// scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
}

// Two 32-column loads (columns at a0.. and a1..) under one wait, so their
// latencies overlap.
__device__ __forceinline__ void tmem_ld32x2(uint32_t a0, uint32_t a1, float* v0, float* v1) {
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
        "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%65];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(a0), "r"(a1));
#pragma unroll
    for (int i = 0; i < 32; i++) {
        v0[i] = __uint_as_float(r[i]);
        v1[i] = __uint_as_float(r[32 + i]);
    }
}

// Shared-memory matrix descriptor (sm_100 layout): K-major tile whose rows are
// 128 bytes, stored in 8-row x 128-byte swizzle atoms (TMA SWIZZLE_128B), atoms
// 1024 bytes apart.  Fields: start address >> 4 [0,14), leading byte offset >> 4
// [16,30) (unused for this layout), stride byte offset >> 4 [32,46), version 1
// [46,48), layout type 2 = 128-byte swizzle [61,64).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(1) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Shared-memory descriptor of a scale-factor chunk for tcgen05.cp: 32 rows of
// 16 bytes, no swizzle, K-major; 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sdesc_sf_chunk(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(1) << 16;
    d |= static_cast<uint64_t>(128 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    return d;   // layout type 0 = no swizzle
}

// Instruction descriptor of kind::mxf4nvf4 with block scaling: A and B E2M1
// (format 1 at [7,10) and [10,13)), both K-major, N >> 3 at [17,23), scale
// factors E4M3 ([23] = 0), M >> 4 at [24,29), scale-factor ids 0, dense K = 64.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
    return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor of kind::f8f6f4: fp32 accumulate [4,6) = 1, A and B
// e4m3 [7,10) = [10,13) = 0, both K-major, N >> 3 at [17,23), M >> 4 at [24,29).
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
    return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Byte offset of block scale factor (row, column c) in the chunked layout the
// block-scaled tensor-core MMAs read: per 128-row tile, per 4 scale columns,
// 512 bytes with row r of the tile at (r % 32) * 16 + (r / 32) * 4 + c % 4.
// sf_cols = scale columns per row (K / 16 for NVFP4, K / 32 for MX).
__host__ __device__ __forceinline__ size_t sf_offset(long long row, int c, int sf_cols) {
    const long long tile = row >> 7;
    const int r = static_cast<int>(row & 127);
    return (static_cast<size_t>(tile) * (sf_cols >> 2) + (c >> 2)) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (c & 3);
}

// MX (UE8M0) block exponent: the smallest e with amax <= 448 * 2^e; amax =
// m 2^x with m in [0.5, 1) and 448 = 0.875 2^9 give e = x - 9 when m <= 0.875,
// else x - 8.  amax == 0 -> -127.  Clamped to [-127, 127].
__device__ __forceinline__ int mx_exponent(float amax) {
    if (amax == 0.0f) return -127;
    int x;
    const float m = frexpf(amax, &x);
    const int e = (m <= 0.875f) ? x - 9 : x - 8;
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}
// 2^-e as a float for e in [-126, 127] (2^-127 is the subnormal 2^-127)
__device__ __forceinline__ float mx_inv_scale(int e) {
    return e >= 127 ? 5.877471754111438e-39f : __int_as_float((127 - e) << 23);
}

// ------------------------------------------------------------------ numerics
// e4m3 of two floats, round to nearest even, saturating; .x -> low byte.
__device__ __forceinline__ uint16_t f2_to_e4m3x2(float a, float b) {
    return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}
// e2m1 of two floats, round to nearest even, saturating; a -> low nibble.
__device__ __forceinline__ uint8_t f2_to_e2m1x2(float a, float b) {
    return static_cast<uint8_t>(__nv_cvt_float2_to_fp4x2(make_float2(a, b), __NV_E2M1, cudaRoundNearest));
}
__device__ __forceinline__ uint8_t f_to_e4m3(float a) {
    return static_cast<uint8_t>(__nv_cvt_float_to_fp8(a, __NV_SATFINITE, __NV_E4M3));
}
__device__ __forceinline__ float e4m3_to_f(uint8_t c) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
    return __half2float(__half(h));
}
// Gated activation h = act(g, u) of the expert MLP in fp32 (LightMoE README,
// "Compatibility"): 0 SwiGLU silu(g) u; 1 bounded SwiGLU silu(min(g, L))
// clamp(u, -L, L); 2 SwiGLU-OAI g' sigmoid(alpha g') (u' + 1) with the same
// clamps; 3 GeGLU 0.5 g (1 + erf(g / sqrt 2)) u; 4 ReGLU max(g, 0) u.
// The GEMM kernels are instantiated per activation (ACT is a compile-time
// constant there), so each epilogue is straight-line code for its activation.
template <int ACT>
__device__ __forceinline__ float glu(float g, float u, float alpha, float limit) {
    if constexpr (ACT == 0) {
        return g / (1.0f + expf(-g)) * u;
    } else if constexpr (ACT == 1 || ACT == 2) {
        const float gc = fminf(g, limit), uc = fminf(fmaxf(u, -limit), limit);
        if constexpr (ACT == 1) return gc / (1.0f + expf(-gc)) * uc;
        else return gc / (1.0f + expf(-alpha * gc)) * (uc + 1.0f);
    } else if constexpr (ACT == 3) {
        return 0.5f * g * (1.0f + erff(g * 0.70710678118654752f)) * u;
    } else {
        return fmaxf(g, 0.0f) * u;
    }
}

// The same activations for an e4m3 hidden: the sigmoid uses the hardware
// exponential and reciprocal (__expf, __fdividef: a few ulp of fp32). The
// result is rounded to an e4m3 code (a 2^-4 relative step) right after, so a
// code changes only when the value sits within those ulp of a rounding
// boundary; the parity tests bound the fraction of such codes.  (An e2m1
// hidden keeps glu: one of its codes moves a value by up to half.)  For
// g < -88 exp overflows and __fdividef(g, inf) is 0, the limit of silu.
template <int ACT>
__device__ __forceinline__ float glu_e4m3(float g, float u, float alpha, float limit) {
    if constexpr (ACT == 0) {
        return __fdividef(g, 1.0f + __expf(-g)) * u;
    } else if constexpr (ACT == 1 || ACT == 2) {
        const float gc = fminf(g, limit), uc = fminf(fmaxf(u, -limit), limit);
        if constexpr (ACT == 1) return __fdividef(gc, 1.0f + __expf(-gc)) * uc;
        else return __fdividef(gc, 1.0f + __expf(-alpha * gc)) * (uc + 1.0f);
    } else {
        return glu<ACT>(g, u, alpha, limit);
    }
}

// ReLU^2 experts (no gate): h = max(u, 0)^2
__device__ __forceinline__ float relu_sq(float u) {
    const float r = fmaxf(u, 0.0f);
    return r * r;
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

}  // namespace moe
