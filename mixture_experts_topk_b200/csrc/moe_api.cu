// moe_api.cu -- the C ABI declared in include/moe_b200.h: argument checks,
// workspace and packed-weight layouts, tensor maps, and the launch sequence
// route -> dispatch -> gate/up GEMM -> down GEMM -> combine.
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>

#include "moe_b200.h"
#include "common.cuh"
#include "dispatch.cuh"
#include "gemm.cuh"
#include "gemm_fp4.cuh"
#include "gemm_mx.cuh"
#include "router.cuh"
#include "router_tc.cuh"

using namespace moe;

// ------------------------------------------------------------------ errors
static thread_local char g_err[512] = "";

static moe_status fail(moe_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return st;
}

#define CUDA_TRY(expr)                                                                       \
    do {                                                                                     \
        cudaError_t err_ = (expr);                                                           \
        if (err_ != cudaSuccess)                                                             \
            return fail(MOE_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(err_));     \
    } while (0)

#define LAUNCH_CHECK(name)                                                                   \
    do {                                                                                     \
        cudaError_t err_ = cudaGetLastError();                                               \
        if (err_ != cudaSuccess)                                                             \
            return fail(MOE_ERR_CUDA, "launch of %s failed: %s", name, cudaGetErrorString(err_)); \
    } while (0)

extern "C" const char* moe_last_error(void) { return g_err; }

// Launch a kernel of the layer.  With pdl set the launch carries the
// programmatic-stream-serialization attribute: the kernel may be scheduled
// while its predecessor finishes, and its own pdl_wait() orders its memory
// accesses after that predecessor's.
template <typename... KP, typename... Args>
static cudaError_t launch_k(bool pdl, void (*kern)(KP...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                            Args&&... args) {
    cudaLaunchConfig_t lc;
    memset(&lc, 0, sizeof(lc));
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    lc.attrs = attr;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, kern, std::forward<Args>(args)...);
}

// the same for a grid of 2-CTA clusters (CTA pairs)
template <typename... KP, typename... Args>
static cudaError_t launch_k_pairs(bool pdl, void (*kern)(KP...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                  Args&&... args) {
    cudaLaunchConfig_t lc;
    memset(&lc, 0, sizeof(lc));
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = 2;
    return cudaLaunchKernelEx(&lc, kern, std::forward<Args>(args)...);
}

#define LAUNCH(pdl, name, kern, grid, block, smem, st, ...)                                  \
    do {                                                                                     \
        cudaError_t err_ = launch_k((pdl), kern, dim3(grid), dim3(block), (smem), (st), __VA_ARGS__); \
        if (err_ != cudaSuccess)                                                             \
            return fail(MOE_ERR_CUDA, "launch of %s failed: %s", name, cudaGetErrorString(err_)); \
    } while (0)

// ------------------------------------------------------------------ layouts
static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct WsLayout {
    size_t status, ids, w, logits, counts, offsets, num_tiles, tile_ptr, pick, gu_done, chunk, tiles, perm, inv, xglobal, xq, xs, hq, hs, o, oe;
    // fixed-point rows of the tensor-core router (0 when the workspace has none)
    size_t rxh, rxl, rwh, rwl, rx_exp, rx_sum, rx_max, rw_exp, rw_sum, rw_sumq, rw_max;
    size_t total;
};
struct WLayout {
    size_t gu_q, gu_s, d_q, d_s, gu_g, d_g, total;
};

struct moe_handle {
    moe_config cfg;
    int device;
    int num_sms;
    WsLayout ws;
    WLayout wl;
    long long spin_limit;
    int down_bn;          // 0 = picked per call, else 64 / 128 / 256
    int gemm_pairs;       // large FP8_ROW batches run the gate/up GEMM on CTA pairs
    int gu_bn;            // gated FP8_ROW gate/up tile width: 0 = picked on the device, else 128 / 256
    PickerParams picker;
    int pdl;              // launch with programmatic dependent launch allowed
};

static size_t code_bytes(int fmt, int K) { return fmt == MOE_FMT_NVFP4 ? K / 2 : K; }
static size_t act_scale_bytes(int fmt, int K) {
    if (fmt == MOE_FMT_FP8_ROW) return 4;
    if (fmt == MOE_FMT_FP8_BLOCK128) return 4 * (K / 128);
    return K / 16;
}
// scale bytes per hidden row: MX (power of two per 32) for FP8_ROW, fp32 per 128
// for FP8_BLOCK128, e4m3 per 16 for NVFP4
static size_t hidden_scale_bytes(int fmt, int I) {
    if (fmt == MOE_FMT_FP8_ROW) return I / 32;
    return fmt == MOE_FMT_NVFP4 ? I / 16 : 4 * (I / 128);
}
// rows of the X / hidden buffers: 128-padded per expert where block-scaled
// tensor-core MMAs read them (NVFP4 X and hidden, FP8_ROW hidden)
// Unpadded buffers (rows in slot order) get TILE_M rows of slack: a row tile
// starting at any slot stays inside the tensor map, so the TMA box never
// zero-fills past the end (which slows the copy); the slack rows feed only
// accumulator rows the epilogue does not store.
static size_t padded_rows(const moe_config& c) {
    const size_t A = static_cast<size_t>(c.max_T) * c.k;
    return c.fmt == MOE_FMT_NVFP4 ? A + static_cast<size_t>(TILE_M) * c.E : A + TILE_M;
}
static size_t hidden_rows(const moe_config& c) {
    const size_t A = static_cast<size_t>(c.max_T) * c.k;
    return c.fmt == MOE_FMT_FP8_BLOCK128 ? A + TILE_M : A + static_cast<size_t>(TILE_M) * c.E;
}

// rows of the fp32 down output: A, plus room for up to 8 K-split copies of
// batches of at most 256 assignments where the down GEMM may split its K
static size_t o_rows(const moe_config& c) {
    const size_t A = static_cast<size_t>(c.max_T) * c.k;
    return c.fmt == MOE_FMT_FP8_ROW ? A + 7 * std::min<size_t>(A, 256) : A;
}

// The large-batch router (router_tc.cuh): batches above 128 tokens with more
// than 8 experts.  Expert tiles of 128, or of E rounded up to 16.
static bool router_tc_sized(const moe_config& c) { return c.max_T > 128 && c.E > 8 && c.H <= RTC_MAX_H; }
// experts per tile: 128, or 64 when 128-wide tiles would leave over half of
// the SMs idle; E rounded up to 16 when E <= 128
static int router_tc_nt(int E, int T, int num_sms) {
    if (E <= RTC_NT_MAX) return (E + 15) / 16 * 16;
    const int tiles = (T + RTC_BM - 1) / RTC_BM * ((E + RTC_NT_MAX - 1) / RTC_NT_MAX);
    return 2 * tiles < num_sms ? RTC_NT_MAX / 2 : RTC_NT_MAX;
}
// Wr rows padded to whole tiles (the workspace holds the widest padding)
static int router_tc_epad(int E, int nt) { return (E + nt - 1) / nt * nt; }
static int router_tc_epad_max(int E) {
    return E <= RTC_NT_MAX ? (E + 15) / 16 * 16 : (E + RTC_NT_MAX - 1) / RTC_NT_MAX * RTC_NT_MAX;
}

static WsLayout make_ws_layout(const moe_config& c) {
    const size_t A = static_cast<size_t>(c.max_T) * c.k;
    const size_t nchunks = (A + DISPATCH_CHUNK - 1) / DISPATCH_CHUNK;
    const size_t tiles_cap = A / TILE_M + c.E + 1;
    WsLayout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    L.status = take(64 * 4);
    L.ids = take(A * 4);
    L.w = take(A * 4);
    L.logits = take(static_cast<size_t>(c.max_T) * c.E * 4);
    L.counts = take(c.E * 4);
    L.offsets = take((c.E + 1) * 4);
    L.num_tiles = take(4);
    L.tile_ptr = take((c.E + 1) * 4);
    L.pick = take(16);
    L.gu_done = take(c.E * 4);
    L.chunk = take(nchunks * c.E * 4);
    L.tiles = take(tiles_cap * 8);
    L.perm = take(A * 4);
    L.inv = take(A * 4);
    L.xglobal = take(16);
    // NVFP4 rows are padded to 128 per expert, so each row tile owns whole
    // scale-factor chunks
    const size_t R = padded_rows(c), RH = hidden_rows(c);
    L.xq = take(R * code_bytes(c.fmt, c.H));
    L.xs = take(R * act_scale_bytes(c.fmt, c.H));
    L.hq = take(RH * code_bytes(c.fmt, c.I));
    L.hs = take(RH * hidden_scale_bytes(c.fmt, c.I));
    L.o = take(o_rows(c) * c.H * 2);        // fp16 rows
    L.oe = take(o_rows(c) * (c.H / 32));    // their block exponents
    L.rxh = L.rxl = L.rwh = L.rwl = L.rx_exp = L.rx_sum = L.rx_max = L.rw_exp = L.rw_sum = L.rw_sumq = L.rw_max = 0;
    if (router_tc_sized(c)) {
        const size_t T = c.max_T, H = c.H, Ep = router_tc_epad_max(c.E);
        L.rxh = take(T * H);
        L.rxl = take(T * H);
        L.rwh = take(Ep * H);
        L.rwl = take(Ep * H);
        L.rx_exp = take(T * 4);
        L.rx_sum = take(T * 8);
        L.rx_max = take(T * 4);
        L.rw_exp = take(Ep * 4);
        L.rw_sum = take(Ep * 8);
        L.rw_sumq = take(Ep * 8);
        L.rw_max = take(Ep * 4);
    }
    L.total = off;
    return L;
}

static WLayout make_w_layout(const moe_config& c) {
    const size_t E = c.E, H = c.H, I = c.I;
    WLayout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    L.gu_q = take(E * 2 * I * code_bytes(c.fmt, c.H));
    L.d_q = take(E * H * code_bytes(c.fmt, c.I));
    if (c.fmt == MOE_FMT_FP8_ROW) {
        L.gu_s = take(E * 2 * I * 4);
        L.d_s = take(E * H * 4);
    } else if (c.fmt == MOE_FMT_FP8_BLOCK128) {
        L.gu_s = take(E * (2 * I / 128) * (H / 128) * 4);
        L.d_s = take(E * (H / 128) * (I / 128) * 4);
    } else {
        L.gu_s = take(E * 2 * I * (H / 16));
        L.d_s = take(E * H * (I / 16));
    }
    L.gu_g = take(E * 2 * 4);
    L.d_g = take(E * 4);
    L.total = off;
    return L;
}

// ------------------------------------------------------------------ init
// Gate/up mode model: per-unit cost kb * a + b (ps) on 256-wide single CTAs,
// CTA pairs and 128-wide single CTAs.  a_0 is the per-K-block cost of a
// 128 x 256 unit from a least-squares fit of an interleaved B200 sweep of the
// modes; the others are set against it so that the rule reproduces the
// fastest measured mode of each point of that sweep (gated FP8_ROW workloads
// at every batch size and two more shapes): a_1 = a_0 / 1.069 and b_1 = 0.2 us
// (a pair unit's fixed cost: one-wave batches stay on single CTAs); a_2 =
// 0.634 a_0, the middle of the range (0.60-0.66 a_0) that separates the
// points where 128-wide tiles measured faster from those where they did not.
static const long long GU_MODE_FIT[6] = {527000, 0, 493000, 200000, 334000, 0};

// allowed gate/up modes (bit 0 wide single, 1 pairs, 2 narrow) under the
// host's options, 0 when they contradict each other
static int gu_allow_of(int gemm_pairs, int gu_bn) {
    int allow = 7;
    if (gemm_pairs == 0) allow &= ~2;
    if (gemm_pairs == 2) allow &= 2;
    if (gu_bn == 128) allow &= 4;
    if (gu_bn == 256) allow &= ~4;
    return allow;
}

extern "C" moe_status moe_init(const moe_config* cfg, moe_handle** out) {
    if (!cfg || !out) return fail(MOE_ERR_INVALID_ARG, "moe_init: null argument");
    const moe_config& c = *cfg;
    if (c.H <= 0 || c.I <= 0 || c.E <= 0 || c.k <= 0 || c.max_T <= 0)
        return fail(MOE_ERR_INVALID_ARG, "moe_init: sizes must be positive");
    if (c.score != MOE_SCORE_SOFTMAX && c.score != MOE_SCORE_SIGMOID)
        return fail(MOE_ERR_INVALID_ARG, "moe_init: unknown score function %d", c.score);
    if (c.fmt != MOE_FMT_FP8_ROW && c.fmt != MOE_FMT_FP8_BLOCK128 && c.fmt != MOE_FMT_NVFP4)
        return fail(MOE_ERR_INVALID_ARG, "moe_init: unknown format %d", c.fmt);
    if (c.H % 256 != 0 || c.I % 128 != 0)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_init: H must be a multiple of 256 and I of 128 (H=%d I=%d)", c.H, c.I);
    if (c.k > 8 || c.k > c.E || c.E > 256)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_init: need 1 <= k <= 8, k <= E <= 256 (E=%d k=%d)", c.E, c.k);
    if (static_cast<long long>(c.max_T) * c.k > 131072)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_init: max_T * k must be <= 131072");
    if (c.fmt == MOE_FMT_NVFP4 && c.I % 256 != 0)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_init: NVFP4 needs I to be a multiple of 256 (I=%d)", c.I);
    if (c.fmt == MOE_FMT_NVFP4 && !(c.hidden_global_scale > 0.0f))
        return fail(MOE_ERR_INVALID_ARG, "moe_init: NVFP4 needs a positive hidden_global_scale");
    if (c.act < MOE_ACT_SWIGLU || c.act > MOE_ACT_RELU2)
        return fail(MOE_ERR_INVALID_ARG, "moe_init: unknown activation %d", c.act);
    if (c.act == MOE_ACT_RELU2 && c.I % 256 != 0)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_init: ReLU^2 experts need I to be a multiple of 256 (I=%d)", c.I);
    if ((c.act == MOE_ACT_SWIGLU_BOUNDED || c.act == MOE_ACT_SWIGLU_OAI) && !(c.act_limit > 0.0f))
        return fail(MOE_ERR_INVALID_ARG, "moe_init: this activation needs a positive act_limit");
    if (c.act == MOE_ACT_SWIGLU_OAI && !(c.act_alpha > 0.0f))
        return fail(MOE_ERR_INVALID_ARG, "moe_init: SWIGLU_OAI needs a positive act_alpha");
    moe_handle* h = new (std::nothrow) moe_handle;
    if (!h) return fail(MOE_ERR_INVALID_ARG, "moe_init: out of host memory");
    h->cfg = c;
    CUDA_TRY(cudaGetDevice(&h->device));
    CUDA_TRY(cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device));
    h->ws = make_ws_layout(c);
    h->wl = make_w_layout(c);
    h->spin_limit = 2000000000LL;   // ~1 s of SM clock per wait
    h->down_bn = 0;
    h->picker.alpha_ps = 334419;       // least-squares fit to a B200 tile sweep
    h->picker.beta_ps = 2114;
    h->picker.bw_cta = 38684;
    h->picker.gamma_ps = 17030139;
    h->picker.num_sms = h->num_sms;
    h->pdl = 1;
    h->gemm_pairs = 1;
    h->gu_bn = 0;
    h->picker.H = c.H;
    h->picker.I = c.I;
    h->picker.split_nb = c.fmt == MOE_FMT_FP8_ROW ? c.H / MX_BN : 0;
    h->picker.split_kb = c.I / 128;
    h->picker.o_rows = static_cast<int>(o_rows(c));
    // gate/up CTA mode (FP8_ROW SwiGLU), per-unit costs fitted to a B200 sweep
    h->picker.gu_nb = (c.fmt == MOE_FMT_FP8_ROW && c.act != MOE_ACT_RELU2) ? 2 * c.I / 256 : 0;
    h->picker.gu_kb = c.H / 128;
    h->picker.gu_allow = gu_allow_of(h->gemm_pairs, h->gu_bn);
    for (int i = 0; i < 6; i++) h->picker.gu_ps[i] = GU_MODE_FIT[i];
    *out = h;
    return MOE_OK;
}

extern "C" moe_status moe_destroy(moe_handle* h) {
    delete h;
    return MOE_OK;
}

extern "C" moe_status moe_weights_size(const moe_handle* h, size_t* bytes) {
    if (!h || !bytes) return fail(MOE_ERR_INVALID_ARG, "moe_weights_size: null argument");
    *bytes = h->wl.total;
    return MOE_OK;
}

extern "C" moe_status moe_workspace_size(const moe_handle* h, size_t* bytes) {
    if (!h || !bytes) return fail(MOE_ERR_INVALID_ARG, "moe_workspace_size: null argument");
    *bytes = h->ws.total;
    return MOE_OK;
}

extern "C" moe_status moe_workspace_view_get(const moe_handle* h, void* ws, moe_workspace_view* v) {
    if (!h || !ws || !v) return fail(MOE_ERR_INVALID_ARG, "moe_workspace_view_get: null argument");
    uint8_t* b = static_cast<uint8_t*>(ws);
    const WsLayout& L = h->ws;
    v->status = reinterpret_cast<int32_t*>(b + L.status);
    v->ids = reinterpret_cast<int32_t*>(b + L.ids);
    v->w = reinterpret_cast<float*>(b + L.w);
    v->counts = reinterpret_cast<int32_t*>(b + L.counts);
    v->offsets = reinterpret_cast<int32_t*>(b + L.offsets);
    v->num_tiles = reinterpret_cast<int32_t*>(b + L.num_tiles);
    v->tile_ptr = reinterpret_cast<int32_t*>(b + L.tile_ptr);
    v->pick = reinterpret_cast<int32_t*>(b + L.pick);
    v->tiles = reinterpret_cast<int32_t*>(b + L.tiles);
    v->perm = reinterpret_cast<int32_t*>(b + L.perm);
    v->inv = reinterpret_cast<int32_t*>(b + L.inv);
    v->x_global = reinterpret_cast<float*>(b + L.xglobal);
    v->xq = b + L.xq;
    v->xs = b + L.xs;
    v->hq = b + L.hq;
    v->hs = b + L.hs;
    v->o = reinterpret_cast<uint16_t*>(b + L.o);
    v->o_exp = reinterpret_cast<int8_t*>(b + L.oe);
    v->logits = reinterpret_cast<float*>(b + L.logits);
    return MOE_OK;
}

static bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }

// per-expert count of finished gate/up parts (reset by the dispatch's scan)
static int32_t* gu_done_of(const moe_handle* h, void* ws) {
    return reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + h->ws.gu_done);
}

static moe_status check_T(const moe_handle* h, int T, const char* who) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "%s: null handle", who);
    if (T < 0 || T > h->cfg.max_T) return fail(MOE_ERR_INVALID_ARG, "%s: T=%d outside [0, max_T=%d]", who, T, h->cfg.max_T);
    return MOE_OK;
}

// ------------------------------------------------------------------ pack
extern "C" moe_status moe_pack_weights(const moe_handle* h, const moe_weights* src, void* packed, moe_stream_t stream) {
    if (!h || !src || !packed) return fail(MOE_ERR_INVALID_ARG, "moe_pack_weights: null argument");
    const bool relu2 = h->cfg.act == MOE_ACT_RELU2;   // up and down only
    if ((!relu2 && (!src->gate_q || !src->gate_s)) || !src->up_q || !src->down_q || !src->up_s || !src->down_s)
        return fail(MOE_ERR_INVALID_ARG, "moe_pack_weights: null weight pointer");
    if (!aligned256(packed)) return fail(MOE_ERR_INVALID_ARG, "moe_pack_weights: packed must be 256-byte aligned");
    const moe_config& c = h->cfg;
    uint8_t* b = static_cast<uint8_t*>(packed);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int grid = 4 * h->num_sms;
    if (relu2) {
        // the up projection alone, in row order: W_u [E, I, K-bytes] and its scales
        const size_t E = c.E, I = c.I, H = c.H;
        CUDA_TRY(cudaMemcpyAsync(b + h->wl.gu_q, src->up_q, E * I * code_bytes(c.fmt, c.H), cudaMemcpyDeviceToDevice,
                                 st));
        if (c.fmt == MOE_FMT_NVFP4) {
            if (!src->up_g || !src->down_g)
                return fail(MOE_ERR_INVALID_ARG, "moe_pack_weights: NVFP4 needs the global scales");
            pack_sf_kernel<<<grid, 256, 0, st>>>(static_cast<const uint8_t*>(src->up_s), nullptr, b + h->wl.gu_s, c.E,
                                                 c.I, 0, c.H / 16, 0);
            LAUNCH_CHECK("pack_sf_kernel(up)");
            pack_sf_kernel<<<grid, 256, 0, st>>>(static_cast<const uint8_t*>(src->down_s), nullptr, b + h->wl.d_s,
                                                 c.E, c.H, 0, c.I / 16, 0);
            LAUNCH_CHECK("pack_sf_kernel(down)");
            CUDA_TRY(cudaMemcpyAsync(b + h->wl.d_q, src->down_q, E * H * (I / 2), cudaMemcpyDeviceToDevice, st));
            // [E][2] global scales as for gated experts, both entries the up scale
            CUDA_TRY(cudaMemcpy2DAsync(b + h->wl.gu_g, 8, src->up_g, 4, 4, c.E, cudaMemcpyDeviceToDevice, st));
            CUDA_TRY(cudaMemcpy2DAsync(b + h->wl.gu_g + 4, 8, src->up_g, 4, 4, c.E, cudaMemcpyDeviceToDevice, st));
            CUDA_TRY(cudaMemcpyAsync(b + h->wl.d_g, src->down_g, E * 4, cudaMemcpyDeviceToDevice, st));
            return MOE_OK;
        }
        const size_t us = c.fmt == MOE_FMT_FP8_ROW ? E * I * 4 : E * (I / 128) * (H / 128) * 4;
        const size_t ds = c.fmt == MOE_FMT_FP8_ROW ? E * H * 4 : E * (H / 128) * (I / 128) * 4;
        CUDA_TRY(cudaMemcpyAsync(b + h->wl.gu_s, src->up_s, us, cudaMemcpyDeviceToDevice, st));
        CUDA_TRY(cudaMemcpyAsync(b + h->wl.d_s, src->down_s, ds, cudaMemcpyDeviceToDevice, st));
        CUDA_TRY(cudaMemcpyAsync(b + h->wl.d_q, src->down_q, E * H * I, cudaMemcpyDeviceToDevice, st));
        return MOE_OK;
    }
    if (c.fmt == MOE_FMT_NVFP4) {
        if (!src->gate_g || !src->up_g || !src->down_g)
            return fail(MOE_ERR_INVALID_ARG, "moe_pack_weights: NVFP4 needs the global scales");
        // gate/up interleaved in 64-row groups (a 128-row tile = 64 gate + 64 up)
        interleave_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const uint32_t*>(src->gate_q),
                                                     static_cast<const uint32_t*>(src->up_q),
                                                     reinterpret_cast<uint32_t*>(b + h->wl.gu_q), c.E, c.I, 64, c.H / 8);
        LAUNCH_CHECK("interleave_rows_kernel(nvfp4 codes)");
        pack_sf_kernel<<<grid, 256, 0, st>>>(static_cast<const uint8_t*>(src->gate_s),
                                             static_cast<const uint8_t*>(src->up_s), b + h->wl.gu_s, c.E, c.I, 64,
                                             c.H / 16, 1);
        LAUNCH_CHECK("pack_sf_kernel(gate/up)");
        pack_sf_kernel<<<grid, 256, 0, st>>>(static_cast<const uint8_t*>(src->down_s), nullptr, b + h->wl.d_s, c.E,
                                             c.H, 0, c.I / 16, 0);
        LAUNCH_CHECK("pack_sf_kernel(down)");
        CUDA_TRY(cudaMemcpyAsync(b + h->wl.d_q, src->down_q, static_cast<size_t>(c.E) * c.H * (c.I / 2),
                                 cudaMemcpyDeviceToDevice, st));
        CUDA_TRY(cudaMemcpy2DAsync(b + h->wl.gu_g, 8, src->gate_g, 4, 4, c.E, cudaMemcpyDeviceToDevice, st));
        CUDA_TRY(cudaMemcpy2DAsync(b + h->wl.gu_g + 4, 8, src->up_g, 4, 4, c.E, cudaMemcpyDeviceToDevice, st));
        CUDA_TRY(cudaMemcpyAsync(b + h->wl.d_g, src->down_g, static_cast<size_t>(c.E) * 4, cudaMemcpyDeviceToDevice,
                                 st));
        return MOE_OK;
    }
    interleave_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const uint32_t*>(src->gate_q),
                                                 static_cast<const uint32_t*>(src->up_q),
                                                 reinterpret_cast<uint32_t*>(b + h->wl.gu_q), c.E, c.I, 128,
                                                 static_cast<int>(code_bytes(c.fmt, c.H) / 4));
    LAUNCH_CHECK("interleave_rows_kernel(codes)");
    if (c.fmt == MOE_FMT_FP8_ROW) {
        interleave_rows_kernel<<<grid, 32, 0, st>>>(static_cast<const uint32_t*>(src->gate_s),
                                                    static_cast<const uint32_t*>(src->up_s),
                                                    reinterpret_cast<uint32_t*>(b + h->wl.gu_s), c.E, c.I, 128, 1);
        CUDA_TRY(cudaMemcpyAsync(b + h->wl.d_s, src->down_s, static_cast<size_t>(c.E) * c.H * 4,
                                 cudaMemcpyDeviceToDevice, st));
    } else {
        interleave_rows_kernel<<<grid, 32, 0, st>>>(static_cast<const uint32_t*>(src->gate_s),
                                                    static_cast<const uint32_t*>(src->up_s),
                                                    reinterpret_cast<uint32_t*>(b + h->wl.gu_s), c.E, c.I / 128, 1,
                                                    c.H / 128);
        CUDA_TRY(cudaMemcpyAsync(b + h->wl.d_s, src->down_s,
                                 static_cast<size_t>(c.E) * (c.H / 128) * (c.I / 128) * 4, cudaMemcpyDeviceToDevice, st));
    }
    LAUNCH_CHECK("interleave_rows_kernel(scales)");
    CUDA_TRY(cudaMemcpyAsync(b + h->wl.d_q, src->down_q, static_cast<size_t>(c.E) * c.H * code_bytes(c.fmt, c.I),
                             cudaMemcpyDeviceToDevice, st));
    return MOE_OK;
}

// ------------------------------------------------------------------ route
static moe_status make_tmap(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch,
                            uint32_t box_inner, uint32_t box_rows, bool swizzle = true);

// Large batches: fixed-point rows, exact int8 tensor-core products, and the
// certified candidate filter with canonical logits for the candidates
// (router_tc.cuh).  Same ids and weights as the SIMT kernels.
static moe_status route_tc(const moe_handle* h, const void* x, int T, const float* wr, const RouterParams& p, void* ws,
                           cudaStream_t st) {
    const moe_config& c = h->cfg;
    uint8_t* b = static_cast<uint8_t*>(ws);
    const WsLayout& L = h->ws;
    RouterFix f;
    f.xh = reinterpret_cast<int8_t*>(b + L.rxh);
    f.xl = reinterpret_cast<int8_t*>(b + L.rxl);
    f.wh = reinterpret_cast<int8_t*>(b + L.rwh);
    f.wl = reinterpret_cast<int8_t*>(b + L.rwl);
    f.x_exp = reinterpret_cast<int32_t*>(b + L.rx_exp);
    f.x_sum = reinterpret_cast<double*>(b + L.rx_sum);
    f.x_max = reinterpret_cast<float*>(b + L.rx_max);
    f.w_exp = reinterpret_cast<int32_t*>(b + L.rw_exp);
    f.w_sum = reinterpret_cast<double*>(b + L.rw_sum);
    f.w_sumq = reinterpret_cast<double*>(b + L.rw_sumq);
    f.w_max = reinterpret_cast<float*>(b + L.rw_max);
    const int NT = router_tc_nt(c.E, T, h->num_sms), Ep = router_tc_epad(c.E, NT);
    const int nbx = (T + 7) / 8, nbw = (Ep + 7) / 8;
    LAUNCH(h->pdl, "router_fixpoint_kernel", router_fixpoint_kernel, nbx + nbw, 256, 0, st,
           static_cast<const __nv_bfloat16*>(x), wr, T, c.H, c.E, Ep, nbx, f);
    CUtensorMap txh, txl, twh, twl;
    moe_status r = make_tmap(&txh, f.xh, c.H, T, c.H, RTC_BK, RTC_BM);
    if (r != MOE_OK) return r;
    r = make_tmap(&txl, f.xl, c.H, T, c.H, RTC_BK, RTC_BM);
    if (r != MOE_OK) return r;
    r = make_tmap(&twh, f.wh, c.H, Ep, c.H, RTC_BK, NT);
    if (r != MOE_OK) return r;
    r = make_tmap(&twl, f.wl, c.H, Ep, c.H, RTC_BK, NT);
    if (r != MOE_OK) return r;
    RouterI8Params q;
    q.T = T;
    q.H = c.H;
    q.E = c.E;
    q.NT = NT;
    q.x_exp = f.x_exp;
    q.w_exp = f.w_exp;
    q.bias = p.bias;
    q.logits = p.logits;
    q.status = reinterpret_cast<int32_t*>(b + L.status);
    q.spin_limit = h->spin_limit;
    CUDA_TRY(cudaFuncSetAttribute(router_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, RTC_SMEM));
    LAUNCH(h->pdl, "router_i8_kernel", router_i8_kernel, dim3((T + RTC_BM - 1) / RTC_BM, Ep / NT), RTC_THREADS,
           RTC_SMEM, st, txh, txl, twh, twl, q);
    LAUNCH(h->pdl, "router_select_kernel", router_select_kernel, std::min((T + 7) / 8, 16 * h->num_sms), 256, 0, st,
           p, f);
    return MOE_OK;
}

extern "C" moe_status moe_route(const moe_handle* h, const void* x, int T, const float* wr, const float* bias,
                                int32_t* ids, float* w, void* ws, moe_stream_t stream) {
    moe_status st0 = check_T(h, T, "moe_route");
    if (st0 != MOE_OK) return st0;
    if (T == 0) return MOE_OK;
    if (!x || !wr || !ids || !w) return fail(MOE_ERR_INVALID_ARG, "moe_route: null argument");
    if (h->cfg.has_bias && !bias) return fail(MOE_ERR_INVALID_ARG, "moe_route: config has a bias but bias is null");
    if (!h->cfg.has_bias) bias = nullptr;
    if (!aligned256(x) || !aligned256(wr)) return fail(MOE_ERR_INVALID_ARG, "moe_route: x and wr must be 256-byte aligned");
    if (!ws || !aligned256(ws)) return fail(MOE_ERR_INVALID_ARG, "moe_route: ws must be a 256-byte aligned workspace");
    RouterParams p;
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.wr = wr;
    p.bias = bias;
    p.logits = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + h->ws.logits);
    p.ids = ids;
    p.w = w;
    p.T = T;
    p.H = h->cfg.H;
    p.E = h->cfg.E;
    p.k = h->cfg.k;
    p.score = h->cfg.score;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (T > 128 && router_tc_sized(h->cfg)) return route_tc(h, x, T, wr, p, ws, st);
    if (T <= 128 && h->cfg.E <= RF_MAX_E) {
        // logits and top-k in one launch
        LAUNCH(h->pdl, "router_small_fused_kernel", router_small_fused_kernel, (T + RS_TG - 1) / RS_TG,
               32 * std::max(h->cfg.E, RS_TG), 0, st, p);
        return MOE_OK;
    }
    if (T <= 128) {
        LAUNCH(h->pdl, "router_logits_small_kernel", router_logits_small_kernel,
               dim3((T + RS_TG - 1) / RS_TG, (h->cfg.E + RS_WARPS - 1) / RS_WARPS), RS_WARPS * 32, 0, st, p);
    } else if (h->cfg.E <= 8) {
        // 32-token tiles (4-token x 8-expert micro-tiles), so that T = 4096 keeps
        // 128 SMs busy rather than 64
        using RT = RouterTile<32, 8, 4>;
        CUDA_TRY(cudaFuncSetAttribute(router_logits_kernel<32, 8, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      RT::SMEM));
        auto kern = router_logits_kernel<32, 8, 4>;
        LAUNCH(h->pdl, "router_logits_kernel", kern, dim3((T + 31) / 32, 1), RT::NT, RT::SMEM, st, p);
    } else {
        using RT = RouterTile<64, 16, 16>;
        CUDA_TRY(cudaFuncSetAttribute(router_logits_kernel<64, 16, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      RT::SMEM));
        auto kern = router_logits_kernel<64, 16, 16>;
        LAUNCH(h->pdl, "router_logits_kernel", kern, dim3((T + 63) / 64, (h->cfg.E + 15) / 16), RT::NT,
               RT::SMEM, st, p);
    }
    LAUNCH(h->pdl, "router_topk_kernel", router_topk_kernel, std::min((T + 7) / 8, 16 * h->num_sms), 256, 0, st, p);
    return MOE_OK;
}

// ------------------------------------------------------------------ dispatch
extern "C" moe_status moe_dispatch(const moe_handle* h, const void* x, const int32_t* ids, int T, void* ws,
                                   moe_stream_t stream) {
    moe_status st0 = check_T(h, T, "moe_dispatch");
    if (st0 != MOE_OK) return st0;
    if (!ws) return fail(MOE_ERR_INVALID_ARG, "moe_dispatch: null workspace");
    if (T > 0 && (!x || !ids)) return fail(MOE_ERR_INVALID_ARG, "moe_dispatch: null argument");
    if (!aligned256(ws) || (T > 0 && !aligned256(x)))
        return fail(MOE_ERR_INVALID_ARG, "moe_dispatch: x and ws must be 256-byte aligned");
    const moe_config& c = h->cfg;
    moe_workspace_view v;
    moe_workspace_view_get(h, ws, &v);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int A = T * c.k;
    const int nchunks = (A + DISPATCH_CHUNK - 1) / DISPATCH_CHUNK;
    int32_t* chunk = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + h->ws.chunk);
    if (A > 0 && nchunks == 1 && c.fmt != MOE_FMT_NVFP4) {
        // one chunk: the dispatch and the quantisation in one launch, a CTA per token
        LAUNCH(h->pdl, "dispatch_quant_small_kernel",
               c.fmt == MOE_FMT_FP8_ROW ? dispatch_quant_small_kernel<0> : dispatch_quant_small_kernel<1>,
               std::min(T, 8 * h->num_sms), 256, 0, st, ids, A, c.E, T, c.H, c.k,
               static_cast<const __nv_bfloat16*>(x), v.counts, v.offsets, v.tiles, v.num_tiles, v.tile_ptr, v.pick,
               h->picker, v.perm, v.inv, v.status, gu_done_of(h, ws), v.xq, static_cast<float*>(v.xs));
        return MOE_OK;
    }
    if (A > 0 && nchunks == 1) {
        // one chunk: histogram, scan and ranks in one CTA
        LAUNCH(h->pdl, "dispatch_small_kernel", dispatch_small_kernel, 1, DISPATCH_CHUNK, 0, st, ids, A, c.E,
               v.counts, v.offsets, v.tiles, v.num_tiles, v.tile_ptr, v.pick, h->picker, v.perm, v.inv, v.status,
               gu_done_of(h, ws));
    } else {
        if (A > 0) {
            LAUNCH(h->pdl, "hist_kernel", hist_kernel, nchunks, DISPATCH_CHUNK, 0, st, ids, A, c.E, chunk, v.status);
        }
        const int scan_smem = nchunks * c.E * 4;   // at most 128 chunks x 256 experts
        CUDA_TRY(cudaFuncSetAttribute(scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SCAN_SMEM_MAX));
        LAUNCH(h->pdl, "scan_kernel", scan_kernel, 1, 256, scan_smem, st, chunk, nchunks, c.E, v.counts, v.offsets, v.tiles,
               v.num_tiles, v.tile_ptr, v.pick, h->picker, gu_done_of(h, ws));
        if (A == 0) return MOE_OK;
        LAUNCH(h->pdl, "rank_kernel", rank_kernel, nchunks, DISPATCH_CHUNK, 0, st, ids, A, c.E, chunk, v.perm, v.inv);
    }
    const int qgrid = std::min((T + 7) / 8, 8 * h->num_sms);
    if (c.fmt == MOE_FMT_NVFP4) {
        int32_t* amax = reinterpret_cast<int32_t*>(v.x_global);
        CUDA_TRY(cudaMemsetAsync(amax, 0, sizeof(int32_t), st));
        const long long n8 = static_cast<long long>(T) * c.H / 8;
        LAUNCH(h->pdl, "amax_kernel", amax_kernel,
               static_cast<int>(std::min<long long>((n8 + 255) / 256, 4LL * h->num_sms)), 256, 0, st,
               static_cast<const __nv_bfloat16*>(x), n8, amax);
        LAUNCH(h->pdl, "quant_scatter_nvfp4_kernel", quant_scatter_nvfp4_kernel, qgrid, 256, 0, st,
               static_cast<const __nv_bfloat16*>(x), T, c.H, c.k, ids, v.inv, v.offsets, v.tile_ptr,
               static_cast<const int32_t*>(amax), v.xq, static_cast<uint8_t*>(v.xs));
        return MOE_OK;
    }
    if (T <= 4 * h->num_sms) {
        // one CTA per token while the batch leaves SMs to spare
        LAUNCH(h->pdl, "quant_scatter_row_kernel",
               c.fmt == MOE_FMT_FP8_ROW ? quant_scatter_row_kernel<0> : quant_scatter_row_kernel<1>, T, 256, 0, st,
               static_cast<const __nv_bfloat16*>(x), T, c.H, c.k, static_cast<const int32_t*>(v.inv), v.xq,
               static_cast<float*>(v.xs));
        return MOE_OK;
    }
    LAUNCH(h->pdl, "quant_scatter_kernel",
           c.fmt == MOE_FMT_FP8_ROW ? quant_scatter_kernel<0> : quant_scatter_kernel<1>, qgrid, 256, 0, st,
           static_cast<const __nv_bfloat16*>(x), T, c.H, c.k, static_cast<const int32_t*>(v.inv), v.xq,
           static_cast<float*>(v.xs));
    return MOE_OK;
}

// ------------------------------------------------------------------ NVFP4 GEMMs
static int max_m_tiles(const moe_config& c, int T);

template <int KIND, int ACT = 0>
static moe_status launch_fp4(bool pdl, const CUtensorMap& ta, const CUtensorMap& tb, const Fp4Params& p, int grid,
                             cudaStream_t st) {
    auto kern = grouped_gemm_fp4_kernel<KIND, ACT>;
    constexpr int smem = Fp4Layout<KIND, ACT>::TOTAL;
    CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    LAUNCH(pdl, "grouped_gemm_fp4_kernel", kern, grid, GEMM_THREADS, smem, st, ta, tb, p);
    return MOE_OK;
}

static moe_status fp4_gemm(const moe_handle* h, const void* packed, const float* w, int T, void* ws,
                           moe_stream_t stream, bool gate_up) {
    const moe_config& c = h->cfg;
    moe_workspace_view v;
    moe_workspace_view_get(h, ws, &v);
    const uint8_t* pw = static_cast<const uint8_t*>(packed);
    const size_t R = padded_rows(c);
    const int K = gate_up ? c.H : c.I;
    const int N = gate_up ? (c.act == MOE_ACT_RELU2 ? c.I : 2 * c.I) : c.H;
    CUtensorMap ta, tb;
    moe_status r = make_tmap(&ta, gate_up ? v.xq : v.hq, K / 2, R, K / 2, 128, 128);
    if (r != MOE_OK) return r;
    // gated gate/up (two packed 64 gate + 64 up blocks) and down: 256-row
    // tiles of B; ReLU^2 gate/up: 128-row tiles
    const int bn = (gate_up && c.act == MOE_ACT_RELU2) ? 128 : 256;
    r = make_tmap(&tb, pw + (gate_up ? h->wl.gu_q : h->wl.d_q), K / 2, static_cast<uint64_t>(c.E) * N, K / 2, 128,
                  bn);
    if (r != MOE_OK) return r;
    Fp4Params p;
    memset(&p, 0, sizeof(p));
    p.tiles = v.tiles;
    p.num_tiles = v.num_tiles;
    p.tile_ptr = v.tile_ptr;
    p.offsets = v.offsets;
    p.E = c.E;
    p.n_blocks = N / bn;
    p.num_kb = K / 256;
    p.sf_cols = K / 16;
    p.b_rows = N;
    p.sfa = static_cast<const uint8_t*>(gate_up ? v.xs : v.hs);
    p.sfb = pw + (gate_up ? h->wl.gu_s : h->wl.d_s);
    p.x_amax = reinterpret_cast<const int32_t*>(v.x_global);
    p.w_global = reinterpret_cast<const float*>(pw + (gate_up ? h->wl.gu_g : h->wl.d_g));
    p.h_global = c.hidden_global_scale;
    p.act = c.act;
    p.act_alpha = c.act_alpha;
    p.act_limit = c.act_limit;
    p.hq = v.hq;
    p.hsf = static_cast<uint8_t*>(v.hs);
    p.I = c.I;
    p.o = v.o;
    p.oe = v.o_exp;
    p.H = c.H;
    p.perm = v.perm;
    p.route_w = w;
    p.status = v.status;
    p.spin_limit = h->spin_limit;
    const int grid = std::max(1, std::min(h->num_sms, max_m_tiles(c, T) * p.n_blocks));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (!gate_up) return launch_fp4<KIND_DOWN>(h->pdl, ta, tb, p, grid, st);
    switch (c.act) {
    case MOE_ACT_SWIGLU_BOUNDED: return launch_fp4<KIND_GATE_UP, MOE_ACT_SWIGLU_BOUNDED>(h->pdl, ta, tb, p, grid, st);
    case MOE_ACT_SWIGLU_OAI: return launch_fp4<KIND_GATE_UP, MOE_ACT_SWIGLU_OAI>(h->pdl, ta, tb, p, grid, st);
    case MOE_ACT_GEGLU: return launch_fp4<KIND_GATE_UP, MOE_ACT_GEGLU>(h->pdl, ta, tb, p, grid, st);
    case MOE_ACT_REGLU: return launch_fp4<KIND_GATE_UP, MOE_ACT_REGLU>(h->pdl, ta, tb, p, grid, st);
    case MOE_ACT_RELU2: return launch_fp4<KIND_GATE_UP, MOE_ACT_RELU2>(h->pdl, ta, tb, p, grid, st);
    default: return launch_fp4<KIND_GATE_UP, MOE_ACT_SWIGLU>(h->pdl, ta, tb, p, grid, st);
    }
}

// ------------------------------------------------------------------ tensor maps
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2D byte matrix [rows][inner] with row pitch `pitch`, boxes of box_inner
// bytes x box_rows rows, 128-byte swizzled (else stored as they are in memory);
// rows past the end read as zero.
static moe_status make_tmap(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch,
                            uint32_t box_inner, uint32_t box_rows, bool swizzle) {
    auto fn = encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {pitch};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    return MOE_OK;
}

template <int KIND, int BSCALE, bool PROMOTE, int BN, int STAGES, int EPI = 8, int ACT = 0>
static moe_status launch_gemm(bool pdl, const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p, int grid,
                              cudaStream_t st) {
    using S = GemmSmem<BN, STAGES, EPI>;
    static_assert(S::TOTAL <= 232448, "shared memory of the GEMM exceeds 227 KB");
    auto kern = grouped_gemm_kernel<KIND, BSCALE, PROMOTE, BN, STAGES, EPI, ACT>;
    CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::TOTAL));
    LAUNCH(pdl, "grouped_gemm_kernel", kern, grid, (gemm_threads<EPI, PROMOTE>()), S::TOTAL, st, ta, tb, p);
    return MOE_OK;
}

// The gated FP8_ROW gate/up GEMM as 2-CTA clusters running the picked mode
template <int ACT>
static cudaError_t launch_gu_poly(bool pdl, int grid, cudaStream_t st, const CUtensorMap& ta, const CUtensorMap& tb256,
                                  const CUtensorMap& tb128, const CUtensorMap& tb64, const GemmParams& p,
                                  const int32_t* mode) {
    auto kern = grouped_gemm_gu_poly_kernel<ACT>;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GU_POLY_SMEM);
    if (e != cudaSuccess) return e;
    return launch_k_pairs(pdl, kern, dim3(grid), dim3(gemm_threads<16>()), GU_POLY_SMEM, st, ta, tb256, tb128, tb64, p,
                          mode);
}

// upper bound of the m-tiles the schedule can hold for T tokens
static int max_m_tiles(const moe_config& c, int T) {
    const int A = T * c.k;
    return A / TILE_M + std::min(c.E, A);
}

// ------------------------------------------------------------------ gate/up
// publish: the FP8_ROW gate/up epilogue counts each finished part of a tile
// per expert (a fence and an atomic per warp and tile) for a down GEMM chained
// behind it (mx_down with chained = true); without such a consumer it does not.
static moe_status gate_up_impl(const moe_handle* h, const void* packed, int T, void* ws, moe_stream_t stream,
                               bool publish);

extern "C" moe_status moe_gate_up(const moe_handle* h, const void* packed, int T, void* ws, moe_stream_t stream) {
    return gate_up_impl(h, packed, T, ws, stream, false);
}

static moe_status gate_up_impl(const moe_handle* h, const void* packed, int T, void* ws, moe_stream_t stream,
                               bool publish) {
    moe_status st0 = check_T(h, T, "moe_gate_up");
    if (st0 != MOE_OK) return st0;
    if (T == 0) return MOE_OK;
    if (!packed || !ws) return fail(MOE_ERR_INVALID_ARG, "moe_gate_up: null argument");
    if (!aligned256(packed) || !aligned256(ws)) return fail(MOE_ERR_INVALID_ARG, "moe_gate_up: pointers must be 256-byte aligned");
    if (h->cfg.fmt == MOE_FMT_NVFP4) return fp4_gemm(h, packed, nullptr, T, ws, stream, true);
    const moe_config& c = h->cfg;
    moe_workspace_view v;
    moe_workspace_view_get(h, ws, &v);
    const uint8_t* pw = static_cast<const uint8_t*>(packed);
    CUtensorMap ta, tb;
    moe_status r = make_tmap(&ta, v.xq, c.H, padded_rows(c), c.H, GEMM_BK, GEMM_BM);
    if (r != MOE_OK) return r;
    const int n_gu = c.act == MOE_ACT_RELU2 ? c.I : 2 * c.I;   // rows of the packed gate/up weights
    r = make_tmap(&tb, pw + h->wl.gu_q, c.H, static_cast<uint64_t>(c.E) * n_gu, c.H, GEMM_BK, 256);
    if (r != MOE_OK) return r;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.tiles = v.tiles;
    p.num_tiles = v.num_tiles;
    p.tile_ptr = v.tile_ptr;
    p.E = c.E;
    p.offsets = v.offsets;
    p.n_blocks = n_gu / 256;
    p.num_kb = c.H / GEMM_BK;
    p.b_rows = n_gu;
    p.a_scale = static_cast<const float*>(v.xs);
    p.a_ld = (c.fmt == MOE_FMT_FP8_ROW) ? 1 : c.H / 128;
    p.b_scale = reinterpret_cast<const float*>(pw + h->wl.gu_s);
    p.hq = v.hq;
    p.hs = static_cast<float*>(v.hs);
    p.hsf = static_cast<uint8_t*>(v.hs);
    p.I = c.I;
    p.H = c.H;
    p.act = c.act;
    p.act_alpha = c.act_alpha;
    p.act_limit = c.act_limit;
    p.gu_done = (c.fmt == MOE_FMT_FP8_ROW && publish) ? gu_done_of(h, ws) : nullptr;
    p.status = v.status;
    p.spin_limit = h->spin_limit;
    const int grid = std::max(1, std::min(h->num_sms, max_m_tiles(c, T) * p.n_blocks));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (c.fmt == MOE_FMT_FP8_ROW && c.act != MOE_ACT_RELU2) {
        // 2-CTA clusters that run the mode the dispatch picked (pick[2]): single
        // CTAs on 256- or 128-wide tiles, or CTA pairs; weight maps with boxes of
        // 256 rows (wide), 128 (half of a pair's tile) and 64 (narrow: 64 gate
        // rows, then the 64 matching up rows); an even grid that covers the
        // largest unit count of the three
        CUtensorMap tb128, tb64;
        r = make_tmap(&tb128, pw + h->wl.gu_q, c.H, static_cast<uint64_t>(c.E) * n_gu, c.H, GEMM_BK, 128);
        if (r != MOE_OK) return r;
        r = make_tmap(&tb64, pw + h->wl.gu_q, c.H, static_cast<uint64_t>(c.E) * n_gu, c.H, GEMM_BK, 64);
        if (r != MOE_OK) return r;
        const int g2 = std::max(2, (std::min(h->num_sms, max_m_tiles(c, T) * 2 * p.n_blocks) + 1) / 2 * 2);
        static_assert(GU_POLY_SMEM <= 232448, "shared memory of the GEMM exceeds 227 KB");
        const int32_t* mode = static_cast<const int32_t*>(v.pick + 2);
        cudaError_t err;
        switch (c.act) {
        case MOE_ACT_SWIGLU_BOUNDED:
            err = launch_gu_poly<MOE_ACT_SWIGLU_BOUNDED>(h->pdl, g2, st, ta, tb, tb128, tb64, p, mode);
            break;
        case MOE_ACT_SWIGLU_OAI:
            err = launch_gu_poly<MOE_ACT_SWIGLU_OAI>(h->pdl, g2, st, ta, tb, tb128, tb64, p, mode);
            break;
        case MOE_ACT_GEGLU:
            err = launch_gu_poly<MOE_ACT_GEGLU>(h->pdl, g2, st, ta, tb, tb128, tb64, p, mode);
            break;
        case MOE_ACT_REGLU:
            err = launch_gu_poly<MOE_ACT_REGLU>(h->pdl, g2, st, ta, tb, tb128, tb64, p, mode);
            break;
        default:
            err = launch_gu_poly<MOE_ACT_SWIGLU>(h->pdl, g2, st, ta, tb, tb128, tb64, p, mode);
            break;
        }
        if (err != cudaSuccess)
            return fail(MOE_ERR_CUDA, "launch of grouped_gemm_gu_poly_kernel failed: %s", cudaGetErrorString(err));
        return MOE_OK;
    }
    if (c.fmt == MOE_FMT_FP8_ROW)   // ReLU^2: the up projection alone, 256 rows per tile
        return launch_gemm<KIND_GATE_UP, BSCALE_ROW, false, 256, 4, 16, MOE_ACT_RELU2>(h->pdl, ta, tb, p, grid, st);
    switch (c.act) {
    case MOE_ACT_SWIGLU_BOUNDED:
        return launch_gemm<KIND_GATE_UP, BSCALE_BLOCK128, true, 256, 4, 8, MOE_ACT_SWIGLU_BOUNDED>(h->pdl, ta, tb, p, grid, st);
    case MOE_ACT_SWIGLU_OAI:
        return launch_gemm<KIND_GATE_UP, BSCALE_BLOCK128, true, 256, 4, 8, MOE_ACT_SWIGLU_OAI>(h->pdl, ta, tb, p, grid, st);
    case MOE_ACT_GEGLU:
        return launch_gemm<KIND_GATE_UP, BSCALE_BLOCK128, true, 256, 4, 8, MOE_ACT_GEGLU>(h->pdl, ta, tb, p, grid, st);
    case MOE_ACT_REGLU:
        return launch_gemm<KIND_GATE_UP, BSCALE_BLOCK128, true, 256, 4, 8, MOE_ACT_REGLU>(h->pdl, ta, tb, p, grid, st);
    case MOE_ACT_RELU2:
        return launch_gemm<KIND_GATE_UP, BSCALE_BLOCK128, true, 256, 4, 8, MOE_ACT_RELU2>(h->pdl, ta, tb, p, grid, st);
    default:
        return launch_gemm<KIND_GATE_UP, BSCALE_BLOCK128, true, 256, 4, 8, MOE_ACT_SWIGLU>(h->pdl, ta, tb, p, grid, st);
    }
}

// ------------------------------------------------------------------ down
// FP8_ROW: MX-scaled hidden (tensor cores apply its scales), one tile width.
// chained: launched right after this call's gate/up GEMM (moe_forward_routed);
// the kernel then waits per expert for the gate/up parts instead of for the
// whole gate/up kernel, so down tiles of finished experts overlap its tail.
static moe_status mx_down(const moe_handle* h, const void* packed, const float* w, int T, void* ws,
                          moe_stream_t stream, bool chained) {
    const moe_config& c = h->cfg;
    moe_workspace_view v;
    moe_workspace_view_get(h, ws, &v);
    const uint8_t* pw = static_cast<const uint8_t*>(packed);
    // Large batches with deep K: CTA pairs (M = 256), each CTA loading 128 of a
    // tile's 256 B rows, when the experts average at least 4 row tiles (as for
    // the gate/up GEMM) and no K split can be chosen; shallow K keeps single
    // CTAs and the box stores.
    const bool pairs = c.I / 128 > MX_BOX_MAX_KB && split_limit(h->picker, T * c.k) == 1 &&
                       (h->gemm_pairs == 2 || (h->gemm_pairs == 1 && T * c.k >= 4 * TILE_M * c.E)) &&
                       h->down_bn != 128;
    // 128-wide tiles with two accumulators in TMEM (moe_set_tile_config(h, 128))
    const bool narrow = !pairs && h->down_bn == 128;
    const int bn = narrow ? 128 : MX_BN;
    CUtensorMap ta, tb, to, ts;
    moe_status r = make_tmap(&ta, v.hq, c.I, hidden_rows(c), c.I, GEMM_BK, GEMM_BM);
    if (r != MOE_OK) return r;
    r = make_tmap(&tb, pw + h->wl.d_q, c.I, static_cast<uint64_t>(c.E) * c.H, c.I, GEMM_BK, pairs ? MX_BN / 2 : bn);
    if (r != MOE_OK) return r;
    // hidden scales as rows of 256 bytes (a 512-byte chunk per row tile and K
    // stage is two rows), copied as they are: the pairs' scale loads
    const uint64_t hs_bytes = hidden_rows(c) * hidden_scale_bytes(c.fmt, c.I);
    r = make_tmap(&ts, v.hs, 256, hs_bytes / 256, 256, 256, 2, false);
    if (r != MOE_OK) return r;
    // output rows (fp16 as bytes): boxes of 32 rows x 64 values for the epilogue's stores
    r = make_tmap(&to, v.o, static_cast<uint64_t>(c.H) * 2, o_rows(c), static_cast<uint64_t>(c.H) * 2, 128, 32);
    if (r != MOE_OK) return r;
    MxDownParams p;
    memset(&p, 0, sizeof(p));
    p.tiles = v.tiles;
    p.num_tiles = v.num_tiles;
    p.tile_ptr = v.tile_ptr;
    p.offsets = v.offsets;
    p.E = c.E;
    p.n_blocks = c.H / bn;
    p.num_kb = c.I / 128;
    p.b_rows = c.H;
    p.sfa = static_cast<const uint8_t*>(v.hs);
    p.w_scale = reinterpret_cast<const float*>(pw + h->wl.d_s);
    p.o = v.o;
    p.oe = v.o_exp;
    p.H = c.H;
    p.A = T * c.k;
    p.split = v.pick + 1;
    p.s_max = split_limit(h->picker, p.A);
    p.gu_done = chained ? gu_done_of(h, ws) : nullptr;
    p.gu_per_mtile = ((c.act == MOE_ACT_RELU2 ? c.I : 2 * c.I) / 256) * 16;   // gate/up n-blocks x 16 epilogue warps
    p.perm = v.perm;
    p.route_w = w;
    p.status = v.status;
    p.spin_limit = h->spin_limit;
    const int grid = std::max(1, std::min(h->num_sms, max_m_tiles(c, T) * p.n_blocks * p.s_max));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (pairs) {
        using Lp = MxSmem<MX_PAIR_STAGES, false, true>;
        auto kern = grouped_gemm_mx_down_kernel<MX_PAIR_STAGES, false, true>;
        const int npairs = std::max(1, std::min(h->num_sms / 2, (max_m_tiles(c, T) + 1) / 2 * p.n_blocks * p.s_max));
        CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lp::TOTAL));
        const cudaError_t err =
            launch_k_pairs(h->pdl, kern, dim3(2 * npairs), dim3(GEMM_THREADS), Lp::TOTAL, st, ta, tb, to, ts, p);
        if (err != cudaSuccess)
            return fail(MOE_ERR_CUDA, "launch of grouped_gemm_mx_down_kernel (pairs) failed: %s", cudaGetErrorString(err));
        return MOE_OK;
    }
    if (narrow && p.num_kb <= MX_BOX_MAX_KB) {
        using Ln = MxSmem<MX_NARROW_BOX_STAGES, true, false, 128>;
        auto kern = grouped_gemm_mx_down_kernel<MX_NARROW_BOX_STAGES, true, false, 128>;
        CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ln::TOTAL));
        LAUNCH(h->pdl, "grouped_gemm_mx_down_kernel", kern, grid, GEMM_THREADS, Ln::TOTAL, st, ta, tb, to, ts, p);
    } else if (narrow) {
        using Ln = MxSmem<MX_NARROW_STAGES, false, false, 128>;
        auto kern = grouped_gemm_mx_down_kernel<MX_NARROW_STAGES, false, false, 128>;
        CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ln::TOTAL));
        LAUNCH(h->pdl, "grouped_gemm_mx_down_kernel", kern, grid, GEMM_THREADS, Ln::TOTAL, st, ta, tb, to, ts, p);
    } else if (p.num_kb <= MX_BOX_MAX_KB) {
        using Lb = MxSmem<3, true>;
        auto kern = grouped_gemm_mx_down_kernel<3, true>;
        CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lb::TOTAL));
        LAUNCH(h->pdl, "grouped_gemm_mx_down_kernel", kern, grid, GEMM_THREADS, Lb::TOTAL, st, ta, tb, to, ts, p);
    } else {
        using Lr = MxSmem<4, false>;
        auto kern = grouped_gemm_mx_down_kernel<4, false>;
        CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lr::TOTAL));
        LAUNCH(h->pdl, "grouped_gemm_mx_down_kernel", kern, grid, GEMM_THREADS, Lr::TOTAL, st, ta, tb, to, ts, p);
    }
    return MOE_OK;
}

extern "C" moe_status moe_down(const moe_handle* h, const void* packed, const float* w, int T, void* ws,
                               moe_stream_t stream) {
    moe_status st0 = check_T(h, T, "moe_down");
    if (st0 != MOE_OK) return st0;
    if (T == 0) return MOE_OK;
    if (!packed || !ws || !w) return fail(MOE_ERR_INVALID_ARG, "moe_down: null argument");
    if (!aligned256(packed) || !aligned256(ws)) return fail(MOE_ERR_INVALID_ARG, "moe_down: pointers must be 256-byte aligned");
    if (h->cfg.fmt == MOE_FMT_NVFP4) return fp4_gemm(h, packed, w, T, ws, stream, false);
    if (h->cfg.fmt == MOE_FMT_FP8_ROW) return mx_down(h, packed, w, T, ws, stream, false);
    const moe_config& c = h->cfg;
    moe_workspace_view v;
    moe_workspace_view_get(h, ws, &v);
    const uint8_t* pw = static_cast<const uint8_t*>(packed);
    const int BN = h->down_bn ? h->down_bn : 256;
    CUtensorMap ta, tb, tb128, tb64;
    moe_status r = make_tmap(&ta, v.hq, c.I, hidden_rows(c), c.I, GEMM_BK, GEMM_BM);
    if (r != MOE_OK) return r;
    r = make_tmap(&tb, pw + h->wl.d_q, c.I, static_cast<uint64_t>(c.E) * c.H, c.I, GEMM_BK, BN);
    if (r != MOE_OK) return r;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.tiles = v.tiles;
    p.num_tiles = v.num_tiles;
    p.tile_ptr = v.tile_ptr;
    p.E = c.E;
    p.offsets = v.offsets;
    p.n_blocks = c.H / BN;
    p.num_kb = c.I / GEMM_BK;
    p.b_rows = c.H;
    p.a_scale = static_cast<const float*>(v.hs);
    p.a_ld = c.I / 128;
    p.b_scale = reinterpret_cast<const float*>(pw + h->wl.d_s);
    p.o = v.o;
    p.oe = v.o_exp;
    p.H = c.H;
    p.I = c.I;
    p.perm = v.perm;
    p.route_w = w;
    p.status = v.status;
    p.spin_limit = h->spin_limit;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (h->down_bn == 0) {
        // tile width chosen on the device from the histogram (scan kernel)
        r = make_tmap(&tb128, pw + h->wl.d_q, c.I, static_cast<uint64_t>(c.E) * c.H, c.I, GEMM_BK, 128);
        if (r != MOE_OK) return r;
        r = make_tmap(&tb64, pw + h->wl.d_q, c.I, static_cast<uint64_t>(c.E) * c.H, c.I, GEMM_BK, 64);
        if (r != MOE_OK) return r;
        const int grid = std::max(1, std::min(h->num_sms, max_m_tiles(c, T) * (c.H / 64)));
        CUDA_TRY(cudaFuncSetAttribute(down_gemm_poly_kernel<BSCALE_BLOCK128>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, POLY_SMEM));
        LAUNCH(h->pdl, "down_gemm_poly_kernel", down_gemm_poly_kernel<BSCALE_BLOCK128>, grid, (gemm_threads<8, true>()),
               POLY_SMEM, st, ta, tb, tb128, tb64, p, static_cast<const int32_t*>(v.pick));
        return MOE_OK;
    }
    const int grid = std::max(1, std::min(h->num_sms, max_m_tiles(c, T) * p.n_blocks));
    if (BN == 256) return launch_gemm<KIND_DOWN, BSCALE_BLOCK128, true, 256, 4>(h->pdl, ta, tb, p, grid, st);
    if (BN == 128) return launch_gemm<KIND_DOWN, BSCALE_BLOCK128, true, 128, 6>(h->pdl, ta, tb, p, grid, st);
    return launch_gemm<KIND_DOWN, BSCALE_BLOCK128, true, 64, 8>(h->pdl, ta, tb, p, grid, st);
}

extern "C" moe_status moe_set_picker_params(moe_handle* h, const long long* params) {
    if (!h || !params) return fail(MOE_ERR_INVALID_ARG, "moe_set_picker_params: null argument");
    if (params[0] < 0 || params[1] < 0 || params[2] <= 0 || params[3] < 0)
        return fail(MOE_ERR_INVALID_ARG, "moe_set_picker_params: need alpha, beta, gamma >= 0 and bw > 0");
    h->picker.alpha_ps = params[0];
    h->picker.beta_ps = params[1];
    h->picker.bw_cta = params[2];
    h->picker.gamma_ps = params[3];
    return MOE_OK;
}

extern "C" moe_status moe_get_picker_params(const moe_handle* h, long long* params) {
    if (!h || !params) return fail(MOE_ERR_INVALID_ARG, "moe_get_picker_params: null argument");
    params[0] = h->picker.alpha_ps;
    params[1] = h->picker.beta_ps;
    params[2] = h->picker.bw_cta;
    params[3] = h->picker.gamma_ps;
    params[4] = h->picker.num_sms;
    return MOE_OK;
}

extern "C" moe_status moe_set_gate_up_model(moe_handle* h, const long long* params) {
    if (!h || !params) return fail(MOE_ERR_INVALID_ARG, "moe_set_gate_up_model: null argument");
    for (int i = 0; i < 6; i++)
        if (params[i] < 0) return fail(MOE_ERR_INVALID_ARG, "moe_set_gate_up_model: costs must be >= 0");
    for (int i = 0; i < 6; i++) h->picker.gu_ps[i] = params[i];
    return MOE_OK;
}

extern "C" moe_status moe_get_gate_up_model(const moe_handle* h, long long* params) {
    if (!h || !params) return fail(MOE_ERR_INVALID_ARG, "moe_get_gate_up_model: null argument");
    for (int i = 0; i < 6; i++) params[i] = h->picker.gu_ps[i];
    params[6] = h->picker.gu_nb;
    params[7] = h->picker.gu_kb;
    params[8] = h->picker.num_sms;
    params[9] = h->picker.gu_allow;
    return MOE_OK;
}

extern "C" moe_status moe_set_tile_config(moe_handle* h, int down_bn) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "moe_set_tile_config: null handle");
    if (down_bn != 0 && down_bn != 64 && down_bn != 128 && down_bn != 256)
        return fail(MOE_ERR_INVALID_ARG, "moe_set_tile_config: down_bn must be 0, 64, 128 or 256 (got %d)", down_bn);
    h->down_bn = down_bn;
    return MOE_OK;
}

extern "C" moe_status moe_set_wait_limit(moe_handle* h, long long cycles) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "moe_set_wait_limit: null handle");
    if (cycles <= 0) return fail(MOE_ERR_INVALID_ARG, "moe_set_wait_limit: cycles must be positive (got %lld)", cycles);
    h->spin_limit = cycles;
    return MOE_OK;
}

extern "C" moe_status moe_set_launch_options(moe_handle* h, int pdl) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "moe_set_launch_options: null handle");
    if (pdl != 0 && pdl != 1) return fail(MOE_ERR_INVALID_ARG, "moe_set_launch_options: pdl must be 0 or 1 (got %d)", pdl);
    h->pdl = pdl;
    return MOE_OK;
}

extern "C" moe_status moe_set_gate_up_tile(moe_handle* h, int bn) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "moe_set_gate_up_tile: null handle");
    if (bn != 0 && bn != 128 && bn != 256)
        return fail(MOE_ERR_INVALID_ARG, "moe_set_gate_up_tile: bn must be 0, 128 or 256 (got %d)", bn);
    if (bn == 128 && (h->cfg.fmt != MOE_FMT_FP8_ROW || h->cfg.act == MOE_ACT_RELU2))
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_set_gate_up_tile: 128-wide tiles need a gated FP8_ROW layer");
    const int allow = gu_allow_of(h->gemm_pairs, bn);
    if (allow == 0)
        return fail(MOE_ERR_INVALID_ARG, "moe_set_gate_up_tile: 128-wide tiles contradict CTA pairs forced on");
    h->gu_bn = bn;
    h->picker.gu_allow = allow;
    return MOE_OK;
}

extern "C" moe_status moe_set_gemm_options(moe_handle* h, int cta_pairs) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "moe_set_gemm_options: null handle");
    if (cta_pairs < 0 || cta_pairs > 2)
        return fail(MOE_ERR_INVALID_ARG, "moe_set_gemm_options: cta_pairs must be 0, 1 or 2 (got %d)", cta_pairs);
    const int allow = gu_allow_of(cta_pairs, h->gu_bn);
    if (allow == 0)
        return fail(MOE_ERR_INVALID_ARG, "moe_set_gemm_options: CTA pairs contradict 128-wide gate/up tiles forced on");
    h->gemm_pairs = cta_pairs;
    h->picker.gu_allow = allow;
    return MOE_OK;
}

// ------------------------------------------------------------------ combine
extern "C" moe_status moe_combine(const moe_handle* h, int T, void* y, void* ws, moe_stream_t stream) {
    moe_status st0 = check_T(h, T, "moe_combine");
    if (st0 != MOE_OK) return st0;
    if (T == 0) return MOE_OK;
    if (!y || !ws) return fail(MOE_ERR_INVALID_ARG, "moe_combine: null argument");
    if (!aligned256(y) || !aligned256(ws)) return fail(MOE_ERR_INVALID_ARG, "moe_combine: pointers must be 256-byte aligned");
    if (T == 0) return MOE_OK;
    moe_workspace_view v;
    moe_workspace_view_get(h, ws, &v);
    const int s_max = split_limit(h->picker, T * h->cfg.k);
    // one CTA per (group of 8 / k tokens, 2048-column slice): small batches still spread.
    // Launched without the PDL attribute: launched early, its CTAs would be
    // placed on the few SMs the down GEMM leaves room on and run ~2x slower
    // (Qwen3.5 T=64: 5.4 vs 2.6 us) than when placed after the GEMM ends.
    constexpr int span = COMBINE_COLS * COMBINE_THREADS;
    const int ncb = (h->cfg.H + span - 1) / span;
    const int groups = (T + combine_group(h->cfg.k) - 1) / combine_group(h->cfg.k);
    const dim3 grid(std::max(1, std::min(groups, 16 * h->num_sms / ncb)), ncb);
    LAUNCH(false, "combine_kernel", combine_kernel, grid, COMBINE_THREADS, 0, reinterpret_cast<cudaStream_t>(stream),
           static_cast<const uint16_t*>(v.o), static_cast<const int8_t*>(v.o_exp), static_cast<const int32_t*>(v.inv),
           T, h->cfg.H, h->cfg.k,
           static_cast<const int32_t*>(h->cfg.fmt == MOE_FMT_FP8_ROW ? v.pick + 1 : nullptr), s_max,
           static_cast<__nv_bfloat16*>(y));
    return MOE_OK;
}

// ------------------------------------------------------------------ layer
constexpr long long CHAIN_MAX_A = 4096;

extern "C" moe_status moe_forward_routed(const moe_handle* h, const void* x, int T, const int32_t* ids, const float* w,
                                         const void* packed, void* y, void* ws, moe_stream_t stream) {
    moe_status r = moe_dispatch(h, x, ids, T, ws, stream);
    if (r != MOE_OK) return r;
    // FP8_ROW batches of at most CHAIN_MAX_A assignments chain the down GEMM
    // behind the gate/up GEMM (per-expert waits, so it starts on the SMs the
    // gate/up GEMM's last wave leaves idle); larger batches fill every SM with
    // gate/up tiles to the end, where the per-tile counting only costs time
    const bool chained = h->cfg.fmt == MOE_FMT_FP8_ROW && T > 0 && h->pdl &&
                         static_cast<long long>(T) * h->cfg.k <= CHAIN_MAX_A;
    r = gate_up_impl(h, packed, T, ws, stream, chained);
    if (r != MOE_OK) return r;
    if (chained) {
        if (!w) return fail(MOE_ERR_INVALID_ARG, "moe_forward_routed: null argument");
        r = mx_down(h, packed, w, T, ws, stream, true);
    } else {
        r = moe_down(h, packed, w, T, ws, stream);
    }
    if (r != MOE_OK) return r;
    return moe_combine(h, T, y, ws, stream);
}

extern "C" moe_status moe_forward(const moe_handle* h, const void* x, int T, const float* wr, const float* bias,
                                  const void* packed, void* y, void* ws, moe_stream_t stream) {
    moe_status st0 = check_T(h, T, "moe_forward");
    if (st0 != MOE_OK) return st0;
    if (!ws) return fail(MOE_ERR_INVALID_ARG, "moe_forward: null workspace");
    moe_workspace_view v;
    moe_workspace_view_get(h, ws, &v);
    moe_status r = moe_route(h, x, T, wr, bias, v.ids, v.w, ws, stream);
    if (r != MOE_OK) return r;
    return moe_forward_routed(h, x, T, v.ids, v.w, packed, y, ws, stream);
}

// ------------------------------------------------------------------ status
extern "C" moe_status moe_workspace_init(const moe_handle* h, void* ws, moe_stream_t stream) {
    if (!h || !ws) return fail(MOE_ERR_INVALID_ARG, "moe_workspace_init: null argument");
    CUDA_TRY(cudaMemsetAsync(static_cast<uint8_t*>(ws) + h->ws.status, 0, 64 * 4,
                             reinterpret_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

extern "C" moe_status moe_get_status(const moe_handle* h, void* ws, moe_stream_t stream) {
    if (!h || !ws) return fail(MOE_ERR_INVALID_ARG, "moe_get_status: null argument");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    CUDA_TRY(cudaStreamSynchronize(st));
    int32_t s[2] = {0, 0};
    int32_t* dev = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + h->ws.status);
    CUDA_TRY(cudaMemcpy(s, dev, sizeof(s), cudaMemcpyDeviceToHost));
    if (s[0] == 0) return MOE_OK;
    CUDA_TRY(cudaMemset(dev, 0, sizeof(s)));
    static const char* where[] = {"?", "GEMM producer", "GEMM MMA issuer", "GEMM epilogue", "dispatch",
                                  "router", "combine", "GEMM schedule"};
    const char* wn = (s[1] >= 0 && s[1] < 8) ? where[s[1]] : "?";
    if (s[0] == MOE_ERR_DEVICE_TIMEOUT) return fail(MOE_ERR_DEVICE_TIMEOUT, "device wait ran out in %s", wn);
    if (s[0] == MOE_ERR_DEVICE_BOUNDS) return fail(MOE_ERR_DEVICE_BOUNDS, "index out of range in %s", wn);
    return fail(static_cast<moe_status>(s[0]), "device error %d in %s", s[0], wn);
}

// ------------------------------------------------------------------ dispatch without a workspace
// For callers that cannot allocate device memory at all: a service whose host
// framework owns every device allocation and hands the layer only its input
// and output buffers, so there is nowhere to put a caller-sized workspace.
// The only scratch the dispatch needs, the per-chunk expert counts, lives in
// this file-scope device array instead: at most 128 chunks of 1024
// assignments x 256 experts = 128 KB.  Every GPU that loads this library holds
// it until the process exits.
constexpr int NOALLOC_MAX_CHUNKS = 131072 / DISPATCH_CHUNK;
constexpr int NOALLOC_SCRATCH_INTS = NOALLOC_MAX_CHUNKS * 256;
static __device__ __align__(256) int32_t g_dispatch_scratch[NOALLOC_SCRATCH_INTS];

// Device address of g_dispatch_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress with that device current.  The lookup is repeated on
// every call made outside stream capture (a host-side table lookup once the
// module is loaded), so an address cached before a cudaDeviceReset, whose
// context and module are then recreated, is never used afterwards.  Under
// capture the address of the last uncaptured call on the device is used; the
// first call on a device must therefore come before any capture.
static moe_status dispatch_scratch(cudaStream_t st, int32_t** out) {
    static std::mutex mu;
    static int32_t* addr[64] = {nullptr};
    int dev = 0;
    CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return fail(MOE_ERR_CUDA, "moe_dispatch_noalloc: device index %d out of range", dev);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    CUDA_TRY(cudaStreamIsCapturing(st, &cap));
    std::lock_guard<std::mutex> lock(mu);
    if (cap == cudaStreamCaptureStatusNone || !addr[dev]) {
        if (cap != cudaStreamCaptureStatusNone)
            return fail(MOE_ERR_INVALID_ARG,
                        "moe_dispatch_noalloc: the first call on device %d is under stream capture; make one "
                        "call before capturing",
                        dev);
        void* p = nullptr;
        CUDA_TRY(cudaGetSymbolAddress(&p, g_dispatch_scratch));
        addr[dev] = static_cast<int32_t*>(p);
    }
    *out = addr[dev];
    return MOE_OK;
}

extern "C" moe_status moe_dispatch_noalloc(const moe_handle* h, const void* x, const int32_t* ids, int T,
                                           int32_t* counts, int32_t* offsets, int32_t* num_tiles, int32_t* tiles,
                                           int32_t* perm, int32_t* inv, uint8_t* xq, void* xs, int32_t* status,
                                           moe_stream_t stream) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "moe_dispatch_noalloc: null handle");
    const moe_config& c = h->cfg;
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "moe_dispatch_noalloc: T=%d is negative", T);
    const long long A = static_cast<long long>(T) * c.k;
    const long long nchunks = (A + DISPATCH_CHUNK - 1) / DISPATCH_CHUNK;
    // the scan packs each count with its row-tile count into one int32, which
    // holds for at most 131072 assignments whatever E is
    if (A > 131072)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                    "moe_dispatch_noalloc: T*k=%lld assignments, more than the 131072 this entry point handles", A);
    if (nchunks * c.E > NOALLOC_SCRATCH_INTS)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                    "moe_dispatch_noalloc: T*k=%lld assignments need %lld scratch counts, more than the %d "
                    "this library holds (at most 131072 assignments with 256 experts)",
                    A, nchunks * c.E, NOALLOC_SCRATCH_INTS);
    if (c.fmt == MOE_FMT_NVFP4)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_dispatch_noalloc: NVFP4 is not supported");
    if (!counts || !offsets || !num_tiles || !tiles || !status)
        return fail(MOE_ERR_INVALID_ARG, "moe_dispatch_noalloc: null output");
    if (A > 0 && (!x || !ids || !perm || !inv || !xq || !xs))
        return fail(MOE_ERR_INVALID_ARG, "moe_dispatch_noalloc: null argument");
    if (A > 0 && (!aligned256(x) || !aligned256(xq)))
        return fail(MOE_ERR_INVALID_ARG, "moe_dispatch_noalloc: x and xq must be 256-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t* chunk = nullptr;
    moe_status r = dispatch_scratch(st, &chunk);
    if (r != MOE_OK) return r;
    CUDA_TRY(cudaMemsetAsync(status, 0, 2 * sizeof(int32_t), st));
    const int n = static_cast<int>(nchunks), a = static_cast<int>(A);
    // the histogram writes every count of every chunk it covers, so the
    // scratch left by an earlier call needs no clearing
    if (a > 0) {
        hist_kernel<<<n, DISPATCH_CHUNK, 0, st>>>(ids, a, c.E, chunk, status);
        LAUNCH_CHECK("hist_kernel");
    }
    CUDA_TRY(cudaFuncSetAttribute(scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SCAN_SMEM_MAX));
    scan_kernel<<<1, 256, n * c.E * 4, st>>>(chunk, n, c.E, counts, offsets, tiles, num_tiles, nullptr, nullptr, h->picker,
                                   nullptr);
    LAUNCH_CHECK("scan_kernel");
    if (a == 0) return MOE_OK;
    rank_kernel<<<n, DISPATCH_CHUNK, 0, st>>>(ids, a, c.E, chunk, perm, inv);
    LAUNCH_CHECK("rank_kernel");
    const int qgrid = std::min((T + 7) / 8, 8 * h->num_sms);
    if (c.fmt == MOE_FMT_FP8_ROW)
        quant_scatter_kernel<0><<<qgrid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), T, c.H, c.k, inv, xq,
                                                       static_cast<float*>(xs));
    else
        quant_scatter_kernel<1><<<qgrid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), T, c.H, c.k, inv, xq,
                                                       static_cast<float*>(xs));
    LAUNCH_CHECK("quant_scatter_kernel");
    return MOE_OK;
}

#ifdef MOE_TRACE
// Timeline trace of a build made with -DMOE_TRACE: slot 2i holds the earliest
// entry of kernel i, slot 2i+1 its latest warp exit (global timer, ns).
extern "C" int moe_trace_clear(void) {
    unsigned long long init[2 * TRACE_SLOTS];
    for (int i = 0; i < TRACE_SLOTS; i++) {
        init[2 * i] = ~0ull;
        init[2 * i + 1] = 0;
    }
    return cudaMemcpyToSymbol(moe_trace_buf, init, sizeof(init)) == cudaSuccess ? 0 : -1;
}
extern "C" int moe_trace_blk_read(unsigned long long* out) {
    return cudaMemcpyFromSymbol(out, moe::moe_trace_blk, sizeof(unsigned long long) * TRACE_BLKS * 8) == cudaSuccess
               ? 0
               : -1;
}
extern "C" int moe_trace_read(unsigned long long* out) {
    return cudaMemcpyFromSymbol(out, moe_trace_buf, sizeof(unsigned long long) * 2 * TRACE_SLOTS) == cudaSuccess
               ? 0
               : -1;
}
#endif
