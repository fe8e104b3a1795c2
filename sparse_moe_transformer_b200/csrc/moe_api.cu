// moe_api.cu -- host runtime behind include/moe.h: handle, owned weight copies,
// workspace, second stream for the shared expert, TMA descriptors, error words.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "moe.h"
#include "layer.h"

using namespace moe;

namespace {

thread_local char g_err[512] = "";

moe_status fail(moe_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return s;
}

#define CUDA_TRY(expr)                                                                   \
    do {                                                                                 \
        cudaError_t e_ = (expr);                                                         \
        if (e_ != cudaSuccess)                                                           \
            return fail(e_ == cudaErrorMemoryAllocation ? MOE_ERR_OOM : MOE_ERR_CUDA,    \
                        "%s: %s (%s:%d)", #expr, cudaGetErrorString(e_), __FILE__, __LINE__); \
    } while (0)

// Restores the caller's current device on scope exit.
struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(int dev) {
        cudaGetDevice(&prev);
        if (prev != dev) cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        int cur = -1;
        cudaGetDevice(&cur);
        if (prev >= 0 && cur != prev) cudaSetDevice(prev);
    }
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2D bf16 tensor map over a row-major [rows][cols] matrix: boxes of 64 columns
// (one 128-byte swizzle row) by box_rows rows, 128-byte swizzle, zero fill.
moe_status make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    if ((reinterpret_cast<uintptr_t>(base) & 15) || (cols * 2) % 16)
        return fail(MOE_ERR_INVALID_ARG, "tensor map base/stride not 16-byte aligned");
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return MOE_OK;
}

constexpr int kRouteBlock = 16;      // routing block with CUDA-core logits (T < 256)
constexpr int kRouteBlockWide = 128; // routing block after tensor-core logits
constexpr int kNarrow = 32, kWide = 256;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

namespace moe {
// Sets the thread-local moe_last_error text (used by entry points in other files).
void set_last_error(const char* msg) { snprintf(g_err, sizeof g_err, "%s", msg); }
}  // namespace moe

struct moe_layer {
    moe_config cfg;
    Dims d;
    int device = 0;
    int dtype = 1;
    size_t esz = 2;
    bool tc_ok = false;
    int num_sms = 148;
    // owned weight copies
    void *w_router = nullptr, *w_gate = nullptr, *w_up = nullptr, *w_down = nullptr;
    void *ws_gate = nullptr, *ws_up = nullptr, *ws_down = nullptr, *rms_w = nullptr;
    void* w_router_packed = nullptr;   // tensor-core router (E % 128 == 0, no pre-norm)
    void* w_router_kp = nullptr;       // W_r as k-pairs: one-CTA router for a few tokens
    // workspace
    int max_T = 0;
    int max_units = 0;
    char* ws = nullptr;
    RouteBufs rb{};
    void *x_norm = nullptr, *xp = nullptr, *hbuf = nullptr, *obuf = nullptr;
    void *hs = nullptr, *sbuf = nullptr;
    void *x_stage = nullptr, *r_stage = nullptr, *y_stage = nullptr;
    int32_t *sync_routed = nullptr, *sync_shared = nullptr, *sync_router = nullptr;
    int32_t* sync_fused = nullptr;
    float* o_part = nullptr;      // few-token path: [max(I, Is)/128][T*k + T][H] fp32
    bool last_fused = false;      // the last forward took the few-token path
    TcMaps routed_maps{}, shared_maps{};
    // status words
    int* err_dev = nullptr;
    int* err_host = nullptr;
    int* err_host_dev = nullptr;
    // streams
    cudaStream_t s2 = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
    // options
    uint64_t wait_limit_ns = 1000000000ull;
    int inject_stuck = 0, shared_stream = 1, fuse = 1, force_simt = 0, timing = 0;
    int last_T = 0;
    // kernel statistics
    struct Pending { int cls; cudaEvent_t a, b; };
    std::vector<cudaEvent_t> ev_pool;
    std::vector<Pending> pending;
    double k_ms[MOE_KERNEL_CLASSES] = {};
    int64_t k_launches[MOE_KERNEL_CLASSES] = {};

    DeviceStatus status() const { return DeviceStatus{err_dev, err_host_dev}; }
};

namespace {

moe_status copy_weight(void** dst, const void* src, size_t bytes) {
    if (!bytes) return MOE_OK;
    CUDA_TRY(cudaMalloc(dst, bytes));
    CUDA_TRY(cudaMemcpy(*dst, src, bytes, cudaMemcpyDeviceToDevice));
    return MOE_OK;
}

// Allocate and fill a tile-contiguous copy of one or two expert-major matrices
// (see packed_gu_offset / packed_down_offset).
moe_status pack_weight(void** dst, const void* src0, const void* src1, int E, int R, int C) {
    const size_t bytes = src1 ? (size_t)E * R * C * 2 * 2 : packed_down_elems(E, R, C) * 2;
    CUDA_TRY(cudaMalloc(dst, bytes));
    CUDA_TRY(cudaMemset(*dst, 0, bytes));
    CUDA_TRY(launch_pack_tiles(src0, src1, *dst, E, R, C, 0));
    CUDA_TRY(cudaStreamSynchronize(0));
    return MOE_OK;
}

// W_r [R][C] as k-pairs (launch_pack_kpairs) for the one-CTA tensor-core router.
moe_status pack_kpair_weight(void** dst, const void* src, int R, int C) {
    CUDA_TRY(cudaMalloc(dst, (size_t)R * C * 2));
    CUDA_TRY(launch_pack_kpairs(src, *dst, R, C, 0));
    CUDA_TRY(cudaStreamSynchronize(0));
    return MOE_OK;
}

void free_workspace(moe_layer* h) {
    if (h->ws) cudaFree(h->ws);
    h->ws = nullptr;
    h->max_T = 0;
}

moe_status pending_device_error(moe_layer* h) {
    int code = h->err_host ? *(volatile int*)h->err_host : 0;
    if (code == MOE_ERR_TIMEOUT)
        return fail(MOE_ERR_TIMEOUT, "a bounded device-side wait ran out in an earlier call; "
                                     "call moe_check() to clear");
    if (code)
        return fail(MOE_ERR_DEVICE_CHECK, "device-side check failed in an earlier call (%d); "
                                          "call moe_check() to clear", code);
    return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

cudaEvent_t take_event(moe_layer* h) {
    if (!h->ev_pool.empty()) {
        cudaEvent_t e = h->ev_pool.back();
        h->ev_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Counts one launch of class `cls` and, with MOE_OPT_KERNEL_TIMING, brackets it
// with events recorded on the stream the kernel is launched on.
struct KernelScope {
    moe_layer* h;
    int cls;
    cudaStream_t s;
    cudaEvent_t a = nullptr;
    KernelScope(moe_layer* h_, int cls_, cudaStream_t s_) : h(h_), cls(cls_), s(s_) {
        h->k_launches[cls]++;
        if (h->timing) {
            a = take_event(h);
            if (a) cudaEventRecord(a, s);
        }
    }
    ~KernelScope() {
        if (!a) return;
        cudaEvent_t b = take_event(h);
        if (!b) return;
        cudaEventRecord(b, s);
        h->pending.push_back({cls, a, b});
    }
};

}  // namespace

extern "C" {

const char* moe_version(void) { return "sparse_moe_b200 0.1 sm_100a"; }

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_OOM: return "out of memory";
        case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case MOE_ERR_TIMEOUT: return "device-side wait timed out";
        case MOE_ERR_DEVICE_CHECK: return "device-side check failed";
    }
    return "unknown status";
}

const char* moe_last_error(moe_handle) { return g_err; }

moe_status moe_create(const moe_config* cfg, int device, const void* w_router, const void* w_gate,
                      const void* w_up, const void* w_down, const void* ws_gate,
                      const void* ws_up, const void* ws_down, const void* rms_weight,
                      moe_handle* out) {
    if (!cfg || !out) return fail(MOE_ERR_INVALID_ARG, "cfg and out must not be NULL");
    *out = nullptr;
    const moe_config& c = *cfg;
    if (c.hidden <= 0 || c.n_experts <= 0 || c.n_experts > 1024 || c.top_k <= 0 ||
        c.top_k > c.n_experts || c.top_k > 16 || c.expert_inter <= 0 || c.shared_inter < 0)
        return fail(MOE_ERR_INVALID_ARG, "bad layer sizes");
    if (c.dtype != MOE_DTYPE_F32 && c.dtype != MOE_DTYPE_BF16)
        return fail(MOE_ERR_INVALID_ARG, "dtype must be MOE_DTYPE_F32 or MOE_DTYPE_BF16");
    if (c.norm_topk_prob != 1)
        return fail(MOE_ERR_UNSUPPORTED, "only norm_topk_prob = 1 is implemented");
    if (!w_router || !w_gate || !w_up || !w_down)
        return fail(MOE_ERR_INVALID_ARG, "routed weights must not be NULL");
    if (c.shared_inter > 0 && (!ws_gate || !ws_up || !ws_down))
        return fail(MOE_ERR_INVALID_ARG, "shared weights must not be NULL when shared_inter > 0");
    if (rms_weight && !(c.rms_eps >= 0.f))
        return fail(MOE_ERR_INVALID_ARG, "rms_eps must be >= 0");
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev)
        return fail(MOE_ERR_INVALID_ARG, "device %d not available", device);
    DeviceGuard g(device);

    moe_layer* h = new moe_layer();
    h->cfg = c;
    h->d = Dims{c.hidden, c.n_experts, c.top_k, c.expert_inter, c.shared_inter};
    h->device = device;
    h->dtype = c.dtype == MOE_DTYPE_F32 ? 0 : 1;
    h->esz = h->dtype == 0 ? 4 : 2;
    cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, device);
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device);
    h->tc_ok = h->dtype == 1 && major == 10 && minor == 0 && c.hidden % 128 == 0 &&
               c.expert_inter % 128 == 0 && c.shared_inter % 128 == 0;

    const size_t H = c.hidden, E = c.n_experts, I = c.expert_inter, Is = c.shared_inter;
    const size_t es = h->esz;
    moe_status st = MOE_OK;
    auto chk = [&](moe_status s) { if (st == MOE_OK) st = s; };
    chk(copy_weight(&h->w_router, w_router, E * H * es));
    if (h->tc_ok) {
        // tile-contiguous copies: gate/up interleaved in w_gate, w_up unused
        chk(pack_weight(&h->w_gate, w_gate, w_up, (int)E, (int)I, (int)H));
        chk(pack_weight(&h->w_down, w_down, nullptr, (int)E, (int)H, (int)I));
        if (E % 128 == 0 && !rms_weight)
            chk(pack_weight(&h->w_router_packed, w_router, nullptr, 1, (int)E, (int)H));
        if (!rms_weight && router_tc_supported((int)E, (int)H, c.top_k, 1))
            chk(pack_kpair_weight(&h->w_router_kp, w_router, (int)E, (int)H));
        if (Is) {
            chk(pack_weight(&h->ws_gate, ws_gate, ws_up, 1, (int)Is, (int)H));
            chk(pack_weight(&h->ws_down, ws_down, nullptr, 1, (int)H, (int)Is));
        }
    } else {
        chk(copy_weight(&h->w_gate, w_gate, E * I * H * es));
        chk(copy_weight(&h->w_up, w_up, E * I * H * es));
        chk(copy_weight(&h->w_down, w_down, E * H * I * es));
        if (Is) {
            chk(copy_weight(&h->ws_gate, ws_gate, Is * H * es));
            chk(copy_weight(&h->ws_up, ws_up, Is * H * es));
            chk(copy_weight(&h->ws_down, ws_down, H * Is * es));
        }
    }
    if (rms_weight) chk(copy_weight(&h->rms_w, rms_weight, H * es));
    if (st == MOE_OK) {
        cudaError_t e = cudaMalloc(&h->err_dev, sizeof(int));
        if (e == cudaSuccess) e = cudaMemset(h->err_dev, 0, sizeof(int));
        if (e == cudaSuccess) e = cudaHostAlloc(&h->err_host, sizeof(int), cudaHostAllocMapped);
        if (e == cudaSuccess) *h->err_host = 0;
        if (e == cudaSuccess) e = cudaHostGetDevicePointer(&h->err_host_dev, h->err_host, 0);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->s2, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming);
        if (e != cudaSuccess)
            chk(fail(e == cudaErrorMemoryAllocation ? MOE_ERR_OOM : MOE_ERR_CUDA, "create: %s",
                     cudaGetErrorString(e)));
    }
    if (st != MOE_OK) {
        char keep[sizeof g_err];
        memcpy(keep, g_err, sizeof keep);
        moe_destroy(h);
        memcpy(g_err, keep, sizeof keep);
        return st;
    }
    *out = h;
    return MOE_OK;
}

moe_status moe_reserve(moe_handle h, int max_tokens) {
    if (!h || max_tokens < 0) return fail(MOE_ERR_INVALID_ARG, "bad handle or max_tokens");
    if (max_tokens <= h->max_T) return MOE_OK;
    // The kernels index the per-row buffers (T k + T rows of up to max(H, I, I_s)
    // elements) with 32-bit integers.
    const uint64_t width = std::max({(uint64_t)h->d.H, (uint64_t)h->d.I, (uint64_t)h->d.Is});
    if ((uint64_t)max_tokens * (uint64_t)(h->d.k + 1) * width >= (1ull << 31))
        return fail(MOE_ERR_UNSUPPORTED,
                    "max_tokens=%d: T*(k+1)*max(H, I, I_s) must stay below 2^31 "
                    "(32-bit row indexing); split the batch", max_tokens);
    DeviceGuard g(h->device);
    CUDA_TRY(cudaDeviceSynchronize());
    free_workspace(h);
    const size_t T = max_tokens, H = h->d.H, E = h->d.E, k = h->d.k, I = h->d.I, Is = h->d.Is;
    const size_t es = h->esz, S = T * k;
    const size_t nblocks = (T + kRouteBlock - 1) / kRouteBlock;
    const int max_units = (int)((S + kNarrow - 1) / kNarrow + E);
    const int max_shared_units = (int)((T + kNarrow - 1) / kNarrow);

    struct Part { void** ptr; size_t bytes; };
    std::vector<Part> parts = {
        {(void**)&h->rb.logits, T * E * 4},
        {(void**)&h->rb.topk_idx, S * 4},
        {(void**)&h->rb.topk_w, S * 4},
        {(void**)&h->rb.block_hist, nblocks * E * 4},
        {(void**)&h->rb.block_off, nblocks * E * 4},
        {(void**)&h->rb.counts, E * 4},
        {(void**)&h->rb.offsets, (E + 1) * 4},
        {(void**)&h->rb.units, (size_t)max_units * sizeof(Unit)},
        {(void**)&h->rb.n_units, 4},
        {(void**)&h->rb.token_slot, S * 4},
        {(void**)&h->rb.slot_token, S * 4},
        {(void**)&h->rb.slot_expert, S * 4},
        {(void**)&h->rb.tickets, ((T + 7) / 8 + 1) * 4},        // CTA groups of >= 8 tokens
        {(void**)&h->sync_routed, (2 + (size_t)max_units) * 4},
        {(void**)&h->sync_shared, (2 + (size_t)max_shared_units) * 4},
        {(void**)&h->sync_router, (2 + (size_t)max_shared_units) * 4},
        {(void**)&h->sync_fused, 16},
        {(void**)&h->o_part, h->tc_ok ? (size_t)(std::max(I, Is) / 128) *
                                            (std::min<size_t>(S, 1024) + std::min<size_t>(T, 1024)) * H * 4
                                      : 0},
        {&h->x_norm, h->rms_w ? T * H * es : 0},
        {&h->xp, S * H * es},
        {&h->hbuf, S * I * es},
        {&h->obuf, S * H * es},
        {&h->hs, T * (Is ? Is : 1) * es},
        {&h->sbuf, T * H * es},
        {&h->x_stage, T * H * es},
        {&h->r_stage, T * H * es},
        {&h->y_stage, T * H * es},
    };
    size_t total = 0;
    for (auto& p : parts) total += align_up(p.bytes ? p.bytes : 16, 256);
    char* base = nullptr;
    CUDA_TRY(cudaMalloc(&base, total));
    CUDA_TRY(cudaMemset(base, 0, total));
    size_t off = 0;
    for (auto& p : parts) {
        *p.ptr = base + off;
        off += align_up(p.bytes ? p.bytes : 16, 256);
    }
    if (!h->rms_w) h->x_norm = nullptr;
    h->ws = base;
    h->max_T = max_tokens;
    h->max_units = max_units;
    if (h->tc_ok) {
        moe_status st = make_map(&h->routed_maps.b_x, h->xp, S, H, 16);
        if (st == MOE_OK) st = make_map(&h->routed_maps.b_h, h->hbuf, S, I, 16);
        if (st == MOE_OK && Is) st = make_map(&h->shared_maps.b_h, h->hs, T, Is, 16);
        if (st != MOE_OK) { free_workspace(h); return st; }
    }
    return MOE_OK;
}

}  // extern "C"

namespace {

int choose_width(const moe_layer* h, int T) {
    return (int64_t)T * h->d.k > (int64_t)16 * h->d.E ? kWide : kNarrow;
}

// Tensor-core router logits for large T: W_r (packed) x tokens, fp32 into rb.logits.
bool use_tc_router(const moe_layer* h, int T) {
    return h->w_router_packed && !h->force_simt && T >= 256;
}

moe_status run_tc_router(moe_layer* h, const void* x, int T, const RouteBufs& rb,
                         cudaStream_t s, int pdl = 0) {
    const Dims& d = h->d;
    TcMaps maps{};
    moe_status st = make_map(&maps.b_x, x, (uint64_t)T, d.H, 16);
    if (st != MOE_OK) return st;
    maps.b_h = maps.b_x;
    TcArgs a{};
    a.w_gu = h->w_router_packed; a.w_down = nullptr;
    a.H = d.H; a.I = d.E; a.phases = 4; a.logits = rb.logits;
    a.dense_T = T; a.unit_width = kNarrow;
    a.sync = h->sync_router;
    a.st = h->status(); a.wait_limit_ns = h->wait_limit_ns; a.inject_stuck = 0;
    const int tiles = (T + kNarrow - 1) / kNarrow * ((d.E / 128 + 1) / 2);
    CUDA_TRY(launch_tc_experts(maps, a, kNarrow, std::min(tiles, h->num_sms), s, pdl));
    return MOE_OK;
}

// CUDA-core shared expert (fp32 layers and forced CUDA-core runs); the tensor-core
// paths run the shared expert's tiles inside their expert kernel.
moe_status run_shared(moe_layer* h, const void* x_in, int T, cudaStream_t s) {
    const Dims& d = h->d;
    if (!d.Is) return MOE_OK;
    {
        KernelScope ks(h, MOE_KERNEL_SHARED, s);
        CUDA_TRY(launch_simt_gate_up(h->dtype, x_in, h->ws_gate, h->ws_up, h->tc_ok, nullptr,
                                     nullptr, T, d.H, d.Is, h->hs, s));
    }
    KernelScope ks(h, MOE_KERNEL_SHARED, s);
    CUDA_TRY(launch_simt_down(h->dtype, h->hs, h->ws_down, h->tc_ok, nullptr, nullptr, T, d.H,
                              d.Is, h->sbuf, s));
    return MOE_OK;
}

// Few-token path: route only, then one persistent kernel over the feature
// blocks of the shared expert and of the selected experts (gate/up, SiLU*up and
// the down partial on chip), then the partial combine.  The expert kernel and
// the combine are programmatic dependents: each starts while its predecessor
// finishes and waits on the device for the predecessor's results.
moe_status run_layer_fused(moe_layer* h, const void* x, const void* residual, void* y, int T,
                           int32_t* idx_out, float* w_out, cudaStream_t s) {
    const Dims& d = h->d;
    RouteBufs rb = h->rb;
    const void* x_in = h->rms_w ? h->x_norm : x;
    // with per-kernel timing on, events separate the kernels and the overlap is off
    const int pdl = h->timing ? 0 : 1;
    {
        KernelScope ks(h, MOE_KERNEL_ROUTER, s);
        if (h->w_router_kp && router_tc_supported(d.E, d.H, d.k, T)) {
            // a handful of tokens: one CTA forms the logits on the tensor cores
            CUtensorMap xmap;
            moe_status st = make_map(&xmap, x, (uint64_t)T, d.H, (T + 15) / 16 * 16);
            if (st != MOE_OK) return st;
            RouterTcArgs ra{};
            ra.w_router_kp = h->w_router_kp; ra.topk_idx = rb.topk_idx; ra.topk_w = rb.topk_w;
            ra.H = d.H; ra.k = d.k; ra.T = T;
            ra.st = h->status(); ra.wait_limit_ns = h->wait_limit_ns;
            CUDA_TRY(launch_router_tc(xmap, ra, pdl, s));
        } else {
            CUDA_TRY(launch_router(h->dtype, x, h->w_router, h->rms_w, h->cfg.rms_eps, h->x_norm,
                                   0, nullptr, d, T, kRouteBlock, rb, 0, kNarrow, h->max_units,
                                   0, h->status(), s, pdl));
        }
    }
    const int S = T * d.k;
    {
        FusedArgs a{};
        a.w_gu = h->w_gate; a.w_down = h->w_down;
        a.ws_gu = d.Is ? h->ws_gate : nullptr; a.ws_down = d.Is ? h->ws_down : nullptr;
        // x_early = 0: every CTA waits for the router before reading x.  The router
        // lets this kernel launch before its own wait on the previous kernel, and the
        // previous call's combine lets the router launch before it writes y, so when a
        // call's x is the previous call's y (a residual stream, in place or not) only
        // the dependency wait orders the read of x after that write.
        a.x_rows = x_in; a.x_early = 0;
        a.topk_idx = rb.topk_idx; a.o_part = h->o_part;
        a.H = d.H; a.I = d.I; a.Is = d.Is; a.E = d.E; a.k = d.k; a.T = T;
        a.zero_word = h->sync_fused + 2;
        a.st = h->status(); a.wait_limit_ns = h->wait_limit_ns;
        a.inject_stuck = h->inject_stuck;
        const int unit_rows = fused_unit_rows();
        const int max_units = std::min(d.E, S) + (S + unit_rows - 1) / unit_rows;
        const int tiles = max_units * (d.I / 128) + (T + unit_rows - 1) / unit_rows * (d.Is / 128);
        const int grid = std::min(tiles, h->num_sms);
        KernelScope ks(h, MOE_KERNEL_EXPERTS, s);
        CUDA_TRY(launch_fused_experts(a, grid, pdl, s));
        h->inject_stuck = 0;
    }
    {
        KernelScope ks(h, MOE_KERNEL_COMBINE, s);
        CUDA_TRY(launch_combine_partials(h->o_part, d.I / 128, d.Is / 128, residual, y, rb.topk_w,
                                         d, T, pdl, s));
    }
    if (idx_out)
        CUDA_TRY(cudaMemcpyAsync(idx_out, rb.topk_idx, (size_t)S * 4, cudaMemcpyDeviceToDevice, s));
    if (w_out)
        CUDA_TRY(cudaMemcpyAsync(w_out, rb.topk_w, (size_t)S * 4, cudaMemcpyDeviceToDevice, s));
    h->last_T = T;
    h->last_fused = true;
    return MOE_OK;
}

bool use_fused(const moe_layer* h, int T) {
    return h->tc_ok && !h->force_simt && h->fuse &&
           fused_supported(h->d.H, h->d.I, h->d.Is, h->d.E, h->d.k, T * h->d.k);
}

moe_status run_layer(moe_layer* h, const void* x, const void* residual, void* y, int T,
                     int32_t* idx_out, float* w_out, cudaStream_t s) {
    if (use_fused(h, T)) return run_layer_fused(h, x, residual, y, T, idx_out, w_out, s);
    h->last_fused = false;
    const Dims& d = h->d;
    const bool tc = h->tc_ok && !h->force_simt;
    const int width = choose_width(h, T);
    RouteBufs rb = h->rb;
    if (idx_out) rb.topk_idx = idx_out;
    if (w_out) rb.topk_w = w_out;
    const void* x_in = h->rms_w ? h->x_norm : x;
    // tensor cores: the shared expert's tiles join the routed experts' launch (two
    // persistent kernels would only compete for the SMs; on a side stream it held
    // every SM while the router waited).  CUDA cores: optionally a second stream.
    const bool merged = tc && d.Is > 0;
    const bool side = !merged && h->shared_stream && d.Is > 0;
    // Programmatic dependent launch is off on this path: measured at 4096 tokens it
    // cost 7 us per layer (the persistent expert kernel's early CTAs took SMs from the
    // permutation kernel); the few-token path uses it.
    const int pdl = 0;

    if (side && !h->rms_w) {     // the shared expert needs only x: start it right away
        CUDA_TRY(cudaEventRecord(h->ev_fork, s));
        CUDA_TRY(cudaStreamWaitEvent(h->s2, h->ev_fork, 0));
        moe_status st = run_shared(h, x_in, T, h->s2);
        if (st != MOE_OK) return st;
        CUDA_TRY(cudaEventRecord(h->ev_join, h->s2));
    }
    const bool tc_route = use_tc_router(h, T);
    const int tb = tc_route ? kRouteBlockWide : kRouteBlock;
    const bool fused_permute = T <= tb;      // one routing block: the router permutes it
    // narrow tensor-core tiles read their token rows from x in place: no permuted copy
    const bool gather = tc && width == kNarrow;
    void* xp_copy = gather ? nullptr : h->xp;
    {
        KernelScope ks(h, MOE_KERNEL_ROUTER, s);
        if (tc_route) {
            moe_status st = run_tc_router(h, x, T, rb, s, pdl);
            if (st != MOE_OK) return st;
        }
        CUDA_TRY(launch_router(h->dtype, x, h->w_router, h->rms_w, h->cfg.rms_eps, h->x_norm,
                               fused_permute, xp_copy, d, T, tb, rb, 1, width, h->max_units,
                               tc_route, h->status(), s, pdl));
    }
    if (side && h->rms_w) {      // with a pre-norm it needs the router's normalised x
        CUDA_TRY(cudaEventRecord(h->ev_fork, s));
        CUDA_TRY(cudaStreamWaitEvent(h->s2, h->ev_fork, 0));
        moe_status st = run_shared(h, x_in, T, h->s2);
        if (st != MOE_OK) return st;
        CUDA_TRY(cudaEventRecord(h->ev_join, h->s2));
    }
    if (!fused_permute) {
        KernelScope ks(h, MOE_KERNEL_PERMUTE, s);
        CUDA_TRY(launch_permute(h->dtype, x_in, xp_copy, d, T, tb, rb, s, pdl));
    }
    const int S = T * d.k;
    if (tc) {
        TcArgs a{};
        a.w_gu = h->w_gate; a.w_down = h->w_down;
        a.H = d.H; a.I = d.I; a.phases = h->fuse ? 3 : 1;
        a.dense_T = 0; a.unit_width = width;
        a.units = rb.units; a.n_units = rb.n_units;
        a.x_rows = x_in; a.row_token = gather ? rb.slot_token : nullptr;
        a.sync = h->sync_routed; a.hbuf = h->hbuf; a.out = h->obuf;
        a.st = h->status(); a.wait_limit_ns = h->wait_limit_ns;
        a.inject_stuck = h->inject_stuck && h->fuse;
        const int max_units = std::min(h->max_units, (S + width - 1) / width + d.E);
        int tiles = max_units * (d.I / 128 + (d.H / 128 + 1) / 2);
        TcMaps maps = h->routed_maps;
        if (merged) {
            a.w_gu2 = h->ws_gate; a.w_down2 = h->ws_down;
            a.I2 = d.Is; a.dense2_T = T;
            a.hbuf2 = h->hs; a.out2 = h->sbuf;
            a.done2 = h->sync_shared + 2;
            maps.b_h2 = h->shared_maps.b_h;
            moe_status st = make_map(&maps.b_x2, x_in, (uint64_t)T, d.H, 16);
            if (st != MOE_OK) return st;
            tiles += (T + width - 1) / width * (d.Is / 128 + (d.H / 128 + 1) / 2);
        }
        const int grid = std::min(tiles, h->num_sms);
        {
            KernelScope ks(h, MOE_KERNEL_EXPERTS, s);
            CUDA_TRY(launch_tc_experts(maps, a, width, grid, s, pdl));
        }
        if (!h->fuse) {
            a.phases = 2;
            KernelScope ks(h, MOE_KERNEL_EXPERTS, s);
            CUDA_TRY(launch_tc_experts(maps, a, width, grid, s, pdl));
        }
        h->inject_stuck = 0;
    } else {
        const int32_t* n_rows = rb.offsets + d.E;
        {
            KernelScope ks(h, MOE_KERNEL_EXPERTS, s);
            CUDA_TRY(launch_simt_gate_up(h->dtype, h->xp, h->w_gate, h->w_up, h->tc_ok,
                                         rb.slot_expert, n_rows, S, d.H, d.I, h->hbuf, s));
        }
        KernelScope ks(h, MOE_KERNEL_EXPERTS, s);
        CUDA_TRY(launch_simt_down(h->dtype, h->hbuf, h->w_down, h->tc_ok, rb.slot_expert, n_rows,
                                  S, d.H, d.I, h->obuf, s));
    }
    if (d.Is > 0 && !merged) {
        if (side) {
            CUDA_TRY(cudaStreamWaitEvent(s, h->ev_join, 0));
        } else {
            moe_status st = run_shared(h, x_in, T, s);
            if (st != MOE_OK) return st;
        }
    }
    {
        KernelScope ks(h, MOE_KERNEL_COMBINE, s);
        CUDA_TRY(launch_combine(h->dtype, h->obuf, d.Is > 0 ? h->sbuf : nullptr, residual, y,
                                rb.topk_w, rb.token_slot, d, T, s, pdl));
    }
    h->last_T = T;
    return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_route(moe_handle h, const void* x, int T, int32_t* topk_idx, float* topk_w,
                     void* stream) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "NULL handle");
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0");
    if (T == 0) return MOE_OK;
    if (!x || !topk_idx || !topk_w) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(x)) return fail(MOE_ERR_INVALID_ARG, "x must be 16-byte aligned");
    if (T > h->max_T) return fail(MOE_ERR_INVALID_ARG, "T=%d exceeds reserved %d", T, h->max_T);
    moe_status pe = pending_device_error(h);
    if (pe != MOE_OK) return pe;
    DeviceGuard g(h->device);
    RouteBufs rb = h->rb;
    rb.topk_idx = topk_idx;
    rb.topk_w = topk_w;
    KernelScope ks(h, MOE_KERNEL_ROUTER, (cudaStream_t)stream);
    if (use_tc_router(h, T)) {
        moe_status st = run_tc_router(h, x, T, rb, (cudaStream_t)stream);
        if (st != MOE_OK) return st;
    }
    const bool tc_route = use_tc_router(h, T);
    CUDA_TRY(launch_router(h->dtype, x, h->w_router, h->rms_w, h->cfg.rms_eps, nullptr, 0,
                           nullptr, h->d, T, tc_route ? kRouteBlockWide : kRouteBlock, rb, 0,
                           kNarrow, h->max_units, tc_route, h->status(), (cudaStream_t)stream));
    return MOE_OK;
}

moe_status moe_forward(moe_handle h, const void* x, const void* residual, void* y, int T,
                       int32_t* topk_idx_out, float* topk_w_out, void* stream) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "NULL handle");
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0");
    if (T == 0) return MOE_OK;
    if (!x || !y) return fail(MOE_ERR_INVALID_ARG, "x and y must not be NULL");
    if (!aligned16(x) || !aligned16(y) || (residual && !aligned16(residual)))
        return fail(MOE_ERR_INVALID_ARG, "x, residual and y must be 16-byte aligned");
    if (T > h->max_T) return fail(MOE_ERR_INVALID_ARG, "T=%d exceeds reserved %d", T, h->max_T);
    moe_status pe = pending_device_error(h);
    if (pe != MOE_OK) return pe;
    DeviceGuard g(h->device);
    return run_layer(h, x, residual, y, T, topk_idx_out, topk_w_out, (cudaStream_t)stream);
}

moe_status moe_forward_host(moe_handle h, const void* x_host, const void* residual_host,
                            void* y_host, int T, void* stream) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "NULL handle");
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0");
    if (T == 0) return MOE_OK;
    if (!x_host || !y_host) return fail(MOE_ERR_INVALID_ARG, "x_host and y_host must not be NULL");
    if (T > h->max_T) return fail(MOE_ERR_INVALID_ARG, "T=%d exceeds reserved %d", T, h->max_T);
    moe_status pe = pending_device_error(h);
    if (pe != MOE_OK) return pe;
    DeviceGuard g(h->device);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t bytes = (size_t)T * h->d.H * h->esz;
    CUDA_TRY(cudaMemcpyAsync(h->x_stage, x_host, bytes, cudaMemcpyHostToDevice, s));
    if (residual_host)
        CUDA_TRY(cudaMemcpyAsync(h->r_stage, residual_host, bytes, cudaMemcpyHostToDevice, s));
    moe_status st = run_layer(h, h->x_stage, residual_host ? h->r_stage : nullptr, h->y_stage, T,
                              nullptr, nullptr, s);
    if (st != MOE_OK) return st;
    CUDA_TRY(cudaMemcpyAsync(y_host, h->y_stage, bytes, cudaMemcpyDeviceToHost, s));
    CUDA_TRY(cudaStreamSynchronize(s));
    return MOE_OK;
}

moe_status moe_last_routing(moe_handle h, int32_t* counts, int32_t* offsets, int32_t* token_slot,
                            void* stream) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "NULL handle");
    if (!h->ws) return fail(MOE_ERR_INVALID_ARG, "no workspace reserved");
    DeviceGuard g(h->device);
    cudaStream_t s = (cudaStream_t)stream;
    CUDA_TRY(cudaStreamSynchronize(s));
    if (h->last_fused) {
        // the few-token path builds its expert lists inside the kernel; derive the
        // same expert-major, token-ordered bookkeeping from the recorded Top-k
        const int E = h->d.E, k = h->d.k, S = h->last_T * k;
        std::vector<int32_t> idx(S), cnt(E, 0), off(E + 1, 0);
        if (S) CUDA_TRY(cudaMemcpy(idx.data(), h->rb.topk_idx, (size_t)S * 4, cudaMemcpyDeviceToHost));
        for (int i = 0; i < S; ++i) {
            if (idx[i] < 0 || idx[i] >= E)     // only after a failed call: never index with it
                return fail(MOE_ERR_DEVICE_CHECK, "recorded expert index %d out of range", idx[i]);
            cnt[idx[i]]++;
        }
        for (int e = 0; e < E; ++e) off[e + 1] = off[e] + cnt[e];
        if (counts) memcpy(counts, cnt.data(), (size_t)E * 4);
        if (offsets) memcpy(offsets, off.data(), (size_t)(E + 1) * 4);
        if (token_slot) {
            std::vector<int32_t> next(off.begin(), off.end() - 1);
            for (int i = 0; i < S; ++i) token_slot[i] = next[idx[i]]++;
        }
        return MOE_OK;
    }
    if (counts)
        CUDA_TRY(cudaMemcpy(counts, h->rb.counts, h->d.E * 4, cudaMemcpyDeviceToHost));
    if (offsets)
        CUDA_TRY(cudaMemcpy(offsets, h->rb.offsets, (h->d.E + 1) * 4, cudaMemcpyDeviceToHost));
    if (token_slot && h->last_T)
        CUDA_TRY(cudaMemcpy(token_slot, h->rb.token_slot, (size_t)h->last_T * h->d.k * 4,
                            cudaMemcpyDeviceToHost));
    return MOE_OK;
}

moe_status moe_check(moe_handle h, void* stream) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "NULL handle");
    DeviceGuard g(h->device);
    CUDA_TRY(cudaStreamSynchronize((cudaStream_t)stream));
    CUDA_TRY(cudaStreamSynchronize(h->s2));
    int code = 0;
    CUDA_TRY(cudaMemcpy(&code, h->err_dev, sizeof(int), cudaMemcpyDeviceToHost));
    if (!code) code = *(volatile int*)h->err_host;
    CUDA_TRY(cudaMemset(h->err_dev, 0, sizeof(int)));
    *(volatile int*)h->err_host = 0;
    if (code == MOE_ERR_TIMEOUT) return fail(MOE_ERR_TIMEOUT, "a bounded device-side wait ran out");
    if (code) return fail(MOE_ERR_DEVICE_CHECK, "device-side check failed (%d)", code);
    return MOE_OK;
}

moe_status moe_set_option(moe_handle h, moe_option opt, int64_t value) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "NULL handle");
    switch (opt) {
        case MOE_OPT_WAIT_LIMIT_NS:
            if (value < 0) return fail(MOE_ERR_INVALID_ARG, "wait limit < 0");
            h->wait_limit_ns = (uint64_t)value;
            return MOE_OK;
        case MOE_OPT_INJECT_STUCK_WAIT: h->inject_stuck = value != 0; return MOE_OK;
        case MOE_OPT_SHARED_STREAM: h->shared_stream = value != 0; return MOE_OK;
        case MOE_OPT_FUSE_PHASES: h->fuse = value != 0; return MOE_OK;
        case MOE_OPT_FORCE_SIMT: h->force_simt = value != 0; return MOE_OK;
        case MOE_OPT_KERNEL_TIMING: h->timing = value != 0; return MOE_OK;
    }
    return fail(MOE_ERR_INVALID_ARG, "unknown option %d", (int)opt);
}

moe_status moe_kernel_stats(moe_handle h, double* total_ms, int64_t* launches, int reset) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "NULL handle");
    DeviceGuard g(h->device);
    CUDA_TRY(cudaDeviceSynchronize());
    for (auto& p : h->pending) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) h->k_ms[p.cls] += ms;
        h->ev_pool.push_back(p.a);
        h->ev_pool.push_back(p.b);
    }
    h->pending.clear();
    for (int c = 0; c < MOE_KERNEL_CLASSES; ++c) {
        if (total_ms) total_ms[c] = h->k_ms[c];
        if (launches) launches[c] = h->k_launches[c];
        if (reset) { h->k_ms[c] = 0.0; h->k_launches[c] = 0; }
    }
    return MOE_OK;
}

moe_status moe_destroy(moe_handle h) {
    if (!h) return MOE_OK;
    DeviceGuard g(h->device);
    if (h->s2) cudaStreamSynchronize(h->s2);
    cudaDeviceSynchronize();
    for (auto& p : h->pending) { cudaEventDestroy(p.a); cudaEventDestroy(p.b); }
    for (cudaEvent_t e : h->ev_pool) cudaEventDestroy(e);
    free_workspace(h);
    void* bufs[] = {h->w_router, h->w_gate, h->w_up,  h->w_down,  h->ws_gate,
                    h->ws_up,    h->ws_down, h->rms_w, h->err_dev, h->w_router_packed,
                    h->w_router_kp};
    for (void* p : bufs)
        if (p) cudaFree(p);
    if (h->err_host) cudaFreeHost(h->err_host);
    if (h->ev_fork) cudaEventDestroy(h->ev_fork);
    if (h->ev_join) cudaEventDestroy(h->ev_join);
    if (h->s2) cudaStreamDestroy(h->s2);
    delete h;
    return MOE_OK;
}

}  // extern "C"
