// noalloc.cu -- moe_route_noalloc: the router without any memory allocation.
//
// Some callers cannot call cudaMalloc: a streaming audio thread that must never
// block (cudaMalloc can synchronise the device and wait on driver locks), a
// process whose device memory is already fully reserved by another allocator,
// or a service that must keep its device footprint fixed after start-up.  For
// them this entry point runs the same router kernel as moe_route, with every
// scratch buffer the kernel needs placed in one fixed array below instead of a
// handle's workspace.  The router weights come straight from the caller.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "layer.h"
#include "moe.h"

namespace moe {
void set_last_error(const char* msg);   // moe_api.cu: thread-local moe_last_error text
}

using namespace moe;

namespace {

// Scratch of moe_route_noalloc: 256 bytes of control words (device status
// word), then the router's arrival counters, then its fp32 logits [T][E].
// Every device that loads this library holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB
__device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

constexpr size_t kCtrlBytes = 256;
constexpr int kMaxDevices = 256;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};   // device address of g_route_scratch, per device

size_t align256(size_t v) { return (v + 255) / 256 * 256; }
size_t ticket_bytes(int T) { return align256(((size_t)T + 7) / 8 * 4 + 4); }

moe_status fail(moe_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    set_last_error(buf);
    return s;
}

// Device address of the scratch array on the current device (resolved once).
moe_status scratch_on(int dev, void** out) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess || !p)
            return fail(MOE_ERR_CUDA, "cudaGetSymbolAddress(route scratch) failed: %s",
                        cudaGetErrorString(e));
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_route_noalloc(const moe_config* cfg, const void* x,
                                        const void* w_router, const void* rms_weight, int T,
                                        int32_t* topk_idx, float* topk_w, void* stream) {
    if (!cfg) return fail(MOE_ERR_INVALID_ARG, "cfg must not be NULL");
    const moe_config& c = *cfg;
    if (c.hidden <= 0 || c.n_experts <= 0 || c.n_experts > 1024 || c.top_k <= 0 ||
        c.top_k > c.n_experts || c.top_k > 16)
        return fail(MOE_ERR_INVALID_ARG, "bad layer sizes");
    if (c.dtype != MOE_DTYPE_F32 && c.dtype != MOE_DTYPE_BF16)
        return fail(MOE_ERR_INVALID_ARG, "dtype must be MOE_DTYPE_F32 or MOE_DTYPE_BF16");
    if (c.norm_topk_prob != 1) return fail(MOE_ERR_UNSUPPORTED, "only norm_topk_prob = 1");
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0");
    if (T == 0) return MOE_OK;
    if (!x || !w_router || !topk_idx || !topk_w)
        return fail(MOE_ERR_INVALID_ARG, "x, w_router, topk_idx and topk_w must not be NULL");
    if (reinterpret_cast<uintptr_t>(x) & 15)
        return fail(MOE_ERR_INVALID_ARG, "x must be 16-byte aligned");
    const size_t need = kCtrlBytes + ticket_bytes(T) + (size_t)T * c.n_experts * 4;
    if (need > kNoAllocScratchBytes)
        return fail(MOE_ERR_INVALID_ARG,
                    "T=%d with %d experts needs %zu bytes of router scratch; "
                    "moe_route_noalloc has a fixed %zu bytes (use moe_route for larger calls)",
                    T, c.n_experts, need, kNoAllocScratchBytes);
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return fail(MOE_ERR_CUDA, "no current CUDA device: %s", cudaGetErrorString(e));
    void* base = nullptr;
    moe_status st = scratch_on(dev, &base);
    if (st != MOE_OK) return st;

    char* p = static_cast<char*>(base);
    RouteBufs rb{};
    DeviceStatus ds{reinterpret_cast<int*>(p), nullptr};
    rb.tickets = reinterpret_cast<int32_t*>(p + kCtrlBytes);
    rb.logits = reinterpret_cast<float*>(p + kCtrlBytes + ticket_bytes(T));
    rb.topk_idx = topk_idx;
    rb.topk_w = topk_w;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the status word and the arrival counters must start at zero on every call
    e = cudaMemsetAsync(p, 0, kCtrlBytes + ticket_bytes(T), s);
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    const Dims d{c.hidden, c.n_experts, c.top_k, 0, 0};
    e = launch_router(c.dtype == MOE_DTYPE_F32 ? 0 : 1, x, w_router, rms_weight, c.rms_eps,
                      nullptr, 0, nullptr, d, T, 16, rb, 0, 32, 0, 0, ds, s);
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "router launch: %s", cudaGetErrorString(e));
    return MOE_OK;
}
