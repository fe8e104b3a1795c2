/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse MoE feed-forward layer.
 *
 * The operation (page "3C . Talker MoE (20 lop, 128 Experts Top-6) & Dau ra ma
 * ngu nghia c_0", section 3 "Giai phap", the routing / combine equation):
 *
 *   p   = softmax(W_r x)                       router over E experts
 *   S   = Top-k(p)                             ties -> lower expert index
 *   w_i = p_i / sum_{j in S} p_j               norm_topk_prob = True
 *   y   = Shared(x) + sum_{i in S} w_i Expert_i(x)   [+ residual]
 *
 * Expert_i and Shared are SwiGLU MLPs without bias, down(SiLU(gate x) * up x)
 * (page "print(model) Qwen3-TTS", SwiGLU feed-forward section).  Optionally the
 * layer input is first RMS-normalised, x / sqrt(mean(x^2) + eps) * g (the
 * "rmsnorm" helper of the lab page "Bai Lab tong hop -- Qwen3-Omni &
 * Qwen3-TTS-12Hz Architecture", section [3C]).  Sizes on the Talker page,
 * section 1: hidden 1024, 128 experts, Top-6, expert 384, shared expert 768.
 *
 * Conventions for every entry point:
 *  - Matrices are row-major in the nn.Linear [out, in] convention.
 *  - "device" pointers are CUDA global memory of the handle's device; "host"
 *    pointers are ordinary (preferably pinned) host memory.
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy default
 *    stream.  Every call is asynchronous on that stream unless stated.
 *  - Errors are returned, never raised: no call aborts the process.  After an
 *    error, moe_last_error() gives a thread-local description.  A device-side
 *    failure (a bounded wait that ran out, a failed device check) is recorded
 *    by the kernels in host-visible memory; moe_check() reports and clears it,
 *    and until then every call that starts after the faulty work has finished
 *    returns it without launching anything.
 *  - The library never takes ownership of caller memory.
 *  - A handle is not thread-safe: calls on one handle share its workspace and
 *    must be serialised by the caller (and, across streams, ordered on the GPU).
 *    Different handles are independent; moe_route_noalloc has its own rule.
 */
#ifndef SPARSE_MOE_B200_MOE_H
#define SPARSE_MOE_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or option      */
    MOE_ERR_CUDA = 2,          /* a CUDA runtime/driver call failed           */
    MOE_ERR_OOM = 3,           /* device or pinned-host allocation failed      */
    MOE_ERR_UNSUPPORTED = 4,   /* shape/dtype the library has no kernel for   */
    MOE_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out           */
    MOE_ERR_DEVICE_CHECK = 6   /* a device-side consistency check failed       */
} moe_status;

typedef enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 } moe_dtype;

typedef struct {
    int hidden;          /* H                                                 */
    int n_experts;       /* E, 1..1024                                        */
    int top_k;           /* k, 1..min(E, 16)                                  */
    int expert_inter;    /* I, routed expert intermediate size                */
    int shared_inter;    /* I_s, shared expert intermediate size (0 = none)   */
    moe_dtype dtype;     /* storage type of x, residual, y and every weight   */
    int norm_topk_prob;  /* must be 1: the selected weights are renormalised  */
    float rms_eps;       /* epsilon of the optional pre-RMSNorm               */
} moe_config;

typedef struct moe_layer* moe_handle;

/*
 * Create a layer on `device` from DEVICE weight pointers (the caller keeps
 * ownership; the library copies them into its own packed buffers, so they may
 * be freed when this returns).  Shapes:
 *   w_router [E][H], w_gate [E][I][H], w_up [E][I][H], w_down [E][H][I],
 *   ws_gate [I_s][H], ws_up [I_s][H], ws_down [H][I_s] (NULL when I_s == 0),
 *   rms_weight [H] or NULL (NULL = no pre-RMSNorm).
 * bf16 layers run the routed and shared experts on tcgen05 tensor cores and
 * need H % 128 == 0, I % 128 == 0 and I_s % 128 == 0; other shapes, and f32
 * layers, use exact-fp32 CUDA-core kernels.  On success *out holds the handle.
 * Errors: INVALID_ARG (NULL pointer, bad config), OOM, CUDA.
 */
moe_status moe_create(const moe_config* cfg, int device,
                      const void* w_router, const void* w_gate, const void* w_up,
                      const void* w_down, const void* ws_gate, const void* ws_up,
                      const void* ws_down, const void* rms_weight, moe_handle* out);

/*
 * Reserve the device workspace for up to `max_tokens` tokens per call.  Calls
 * with T <= max_tokens then allocate nothing, which is what makes a forward
 * capturable in a CUDA graph.  Synchronous.  The kernels index rows with 32-bit
 * integers, so max_tokens * (k + 1) * max(H, I, I_s) must stay below 2^31 (at the
 * Talker sizes: up to 299,593 tokens per call); larger reservations return
 * UNSUPPORTED and the caller splits the batch.  Errors: INVALID_ARG, UNSUPPORTED,
 * OOM, CUDA.
 */
moe_status moe_reserve(moe_handle h, int max_tokens);

/*
 * Router only (Talker page, section 3: p = softmax(W_r x), Top-k, renormalise).
 * x: device [T][H] in the layer dtype (16-byte aligned).  Writes device
 * topk_idx [T][k] (int32, in selection order: descending logit, ties to the
 * lower index) and topk_w [T][k] (fp32, sums to 1 per token).  Logits are
 * accumulated in fp32.  With a pre-RMSNorm the router sees the normalised x.
 * T == 0 is a no-op.  T must not exceed the reserved token count.
 */
moe_status moe_route(moe_handle h, const void* x, int T, int32_t* topk_idx,
                     float* topk_w, void* stream);

/*
 * Full layer: y = Shared(x') + sum_{i in S} w_i Expert_i(x') [+ residual],
 * x' = x or RMSNorm(x) * g.  x, residual (nullable) and y are device [T][H] in
 * the layer dtype, 16-byte aligned.  y may alias x or residual (the inputs are
 * consumed before y is written).  topk_idx_out / topk_w_out (nullable, device
 * [T][k]) receive the routing the call used.  T == 0 is a no-op.
 * Few tokens (T * k <= 1024, bf16, H a multiple of 256 up to 1024, k <= 8) run
 * as router + one expert kernel (the shared expert's blocks among its tiles) +
 * combine, each kernel a programmatic dependent of the one before.  Up to 64
 * tokens with 128 experts and no pre-norm, the router is one CTA that forms the
 * logits on the tensor cores (fp32 accumulate), so its routing can differ from
 * moe_route's CUDA-core logits by fp32 rounding (weights) and at exact
 * near-ties.  Larger calls run router, permutation, one grouped expert GEMM
 * launch (the shared expert's tiles among the routed experts') and combine.
 */
moe_status moe_forward(moe_handle h, const void* x, const void* residual, void* y,
                       int T, int32_t* topk_idx_out, float* topk_w_out, void* stream);

/*
 * moe_forward from HOST buffers: copies x (and residual) host->device into the
 * handle's staging buffers on `stream`, runs the layer, copies y back to
 * y_host and synchronises the stream before returning.  Pinned host memory
 * gives full copy bandwidth.  Errors as moe_forward, plus CUDA on copy failure.
 */
moe_status moe_forward_host(moe_handle h, const void* x_host, const void* residual_host,
                            void* y_host, int T, void* stream);

/*
 * Routing bookkeeping of the last moe_forward, copied to HOST arrays after a
 * stream synchronise (for tests and diagnostics).  Any pointer may be NULL.
 * counts [E]: tokens per expert; offsets [E+1]: exclusive prefix sum of counts
 * (first permuted row of each expert); token_slot [T][k]: permuted row of
 * token t's j-th selected expert, rows of one expert ordered by token index.
 * Errors: INVALID_ARG (NULL handle, no workspace), CUDA, DEVICE_CHECK (the
 * recorded routing holds an invalid expert index, possible only after a failed
 * call).
 */
moe_status moe_last_routing(moe_handle h, int32_t* counts, int32_t* offsets,
                            int32_t* token_slot, void* stream);

/* Synchronise `stream`, then report (and clear) any device-side failure
 * recorded since the last check: TIMEOUT or DEVICE_CHECK, else OK. */
moe_status moe_check(moe_handle h, void* stream);

typedef enum {
    MOE_OPT_WAIT_LIMIT_NS = 0,     /* bound of every device-side wait (ns), default 1e9 */
    MOE_OPT_INJECT_STUCK_WAIT = 1, /* 1: the next forward's first cross-tile dependency
                                      wait targets a count that is never reached, so it
                                      runs out (test hook for the bounded-wait path)    */
    MOE_OPT_SHARED_STREAM = 2,     /* 1 (default): on the CUDA-core path the shared
                                      expert runs on the second stream (the tensor-core
                                      kernels run it among their own tiles)            */
    MOE_OPT_FUSE_PHASES = 3,       /* 1 (default): gate/up and down in one launch: for
                                      T*k <= 1024 a kernel whose tiles keep h on chip
                                      and emit fp32 partial sums (the shared expert's
                                      blocks among them); otherwise one
                                      persistent launch with per-tile dependency
                                      counters.  0: separate launches.                */
    MOE_OPT_FORCE_SIMT = 4,        /* 1: run bf16 experts on the CUDA-core kernels      */
    MOE_OPT_KERNEL_TIMING = 5      /* 1: bracket every kernel launch with CUDA events on
                                      its own stream (read with moe_kernel_stats); this
                                      also turns off the programmatic launch overlap of
                                      the few-token path, so each kernel is timed alone */
} moe_option;

/* Set an option; takes effect at the next call.  Errors: INVALID_ARG. */
moe_status moe_set_option(moe_handle h, moe_option opt, int64_t value);

/* Kernel classes reported by moe_kernel_stats. */
typedef enum {
    MOE_KERNEL_ROUTER = 0,     /* logits, Top-k, weights, histogram, scan            */
    MOE_KERNEL_PERMUTE = 1,    /* gather of token rows into expert-contiguous order  */
    MOE_KERNEL_EXPERTS = 2,    /* expert GEMMs (gate/up + SiLU*up, down); on tensor
                                  cores the shared expert's tiles run in them too   */
    MOE_KERNEL_SHARED = 3,     /* shared expert GEMMs on CUDA cores (fp32 layers)    */
    MOE_KERNEL_COMBINE = 4,    /* weighted combine + shared + residual               */
    MOE_KERNEL_CLASSES = 5
} moe_kernel_class;

/*
 * Per-class kernel statistics since the last reset, after synchronising the
 * handle's device: launches[c] counts every launch of class c (always on);
 * total_ms[c] sums the CUDA-event time of those launches, measured on the
 * stream each kernel runs on, while MOE_OPT_KERNEL_TIMING is 1 (else 0).
 * Both arrays hold MOE_KERNEL_CLASSES entries (HOST memory, nullable).
 * reset != 0 clears the counters after reading.
 */
moe_status moe_kernel_stats(moe_handle h, double* total_ms, int64_t* launches, int reset);

/* Free everything the handle owns (after synchronising its streams). */
moe_status moe_destroy(moe_handle h);

/*
 * Router with no memory allocation (the pages have no counterpart: this is a
 * deployment convenience of this library).  For callers that cannot call
 * cudaMalloc -- e.g. a streaming audio thread that must never block, since
 * cudaMalloc can synchronise the device and wait on driver locks, or a process
 * whose device memory is fully reserved by another allocator -- this routes T
 * tokens like moe_route without a handle: the caller passes the layer sizes
 * (cfg), x [T][H] (16-byte aligned), the router weights w_router [E][H] and
 * rms_weight [H] or NULL, all on the current device, and receives topk_idx /
 * topk_w [T][k] (device).  The router's scratch lives in one fixed 4 MiB
 * device array that every GPU loading this library holds until the process
 * exits; a call needs T * E * 4 bytes of logits plus about T / 2 + 512 bytes
 * of counters in it (T up to 8183 at E = 128); larger calls return
 * MOE_ERR_INVALID_ARG.  Nothing is allocated or freed.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress), so make
 * that first call before any stream capture on that device.  All calls share
 * the array: calls whose work overlaps on the GPU (different streams, or other
 * threads) race and must be serialised by the caller.  Logits are always
 * formed on CUDA cores (fp32), so for T >= 256 results can differ from
 * moe_route's tensor-core logits by rounding (near-tie tokens only).  The
 * router has no device-side wait; its one device check (a selected index out
 * of range, impossible for 1 <= k <= E) is not reported by this entry point,
 * which has no handle for moe_check.  Errors: INVALID_ARG (NULL cfg or
 * pointer, bad sizes or dtype, misaligned x, T too large), UNSUPPORTED
 * (norm_topk_prob != 1), CUDA (no current device, launch failure).
 */
moe_status moe_route_noalloc(const moe_config* cfg, const void* x, const void* w_router,
                             const void* rms_weight, int T, int32_t* topk_idx, float* topk_w,
                             void* stream);

/* Static text for a status code. */
const char* moe_status_string(moe_status s);

/* Thread-local description of the last error on this thread (h may be NULL). */
const char* moe_last_error(moe_handle h);

/* Library version string, e.g. "sparse_moe_b200 0.1 sm_100a". */
const char* moe_version(void);

#ifdef __cplusplus
}
#endif
#endif
