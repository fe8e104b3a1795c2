// router_tc.cu -- router for a handful of tokens in one CTA, on the tensor cores.
//
// Router equation: page "3C . Talker MoE (20 lop, 128 Experts Top-6) & Dau ra
// ma ngu nghia c_0", section 3: p = softmax(W_r x), S = Top-k, w_i = p_i /
// sum_{j in S} p_j (the selection and weights as in topk.cuh).
//
// With few tokens the router is latency, not work: 128 x 1024 x T multiply-adds.
// The multi-CTA CUDA-core router spends its time in round trips -- logits to
// global memory, an arrival counter, the last CTA reloading them.  Here one CTA
// streams W_r (packed as k-pairs: 128 experts x 128 columns, one 32 KB bulk copy)
// through a 4-stage ring, together with the matching 128 columns of the tokens
// (one TMA box, rows past T read as zeros), forms the logits
// L[e][t] = sum_j W_r[e][j] x[t][j] with tcgen05.mma (bf16 in, fp32 accumulate,
// M = 128 experts, N = the tokens rounded up to 16), moves them TMEM -> shared
// memory, and takes each token's Top-k with one warp.  W_r is a constant: its
// first stages are issued before the wait on the previous kernel (programmatic
// dependent launch), the tokens after it.
//
// Warp roles: warp 0 lane 0 issues the copies, warp 1 lane 0 the MMAs, warps 2-9
// drain TMEM and run the Top-k.  Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "device.cuh"
#include "layer.h"
#include "topk.cuh"

namespace moe {
namespace {

constexpr int kE = 128;                  // experts (one MMA M block)
constexpr int kMaxN = 64;                // tokens (MMA N, multiple of 16)
constexpr int kStages = 4;
constexpr int kWBytes = 2 * kE * 64 * 2; // a k-pair of W_r: two 128 x 64 swizzled tiles
constexpr int kXTile = kMaxN * 128;      // one 64-column box of the tokens (max rows)
constexpr int kStageBytes = kWBytes + 2 * kXTile;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kLgStride = kMaxN + 1;     // logits row stride in shared memory (floats)
constexpr int kLgBytes = kE * kLgStride * 4;
constexpr int kSmem = kStages * kStageBytes + kLgBytes + 256 + 1024;   // + barriers, alignment
constexpr uint64_t kDrainLimitNs = 200ull * 1000 * 1000;
static_assert(kStageBytes % 1024 == 0, "stage alignment");
static_assert(kSmem <= 232448, "shared memory per CTA");

__global__ void __launch_bounds__(kThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap xmap, const RouterTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float* lg = reinterpret_cast<float*>(smem + kStages * kStageBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes + kLgBytes);
    uint64_t* empty = full + kStages;
    uint64_t* accfull = empty + kStages;
    uint64_t* lgbar = accfull + 1;       // epilogue warps: every logit written
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lgbar + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = a.T, k = a.k, KP = a.H / 128;
    const int NT = (T + 15) / 16 * 16;
    const uint32_t x_bytes = 2u * NT * 128u;
    const uint64_t limit = a.wait_limit_ns;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        mbar_init(accfull, 1);
        mbar_init(lgbar, kEpiWarps);
        mbar_fence_init();
        tma_prefetch_desc(&xmap);
    }
    if (warp == 1) tmem_alloc(tmem_slot, kMaxN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    grid_dependents_launch();                // the expert kernel may start its prologue

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_x = policy_evict_last();
            const uint8_t* wr = static_cast<const uint8_t*>(a.w_router_kp);
            const int pre = min(kStages, KP);
            bool ok = true;
            // the router weights of the first stages do not depend on the previous kernel
            for (int q = 0; q < pre; ++q) {
                mbar_arrive_expect_tx(&full[q], kWBytes + x_bytes);
                bulk_load(smem + q * kStageBytes, wr + (size_t)q * kWBytes, kWBytes, &full[q], pol_w);
            }
            grid_dependency_wait();          // x is the previous kernel's output
            for (int q = 0; q < pre; ++q) {
                uint8_t* X = smem + q * kStageBytes + kWBytes;
                tma_load_2d(X, &xmap, &full[q], (2 * q) * 64, 0, pol_x);
                tma_load_2d(X + NT * 128, &xmap, &full[q], (2 * q + 1) * 64, 0, pol_x);
            }
            int issued = pre;                // stages whose copies are in flight or landed
            for (int q = pre; q < KP && ok; ++q) {
                const int s = q % kStages;
                if (!mbar_wait(&empty[s], ((q / kStages) & 1) ^ 1, a.st, limit)) { ok = false; break; }
                issued = q + 1;
                uint8_t* W = smem + s * kStageBytes;
                mbar_arrive_expect_tx(&full[s], kWBytes + x_bytes);
                bulk_load(W, wr + (size_t)q * kWBytes, kWBytes, &full[s], pol_w);
                tma_load_2d(W + kWBytes, &xmap, &full[s], (2 * q) * 64, 0, pol_x);
                tma_load_2d(W + kWBytes + NT * 128, &xmap, &full[s], (2 * q + 1) * 64, 0, pol_x);
            }
            // copies still in flight must land before the CTA exits (a stage's full
            // barrier completes once its bytes have arrived)
            for (int q = max(0, issued - kStages); q < issued; ++q)
                mbar_wait(&full[q % kStages], (q / kStages) & 1, a.st, kDrainLimitNs);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kE, NT);
            bool ok = true;
            for (int q = 0; q < KP; ++q) {
                const int s = q % kStages;
                if (!mbar_wait(&full[s], (q / kStages) & 1, a.st, limit)) { ok = false; break; }
                tc_fence_after();
                const uint32_t w0 = smem_u32(smem + s * kStageBytes);
                const uint32_t x0 = w0 + kWBytes;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_bf16(tmem_base, smem_desc_sw128(w0 + h * (kWBytes / 2) + kk * 32),
                                    smem_desc_sw128(x0 + h * NT * 128 + kk * 32), idesc,
                                    (q | h | kk) != 0);
                tc_commit(&empty[s]);
            }
            tc_commit(accfull);                // also when a wait ran out: the epilogue goes on
            (void)ok;
        }
        __syncwarp();
    } else {
        // ---- logits TMEM -> shared memory: warp (q, half) reads experts 32 q + lane,
        // columns [32 half, 32 half + 32)
        const int ew = warp - 2, q = warp & 3, half = ew >> 2;
        const bool got = mbar_wait(accfull, 0, a.st, limit);
        tc_fence_after();
        const uint32_t lanes = static_cast<uint32_t>(q * 32) << 16;
        const int e = q * 32 + lane;
        if (got) {
            for (int c = 2 * half; c < 2 * half + 2 && c * 16 < NT; ++c) {
                float v[16];
                tmem_ld16(tmem_base + lanes + c * 16, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) lg[e * kLgStride + c * 16 + j] = v[j];
            }
        }
        tc_fence_before();
        __threadfence_block();
        __syncwarp();
        if (lane == 0) mbar_arrive(lgbar);
        // a wait that runs out has recorded its error; the warps still finish together
        mbar_wait(lgbar, 0, a.st, limit);
        // ---- Top-k of token t by warp t % 8 (lower-index ties, renormalised weights)
        for (int t = ew; t < T; t += kEpiWarps) {
            float lv[kE / 32];
#pragma unroll
            for (int i = 0; i < kE / 32; ++i) lv[i] = lg[(lane + 32 * i) * kLgStride + t];
            int my_e;
            float my_w;
            warp_topk_select<kE / 32>(lv, kE, k, my_e, my_w, a.st);
            if (lane < k) {
                a.topk_idx[(size_t)t * k + lane] = my_e;
                a.topk_w[(size_t)t * k + lane] = my_w;
            }
        }
    }

    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kMaxN);
    }
}

}  // namespace

bool router_tc_supported(int E, int H, int k, int T) {
    return E == kE && H % 128 == 0 && H >= 128 && k >= 1 && k <= kE && T >= 1 && T <= kMaxN;
}

cudaError_t launch_router_tc(const CUtensorMap& xmap, const RouterTcArgs& a, int pdl,
                             cudaStream_t s) {
    if (!router_tc_supported(kE, a.H, a.k, a.T)) return cudaErrorInvalidValue;
    static std::once_flag configured[16];    // the attribute is set per device
    cudaError_t e = once_per_device(configured, [] {
        return cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kSmem);
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, router_tc_kernel, xmap, a);
}

}  // namespace moe
