// routing.cu -- router (logits, Top-k, renormalised weights, histogram, scan)
// and token permutation into expert-contiguous rows.
//
// Router equation: page "3C . Talker MoE (20 lop, 128 Experts Top-6) & Dau ra
// ma ngu nghia c_0", section 3: p = softmax(W_r x), S = Top-k, w_i = p_i /
// sum_{j in S} p_j.  Because softmax is strictly increasing, S is taken on the
// fp32 logits, and w_i = exp(l_i - l_max) / sum_{j in S} exp(l_j - l_max) needs
// only the k selected logits.  Optional pre-RMSNorm: "rmsnorm" helper of the lab
// page, section [3C], x / sqrt(mean(x^2) + eps) * g, applied in fp32 before the
// logits (the router never sees a rounded normalised input).
#include <cuda_bf16.h>
#include <stdint.h>

#include "device.cuh"
#include "layer.h"

namespace moe {
namespace {

constexpr int kRouterThreads = 256;
constexpr int kEG = 16;        // experts per router CTA
constexpr int kMaxTB = 16;     // tokens per router CTA (= routing block)
constexpr int kKC = 128;       // K chunk staged in shared memory
constexpr int kMaxE = 1024;
constexpr int kMaxK = 16;

// "a before b" in the Top-k order: larger logit first, ties to the lower index.
__device__ __forceinline__ bool before(float va, int ia, float vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

template <typename Tin>
__global__ void __launch_bounds__(kRouterThreads)
router_kernel(const Tin* __restrict__ x, const Tin* __restrict__ w_router,
              const Tin* __restrict__ rms_w, float rms_eps, Tin* __restrict__ x_norm, Dims d,
              int T, int tb, RouteBufs rb, int do_scan, int unit_width, int max_units,
              DeviceStatus st) {
    __shared__ float xs[kMaxTB][kKC + 1];
    __shared__ float ws[kEG][kKC + 1];
    __shared__ float inv_rms[kMaxTB];
    __shared__ int hist[kMaxE];
    __shared__ int unit_base[kMaxE + 1];
    __shared__ int s_flag;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = d.H, E = d.E, k = d.k;
    const int n_groups = gridDim.x, nblocks = gridDim.y;
    const int g = blockIdx.x, b = blockIdx.y;
    const int t0 = b * tb, nt = min(tb, T - t0);
    const int e0 = g * kEG;

    // ---- pre-RMSNorm scale per token (fp32), one warp per token
    if (rms_w) {
        for (int tl = warp; tl < nt; tl += kRouterThreads / 32) {
            const Tin* row = x + (size_t)(t0 + tl) * H;
            float ss = 0.f;
            for (int j = lane; j < H; j += 32) {
                float v = to_f32(row[j]);
                ss += v * v;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if (lane == 0) inv_rms[tl] = 1.0f / sqrtf(ss / (float)H + rms_eps);
        }
        __syncthreads();
        if (g == 0 && x_norm) {   // materialise the normalised input for the experts
            for (int i = tid; i < nt * H; i += kRouterThreads) {
                int tl = i / H, j = i - tl * H;
                float v = to_f32(x[(size_t)(t0 + tl) * H + j]) * inv_rms[tl] * to_f32(rms_w[j]);
                x_norm[(size_t)(t0 + tl) * H + j] = from_f32<Tin>(v);
            }
        }
    }

    // ---- logits for nt tokens x kEG experts; thread = (token, expert)
    const int tl_me = tid / kEG, el_me = tid % kEG;
    float acc = 0.f;
    for (int kc = 0; kc < H; kc += kKC) {
        const int kn = min(kKC, H - kc);
        for (int i = tid; i < kMaxTB * kKC; i += kRouterThreads) {
            int tl = i / kKC, j = i - tl * kKC;
            float v = 0.f;
            if (tl < nt && j < kn) {
                v = to_f32(x[(size_t)(t0 + tl) * H + kc + j]);
                if (rms_w) v = v * inv_rms[tl] * to_f32(rms_w[kc + j]);
            }
            xs[tl][j] = v;
        }
        for (int i = tid; i < kEG * kKC; i += kRouterThreads) {
            int el = i / kKC, j = i - el * kKC;
            ws[el][j] = (e0 + el < E && j < kn) ? to_f32(w_router[(size_t)(e0 + el) * H + kc + j])
                                                : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int j = 0; j < kKC; ++j) acc = fmaf(xs[tl_me][j], ws[el_me][j], acc);
        __syncthreads();
    }
    if (tl_me < nt && e0 + el_me < E) rb.logits[(size_t)(t0 + tl_me) * E + e0 + el_me] = acc;

    // ---- the last CTA of this token block selects the Top-k
    __threadfence();
    __syncthreads();
    if (tid == 0) s_flag = (atomicAdd(&rb.tickets[b], 1) == n_groups - 1);
    __syncthreads();
    if (!s_flag) return;
    __threadfence();
    for (int e = tid; e < E; e += kRouterThreads) hist[e] = 0;
    __syncthreads();

    for (int tl = warp; tl < nt; tl += kRouterThreads / 32) {
        const int t = t0 + tl;
        const float* lrow = rb.logits + (size_t)t * E;
        uint32_t taken = 0;     // bit i: element lane + 32 i already selected
        float sel_v[kMaxK];
        int sel_i[kMaxK];
        for (int r = 0; r < k; ++r) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
            for (int i = 0; lane + 32 * i < E; ++i) {
                if (taken & (1u << i)) continue;
                int e = lane + 32 * i;
                float v = __ldcg(lrow + e);
                if (bi == 0x7fffffff || before(v, e, bv, bi)) { bv = v; bi = e; }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (oi != 0x7fffffff && (bi == 0x7fffffff || before(ov, oi, bv, bi))) {
                    bv = ov; bi = oi;
                }
            }
            if (bi != 0x7fffffff && (bi & 31) == lane) taken |= 1u << (bi >> 5);
            sel_v[r] = bv;
            sel_i[r] = bi;
        }
        if (lane == 0) {
            float z = 0.f, ex[kMaxK];
            for (int r = 0; r < k; ++r) { ex[r] = expf(sel_v[r] - sel_v[0]); z += ex[r]; }
            for (int r = 0; r < k; ++r) {
                int e = sel_i[r];
                if (e < 0 || e >= E) { report_error(st, kErrDeviceCheck); e = 0; }
                rb.topk_idx[(size_t)t * k + r] = e;
                rb.topk_w[(size_t)t * k + r] = ex[r] / z;
                atomicAdd(&hist[e], 1);
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += kRouterThreads) rb.block_hist[(size_t)b * E + e] = hist[e];
    if (tid == 0) rb.tickets[b] = 0;   // every CTA of this block has arrived
    if (!do_scan) return;

    // ---- the last token block computes the global scan and the unit list
    __threadfence();
    __syncthreads();
    if (tid == 0) s_flag = (atomicAdd(&rb.tickets[nblocks], 1) == nblocks - 1);
    __syncthreads();
    if (!s_flag) return;
    __threadfence();
    for (int e = tid; e < E; e += kRouterThreads) {
        int run = 0;
        for (int bb = 0; bb < nblocks; ++bb) {
            rb.block_off[(size_t)bb * E + e] = run;
            run += __ldcg(rb.block_hist + (size_t)bb * E + e);
        }
        hist[e] = run;
        rb.counts[e] = run;
    }
    __syncthreads();
    if (tid == 0) {
        int off = 0, nu = 0;
        for (int e = 0; e < E; ++e) {
            rb.offsets[e] = off;
            unit_base[e] = nu;
            off += hist[e];
            nu += (hist[e] + unit_width - 1) / unit_width;
        }
        rb.offsets[E] = off;
        unit_base[E] = nu;
        if (nu > max_units) { report_error(st, kErrDeviceCheck); nu = max_units; }
        *rb.n_units = nu;
        rb.tickets[nblocks] = 0;
    }
    __syncthreads();
    for (int e = tid; e < E; e += kRouterThreads) {
        int c = hist[e], base = rb.offsets[e];
        for (int u = 0; u * unit_width < c; ++u) {
            int idx = unit_base[e] + u;
            if (idx >= max_units) break;
            Unit un;
            un.expert = e;
            un.row_start = base + u * unit_width;
            un.n_len = min(unit_width, c - u * unit_width);
            un.pad = 0;
            rb.units[idx] = un;
        }
    }
}

// ---------------------------------------------------------------- permute
// One CTA per routing block of tb <= 128 tokens.  Rows of one expert are placed
// in token order: rank = number of earlier tokens of the block that picked the
// same expert (from a 128-bit token mask per expert) + earlier blocks' counts.
template <typename Tin>
__global__ void __launch_bounds__(256)
permute_kernel(const Tin* __restrict__ x_in, Tin* __restrict__ xp, Dims d, int T, int tb,
               RouteBufs rb) {
    extern __shared__ uint32_t bits[];   // [E][4]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = d.E, k = d.k, H = d.H;
    const int b = blockIdx.x, t0 = b * tb, nt = min(tb, T - t0);
    for (int i = tid; i < E * 4; i += blockDim.x) bits[i] = 0;
    __syncthreads();
    for (int i = tid; i < nt * k; i += blockDim.x) {
        int tl = i / k;
        int e = rb.topk_idx[(size_t)t0 * k + i];
        atomicOr(&bits[e * 4 + (tl >> 5)], 1u << (tl & 31));
    }
    __syncthreads();
    for (int i = tid; i < nt * k; i += blockDim.x) {
        int tl = i / k, t = t0 + tl;
        int e = rb.topk_idx[(size_t)t0 * k + i];
        int rank = 0;
        for (int w = 0; w < (tl >> 5); ++w) rank += __popc(bits[e * 4 + w]);
        rank += __popc(bits[e * 4 + (tl >> 5)] & ((1u << (tl & 31)) - 1u));
        int pos = rb.offsets[e] + rb.block_off[(size_t)b * E + e] + rank;
        rb.token_slot[(size_t)t0 * k + i] = pos;
        rb.slot_token[pos] = t;
        rb.slot_expert[pos] = e;
    }
    __syncthreads();
    // copy rows: one warp per (token, slot) pair, 16-byte vectors when possible
    const bool vec = ((H * (int)sizeof(Tin)) % 16) == 0;
    for (int i = warp; i < nt * k; i += blockDim.x / 32) {
        int tl = i / k;
        int pos = rb.token_slot[(size_t)t0 * k + i];
        const Tin* src = x_in + (size_t)(t0 + tl) * H;
        Tin* dst = xp + (size_t)pos * H;
        if (vec) {
            const int nv = H * (int)sizeof(Tin) / 16;
            const uint4* s4 = reinterpret_cast<const uint4*>(src);
            uint4* d4 = reinterpret_cast<uint4*>(dst);
            for (int v = lane; v < nv; v += 32) d4[v] = s4[v];
        } else {
            for (int j = lane; j < H; j += 32) dst[j] = src[j];
        }
    }
}

}  // namespace

cudaError_t launch_router(int dtype, const void* x, const void* w_router, const void* rms_w,
                          float rms_eps, void* x_norm, const Dims& d, int T, int tb,
                          const RouteBufs& rb, int do_scan, int unit_width, int max_units,
                          const DeviceStatus& ds, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    if (tb > kMaxTB || d.E > kMaxE || d.k > kMaxK) return cudaErrorInvalidValue;
    dim3 grid((d.E + kEG - 1) / kEG, (T + tb - 1) / tb);
    if (dtype == 0)
        router_kernel<float><<<grid, kRouterThreads, 0, s>>>(
            (const float*)x, (const float*)w_router, (const float*)rms_w, rms_eps,
            (float*)x_norm, d, T, tb, rb, do_scan, unit_width, max_units, ds);
    else
        router_kernel<__nv_bfloat16><<<grid, kRouterThreads, 0, s>>>(
            (const __nv_bfloat16*)x, (const __nv_bfloat16*)w_router,
            (const __nv_bfloat16*)rms_w, rms_eps, (__nv_bfloat16*)x_norm, d, T, tb, rb, do_scan,
            unit_width, max_units, ds);
    return cudaGetLastError();
}

cudaError_t launch_permute(int dtype, const void* x_in, void* xp, const Dims& d, int T, int tb,
                           const RouteBufs& rb, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    if (tb > 128) return cudaErrorInvalidValue;
    int nblocks = (T + tb - 1) / tb;
    size_t smem = (size_t)d.E * 4 * sizeof(uint32_t);
    if (dtype == 0)
        permute_kernel<float><<<nblocks, 256, smem, s>>>((const float*)x_in, (float*)xp, d, T, tb,
                                                        rb);
    else
        permute_kernel<__nv_bfloat16><<<nblocks, 256, smem, s>>>(
            (const __nv_bfloat16*)x_in, (__nv_bfloat16*)xp, d, T, tb, rb);
    return cudaGetLastError();
}

}  // namespace moe
