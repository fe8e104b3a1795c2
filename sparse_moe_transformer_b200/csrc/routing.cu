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
//
// These kernels run once per layer call on little data, so they are written to
// be latency-lean: short rolled loops (the code is fetched cold on every
// launch), loads issued together, and block-wide parallel scans instead of
// single-thread loops.
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

#include "device.cuh"
#include "layer.h"
#include "topk.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kEG = 2;              // experts per logits CTA: 4 warps per expert
constexpr int kMaxTB = 16;          // tokens per logits CTA
constexpr int kMaxE = 1024;
constexpr int kMaxK = 16;
constexpr int kMaxRouterSmem = 200 * 1024;   // dynamic shared memory of a router launch

// VEC consecutive elements as fp32 (VEC * sizeof(T) == 16: one vector load).
template <typename T, int VEC>
__device__ __forceinline__ void load_vec(const T* p, float (&v)[VEC]) {
    if constexpr (VEC * sizeof(T) == 16) {
        uint4 raw = *reinterpret_cast<const uint4*>(p);
        const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
        for (int i = 0; i < VEC; ++i) v[i] = to_f32(e[i]);
    } else {
#pragma unroll
        for (int i = 0; i < VEC; ++i) v[i] = to_f32(p[i]);
    }
}

// In-place exclusive scan of v[0..n) (n <= 1024) by all kThreads threads;
// returns the total.  `tmp` holds kWarps + 1 ints of shared memory.
__device__ int block_exclusive_scan(int* v, int n, int* tmp) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + kThreads - 1) / kThreads;
    const int b0 = min(n, tid * per), b1 = min(n, b0 + per);
    int s = 0;
    for (int i = b0; i < b1; ++i) s += v[i];
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int w = 0; w < kWarps; ++w) { const int t = tmp[w]; tmp[w] = run; run += t; }
        tmp[kWarps] = run;
    }
    __syncthreads();
    int run = tmp[warp] + incl - s;
    for (int i = b0; i < b1; ++i) { const int t = v[i]; v[i] = run; run += t; }
    const int total = tmp[kWarps];
    __syncthreads();
    return total;
}

// Top-k of one token (one warp), written to the routing buffers; the
// selections are counted into the token's routing block (hist = its row, nullable).
template <int EPL>
__device__ void warp_topk_vals(const float (&lv)[EPL], int E, int k, int t, RouteBufs& rb,
                               int* hist, const DeviceStatus& st) {
    const int lane = threadIdx.x & 31;
    int my_e;
    float my_w;
    warp_topk_select<EPL>(lv, E, k, my_e, my_w, st);
    if (lane < k) {
        rb.topk_idx[(size_t)t * k + lane] = my_e;
        rb.topk_w[(size_t)t * k + lane] = my_w;
        if (hist) atomicAdd(hist + my_e, 1);
    }
}

template <int EPL>
__device__ void warp_topk(const float* lrow, int E, int k, int t, RouteBufs& rb, int* hist,
                          const DeviceStatus& st) {
    const int lane = threadIdx.x & 31;
    float lv[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i)
        lv[i] = (lane + 32 * i < E) ? __ldcg(lrow + lane + 32 * i) : -INFINITY;
    warp_topk_vals<EPL>(lv, E, k, t, rb, hist, st);
}

// Permutation of routing block b (tb <= 128 tokens): rows of one expert in token
// order.  rank = earlier tokens of the block that chose the same expert (from a
// 128-bit token mask per expert) + earlier blocks' counts.  part / split: this
// CTA copies every split-th 16-byte vector of the block's rows (no copy when xp is
// null: bookkeeping only).  `sm` holds E * 4 + tb * k ints of shared memory.
template <typename Tin>
__device__ void permute_block(const Tin* __restrict__ x_in, Tin* __restrict__ xp, const Dims& d,
                              int T, int tb, int b, int part, int split, const RouteBufs& rb,
                              uint32_t* sm) {
    const int tid = threadIdx.x;
    const int E = d.E, k = d.k, H = d.H;
    const int t0 = b * tb, nt = min(tb, T - t0), pairs = nt * k;
    uint32_t* bits = sm;
    int* pos_s = reinterpret_cast<int*>(sm + E * 4);
    for (int i = tid; i < E * 4; i += blockDim.x) bits[i] = 0;
    __syncthreads();
    for (int i = tid; i < pairs; i += blockDim.x) {
        const int tl = i / k;
        const int e = __ldcg(rb.topk_idx + (size_t)t0 * k + i);
        atomicOr(&bits[e * 4 + (tl >> 5)], 1u << (tl & 31));
    }
    __syncthreads();
    for (int i = tid; i < pairs; i += blockDim.x) {
        const int tl = i / k;
        const int e = __ldcg(rb.topk_idx + (size_t)t0 * k + i);
        int rank = __popc(bits[e * 4 + (tl >> 5)] & ((1u << (tl & 31)) - 1u));
        for (int w = 0; w < (tl >> 5); ++w) rank += __popc(bits[e * 4 + w]);
        const int pos = __ldcg(rb.offsets + e) + __ldcg(rb.block_off + (size_t)b * E + e) + rank;
        pos_s[i] = pos;
        if (part == 0) {
            rb.token_slot[(size_t)t0 * k + i] = pos;
            rb.slot_token[pos] = t0 + tl;
            rb.slot_expert[pos] = e;
        }
    }
    __syncthreads();
    if (!xp) return;                                       // bookkeeping only
    if ((H * (int)sizeof(Tin)) % 16 == 0) {
        const int nv = H * (int)sizeof(Tin) / 16;            // vectors per row
        const int total = pairs * nv;
        const int stride = blockDim.x * split;
#pragma unroll 1
        for (int q0 = part * blockDim.x + tid; q0 < total; q0 += 8 * stride) {
            uint4 v[8];
            int dst[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {                    // eight loads in flight
                const int q = q0 + u * stride;
                dst[u] = -1;
                if (q < total) {
                    const int i = q / nv, c = q - i * nv;
                    v[u] = *(reinterpret_cast<const uint4*>(x_in + (size_t)(t0 + i / k) * H) + c);
                    dst[u] = pos_s[i] * nv + c;
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (dst[u] >= 0) reinterpret_cast<uint4*>(xp)[dst[u]] = v[u];
        }
    } else {
        for (int q = part * blockDim.x + tid; q < pairs * H; q += blockDim.x * split) {
            const int i = q / H, j = q - i * H;
            xp[(size_t)pos_s[i] * H + j] = x_in[(size_t)(t0 + i / k) * H + j];
        }
    }
}

// Part sums of the column scan live after the chunk rows in dynamic shared memory.
__device__ __forceinline__ int* scan_tmp_big(uint8_t* dyn, int rows, int E) {
    return reinterpret_cast<int*>(dyn) + (size_t)rows * E;
}

struct RouterArgs {
    const void* x;
    const void* w_router;
    const void* rms_w;
    float rms_eps;
    void* x_norm;
    int permute;         // 1: with a single routing block, the last CTA also permutes
    void* xp;            //    ... and copies rows into xp when it is non-null
    Dims d;
    int T, tb, tt;       // routing block, tokens per CTA group
    int do_scan, unit_width, max_units, select_only;
    int scan_rows;       // histogram rows per scan chunk
    RouteBufs rb;
    DeviceStatus st;
};

// Grid (ceil(E / 2), ceil(T / tt)), tt tokens per CTA group.  In a logits CTA
// four warps share an expert row and take four tokens each, reading W_r, x and
// the RMSNorm scale straight from global memory with every load of a step in
// flight (the normalised input is never rounded before the logits).
// The last CTA of a group (arrival counter) takes the group's Top-k (with
// select_only the grid is (1, ceil(T / tt)) and the logits are already there).
// Selections are counted per routing block of tb tokens (global atomics); the
// last CTA overall scans those histograms into offsets and GEMM units.
template <typename Tin, int VEC, int EPL>
__global__ void __launch_bounds__(kThreads) router_kernel(RouterArgs a) {
    extern __shared__ __align__(16) uint8_t dyn[];
    __shared__ int hist[kMaxE];
    __shared__ int scan_tmp[kWarps + 1];
    __shared__ int s_flag;

    // Launched as a programmatic dependent, wait for the producer of x before
    // touching anything it writes; then let the next kernel (the few-token expert
    // kernel, which waits on the device for this grid's results) start its
    // prologue.  The router rows are constants: their L2 prefetch goes first.
    if (!a.select_only && threadIdx.x == 0 && blockIdx.y == 0) {
        const int e0 = blockIdx.x * kEG;
        const int ne = min(kEG, a.d.E - e0);
        const size_t row_bytes = (size_t)a.d.H * sizeof(Tin);
        const Tin* wr = static_cast<const Tin*>(a.w_router) + (size_t)e0 * a.d.H;
        auto aligned16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
        if (ne > 0 && (row_bytes * ne) % 16 == 0 && aligned16(wr))
            prefetch_l2_bulk(wr, (uint32_t)(row_bytes * ne));
        if (a.rms_w && row_bytes % 16 == 0 && blockIdx.x == 0 && aligned16(a.rms_w))
            prefetch_l2_bulk(a.rms_w, (uint32_t)row_bytes);
    }
    grid_dependency_wait();
    grid_dependents_launch();
    const Tin* x = static_cast<const Tin*>(a.x);
    const Tin* w_router = static_cast<const Tin*>(a.w_router);
    const Tin* rms_w = static_cast<const Tin*>(a.rms_w);
    RouteBufs& rb = a.rb;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.d.H, E = a.d.E, k = a.d.k;
    const int n_groups = gridDim.x, nblocks = gridDim.y;
    const int g = blockIdx.x, b = blockIdx.y;
    const int t0 = b * a.tt, nt = min(a.tt, a.T - t0);
    constexpr int kStride = 32 * VEC;

    if (!a.select_only) {
        // warp w: expert 2 g + (w >> 2), tokens 4 (w & 3) .. +3 of this group.
        // l = sum_j W_r[e][j] x'_j with x' = x (no pre-norm) or x * g * inv_rms; the
        // pre-norm is folded in: l = inv_rms * sum_j W_r[e][j] g_j x_j, fp32 throughout.
        const int e = g * kEG + (warp >> 2);
        const int tq = (warp & 3) * 4;
        if (e < E && tq < nt) {
            const Tin* wrow = w_router + (size_t)e * H;
            const Tin* xr[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) xr[j] = x + (size_t)(t0 + min(tq + j, nt - 1)) * H;
            float acc[4] = {0.f, 0.f, 0.f, 0.f}, ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
            for (int c = lane * VEC; c < H; c += kStride) {
                float wv[VEC], xv[4][VEC];
                load_vec<Tin, VEC>(wrow + c, wv);
                if (rms_w) {
                    float gv[VEC];
                    load_vec<Tin, VEC>(rms_w + c, gv);
#pragma unroll
                    for (int i = 0; i < VEC; ++i) wv[i] *= gv[i];
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) load_vec<Tin, VEC>(xr[j] + c, xv[j]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
#pragma unroll
                    for (int i = 0; i < VEC; ++i) {
                        acc[j] = fmaf(wv[i], xv[j][i], acc[j]);
                        ss[j] = fmaf(xv[j][i], xv[j][i], ss[j]);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
                    ss[j] += __shfl_xor_sync(0xffffffffu, ss[j], o);
                }
            }
            if (lane < 4 && tq + lane < nt) {
                float v = acc[0], q = ss[0];
#pragma unroll
                for (int j = 1; j < 4; ++j) if (lane == j) { v = acc[j]; q = ss[j]; }
                if (rms_w) v *= 1.0f / sqrtf(q / (float)H + a.rms_eps);
                rb.logits[(size_t)(t0 + tq + lane) * E + e] = v;
            }
            // the first expert's warps also write the normalised tokens for the experts
            if (rms_w && a.x_norm && e == 0) {
                float inv[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) inv[j] = 1.0f / sqrtf(ss[j] / (float)H + a.rms_eps);
#pragma unroll 1
                for (int j = 0; j < 4 && tq + j < nt; ++j) {
                    for (int c = lane * VEC; c < H; c += kStride) {
                        float xv[VEC], gv[VEC];
                        load_vec<Tin, VEC>(xr[j] + c, xv);
                        load_vec<Tin, VEC>(rms_w + c, gv);
#pragma unroll
                        for (int i = 0; i < VEC; ++i)
                            static_cast<Tin*>(a.x_norm)[(size_t)(t0 + tq + j) * H + c + i] =
                                from_f32<Tin>(xv[i] * inv[j] * gv[i]);
                    }
                }
            }
        }
        // the last logits CTA of this group continues
        __threadfence();
        __syncthreads();
        if (tid == 0) s_flag = (atomicAdd(&rb.tickets[b], 1) == n_groups - 1);
        __syncthreads();
        if (!s_flag) return;
        __threadfence();
    }

    // ---- Top-k of this CTA's tokens, one warp per token; counts per routing block
#pragma unroll 1
    for (int tl = warp; tl < nt; tl += kWarps) {
        const int t = t0 + tl;
        warp_topk<EPL>(rb.logits + (size_t)t * E, E, k, t, rb,
                       a.do_scan ? rb.block_hist + (size_t)(t / a.tb) * E : nullptr, a.st);
    }
    if (tid == 0 && !a.select_only) rb.tickets[b] = 0;   // every CTA of this group has arrived
    if (!a.do_scan) return;

    // ---- the last CTA scans the per-block histograms (and zeroes them for the next call)
    __threadfence();
    __syncthreads();
    if (nblocks > 1) {                 // with a single CTA group this CTA is the last
        if (tid == 0) s_flag = (atomicAdd(&rb.tickets[nblocks], 1) == nblocks - 1);
        __syncthreads();
        if (!s_flag) return;
        __threadfence();
    }
    const int nrb = (a.T + a.tb - 1) / a.tb;              // routing blocks
    // Column scan of the [nrb][E] histograms: block_off[b][e] = sum_{b' < b} hist[b'][e].
    // A chunk of rows is loaded with many loads in flight; P = kThreads / E threads
    // share an expert's column (two passes over the chunk, then a fix-up).
    int* chunk = reinterpret_cast<int*>(dyn);          // [cb][E] histogram rows
    const int cb = a.scan_rows;                        // rows per chunk (fits the smem)
    const int P = max(1, kThreads / E);                // threads per expert column
    int* psum = scan_tmp_big(dyn, cb, E);              // [P][E] part sums
    for (int e = tid; e < E; e += kThreads) hist[e] = 0;    // running count per expert
#pragma unroll 1
    for (int b0 = 0; b0 < nrb; b0 += cb) {
        const int nb = min(cb, nrb - b0);
        __syncthreads();
        const int n = nb * E;
        const int* src = rb.block_hist + (size_t)b0 * E;
#pragma unroll 1
        for (int i0 = tid; i0 < n; i0 += 16 * kThreads) {
            int v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int i = i0 + j * kThreads;
                v[j] = i < n ? __ldcg(src + i) : 0;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int i = i0 + j * kThreads;
                if (i < n) { chunk[i] = v[j]; rb.block_hist[(size_t)b0 * E + i] = 0; }
            }
        }
        __syncthreads();
        const int e = tid % E, part = tid / E;
        const int per = (nb + P - 1) / P;
        const int j0 = min(nb, part * per), j1 = min(nb, j0 + per);
        if (tid < P * E) {
            int sum = 0;
#pragma unroll 8
            for (int j = j0; j < j1; ++j) sum += chunk[j * E + e];
            psum[part * E + e] = sum;
        }
        __syncthreads();
        if (tid < P * E) {
            int run = hist[e];
            for (int q = 0; q < part; ++q) run += psum[q * E + e];
#pragma unroll 8
            for (int j = j0; j < j1; ++j) {
                rb.block_off[(size_t)(b0 + j) * E + e] = run;
                run += chunk[j * E + e];
            }
        }
        __syncthreads();
        if (tid < E) {
            int tot = hist[tid];
            for (int q = 0; q < P; ++q) tot += psum[q * E + tid];
            hist[tid] = tot;
        }
    }
    __syncthreads();
    int* cnt = chunk;                  // counts, then offsets
    int* ub = chunk + kMaxE;           // units per expert, then unit base
    for (int e = tid; e < E; e += kThreads) {
        cnt[e] = hist[e];
        rb.counts[e] = hist[e];
        ub[e] = (hist[e] + a.unit_width - 1) / a.unit_width;
    }
    __syncthreads();
    const int total = block_exclusive_scan(cnt, E, scan_tmp);
    int nu = block_exclusive_scan(ub, E, scan_tmp);
    if (nu > a.max_units) {
        if (tid == 0) report_error(a.st, kErrDeviceCheck);
        nu = a.max_units;
    }
    for (int e = tid; e < E; e += kThreads) {
        rb.offsets[e] = cnt[e];
        const int c = hist[e];
        for (int u = 0; u * a.unit_width < c; ++u) {
            const int idx = ub[e] + u;
            if (idx >= a.max_units) break;
            Unit un;
            un.expert = e;
            un.row_start = cnt[e] + u * a.unit_width;
            un.n_len = min(a.unit_width, c - u * a.unit_width);
            un.pad = 0;
            rb.units[idx] = un;
        }
    }
    if (tid == 0) {
        rb.offsets[E] = total;
        *rb.n_units = nu;
        if (nblocks > 1) rb.tickets[nblocks] = 0;
    }
    if (a.permute && nrb == 1) {       // decode: permute the single routing block right here
        __threadfence();
        __syncthreads();
        const Tin* x_in = a.x_norm ? static_cast<const Tin*>(a.x_norm) : x;
        permute_block<Tin>(x_in, static_cast<Tin*>(a.xp), a.d, a.T, a.tb, 0, 0, 1, rb,
                           reinterpret_cast<uint32_t*>(dyn + 2 * kMaxE * 4));
    }
}

template <typename Tin>
__global__ void __launch_bounds__(kThreads)
permute_kernel(const Tin* __restrict__ x_in, Tin* __restrict__ xp, Dims d, int T, int tb,
               RouteBufs rb) {
    extern __shared__ uint32_t sm[];
    grid_dependency_wait();          // the router's histograms (no-op unless a dependent launch)
    grid_dependents_launch();
    permute_block<Tin>(x_in, xp, d, T, tb, blockIdx.x, blockIdx.y, gridDim.y, rb, sm);
}

template <typename Tin, int VEC>
cudaError_t launch_router_t(const RouterArgs& a, dim3 grid, size_t smem, int pdl, cudaStream_t s) {
    const int epl = (a.d.E + 31) / 32;
    // Every instance may take up to kMaxRouterSmem bytes of dynamic shared memory; the
    // attribute is set once per instance (the three instances share one signature, so
    // a per-call "already allowed" record could not tell them apart).
    static std::once_flag configured[16];    // the attribute is set per device
    cudaError_t e = once_per_device(configured, [] {
        for (auto kernel : {router_kernel<Tin, VEC, 4>, router_kernel<Tin, VEC, 8>,
                            router_kernel<Tin, VEC, 32>}) {
            cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kMaxRouterSmem);
            if (r != cudaSuccess) return r;
        }
        return cudaSuccess;
    });
    if (e != cudaSuccess) return e;
    auto go = [&](auto kernel) -> cudaError_t {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = pdl ? 1 : 0;
        return cudaLaunchKernelEx(&cfg, kernel, a);
    };
    if (epl <= 4) return go(router_kernel<Tin, VEC, 4>);
    if (epl <= 8) return go(router_kernel<Tin, VEC, 8>);
    return go(router_kernel<Tin, VEC, 32>);
}

}  // namespace

cudaError_t launch_router(int dtype, const void* x, const void* w_router, const void* rms_w,
                          float rms_eps, void* x_norm, int permute, void* xp, const Dims& d,
                          int T, int tb, const RouteBufs& rb, int do_scan, int unit_width,
                          int max_units, int select_only, const DeviceStatus& ds,
                          cudaStream_t s, int pdl) {
    if (T <= 0) return cudaSuccess;
    if (d.E > kMaxE || d.k > kMaxK || tb > 128) return cudaErrorInvalidValue;
    const int tt = select_only ? kWarps : kMaxTB;   // select: one token per warp
    if (!select_only && tb != kMaxTB) return cudaErrorInvalidValue;
    const int nrb = (T + tb - 1) / tb;
    const int parts = std::max(1, kThreads / d.E);
    // scan chunk: up to 48 KB of histogram rows (all of them when they fit)
    const int scan_rows = std::max(1, std::min(nrb, (48 * 1024) / (d.E * 4)));
    RouterArgs a{x, w_router, rms_w, rms_eps, x_norm, permute, xp, d, T, tb, tt, do_scan,
                 unit_width, max_units, select_only, scan_rows, rb, ds};
    dim3 grid(select_only ? 1 : (d.E + kEG - 1) / kEG, (T + tt - 1) / tt);
    size_t smem = do_scan ? (size_t)(scan_rows + parts) * d.E * 4 : 0;            // scan chunk
    smem = std::max(smem, (size_t)2 * kMaxE * 4 + (size_t)d.E * 16 + (size_t)tb * d.k * 4);
    if (smem > (size_t)kMaxRouterSmem) return cudaErrorInvalidValue;
    if (dtype == 0)
        return d.H % 4 == 0 ? launch_router_t<float, 4>(a, grid, smem, pdl, s)
                            : launch_router_t<float, 1>(a, grid, smem, pdl, s);
    return d.H % 8 == 0 ? launch_router_t<__nv_bfloat16, 8>(a, grid, smem, pdl, s)
                        : launch_router_t<__nv_bfloat16, 1>(a, grid, smem, pdl, s);
}

cudaError_t launch_permute(int dtype, const void* x_in, void* xp, const Dims& d, int T, int tb,
                           const RouteBufs& rb, cudaStream_t s, int pdl) {
    if (T <= 0) return cudaSuccess;
    if (tb > 128) return cudaErrorInvalidValue;
    const int nblocks = (T + tb - 1) / tb;
    const int split = std::max(1, std::min(16, (2 * 148 + nblocks - 1) / nblocks));   // >= 2 CTAs/SM
    const size_t smem = (size_t)d.E * 4 * sizeof(uint32_t) + (size_t)tb * d.k * sizeof(int);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nblocks, split);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (dtype == 0)
        return cudaLaunchKernelEx(&cfg, permute_kernel<float>, (const float*)x_in, (float*)xp, d,
                                  T, tb, rb);
    return cudaLaunchKernelEx(&cfg, permute_kernel<__nv_bfloat16>, (const __nv_bfloat16*)x_in,
                              (__nv_bfloat16*)xp, d, T, tb, rb);
}

}  // namespace moe
