// combine_simt.cu -- the weighted combine and the CUDA-core expert kernels.
//
// Combine (page "3C . Talker MoE (20 lop, 128 Experts Top-6) & Dau ra ma ngu
// nghia c_0", section 3): y_t = Shared(x_t) + sum_{i in S_t} w_ti Expert_i(x_t),
// plus the residual when one is given (lab page, section [3C]: the layer input
// is added back).  Sum order is fixed (slot 0..k-1, then shared, then residual)
// so results are deterministic.
//
// The CUDA-core expert kernels compute the SwiGLU experts (page "print(model)
// Qwen3-TTS", SwiGLU section: down(SiLU(gate x) * up x)) with fp32 FMA
// accumulation.  They serve fp32 layers (where a 1e-5 tolerance rules out TF32
// tensor cores) and bf16 shapes the tensor-core kernel does not tile.
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

#include "device.cuh"
#include "layer.h"

namespace moe {
namespace {

template <typename T, int VEC>
__global__ void __launch_bounds__(128)
combine_kernel(const T* __restrict__ o, const T* __restrict__ sh, const T* res, T* y,
               const float* __restrict__ topk_w,
               const int32_t* __restrict__ token_slot, int H, int k) {
    grid_dependency_wait();          // expert outputs (no-op unless a dependent launch)
    grid_dependents_launch();
    const int t = blockIdx.x;
    __shared__ int slot[16];
    __shared__ float wt[16];
    if (threadIdx.x < k) {
        slot[threadIdx.x] = token_slot[(size_t)t * k + threadIdx.x];
        wt[threadIdx.x] = topk_w[(size_t)t * k + threadIdx.x];
    }
    __syncthreads();
    for (int j0 = threadIdx.x * VEC; j0 < H; j0 += blockDim.x * VEC) {
        float acc[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
        // slot rows in groups of 8 with all loads of a group in flight, summed in slot order
#pragma unroll 1
        for (int i0 = 0; i0 < k; i0 += 8) {
            T vals[8][VEC];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i0 + i < k) {
                    const T* src = o + (size_t)slot[i0 + i] * H + j0;
                    if (VEC * sizeof(T) == 16) {
                        *reinterpret_cast<uint4*>(vals[i]) = __ldg(reinterpret_cast<const uint4*>(src));
                    } else {
#pragma unroll
                        for (int v = 0; v < VEC; ++v) vals[i][v] = src[v];
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i0 + i < k) {
#pragma unroll
                    for (int v = 0; v < VEC; ++v) acc[v] = fmaf(wt[i0 + i], to_f32(vals[i][v]), acc[v]);
                }
            }
        }
        const size_t base = (size_t)t * H + j0;
        if (sh) {
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[v] += to_f32(sh[base + v]);
        }
        if (res) {
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[v] += to_f32(res[base + v]);
        }
        T out[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) out[v] = from_f32<T>(acc[v]);
        if (VEC * sizeof(T) == 16) {
            *reinterpret_cast<uint4*>(y + base) = *reinterpret_cast<const uint4*>(out);
        } else {
#pragma unroll
            for (int v = 0; v < VEC; ++v) y[base + v] = out[v];
        }
    }
}

// h[r][f] = SiLU(x_r . Wg[e][f]) * (x_r . Wu[e][f]), one thread per (row, f).
template <typename T, bool PACKED>
__global__ void __launch_bounds__(256)
simt_gate_up_kernel(const T* __restrict__ xin, const T* __restrict__ wg, const T* __restrict__ wu,
                    const int32_t* __restrict__ slot_expert, const int32_t* __restrict__ n_rows,
                    int max_rows, int H, int I, T* __restrict__ h) {
    const int rows = n_rows ? min(*n_rows, max_rows) : max_rows;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < (size_t)rows * I;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int r = (int)(idx / I), f = (int)(idx % I);
        const int e = slot_expert ? slot_expert[r] : 0;
        const T* xr = xin + (size_t)r * H;
        float ag = 0.f, au = 0.f;
        for (int j = 0; j < H; ++j) {
            const float xv = to_f32(xr[j]);
            if (PACKED) {
                ag = fmaf(xv, to_f32(wg[packed_gu_offset(e, f, j, 0, I, H)]), ag);
                au = fmaf(xv, to_f32(wg[packed_gu_offset(e, f, j, 1, I, H)]), au);
            } else {
                ag = fmaf(xv, to_f32(wg[((size_t)e * I + f) * H + j]), ag);
                au = fmaf(xv, to_f32(wu[((size_t)e * I + f) * H + j]), au);
            }
        }
        h[(size_t)r * I + f] = from_f32<T>(silu_exact(ag) * au);
    }
}

// out[r][j] = h_r . Wd[e][j], one thread per (row, j).
template <typename T, bool PACKED>
__global__ void __launch_bounds__(256)
simt_down_kernel(const T* __restrict__ h, const T* __restrict__ wd,
                 const int32_t* __restrict__ slot_expert, const int32_t* __restrict__ n_rows,
                 int max_rows, int H, int I, T* __restrict__ out) {
    const int rows = n_rows ? min(*n_rows, max_rows) : max_rows;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < (size_t)rows * H;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int r = (int)(idx / H), j = (int)(idx % H);
        const int e = slot_expert ? slot_expert[r] : 0;
        const T* hr = h + (size_t)r * I;
        float a = 0.f;
        for (int f = 0; f < I; ++f) {
            const size_t off = PACKED ? packed_down_offset(e, j, f, H, I) : ((size_t)e * H + j) * I + f;
            a = fmaf(to_f32(hr[f]), to_f32(wd[off]), a);
        }
        out[(size_t)r * H + j] = from_f32<T>(a);
    }
}

// dst[v] for v over 16-byte vectors of the tile-contiguous layout (see layer.h):
// vector v holds physical chunk (v & 7) of row r, i.e. logical chunk (v & 7) ^ (r & 7).
// Gate/up (src1 != nullptr): pair index (e, mt, kb), member = gate / up.
// Down (src1 == nullptr): pair index (e, mt2, kb), member = row block 2 mt2 + member.
__global__ void __launch_bounds__(256)
pack_tiles_kernel(const uint4* __restrict__ src0, const uint4* __restrict__ src1,
                  uint4* __restrict__ dst, int E, int R, int C, int kpair, size_t total) {
    const int MT = R / 128, KB = C / 64;
    const int NB = (src1 || kpair) ? MT : (MT + 1) / 2;   // row blocks (or block pairs) per expert
    const int KP = kpair ? KB / 2 : KB;                     // pairs along the columns
    for (size_t v = blockIdx.x * (size_t)blockDim.x + threadIdx.x; v < total;
         v += (size_t)gridDim.x * blockDim.x) {
        const int r = (int)((v >> 3) & 127);
        const int c8 = (int)(v & 7) ^ (r & 7);
        size_t rest = v >> 10;
        const int member = (int)(rest & 1); rest >>= 1;
        int kb = (int)(rest % KP); rest /= KP;
        const int nb = (int)(rest % NB);
        const int e = (int)(rest / NB);
        const uint4* src = src0;
        int mt = nb;
        if (kpair) {
            kb = 2 * kb + member;
        } else if (src1) {
            src = member ? src1 : src0;
        } else {
            mt = 2 * nb + member;
            if (mt >= MT) continue;                    // the zero-filled odd half
        }
        dst[v] = src[(((size_t)e * R + mt * 128 + r) * C + kb * 64) / 8 + c8];
    }
}

// y_t = sum_j w_tj (sum_b o_part[b][t k + j]) + sum_b o_part[b][T k + t] [+ r_t].
// Eight threads (lanes 8 g .. 8 g + 7 of a warp) share 4 columns of one token
// (k <= 8): thread s takes routed slot j = s (the sum of its block partials in
// block order, times w_tj) and the shared expert's blocks b = s, s + 8, ...; the
// eight values are then added in a fixed butterfly order, so the result does not
// depend on timing.  Every load of a thread is issued before its first add.
constexpr int kCombineSub = 8;
constexpr int kCombineMaxLoads = 16;
__global__ void __launch_bounds__(256)
combine_partials_kernel(const float* __restrict__ o_part, int n_blk, int n_blk_s,
                        const __nv_bfloat16* res, __nv_bfloat16* y,
                        const float* __restrict__ topk_w, int T, int H, int k) {
    grid_dependency_wait();                    // partials of the expert kernel
    grid_dependents_launch();                  // the next router may start its prologue
    const int per_t = H / 4;
    const int gid = blockIdx.x * (blockDim.x / kCombineSub) + threadIdx.x / kCombineSub;
    const int sub = threadIdx.x % kCombineSub;
    const bool live = gid < T * per_t;
    const int t = live ? gid / per_t : 0, c4 = live ? (gid - t * per_t) * 4 : 0;
    const size_t S = (size_t)T * k, bstride = (S + T) * H;
    // thread `sub` holds routed slot j = sub (k <= kCombineSub: at most one) as
    // items 0 .. n_r - 1, then shared blocks sub, sub + 8, ... as the next items
    const bool has_slot = live && sub < k;
    const int n_r = has_slot ? n_blk : 0;
    const int n_s = live && sub < n_blk_s ? (n_blk_s - sub + kCombineSub - 1) / kCombineSub : 0;
    const float* pr = o_part + ((size_t)t * k + sub) * H + c4;
    const float* ps = o_part + (S + t) * H + c4 + (size_t)sub * bstride;
    const float w = has_slot ? __ldg(topk_w + (size_t)t * k + sub) : 0.f;
    float4 v[kCombineMaxLoads];
#pragma unroll
    for (int i = 0; i < kCombineMaxLoads; ++i) {
        if (i < n_r) v[i] = __ldg(reinterpret_cast<const float4*>(pr + (size_t)i * bstride));
        else if (i < n_r + n_s)
            v[i] = __ldg(reinterpret_cast<const float4*>(ps + (size_t)(i - n_r) * kCombineSub * bstride));
    }
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f), sh = sum;
#pragma unroll
    for (int i = 0; i < kCombineMaxLoads; ++i) {
        if (i < n_r) { sum.x += v[i].x; sum.y += v[i].y; sum.z += v[i].z; sum.w += v[i].w; }
        else if (i < n_r + n_s) { sh.x += v[i].x; sh.y += v[i].y; sh.z += v[i].z; sh.w += v[i].w; }
    }
    float4 acc = make_float4(fmaf(w, sum.x, sh.x), fmaf(w, sum.y, sh.y), fmaf(w, sum.z, sh.z),
                             fmaf(w, sum.w, sh.w));
#pragma unroll
    for (int o = 1; o < kCombineSub; o <<= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
    }
    if (!live || sub != 0) return;
    float o[4] = {acc.x, acc.y, acc.z, acc.w};
    __nv_bfloat16 out[4];
    if (res) {
        const uint2 rv = *reinterpret_cast<const uint2*>(res + (size_t)t * H + c4);
        const __nv_bfloat16* r4 = reinterpret_cast<const __nv_bfloat16*>(&rv);
#pragma unroll
        for (int q = 0; q < 4; ++q) o[q] += __bfloat162float(r4[q]);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) out[q] = __float2bfloat16_rn(o[q]);
    *reinterpret_cast<uint2*>(y + (size_t)t * H + c4) = *reinterpret_cast<const uint2*>(out);
}

int simt_grid(size_t work) {
    size_t blocks = (work + 255) / 256;
    return (int)(blocks < 148 * 16 ? (blocks ? blocks : 1) : 148 * 16);
}

}  // namespace

cudaError_t launch_combine(int dtype, const void* o, const void* sh, const void* res, void* y,
                           const float* topk_w, const int32_t* token_slot, const Dims& d, int T,
                           cudaStream_t s, int pdl) {
    if (T <= 0) return cudaSuccess;
    if (d.k > 16) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(T);
    cfg.blockDim = dim3(128);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    using bf = __nv_bfloat16;
    if (dtype == 0) {
        const float *o_ = (const float*)o, *sh_ = (const float*)sh, *res_ = (const float*)res;
        if (d.H % 4 == 0)
            return cudaLaunchKernelEx(&cfg, combine_kernel<float, 4>, o_, sh_, res_, (float*)y,
                                      topk_w, token_slot, d.H, d.k);
        return cudaLaunchKernelEx(&cfg, combine_kernel<float, 1>, o_, sh_, res_, (float*)y, topk_w,
                                  token_slot, d.H, d.k);
    }
    const bf *o_ = (const bf*)o, *sh_ = (const bf*)sh, *res_ = (const bf*)res;
    if (d.H % 8 == 0)
        return cudaLaunchKernelEx(&cfg, combine_kernel<bf, 8>, o_, sh_, res_, (bf*)y, topk_w,
                                  token_slot, d.H, d.k);
    return cudaLaunchKernelEx(&cfg, combine_kernel<bf, 1>, o_, sh_, res_, (bf*)y, topk_w,
                              token_slot, d.H, d.k);
}

cudaError_t launch_combine_partials(const float* o_part, int n_blk, int n_blk_s,
                                    const void* residual, void* y, const float* topk_w,
                                    const Dims& d, int T, int pdl, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    if (d.H % 4 || n_blk < 1) return cudaErrorInvalidValue;
    // loads per thread: its slot's blocks plus its shared blocks
    if (d.k > kCombineSub || n_blk + (n_blk_s + kCombineSub - 1) / kCombineSub > kCombineMaxLoads)
        return cudaErrorInvalidValue;
    using bf = __nv_bfloat16;
    const int groups = T * (d.H / 4);
    const int per_block = 256 / kCombineSub;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((groups + per_block - 1) / per_block);
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, combine_partials_kernel, o_part, n_blk, n_blk_s,
                              (const bf*)residual, (bf*)y, topk_w, T, d.H, d.k);
}

cudaError_t launch_simt_gate_up(int dtype, const void* xin, const void* w_gate, const void* w_up,
                                int packed, const int32_t* slot_expert, const int32_t* n_rows_dev,
                                int max_rows, int H, int I, void* hbuf, cudaStream_t s) {
    if (max_rows <= 0) return cudaSuccess;
    int grid = simt_grid((size_t)max_rows * I);
    using bf = __nv_bfloat16;
    if (dtype == 0)
        simt_gate_up_kernel<float, false><<<grid, 256, 0, s>>>(
            (const float*)xin, (const float*)w_gate, (const float*)w_up, slot_expert, n_rows_dev,
            max_rows, H, I, (float*)hbuf);
    else if (packed)
        simt_gate_up_kernel<bf, true><<<grid, 256, 0, s>>>(
            (const bf*)xin, (const bf*)w_gate, (const bf*)w_up, slot_expert, n_rows_dev, max_rows,
            H, I, (bf*)hbuf);
    else
        simt_gate_up_kernel<bf, false><<<grid, 256, 0, s>>>(
            (const bf*)xin, (const bf*)w_gate, (const bf*)w_up, slot_expert, n_rows_dev, max_rows,
            H, I, (bf*)hbuf);
    return cudaGetLastError();
}

cudaError_t launch_simt_down(int dtype, const void* hbuf, const void* w_down, int packed,
                             const int32_t* slot_expert, const int32_t* n_rows_dev, int max_rows,
                             int H, int I, void* out, cudaStream_t s) {
    if (max_rows <= 0) return cudaSuccess;
    int grid = simt_grid((size_t)max_rows * H);
    using bf = __nv_bfloat16;
    if (dtype == 0)
        simt_down_kernel<float, false><<<grid, 256, 0, s>>>(
            (const float*)hbuf, (const float*)w_down, slot_expert, n_rows_dev, max_rows, H, I,
            (float*)out);
    else if (packed)
        simt_down_kernel<bf, true><<<grid, 256, 0, s>>>((const bf*)hbuf, (const bf*)w_down,
                                                        slot_expert, n_rows_dev, max_rows, H, I,
                                                        (bf*)out);
    else
        simt_down_kernel<bf, false><<<grid, 256, 0, s>>>((const bf*)hbuf, (const bf*)w_down,
                                                         slot_expert, n_rows_dev, max_rows, H, I,
                                                         (bf*)out);
    return cudaGetLastError();
}

cudaError_t launch_pack_tiles(const void* src0, const void* src1, void* dst, int E, int R, int C,
                              cudaStream_t s) {
    if (R % 128 || C % 64) return cudaErrorInvalidValue;
    const int NB = src1 ? R / 128 : (R / 128 + 1) / 2;
    const size_t total = (size_t)E * NB * (C / 64) * 2 * 1024;     // 16-byte vectors
    const int grid = (int)std::min<size_t>((total + 255) / 256, 148 * 32);
    pack_tiles_kernel<<<grid, 256, 0, s>>>((const uint4*)src0, (const uint4*)src1, (uint4*)dst,
                                           E, R, C, 0, total);
    return cudaGetLastError();
}

cudaError_t launch_pack_kpairs(const void* src, void* dst, int R, int C, cudaStream_t s) {
    if (R % 128 || C % 128) return cudaErrorInvalidValue;
    const size_t total = (size_t)(R / 128) * (C / 128) * 2 * 1024;  // 16-byte vectors
    const int grid = (int)std::min<size_t>((total + 255) / 256, 148 * 32);
    pack_tiles_kernel<<<grid, 256, 0, s>>>((const uint4*)src, nullptr, (uint4*)dst, 1, R, C, 1,
                                           total);
    return cudaGetLastError();
}

}  // namespace moe
