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

#include "device.cuh"
#include "layer.h"

namespace moe {
namespace {

template <typename T, int VEC>
__global__ void __launch_bounds__(128)
combine_kernel(const T* __restrict__ o, const T* __restrict__ sh, const T* __restrict__ res,
               T* __restrict__ y, const float* __restrict__ topk_w,
               const int32_t* __restrict__ token_slot, int H, int k) {
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
        for (int i = 0; i < k; ++i) {
            const T* src = o + (size_t)slot[i] * H + j0;
            T vals[VEC];
            if (VEC * sizeof(T) == 16) {
                *reinterpret_cast<uint4*>(vals) = __ldg(reinterpret_cast<const uint4*>(src));
            } else {
#pragma unroll
                for (int v = 0; v < VEC; ++v) vals[v] = src[v];
            }
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[v] = fmaf(wt[i], to_f32(vals[v]), acc[v]);
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
template <typename T>
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
        const T* g = wg + ((size_t)e * I + f) * H;
        const T* u = wu + ((size_t)e * I + f) * H;
        float ag = 0.f, au = 0.f;
        for (int j = 0; j < H; ++j) {
            float xv = to_f32(xr[j]);
            ag = fmaf(xv, to_f32(g[j]), ag);
            au = fmaf(xv, to_f32(u[j]), au);
        }
        h[(size_t)r * I + f] = from_f32<T>(silu_exact(ag) * au);
    }
}

// out[r][j] = h_r . Wd[e][j], one thread per (row, j).
template <typename T>
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
        const T* w = wd + ((size_t)e * H + j) * I;
        float a = 0.f;
        for (int f = 0; f < I; ++f) a = fmaf(to_f32(hr[f]), to_f32(w[f]), a);
        out[(size_t)r * H + j] = from_f32<T>(a);
    }
}

int simt_grid(size_t work) {
    size_t blocks = (work + 255) / 256;
    return (int)(blocks < 148 * 16 ? (blocks ? blocks : 1) : 148 * 16);
}

}  // namespace

cudaError_t launch_combine(int dtype, const void* o, const void* sh, const void* res, void* y,
                           const float* topk_w, const int32_t* token_slot, const Dims& d, int T,
                           cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    if (d.k > 16) return cudaErrorInvalidValue;
    if (dtype == 0) {
        if (d.H % 4 == 0)
            combine_kernel<float, 4><<<T, 128, 0, s>>>((const float*)o, (const float*)sh,
                                                       (const float*)res, (float*)y, topk_w,
                                                       token_slot, d.H, d.k);
        else
            combine_kernel<float, 1><<<T, 128, 0, s>>>((const float*)o, (const float*)sh,
                                                       (const float*)res, (float*)y, topk_w,
                                                       token_slot, d.H, d.k);
    } else {
        using bf = __nv_bfloat16;
        if (d.H % 8 == 0)
            combine_kernel<bf, 8><<<T, 128, 0, s>>>((const bf*)o, (const bf*)sh, (const bf*)res,
                                                    (bf*)y, topk_w, token_slot, d.H, d.k);
        else
            combine_kernel<bf, 1><<<T, 128, 0, s>>>((const bf*)o, (const bf*)sh, (const bf*)res,
                                                    (bf*)y, topk_w, token_slot, d.H, d.k);
    }
    return cudaGetLastError();
}

cudaError_t launch_simt_gate_up(int dtype, const void* xin, const void* w_gate, const void* w_up,
                                const int32_t* slot_expert, const int32_t* n_rows_dev,
                                int max_rows, int H, int I, void* hbuf, cudaStream_t s) {
    if (max_rows <= 0) return cudaSuccess;
    int grid = simt_grid((size_t)max_rows * I);
    if (dtype == 0)
        simt_gate_up_kernel<float><<<grid, 256, 0, s>>>((const float*)xin, (const float*)w_gate,
                                                       (const float*)w_up, slot_expert,
                                                       n_rows_dev, max_rows, H, I, (float*)hbuf);
    else
        simt_gate_up_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
            (const __nv_bfloat16*)xin, (const __nv_bfloat16*)w_gate, (const __nv_bfloat16*)w_up,
            slot_expert, n_rows_dev, max_rows, H, I, (__nv_bfloat16*)hbuf);
    return cudaGetLastError();
}

cudaError_t launch_simt_down(int dtype, const void* hbuf, const void* w_down,
                             const int32_t* slot_expert, const int32_t* n_rows_dev, int max_rows,
                             int H, int I, void* out, cudaStream_t s) {
    if (max_rows <= 0) return cudaSuccess;
    int grid = simt_grid((size_t)max_rows * H);
    if (dtype == 0)
        simt_down_kernel<float><<<grid, 256, 0, s>>>((const float*)hbuf, (const float*)w_down,
                                                    slot_expert, n_rows_dev, max_rows, H, I,
                                                    (float*)out);
    else
        simt_down_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
            (const __nv_bfloat16*)hbuf, (const __nv_bfloat16*)w_down, slot_expert, n_rows_dev,
            max_rows, H, I, (__nv_bfloat16*)out);
    return cudaGetLastError();
}

}  // namespace moe
