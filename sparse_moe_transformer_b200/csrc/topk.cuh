// topk.cuh -- warp Top-k selection with renormalised weights, shared by the
// CUDA-core router (routing.cu) and the one-CTA tensor-core router (router_tc.cu).
//
// Router equation: page "3C . Talker MoE (20 lop, 128 Experts Top-6) & Dau ra
// ma ngu nghia c_0", section 3: p = softmax(W_r x), S = Top-k, w_i = p_i /
// sum_{j in S} p_j.  Softmax is strictly increasing, so S is taken on the fp32
// logits, and w_i = exp(l_i - l_max) / sum_{j in S} exp(l_j - l_max) needs only
// the k selected logits.
#pragma once

#include <stdint.h>

#include "device.cuh"

namespace moe {

// Order-preserving map of an fp32 value to uint32 (larger float -> larger key;
// -0 and +0 map to the same key, so they tie like equal values).
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k of one token (one warp): EPL logits per lane (experts lane + 32 i).
// Each round: every lane proposes its best unselected expert; the warp takes
// the largest key (redux.sync max) and, among equal keys, the lowest expert
// index (redux.sync min) -- the lower-index tie rule.  On return lane j < k
// holds selection j: its expert in my_e and its renormalised weight in my_w.
template <int EPL>
__device__ __forceinline__ void warp_topk_select(const float (&lv)[EPL], int E, int k, int& my_e,
                                                 float& my_w, const DeviceStatus& st) {
    const int lane = threadIdx.x & 31;
    uint32_t taken = 0;                 // bit i: element lane + 32 i already selected
    float vmax = 0.f, z = 0.f, my_v = 0.f;
    my_e = -1;
#pragma unroll 1
    for (int r = 0; r < k; ++r) {
        uint32_t bk = 0;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            const uint32_t key = order_key(lv[i]);
            if (e < E && !(taken & (1u << i)) && (bi == 0x7fffffff || key > bk)) { bk = key; bi = e; }
        }
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, bk);
        int e_win = (int)__reduce_min_sync(0xffffffffu, (bi != 0x7fffffff && bk == kmax)
                                                            ? (uint32_t)bi : 0xffffffffu);
        if (e_win < 0 || e_win >= E) {            // cannot happen for k <= E
            if (lane == 0) report_error(st, kErrDeviceCheck);
            e_win = r;
        }
        if ((e_win & 31) == lane) taken |= 1u << (e_win >> 5);
        float bv = 0.f;
#pragma unroll
        for (int i = 0; i < EPL; ++i) if (lane + 32 * i == e_win) bv = lv[i];
        bv = __shfl_sync(0xffffffffu, bv, e_win & 31);
        if (r == 0) vmax = bv;
        const float ex = expf(bv - vmax);
        z += ex;
        if (lane == r) { my_e = e_win; my_v = ex; }   // lane r keeps selection r
    }
    my_w = my_v / z;
}

}  // namespace moe
