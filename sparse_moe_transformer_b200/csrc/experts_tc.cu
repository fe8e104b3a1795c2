// experts_tc.cu -- grouped SwiGLU expert GEMM on sm_100a tensor cores.
//
// Each expert is down(SiLU(gate x) * up x) with no bias (page "print(model)
// Qwen3-TTS", SwiGLU feed-forward section); the routed experts are 1024->384->1024
// and the shared one 1024->768->1024 (page "3C . Talker MoE", section 1).
//
// Design (swap-AB): the MMA's M side is 128 weight rows (output features), its N
// side the tokens of one expert (any multiple of 16 up to the tile width), so a
// ragged token count costs at most 15 padded columns instead of a 128-row tile.
//   gate/up tile: D_gate = Wg[e][128 rows] . X^T and D_up = Wu[e][128 rows] . X^T
//                 share the B operand; the epilogue forms SiLU(D_gate) * D_up.
//   down tile:    D = Wd[e][128 rows] . Hrows^T.
// A and B are staged by TMA (128-byte swizzle, no multicast) into a ring of
// shared-memory stages; one thread issues tcgen05.mma into TMEM accumulators;
// four epilogue warps read TMEM with tcgen05.ld and store bf16 rows.
//
// The kernel is persistent: CTAs take tiles from a global counter, gate/up tiles
// first, then down tiles.  When both phases run in one launch, a down tile of a
// unit waits (bounded by a time limit) until the unit's gate/up tiles have
// published their h rows; every gate/up tile is taken before any down tile and
// never waits, so the wait always ends.  Every wait in the kernel is bounded; a
// wait that runs out records MOE_ERR_TIMEOUT and the CTA drains and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "device.cuh"
#include "layer.h"

namespace moe {
namespace {

constexpr int kBM = 128;           // weight rows per tile (MMA M)
constexpr int kBK = 64;            // K elements per stage: one 128-byte swizzle atom
constexpr int kThreads = 192;      // warp 0 TMA producer, warp 1 MMA, warps 2-5 epilogue
constexpr int kRing = 4;           // tile-info ring depth
constexpr int kABytes = kBM * kBK * 2;
constexpr int kBoxRows = 16;       // activation rows per TMA box
constexpr int kBoxBytes = kBoxRows * kBK * 2;
constexpr uint64_t kDrainLimitNs = 200ull * 1000 * 1000;

constexpr int pow2_at_least(int v) {
    int p = 32;
    while (p < v) p <<= 1;
    return p;
}

template <int BN>
struct TcCfg {
    static constexpr int kStages = BN <= 32 ? 6 : (BN <= 128 ? 4 : 3);
    static constexpr int kAcc = (4 * BN <= 512) ? 2 : 1;           // accumulator buffers
    static constexpr int kTmemCols = pow2_at_least(kAcc * 2 * BN);
    static constexpr int kBBytes = BN * kBK * 2;
    static constexpr int kStageBytes = 2 * kABytes + kBBytes;
    static constexpr int kCtrlBytes = 1024;
    static constexpr int kSmem = kStages * kStageBytes + kCtrlBytes + 1024;   // + align slack
    static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
    static_assert(kTmemCols <= 512, "TMEM has 512 columns");
};

struct Tile {
    int phase;       // 0 gate/up, 1 down, -1 no more work
    int unit;
    int mt;          // 128-row block of the weight matrix
    int expert;
    int row_start;   // first activation row
    int n_len;       // activation rows (MMA N before rounding to 16)
};

__device__ __forceinline__ Tile decode_tile(int i, int n_units, const TcArgs& a, int mt_gu,
                                            int mt_dn, int bn) {
    Tile t;
    const int n_gu = (a.phases & 1) ? n_units * mt_gu : 0;
    const int n_dn = (a.phases & 2) ? n_units * mt_dn : 0;
    if (i < n_gu) {
        t.phase = 0; t.unit = i / mt_gu; t.mt = i - t.unit * mt_gu;
    } else if (i - n_gu < n_dn) {
        const int j = i - n_gu;
        t.phase = 1; t.unit = j / mt_dn; t.mt = j - t.unit * mt_dn;
    } else {
        t.phase = -1; t.unit = t.mt = t.expert = t.row_start = t.n_len = 0;
        return t;
    }
    if (a.dense_T > 0) {
        t.expert = 0;
        t.row_start = t.unit * bn;
        t.n_len = min(bn, a.dense_T - t.row_start);
    } else {
        const Unit u = a.units[t.unit];
        t.expert = u.expert; t.row_start = u.row_start; t.n_len = u.n_len;
    }
    return t;
}

template <int BN>
__device__ __forceinline__ void tc_experts_body(const TcMaps& maps, const TcArgs& a) {
    using C = TcCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* ctrl = smem + C::kStages * C::kStageBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
    uint64_t* empty = full + C::kStages;
    uint64_t* accfull = empty + C::kStages;
    uint64_t* accempty = accfull + C::kAcc;
    uint64_t* tfull = accempty + C::kAcc;
    uint64_t* tempty = tfull + kRing;
    uint64_t* pubbar = tempty + kRing;      // 4 epilogue warps finished a gate/up tile
    uint64_t* drainbar = pubbar + 1;        // all MMAs of this CTA completed
    Tile* ring = reinterpret_cast<Tile*>(drainbar + 1);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring + kRing);
    int* s_misc = reinterpret_cast<int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int mt_gu = a.I / kBM, mt_dn = a.H / kBM;
    int* tile_counter = a.sync;
    int* exit_counter = a.sync + 1;
    int* done = a.sync + 2;
    const uint64_t limit = a.wait_limit_ns;

    const int n_units = a.dense_T > 0 ? (a.dense_T + BN - 1) / BN : *a.n_units;
    const int n_tiles = n_units * (((a.phases & 1) ? mt_gu : 0) + ((a.phases & 2) ? mt_dn : 0));

    if (tid == 0) {
        for (int s = 0; s < C::kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int s = 0; s < C::kAcc; ++s) { mbar_init(&accfull[s], 1); mbar_init(&accempty[s], 4); }
        for (int s = 0; s < kRing; ++s) { mbar_init(&tfull[s], 1); mbar_init(&tempty[s], 5); }
        mbar_init(pubbar, 4);
        mbar_init(drainbar, 1);
        mbar_fence_init();
        tma_prefetch_desc(&maps.a_gate); tma_prefetch_desc(&maps.a_up);
        tma_prefetch_desc(&maps.a_down); tma_prefetch_desc(&maps.b_x);
        tma_prefetch_desc(&maps.b_h);
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ scheduler + TMA producer
        const uint64_t pol_w = policy_evict_first();   // weights stream through once
        const uint64_t pol_x = policy_evict_last();    // activations are re-read per tile
        uint32_t it = 0;
        int tc = 0;
        bool ok = true, stuck_pending = a.inject_stuck != 0;
        while (true) {
            int i = (ok && !error_pending(a.st)) ? atomicAdd(tile_counter, 1) : n_tiles;
            Tile t = decode_tile(i, n_units, a, mt_gu, mt_dn, BN);
            const int r = tc % kRing;
            if (!mbar_wait(&tempty[r], ((tc / kRing) & 1) ^ 1, a.st, limit)) { ok = false; break; }
            ring[r] = t;
            mbar_arrive(&tfull[r]);
            ++tc;
            if (t.phase < 0) break;
            if (t.phase == 1 && (a.phases & 1)) {
                // dependency: the unit's gate/up tiles must have published their h rows
                const int target = mt_gu + (stuck_pending ? 1 : 0);
                stuck_pending = false;
                const int* flag = done + t.unit;
                if (ld_acquire_gpu(flag) < target) {
                    const uint64_t t0 = globaltimer_ns();
                    while (ld_acquire_gpu(flag) < target) {
                        __nanosleep(64);
                        if (globaltimer_ns() - t0 > limit) {
                            report_error(a.st, kErrTimeout);
                            ok = false;     // finish this tile (output invalid), take no more
                            break;
                        }
                    }
                }
                fence_proxy_async_global();
            }
            const int nb16 = (t.n_len + kBoxRows - 1) / kBoxRows;
            const int KB = (t.phase == 0 ? a.H : a.I) / kBK;
            const uint32_t bytes = (t.phase == 0 ? 2 : 1) * kABytes + nb16 * kBoxBytes;
            bool fail = false;
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const int s = it % C::kStages;
                if (!mbar_wait(&empty[s], ((it / C::kStages) & 1) ^ 1, a.st, limit)) {
                    fail = true;
                    break;
                }
                uint8_t* A0 = smem + s * C::kStageBytes;
                uint8_t* B = A0 + 2 * kABytes;
                mbar_arrive_expect_tx(&full[s], bytes);
                if (t.phase == 0) {
                    const int row = t.expert * a.I + t.mt * kBM;
                    tma_load_2d(A0, &maps.a_gate, &full[s], kb * kBK, row, pol_w);
                    tma_load_2d(A0 + kABytes, &maps.a_up, &full[s], kb * kBK, row, pol_w);
                    for (int j = 0; j < nb16; ++j)
                        tma_load_2d(B + j * kBoxBytes, &maps.b_x, &full[s], kb * kBK,
                                    t.row_start + j * kBoxRows, pol_x);
                } else {
                    const int row = t.expert * a.H + t.mt * kBM;
                    tma_load_2d(A0, &maps.a_down, &full[s], kb * kBK, row, pol_w);
                    for (int j = 0; j < nb16; ++j)
                        tma_load_2d(B + j * kBoxBytes, &maps.b_h, &full[s], kb * kBK,
                                    t.row_start + j * kBoxRows, pol_x);
                }
            }
            if (fail) { ok = false; break; }
        }
        // drain: copies still in flight must land before the CTA exits
        for (uint32_t q = (it > (uint32_t)C::kStages ? it - C::kStages : 0); q < it; ++q)
            mbar_wait(&full[q % C::kStages], (q / C::kStages) & 1, a.st, kDrainLimitNs);
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        uint32_t it = 0;
        int tc = 0, ac = 0;
        while (true) {
            const int r = tc % kRing;
            if (!mbar_wait(&tfull[r], (tc / kRing) & 1, a.st, limit)) break;
            const Tile t = ring[r];
            mbar_arrive(&tempty[r]);
            ++tc;
            if (t.phase < 0) break;
            const int acc = ac % C::kAcc;
            if (!mbar_wait(&accempty[acc], ((ac / C::kAcc) & 1) ^ 1, a.st, limit)) break;
            tc_fence_after();
            const int N = ((t.n_len + 15) / 16) * 16;
            const uint32_t idesc = idesc_bf16_f32(kBM, N);
            const uint32_t d_gate = tmem_base + acc * 2 * BN;
            const uint32_t d_up = d_gate + BN;
            const int KB = (t.phase == 0 ? a.H : a.I) / kBK;
            bool fail = false;
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const int s = it % C::kStages;
                if (!mbar_wait(&full[s], (it / C::kStages) & 1, a.st, limit)) { fail = true; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + s * C::kStageBytes);
                const uint32_t a1 = a0 + kABytes;
                const uint32_t b0 = a0 + 2 * kABytes;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    const uint64_t bd = smem_desc_sw128(b0 + kk * 32);
                    const uint32_t accum = (kb | kk) != 0;
                    tc_mma_bf16(d_gate, smem_desc_sw128(a0 + kk * 32), bd, idesc, accum);
                    if (t.phase == 0)
                        tc_mma_bf16(d_up, smem_desc_sw128(a1 + kk * 32), bd, idesc, accum);
                }
                tc_commit(&empty[s]);   // frees the stage once these MMAs have read it
            }
            if (fail) break;
            tc_commit(&accfull[acc]);
            ++ac;
        }
        tc_commit(drainbar);
        mbar_wait(drainbar, 0, a.st, kDrainLimitNs);
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue (TMEM -> bf16 rows)
        const int q = warp & 3;            // TMEM lanes 32q..32q+31 belong to this warp
        __nv_bfloat16* hbuf = static_cast<__nv_bfloat16*>(a.hbuf);
        __nv_bfloat16* outb = static_cast<__nv_bfloat16*>(a.out);
        int tc = 0, ac = 0, pub = 0;
        while (true) {
            const int r = tc % kRing;
            if (!mbar_wait(&tfull[r], (tc / kRing) & 1, a.st, limit)) break;
            const Tile t = ring[r];
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[r]);
            ++tc;
            if (t.phase < 0) break;
            const int acc = ac % C::kAcc;
            if (!mbar_wait(&accfull[acc], (ac / C::kAcc) & 1, a.st, limit)) break;
            tc_fence_after();
            const uint32_t tg = tmem_base + acc * 2 * BN + (static_cast<uint32_t>(q * 32) << 16);
            const uint32_t tu = tg + BN;
            const int f = t.mt * kBM + q * 32 + lane;
            const int nc = (t.n_len + 15) / 16;
            if (t.phase == 0) {
                __nv_bfloat16* dst = hbuf + (size_t)t.row_start * a.I + f;
                for (int c = 0; c < nc; ++c) {
                    float g[16], u[16];
                    tmem_ld16(tg + c * 16, g);
                    tmem_ld16(tu + c * 16, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int n = c * 16 + j;
                        if (n < t.n_len)
                            dst[(size_t)n * a.I] = __float2bfloat16_rn(silu_fast(g[j]) * u[j]);
                    }
                }
            } else {
                __nv_bfloat16* dst = outb + (size_t)t.row_start * a.H + f;
                for (int c = 0; c < nc; ++c) {
                    float v[16];
                    tmem_ld16(tg + c * 16, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int n = c * 16 + j;
                        if (n < t.n_len) dst[(size_t)n * a.H] = __float2bfloat16_rn(v[j]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[acc]);
            ++ac;
            if (t.phase == 0 && (a.phases & 2)) {
                // publish this unit's h rows to the down tiles (other CTAs read them by TMA)
                __threadfence();
                fence_proxy_async_global();
                __syncwarp();
                if (lane == 0) mbar_arrive(pubbar);
                if (warp == 2 && lane == 0) {
                    if (mbar_wait(pubbar, pub & 1, a.st, limit)) red_release_gpu_add(done + t.unit, 1);
                }
                ++pub;
            }
        }
    }

    // ------------------------------------------------ teardown
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
    if (tid == 0) {
        __threadfence();
        s_misc[0] = (atomicAdd(exit_counter, 1) == (int)gridDim.x - 1);
    }
    __syncthreads();
    if (s_misc[0]) {   // last CTA out: reset the counters for the next launch
        __threadfence();
        for (int u = tid; u < n_units; u += kThreads) done[u] = 0;
        if (tid == 0) { *tile_counter = 0; *exit_counter = 0; }
    }
}

// Two entry points with one body, so profiles tell the routed experts (grouped,
// device-built unit list) from the dense shared expert.
template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
tc_routed_experts_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
    tc_experts_body<BN>(maps, a);
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
tc_shared_expert_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
    tc_experts_body<BN>(maps, a);
}

template <int BN>
cudaError_t launch_width(const TcMaps& maps, const TcArgs& a, int grid, cudaStream_t s) {
    static bool configured = false;   // per process; the attribute is per function
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(tc_routed_experts_kernel<BN>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             TcCfg<BN>::kSmem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(tc_shared_expert_kernel<BN>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     TcCfg<BN>::kSmem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    if (a.dense_T > 0)
        tc_shared_expert_kernel<BN><<<grid, kThreads, TcCfg<BN>::kSmem, s>>>(maps, a);
    else
        tc_routed_experts_kernel<BN><<<grid, kThreads, TcCfg<BN>::kSmem, s>>>(maps, a);
    return cudaGetLastError();
}

}  // namespace

int tc_smem_bytes(int width) {
    return width <= 32 ? TcCfg<32>::kSmem : TcCfg<256>::kSmem;
}

cudaError_t launch_tc_experts(const TcMaps& maps, const TcArgs& a, int width, int grid,
                              cudaStream_t s) {
    if (grid <= 0) return cudaSuccess;
    if (a.H % kBM || a.I % kBM) return cudaErrorInvalidValue;
    if (width == 32) return launch_width<32>(maps, a, grid, s);
    if (width == 256) return launch_width<256>(maps, a, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace moe
