// experts_fused.cu -- routed SwiGLU experts for few tokens (decode), one tile =
// one expert's tokens x one 128-feature block of the intermediate dimension.
//
// Each expert is down(SiLU(gate x) * up x) (page "print(model) Qwen3-TTS",
// SwiGLU section).  Splitting the intermediate dimension I into 128-feature
// blocks b, the down projection is a sum over blocks:
//     o = sum_b W_down[:, b] h_b,   h_b = SiLU(W_gate[b] x) * (W_up[b] x),
// so a tile computes h_b on the tensor cores, keeps it on chip (TMEM ->
// registers -> shared memory, where it becomes the B operand of the next MMA)
// and then multiplies it by the matching 128-column slice of W_down for all H
// outputs.  Tiles never wait for one another; each writes an fp32 partial
// o_part[b][slot][H] and the combine sums the blocks in fixed order.
//
// The token lists come straight from the router's Top-k: every CTA builds the
// same expert-ordered unit list from topk_idx in shared memory (tokens of one
// expert in token order, split into runs of at most BN), so no permutation pass
// or global scan runs before this kernel.
//
// Warp roles as in experts_tc.cu: warp 0 schedules and copies (weights by
// contiguous bulk copies of pre-swizzled tile pairs; token rows gathered from x
// by the whole warp and stored with the 128-byte swizzle), warp 1 issues
// tcgen05.mma, warps 2-9 drain TMEM.  All waits are bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "device.cuh"
#include "layer.h"

namespace moe {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kRing = 4;
constexpr int kPairBytes = 2 * kBM * kBK * 2;      // one packed tile pair, 32 KB
constexpr int kBN = 32;                             // rows (token slots) per unit
constexpr int kStages = 5;
constexpr int kBBytes = kBN * kBK * 2;              // gathered rows of one k-step
constexpr int kStageBytes = kPairBytes + kBBytes;
constexpr int kHAtom = kBN / 8 * 1024;              // h as B operand: one 64-wide K atom
constexpr int kHBytes = 2 * kHAtom;                 // 128 features
constexpr int kMaxSlots = 1024;                     // T * k
constexpr int kMaxE = 256;
constexpr int kMaxUnits = 384;
constexpr int kDownBlocks = 8;                      // H / 128 accumulators (H <= 1024)
constexpr int kTmemCols = 512;                      // gate, up (2 x 32) + 8 x 32 down
constexpr uint64_t kDrainLimitNs = 200ull * 1000 * 1000;
static_assert(kStageBytes % 1024 == 0, "stage alignment");

struct FTile {
    int unit;        // -1: no more work
    int blk;         // 128-feature block of the intermediate dimension
    int expert;
    int start;       // first row in the unit row list
    int n_len;
};

struct FUnit {
    int expert, start, n_len;
};

struct SmemLayout {
    static constexpr int kStagesOff = 0;
    static constexpr int kHOff = kStages * kStageBytes;
    static constexpr int kSlotsOff = kHOff + kHBytes;                 // int[kMaxSlots] rows
    static constexpr int kIdxOff = kSlotsOff + kMaxSlots * 4;         // int[kMaxSlots] topk
    static constexpr int kCountOff = kIdxOff + kMaxSlots * 4;         // int[kMaxE] counts
    static constexpr int kStartOff = kCountOff + kMaxE * 4;           // int[kMaxE] starts
    static constexpr int kUBaseOff = kStartOff + kMaxE * 4;           // int[kMaxE + 1]
    static constexpr int kUnitsOff = kUBaseOff + (kMaxE + 4) * 4;     // FUnit[kMaxUnits]
    static constexpr int kCtrlOff = kUnitsOff + kMaxUnits * (int)sizeof(FUnit);
    static constexpr int kTotal = kCtrlOff + 1024 + 1024;             // + alignment slack
};
static_assert(SmemLayout::kTotal <= 232448, "shared memory per CTA");

__device__ __forceinline__ int scan_tmp_sum(int* v, int n, int* tmp) {
    // exclusive scan of v[0..n) by all kThreads threads; returns the total
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kW = kThreads / 32;
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
        for (int w = 0; w < kW; ++w) { const int t = tmp[w]; tmp[w] = run; run += t; }
        tmp[kW] = run;
    }
    __syncthreads();
    int run = tmp[warp] + incl - s;
    for (int i = b0; i < b1; ++i) { const int t = v[i]; v[i] = run; run += t; }
    const int total = tmp[kW];
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(kThreads, 1)
tc_fused_experts_kernel(const FusedArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* hsm = smem + SmemLayout::kHOff;
    int* rows_s = reinterpret_cast<int*>(smem + SmemLayout::kSlotsOff);
    int* idx_s = reinterpret_cast<int*>(smem + SmemLayout::kIdxOff);
    int* cnt_s = reinterpret_cast<int*>(smem + SmemLayout::kCountOff);
    int* start_s = reinterpret_cast<int*>(smem + SmemLayout::kStartOff);
    int* ubase_s = reinterpret_cast<int*>(smem + SmemLayout::kUBaseOff);
    FUnit* units_s = reinterpret_cast<FUnit*>(smem + SmemLayout::kUnitsOff);
    uint8_t* ctrl = smem + SmemLayout::kCtrlOff;
    uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
    uint64_t* empty = full + kStages;
    uint64_t* accA_full = empty + kStages;
    uint64_t* accA_empty = accA_full + 1;
    uint64_t* h_ready = accA_empty + 1;
    uint64_t* accB_full = h_ready + 1;
    uint64_t* accB_empty = accB_full + 1;
    uint64_t* tfull = accB_empty + 1;
    uint64_t* tempty = tfull + kRing;
    uint64_t* drainbar = tempty + kRing;
    FTile* ring = reinterpret_cast<FTile*>(drainbar + 1);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring + kRing);
    int* s_misc = reinterpret_cast<int*>(tmem_slot + 1);          // [0] last CTA, [1] n_units
    int* scan_tmp = s_misc + 4;                                    // kThreads / 32 + 1

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H, I = a.I, E = a.E, k = a.k, T = a.T;
    const int S = T * k;
    const int n_blk = I / kBM;                 // 128-feature blocks (gate/up tiles per unit)
    const int kb_gu = H / kBK;
    const int mt2 = (H / kBM + 1) / 2;         // packed down pairs (256 outputs each)
    const int kb_dn = I / kBK;
    int* tile_counter = a.sync;
    int* exit_counter = a.sync + 1;
    const uint64_t limit = a.wait_limit_ns;

    // ---- barriers and TMEM (thread 0 / warp 1) while the unit list is built
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 2); mbar_init(&empty[s], 1); }
        mbar_init(accA_full, 1);
        mbar_init(accA_empty, kEpiWarps);
        mbar_init(h_ready, kEpiWarps);
        mbar_init(accB_full, 1);
        mbar_init(accB_empty, kEpiWarps);
        for (int s = 0; s < kRing; ++s) { mbar_init(&tfull[s], 1); mbar_init(&tempty[s], 1 + kEpiWarps); }
        mbar_init(drainbar, 1);
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);

    // ---- expert-ordered unit list from the Top-k (identical in every CTA)
    for (int i = tid; i < S; i += kThreads) idx_s[i] = a.topk_idx[i];
    for (int e = tid; e < E; e += kThreads) cnt_s[e] = 0;
    __syncthreads();
    for (int i = tid; i < S; i += kThreads) {
        const int e = idx_s[i];
        if (e >= 0 && e < E) atomicAdd(&cnt_s[e], 1);
        else report_error(a.st, kErrDeviceCheck);
    }
    __syncthreads();
    for (int e = tid; e < E; e += kThreads) {
        start_s[e] = cnt_s[e];
        ubase_s[e] = (cnt_s[e] + kBN - 1) / kBN;
    }
    __syncthreads();
    scan_tmp_sum(start_s, E, scan_tmp);
    int n_units = scan_tmp_sum(ubase_s, E, scan_tmp);
    n_units = min(n_units, kMaxUnits);
    for (int i = tid; i < S; i += kThreads) {        // stable: rank among earlier slots
        const int e = idx_s[i];
        if (e < 0 || e >= E) continue;
        int rank = 0;
        for (int j = 0; j < i; ++j) rank += idx_s[j] == e;
        rows_s[start_s[e] + rank] = i;               // slot id t * k + j
    }
    for (int e = tid; e < E; e += kThreads) {
        const int c = cnt_s[e];
        for (int u = 0; u * kBN < c; ++u) {
            const int id = ubase_s[e] + u;
            if (id < kMaxUnits) units_s[id] = FUnit{e, start_s[e] + u * kBN, min(kBN, c - u * kBN)};
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int n_tiles = n_units * n_blk;

    if (warp == 0) {
        // ------------------------------------------------ scheduler + copy producer
        const uint64_t pol_w = policy_evict_first();
        const uint8_t* w_gu = static_cast<const uint8_t*>(a.w_gu);
        const uint8_t* w_dn = static_cast<const uint8_t*>(a.w_down);
        const __nv_bfloat16* x_rows = static_cast<const __nv_bfloat16*>(a.x_rows);
        uint32_t it = 0;
        int tc = 0;
        bool ok = true;
        while (true) {
            int i = n_tiles;
            if (lane == 0 && ok && !error_pending(a.st)) i = atomicAdd(tile_counter, 1);
            i = __shfl_sync(0xffffffffu, i, 0);
            FTile t{-1, 0, 0, 0, 0};
            if (i < n_tiles) {
                const FUnit u = units_s[i / n_blk];
                t = FTile{i / n_blk, i % n_blk, u.expert, u.start, u.n_len};
            }
            const int r = tc % kRing;
            int w_ok = 1;
            if (lane == 0) {
                w_ok = mbar_wait(&tempty[r], ((tc / kRing) & 1) ^ 1, a.st, limit);
                if (w_ok) { ring[r] = t; mbar_arrive(&tfull[r]); }
            }
            if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
            ++tc;
            if (t.unit < 0) break;
            // lane covers (row, 16-byte chunk) pairs p = lane + 32 j of the unit's rows
            const int my_slot = lane < t.n_len ? rows_s[t.start + lane] : 0;
            const __nv_bfloat16* src_row[8];
            uint4 nx[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int p = lane + 32 * j, rr = p >> 3, cc = p & 7;
                const int slot = __shfl_sync(0xffffffffu, my_slot, rr);
                src_row[j] = rr < t.n_len ? x_rows + (size_t)(slot / k) * H + cc * 8 : nullptr;
                if (src_row[j]) nx[j] = *reinterpret_cast<const uint4*>(src_row[j]);
            }
            const uint8_t* gu_src = w_gu + (size_t)(t.expert * n_blk + t.blk) * kb_gu * kPairBytes;
            int fail = 0;
            // gate/up k-steps: weights by bulk copy, token rows gathered from x
            for (int kb = 0; kb < kb_gu; ++kb, ++it) {
                const int s = it % kStages;
                uint8_t* A0 = smem + s * kStageBytes;
                uint8_t* B = A0 + kPairBytes;
                if (lane == 0) {
                    if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, a.st, limit)) fail = 1;
                    else {
                        mbar_arrive_expect_tx(&full[s], kPairBytes);
                        bulk_load(A0, gu_src + (size_t)kb * kPairBytes, kPairBytes, &full[s], pol_w);
                    }
                }
                if (__shfl_sync(0xffffffffu, fail, 0)) break;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int p = lane + 32 * j, rr = p >> 3, cc = p & 7;
                    if (src_row[j])
                        *reinterpret_cast<uint4*>(B + rr * 128 + ((cc ^ (rr & 7)) << 4)) = nx[j];
                }
                if (kb + 1 < kb_gu) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (src_row[j]) nx[j] = *reinterpret_cast<const uint4*>(src_row[j] + (kb + 1) * kBK);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[s]);
            }
            if (__shfl_sync(0xffffffffu, fail, 0)) { ok = false; break; }
            // down k-steps: the two k-blocks of this feature block for every output pair
            for (int q = 0; q < mt2 * 2; ++q, ++it) {
                const int s = it % kStages;
                const int pair = q >> 1, kbl = q & 1;
                uint8_t* A0 = smem + s * kStageBytes;
                if (lane == 0) {
                    if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, a.st, limit)) fail = 1;
                    else {
                        mbar_arrive_expect_tx(&full[s], kPairBytes);
                        const size_t tile = ((size_t)t.expert * mt2 + pair) * kb_dn + 2 * t.blk + kbl;
                        bulk_load(A0, w_dn + tile * kPairBytes, kPairBytes, &full[s], pol_w);
                        mbar_arrive(&full[s]);
                    }
                }
                if (__shfl_sync(0xffffffffu, fail, 0)) break;
            }
            if (__shfl_sync(0xffffffffu, fail, 0)) { ok = false; break; }
        }
        if (lane == 0)
            for (uint32_t q = (it > (uint32_t)kStages ? it - kStages : 0); q < it; ++q)
                mbar_wait(&full[q % kStages], (q / kStages) & 1, a.st, kDrainLimitNs);
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        uint32_t it = 0;
        int tc = 0, na = 0;
        bool stuck_pending = a.inject_stuck != 0;
        const uint32_t dA = tmem_base;               // gate: cols [0, 32), up: [32, 64)
        const uint32_t dB = tmem_base + 2 * kBN;     // down block r: cols [64 + 32 r, ...)
        while (true) {
            const int r = tc % kRing;
            if (!mbar_wait(&tfull[r], (tc / kRing) & 1, a.st, limit)) break;
            const FTile t = ring[r];
            mbar_arrive(&tempty[r]);
            ++tc;
            if (t.unit < 0) break;
            if (stuck_pending) {       // test hook: a count nobody raises, so the wait runs out
                stuck_pending = false;
                const int* never = a.sync + 2;
                const uint64_t t0 = globaltimer_ns();
                while (ld_acquire_gpu(never) < 1 && globaltimer_ns() - t0 <= limit) __nanosleep(64);
                if (ld_acquire_gpu(never) < 1) report_error(a.st, kErrTimeout);
            }
            const int N = ((t.n_len + 15) / 16) * 16;
            const uint32_t idesc = idesc_bf16_f32(kBM, N);
            bool fail = !mbar_wait(accA_empty, (na & 1) ^ 1, a.st, limit);
            tc_fence_after();
            for (int kb = 0; kb < kb_gu && !fail; ++kb, ++it) {
                const int s = it % kStages;
                if (!mbar_wait(&full[s], (it / kStages) & 1, a.st, limit)) { fail = true; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + s * kStageBytes);
                const uint32_t b0 = a0 + kPairBytes;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    const uint64_t bd = smem_desc_sw128(b0 + kk * 32);
                    const uint32_t acc = (kb | kk) != 0;
                    tc_mma_bf16(dA, smem_desc_sw128(a0 + kk * 32), bd, idesc, acc);
                    tc_mma_bf16(dA + kBN, smem_desc_sw128(a0 + kPairBytes / 2 + kk * 32), bd, idesc, acc);
                }
                tc_commit(&empty[s]);
            }
            if (fail) break;
            tc_commit(accA_full);
            // h (written by the epilogue into shared memory) feeds the down MMAs
            if (!mbar_wait(h_ready, na & 1, a.st, limit)) break;
            if (!mbar_wait(accB_empty, (na & 1) ^ 1, a.st, limit)) break;
            tc_fence_after();
            const uint32_t hs = smem_u32(hsm);
            for (int q = 0; q < mt2 * 2; ++q, ++it) {
                const int s = it % kStages;
                const int pair = q >> 1, kbl = q & 1;
                if (!mbar_wait(&full[s], (it / kStages) & 1, a.st, limit)) { fail = true; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + s * kStageBytes);
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    const uint64_t bd = smem_desc_sw128(hs + kbl * kHAtom + kk * 32);
                    const uint32_t acc = (kbl | kk) != 0;
                    tc_mma_bf16(dB + (2 * pair) * kBN, smem_desc_sw128(a0 + kk * 32), bd, idesc, acc);
                    tc_mma_bf16(dB + (2 * pair + 1) * kBN,
                                smem_desc_sw128(a0 + kPairBytes / 2 + kk * 32), bd, idesc, acc);
                }
                tc_commit(&empty[s]);
            }
            if (fail) break;
            tc_commit(accB_full);
            ++na;
        }
        tc_commit(drainbar);
        mbar_wait(drainbar, 0, a.st, kDrainLimitNs);
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue
        const int ew = warp - 2, q = warp & 3, half = ew >> 2;
        int tc = 0, na = 0;
        float* opart = a.o_part;
        while (true) {
            const int r = tc % kRing;
            if (!mbar_wait(&tfull[r], (tc / kRing) & 1, a.st, limit)) break;
            const FTile t = ring[r];
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[r]);
            ++tc;
            if (t.unit < 0) break;
            const int nc = (t.n_len + 15) / 16;
            const uint32_t lanes = static_cast<uint32_t>(q * 32) << 16;
            // h = SiLU(gate) * up for features 32 q + lane of this block -> shared memory,
            // laid out as the K-major B operand (token rows, 128-byte swizzle)
            if (!mbar_wait(accA_full, na & 1, a.st, limit)) break;
            tc_fence_after();
            const int f = q * 32 + lane;                   // feature within the block
            const int atom = f >> 6, c16 = (f & 63) >> 3, e8 = f & 7;
            for (int c = half; c < nc; c += 2) {
                float g[16], u[16];
                tmem_ld16(tmem_base + lanes + c * 16, g);
                tmem_ld16(tmem_base + kBN + lanes + c * 16, u);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int n = c * 16 + j;
                    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(
                        hsm + atom * kHAtom + (n >> 3) * 1024 + (n & 7) * 128 +
                        ((c16 ^ (n & 7)) << 4)) + e8;
                    *dst = __float2bfloat16_rn(silu_fast(g[j]) * u[j]);
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) { mbar_arrive(accA_empty); mbar_arrive(h_ready); }
            // down partials: o_part[blk][slot][128 rb + 32 q + lane], fp32
            if (!mbar_wait(accB_full, na & 1, a.st, limit)) break;
            tc_fence_after();
            float* ob = opart + (size_t)t.blk * S * H;
            for (int rb = half; rb < kDownBlocks; rb += 2) {
                const int col = rb * kBM + f;
                if (rb * kBM >= H) break;
                for (int c = 0; c < nc; ++c) {
                    float v[16];
                    tmem_ld16(tmem_base + 2 * kBN + rb * kBN + lanes + c * 16, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int n = c * 16 + j;
                        if (n < t.n_len) ob[(size_t)rows_s[t.start + n] * H + col] = v[j];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(accB_empty);
            ++na;
        }
    }

    // ------------------------------------------------ teardown
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
    if (tid == 0) {
        __threadfence();
        s_misc[0] = (atomicAdd(exit_counter, 1) == (int)gridDim.x - 1);
    }
    __syncthreads();
    if (s_misc[0] && tid == 0) {    // last CTA out: reset the counters for the next launch
        __threadfence();
        *tile_counter = 0;
        *exit_counter = 0;
    }
}

}  // namespace

int fused_smem_bytes() { return SmemLayout::kTotal; }

bool fused_supported(int H, int I, int E, int S) {
    return H % 256 == 0 && H <= kDownBlocks * kBM && I % 128 == 0 && E <= kMaxE &&
           S <= kMaxSlots;
}

cudaError_t launch_fused_experts(const FusedArgs& a, int grid, cudaStream_t s) {
    if (grid <= 0) return cudaSuccess;
    if (!fused_supported(a.H, a.I, a.E, a.T * a.k)) return cudaErrorInvalidValue;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(tc_fused_experts_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             SmemLayout::kTotal);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    tc_fused_experts_kernel<<<grid, kThreads, SmemLayout::kTotal, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
