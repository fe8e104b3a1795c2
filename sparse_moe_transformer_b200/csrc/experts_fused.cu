// experts_fused.cu -- routed and shared SwiGLU experts for few tokens (decode),
// one tile = one expert's tokens (or the shared expert's) x one 128-feature block
// of the intermediate dimension.
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
// The token lists come straight from the router's Top-k: every CTA counts the
// selections per expert in shared memory and finds each of its own tiles' expert
// and rows with ballots (the rows of an expert in token order, cut into units of
// at most kBN), so no permutation pass or global scan runs before this kernel.
// CTA b takes tiles b, b + G, b + 2G, ... of [shared-expert tiles | routed tiles];
// the shared tiles need no routing and, when the layer input is used as is,
// start while the router still runs (programmatic dependent launch).
//
// Warp roles: warp 0 schedules tiles and streams weights (contiguous bulk copies
// of pre-swizzled tile pairs, nothing else, so it runs ahead by the full stage
// ring); warp 1 issues tcgen05.mma; warps 2-9 gather each tile's token rows into
// a swizzled x panel (the B operand of all gate/up k-steps, loaded while the
// previous tile's down projection runs) and drain TMEM.  All waits are bounded.
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
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = 64 + kEpiThreads;
constexpr int kRing = 4;
constexpr int kPairBytes = 2 * kBM * kBK * 2;      // one packed tile pair, 32 KB
constexpr int kBN = 16;                             // rows (token slots) per unit
constexpr int kStages = 5;
constexpr int kStageBytes = kPairBytes;
constexpr int kMaxH = 1024;
constexpr int kXAtom = kBN / 8 * 1024;              // kBN rows x 64 columns, 128-byte swizzle
constexpr int kXBytes = kMaxH / kBK * kXAtom;       // x panel: every k-step of the tile
constexpr int kHAtom = kXAtom;                      // h as B operand: one 64-wide K atom
constexpr int kHBytes = 2 * kHAtom;                 // 128 features
constexpr int kMaxSlots = 1024;                     // T * k
constexpr int kMaxE = 256;
constexpr int kDownBlocks = kMaxH / kBM;            // H / 128 accumulators
constexpr int kTmemCols = 256;                      // gate, up (2 x 16) + 8 x 16 down
constexpr uint64_t kDrainLimitNs = 200ull * 1000 * 1000;
static_assert(kStageBytes % 1024 == 0 && kXBytes % 1024 == 0, "alignment");
static_assert(2 * kBN + kDownBlocks * kBN <= kTmemCols, "TMEM columns");

constexpr int kTileRouted = 0;   // an expert's slots (rows in the ring)
constexpr int kTileShared = 1;   // the shared expert: tokens start .. start + n_len - 1

struct FTile {
    int unit;        // -1: no more work
    int blk;         // 128-feature block of the intermediate dimension
    int kind;        // kTileRouted or kTileShared
    int expert;      // routed expert (other kinds: 0)
    int start;       // shared: first token (routed tiles: their slots are in the ring's rows)
    int n_len;
};


struct SmemLayout {
    static constexpr int kXOff = kStages * kStageBytes;
    static constexpr int kHOff = kXOff + kXBytes;
    static constexpr int kIdxOff = kHOff + kHBytes;                   // int[kMaxSlots] topk
    static constexpr int kCountOff = kIdxOff + kMaxSlots * 4;         // int[kMaxE] counts
    static constexpr int kUBaseOff = kCountOff + kMaxE * 4;           // int[kMaxE] unit starts
    static constexpr int kRowsOff = kUBaseOff + kMaxE * 4;            // int[kRing][kBN] tile rows
    static constexpr int kCtrlOff = kRowsOff + kRing * kBN * 4;
    static constexpr int kTotal = kCtrlOff + 1024 + 1024;             // + alignment slack
};
static_assert(SmemLayout::kTotal <= 232448, "shared memory per CTA");

// x panel of one tile: row rr (a token), k-step kb, 16-byte chunk cc at
// kb * kXAtom + rr * 128 + ((cc ^ (rr % 8)) * 16) -- the K-major 128-byte-swizzle
// image of kBN rows the tensor core reads for k-step kb.  Gathered by the
// epilogue warps with plain loads, then published to the async proxy.
__device__ __forceinline__ void gather_x_panel(uint8_t* xs, const __nv_bfloat16* __restrict__ x,
                                               const int* rows, bool by_token, int start, int n_len,
                                               int k, int H) {
    const int et = threadIdx.x - 64;                 // 0 .. kEpiThreads-1
    const int per_row = H / 8;                       // 16-byte chunks of one row
    const int n = n_len * per_row;
    constexpr int kIter = kBN * (kMaxH / 8) / kEpiThreads;
    uint4 v[kIter];
    int dst[kIter];
#pragma unroll
    for (int i = 0; i < kIter; ++i) {
        const int id = et + i * kEpiThreads;
        dst[i] = -1;
        if (id < n) {
            const int rr = id / per_row, ch = id - rr * per_row;
            const int tok = by_token ? start + rr : rows[rr] / k;
            v[i] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)tok * H) + ch);
            const int kb = ch >> 3, cc = ch & 7;
            dst[i] = kb * kXAtom + rr * 128 + ((cc ^ (rr & 7)) << 4);
        }
    }
#pragma unroll
    for (int i = 0; i < kIter; ++i)
        if (dst[i] >= 0) *reinterpret_cast<uint4*>(xs + dst[i]) = v[i];
    fence_proxy_async_smem();
}

// The expert-ordered unit list of the Top-k, in two parts (one warp each).
// Slot i = t k + j selects expert idx[i]; the rows of expert e are its slots in
// increasing order, cut into units of at most kBN rows; units are ordered by
// expert.  count_units (once per CTA) loads idx, counts the rows per expert and
// scans the unit counts into ubase; it returns the number of units (0 and an
// error record on a bad index).
__device__ int count_units(const int32_t* __restrict__ topk_idx, int S, int E, int* idx_s,
                           int* cnt_s, int* ubase_s, const DeviceStatus& st) {
    const int lane = threadIdx.x & 31;
    for (int e = lane; e < E; e += 32) cnt_s[e] = 0;
    __syncwarp();
    bool bad = false;
#pragma unroll 4
    for (int i = lane; i < S; i += 32) {
        const int e = __ldg(topk_idx + i);
        idx_s[i] = e;
        if (e >= 0 && e < E) atomicAdd(&cnt_s[e], 1);
        else bad = true;
    }
    if (__any_sync(0xffffffffu, bad)) {
        if (lane == 0) report_error(st, kErrDeviceCheck);
        return 0;
    }
    __syncwarp();
    // exclusive scan over experts of the unit counts; lane l owns [l * per, (l + 1) * per)
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    int usum = 0;
    for (int e = e0; e < e1; ++e) usum += (cnt_s[e] + kBN - 1) / kBN;
    int uinc = usum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, uinc, o);
        if (lane >= o) uinc += y;
    }
    int u = uinc - usum;
    for (int e = e0; e < e1; ++e) {
        ubase_s[e] = u;
        u += (cnt_s[e] + kBN - 1) / kBN;
    }
    __syncwarp();
    return __shfl_sync(0xffffffffu, uinc, 31);
}

// Unit u: its expert, its row count and (into rows[0 .. n_len)) its slots --
// occurrences q kBN .. q kBN + n_len - 1 of the expert in slot order, where q is
// the unit's index within its expert.  One warp; ballots only.
__device__ void locate_unit(int u, int S, int E, const int* idx_s, const int* cnt_s,
                            const int* ubase_s, int* rows, int& expert, int& n_len) {
    const int lane = threadIdx.x & 31;
    int own = -1, q = 0;
    for (int e = lane; e < E; e += 32) {
        const int ub = ubase_s[e], nu = (cnt_s[e] + kBN - 1) / kBN;
        if (u >= ub && u < ub + nu) { own = e; q = u - ub; }
    }
    const uint32_t m = __ballot_sync(0xffffffffu, own >= 0);
    const int src = __ffs(m) - 1;
    expert = __shfl_sync(0xffffffffu, own, src);
    q = __shfl_sync(0xffffffffu, q, src);
    const int first = q * kBN;
    n_len = min(kBN, cnt_s[expert] - first);
    const uint32_t lt = (1u << lane) - 1u;
    int seen = 0;
    for (int c = 0; c < S && seen < first + n_len; c += 32) {
        const int i = c + lane;
        const bool hit = i < S && idx_s[i] == expert;
        const uint32_t hm = __ballot_sync(0xffffffffu, hit);
        const int occ = seen + __popc(hm & lt);
        if (hit && occ >= first && occ < first + n_len) rows[occ - first] = i;
        seen += __popc(hm);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
tc_fused_experts_kernel(const FusedArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* hsm = smem + SmemLayout::kHOff;
    uint8_t* xsm = smem + SmemLayout::kXOff;
    int* idx_s = reinterpret_cast<int*>(smem + SmemLayout::kIdxOff);
    int* ring_rows = reinterpret_cast<int*>(smem + SmemLayout::kRowsOff);     // [kRing][kBN]
    uint8_t* ctrl = smem + SmemLayout::kCtrlOff;
    uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
    uint64_t* empty = full + kStages;
    uint64_t* accA_full = empty + kStages;
    uint64_t* accA_empty = accA_full + 1;
    uint64_t* h_ready = accA_empty + 1;
    uint64_t* accB_full = h_ready + 1;
    uint64_t* accB_empty = accB_full + 1;
    uint64_t* x_full = accB_empty + 1;
    uint64_t* tfull = x_full + 1;
    uint64_t* tempty = tfull + kRing;
    uint64_t* drainbar = tempty + kRing;
    FTile* ring = reinterpret_cast<FTile*>(drainbar + 1);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring + kRing);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H, k = a.k, T = a.T, E = a.E;
    const int S = T * k;
    const int rows_total = S + T;              // o_part rows: routed slots, then shared tokens
    const int n_blk = a.I / kBM;               // routed 128-feature blocks
    const int n_blk_s = a.Is / kBM;            // shared-expert 128-feature blocks
    const int n_st = (T + kBN - 1) / kBN * n_blk_s;   // shared tiles come first
    const int kb_gu = H / kBK;
    const int mt2 = (H / kBM + 1) / 2;         // packed down pairs (256 outputs each)
    const uint64_t limit = a.wait_limit_ns;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        mbar_init(accA_full, 1);
        mbar_init(accA_empty, kEpiWarps);
        mbar_init(h_ready, kEpiWarps);
        mbar_init(accB_full, 1);
        mbar_init(accB_empty, kEpiWarps);
        mbar_init(x_full, kEpiWarps);
        for (int s = 0; s < kRing; ++s) { mbar_init(&tfull[s], 1); mbar_init(&tempty[s], 1 + kEpiWarps); }
        mbar_init(drainbar, 1);
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    grid_dependents_launch();                  // the combine may start its own prologue

    if (warp == 0) {
        // ------------------------------------------------ scheduler + copy producer
        // Tiles b, b + G, b + 2G, ... of the list [shared tiles | routed tiles].
        // Shared tiles need no routing and start at once (weights are constants);
        // the routed unit list is counted from the router's Top-k, after the grid
        // dependency is satisfied, when the first routed tile comes up.
        const uint64_t pol_w = policy_evict_first();
        int* cnt_s = reinterpret_cast<int*>(smem + SmemLayout::kCountOff);
        int* ubase_s = reinterpret_cast<int*>(smem + SmemLayout::kUBaseOff);
        bool built = false;
        int n_units = 0;
        uint32_t it = 0;
        int tc = 0;
        bool ok = true;
        for (int i = blockIdx.x;; i += gridDim.x) {
            const int rs = tc % kRing;
            int w_ok = 1;
            if (lane == 0) w_ok = mbar_wait(&tempty[rs], ((tc / kRing) & 1) ^ 1, a.st, limit);
            if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
            FTile t{-1, 0, kTileRouted, 0, 0, 0};
            if (ok && (tc == 0 || !error_pending(a.st))) {
                if (i < n_st) {
                    const int u = i / n_blk_s;
                    t = FTile{u, i % n_blk_s, kTileShared, 0, u * kBN, min(kBN, T - u * kBN)};
                } else {
                    if (!built) {
                        grid_dependency_wait();
                        n_units = count_units(a.topk_idx, S, E, idx_s, cnt_s, ubase_s, a.st);
                        built = true;
                    }
                    const int r = i - n_st;
                    if (r < n_units * n_blk) {
                        int e, n_len;
                        locate_unit(r / n_blk, S, E, idx_s, cnt_s, ubase_s, ring_rows + rs * kBN,
                                    e, n_len);
                        t = FTile{r / n_blk, r % n_blk, kTileRouted, e, 0, n_len};
                    }
                }
            }
            __syncwarp();
            if (lane == 0) { ring[rs] = t; mbar_arrive(&tfull[rs]); }
            ++tc;
            if (t.unit < 0) break;
            int fail = 0;
            const bool sh = t.kind == kTileShared;
            const uint8_t* w_gu = static_cast<const uint8_t*>(sh ? a.ws_gu : a.w_gu);
            const uint8_t* w_dn = static_cast<const uint8_t*>(sh ? a.ws_down : a.w_down);
            const int nb = sh ? n_blk_s : n_blk;
            const int kb_dn = 2 * nb;                        // 64-wide k-blocks of the down input
            const uint8_t* gu_src = w_gu + (size_t)(t.expert * nb + t.blk) * kb_gu * kPairBytes;
            // gate/up k-steps: one bulk copy of the packed (gate, up) tile pair each
            for (int kb = 0; kb < kb_gu; ++kb, ++it) {
                const int s = it % kStages;
                if (lane == 0) {
                    if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, a.st, limit)) fail = 1;
                    else {
                        mbar_arrive_expect_tx(&full[s], kPairBytes);
                        bulk_load(smem + s * kStageBytes, gu_src + (size_t)kb * kPairBytes,
                                  kPairBytes, &full[s], pol_w);
                    }
                }
                if (__shfl_sync(0xffffffffu, fail, 0)) break;
            }
            if (__shfl_sync(0xffffffffu, fail, 0)) { ok = false; break; }
            // down k-steps: the two k-blocks of this feature block for every output pair
            for (int q = 0; q < mt2 * 2; ++q, ++it) {
                const int s = it % kStages;
                const int pair = q >> 1, kbl = q & 1;
                if (lane == 0) {
                    if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, a.st, limit)) fail = 1;
                    else {
                        mbar_arrive_expect_tx(&full[s], kPairBytes);
                        const size_t tile = ((size_t)t.expert * mt2 + pair) * kb_dn + 2 * t.blk + kbl;
                        bulk_load(smem + s * kStageBytes, w_dn + tile * kPairBytes, kPairBytes,
                                  &full[s], pol_w);
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
        int tc = 0, nA = 0, nB = 0;     // uses of accumulator A (every tile), B (expert tiles)
        bool stuck_pending = a.inject_stuck != 0;
        const uint32_t dA = tmem_base;               // gate: cols [0, 16), up: [16, 32)
        const uint32_t dB = tmem_base + 2 * kBN;     // down block r: cols [32 + 16 r, ...)
        const uint32_t idesc = idesc_bf16_f32(kBM, kBN);
        const uint32_t xs = smem_u32(xsm);
        while (true) {
            const int r = tc % kRing;
            if (!mbar_wait(&tfull[r], (tc / kRing) & 1, a.st, limit)) break;
            const FTile t = ring[r];
            mbar_arrive(&tempty[r]);
            ++tc;
            if (t.unit < 0) break;
            if (stuck_pending) {       // test hook: a word nobody sets, so the wait runs out
                stuck_pending = false;
                const uint64_t t0 = globaltimer_ns();
                while (ld_acquire_gpu(a.zero_word) < 1 && globaltimer_ns() - t0 <= limit) __nanosleep(64);
                if (ld_acquire_gpu(a.zero_word) < 1) report_error(a.st, kErrTimeout);
            }
            bool fail = !mbar_wait(accA_empty, (nA & 1) ^ 1, a.st, limit) ||
                        !mbar_wait(x_full, nA & 1, a.st, limit);
            tc_fence_after();
            for (int kb = 0; kb < kb_gu && !fail; ++kb, ++it) {
                const int s = it % kStages;
                if (!mbar_wait(&full[s], (it / kStages) & 1, a.st, limit)) { fail = true; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + s * kStageBytes);
                const uint32_t b0 = xs + kb * kXAtom;
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
            ++nA;
            // h (written by the epilogue into shared memory) feeds the down MMAs
            if (!mbar_wait(h_ready, nB & 1, a.st, limit)) break;
            if (!mbar_wait(accB_empty, (nB & 1) ^ 1, a.st, limit)) break;
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
            ++nB;
        }
        tc_commit(drainbar);
        mbar_wait(drainbar, 0, a.st, kDrainLimitNs);
    } else if (warp >= 2) {
        // ------------------------------------------------ x panels + epilogue
        const int ew = warp - 2, q = warp & 3, half = ew >> 2;
        const __nv_bfloat16* x_rows = static_cast<const __nv_bfloat16*>(a.x_rows);
        if (!a.x_early) grid_dependency_wait();      // x_rows is the router's output
        int tc = 0, nA = 0, nB = 0;
        // Take the next ring entry: the tile, this lane's o_part row, and (while the
        // entry is still held) the gathered x panel; then release the entry.
        auto next_tile = [&](FTile& t, int& my_row) -> bool {
            const int r = tc % kRing;
            if (!mbar_wait(&tfull[r], (tc / kRing) & 1, a.st, limit)) return false;
            t = ring[r];
            const int* rows = ring_rows + r * kBN;
            const bool by_token = t.kind != kTileRouted;
            my_row = 0;
            if (t.unit >= 0 && lane < t.n_len) my_row = by_token ? S + t.start + lane : rows[lane];
            if (t.unit >= 0) {
                gather_x_panel(xsm, x_rows, rows, by_token, t.start, t.n_len, k, H);
                __syncwarp();
                if (lane == 0) mbar_arrive(x_full);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[r]);
            ++tc;
            return true;
        };
        FTile t;
        int my_row = 0;
        if (!next_tile(t, my_row)) t.unit = -1;
        while (t.unit >= 0) {
            const uint32_t lanes = static_cast<uint32_t>(q * 32) << 16;
            if (!mbar_wait(accA_full, nA & 1, a.st, limit)) break;
            tc_fence_after();
            ++nA;
            // h = SiLU(gate) * up for features 32 q + lane of this block -> shared memory,
            // laid out as the K-major B operand (token rows, 128-byte swizzle)
            const int f = q * 32 + lane;                   // feature within the block
            if (half == 0) {
                const int atom = f >> 6, c16 = (f & 63) >> 3, e8 = f & 7;
                float g[16], u[16];
                tmem_ld16(tmem_base + lanes, g);
                tmem_ld16(tmem_base + kBN + lanes, u);
                tmem_wait_ld();
#pragma unroll
                for (int n = 0; n < 16; ++n) {
                    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(
                        hsm + atom * kHAtom + (n >> 3) * 1024 + (n & 7) * 128 +
                        ((c16 ^ (n & 7)) << 4)) + e8;
                    *dst = __float2bfloat16_rn(silu_fast(g[n]) * u[n]);
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) { mbar_arrive(accA_empty); mbar_arrive(h_ready); }
            // the gate/up MMAs are done with the x panel: gather the next tile's rows
            // while this tile's down projection runs
            FTile tn;
            int my_row_n = 0;
            if (!next_tile(tn, my_row_n)) break;
            // down partials: o_part[blk][row][128 rb + 32 q + lane], fp32
            if (!mbar_wait(accB_full, nB & 1, a.st, limit)) break;
            tc_fence_after();
            float* ob = a.o_part + (size_t)t.blk * rows_total * H;
            const int n_rb = min(kDownBlocks / 2, (H / kBM - half + 1) / 2);   // this half's blocks
            {
                // every TMEM load of this half in flight before the one wait
                float v[kDownBlocks / 2][16];
#pragma unroll
                for (int i = 0; i < kDownBlocks / 2; ++i)
                    if (i < n_rb) tmem_ld16(tmem_base + 2 * kBN + (half + 2 * i) * kBN + lanes, v[i]);
                tmem_wait_ld();
#pragma unroll
                for (int n = 0; n < 16; ++n) {
                    const int row = __shfl_sync(0xffffffffu, my_row, n);
                    if (n < t.n_len) {
                        float* dst = ob + (size_t)row * H + half * kBM + f;
#pragma unroll
                        for (int i = 0; i < kDownBlocks / 2; ++i)
                            if (i < n_rb) dst[2 * i * kBM] = v[i][n];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(accB_empty);
            ++nB;
            t = tn;
            my_row = my_row_n;
        }
    }

    // ------------------------------------------------ teardown
    // The MMA role runs on lane 0 of warp 1 only: reconverge every warp before
    // the CTA barrier (bar.sync expects whole warps).
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace

int fused_smem_bytes() { return SmemLayout::kTotal; }
int fused_unit_rows() { return kBN; }

bool fused_supported(int H, int I, int Is, int E, int k, int S) {
    return H % 256 == 0 && H <= kMaxH && I % 128 == 0 && Is % 128 == 0 &&
           E <= kMaxE && k >= 1 && k <= 8 && I / 128 + (Is / 128 + 7) / 8 <= 16 &&
           S <= kMaxSlots;
}

cudaError_t launch_fused_experts(const FusedArgs& a, int grid, int pdl, cudaStream_t s) {
    if (grid <= 0) return cudaSuccess;
    if (!fused_supported(a.H, a.I, a.Is, a.E, a.k, a.T * a.k)) return cudaErrorInvalidValue;
    static std::once_flag configured[16];    // the attribute is set per device
    cudaError_t e = once_per_device(configured, [] {
        return cudaFuncSetAttribute(tc_fused_experts_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    SmemLayout::kTotal);
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SmemLayout::kTotal;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, tc_fused_experts_kernel, a);
}

}  // namespace moe
