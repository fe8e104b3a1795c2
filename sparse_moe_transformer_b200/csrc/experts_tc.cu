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
//   down tile:    D_0, D_1 = Wd[e][two 128-row blocks] . Hrows^T (256 outputs),
//                 the same two-panel shape, so both phases move 32 KB of weights
//                 per k-step.
// Weights are pre-packed as the exact 128-byte-swizzled tile images the MMA
// reads, so each k-step's weights arrive by one contiguous bulk copy; token rows
// come by TMA (128-byte swizzle, no multicast).  Stages form a shared-memory
// ring; one thread issues tcgen05.mma into TMEM accumulators; eight epilogue
// warps read TMEM with tcgen05.ld and store bf16 rows with 16-byte stores.
//
// The kernel is persistent: CTAs take tiles from a global counter, gate/up tiles
// first, then down tiles.  A launch may carry a second, dense problem -- the
// shared expert over every token -- whose tiles interleave as [routed gate/up |
// shared gate/up | routed down | shared down].  When both phases run in one
// launch, a down tile of a unit waits (bounded by a time limit) until the unit's
// gate/up tiles have published their h rows; every gate/up tile is taken before
// any down tile and never waits, so the wait always ends.  (Ordering tiles in
// waves of units -- each wave's gate/up then down tiles -- was measured slower:
// down tiles then hold SMs idle while their wave's gate/up tiles still stream.)
// Every wait in the kernel is bounded; a wait that runs out records
// MOE_ERR_TIMEOUT and the CTA drains and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "device.cuh"
#include "layer.h"

namespace moe {
namespace {

constexpr int kBM = 128;           // weight rows per tile (MMA M)
constexpr int kBK = 64;            // K elements per stage: one 128-byte swizzle atom
constexpr int kEpiWarps = 8;       // two warps per TMEM lane quarter, alternating columns
constexpr int kThreads = 64 + 32 * kEpiWarps;   // warp 0 producer, warp 1 MMA, epilogue
constexpr int kRing = 4;           // tile-info ring depth
constexpr int kABytes = kBM * kBK * 2;          // one packed weight tile
constexpr int kBoxRows = 16;       // activation rows per TMA box
constexpr int kBoxBytes = kBoxRows * kBK * 2;
constexpr int kEpiStage = 16 * 32 * 2;          // per-warp transpose buffer: 16 rows x 32 cols
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
    static constexpr int kSmem =
        kStages * kStageBytes + kEpiWarps * kEpiStage + kCtrlBytes + 1024;   // + align slack
    static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
    static_assert(kTmemCols <= 512, "TMEM has 512 columns");
    static_assert(kSmem <= 232448, "shared memory per CTA");
};

struct Tile {
    int phase;       // 0 gate/up, 1 down, 2 router logits, -1 no more work
    int prob;        // 0: the launch's first problem, 1: the second (dense) problem
    int unit;
    int mt;          // 128-row block of the weight matrix
    int expert;
    int row_start;   // first activation row
    int n_len;       // activation rows (MMA N before rounding to 16)
};

// Tile list: [problem 0 gate/up | problem 1 gate/up | problem 0 down | problem 1 down]
// (router launches: one two-panel tile of 256 experts per unit).  Every gate/up
// tile comes before every down tile, so a down tile's wait for its unit's h always
// ends.  n0 / n1: units of the two problems; mt_gu0 / mt_gu1 their gate/up blocks.
__device__ __forceinline__ Tile decode_tile(int i, int n0, int n1, const TcArgs& a, int mt_gu0,
                                            int mt_gu1, int mt_dn, int bn) {
    Tile t;
    t.prob = 0;
    if (a.phases == 4) {
        if (i < n0 * mt_dn) {
            t.phase = 2; t.unit = i / mt_dn; t.mt = i - t.unit * mt_dn;
            t.expert = 0; t.row_start = t.unit * bn; t.n_len = min(bn, a.dense_T - t.row_start);
        } else {
            t.phase = -1; t.unit = t.mt = t.expert = t.row_start = t.n_len = 0;
        }
        return t;
    }
    const int g0 = (a.phases & 1) ? n0 * mt_gu0 : 0, g1 = (a.phases & 1) ? n1 * mt_gu1 : 0;
    const int d0 = (a.phases & 2) ? n0 * mt_dn : 0, d1 = (a.phases & 2) ? n1 * mt_dn : 0;
    if (i < g0) {
        t.phase = 0; t.unit = i / mt_gu0; t.mt = i - t.unit * mt_gu0;
    } else if ((i -= g0) < g1) {
        t.phase = 0; t.prob = 1; t.unit = i / mt_gu1; t.mt = i - t.unit * mt_gu1;
    } else if ((i -= g1) < d0) {
        t.phase = 1; t.unit = i / mt_dn; t.mt = i - t.unit * mt_dn;
    } else if ((i -= d0) < d1) {
        t.phase = 1; t.prob = 1; t.unit = i / mt_dn; t.mt = i - t.unit * mt_dn;
    } else {
        t.phase = -1; t.unit = t.mt = t.expert = t.row_start = t.n_len = 0;
        return t;
    }
    const int dense = t.prob ? a.dense2_T : a.dense_T;
    if (dense > 0) {
        t.expert = 0;
        t.row_start = t.unit * bn;
        t.n_len = min(bn, dense - t.row_start);
    } else {
        const Unit u = a.units[t.unit];
        t.expert = u.expert; t.row_start = u.row_start; t.n_len = u.n_len;
    }
    return t;
}

// Down and router tiles cover two 128-row blocks; with an odd number of blocks the
// last tile's second block is the packed layout's zero fill and is neither loaded
// nor multiplied.
__device__ __forceinline__ bool single_panel(const Tile& t, const TcArgs& a) {
    const int rows = t.phase == 1 ? a.H : t.phase == 2 ? a.I : 0;
    return rows && (2 * t.mt + 1) * kBM >= rows;
}

// Wait (bounded) until `flag` reaches `target`; false after recording a timeout.
__device__ __forceinline__ bool wait_count(const int* flag, int target, const TcArgs& a) {
    if (ld_acquire_gpu(flag) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(flag) < target) {
        __nanosleep(64);
        if (globaltimer_ns() - t0 > a.wait_limit_ns) {
            report_error(a.st, kErrTimeout);
            return false;
        }
    }
    return true;
}

template <int BN>
__device__ __forceinline__ void tc_experts_body(const TcMaps& maps, const TcArgs& a) {
    using C = TcCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* epi_smem = smem + C::kStages * C::kStageBytes;
    uint8_t* ctrl = epi_smem + kEpiWarps * kEpiStage;
    uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
    uint64_t* empty = full + C::kStages;
    uint64_t* accfull = empty + C::kStages;
    uint64_t* accempty = accfull + C::kAcc;
    uint64_t* tfull = accempty + C::kAcc;
    uint64_t* tempty = tfull + kRing;
    uint64_t* pubbar = tempty + kRing;      // epilogue warps finished a gate/up tile
    uint64_t* drainbar = pubbar + 1;        // all MMAs of this CTA completed
    Tile* ring = reinterpret_cast<Tile*>(drainbar + 1);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring + kRing);
    int* s_misc = reinterpret_cast<int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool router = a.phases == 4;
    const int mt_gu0 = a.I / kBM;                     // gate/up tiles: 128 features each
    const int mt_gu1 = a.dense2_T > 0 ? a.I2 / kBM : 1;
    // down tiles: 256 output features each; router tiles: 256 experts each
    const int mt_dn = router ? (a.I / kBM + 1) / 2 : (a.H / kBM + 1) / 2;
    const int kb_gu = a.H / kBK;
    const int kb_dn0 = router ? a.H / kBK : a.I / kBK, kb_dn1 = a.I2 / kBK;
    int* tile_counter = a.sync;
    int* exit_counter = a.sync + 1;
    const uint64_t limit = a.wait_limit_ns;
    const bool fused = (a.phases & 3) == 3;

    const int n_units = a.dense_T > 0 ? (a.dense_T + BN - 1) / BN : *a.n_units;
    const int n_units2 = a.dense2_T > 0 ? (a.dense2_T + BN - 1) / BN : 0;
    const int n_tiles = router ? n_units * mt_dn
                               : ((a.phases & 1) ? n_units * mt_gu0 + n_units2 * mt_gu1 : 0) +
                                 ((a.phases & 2) ? (n_units + n_units2) * mt_dn : 0);

    if (tid == 0) {
        for (int s = 0; s < C::kStages; ++s) { mbar_init(&full[s], 2); mbar_init(&empty[s], 1); }
        for (int s = 0; s < C::kAcc; ++s) {
            mbar_init(&accfull[s], 1);
            mbar_init(&accempty[s], kEpiWarps);
        }
        for (int s = 0; s < kRing; ++s) { mbar_init(&tfull[s], 1); mbar_init(&tempty[s], 1 + kEpiWarps); }
        mbar_init(pubbar, kEpiWarps);
        mbar_init(drainbar, 1);
        mbar_fence_init();
        tma_prefetch_desc(&maps.b_x);
        tma_prefetch_desc(&maps.b_h);
        if (a.dense2_T > 0) { tma_prefetch_desc(&maps.b_x2); tma_prefetch_desc(&maps.b_h2); }
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // when launched as a programmatic dependent, the set-up above overlaps the previous
    // kernel and its results (units, activations) are read only from here on (a no-op
    // otherwise)
    grid_dependency_wait();
    grid_dependents_launch();

    if (warp == 0) {
        // ------------------------------------------------ scheduler + copy producer
        // Lane 0 takes tiles and issues every barrier, bulk and TMA operation.  For
        // routed gate/up tiles with a.row_token set, the whole warp also gathers the
        // unit's token rows straight from x into the stage (stored with the 128-byte
        // swizzle, loaded one k-step ahead), so no permuted copy of x is needed.
        // Every stage's full barrier takes two arrivals: the expect-tx arrival and a
        // completion arrival once this warp has written or issued everything.
        const uint64_t pol_w = policy_evict_first();   // weights stream through once
        const uint64_t pol_x = policy_evict_last();    // activations are re-read per tile
        const uint8_t* w_gu = static_cast<const uint8_t*>(a.w_gu);
        const uint8_t* w_dn = static_cast<const uint8_t*>(a.w_down);
        const __nv_bfloat16* x_rows = static_cast<const __nv_bfloat16*>(a.x_rows);
        uint32_t it = 0;
        int tc = 0;
        bool ok = true, stuck_pending = a.inject_stuck != 0;
        while (true) {
            int i = n_tiles;
            if (lane == 0 && ok && !error_pending(a.st)) i = atomicAdd(tile_counter, 1);
            i = __shfl_sync(0xffffffffu, i, 0);
            Tile t = decode_tile(i, n_units, n_units2, a, mt_gu0, mt_gu1, mt_dn, BN);
            const int r = tc % kRing;
            int w_ok = 1;
            if (lane == 0) {
                w_ok = mbar_wait(&tempty[r], ((tc / kRing) & 1) ^ 1, a.st, limit);
                if (w_ok) { ring[r] = t; mbar_arrive(&tfull[r]); }
            }
            if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
            ++tc;
            if (t.phase < 0) break;
            const bool p1 = t.prob == 1;
            const bool gather = BN <= 32 && t.phase == 0 && !p1 && a.row_token != nullptr;
            const int nb16 = (t.n_len + kBoxRows - 1) / kBoxRows;
            const int mt_gu = p1 ? mt_gu1 : mt_gu0;
            const int kb_dn = p1 ? kb_dn1 : kb_dn0;
            const int KB = t.phase == 0 ? kb_gu : kb_dn;
            // a tile pair per k-step; the zero-filled second panel of an odd count of
            // 128-row blocks (W_down with odd H / 128, W_r with odd E / 128) is skipped
            const uint32_t a_stride = 2 * kABytes;
            const uint32_t a_bytes = single_panel(t, a) ? kABytes : a_stride;
            const uint32_t bytes = a_bytes + (gather ? 0 : nb16 * kBoxBytes);
            const uint8_t* wg = p1 ? static_cast<const uint8_t*>(a.w_gu2) : w_gu;
            const uint8_t* wd = p1 ? static_cast<const uint8_t*>(a.w_down2) : w_dn;
            const uint8_t* a_src =
                t.phase == 0 ? wg + (size_t)(t.expert * mt_gu + t.mt) * kb_gu * a_stride
                : t.phase == 1 ? wd + (size_t)(t.expert * mt_dn + t.mt) * kb_dn * a_stride
                               : w_gu + (size_t)t.mt * kb_dn * a_stride;   // packed W_r
            const CUtensorMap* bmap = t.phase == 1 ? (p1 ? &maps.b_h2 : &maps.b_h)
                                                   : (p1 ? &maps.b_x2 : &maps.b_x);
            int* done = p1 ? a.done2 : a.sync + 2;
            // gather mode: lane covers (row, 16-byte chunk) pairs p = lane + 32 j
            const __nv_bfloat16* src_row[8];
            uint4 nx[8];
            if (gather) {
                const int my_tok = lane < t.n_len ? a.row_token[t.row_start + lane] : 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int p = lane + 32 * j, rr = p >> 3, cc = p & 7;
                    const int tok = __shfl_sync(0xffffffffu, my_tok, rr);
                    src_row[j] = rr < t.n_len ? x_rows + (size_t)tok * a.H + cc * 8 : nullptr;
                    if (src_row[j]) nx[j] = *reinterpret_cast<const uint4*>(src_row[j]);
                }
            }
            // Down tiles of a fused launch first stream their weights (independent of h),
            // then wait until the unit's gate/up tiles have published h, then load h rows.
            const bool gated = t.phase == 1 && fused;
            const int pre = gated ? min(KB, C::kStages) : 0;
            int fail = 0;
            for (int kb = 0; kb < pre; ++kb) {
                const uint32_t q = it + kb;
                const int s = q % C::kStages;
                if (lane == 0) {
                    if (!mbar_wait(&empty[s], ((q / C::kStages) & 1) ^ 1, a.st, limit)) fail = 1;
                    else {
                        mbar_arrive_expect_tx(&full[s], bytes);
                        bulk_load(smem + s * C::kStageBytes, a_src + (size_t)kb * a_stride, a_bytes,
                                  &full[s], pol_w);
                    }
                }
                if (__shfl_sync(0xffffffffu, fail, 0)) break;
            }
            if (__shfl_sync(0xffffffffu, fail, 0)) { ok = false; break; }
            if (gated) {
                if (lane == 0) {
                    const int target = mt_gu + (stuck_pending ? 1 : 0);
                    if (!wait_count(done + t.unit, target, a)) ok = false;   // finish the tile anyway
                    fence_proxy_async_global();
                    for (int kb = 0; kb < pre; ++kb) {
                        const int s = (it + kb) % C::kStages;
                        uint8_t* B = smem + s * C::kStageBytes + 2 * kABytes;
                        for (int j = 0; j < nb16; ++j)
                            tma_load_2d(B + j * kBoxBytes, bmap, &full[s], kb * kBK,
                                        t.row_start + j * kBoxRows, pol_x);
                        mbar_arrive(&full[s]);
                    }
                }
                stuck_pending = false;
                ok = __shfl_sync(0xffffffffu, (int)ok, 0);
                it += pre;
            }
            for (int kb = pre; kb < KB; ++kb, ++it) {
                const int s = it % C::kStages;
                uint8_t* A0 = smem + s * C::kStageBytes;
                uint8_t* B = A0 + 2 * kABytes;
                if (lane == 0) {
                    if (!mbar_wait(&empty[s], ((it / C::kStages) & 1) ^ 1, a.st, limit)) fail = 1;
                    else {
                        mbar_arrive_expect_tx(&full[s], bytes);
                        bulk_load(A0, a_src + (size_t)kb * a_stride, a_bytes, &full[s], pol_w);
                        if (!gather)
                            for (int j = 0; j < nb16; ++j)
                                tma_load_2d(B + j * kBoxBytes, bmap, &full[s], kb * kBK,
                                            t.row_start + j * kBoxRows, pol_x);
                    }
                }
                if (__shfl_sync(0xffffffffu, fail, 0)) break;
                if (gather) {
                    // rows of this k-step into the stage, then the next k-step's loads
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int p = lane + 32 * j, rr = p >> 3, cc = p & 7;
                        if (src_row[j])
                            *reinterpret_cast<uint4*>(B + rr * 128 + ((cc ^ (rr & 7)) << 4)) = nx[j];
                    }
                    if (kb + 1 < KB) {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            if (src_row[j])
                                nx[j] = *reinterpret_cast<const uint4*>(src_row[j] + (kb + 1) * kBK);
                    }
                    fence_proxy_async_smem();     // generic stores -> tensor-core reads
                    __syncwarp();
                }
                if (lane == 0) mbar_arrive(&full[s]);
            }
            if (__shfl_sync(0xffffffffu, fail, 0)) { ok = false; break; }
        }
        // drain: copies still in flight must land before the CTA exits
        if (lane == 0)
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
            const int KB = t.phase == 0 ? kb_gu : (t.prob ? kb_dn1 : kb_dn0);
            const bool one = single_panel(t, a);
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
                    // gate/up: (gate, up) panels; down: two 128-row output blocks
                    tc_mma_bf16(d_gate, smem_desc_sw128(a0 + kk * 32), bd, idesc, accum);
                    if (!one) tc_mma_bf16(d_up, smem_desc_sw128(a1 + kk * 32), bd, idesc, accum);
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
        // Warp pairs (q, q + 4) share TMEM lanes 32q..32q+31 and take alternate
        // 16-column chunks.  A chunk (32 features x 16 rows) is transposed through
        // shared memory so that each store writes 16 contiguous bytes of a row.
        const int ew = warp - 2;
        const int q = warp & 3;
        const int half = ew >> 2;
        __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(epi_smem + ew * kEpiStage);

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
            const int nc = (t.n_len + 15) / 16;
            // gate/up: h[rows][mt*128 + 32q + lane] = SiLU(gate) * up
            // down:    out[rows][mt*256 + p*128 + 32q + lane] = panel p, p = 0, 1
            if (t.phase == 2) {
                // router logits: logits[rows][256 mt + 128 p + 32 q + lane], fp32
                const int e0 = t.mt * 2 * kBM + q * 32 + lane;
                float* lg = a.logits + (size_t)t.row_start * a.I;
                const int rpanels = single_panel(t, a) ? 1 : 2;
                for (int c = half; c < nc; c += 2) {
                    for (int p = 0; p < rpanels; ++p) {
                        float v[16];
                        tmem_ld16((p ? tu : tg) + c * 16, v);
                        tmem_wait_ld();
                        const int e = e0 + p * kBM;
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (c * 16 + j < t.n_len && e < a.I) lg[(size_t)(c * 16 + j) * a.I + e] = v[j];
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&accempty[acc]);
                ++ac;
                continue;
            }
            const int ld = t.phase == 0 ? (t.prob ? a.I2 : a.I) : a.H;
            const int col0 = t.phase == 0 ? t.mt * kBM : t.mt * 2 * kBM;
            const int panels = t.phase == 0 ? 1 : (col0 + kBM < a.H ? 2 : 1);
            void* base = t.phase == 0 ? (t.prob ? a.hbuf2 : a.hbuf) : (t.prob ? a.out2 : a.out);
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(base) + (size_t)t.row_start * ld +
                                 col0 + q * 32;
            for (int c = half; c < nc; c += 2) {
                for (int p = 0; p < panels; ++p) {
                    float v[16];
                    if (t.phase == 0) {
                        float u[16];
                        tmem_ld16(tg + c * 16, v);
                        tmem_ld16(tu + c * 16, u);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) v[j] = silu_fast(v[j]) * u[j];
                    } else {
                        tmem_ld16((p ? tu : tg) + c * 16, v);
                        tmem_wait_ld();
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) stage[j * 32 + lane] = __float2bfloat16_rn(v[j]);
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int vid = lane + 32 * i, row = vid >> 2, seg = vid & 3;
                        if (c * 16 + row < t.n_len)
                            *reinterpret_cast<uint4*>(dst + (size_t)(c * 16 + row) * ld + p * kBM +
                                                      seg * 8) =
                                *reinterpret_cast<const uint4*>(stage + row * 32 + seg * 8);
                    }
                    __syncwarp();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[acc]);
            ++ac;
            if (t.phase == 0 && fused) {
                // publish this unit's h rows to the down tiles (other CTAs read them by TMA)
                __threadfence();
                fence_proxy_async_global();
                __syncwarp();
                if (lane == 0) mbar_arrive(pubbar);
                if (ew == 0 && lane == 0) {
                    int* done = t.prob ? a.done2 : a.sync + 2;
                    if (mbar_wait(pubbar, pub & 1, a.st, limit)) red_release_gpu_add(done + t.unit, 1);
                }
                ++pub;
            }
        }
    }

    // ------------------------------------------------ teardown
    // The MMA role runs on lane 0 of warp 1 only: reconverge every warp before
    // the CTA barrier (bar.sync expects whole warps).
    __syncwarp();
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
        for (int u = tid; u < n_units; u += kThreads) a.sync[2 + u] = 0;
        for (int u = tid; u < n_units2; u += kThreads) a.done2[u] = 0;
        if (tid == 0) { *tile_counter = 0; *exit_counter = 0; }
    }
}

// Two entry points with one body, so profiles tell the expert GEMMs (grouped
// routed experts, with the shared expert's dense tiles) from the router logits.
template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
tc_routed_experts_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
    tc_experts_body<BN>(maps, a);
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
tc_router_logits_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
    tc_experts_body<BN>(maps, a);
}

template <int BN>
cudaError_t launch_width(const TcMaps& maps, const TcArgs& a, int grid, int pdl, cudaStream_t s) {
    static std::once_flag configured[16];    // the attribute is set per device
    cudaError_t e = once_per_device(configured, [] {
        cudaError_t r = cudaFuncSetAttribute(tc_routed_experts_kernel<BN>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             TcCfg<BN>::kSmem);
        if (r == cudaSuccess)
            r = cudaFuncSetAttribute(tc_router_logits_kernel<BN>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     TcCfg<BN>::kSmem);
        return r;
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = TcCfg<BN>::kSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (a.phases == 4) return cudaLaunchKernelEx(&cfg, tc_router_logits_kernel<BN>, maps, a);
    return cudaLaunchKernelEx(&cfg, tc_routed_experts_kernel<BN>, maps, a);
}

}  // namespace

int tc_smem_bytes(int width) {
    return width <= 32 ? TcCfg<32>::kSmem : TcCfg<256>::kSmem;
}

cudaError_t launch_tc_experts(const TcMaps& maps, const TcArgs& a, int width, int grid,
                              cudaStream_t s, int pdl) {
    if (grid <= 0) return cudaSuccess;
    if (a.H % kBM || a.I % kBM) return cudaErrorInvalidValue;   // I, H multiples of 128
    if (a.dense2_T > 0 && (a.I2 % kBM || !a.w_gu2 || !a.w_down2 || !a.done2))
        return cudaErrorInvalidValue;
    if (width == 32) return launch_width<32>(maps, a, grid, pdl, s);
    if (width == 256) return launch_width<256>(maps, a, grid, pdl, s);
    return cudaErrorInvalidValue;
}

}  // namespace moe
