// layer.h -- internal declarations shared by the host runtime and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace moe {

// device-side error codes (same values as the public moe_status)
constexpr int kErrTimeout = 5;
constexpr int kErrDeviceCheck = 6;

// Where kernels record failures.  err_host is host-mapped pinned memory (may be null).
struct DeviceStatus {
    int* err_dev;
    int* err_host;
};

// A run of permuted rows that belong to one expert and fit one GEMM tile.
struct Unit {
    int expert;
    int row_start;   // first permuted row
    int n_len;       // rows in this unit, 1..tile width
    int pad;
};

// Dimensions of one layer.
struct Dims {
    int H, E, k, I, Is;
};

// Routing bookkeeping buffers (device).
struct RouteBufs {
    float* logits;        // [T][E] fp32 scratch (multi-CTA router)
    int32_t* topk_idx;    // [T][k]
    float* topk_w;        // [T][k]
    int32_t* block_hist;  // [nblocks][E] selections per routing block (zeroed by the scan)
    int32_t* block_off;   // [nblocks][E] exclusive prefix over blocks
    int32_t* counts;      // [E]
    int32_t* offsets;     // [E+1]
    Unit* units;          // [max_units]
    int32_t* n_units;     // [1]
    int32_t* token_slot;  // [T*k]  permuted row of (t, j)
    int32_t* slot_token;  // [T*k]  token of permuted row
    int32_t* slot_expert; // [T*k]  expert of permuted row
    int32_t* tickets;     // [T / 8 + 1] arrival counters (self-resetting)
};

// A launcher's once-per-device set-up (kernel attributes are set per device): runs
// `setup` the first time any thread asks for the current device; other threads
// asking meanwhile wait for it.  Returns setup's result to the thread that ran it.
template <typename Setup>
inline cudaError_t once_per_device(std::once_flag (&flags)[16], Setup&& setup) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return setup();
    cudaError_t e = cudaSuccess;
    std::call_once(flags[dev], [&] { e = setup(); });
    return e;
}

// ---------------------------------------------------------------- launchers
// Router: logits (fp32 accumulate), optional fused pre-RMSNorm, Top-k with the
// lower-index tie rule, renormalised weights, per-block histograms and (when
// do_scan) the global scan, expert offsets and the GEMM unit list.  With
// select_only the logits already sit in rb.logits (tensor-core router).
// With permute and a single routing block (T <= tb) the last CTA also performs
// the permutation (what launch_permute would do; the row copy only if xp != null).
// pdl: launch as a programmatic dependent of the previous kernel in the stream
// (the router waits on the device for it before reading anything).
cudaError_t launch_router(int dtype, const void* x, const void* w_router, const void* rms_w,
                          float rms_eps, void* x_norm, int permute, void* xp, const Dims& d,
                          int T, int tb, const RouteBufs& rb, int do_scan, int unit_width,
                          int max_units, int select_only, const DeviceStatus& st,
                          cudaStream_t s, int pdl = 0);

// One-CTA tensor-core router for a handful of tokens (bf16, no pre-norm, 128
// experts, T <= 64): W_r packed as k-pairs (launch_pack_kpairs), x by a TMA map
// with 64 x round16(T) boxes.  Writes topk_idx / topk_w.
struct RouterTcArgs {
    const void* w_router_kp;
    int32_t* topk_idx;
    float* topk_w;
    int H, k, T;
    DeviceStatus st;
    uint64_t wait_limit_ns;
};
bool router_tc_supported(int E, int H, int k, int T);
// pdl: launch as a programmatic dependent of the previous kernel in the stream.
cudaError_t launch_router_tc(const CUtensorMap& xmap, const RouterTcArgs& a, int pdl,
                             cudaStream_t s);

// Expert-contiguous order of the token rows: fills token_slot / slot_token /
// slot_expert, and gathers the rows into xp unless xp is null.
cudaError_t launch_permute(int dtype, const void* x_in, void* xp, const Dims& d, int T, int tb,
                           const RouteBufs& rb, cudaStream_t s, int pdl = 0);

// y = [residual +] s + sum_j w_tj * o[token_slot[t][j]]
cudaError_t launch_combine(int dtype, const void* o, const void* shared_out, const void* residual,
                           void* y, const float* topk_w, const int32_t* token_slot,
                           const Dims& d, int T, cudaStream_t s, int pdl = 0);

// Tile-contiguous weight layout of the tensor-core path.  A weight matrix
// [E][R][C] is cut into 128-row x 64-column tiles, each stored as the exact
// 16 KB image the tensor core reads from shared memory: 128 rows of 128 bytes
// whose 16-byte chunks are permuted by the 128-byte swizzle (chunk c of row r
// stored at chunk c ^ (r % 8)).  Tiles come in pairs that one contiguous 32 KB
// bulk copy moves together:
//   gate/up: pair (e, mt, kb) = gate tile (e, mt, kb), then up tile (e, mt, kb);
//   down:    pair (e, mt2, kb) = tiles (e, 2 mt2, kb) and (e, 2 mt2 + 1, kb),
//            i.e. 256 output rows; a missing odd tile is stored as zeros.
// Pairs are ordered e, then row block, then kb.  Offsets of element (e, row, col):
__host__ __device__ inline size_t swizzled_in_tile(int row, int col) {
    const int r = row % 128, c = col % 64;
    return (size_t)r * 64 + (((c >> 3) ^ (r & 7)) << 3) + (c & 7);
}
__host__ __device__ inline size_t packed_gu_offset(int e, int row, int col, int which, int I,
                                                   int H) {
    const int MT = I / 128, KB = H / 64;
    return ((((size_t)e * MT + row / 128) * KB + col / 64) * 2 + which) * 8192 +
           swizzled_in_tile(row, col);
}
__host__ __device__ inline size_t packed_down_offset(int e, int row, int col, int H, int I) {
    const int MT2 = (H / 128 + 1) / 2, KB = I / 64, mt = row / 128;
    return ((((size_t)e * MT2 + mt / 2) * KB + col / 64) * 2 + (mt & 1)) * 8192 +
           swizzled_in_tile(row, col);
}
__host__ __device__ inline size_t packed_down_elems(int E, int H, int I) {
    return (size_t)E * ((H / 128 + 1) / 2) * (I / 64) * 2 * 8192;
}

// Pack weights into the tile-contiguous layout (bf16): gate/up pairs when
// src1 != nullptr, else down row-block pairs (dst must be zeroed when R / 128 is odd).
cudaError_t launch_pack_tiles(const void* src0, const void* src1, void* dst, int E, int R, int C,
                              cudaStream_t s);
// Pack a [R][C] matrix (bf16) as k-pairs: pair (mt, p) = tile (mt, 2p) then tile
// (mt, 2p + 1), pairs ordered mt then p (R % 128 == 0, C % 128 == 0): one 32 KB
// bulk copy carries 128 columns of one 128-row block.
cudaError_t launch_pack_kpairs(const void* src, void* dst, int R, int C, cudaStream_t s);


// CUDA-core expert kernels (exact fp32 accumulate; any shape).
// rows: permuted rows (routed) or tokens (shared, slot_expert == nullptr).
// packed: weights are in the tile-contiguous layout (gate/up in one buffer).
cudaError_t launch_simt_gate_up(int dtype, const void* xin, const void* w_gate, const void* w_up,
                                int packed, const int32_t* slot_expert, const int32_t* n_rows_dev,
                                int max_rows, int H, int I, void* hbuf, cudaStream_t s);
cudaError_t launch_simt_down(int dtype, const void* hbuf, const void* w_down, int packed,
                             const int32_t* slot_expert, const int32_t* n_rows_dev, int max_rows,
                             int H, int I, void* out, cudaStream_t s);

// tcgen05 grouped SwiGLU expert GEMM (bf16, fp32 accumulate).
struct TcMaps {
    CUtensorMap b_x, b_h;   // activations [rows][H], [rows][I], 16-row boxes, 128-byte swizzle
    CUtensorMap b_x2, b_h2; // the second (dense) problem's, when TcArgs::dense2_T > 0
};
struct TcArgs {
    const void* w_gu;     // packed gate/up tiles (see packed_gu_offset); router: packed W_r
    const void* w_down;   // packed down tiles (see packed_down_offset)
    int H, I;             // router launch: I = number of experts E
    int phases;          // 1: gate/up, 2: down, 3: both in one launch with dependencies,
                         // 4: router logits (dense over dense_T tokens, fp32 into `logits`)
    float* logits;       // [dense_T][I] fp32, router launch only
    const void* x_rows;       // gather mode: token rows [T][H] bf16 (x or its normalised copy)
    const int32_t* row_token; // non-null: routed gate/up tiles gather row r from x_rows
                              // [row_token[r]] instead of loading permuted rows by TMA
    int dense_T;         // >0: units are consecutive row runs over dense_T rows (shared expert)
    int unit_width;      // tile width the units were built with
    const Unit* units;
    const int32_t* n_units;
    int32_t* sync;       // [2 + max_units]: tile counter, exit counter, per-unit done counters
    void* hbuf;          // [rows][I] bf16
    void* out;           // [rows][H] bf16
    DeviceStatus st;
    uint64_t wait_limit_ns;
    int inject_stuck;
    // A second, dense problem in the same launch (the shared expert: every row of
    // x, weights w_gu2 / w_down2 packed like an expert's, intermediate size I2).
    // Its gate/up tiles follow the first problem's, its down tiles follow the first
    // problem's down tiles.  dense2_T == 0: none.
    const void* w_gu2;
    const void* w_down2;
    int I2, dense2_T;
    void* hbuf2;         // [dense2_T][I2] bf16
    void* out2;          // [dense2_T][H] bf16
    int32_t* done2;      // [ceil(dense2_T / width)] per-unit counters (self-resetting)
};
// width: 32 (decode) or 256 (prefill) tile-width instance.
// pdl: launch as a programmatic dependent of the previous kernel in the stream.
cudaError_t launch_tc_experts(const TcMaps& maps, const TcArgs& a, int width, int grid,
                              cudaStream_t s, int pdl = 0);
int tc_smem_bytes(int width);

// Few-token (decode) experts: one tile = the tokens of one expert (or of the
// shared expert) x one 128-feature block; h stays on chip; fp32 partials
// o_part[b][row][H] with rows 0..T*k-1 the routed slots t*k+j and rows
// T*k+t the shared expert's tokens.
struct FusedArgs {
    const void* w_gu;          // routed packed gate/up tile pairs
    const void* w_down;        // routed packed down tile pairs
    const void* ws_gu;         // shared-expert packed gate/up (Is > 0)
    const void* ws_down;       // shared-expert packed down (Is > 0)
    const void* x_rows;        // [T][H] bf16 layer input (x or its normalised copy)
    const int32_t* topk_idx;   // [T][k] from the router
    float* o_part;             // [max(I, Is) / 128][T*k + T][H] fp32
    int H, I, Is, E, k, T;
    int x_early;               // 1: x_rows may be read before the grid dependency wait
                               // (only safe when nothing in flight writes it)
    const int32_t* zero_word;  // a word that stays 0 (bounded-wait test hook)
    DeviceStatus st;
    uint64_t wait_limit_ns;
    int inject_stuck;
};
bool fused_supported(int H, int I, int Is, int E, int k, int S);
int fused_smem_bytes();
int fused_unit_rows();     // token rows per tile
// pdl: launch as a programmatic dependent of the previous kernel in the stream.
cudaError_t launch_fused_experts(const FusedArgs& a, int grid, int pdl, cudaStream_t s);

// y_t = sum_j w_tj sum_b o_part[b][t k + j] + sum_b o_part[b][T k + t] [+ r_t], bf16 out.
cudaError_t launch_combine_partials(const float* o_part, int n_blk, int n_blk_s,
                                    const void* residual, void* y, const float* topk_w,
                                    const Dims& d, int T, int pdl, cudaStream_t s);

}  // namespace moe
