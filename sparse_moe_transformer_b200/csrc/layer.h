// layer.h -- internal declarations shared by the host runtime and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

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
    int32_t* block_hist;  // [nblocks][E]
    int32_t* block_off;   // [nblocks][E] exclusive prefix over blocks
    int32_t* counts;      // [E]
    int32_t* offsets;     // [E+1]
    Unit* units;          // [max_units]
    int32_t* n_units;     // [1]
    int32_t* token_slot;  // [T*k]  permuted row of (t, j)
    int32_t* slot_token;  // [T*k]  token of permuted row
    int32_t* slot_expert; // [T*k]  expert of permuted row
    int32_t* tickets;     // [nblocks + 1] arrival counters (self-resetting)
};

// ---------------------------------------------------------------- launchers
// Router: logits (fp32 accumulate), optional fused pre-RMSNorm, Top-k with the
// lower-index tie rule, renormalised weights, per-block histograms and (when
// do_scan) the global scan, expert offsets and the GEMM unit list.
cudaError_t launch_router(int dtype, const void* x, const void* w_router, const void* rms_w,
                          float rms_eps, void* x_norm, const Dims& d, int T, int tb,
                          const RouteBufs& rb, int do_scan, int unit_width, int max_units,
                          const DeviceStatus& st, cudaStream_t s);

// Gather token rows into expert-contiguous order; fills token_slot / slot_token.
cudaError_t launch_permute(int dtype, const void* x_in, void* xp, const Dims& d, int T, int tb,
                           const RouteBufs& rb, cudaStream_t s);

// y = [residual +] s + sum_j w_tj * o[token_slot[t][j]]
cudaError_t launch_combine(int dtype, const void* o, const void* shared_out, const void* residual,
                           void* y, const float* topk_w, const int32_t* token_slot,
                           const Dims& d, int T, cudaStream_t s);

// CUDA-core expert kernels (exact fp32 accumulate; any shape).
// rows: permuted rows (routed) or tokens (shared, slot_expert == nullptr).
cudaError_t launch_simt_gate_up(int dtype, const void* xin, const void* w_gate, const void* w_up,
                                const int32_t* slot_expert, const int32_t* n_rows_dev,
                                int max_rows, int H, int I, void* hbuf, cudaStream_t s);
cudaError_t launch_simt_down(int dtype, const void* hbuf, const void* w_down,
                             const int32_t* slot_expert, const int32_t* n_rows_dev, int max_rows,
                             int H, int I, void* out, cudaStream_t s);

// tcgen05 grouped SwiGLU expert GEMM (bf16, fp32 accumulate).
struct TcMaps {
    CUtensorMap a_gate, a_up, a_down;   // weights [E*I][H], [E*I][H], [E*H][I]
    CUtensorMap b_x, b_h;               // activations [rows][H], [rows][I]
};
struct TcArgs {
    int H, I;
    int phases;          // 1: gate/up, 2: down, 3: both in one launch with dependencies
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
};
// width: 32 (decode) or 256 (prefill) tile-width instance.
cudaError_t launch_tc_experts(const TcMaps& maps, const TcArgs& a, int width, int grid,
                              cudaStream_t s);
int tc_smem_bytes(int width);

}  // namespace moe
