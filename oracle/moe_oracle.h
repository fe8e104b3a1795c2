/*
 * moe_oracle.h -- plain fp64 CPU oracle of one sparse MoE feed-forward layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This oracle exists to check the CUDA path.  Only
 * the test suite, the smoke check and the benchmark's CPU-baseline leg may
 * load it.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (per token t, every step in double precision from the exact
 * values of the stored inputs):
 *
 *   x      = rms ? x_t / sqrt(mean_j x_tj^2 + eps) * g : x_t
 *            ("rmsnorm" helper of the lab script, page "Bai Lab tong hop --
 *             Qwen3-Omni & Qwen3-TTS-12Hz Architecture")
 *   l_e    = sum_j W_r[e][j] x_j                         e = 0..E-1
 *   p      = softmax(l), max-subtracted                  (lab "softmax" helper)
 *   S      = the k experts with the largest p; equal values go to the lower
 *            expert index                                (lab section [3C])
 *   w_i    = p_i / sum_{j in S} p_j                       (norm_topk_prob)
 *   E_i(x) = W_down_i ( SiLU(W_gate_i x) * (W_up_i x) ),  SiLU(z) = z/(1+e^-z)
 *   y      = Shared(x) + sum_{i in S} w_i E_i(x)  [+ residual_t]
 *
 * The routing and combine equations are those of page "3C . Talker MoE (20 lop,
 * 128 Experts Top-6) & Dau ra ma ngu nghia c_0", section 3 "Giai phap"; the
 * SwiGLU expert form down(SiLU(gate(x)) * up(x)) with no biases is from page
 * "print(model) Qwen3-TTS", section on the SwiGLU feed-forward network and the
 * printed Linear(..., bias=False) modules.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Storage formats the oracle can read.  bf16 values are widened exactly. */
enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_F64 = 2 };

typedef struct {
    int hidden;        /* H                                   */
    int n_experts;     /* E                                   */
    int top_k;         /* k, 1 <= k <= E                      */
    int expert_inter;  /* I, routed expert intermediate size  */
    int shared_inter;  /* I_s, 0 = no shared expert           */
    int dtype;         /* storage format of every input array */
    int has_rms;       /* 1 = apply the pre-RMSNorm with rms_w */
    double rms_eps;
} oracle_cfg;

typedef struct {
    const void* w_router;  /* [E][H]   */
    const void* w_gate;    /* [E][I][H] */
    const void* w_up;      /* [E][I][H] */
    const void* w_down;    /* [E][H][I] */
    const void* ws_gate;   /* [I_s][H] */
    const void* ws_up;     /* [I_s][H] */
    const void* ws_down;   /* [H][I_s] */
    const void* rms_w;     /* [H], used when has_rms */
} oracle_weights;

/*
 * Route T tokens: logits (T x E, may be NULL), selected experts (T x k, in
 * selection order: descending logit, ties to the lower index), renormalised
 * weights (T x k) and the k-gap l_(k) - l_(k+1) per token (+inf when k == E).
 * Returns 0 on success, nonzero on a bad argument.
 */
int oracle_route(const oracle_cfg* cfg, const oracle_weights* w,
                 const void* x, int T,
                 double* logits, int32_t* topk_idx, double* topk_w,
                 double* kgap, int nthreads);

/*
 * Full layer for T tokens.  residual (T x H, same storage format) may be NULL.
 * forced_idx (T x k) may be NULL; when given, token t uses that expert set
 * instead of its own Top-k (its weights are still p_i / sum over that set).
 * y is T x H doubles.  topk_idx / topk_w / kgap may be NULL.
 */
int oracle_forward(const oracle_cfg* cfg, const oracle_weights* w,
                   const void* x, const void* residual, int T,
                   const int32_t* forced_idx,
                   double* y, int32_t* topk_idx, double* topk_w, double* kgap,
                   int nthreads);

/* Number of threads the oracle would use when asked for nthreads (<=0: all). */
int oracle_threads(int nthreads);

#ifdef __cplusplus
}
#endif
#endif
