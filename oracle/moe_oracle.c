/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle of one sparse MoE FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY: it checks the CUDA path and is never part of it.
 * Every step below follows the layer's definition literally, one token at a
 * time, with no blocking, fusion or reordering.  The passages each function
 * follows are cited above it; the full statement is in moe_oracle.h.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Exact value of element i of an input array in its storage format.  A bf16
 * value is the upper half of an IEEE binary32, so widening is exact. */
static double load(const void* p, int dtype, size_t i)
{
    if (dtype == ORACLE_F64) return ((const double*)p)[i];
    if (dtype == ORACLE_F32) return (double)((const float*)p)[i];
    uint32_t bits = (uint32_t)((const uint16_t*)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* sum_j W[row][j] * v[j] for a row-major matrix with n columns. */
static double dot_row(const void* W, int dtype, size_t row, int n, const double* v)
{
    double s = 0.0;
    for (int j = 0; j < n; ++j) s += load(W, dtype, row * (size_t)n + j) * v[j];
    return s;
}

/* SiLU(z) = z / (1 + e^-z): the lab script's "silu" helper. */
static double silu(double z) { return z / (1.0 + exp(-z)); }

/*
 * One SwiGLU MLP on one token: down( SiLU(gate v) * (up v) ).
 * gate, up are [inter][H] slices, down is [H][inter]; out gets H values.
 * Form from page "print(model) Qwen3-TTS", SwiGLU feed-forward section.
 */
static void swiglu(const void* gate, const void* up, const void* down, int dtype,
                   size_t gate_row0, size_t down_row0, int H, int inter,
                   const double* v, double* hbuf, double* out)
{
    for (int i = 0; i < inter; ++i) {
        double g = dot_row(gate, dtype, gate_row0 + i, H, v);
        double u = dot_row(up, dtype, gate_row0 + i, H, v);
        hbuf[i] = silu(g) * u;
    }
    for (int o = 0; o < H; ++o) out[o] = dot_row(down, dtype, down_row0 + o, inter, hbuf);
}

/* Layer input for token t: either x_t itself or RMSNorm(x_t) * g with the
 * lab's "rmsnorm" helper: x / sqrt(mean(x^2) + eps) * weight. */
static void layer_input(const oracle_cfg* c, const oracle_weights* w,
                        const void* x, int t, double* v)
{
    const int H = c->hidden;
    for (int j = 0; j < H; ++j) v[j] = load(x, c->dtype, (size_t)t * H + j);
    if (!c->has_rms) return;
    double ms = 0.0;
    for (int j = 0; j < H; ++j) ms += v[j] * v[j];
    ms /= (double)H;
    double r = sqrt(ms + c->rms_eps);
    for (int j = 0; j < H; ++j) v[j] = v[j] / r * load(w->rms_w, c->dtype, (size_t)j);
}

/* "a ranks before b": larger logit first, equal logits go to the lower index. */
static int ranks_before(const double* l, int a, int b)
{
    return l[a] > l[b] || (l[a] == l[b] && a < b);
}

/*
 * Router for one token (page "3C . Talker MoE", section 3: p = softmax(W_r x),
 * S = Top-k of p, w_i = p_i / sum_{j in S} p_j; lab section [3C]).
 * Selection runs on the logits: softmax is strictly increasing, so the order
 * of p and of l is the same, and l avoids ties created by exp rounding.
 * sel gets k experts in selection order; wsel their renormalised weights.
 */
static void route_token(const oracle_cfg* c, const oracle_weights* w, const double* v,
                        double* l, double* p, int* sel, double* wsel, double* gap,
                        const int32_t* forced)
{
    const int H = c->hidden, E = c->n_experts, k = c->top_k;
    for (int e = 0; e < E; ++e) l[e] = dot_row(w->w_router, c->dtype, (size_t)e, H, v);

    double m = l[0];
    for (int e = 1; e < E; ++e) if (l[e] > m) m = l[e];
    double z = 0.0;
    for (int e = 0; e < E; ++e) { p[e] = exp(l[e] - m); z += p[e]; }
    for (int e = 0; e < E; ++e) p[e] /= z;

    /* k+1 rounds of "pick the best expert not yet picked" */
    int order[k + 1 <= E ? k + 1 : E];
    int n_order = k + 1 <= E ? k + 1 : E;
    for (int r = 0; r < n_order; ++r) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            int taken = 0;
            for (int q = 0; q < r; ++q) if (order[q] == e) taken = 1;
            if (taken) continue;
            if (best < 0 || ranks_before(l, e, best)) best = e;
        }
        order[r] = best;
    }
    *gap = (k < E) ? l[order[k - 1]] - l[order[k]] : INFINITY;

    for (int i = 0; i < k; ++i) sel[i] = forced ? forced[i] : order[i];
    double psum = 0.0;
    for (int i = 0; i < k; ++i) psum += p[sel[i]];
    for (int i = 0; i < k; ++i) wsel[i] = p[sel[i]] / psum;
}

static int check(const oracle_cfg* c, const oracle_weights* w, const void* x, int T)
{
    if (!c || !w || T < 0 || (T > 0 && !x)) return 1;
    if (c->hidden <= 0 || c->n_experts <= 0 || c->expert_inter <= 0) return 1;
    if (c->top_k < 1 || c->top_k > c->n_experts || c->shared_inter < 0) return 1;
    if (c->dtype != ORACLE_F32 && c->dtype != ORACLE_BF16 && c->dtype != ORACLE_F64) return 1;
    if (!w->w_router || !w->w_gate || !w->w_up || !w->w_down) return 1;
    if (c->shared_inter > 0 && (!w->ws_gate || !w->ws_up || !w->ws_down)) return 1;
    if (c->has_rms && !w->rms_w) return 1;
    return 0;
}

int oracle_threads(int nthreads)
{
#ifdef _OPENMP
    return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

int oracle_route(const oracle_cfg* c, const oracle_weights* w, const void* x, int T,
                 double* logits, int32_t* topk_idx, double* topk_w, double* kgap,
                 int nthreads)
{
    if (check(c, w, x, T)) return 1;
    const int H = c->hidden, E = c->n_experts, k = c->top_k;
    int bad = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(oracle_threads(nthreads))
#else
    (void)nthreads;
#endif
    for (int t = 0; t < T; ++t) {
        double* v = malloc(sizeof(double) * ((size_t)H + 2 * (size_t)E + k));
        int* sel = malloc(sizeof(int) * (size_t)k);
        if (!v || !sel) { free(v); free(sel); bad = 1; continue; }
        double *l = v + H, *p = l + E, *ws = p + E;
        double gap;
        layer_input(c, w, x, t, v);
        route_token(c, w, v, l, p, sel, ws, &gap, NULL);
        if (logits) for (int e = 0; e < E; ++e) logits[(size_t)t * E + e] = l[e];
        for (int i = 0; i < k; ++i) {
            if (topk_idx) topk_idx[(size_t)t * k + i] = sel[i];
            if (topk_w) topk_w[(size_t)t * k + i] = ws[i];
        }
        if (kgap) kgap[t] = gap;
        free(v);
        free(sel);
    }
    return bad ? 2 : 0;
}

int oracle_forward(const oracle_cfg* c, const oracle_weights* w, const void* x,
                   const void* residual, int T, const int32_t* forced_idx,
                   double* y, int32_t* topk_idx, double* topk_w, double* kgap,
                   int nthreads)
{
    if (check(c, w, x, T) || (T > 0 && !y)) return 1;
    const int H = c->hidden, E = c->n_experts, k = c->top_k;
    const int I = c->expert_inter, Is = c->shared_inter;
    const int hmax = I > Is ? I : Is;
    int bad = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(oracle_threads(nthreads))
#else
    (void)nthreads;
#endif
    for (int t = 0; t < T; ++t) {
        size_t nd = (size_t)H * 3 + 2 * (size_t)E + k + hmax;
        double* v = malloc(sizeof(double) * nd);
        int* sel = malloc(sizeof(int) * (size_t)k);
        if (!v || !sel) { free(v); free(sel); bad = 1; continue; }
        double *l = v + H, *p = l + E, *ws = p + E, *hb = ws + k;
        double *eo = hb + hmax, *acc = eo + H;
        double gap;

        layer_input(c, w, x, t, v);
        route_token(c, w, v, l, p, sel, ws, &gap,
                    forced_idx ? forced_idx + (size_t)t * k : NULL);

        /* y = Shared(x) + sum_{i in S} w_i Expert_i(x) */
        for (int o = 0; o < H; ++o) acc[o] = 0.0;
        if (Is > 0) {
            swiglu(w->ws_gate, w->ws_up, w->ws_down, c->dtype, 0, 0, H, Is, v, hb, eo);
            for (int o = 0; o < H; ++o) acc[o] += eo[o];
        }
        for (int i = 0; i < k; ++i) {
            size_t e = (size_t)sel[i];
            swiglu(w->w_gate, w->w_up, w->w_down, c->dtype, e * I, e * H, H, I, v, hb, eo);
            for (int o = 0; o < H; ++o) acc[o] += ws[i] * eo[o];
        }
        for (int o = 0; o < H; ++o) {
            double r = residual ? load(residual, c->dtype, (size_t)t * H + o) : 0.0;
            y[(size_t)t * H + o] = acc[o] + r;
        }
        for (int i = 0; i < k; ++i) {
            if (topk_idx) topk_idx[(size_t)t * k + i] = sel[i];
            if (topk_w) topk_w[(size_t)t * k + i] = ws[i];
        }
        if (kgap) kgap[t] = gap;
        free(v);
        free(sel);
    }
    return bad ? 2 : 0;
}
