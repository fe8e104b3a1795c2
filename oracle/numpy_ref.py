"""Second, independent fp64 statement of the MoE layer in NumPy -- TEST ONLY.

It exists to cross-check the C oracle (a slip in one is unlikely to repeat in
the other: different language, different loop structure, library matmuls).
Same definition as ``moe_oracle.h``: page "3C . Talker MoE", section 3 (router
softmax, Top-k, renormalised weights, shared + weighted routed sum); SwiGLU
expert form from page "print(model) Qwen3-TTS"; SiLU / RMSNorm / softmax as the
lab script's helpers define them.
"""
from __future__ import annotations

import numpy as np


def widen(a: np.ndarray) -> np.ndarray:
    """Exact fp64 value of a float32/float64 array or bf16 bit patterns (uint16)."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def layer(x, w_router, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, top_k,
          rms_w=None, rms_eps=1e-6, residual=None):
    """Returns (y [T,H], topk_idx [T,k], topk_w [T,k])."""
    x = widen(x)
    Wr, Wg, Wu, Wd = widen(w_router), widen(w_gate), widen(w_up), widen(w_down)
    if rms_w is not None:
        ms = np.mean(x * x, axis=-1, keepdims=True)
        x = x / np.sqrt(ms + rms_eps) * widen(rms_w)
    T, H = x.shape
    E = Wr.shape[0]
    y = np.zeros((T, H))
    idx = np.zeros((T, top_k), np.int32)
    wts = np.zeros((T, top_k))
    silu = lambda z: z / (1.0 + np.exp(-z))
    for t in range(T):
        v = x[t]
        logit = Wr @ v
        p = np.exp(logit - logit.max())
        p = p / p.sum()
        # descending logit, ties to the lower expert index (lexsort: last key primary)
        order = np.lexsort((np.arange(E), -logit))
        S = order[:top_k]
        w = p[S] / p[S].sum()
        out = np.zeros(H)
        if ws_gate is not None:
            hs = silu(widen(ws_gate) @ v) * (widen(ws_up) @ v)
            out += widen(ws_down) @ hs
        for wi, e in zip(w, S):
            h = silu(Wg[e] @ v) * (Wu[e] @ v)
            out += wi * (Wd[e] @ h)
        y[t] = out
        idx[t] = S
        wts[t] = w
    if residual is not None:
        y = y + widen(residual)
    return y, idx, wts
