"""Seeded synthetic inputs for the sparse MoE layer (shared by tests and bench).

This module only draws and stores numbers: it holds none of the layer's
arithmetic.  Both the fp64 oracle and the CUDA library consume the exact arrays
produced here (bf16 as uint16 bit patterns, or float32).

Workloads (sizes from the Talker MoE layer: hidden 1024, 128 routed experts,
Top-6, expert SwiGLU 1024->384->1024, shared SwiGLU 1024->768->1024):

  tiny_fp32              T=4,     H=8, E=6, k=2, I=16, Is=32, fp32, all ~0.5*N(0,1), seed 30
  talker_decode          T=8,     bf16, x ~ N(0,1), every weight ~ N(0, 0.02)
  talker_prefill         T=4096,  as decode
  talker_prefill_skewed  T=16384, as decode plus a shared skew direction (below)
  talker_stack20         T=64, 20 layers, each with pre-RMSNorm scale ~ 1 + N(0, 0.01)

Draw order inside one layer: x, W_router, W_gate, W_up, W_down, Ws_gate,
Ws_up, Ws_down, then the RMSNorm scale.  Draws are float32 standard normals
(numpy PCG64), scaled in float32 and rounded to bf16 with round-to-nearest-even.
"""
from __future__ import annotations

import json
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                          "tests", "golden")
SKEW_FILE = os.path.join(GOLDEN_DIR, "skew_talker_prefill_skewed.json")


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 (or float64 via float32) values to bf16, nearest-even; returns uint16 bits."""
    u = np.array(a, dtype=np.float32, copy=True).view(np.uint32)
    lsb = u >> np.uint32(16)
    lsb &= np.uint32(1)
    u += lsb
    u += np.uint32(0x7FFF)
    u >>= np.uint32(16)
    return u.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact float32 value of bf16 bit patterns."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    T: int
    H: int
    E: int
    k: int
    I: int
    Is: int
    dtype: str            # "f32" or "bf16"
    x_scale: float
    w_scale: float
    n_layers: int = 1
    rms: bool = False
    rms_eps: float = 1e-6
    skewed: bool = False
    seed: int = 30


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 0, 4, 8, 6, 2, 16, 32, "f32", 0.5, 0.5, seed=30),
    "talker_decode": Workload("talker_decode", 1, 8, 1024, 128, 6, 384, 768, "bf16", 1.0, 0.02,
                              seed=31),
    "talker_prefill": Workload("talker_prefill", 2, 4096, 1024, 128, 6, 384, 768, "bf16", 1.0,
                               0.02, seed=32),
    "talker_prefill_skewed": Workload("talker_prefill_skewed", 3, 16384, 1024, 128, 6, 384, 768,
                                      "bf16", 1.0, 0.02, skewed=True, seed=33),
    "talker_stack20": Workload("talker_stack20", 4, 64, 1024, 128, 6, 384, 768, "bf16", 1.0, 0.02,
                               n_layers=20, rms=True, seed=34),
}


@dataclass
class Layer:
    """One layer's weights in nn.Linear [out, in] layout, storage format."""
    w_router: np.ndarray
    w_gate: np.ndarray
    w_up: np.ndarray
    w_down: np.ndarray
    ws_gate: np.ndarray
    ws_up: np.ndarray
    ws_down: np.ndarray
    rms_w: np.ndarray | None = None

    def arrays(self) -> dict:
        return {k: v for k, v in self.__dict__.items() if v is not None}

    @property
    def nbytes(self) -> int:
        return sum(a.nbytes for a in self.arrays().values())


@dataclass
class Inputs:
    workload: Workload
    x: np.ndarray
    layers: list = field(default_factory=list)
    skew: dict | None = None


def _store(wl: Workload, a32: np.ndarray) -> np.ndarray:
    return a32.astype(np.float32) if wl.dtype == "f32" else bf16_bits(a32)


def _normal(rng, shape, scale) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    return a


def draw_layer_weights(wl: Workload, rng, H=None, E=None, I=None, Is=None,
                       router_rows_hook=None) -> Layer:
    """Weights of one layer in the fixed draw order (after x, which the caller drew)."""
    H = H or wl.H; E = E or wl.E; I = I or wl.I; Is = wl.Is if Is is None else Is
    s = wl.w_scale
    wr = _normal(rng, (E, H), s)
    if router_rows_hook is not None:
        wr = router_rows_hook(wr)
    layer = Layer(
        w_router=_store(wl, wr),
        w_gate=_store(wl, _normal(rng, (E, I, H), s)),
        w_up=_store(wl, _normal(rng, (E, I, H), s)),
        w_down=_store(wl, _normal(rng, (E, H, I), s)),
        ws_gate=_store(wl, _normal(rng, (Is, H), s)),
        ws_up=_store(wl, _normal(rng, (Is, H), s)),
        ws_down=_store(wl, _normal(rng, (H, Is), s)),
    )
    if wl.rms:
        layer.rms_w = _store(wl, np.float32(1.0) + _normal(rng, (H,), 0.01))
    return layer


def load_skew() -> dict:
    with open(SKEW_FILE) as f:
        return json.load(f)


def skew_sets(wl: Workload, E: int):
    """Hot (8) and dead (48) expert ids of the skewed workload: a seeded permutation."""
    perm = np.random.default_rng((wl.seed, 7)).permutation(E)
    return sorted(int(e) for e in perm[:8]), sorted(int(e) for e in perm[8:56])


def make_skewed(wl: Workload, T: int, s: float, dead_steps: int, hot_bias: float = 0.05,
                router_only: bool = False) -> Inputs:
    """Skewed routing: 8 hot router rows get +hot_bias along a shared unit
    direction d that is also added (times s) to every token; 48 "dead" rows get
    -dead_steps*hot_bias along d so that they receive no token.  With
    router_only, the expert weights (drawn after x and W_router) are left out."""
    rng = np.random.default_rng(wl.seed)
    x32 = _normal(rng, (T, wl.H), wl.x_scale)
    d = np.random.default_rng((wl.seed, 11)).standard_normal(wl.H)
    d = d / np.sqrt(np.sum(d * d))
    hot, dead = skew_sets(wl, wl.E)

    def hook(wr):
        wr = wr.astype(np.float64)
        wr[hot] += hot_bias * d
        wr[dead] -= dead_steps * hot_bias * d
        return wr.astype(np.float32)

    if router_only:
        wr = hook(_normal(rng, (wl.E, wl.H), wl.w_scale))
        layer = Layer(_store(wl, wr), *(None,) * 6)
    else:
        layer = draw_layer_weights(wl, rng, router_rows_hook=hook)
    x = (x32.astype(np.float64) + s * d).astype(np.float32)
    return Inputs(wl, _store(wl, x), [layer],
                  skew=dict(s=s, dead_steps=dead_steps, hot=hot, dead=dead, hot_bias=hot_bias))


def make(name: str, T: int | None = None) -> Inputs:
    """Inputs of a named workload (optionally with a different token count T)."""
    wl = WORKLOADS[name]
    T = wl.T if T is None else T
    if wl.skewed:
        p = load_skew()
        return make_skewed(wl, T, p["s"], p["dead_steps"], p.get("hot_bias", 0.05))
    if wl.n_layers > 1:
        x = _store(wl, _normal(np.random.default_rng((wl.seed, 0)), (T, wl.H), wl.x_scale))
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            layers = list(ex.map(lambda l: draw_layer_weights(
                wl, np.random.default_rng((wl.seed, 1 + l))), range(wl.n_layers)))
        return Inputs(wl, x, layers)
    rng = np.random.default_rng(wl.seed)
    x = _store(wl, _normal(rng, (T, wl.H), wl.x_scale))
    return Inputs(wl, x, [draw_layer_weights(wl, rng)])


def make_extra_weights(name: str, copy: int) -> Layer:
    """Independent weight copy number `copy` >= 1 of a workload (for L2 rotation)."""
    wl = WORKLOADS[name]
    return draw_layer_weights(wl, np.random.default_rng((wl.seed, 100 + copy)))


def make_custom(H: int, E: int, k: int, I: int, Is: int, T: int, dtype: str = "bf16",
                seed: int = 0, x_scale: float = 1.0, w_scale: float = 0.02,
                rms: bool = False) -> Inputs:
    """Small parity-test layers of arbitrary shape, same recipe as the workloads."""
    wl = Workload(f"custom_H{H}_E{E}_k{k}_I{I}_Is{Is}", -1, T, H, E, k, I, Is, dtype, x_scale,
                  w_scale, rms=rms, seed=seed)
    rng = np.random.default_rng((seed, H, E, k, I, Is))
    x = _store(wl, _normal(rng, (T, H), x_scale))
    return Inputs(wl, x, [draw_layer_weights(wl, rng)])


def make_tokens(wl: Workload, T: int, seed: int) -> np.ndarray:
    """Fresh token activations for an existing layer (x ~ x_scale * N(0,1))."""
    return _store(wl, _normal(np.random.default_rng((wl.seed, 200 + seed)), (T, wl.H),
                              wl.x_scale))
