"""fp64 CPU oracle of the sparse MoE feed-forward layer -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It shares nothing with the CUDA library: the C
oracle (``moe_oracle.c``) is compiled here with gcc into ``liboracle.so`` and
called through ctypes; ``numpy_ref`` is a second, independent fp64 statement of
the same layer used to cross-check the C code.

Inputs are numpy arrays in their storage format: ``float32``, ``float64`` or
bf16 held as ``uint16`` bit patterns.  Every value is widened exactly to fp64
inside the oracle.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_HDR = os.path.join(_HERE, "moe_oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16, F64 = 0, 1, 2
_lock = threading.Lock()
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the C oracle with gcc (OpenMP over tokens).  Returns the path."""
    stale = force or not os.path.exists(out) or any(
        os.path.getmtime(p) > os.path.getmtime(out) for p in (src, _HDR))
    if stale:
        # a private temporary per process, then an atomic replace: several processes
        # (e.g. the ranks of a multi-process test) may rebuild at the same time
        tmp = f"{out}.{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-I", _HERE, src, "-o", tmp, "-lm"]
        try:
            subprocess.run(cmd, check=True)
            os.replace(tmp, out)
        finally:
            if os.path.exists(tmp):
                os.remove(tmp)
    return out


class _Cfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("expert_inter", ctypes.c_int),
                ("shared_inter", ctypes.c_int), ("dtype", ctypes.c_int),
                ("has_rms", ctypes.c_int), ("rms_eps", ctypes.c_double)]


class _W(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w_router", "w_gate", "w_up", "w_down", "ws_gate", "ws_up",
                 "ws_down", "rms_w")]


def load_library(path: str | None = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    with _lock:
        if path is not None:
            lib = ctypes.CDLL(path)
        elif _lib is not None:
            return _lib
        else:
            lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        lib.oracle_route.argtypes = [ctypes.POINTER(_Cfg), ctypes.POINTER(_W), P,
                                     ctypes.c_int, P, P, P, P, ctypes.c_int]
        lib.oracle_route.restype = ctypes.c_int
        lib.oracle_forward.argtypes = [ctypes.POINTER(_Cfg), ctypes.POINTER(_W), P, P,
                                       ctypes.c_int, P, P, P, P, P, ctypes.c_int]
        lib.oracle_forward.restype = ctypes.c_int
        lib.oracle_threads.argtypes = [ctypes.c_int]
        lib.oracle_threads.restype = ctypes.c_int
        if path is None:
            _lib = lib
        return lib


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.float64:
        return F64
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle input dtype {a.dtype} not supported")


@dataclass
class LayerWeights:
    """One layer's weights in nn.Linear [out, in] layout (storage format)."""
    w_router: np.ndarray          # [E, H]
    w_gate: np.ndarray            # [E, I, H]
    w_up: np.ndarray              # [E, I, H]
    w_down: np.ndarray            # [E, H, I]
    ws_gate: np.ndarray | None    # [Is, H]
    ws_up: np.ndarray | None      # [Is, H]
    ws_down: np.ndarray | None    # [H, Is]
    rms_w: np.ndarray | None = None   # [H]
    rms_eps: float = 1e-6
    top_k: int = 1

    @property
    def dims(self):
        E, I, H = self.w_gate.shape
        Is = 0 if self.ws_gate is None else self.ws_gate.shape[0]
        return H, E, self.top_k, I, Is


class Oracle:
    """ctypes front end of the C oracle for one layer's weights."""

    def __init__(self, w: LayerWeights, lib=None):
        self.w = w
        self.lib = lib or load_library()
        H, E, k, I, Is = w.dims
        arrays = [w.w_router, w.w_gate, w.w_up, w.w_down]
        if Is:
            arrays += [w.ws_gate, w.ws_up, w.ws_down]
        if w.rms_w is not None:
            arrays.append(w.rms_w)
        codes = {_dtype_code(a) for a in arrays}
        if len(codes) != 1:
            raise TypeError("all weights must share one storage format")
        self.dtype = codes.pop()
        self._cfg = _Cfg(H, E, k, I, Is, self.dtype, int(w.rms_w is not None), w.rms_eps)
        names = [f[0] for f in _W._fields_]
        # keep contiguous copies alive for as long as the C side holds pointers
        self._keep = {n: (None if getattr(w, n) is None else np.ascontiguousarray(getattr(w, n)))
                      for n in names}
        self._w = _W(*[None if self._keep[n] is None else self._keep[n].ctypes.data
                       for n in names])

    def _x(self, x: np.ndarray) -> np.ndarray:
        x = np.ascontiguousarray(x)
        if _dtype_code(x) != self.dtype:
            raise TypeError("x must use the weights' storage format")
        return x

    def route(self, x: np.ndarray, nthreads: int = 0):
        """Returns (logits [T,E], topk_idx [T,k] int32, topk_w [T,k], kgap [T])."""
        x = self._x(x)
        H, E, k, _, _ = self.w.dims
        T = x.shape[0]
        logits = np.empty((T, E)); idx = np.empty((T, k), np.int32)
        wts = np.empty((T, k)); gap = np.empty(T)
        rc = self.lib.oracle_route(ctypes.byref(self._cfg), ctypes.byref(self._w),
                                   x.ctypes.data, T, logits.ctypes.data, idx.ctypes.data,
                                   wts.ctypes.data, gap.ctypes.data, nthreads)
        if rc:
            raise RuntimeError(f"oracle_route failed ({rc})")
        return logits, idx, wts, gap

    def forward(self, x: np.ndarray, residual: np.ndarray | None = None,
                forced_idx: np.ndarray | None = None, nthreads: int = 0):
        """Returns (y [T,H] fp64, topk_idx, topk_w, kgap)."""
        x = self._x(x)
        H, E, k, _, _ = self.w.dims
        T = x.shape[0]
        if residual is not None:
            residual = self._x(residual)
        if forced_idx is not None:
            forced_idx = np.ascontiguousarray(forced_idx, dtype=np.int32)
            assert forced_idx.shape == (T, k)
        y = np.empty((T, H)); idx = np.empty((T, k), np.int32)
        wts = np.empty((T, k)); gap = np.empty(T)
        rc = self.lib.oracle_forward(
            ctypes.byref(self._cfg), ctypes.byref(self._w), x.ctypes.data,
            None if residual is None else residual.ctypes.data, T,
            None if forced_idx is None else forced_idx.ctypes.data,
            y.ctypes.data, idx.ctypes.data, wts.ctypes.data, gap.ctypes.data, nthreads)
        if rc:
            raise RuntimeError(f"oracle_forward failed ({rc})")
        return y, idx, wts, gap

    def threads(self, nthreads: int = 0) -> int:
        return int(self.lib.oracle_threads(nthreads))
