"""Python binding of the B200 sparse MoE layer library (libmoe_b200.so).

Argument marshalling only: every step of the layer runs in the CUDA library
behind include/moe.h.  PyTorch supplies device memory and streams.  There is no
fallback: if the compiled library is missing this module raises at load time.

    layer = MoELayer(cfg, w_router, w_gate, w_up, w_down, ws_gate, ws_up, ws_down)
    y = layer.forward(x)                              # x: [T, H] CUDA tensor
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_CUDA, MOE_ERR_OOM = 0, 1, 2, 3
MOE_ERR_UNSUPPORTED, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE_CHECK = 4, 5, 6
DTYPE_F32, DTYPE_BF16 = 0, 1
OPTIONS = {"wait_limit_ns": 0, "inject_stuck_wait": 1, "shared_stream": 2, "fuse_phases": 3,
           "force_simt": 4, "kernel_timing": 5}
KERNEL_CLASSES = ("router", "permute", "experts", "shared", "combine")

# Every entry point include/moe.h declares (checked by the export test).
EXPORTS = ("moe_create", "moe_reserve", "moe_route", "moe_forward", "moe_forward_host",
           "moe_last_routing", "moe_check", "moe_set_option", "moe_kernel_stats", "moe_destroy",
           "moe_route_noalloc", "moe_status_string", "moe_last_error", "moe_version")


class MoEError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"[{status}] {msg}")
        self.status = status


class _Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int),
                ("expert_inter", ctypes.c_int), ("shared_inter", ctypes.c_int),
                ("dtype", ctypes.c_int), ("norm_topk_prob", ctypes.c_int),
                ("rms_eps", ctypes.c_float)]


_lib = None


def load(path: str = LIB_PATH):
    """Load the compiled library (raises OSError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"{path} is missing: build it with "
                      "`python -m sparse_moe_transformer_b200.build`")
    lib = ctypes.CDLL(path)
    P, I = ctypes.c_void_p, ctypes.c_int
    sig = {
        "moe_create": ([ctypes.POINTER(_Config), I] + [P] * 8 + [ctypes.POINTER(P)], I),
        "moe_reserve": ([P, I], I),
        "moe_route": ([P, P, I, P, P, P], I),
        "moe_forward": ([P, P, P, P, I, P, P, P], I),
        "moe_forward_host": ([P, P, P, P, I, P], I),
        "moe_last_routing": ([P, P, P, P, P], I),
        "moe_check": ([P, P], I),
        "moe_set_option": ([P, I, ctypes.c_int64], I),
        "moe_kernel_stats": ([P, P, P, I], I),
        "moe_route_noalloc": ([ctypes.POINTER(_Config), P, P, P, I, P, P, P], I),
        "moe_destroy": ([P], I),
        "moe_status_string": ([I], ctypes.c_char_p),
        "moe_last_error": ([P], ctypes.c_char_p),
        "moe_version": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _check(status: int, handle=None):
    if status != MOE_OK:
        lib = load()
        raise MoEError(status, f"{lib.moe_status_string(status).decode()}: "
                               f"{lib.moe_last_error(handle).decode()}")


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


@dataclass(frozen=True)
class LayerConfig:
    hidden: int
    n_experts: int
    top_k: int
    expert_inter: int
    shared_inter: int
    dtype: str = "bf16"          # "bf16" or "f32"
    rms_eps: float = 1e-6


class MoELayer:
    """One sparse MoE FFN layer held by the CUDA library."""

    def __init__(self, cfg: LayerConfig, w_router, w_gate, w_up, w_down, ws_gate=None,
                 ws_up=None, ws_down=None, rms_weight=None, device: int | None = None,
                 max_tokens: int = 0):
        import torch
        self.lib = load()
        self.cfg = cfg
        self.device = w_router.device.index if device is None else device
        self.torch_dtype = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
        H, E, I, Is = cfg.hidden, cfg.n_experts, cfg.expert_inter, cfg.shared_inter
        want = {"w_router": (w_router, (E, H)), "w_gate": (w_gate, (E, I, H)),
                "w_up": (w_up, (E, I, H)), "w_down": (w_down, (E, H, I)),
                "ws_gate": (ws_gate, (Is, H)), "ws_up": (ws_up, (Is, H)),
                "ws_down": (ws_down, (H, Is)), "rms_weight": (rms_weight, (H,))}
        for name, (t, shape) in want.items():
            if t is None:
                if name.startswith("w_") or (name.startswith("ws_") and Is > 0):
                    raise ValueError(f"{name} is required")
                continue
            if not (t.is_cuda and t.is_contiguous() and t.dtype == self.torch_dtype and
                    tuple(t.shape) == shape):
                raise ValueError(f"{name} must be a contiguous {list(shape)} "
                                 f"{self.torch_dtype} CUDA tensor")
        c = _Config(cfg.hidden, cfg.n_experts, cfg.top_k, cfg.expert_inter, cfg.shared_inter,
                    DTYPE_BF16 if cfg.dtype == "bf16" else DTYPE_F32, 1, cfg.rms_eps)
        h = ctypes.c_void_p()
        torch.cuda.synchronize(self.device)
        _check(self.lib.moe_create(ctypes.byref(c), self.device, _ptr(w_router), _ptr(w_gate),
                                   _ptr(w_up), _ptr(w_down), _ptr(ws_gate), _ptr(ws_up),
                                   _ptr(ws_down), _ptr(rms_weight), ctypes.byref(h)))
        self.handle = h
        self.reserved = 0
        if max_tokens:
            self.reserve(max_tokens)

    @classmethod
    def from_numpy(cls, cfg: LayerConfig, arrays: dict, device: int = 0, max_tokens: int = 0):
        """Upload numpy weights (bf16 as uint16 bits, or float32) and create the layer."""
        ts = {k: to_device(v, device) for k, v in arrays.items() if v is not None}
        layer = cls(cfg, ts["w_router"], ts["w_gate"], ts["w_up"], ts["w_down"],
                    ts.get("ws_gate"), ts.get("ws_up"), ts.get("ws_down"), ts.get("rms_w"),
                    device=device, max_tokens=max_tokens)
        return layer       # the library keeps its own copies; ts may be freed

    def reserve(self, max_tokens: int):
        _check(self.lib.moe_reserve(self.handle, int(max_tokens)), self.handle)
        self.reserved = max(self.reserved, int(max_tokens))

    def _ensure(self, T: int):
        if T > self.reserved:
            self.reserve(T)

    def _check_tokens(self, x, **others):
        """x: a contiguous [T, hidden] tensor of the layer dtype on a CUDA device; each
        other tensor (residual, out) either None or of exactly x's shape, dtype, device
        and layout (the library reads and writes T x hidden elements through them)."""
        if not (x.is_cuda and x.is_contiguous() and x.dtype == self.torch_dtype and
                x.dim() == 2 and x.shape[1] == self.cfg.hidden):
            raise ValueError(f"x must be a contiguous [T, {self.cfg.hidden}] "
                             f"{self.torch_dtype} CUDA tensor")
        for name, t in others.items():
            if t is not None and not (t.shape == x.shape and t.dtype == x.dtype and
                                      t.device == x.device and t.is_contiguous()):
                raise ValueError(f"{name} must match x (shape, dtype, device, contiguous)")

    def route(self, x, stream=None):
        import torch
        self._check_tokens(x)
        T = x.shape[0]
        self._ensure(T)
        idx = torch.empty((T, self.cfg.top_k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, self.cfg.top_k), dtype=torch.float32, device=x.device)
        _check(self.lib.moe_route(self.handle, _ptr(x), T, _ptr(idx), _ptr(w), _stream(stream)),
               self.handle)
        return idx, w

    def forward(self, x, residual=None, out=None, return_routing=False, stream=None):
        import torch
        self._check_tokens(x, residual=residual, out=out)
        T = x.shape[0]
        self._ensure(T)
        y = torch.empty_like(x) if out is None else out
        idx = w = None
        if return_routing:
            idx = torch.empty((T, self.cfg.top_k), dtype=torch.int32, device=x.device)
            w = torch.empty((T, self.cfg.top_k), dtype=torch.float32, device=x.device)
        _check(self.lib.moe_forward(self.handle, _ptr(x), _ptr(residual), _ptr(y), T, _ptr(idx),
                                    _ptr(w), _stream(stream)), self.handle)
        return (y, idx, w) if return_routing else y

    def forward_host(self, x_host, y_host, residual_host=None, stream=None):
        """x_host / y_host: (pinned) CPU tensors [T, H]; synchronous."""
        for name, t in (("x_host", x_host), ("y_host", y_host), ("residual_host", residual_host)):
            if t is not None and not (not t.is_cuda and t.is_contiguous() and
                                      t.dtype == self.torch_dtype and t.dim() == 2 and
                                      t.shape == x_host.shape and
                                      t.shape[1] == self.cfg.hidden):
                raise ValueError(f"{name} must be a contiguous [T, {self.cfg.hidden}] "
                                 f"{self.torch_dtype} host tensor shaped like x_host")
        T = x_host.shape[0]
        self._ensure(T)
        _check(self.lib.moe_forward_host(self.handle, _ptr(x_host), _ptr(residual_host),
                                         _ptr(y_host), T, _stream(stream)), self.handle)
        return y_host

    def last_routing(self, T: int, stream=None):
        E, k = self.cfg.n_experts, self.cfg.top_k
        counts = np.zeros(E, np.int32)
        offsets = np.zeros(E + 1, np.int32)
        slots = np.zeros((T, k), np.int32)
        _check(self.lib.moe_last_routing(self.handle, counts.ctypes.data, offsets.ctypes.data,
                                         slots.ctypes.data, _stream(stream)), self.handle)
        return counts, offsets, slots

    def check(self, stream=None) -> int:
        """Synchronise; returns the device-side status code (0 = ok) and clears it."""
        return int(self.lib.moe_check(self.handle, _stream(stream)))

    def set_option(self, name: str, value: int):
        _check(self.lib.moe_set_option(self.handle, OPTIONS[name], int(value)), self.handle)

    def kernel_stats(self, reset: bool = False) -> dict:
        """{class: (launches, total_ms)} since the last reset (synchronises the device)."""
        n = len(KERNEL_CLASSES)
        ms = np.zeros(n, np.float64)
        cnt = np.zeros(n, np.int64)
        _check(self.lib.moe_kernel_stats(self.handle, ms.ctypes.data, cnt.ctypes.data,
                                         int(reset)), self.handle)
        return {c: (int(cnt[i]), float(ms[i])) for i, c in enumerate(KERNEL_CLASSES)}

    def close(self):
        if getattr(self, "handle", None):
            self.lib.moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def to_device(a: np.ndarray, device: int = 0):
    """numpy (bf16 bits as uint16, or float32) -> torch CUDA tensor of the same values."""
    import torch
    if a.dtype == np.uint16:
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(f"cuda:{device}")


def to_numpy(t) -> np.ndarray:
    """torch tensor (bf16 or float32) -> numpy (bf16 bits as uint16, or float32)."""
    import torch
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def version() -> str:
    return load().moe_version().decode()
