"""Muon optimizer step on B200 (sm_100a): Python binding of the C ABI in
``include/muon.h``.

This module only marshals arguments (device pointers, shapes, the current
CUDA stream) into the shared library ``libmuon_b200.so``; every step of the
computation runs in the library's CUDA kernels.  If the library is missing,
every entry point raises: there is no fallback.

The update (Modded-NanoGPT article, "Muon optimizer" section): Nesterov
momentum ``buf <- mu*buf + g``, ``G = g + mu*buf``; orthogonalisation by the
zeroth_power_via_newtonschulz5 quintic iteration in bf16; ``W <- W - lr*O``.
"""

from __future__ import annotations

import ctypes
import os
import re

__all__ = [
    "step", "orthogonalize", "step_host", "step_noalloc", "workspace_size", "sync_status", "last_error", "release",
    "profile_enable", "profile_read", "launch_count", "debug_set", "lib", "MuonError", "KINDS",
    "NS_A", "NS_B", "NS_C", "NS_STEPS", "NS_EPS", "LIB_PATH", "header_functions",
]

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmuon_b200.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "muon.h")

NS_A, NS_B, NS_C, NS_STEPS, NS_EPS = 3.4445, -4.7750, 2.0315, 5, 1e-7
KINDS = ("prologue", "gram", "poly", "update", "update_apply", "apply_x0", "small")

STATUS = {0: "MUON_OK", -1: "MUON_ERR_INVALID_ARG", -2: "MUON_ERR_SHAPE", -3: "MUON_ERR_CUDA",
          -4: "MUON_ERR_NOMEM", -5: "MUON_ERR_TIMEOUT", -6: "MUON_ERR_DEVICE", -7: "MUON_ERR_UNSUPPORTED"}


class MuonError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


_lib = None
_P = ctypes.c_void_p
_PP = ctypes.POINTER(ctypes.c_void_p)
_I64P = ctypes.POINTER(ctypes.c_int64)


def header_functions() -> list:
    """Names of the functions declared in include/muon.h."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:int|size_t|void|int64_t|const char\*)\s+\**(muon_\w+)\s*\(", text, flags=re.M)


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                           "`python -m muon_newton_schulz_02_b200.build` (no CPU fallback exists)")
    L = ctypes.CDLL(LIB_PATH)
    step_args = [_PP, _PP, _PP, _I64P, ctypes.c_int, ctypes.c_float, ctypes.c_float, ctypes.c_int]
    L.muon_step.argtypes = step_args + [_P]
    L.muon_step.restype = ctypes.c_int
    L.muon_step_ex.argtypes = step_args + [ctypes.c_float] * 4 + [ctypes.c_int, _P]
    L.muon_step_ex.restype = ctypes.c_int
    L.muon_step_host.argtypes = step_args + [_P]
    L.muon_step_host.restype = ctypes.c_int
    L.muon_step_noalloc.argtypes = step_args + [_P]
    L.muon_step_noalloc.restype = ctypes.c_int
    L.muon_orthogonalize.argtypes = [_PP, _PP, _I64P, ctypes.c_int, ctypes.c_int, _P]
    L.muon_orthogonalize.restype = ctypes.c_int
    L.muon_workspace_size.argtypes = [_I64P, ctypes.c_int]
    L.muon_workspace_size.restype = ctypes.c_size_t
    L.muon_sync_status.argtypes = [_P]
    L.muon_sync_status.restype = ctypes.c_int
    L.muon_last_error.argtypes = []
    L.muon_last_error.restype = ctypes.c_char_p
    L.muon_release.argtypes = []
    L.muon_release.restype = None
    L.muon_profile_enable.argtypes = [ctypes.c_int]
    L.muon_profile_enable.restype = ctypes.c_int
    L.muon_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double), _I64P, ctypes.c_int]
    L.muon_profile_read.restype = ctypes.c_int
    L.muon_launch_count.argtypes = []
    L.muon_launch_count.restype = ctypes.c_int64
    L.muon_debug_set.argtypes = [ctypes.c_int, ctypes.c_int64]
    L.muon_debug_set.restype = ctypes.c_int
    _lib = L
    return L


def last_error() -> str:
    return lib().muon_last_error().decode()


def _check(rc: int):
    if rc != 0:
        raise MuonError(rc, last_error())


def _ptrs(xs):
    return (ctypes.c_void_p * len(xs))(*[ctypes.c_void_p(p) for p in xs])


def _shapes(shapes):
    flat = [int(v) for s in shapes for v in s]
    return (ctypes.c_int64 * len(flat))(*flat)


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    if hasattr(stream, "cuda_stream"):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


def _check_tensors(name, ts, device_kind="cuda"):
    import torch
    for i, t in enumerate(ts):
        if t.dim() != 2:
            raise ValueError(f"{name}[{i}] must be 2-D (the method is defined for matrices)")
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{name}[{i}] must be contiguous float32")
        if t.device.type != device_kind:
            raise ValueError(f"{name}[{i}] must live on {device_kind}")


def step(params, grads, bufs, lr: float, mu: float, ns_steps: int = NS_STEPS, *, a: float = NS_A,
         b: float = NS_B, c: float = NS_C, eps: float = NS_EPS, nesterov: bool = True, stream=None):
    """One Muon step, in place on ``params`` and ``bufs`` (lists of CUDA fp32 matrices)."""
    n = len(params)
    if not (len(grads) == n == len(bufs)) or n == 0:
        raise ValueError("params, grads and bufs must be equally long, non-empty lists")
    for name, ts in (("params", params), ("grads", grads), ("bufs", bufs)):
        _check_tensors(name, ts)
    for i in range(n):
        if not (params[i].shape == grads[i].shape == bufs[i].shape):
            raise ValueError(f"matrix {i}: params, grads and bufs shapes differ")
    L = lib()
    rc = L.muon_step_ex(_ptrs([t.data_ptr() for t in params]), _ptrs([t.data_ptr() for t in grads]),
                        _ptrs([t.data_ptr() for t in bufs]), _shapes([t.shape for t in params]), n,
                        float(lr), float(mu), int(ns_steps), float(a), float(b), float(c), float(eps),
                        1 if nesterov else 0, _stream(stream))
    _check(rc)


def orthogonalize(G, O=None, ns_steps: int = NS_STEPS, stream=None):
    """O_i = NS5(G_i) for a list of CUDA fp32 matrices; returns the list O."""
    import torch
    _check_tensors("G", G)
    if O is None:
        O = [torch.empty_like(g) for g in G]
    _check_tensors("O", O)
    rc = lib().muon_orthogonalize(_ptrs([t.data_ptr() for t in G]), _ptrs([t.data_ptr() for t in O]),
                                  _shapes([t.shape for t in G]), len(G), int(ns_steps), _stream(stream))
    _check(rc)
    return O


def step_host(params, grads, bufs, lr: float, mu: float, ns_steps: int = NS_STEPS, stream=None):
    """Muon step on host (CPU, ideally pinned) fp32 matrices; blocks until done."""
    for name, ts in (("params", params), ("grads", grads), ("bufs", bufs)):
        _check_tensors(name, ts, device_kind="cpu")
    rc = lib().muon_step_host(_ptrs([t.data_ptr() for t in params]), _ptrs([t.data_ptr() for t in grads]),
                              _ptrs([t.data_ptr() for t in bufs]), _shapes([t.shape for t in params]),
                              len(params), float(lr), float(mu), int(ns_steps), _stream(stream))
    _check(rc)


def step_noalloc(params, grads, bufs, lr: float, mu: float, ns_steps: int = NS_STEPS, stream=None):
    """muon_step for callers that cannot allocate device memory: the library's
    scratch is a fixed 64 MiB static device array instead of cudaMalloc'd
    workspace (see include/muon.h for the limits)."""
    for name, ts in (("params", params), ("grads", grads), ("bufs", bufs)):
        _check_tensors(name, ts)
    rc = lib().muon_step_noalloc(_ptrs([t.data_ptr() for t in params]), _ptrs([t.data_ptr() for t in grads]),
                                 _ptrs([t.data_ptr() for t in bufs]), _shapes([t.shape for t in params]),
                                 len(params), float(lr), float(mu), int(ns_steps), _stream(stream))
    _check(rc)


def workspace_size(shapes) -> int:
    return int(lib().muon_workspace_size(_shapes(shapes), len(shapes)))


def sync_status(stream=None) -> int:
    return int(lib().muon_sync_status(_stream(stream)))


def release():
    lib().muon_release()


def profile_enable(flag: bool = True):
    _check(lib().muon_profile_enable(1 if flag else 0))


def profile_read() -> dict:
    """{kind: (total_ms, launches)} accumulated since the last read."""
    ms = (ctypes.c_double * len(KINDS))()
    cnt = (ctypes.c_int64 * len(KINDS))()
    _check(lib().muon_profile_read(ms, cnt, len(KINDS)))
    return {k: (ms[i], cnt[i]) for i, k in enumerate(KINDS)}


def launch_count() -> int:
    return int(lib().muon_launch_count())


def debug_set(flags: int = 0, wait_limit_ns: int = 0):
    _check(lib().muon_debug_set(int(flags), int(wait_limit_ns)))
