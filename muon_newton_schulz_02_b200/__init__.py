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
from array import array

__all__ = [
    "step", "PreparedStep", "orthogonalize", "step_host", "step_noalloc", "workspace_size", "sync_status", "last_error", "release",
    "profile_enable", "profile_read", "launch_count", "chain_clusters", "debug_set", "guard_check", "chain_plan", "lib",
    "MuonError", "KINDS",
    "update_bf16", "apply_bf16",
    "NS_A", "NS_B", "NS_C", "NS_STEPS", "NS_EPS", "LIB_PATH", "DEBUG_LIB_PATH", "header_functions",
]

HERE = os.path.dirname(os.path.abspath(__file__))
# the same library with device bounds checks compiled in (tests and debugging):
# MUON_BOUNDS_CHECKS=1 in the environment, or LIB_PATH set to it before the first call
DEBUG_LIB_PATH = os.path.join(HERE, "libmuon_b200_debug.so")
LIB_PATH = DEBUG_LIB_PATH if os.environ.get("MUON_BOUNDS_CHECKS") == "1" else os.path.join(HERE, "libmuon_b200.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "muon.h")

NS_A, NS_B, NS_C, NS_STEPS, NS_EPS = 3.4445, -4.7750, 2.0315, 5, 1e-7
KINDS = ("prologue", "gram", "poly", "update", "update_apply", "apply_x0", "small", "pair", "chain", "o16", "quad")

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
    L.muon_step_fp8.argtypes = step_args + [ctypes.c_float] * 4 + [ctypes.c_int, ctypes.c_int, _P]
    L.muon_step_fp8.restype = ctypes.c_int
    L.muon_step_host.argtypes = step_args + [_P]
    L.muon_step_host.restype = ctypes.c_int
    L.muon_step_noalloc.argtypes = step_args + [_P]
    L.muon_step_noalloc.restype = ctypes.c_int
    L.muon_update_bf16.argtypes = [_PP, _PP, _PP, _I64P, ctypes.c_int, ctypes.c_float, ctypes.c_int] + \
        [ctypes.c_float] * 4 + [ctypes.c_int, _P]
    L.muon_update_bf16.restype = ctypes.c_int
    L.muon_apply_bf16.argtypes = [_PP, _PP, _I64P, ctypes.c_int, ctypes.c_float, _P]
    L.muon_apply_bf16.restype = ctypes.c_int
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
    L.muon_chain_clusters.argtypes = []
    L.muon_chain_clusters.restype = ctypes.c_int
    L.muon_debug_set.argtypes = [ctypes.c_int, ctypes.c_int64]
    L.muon_debug_set.restype = ctypes.c_int
    L.muon_guard_check.argtypes = [ctypes.c_void_p]
    L.muon_guard_check.restype = ctypes.c_int
    L.muon_chain_plan.argtypes = [_I64P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int32),
                                  ctypes.c_int64, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64)]
    L.muon_chain_plan.restype = ctypes.c_int
    _lib = L
    return L


def last_error() -> str:
    return lib().muon_last_error().decode()


def _check(rc: int):
    if rc != 0:
        raise MuonError(rc, last_error())


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


def _bad(name, i, t, device_kind, dtype=None):
    """The error for a tensor that failed the quick check (slow path, only on failure)."""
    import torch
    dtype = dtype or torch.float32
    if t.dim() != 2:
        return ValueError(f"{name}[{i}] must be 2-D (the method is defined for matrices)")
    if t.dtype != dtype or not t.is_contiguous():
        return ValueError(f"{name}[{i}] must be contiguous {str(dtype).replace('torch.', '')}")
    return ValueError(f"{name}[{i}] must live on {device_kind}")


def _marshal(name, ts, device_kind="cuda", shapes=None, dtype=None):
    """One pass over a tensor list: checks (2-D, contiguous, of `dtype` --
    fp32 by default -- on the device kind -- for CUDA, the current device,
    where the library launches -- and equal shapes to `shapes` when given)
    and returns (pointer array, list of shapes).  The arrays are ctypes
    views of array('q') buffers."""
    import torch
    f32, on_cuda = dtype or torch.float32, device_kind == "cuda"
    dev = None
    ptrs, shp = array("q"), []
    for i, t in enumerate(ts):
        if t.dtype is not f32 or t.is_cuda is not on_cuda or not t.is_contiguous() or t.dim() != 2:
            raise _bad(name, i, t, device_kind, f32)
        if on_cuda:
            if dev is None:
                dev = torch.cuda.current_device()
            if t.get_device() != dev:
                raise ValueError(f"{name}[{i}] is on cuda:{t.get_device()} but the current device is cuda:{dev}")
        sz = t.shape
        if shapes is not None and sz != shapes[i]:
            raise ValueError(f"matrix {i}: params, grads and bufs shapes differ")
        shp.append(sz)
        ptrs.append(t.data_ptr())
    return (ctypes.c_void_p * len(ptrs)).from_buffer(ptrs), shp


def _shape_array(shp):
    flat = array("q")
    for r, c in shp:
        flat.append(r)
        flat.append(c)
    return (ctypes.c_int64 * len(flat)).from_buffer(flat)


def _marshal_step(params, grads, bufs, device_kind="cuda"):
    n = len(params)
    if not (len(grads) == n == len(bufs)) or n == 0:
        raise ValueError("params, grads and bufs must be equally long, non-empty lists")
    pp, shp = _marshal("params", params, device_kind)
    gp, _ = _marshal("grads", grads, device_kind, shp)
    bp, _ = _marshal("bufs", bufs, device_kind, shp)
    return pp, gp, bp, _shape_array(shp), n


def step(params, grads, bufs, lr: float, mu: float, ns_steps: int = NS_STEPS, *, a: float = NS_A,
         b: float = NS_B, c: float = NS_C, eps: float = NS_EPS, nesterov: bool = True, fp8_iters: int = 0,
         stream=None):
    """One Muon step, in place on ``params`` and ``bufs`` (lists of CUDA fp32 matrices).
    ``fp8_iters`` > 0 selects the reduced-precision variant ``muon_step_fp8``
    (e4m3 operands in the first one or two iterations)."""
    pp, gp, bp, sh, n = _marshal_step(params, grads, bufs)
    if fp8_iters:
        rc = lib().muon_step_fp8(pp, gp, bp, sh, n, float(lr), float(mu), int(ns_steps), float(a), float(b),
                                 float(c), float(eps), 1 if nesterov else 0, int(fp8_iters), _stream(stream))
    else:
        rc = lib().muon_step_ex(pp, gp, bp, sh, n, float(lr), float(mu), int(ns_steps), float(a), float(b),
                                float(c), float(eps), 1 if nesterov else 0, _stream(stream))
    _check(rc)


class PreparedStep:
    """A Muon step bound to fixed ``params`` and ``bufs`` (the usual training
    loop: the same weight and momentum tensors every step).  Their checks and
    pointer arrays are built once; each call checks and marshals only the
    gradients, then makes the same library call as :func:`step`.
    The bound tensors must keep their storage (no re-allocation) while the
    object is in use."""

    def __init__(self, params, bufs, lr: float, mu: float, ns_steps: int = NS_STEPS, *, a: float = NS_A,
                 b: float = NS_B, c: float = NS_C, eps: float = NS_EPS, nesterov: bool = True, fp8_iters: int = 0):
        n = len(params)
        if len(bufs) != n or n == 0:
            raise ValueError("params and bufs must be equally long, non-empty lists")
        self._pp, self._shp = _marshal("params", params)
        self._bp, _ = _marshal("bufs", bufs, shapes=self._shp)
        self._sh = _shape_array(self._shp)
        self._keep = (list(params), list(bufs))
        self.n = n
        self.lr, self.mu, self.ns_steps = float(lr), float(mu), int(ns_steps)
        self._abc = (float(a), float(b), float(c), float(eps), 1 if nesterov else 0)
        self.fp8_iters = int(fp8_iters)

    def __call__(self, grads, lr: float = None, stream=None):
        if len(grads) != self.n:
            raise ValueError("params, grads and bufs must be equally long, non-empty lists")
        gp, _ = _marshal("grads", grads, shapes=self._shp)
        lr = self.lr if lr is None else float(lr)
        if self.fp8_iters:
            rc = lib().muon_step_fp8(self._pp, gp, self._bp, self._sh, self.n, lr, self.mu, self.ns_steps,
                                     *self._abc, self.fp8_iters, _stream(stream))
        else:
            rc = lib().muon_step_ex(self._pp, gp, self._bp, self._sh, self.n, lr, self.mu, self.ns_steps,
                                    *self._abc, _stream(stream))
        _check(rc)


def update_bf16(grads, bufs, mu: float, ns_steps: int = NS_STEPS, O=None, *, a: float = NS_A, b: float = NS_B,
                c: float = NS_C, eps: float = NS_EPS, nesterov: bool = True, stream=None):
    """Momentum and NS5 without the weight update: returns the orthogonalised
    updates O_i as CUDA bfloat16 matrices (written into ``O`` when given) and
    updates ``bufs`` in place.  With :func:`apply_bf16`, the two halves of a
    step whose update is exchanged in bf16 between data-parallel ranks."""
    import torch
    n = len(grads)
    if len(bufs) != n or n == 0:
        raise ValueError("grads and bufs must be equally long, non-empty lists")
    gp, shp = _marshal("grads", grads)
    bp, _ = _marshal("bufs", bufs, shapes=shp)
    if O is None:
        O = [torch.empty(s, dtype=torch.bfloat16, device=g.device) for s, g in zip(shp, grads)]
    if len(O) != n:
        raise ValueError("O must have one matrix per gradient")
    op, _ = _marshal("O", O, shapes=shp, dtype=torch.bfloat16)
    rc = lib().muon_update_bf16(gp, bp, op, _shape_array(shp), n, float(mu), int(ns_steps), float(a), float(b),
                                float(c), float(eps), 1 if nesterov else 0, _stream(stream))
    _check(rc)
    return O


def apply_bf16(params, O, lr: float, stream=None):
    """W_i -= lr * O_i for CUDA fp32 ``params`` and bfloat16 ``O`` (in place)."""
    import torch
    if len(params) != len(O) or not params:
        raise ValueError("params and O must be equally long, non-empty lists")
    pp, shp = _marshal("params", params)
    op, _ = _marshal("O", O, shapes=shp, dtype=torch.bfloat16)
    _check(lib().muon_apply_bf16(pp, op, _shape_array(shp), len(params), float(lr), _stream(stream)))


def orthogonalize(G, O=None, ns_steps: int = NS_STEPS, stream=None):
    """O_i = NS5(G_i) for a list of CUDA fp32 matrices; returns the list O."""
    import torch
    gp, shp = _marshal("G", G)
    if O is None:
        O = [torch.empty_like(g) for g in G]
    if len(O) != len(G):
        raise ValueError("G and O must be equally long lists")
    op, _ = _marshal("O", O, shapes=shp)
    rc = lib().muon_orthogonalize(gp, op, _shape_array(shp), len(G), int(ns_steps), _stream(stream))
    _check(rc)
    return O


def step_host(params, grads, bufs, lr: float, mu: float, ns_steps: int = NS_STEPS, stream=None):
    """Muon step on host (CPU, ideally pinned) fp32 matrices; blocks until done."""
    pp, gp, bp, sh, n = _marshal_step(params, grads, bufs, device_kind="cpu")
    rc = lib().muon_step_host(pp, gp, bp, sh, n, float(lr), float(mu), int(ns_steps), _stream(stream))
    _check(rc)


def step_noalloc(params, grads, bufs, lr: float, mu: float, ns_steps: int = NS_STEPS, stream=None):
    """muon_step for callers that cannot allocate device memory: the library's
    scratch is a fixed 64 MiB static device array instead of cudaMalloc'd
    workspace (see include/muon.h for the limits)."""
    pp, gp, bp, sh, n = _marshal_step(params, grads, bufs)
    rc = lib().muon_step_noalloc(pp, gp, bp, sh, n, float(lr), float(mu), int(ns_steps), _stream(stream))
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


def chain_clusters() -> int:
    """Clusters of two CTAs the chained launch uses on the current device."""
    return int(lib().muon_chain_clusters())


def debug_set(flags: int = 0, wait_limit_ns: int = 0):
    _check(lib().muon_debug_set(int(flags), int(wait_limit_ns)))


def guard_check(stream=None) -> int:
    """Guard-band bytes of the last group run on the stream that a launch
    changed (0: none); raises MuonError when the library was loaded without
    MUON_GUARD_BANDS=1."""
    rc = lib().muon_guard_check(_stream(stream))
    if rc < 0:
        _check(rc)
    return rc


def chain_plan(shapes, ns_steps: int = NS_STEPS, nclusters: int = 74):
    """The chained launch's work lists for these shapes (host only): returns
    (items, cluster_off) with items a list of (need, matrix, class, index,
    tile row, tile column, phase, iteration) tuples."""
    sh = _shapes(shapes)
    off = (ctypes.c_int32 * (nclusters + 1))()
    cnt = ctypes.c_int64(0)
    rc = lib().muon_chain_plan(sh, len(shapes), int(ns_steps), int(nclusters), None, 0, off, ctypes.byref(cnt))
    if rc not in (0, -1):
        _check(rc)
    buf = (ctypes.c_int32 * (8 * max(1, cnt.value)))()
    _check(lib().muon_chain_plan(sh, len(shapes), int(ns_steps), int(nclusters), buf, cnt.value, off,
                                 ctypes.byref(cnt)))
    items = [tuple(buf[8 * i:8 * i + 8]) for i in range(cnt.value)]
    return items, list(off)
