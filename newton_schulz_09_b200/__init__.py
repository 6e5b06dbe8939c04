"""B200-native (sm_100a) batched Muon update: momentum, Nesterov, Frobenius
normalisation, cubic Newton-Schulz and the decoupled weight update, done by
hand-written tcgen05/TMA kernels behind the C ABI of ``include/dmuon.h``.

This module is argument marshalling only: it passes tensor addresses, shapes
and the current CUDA stream to ``libdmuon.so``.  Every step of the update
runs in that library; there is no Python or CPU fallback, and the functions
raise if the library or a CUDA device is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "DMUON_F32", "DMUON_BF16", "DmuonError", "load_library", "library_path",
    "dmuon_ns_orthogonalize", "dmuon_ns_orthogonalize_ex", "dmuon_ns_workspace_bytes",
    "dmuon_muon_step_batched", "dmuon_muon_step_batched_ex", "dmuon_workspace_bytes",
    "dmuon_last_error", "dmuon_backend_string", "dmuon_device_status", "dmuon_release_cache",
    "dmuon_debug_fail_allocations", "dmuon_debug_wait_timeout", "dmuon_stage_timing",
    "dmuon_stage_times", "dmuon_launch_count", "KERNEL_KINDS", "dmuon_ns_orthogonalize_noalloc",
    "dmuon_plan_builds", "dmuon_debug_check_pointer", "dmuon_debug_last_plan",
    "dmuon_muon_step_batched_opts", "DmuonStepOptions", "DMUON_LR_PLAIN", "DMUON_LR_SQRT_MAX",
    "dmuon_adamw_step_batched", "DmuonTensorDesc", "dmuon_muon_step_batched_host",
    "dmuon_muon_step_batched_reduce", "dmuon_clip_grad_norm_buckets", "dmuon_clip_workspace_bytes",
    "DmuonGradDesc", "DMUON_MAX_CHUNKS", "DMUON_MAX_SEGMENTS",
]

#: Kernel kinds of dmuon_stage_times(), in order.
KERNEL_KINDS = ("prologue", "finalize", "syrk", "gemm", "apply", "adamw", "clip", "square")

DMUON_F32 = 0
DMUON_BF16 = 1
ERRORS = {0: "DMUON_OK", -1: "DMUON_ERR_INVALID_ARG", -2: "DMUON_ERR_UNSUPPORTED",
          -3: "DMUON_ERR_NO_WORKSPACE", -4: "DMUON_ERR_CUDA", -5: "DMUON_ERR_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libdmuon.so")
_lib = None


class DmuonError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


class DmuonShape(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("param_dtype", ctypes.c_int32), ("grad_dtype", ctypes.c_int32)]


DMUON_LR_PLAIN = 0
DMUON_LR_SQRT_MAX = 1
DMUON_MAX_CHUNKS = 32
DMUON_MAX_SEGMENTS = 64


class DmuonGradDesc(ctypes.Structure):
    _fields_ = [("numel", ctypes.c_int64), ("dtype", ctypes.c_int32), ("segment", ctypes.c_int32)]


class DmuonTensorDesc(ctypes.Structure):
    _fields_ = [("numel", ctypes.c_int64), ("param_dtype", ctypes.c_int32),
                ("grad_dtype", ctypes.c_int32)]


class DmuonStepOptions(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_size_t), ("lr", ctypes.c_float),
                ("momentum", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("nesterov", ctypes.c_int), ("ns_steps", ctypes.c_int),
                ("ns_a", ctypes.c_float), ("ns_b", ctypes.c_float), ("lr_scale", ctypes.c_int),
                ("max_grad_norm", ctypes.c_float), ("grad_norm_out", ctypes.c_void_p),
                ("ns_c", ctypes.c_float)]


def _set_coefficients(o: "DmuonStepOptions", coeffs) -> None:
    """(a, b): the cubic step; (a, b, c): the quintic step."""
    if len(coeffs) == 2:
        o.ns_a, o.ns_b = coeffs
        o.ns_c = 0.0
    elif len(coeffs) == 3:
        o.ns_a, o.ns_b, o.ns_c = coeffs
    else:
        raise ValueError("ns_coefficients must be (a, b) or (a, b, c)")


def library_path() -> str:
    return _LIB_PATH


def load_library() -> ctypes.CDLL:
    """Loads libdmuon.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m newton_schulz_09_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i64, i32, f32, sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                             ctypes.c_float, ctypes.c_size_t)
    pp = ctypes.POINTER(ctypes.c_void_p)
    sp = ctypes.POINTER(DmuonShape)
    sig = {
        "dmuon_ns_orthogonalize": (i32, [vp, i64, i64, i32, vp]),
        "dmuon_ns_orthogonalize_ex": (i32, [vp, i64, i64, i32, i32, vp, sz, vp]),
        "dmuon_ns_workspace_bytes": (sz, [i64, i64, i32]),
        "dmuon_muon_step_batched": (i32, [pp, pp, pp, sp, i32, f32, f32, i32, f32, i32, vp]),
        "dmuon_muon_step_batched_ex": (i32, [pp, pp, pp, sp, i32, f32, f32, i32, f32, i32, vp, sz, vp]),
        "dmuon_workspace_bytes": (sz, [sp, i32, i32]),
        "dmuon_last_error": (ctypes.c_char_p, []),
        "dmuon_backend_string": (ctypes.c_char_p, []),
        "dmuon_device_status": (i32, [i32]),
        "dmuon_release_cache": (None, []),
        "dmuon_debug_fail_allocations": (None, [i32]),
        "dmuon_debug_wait_timeout": (i32, [i32, vp]),
        "dmuon_stage_timing": (i32, [i32]),
        "dmuon_stage_times": (i32, [ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(ctypes.c_int64), i32, i32]),
        "dmuon_launch_count": (ctypes.c_int64, []),
        "dmuon_ns_orthogonalize_noalloc": (i32, [vp, i64, i64, i32, vp]),
        "dmuon_step_options_default": (None, [ctypes.POINTER(DmuonStepOptions)]),
        "dmuon_adamw_step_batched": (i32, [pp, pp, pp, pp, ctypes.POINTER(DmuonTensorDesc), i32,
                                           f32, f32, f32, f32, f32, i64, vp]),
        "dmuon_muon_step_batched_opts": (i32, [pp, pp, pp, sp, i32, ctypes.POINTER(DmuonStepOptions),
                                               vp, sz, vp]),
        "dmuon_muon_step_batched_host": (i32, [pp, pp, pp, pp, pp, sp, i32,
                                               ctypes.POINTER(DmuonStepOptions), i32, vp, sz, vp]),
        "dmuon_debug_partition": (i32, [sp, i32, i32, ctypes.POINTER(ctypes.c_int), i32]),
        "dmuon_muon_step_batched_reduce": (i32, [pp, pp, pp, sp, i32, i32, ctypes.POINTER(DmuonStepOptions),
                                                 vp, sz, vp]),
        "dmuon_clip_workspace_bytes": (sz, [ctypes.POINTER(DmuonGradDesc), i32, i32]),
        "dmuon_workspace_bytes_opts": (sz, [sp, i32, ctypes.POINTER(DmuonStepOptions)]),
        "dmuon_plan_builds": (ctypes.c_int64, []),
        "dmuon_debug_check_pointer": (i32, [vp]),
        "dmuon_debug_last_plan": (i32, [ctypes.POINTER(i32), i32]),
        "dmuon_clip_grad_norm_buckets": (i32, [pp, ctypes.POINTER(DmuonGradDesc), i32,
                                               ctypes.POINTER(ctypes.c_float), i32, vp, vp, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(code: int) -> None:
    if code != 0:
        raise DmuonError(code, load_library().dmuon_last_error().decode())


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return DMUON_BF16
    if t == torch.float32:
        return DMUON_F32
    raise TypeError(f"unsupported dtype {t}; use torch.bfloat16 or torch.float32")


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _cuda_matrix(t: torch.Tensor, what: str) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if t.dim() != 2:
        raise ValueError(f"{what} must be 2-D (the Muon path is for matrices)")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous (row-major)")


def _workspace(workspace: Optional[torch.Tensor], device: torch.device):
    """(address, bytes) of a caller's scratch tensor, (None, 0) without one.
    The scratch must be contiguous device memory on the matrices' device: a
    host tensor's address would be written by the kernels."""
    if workspace is None:
        return None, 0
    if (not isinstance(workspace, torch.Tensor) or not workspace.is_cuda
            or workspace.device != device or not workspace.is_contiguous()):
        raise ValueError(f"workspace must be a contiguous CUDA tensor on {device}")
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


# ---------------------------------------------------------------- orthogonalise
def dmuon_ns_workspace_bytes(m: int, n: int, dtype: torch.dtype = torch.bfloat16) -> int:
    return int(load_library().dmuon_ns_workspace_bytes(m, n, _dtype_code(dtype)))


def dmuon_ns_orthogonalize(X: torch.Tensor, steps: int = 5) -> torch.Tensor:
    """In-place cubic Newton-Schulz of one bf16 matrix with library-owned scratch."""
    lib = load_library()
    _cuda_matrix(X, "X")
    if X.dtype != torch.bfloat16:
        raise TypeError("dmuon_ns_orthogonalize takes bf16; use dmuon_ns_orthogonalize_ex for fp32")
    with torch.cuda.device(X.device):
        _check(lib.dmuon_ns_orthogonalize(X.data_ptr(), X.shape[0], X.shape[1], steps,
                                          _stream(X.device)))
    return X


def dmuon_ns_orthogonalize_ex(X: torch.Tensor, steps: int = 5,
                              workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """In-place cubic Newton-Schulz of one bf16 or fp32 matrix; scratch comes
    from ``workspace`` or from PyTorch's allocator."""
    lib = load_library()
    _cuda_matrix(X, "X")
    dt = _dtype_code(X.dtype)
    need = int(lib.dmuon_ns_workspace_bytes(X.shape[0], X.shape[1], dt))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    ws_ptr, ws_bytes = _workspace(workspace, X.device)
    with torch.cuda.device(X.device):
        _check(lib.dmuon_ns_orthogonalize_ex(X.data_ptr(), X.shape[0], X.shape[1], steps, dt,
                                             ws_ptr, ws_bytes, _stream(X.device)))
    return X


# ---------------------------------------------------------------- Muon step
class _Batch:
    """ctypes arrays describing a list of matrices."""

    def __init__(self, params, grads, bufs):
        n = len(params)
        if len(grads) != n or len(bufs) != n:
            raise ValueError("params, grads and bufs must have the same length")
        self.n = n
        self.P = (ctypes.c_void_p * max(n, 1))()
        self.G = (ctypes.c_void_p * max(n, 1))()
        self.B = (ctypes.c_void_p * max(n, 1))()
        self.S = (DmuonShape * max(n, 1))()
        dev = None
        for i, (p, g, b) in enumerate(zip(params, grads, bufs)):
            _cuda_matrix(p, f"params[{i}]")
            _cuda_matrix(b, f"bufs[{i}]")
            if b.dtype != torch.float32 or b.shape != p.shape:
                raise ValueError(f"bufs[{i}] must be fp32 with the parameter's shape")
            if g is not None:
                _cuda_matrix(g, f"grads[{i}]")
                if g.shape != p.shape:
                    raise ValueError(f"grads[{i}] must have the parameter's shape")
            dev = dev or p.device
            for t in (p, b) + ((g,) if g is not None else ()):
                if t.device != dev:
                    raise ValueError("all tensors must be on one device")
            self.P[i] = p.data_ptr()
            self.G[i] = g.data_ptr() if g is not None else None
            self.B[i] = b.data_ptr()
            gd = _dtype_code(g.dtype) if g is not None else _dtype_code(p.dtype)
            self.S[i] = DmuonShape(p.shape[0], p.shape[1], _dtype_code(p.dtype), gd)
        self.device = dev

    def args(self):
        pp = ctypes.POINTER(ctypes.c_void_p)
        return (ctypes.cast(self.P, pp), ctypes.cast(self.G, pp), ctypes.cast(self.B, pp),
                ctypes.cast(self.S, ctypes.POINTER(DmuonShape)), self.n)


def dmuon_workspace_bytes(params: Sequence[torch.Tensor], ns_steps: int = 5,
                          grads: Optional[Sequence[Optional[torch.Tensor]]] = None) -> int:
    lib = load_library()
    n = len(params)
    S = (DmuonShape * max(n, 1))()
    for i, p in enumerate(params):
        g = grads[i] if grads is not None else None
        gd = _dtype_code(g.dtype) if g is not None else _dtype_code(p.dtype)
        S[i] = DmuonShape(p.shape[0], p.shape[1], _dtype_code(p.dtype), gd)
    return int(lib.dmuon_workspace_bytes(S, n, ns_steps))


def dmuon_muon_step_batched(params, grads, bufs, lr: float = 0.02, momentum: float = 0.95,
                            nesterov: bool = True, weight_decay: float = 0.0,
                            ns_steps: int = 5) -> None:
    """One Muon update of all matrices, scratch from the library's arena."""
    lib = load_library()
    b = _Batch(params, grads, bufs)
    if b.n == 0:
        return
    with torch.cuda.device(b.device):
        _check(lib.dmuon_muon_step_batched(*b.args(), lr, momentum, 1 if nesterov else 0,
                                           weight_decay, ns_steps, _stream(b.device)))


def dmuon_muon_step_batched_opts(params, grads, bufs, lr: float = 0.02, momentum: float = 0.95,
                                 nesterov: bool = True, weight_decay: float = 0.0,
                                 ns_steps: int = 5, ns_coefficients=(1.5, -0.5),
                                 lr_scale: str = "plain", max_grad_norm: float = 0.0,
                                 grad_norm_out: Optional[torch.Tensor] = None,
                                 workspace: Optional[torch.Tensor] = None) -> None:
    """One Muon update with the options of dmuon_step_options: custom cubic
    coefficients (a, b), per-matrix lr scale ("plain" or "sqrt_max":
    lr * 0.2 * sqrt(max(rows, cols))), Muon-only global-norm gradient
    clipping (max_grad_norm > 0; the pre-clip norm goes to ``grad_norm_out``,
    a one-element fp32 CUDA tensor, when given).  Scratch from ``workspace``
    or the library arena."""
    lib = load_library()
    b = _Batch(params, grads, bufs)
    if b.n == 0:
        return
    o = DmuonStepOptions()
    lib.dmuon_step_options_default(ctypes.byref(o))
    o.lr, o.momentum, o.weight_decay = lr, momentum, weight_decay
    o.nesterov, o.ns_steps = (1 if nesterov else 0), ns_steps
    _set_coefficients(o, ns_coefficients)
    o.lr_scale = {"plain": DMUON_LR_PLAIN, "sqrt_max": DMUON_LR_SQRT_MAX}[lr_scale]
    o.max_grad_norm = max_grad_norm
    if grad_norm_out is not None:
        if (grad_norm_out.dtype != torch.float32 or not grad_norm_out.is_cuda
                or grad_norm_out.device != b.device or grad_norm_out.numel() < 1):
            raise ValueError("grad_norm_out must be a CUDA fp32 tensor with one element")
        o.grad_norm_out = grad_norm_out.data_ptr()
    ws_ptr, ws_bytes = _workspace(workspace, b.device)
    with torch.cuda.device(b.device):
        _check(lib.dmuon_muon_step_batched_opts(*b.args(), ctypes.byref(o), ws_ptr, ws_bytes,
                                                _stream(b.device)))


def dmuon_muon_step_batched_reduce(params, rank_grads, bufs, lr: float = 0.02, momentum: float = 0.95,
                                   nesterov: bool = True, weight_decay: float = 0.0, ns_steps: int = 5,
                                   ns_coefficients=(1.5, -0.5), lr_scale: str = "plain",
                                   max_grad_norm: float = 0.0,
                                   workspace: Optional[torch.Tensor] = None) -> None:
    """The owner's step with the data-parallel gradient reduction fused in:
    ``rank_grads[r][i]`` is rank r's gradient of parameter i (a CUDA tensor
    this device can read: local, or another GPU's memory mapped here); the
    update uses their mean (fp32 sum in rank order, then one division).
    ``rank_grads[r][i]`` must be None for every rank or for none."""
    lib = load_library()
    world = len(rank_grads)
    n = len(params)
    if world < 1 or any(len(g) != n for g in rank_grads):
        raise ValueError("rank_grads must hold one list of len(params) gradients per rank")
    for r in range(1, world):
        for i in range(n):
            g, g0 = rank_grads[r][i], rank_grads[0][i]
            if (g is None) != (g0 is None):
                raise ValueError(f"gradient {i}: given on some ranks only")
            if g is not None:
                if not g.is_cuda or g.dtype != g0.dtype or g.shape != g0.shape or not g.is_contiguous():
                    raise ValueError(f"rank_grads[{r}][{i}] must match rank 0's gradient (CUDA, dtype, shape)")
    b = _Batch(params, rank_grads[0], bufs)
    if b.n == 0:
        return
    G = (ctypes.c_void_p * (world * n))()
    for r in range(world):
        for i in range(n):
            g = rank_grads[r][i]
            G[r * n + i] = g.data_ptr() if g is not None else None
    o = DmuonStepOptions()
    lib.dmuon_step_options_default(ctypes.byref(o))
    o.lr, o.momentum, o.weight_decay = lr, momentum, weight_decay
    o.nesterov, o.ns_steps = (1 if nesterov else 0), ns_steps
    _set_coefficients(o, ns_coefficients)
    o.lr_scale = {"plain": DMUON_LR_PLAIN, "sqrt_max": DMUON_LR_SQRT_MAX}[lr_scale]
    o.max_grad_norm = max_grad_norm
    ws_ptr, ws_bytes = _workspace(workspace, b.device)
    P, _, B, S, cnt = b.args()
    pp = ctypes.POINTER(ctypes.c_void_p)
    with torch.cuda.device(b.device):
        _check(lib.dmuon_muon_step_batched_reduce(P, ctypes.cast(G, pp), B, S, cnt, world, ctypes.byref(o),
                                                  ws_ptr, ws_bytes, _stream(b.device)))


def dmuon_muon_step_batched_host(params, grads, bufs, host_grads, host_params=None,
                                 lr: float = 0.02, momentum: float = 0.95, nesterov: bool = True,
                                 weight_decay: float = 0.0, ns_steps: int = 5,
                                 ns_coefficients=(1.5, -0.5), lr_scale: str = "plain",
                                 chunks: int = 0, workspace: Optional[torch.Tensor] = None) -> None:
    """One Muon update whose gradients come from page-locked host tensors
    (``host_grads``, copied into the device tensors ``grads``) and whose
    updated weights are copied back into page-locked host tensors
    (``host_params``, optional), with the copies overlapped with the update in
    ``chunks`` groups (0: the library picks).  ``params`` and ``bufs`` stay on
    the device.  Asynchronous on the current stream: synchronise it before
    reading ``host_params`` or reusing ``host_grads``."""
    lib = load_library()
    n = len(params)
    if len(host_grads) != n or (host_params is not None and len(host_params) != n):
        raise ValueError("host_grads and host_params must have one entry per parameter")
    dev_grads = [g if hg is not None else None for g, hg in zip(grads, host_grads)]
    b = _Batch(params, dev_grads, bufs)
    if b.n == 0:
        return
    HG = (ctypes.c_void_p * n)()
    HP = (ctypes.c_void_p * n)()
    for i, (p, g, hg) in enumerate(zip(params, grads, host_grads)):
        if hg is None:
            continue
        hp = host_params[i] if host_params is not None else None
        for t, what, ref in ((hg, "host_grads", g), (hp, "host_params", p)):
            if t is None:
                continue
            if t.is_cuda or not t.is_pinned() or not t.is_contiguous():
                raise ValueError(f"{what}[{i}] must be a contiguous page-locked (pinned) CPU tensor")
            if t.dtype != ref.dtype or t.shape != ref.shape:
                raise ValueError(f"{what}[{i}] must match the device tensor's dtype and shape")
        HG[i] = hg.data_ptr()
        HP[i] = hp.data_ptr() if hp is not None else None
    o = DmuonStepOptions()
    lib.dmuon_step_options_default(ctypes.byref(o))
    o.lr, o.momentum, o.weight_decay = lr, momentum, weight_decay
    o.nesterov, o.ns_steps = (1 if nesterov else 0), ns_steps
    _set_coefficients(o, ns_coefficients)
    o.lr_scale = {"plain": DMUON_LR_PLAIN, "sqrt_max": DMUON_LR_SQRT_MAX}[lr_scale]
    ws_ptr, ws_bytes = _workspace(workspace, b.device)
    P, G, B, S, cnt = b.args()
    pp = ctypes.POINTER(ctypes.c_void_p)
    with torch.cuda.device(b.device):
        _check(lib.dmuon_muon_step_batched_host(P, G, B, ctypes.cast(HG, pp), ctypes.cast(HP, pp), S,
                                                cnt, ctypes.byref(o), chunks, ws_ptr, ws_bytes,
                                                _stream(b.device)))


def dmuon_muon_step_batched_ex(params, grads, bufs, lr: float = 0.02, momentum: float = 0.95,
                               nesterov: bool = True, weight_decay: float = 0.0,
                               ns_steps: int = 5,
                               workspace: Optional[torch.Tensor] = None) -> None:
    """One Muon update of all matrices; scratch from ``workspace`` (a uint8
    CUDA tensor) or from PyTorch's allocator."""
    lib = load_library()
    b = _Batch(params, grads, bufs)
    if b.n == 0:
        return
    need = dmuon_workspace_bytes(params, ns_steps, grads)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=b.device)
    ws_ptr, ws_bytes = _workspace(workspace, b.device)
    with torch.cuda.device(b.device):
        _check(lib.dmuon_muon_step_batched_ex(*b.args(), lr, momentum, 1 if nesterov else 0,
                                              weight_decay, ns_steps, ws_ptr, ws_bytes,
                                              _stream(b.device)))


# ---------------------------------------------------------------- misc
def dmuon_last_error() -> str:
    return load_library().dmuon_last_error().decode()


def dmuon_backend_string() -> str:
    return load_library().dmuon_backend_string().decode()


def dmuon_device_status(clear: bool = False) -> int:
    return int(load_library().dmuon_device_status(1 if clear else 0))


def dmuon_release_cache() -> None:
    load_library().dmuon_release_cache()


def dmuon_debug_fail_allocations(n: int) -> None:
    load_library().dmuon_debug_fail_allocations(n)


def dmuon_debug_wait_timeout(limit_us: int, device: Optional[torch.device] = None) -> None:
    dev = device or torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        _check(load_library().dmuon_debug_wait_timeout(limit_us, _stream(dev)))


def dmuon_stage_timing(enable: bool) -> None:
    _check(load_library().dmuon_stage_timing(1 if enable else 0))


def dmuon_stage_times(reset: bool = False) -> dict:
    """{kind: (milliseconds, launches)} accumulated while timing was enabled."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _check(load_library().dmuon_stage_times(ms, cnt, n, 1 if reset else 0))
    return {k: (ms[i], int(cnt[i])) for i, k in enumerate(KERNEL_KINDS)}


def dmuon_launch_count() -> int:
    return int(load_library().dmuon_launch_count())


def dmuon_plan_builds() -> int:
    """Launch plans built so far (shapes seen before build none)."""
    return int(load_library().dmuon_plan_builds())


def dmuon_debug_last_plan() -> list:
    """Stage kernels of the most recently used launch plan, one dict per
    dtype group: {"syrk256": bool, "gemm_pair": bool, "square256": bool}
    (launches nothing)."""
    lib = load_library()
    n = int(lib.dmuon_debug_last_plan(None, 0))
    words = (ctypes.c_int32 * max(n, 1))()
    lib.dmuon_debug_last_plan(words, n)
    return [{"syrk256": bool(words[i] & 1), "gemm_pair": bool(words[i] & 2), "square256": bool(words[i] & 4)}
            for i in range(n)]


def dmuon_debug_check_pointer(address: int) -> int:
    """The entry points' device-memory check of one address (launches
    nothing): 0 for device memory, DMUON_ERR_INVALID_ARG (-1) otherwise."""
    return int(load_library().dmuon_debug_check_pointer(address))


def dmuon_ns_orthogonalize_noalloc(X: torch.Tensor, steps: int = 5) -> torch.Tensor:
    """In-place cubic Newton-Schulz of one bf16 matrix without allocating
    any device memory: the scratch is a fixed 32 MiB array inside the
    library.  For callers that must not allocate (a framework that owns all
    device memory, a sandbox without cudaMalloc, a path that must not block
    on an allocation).  Calls on different streams that may overlap race on
    the shared scratch; larger matrices are rejected (DMUON_ERR_UNSUPPORTED)."""
    lib = load_library()
    _cuda_matrix(X, "X")
    if X.dtype != torch.bfloat16:
        raise TypeError("dmuon_ns_orthogonalize_noalloc takes bf16")
    with torch.cuda.device(X.device):
        _check(lib.dmuon_ns_orthogonalize_noalloc(X.data_ptr(), X.shape[0], X.shape[1], steps,
                                                  _stream(X.device)))
    return X



def _clip_descs(segments):
    flat, descs = [], []
    dev = None
    for si, seg in enumerate(segments):
        for g in seg:
            if g is None:
                continue
            if not isinstance(g, torch.Tensor) or not g.is_cuda or not g.is_contiguous():
                raise ValueError(f"segment {si}: gradients must be contiguous CUDA tensors")
            dev = dev or g.device
            if g.device != dev:
                raise ValueError("all gradients must be on one device")
            flat.append(g)
            descs.append(DmuonGradDesc(g.numel(), _dtype_code(g.dtype), si))
    D = (DmuonGradDesc * max(len(descs), 1))(*descs)
    return flat, D, dev


def dmuon_clip_workspace_bytes(segments) -> int:
    flat, D, _ = _clip_descs(segments)
    return int(load_library().dmuon_clip_workspace_bytes(D, len(flat), max(len(segments), 1)))


def dmuon_clip_grad_norm_buckets(segments, max_norms, workspace: Optional[torch.Tensor] = None,
                                 device: Optional[torch.device] = None):
    """Clip several gradient groups in place, each with its own norm and
    coefficient: ``segments[s]`` is a list of gradient tensors (bf16 or fp32,
    any shape; None entries are skipped), ``max_norms`` one bound per segment
    (or one for all; ``math.inf`` measures without clipping).  Returns the
    per-segment norms before clipping and the coefficients, as fp32 CUDA
    tensors (asynchronous on the current stream)."""
    lib = load_library()
    nseg = len(segments)
    if isinstance(max_norms, (int, float)):
        max_norms = [float(max_norms)] * nseg
    if len(max_norms) != nseg or nseg < 1:
        raise ValueError("one max_norm per segment, at least one segment")
    flat, D, dev = _clip_descs(segments)
    dev = dev or device or torch.device("cuda", torch.cuda.current_device())
    norms = torch.empty(nseg, dtype=torch.float32, device=dev)
    coefs = torch.empty(nseg, dtype=torch.float32, device=dev)
    G = (ctypes.c_void_p * max(len(flat), 1))(*[g.data_ptr() for g in flat])
    M = (ctypes.c_float * nseg)(*max_norms)
    ws_ptr, ws_bytes = _workspace(workspace, dev)
    with torch.cuda.device(dev):
        _check(lib.dmuon_clip_grad_norm_buckets(ctypes.cast(G, ctypes.POINTER(ctypes.c_void_p)), D,
                                                len(flat), M, nseg, norms.data_ptr(), coefs.data_ptr(),
                                                ws_ptr, ws_bytes, _stream(dev)))
    return norms, coefs


def dmuon_adamw_step_batched(params, grads, exp_avgs, exp_avg_sqs, lr: float = 1e-3,
                             betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 0.01,
                             step: int = 1) -> None:
    """AdamW of the tensors the Muon path does not orthogonalise (any shape,
    contiguous; bf16 or fp32 parameters and gradients, fp32 states), one
    launch for all of them.  ``step`` counts this step (>= 1).  A None
    gradient skips its tensor."""
    lib = load_library()
    n = len(params)
    if not (len(grads) == len(exp_avgs) == len(exp_avg_sqs) == n):
        raise ValueError("params, grads, exp_avgs and exp_avg_sqs must have the same length")
    if n == 0:
        return
    P = (ctypes.c_void_p * n)()
    G = (ctypes.c_void_p * n)()
    M = (ctypes.c_void_p * n)()
    V = (ctypes.c_void_p * n)()
    D = (DmuonTensorDesc * n)()
    dev = None
    for i, (p, g, m, v) in enumerate(zip(params, grads, exp_avgs, exp_avg_sqs)):
        for t, what in ((p, "params"), (m, "exp_avgs"), (v, "exp_avg_sqs")) + (((g, "grads"),) if g is not None else ()):
            if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{what}[{i}] must be a contiguous CUDA tensor")
            if t.numel() != p.numel():
                raise ValueError(f"{what}[{i}] must have the parameter's number of elements")
            dev = dev or t.device
            if t.device != dev:
                raise ValueError("all tensors must be on one device")
        if m.dtype != torch.float32 or v.dtype != torch.float32:
            raise ValueError(f"exp_avgs[{i}] and exp_avg_sqs[{i}] must be fp32")
        P[i], M[i], V[i] = p.data_ptr(), m.data_ptr(), v.data_ptr()
        G[i] = g.data_ptr() if g is not None else None
        D[i] = DmuonTensorDesc(p.numel(), _dtype_code(p.dtype),
                               _dtype_code(g.dtype) if g is not None else _dtype_code(p.dtype))
    pp = ctypes.POINTER(ctypes.c_void_p)
    with torch.cuda.device(dev):
        _check(lib.dmuon_adamw_step_batched(ctypes.cast(P, pp), ctypes.cast(G, pp), ctypes.cast(M, pp),
                                            ctypes.cast(V, pp), D, n, lr, betas[0], betas[1], eps,
                                            weight_decay, step, _stream(dev)))


from .optim import Muon  # noqa: E402  (the optimizer wraps the functions above)

__all__.append("Muon")
