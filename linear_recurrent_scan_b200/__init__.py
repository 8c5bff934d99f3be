"""Mamba-3 selective recurrence on B200 (sm_100a): thin Python binding.

The computation lives in ``libmamba3.so`` (hand-written CUDA, C ABI declared in
``include/mamba3.h``).  This module only marshals torch tensors into the C
calls: it checks shapes and dtypes, passes device pointers and the current
CUDA stream, and raises on a non-zero status.  There is no CPU fallback; if
the library has not been built the import of the C entry points fails.

Entry points (same names as the C ABI):
  mamba3_scan_workspace_bytes(dims)
  mamba3_scan_fwd(x, B, C, theta, dt, lam, A, D=None, init=None, ...)
  mamba3_decode_step(state, x, B, C, theta, dt, lam, A, D=None, ...)
  mamba3_scan_fwd_bcnorm / mamba3_decode_step_bcnorm (raw B, C + BCNorm)
  mamba3_scan_fwd_at / mamba3_decode_step_at (time-varying decay A_t)
  mamba3_mimo_up / mamba3_mimo_down (MIMO rank-R projections, optional fused gate)
  mamba3_device_status(workspace), mamba3_library_status()
  mamba3_set_wait_limit(cycles), mamba3_test_withhold_loads(on)
  mamba3_status_string(code)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmamba3.so")

MAMBA3_OK = 0
MAMBA3_ERR_INVALID = -1
MAMBA3_ERR_UNSUPPORTED = -2
MAMBA3_ERR_WORKSPACE = -3
MAMBA3_ERR_CUDA = -4
MAMBA3_ERR_TIMEOUT = -5
MAMBA3_F32 = 0
MAMBA3_BF16 = 1

_DTYPES = {torch.float32: MAMBA3_F32, torch.bfloat16: MAMBA3_BF16}


class Mamba3Error(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {mamba3_status_string(code)} (status {code})")


ABI_MAJOR = 2


class Dims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("seqlen", ctypes.c_int), ("nheads", ctypes.c_int),
        ("headdim", ctypes.c_int), ("dstate", ctypes.c_int), ("rank", ctypes.c_int),
        ("chunk", ctypes.c_int), ("in_dtype", ctypes.c_int), ("ngroups", ctypes.c_int),
    ]


class _CState(ctypes.Structure):
    _fields_ = [("h", ctypes.c_void_p), ("b_prev", ctypes.c_void_p), ("x_prev", ctypes.c_void_p),
                ("angle", ctypes.c_void_p)]


class _CNorm(ctypes.Structure):
    _fields_ = [("w_B", ctypes.c_void_p), ("w_C", ctypes.c_void_p), ("bias_B", ctypes.c_void_p),
                ("bias_C", ctypes.c_void_p), ("eps", ctypes.c_float)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmamba3.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m linear_recurrent_scan_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz, i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    lib.mamba3_scan_workspace_bytes.argtypes = [ctypes.POINTER(Dims)]
    lib.mamba3_scan_workspace_bytes.restype = sz
    lib.mamba3_scan_fwd.argtypes = [ctypes.POINTER(Dims), vp, vp, vp, vp, vp, vp, vp, vp,
                                    ctypes.POINTER(_CState), vp, ctypes.POINTER(_CState), vp, sz, vp]
    lib.mamba3_scan_fwd.restype = i
    lib.mamba3_decode_step.argtypes = [ctypes.POINTER(Dims), ctypes.POINTER(_CState), vp, vp, vp, vp, vp, vp,
                                       vp, vp, vp, vp]
    lib.mamba3_decode_step.restype = i
    lib.mamba3_device_status.argtypes = [vp, vp]
    lib.mamba3_device_status.restype = i
    lib.mamba3_status_string.argtypes = [i]
    lib.mamba3_status_string.restype = ctypes.c_char_p
    lib.mamba3_version.argtypes = []
    lib.mamba3_version.restype = i
    if lib.mamba3_version() // 100 != ABI_MAJOR:  # Dims must match the library's mamba3_dims
        raise ImportError(f"{path} has ABI {lib.mamba3_version()}, this binding needs {ABI_MAJOR}.xx: rebuild it")
    lib.mamba3_scan_fwd_bcnorm.argtypes = [ctypes.POINTER(Dims), vp, vp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(_CNorm),
                                           ctypes.POINTER(_CState), vp, ctypes.POINTER(_CState), vp, sz, vp]
    lib.mamba3_scan_fwd_bcnorm.restype = i
    lib.mamba3_decode_step_bcnorm.argtypes = [ctypes.POINTER(Dims), ctypes.POINTER(_CState), vp, vp, vp, vp, vp, vp,
                                              vp, vp, ctypes.POINTER(_CNorm), vp, vp]
    lib.mamba3_decode_step_bcnorm.restype = i
    lib.mamba3_scan_fwd_at.argtypes = [ctypes.POINTER(Dims), vp, vp, vp, vp, vp, vp, vp, vp,
                                       ctypes.POINTER(_CState), vp, ctypes.POINTER(_CState), vp, sz, vp]
    lib.mamba3_scan_fwd_at.restype = i
    lib.mamba3_decode_step_at.argtypes = [ctypes.POINTER(Dims), ctypes.POINTER(_CState), vp, vp, vp, vp, vp, vp,
                                          vp, vp, vp, vp]
    lib.mamba3_decode_step_at.restype = i
    lib.mamba3_scan_bwd_workspace_bytes.argtypes = [ctypes.POINTER(Dims)]
    lib.mamba3_scan_bwd_workspace_bytes.restype = sz
    lib.mamba3_scan_bwd.argtypes = [ctypes.POINTER(Dims), vp, vp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(_CState), vp,
                                    ctypes.POINTER(_CState), vp, vp, vp, vp, vp, vp, vp, vp,
                                    ctypes.POINTER(_CState), vp, sz, vp]
    lib.mamba3_scan_bwd.restype = i
    lib.mamba3_scan_bwd_at.argtypes = lib.mamba3_scan_bwd.argtypes
    lib.mamba3_scan_bwd_at.restype = i
    lib.mamba3_gated_norm.argtypes = [ctypes.POINTER(Dims), i, vp, vp, vp, ctypes.c_float, vp, vp]
    lib.mamba3_gated_norm.restype = i
    lib.mamba3_scan_segmented_workspace_bytes.argtypes = [ctypes.POINTER(Dims)]
    lib.mamba3_scan_segmented_workspace_bytes.restype = sz
    lib.mamba3_test_set_segments.argtypes = [i]
    lib.mamba3_test_set_segments.restype = i
    lib.mamba3_scan_fwd_workspace_bytes.argtypes = [ctypes.POINTER(Dims)]
    lib.mamba3_scan_fwd_workspace_bytes.restype = sz
    lib.mamba3_test_set_split.argtypes = [i, i]
    lib.mamba3_test_set_split.restype = i
    lib.mamba3_library_status.argtypes = [vp]
    lib.mamba3_library_status.restype = i
    lib.mamba3_scan_fwd_host_stage_bytes.argtypes = [ctypes.POINTER(Dims)]
    lib.mamba3_scan_fwd_host_stage_bytes.restype = sz
    lib.mamba3_scan_fwd_host.argtypes = [ctypes.POINTER(Dims), vp, vp, vp, vp, vp, vp, vp, vp,
                                         ctypes.POINTER(_CState), vp, ctypes.POINTER(_CState), vp, sz, vp]
    lib.mamba3_scan_fwd_host.restype = i
    lib.mamba3_mimo_up.argtypes = [ctypes.POINTER(Dims), vp, vp, vp, vp]
    lib.mamba3_mimo_up.restype = i
    lib.mamba3_mimo_down.argtypes = [ctypes.POINTER(Dims), vp, vp, vp, vp, ctypes.c_float, vp, vp]
    lib.mamba3_mimo_down.restype = i
    lib.mamba3_set_wait_limit.argtypes = [ctypes.c_longlong]
    lib.mamba3_set_wait_limit.restype = i
    lib.mamba3_test_withhold_loads.argtypes = [i]
    lib.mamba3_test_withhold_loads.restype = i
    _lib = lib
    return lib


@dataclass
class State:
    """Recurrent state (fp32 device tensors): h [b,H,N,P], b_prev [b,H,R,N],
    x_prev [b,H,R,P], angle [b,H,N/2]."""
    h: torch.Tensor
    b_prev: torch.Tensor
    x_prev: torch.Tensor
    angle: torch.Tensor

    @staticmethod
    def zeros(batch, nheads, headdim, dstate, rank, device="cuda") -> "State":
        z = lambda *s: torch.zeros(*s, dtype=torch.float32, device=device)
        return State(z(batch, nheads, dstate, headdim), z(batch, nheads, rank, dstate),
                     z(batch, nheads, rank, headdim), z(batch, nheads, dstate // 2))

    def clone(self) -> "State":
        return State(self.h.clone(), self.b_prev.clone(), self.x_prev.clone(), self.angle.clone())

    def _c(self) -> _CState:
        for t in (self.h, self.b_prev, self.x_prev, self.angle):
            if t.dtype != torch.float32 or not t.is_contiguous():
                raise ValueError("state tensors must be contiguous float32")
        return _CState(self.h.data_ptr(), self.b_prev.data_ptr(), self.x_prev.data_ptr(), self.angle.data_ptr())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(code: int, where: str):
    if code != MAMBA3_OK:
        raise Mamba3Error(code, where)


def make_dims(x: torch.Tensor, B: torch.Tensor, chunk: int = 0, decode: bool = False) -> Dims:
    if decode:
        b, H, R, P = x.shape
        L = 1
    else:
        b, L, H, R, P = x.shape
    if x.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {x.dtype}")
    return Dims(b, L, H, P, B.shape[-1], R, chunk, _DTYPES[x.dtype], B.shape[-3])


def mamba3_status_string(code: int) -> str:
    return load_library().mamba3_status_string(code).decode()


def mamba3_scan_workspace_bytes(dims: Dims) -> int:
    return int(load_library().mamba3_scan_workspace_bytes(ctypes.byref(dims)))


def mamba3_scan_fwd_workspace_bytes(dims: Dims) -> int:
    """Workspace with which mamba3_scan_fwd runs its best schedule (segments for
    few long sequences, else the split last wave; the minimum when neither applies)."""
    return int(load_library().mamba3_scan_fwd_workspace_bytes(ctypes.byref(dims)))


def mamba3_scan_segmented_workspace_bytes(dims: Dims) -> int:
    """Workspace with which a long sequence over few (batch, head) units runs in
    segments (mamba3_scan_workspace_bytes when the dims do not qualify)."""
    return int(load_library().mamba3_scan_segmented_workspace_bytes(ctypes.byref(dims)))


def _check_inputs(x, B, C, theta, dt, lam, A, D, decode):
    lead = x.shape[:-2]
    for name, t in (("x", x), ("B", B), ("C", C), ("theta", theta), ("dt", dt), ("lam", lam)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.dtype != x.dtype:
            raise ValueError(f"{name} must have the dtype of x ({x.dtype})")
        if t.device != x.device:
            raise ValueError(f"{name} must be on the device of x")
    H = x.shape[-3]
    if (B.shape != C.shape or B.dim() != x.dim() or B.shape[:-3] != x.shape[:-3] or B.shape[-2] != x.shape[-2]
            or H % B.shape[-3] != 0):
        raise ValueError("B and C must be [..., G, R, N] with the leading shape of x and G dividing H "
                         "(G = H: one row per head)")
    if theta.shape != lead + (B.shape[-1] // 2,) or dt.shape != lead or lam.shape != lead:
        raise ValueError("theta must be [..., N/2] and dt, lam [...] with the leading shape of x")
    for name, t in (("A", A), ("D", D)):
        if t is not None and (t.dtype != torch.float32 or t.shape != (H,) or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous float32 tensor of shape [H]")


def mamba3_scan_fwd(x, B, C, theta, dt, lam, A, D=None, init: Optional[State] = None,
                    y: Optional[torch.Tensor] = None, final_state: Optional[State] = None,
                    workspace: Optional[torch.Tensor] = None, chunk: int = 0, stream=None):
    """Chunked prefill. Shapes: x [b,L,H,R,P], B/C [b,L,H,R,N] (or [b,L,G,R,N],
    shared by groups of H/G consecutive heads), theta [b,L,H,N/2], dt/lam [b,L,H],
    A/D [H] fp32. Returns y (allocated if not given)."""
    lib = load_library()
    _check_inputs(x, B, C, theta, dt, lam, A, D, decode=False)
    dims = make_dims(x, B, chunk)
    if y is None:
        y = torch.empty_like(x)
    if workspace is None:
        workspace = torch.empty(mamba3_scan_fwd_workspace_bytes(dims), dtype=torch.uint8, device=x.device)
    ci = init._c() if init is not None else None
    cf = final_state._c() if final_state is not None else None
    rc = lib.mamba3_scan_fwd(ctypes.byref(dims), _ptr(x), _ptr(B), _ptr(C), _ptr(theta), _ptr(dt), _ptr(lam),
                             _ptr(A), _ptr(D), ctypes.byref(ci) if ci is not None else None, _ptr(y),
                             ctypes.byref(cf) if cf is not None else None, _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "mamba3_scan_fwd")
    return y


def mamba3_scan_fwd_host_stage_bytes(dims: Dims) -> int:
    """Device stage bytes mamba3_scan_fwd_host needs for ``dims``."""
    return int(load_library().mamba3_scan_fwd_host_stage_bytes(ctypes.byref(dims)))


def mamba3_scan_fwd_host(x, B, C, theta, dt, lam, A, D=None, init: Optional[State] = None,
                         y: Optional[torch.Tensor] = None, final_state: Optional[State] = None,
                         stage: Optional[torch.Tensor] = None, stream=None):
    """The prefill from host tensors (x .. lam on the CPU, page-locked for
    asynchronous copies; the shapes of mamba3_scan_fwd): the library copies
    sub-batches in, runs them and copies y out on overlapping streams.  A, D, init,
    final_state and ``stage`` are device tensors. Returns the host y (allocated,
    page-locked, if not given); it is complete once ``stream`` is synchronised."""
    lib = load_library()
    _check_inputs(x, B, C, theta, dt, lam, A, D, decode=False)
    if x.device.type != "cpu":
        raise ValueError("mamba3_scan_fwd_host takes host tensors; use mamba3_scan_fwd for device tensors")
    dims = make_dims(x, B)
    if y is None:
        y = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    if y.device.type != "cpu" or y.shape != x.shape or y.dtype != x.dtype or not y.is_contiguous():
        raise ValueError("y must be a contiguous host tensor shaped like x")
    if stage is None:
        stage = torch.empty(mamba3_scan_fwd_host_stage_bytes(dims), dtype=torch.uint8, device=A.device)
    ci = init._c() if init is not None else None
    cf = final_state._c() if final_state is not None else None
    rc = lib.mamba3_scan_fwd_host(ctypes.byref(dims), _ptr(x), _ptr(B), _ptr(C), _ptr(theta), _ptr(dt), _ptr(lam),
                                  _ptr(A), _ptr(D), ctypes.byref(ci) if ci is not None else None, _ptr(y),
                                  ctypes.byref(cf) if cf is not None else None, _ptr(stage),
                                  stage.numel() * stage.element_size(), _stream(stream))
    _check(rc, "mamba3_scan_fwd_host")
    return y


def mamba3_decode_step(state: State, x, B, C, theta, dt, lam, A, D=None, y: Optional[torch.Tensor] = None,
                       stream=None):
    """One decode step in place on ``state``. Shapes: x [b,H,R,P], B/C [b,H,R,N]
    (or [b,G,R,N]), theta [b,H,N/2], dt/lam [b,H]. Returns y [b,H,R,P]."""
    lib = load_library()
    _check_inputs(x, B, C, theta, dt, lam, A, D, decode=True)
    dims = make_dims(x, B, decode=True)
    if y is None:
        y = torch.empty_like(x)
    cs = state._c()
    rc = lib.mamba3_decode_step(ctypes.byref(dims), ctypes.byref(cs), _ptr(x), _ptr(B), _ptr(C), _ptr(theta),
                                _ptr(dt), _ptr(lam), _ptr(A), _ptr(D), _ptr(y), _stream(stream))
    _check(rc, "mamba3_decode_step")
    return y


def mamba3_scan_fwd_noalloc(x, B, C, theta, dt, lam, A, D=None, init: Optional[State] = None,
                            y: Optional[torch.Tensor] = None, final_state: Optional[State] = None,
                            chunk: int = 0, stream=None):
    """The prefill with the library's own scratch instead of a workspace tensor,
    for callers that cannot allocate device memory (see mamba3.h).  Passing no
    ``y`` makes this wrapper allocate one with torch; pass ``y`` to allocate nothing."""
    lib = load_library()
    f = lib.mamba3_scan_fwd_noalloc
    f.argtypes = [ctypes.POINTER(Dims), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(_CState),
                  ctypes.c_void_p, ctypes.POINTER(_CState), ctypes.c_void_p]
    f.restype = ctypes.c_int
    _check_inputs(x, B, C, theta, dt, lam, A, D, decode=False)
    dims = make_dims(x, B, chunk)
    if y is None:
        y = torch.empty_like(x)
    ci = init._c() if init is not None else None
    cf = final_state._c() if final_state is not None else None
    rc = f(ctypes.byref(dims), _ptr(x), _ptr(B), _ptr(C), _ptr(theta), _ptr(dt), _ptr(lam), _ptr(A), _ptr(D),
           ctypes.byref(ci) if ci is not None else None, _ptr(y), ctypes.byref(cf) if cf is not None else None,
           _stream(stream))
    _check(rc, "mamba3_scan_fwd_noalloc")
    return y


@dataclass
class BCNorm:
    """Fused B/C normalisation (see mamba3.h): float32 device tensors [H, R, N]
    or None (weight 1, bias 0), and eps."""
    w_B: Optional[torch.Tensor] = None
    w_C: Optional[torch.Tensor] = None
    bias_B: Optional[torch.Tensor] = None
    bias_C: Optional[torch.Tensor] = None
    eps: float = 1e-6

    def _c(self, H, R, N) -> _CNorm:
        for name in ("w_B", "w_C", "bias_B", "bias_C"):
            t = getattr(self, name)
            if t is not None and (t.dtype != torch.float32 or t.shape != (H, R, N) or not t.is_contiguous()):
                raise ValueError(f"{name} must be a contiguous float32 tensor of shape [H, R, N]")
        return _CNorm(_ptr(self.w_B), _ptr(self.w_C), _ptr(self.bias_B), _ptr(self.bias_C), float(self.eps))


def mamba3_scan_fwd_bcnorm(x, B_raw, C_raw, theta, dt, lam, A, D=None, norm: Optional[BCNorm] = None,
                           init: Optional[State] = None, y: Optional[torch.Tensor] = None,
                           final_state: Optional[State] = None, workspace: Optional[torch.Tensor] = None,
                           chunk: int = 0, stream=None):
    """mamba3_scan_fwd on raw B, C projections with the B/C normalisation fused in."""
    lib = load_library()
    _check_inputs(x, B_raw, C_raw, theta, dt, lam, A, D, decode=False)
    norm = norm if norm is not None else BCNorm()
    dims = make_dims(x, B_raw, chunk)
    cn = norm._c(x.shape[2], x.shape[3], B_raw.shape[-1])
    if y is None:
        y = torch.empty_like(x)
    if workspace is None:
        workspace = torch.empty(mamba3_scan_fwd_workspace_bytes(dims), dtype=torch.uint8, device=x.device)
    ci = init._c() if init is not None else None
    cf = final_state._c() if final_state is not None else None
    rc = lib.mamba3_scan_fwd_bcnorm(ctypes.byref(dims), _ptr(x), _ptr(B_raw), _ptr(C_raw), _ptr(theta), _ptr(dt),
                                    _ptr(lam), _ptr(A), _ptr(D), ctypes.byref(cn),
                                    ctypes.byref(ci) if ci is not None else None, _ptr(y),
                                    ctypes.byref(cf) if cf is not None else None, _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "mamba3_scan_fwd_bcnorm")
    return y


def mamba3_decode_step_bcnorm(state: State, x, B_raw, C_raw, theta, dt, lam, A, D=None,
                              norm: Optional[BCNorm] = None, y: Optional[torch.Tensor] = None, stream=None):
    """mamba3_decode_step on the raw B, C projections of the token with the B/C
    normalisation fused in."""
    lib = load_library()
    _check_inputs(x, B_raw, C_raw, theta, dt, lam, A, D, decode=True)
    norm = norm if norm is not None else BCNorm()
    dims = make_dims(x, B_raw, decode=True)
    cn = norm._c(x.shape[1], x.shape[2], B_raw.shape[-1])
    if y is None:
        y = torch.empty_like(x)
    cs = state._c()
    rc = lib.mamba3_decode_step_bcnorm(ctypes.byref(dims), ctypes.byref(cs), _ptr(x), _ptr(B_raw), _ptr(C_raw),
                                       _ptr(theta), _ptr(dt), _ptr(lam), _ptr(A), _ptr(D), ctypes.byref(cn), _ptr(y),
                                       _stream(stream))
    _check(rc, "mamba3_decode_step_bcnorm")
    return y


def _check_at(A_t, dt, x):
    if A_t.shape != dt.shape or A_t.dtype != x.dtype or not A_t.is_contiguous() or A_t.device != x.device:
        raise ValueError("A_t must be a contiguous tensor shaped like dt, with the dtype and device of x")


def mamba3_scan_fwd_at(x, B, C, theta, dt, lam, A_t, D=None, init: Optional[State] = None,
                       y: Optional[torch.Tensor] = None, final_state: Optional[State] = None,
                       workspace: Optional[torch.Tensor] = None, chunk: int = 0, stream=None):
    """mamba3_scan_fwd with a time-varying decay A_t [b, L, H] (dtype of x) in
    place of the per-head A."""
    lib = load_library()
    _check_inputs(x, B, C, theta, dt, lam, None, D, decode=False)
    _check_at(A_t, dt, x)
    dims = make_dims(x, B, chunk)
    if y is None:
        y = torch.empty_like(x)
    if workspace is None:
        workspace = torch.empty(mamba3_scan_fwd_workspace_bytes(dims), dtype=torch.uint8, device=x.device)
    ci = init._c() if init is not None else None
    cf = final_state._c() if final_state is not None else None
    rc = lib.mamba3_scan_fwd_at(ctypes.byref(dims), _ptr(x), _ptr(B), _ptr(C), _ptr(theta), _ptr(dt), _ptr(lam),
                                _ptr(A_t), _ptr(D), ctypes.byref(ci) if ci is not None else None, _ptr(y),
                                ctypes.byref(cf) if cf is not None else None, _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "mamba3_scan_fwd_at")
    return y


def mamba3_decode_step_at(state: State, x, B, C, theta, dt, lam, A_t, D=None, y: Optional[torch.Tensor] = None,
                          stream=None):
    """mamba3_decode_step with the token's decay rate A_t [b, H] (dtype of x)."""
    lib = load_library()
    _check_inputs(x, B, C, theta, dt, lam, None, D, decode=True)
    _check_at(A_t, dt, x)
    dims = make_dims(x, B, decode=True)
    if y is None:
        y = torch.empty_like(x)
    cs = state._c()
    rc = lib.mamba3_decode_step_at(ctypes.byref(dims), ctypes.byref(cs), _ptr(x), _ptr(B), _ptr(C), _ptr(theta),
                                   _ptr(dt), _ptr(lam), _ptr(A_t), _ptr(D), _ptr(y), _stream(stream))
    _check(rc, "mamba3_decode_step_at")
    return y


def mamba3_scan_bwd_workspace_bytes(dims: Dims) -> int:
    return int(load_library().mamba3_scan_bwd_workspace_bytes(ctypes.byref(dims)))


def mamba3_scan_bwd(x, B, C, theta, dt, lam, A, D, dy, init: Optional[State] = None,
                    d_final: Optional[State] = None, grads: Optional[dict] = None,
                    workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """Gradients of mamba3_scan_fwd (see mamba3.h) given dy (shaped like y) and,
    optionally, the gradients of the exported state.  Returns a dict: dx, dB,
    dC, dtheta, ddt, dlam (shaped and typed like the inputs), dA, dD (fp32
    [H]) and d_init (a State: the initial state's gradients).  ``grads`` may
    hold preallocated outputs under those names."""
    return _scan_bwd(x, B, C, theta, dt, lam, A, None, D, dy, init, d_final, grads, workspace, stream)


def mamba3_scan_bwd_at(x, B, C, theta, dt, lam, A_t, D, dy, init: Optional[State] = None,
                       d_final: Optional[State] = None, grads: Optional[dict] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """mamba3_scan_bwd for mamba3_scan_fwd_at: A_t [b, L, H] (dtype of x); the
    dict holds dA_t (shaped and typed like A_t) in place of dA."""
    return _scan_bwd(x, B, C, theta, dt, lam, None, A_t, D, dy, init, d_final, grads, workspace, stream)


def _scan_bwd(x, B, C, theta, dt, lam, A, A_t, D, dy, init, d_final, grads, workspace, stream) -> dict:
    lib = load_library()
    _check_inputs(x, B, C, theta, dt, lam, A, D, decode=False)
    if A_t is not None:
        _check_at(A_t, dt, x)
    if dy.shape != x.shape or dy.dtype != x.dtype or not dy.is_contiguous() or dy.device != x.device:
        raise ValueError("dy must be a contiguous tensor shaped and typed like x")
    dims = make_dims(x, B)
    b, L, H, R, P = x.shape
    N = B.shape[-1]
    out = dict(grads or {})
    for name, like in (("dx", x), ("dB", B), ("dC", C), ("dtheta", theta), ("ddt", dt), ("dlam", lam)):
        if name not in out:
            out[name] = torch.empty_like(like)
    rate_grad = "dA" if A_t is None else "dA_t"
    if rate_grad not in out:
        out[rate_grad] = (torch.empty(H, dtype=torch.float32, device=x.device) if A_t is None
                          else torch.empty_like(A_t))
    if "dD" not in out:
        out["dD"] = torch.empty(H, dtype=torch.float32, device=x.device)
    if "d_init" not in out:
        out["d_init"] = State.zeros(b, H, P, N, R, device=x.device)
    if workspace is None:
        workspace = torch.empty(mamba3_scan_bwd_workspace_bytes(dims), dtype=torch.uint8, device=x.device)
    ci = init._c() if init is not None else None
    cf = d_final._c() if d_final is not None else None
    cd = out["d_init"]._c()
    fn = lib.mamba3_scan_bwd if A_t is None else lib.mamba3_scan_bwd_at
    rc = fn(ctypes.byref(dims), _ptr(x), _ptr(B), _ptr(C), _ptr(theta), _ptr(dt), _ptr(lam),
            _ptr(A if A_t is None else A_t), _ptr(D), ctypes.byref(ci) if ci is not None else None, _ptr(dy),
            ctypes.byref(cf) if cf is not None else None, _ptr(out["dx"]), _ptr(out["dB"]),
            _ptr(out["dC"]), _ptr(out["dtheta"]), _ptr(out["ddt"]), _ptr(out["dlam"]),
            _ptr(out[rate_grad]), _ptr(out["dD"]), ctypes.byref(cd), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "mamba3_scan_bwd" if A_t is None else "mamba3_scan_bwd_at")
    return out


def mamba3_gated_norm(y, z, w=None, groups: Optional[int] = None, eps: float = 1e-6,
                      out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Pre-gate grouped RMS norm and gate of the layer output (see mamba3.h):
    y, z [..., H, R, P] (same shape, dtype, device; contiguous), w fp32
    [H, R, P] or None, ``groups`` norm groups of H / groups consecutive heads
    (default H).  Returns out (allocated if not given; may be y)."""
    lib = load_library()
    if y.shape != z.shape or y.dtype != z.dtype or y.device != z.device or y.dim() < 3:
        raise ValueError("y and z must have the same shape [..., H, R, P], dtype and device")
    for name, t in (("y", y), ("z", z)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if y.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {y.dtype}")
    H, R, P = y.shape[-3:]
    if w is not None and (w.dtype != torch.float32 or w.shape != (H, R, P) or not w.is_contiguous()):
        raise ValueError("w must be a contiguous float32 tensor of shape [H, R, P]")
    groups = H if groups is None else groups
    if out is None:
        out = torch.empty_like(y)
    elif out.shape != y.shape or out.dtype != y.dtype or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor shaped and typed like y")
    tokens = y.numel() // (H * R * P) if H * R * P else 0
    dims = Dims(1, tokens, H, P, 0, R, 0, _DTYPES[y.dtype], 0)
    rc = lib.mamba3_gated_norm(ctypes.byref(dims), int(groups), _ptr(y), _ptr(z), _ptr(w), float(eps), _ptr(out),
                               _stream(stream))
    _check(rc, "mamba3_gated_norm")
    return out


def mamba3_device_status(workspace: torch.Tensor, stream=None) -> int:
    return int(load_library().mamba3_device_status(_ptr(workspace), _stream(stream)))


def mamba3_library_status(stream=None) -> int:
    """Synchronise the stream; return and clear the status words of the calls
    without a workspace (decode steps, MIMO projections) on the current device."""
    return int(load_library().mamba3_library_status(_stream(stream)))


def mamba3_mimo_up(u, Wx, out=None, stream=None):
    """MIMO input projection per head: u [..., H, P] bf16, Wx [H, R P, P] bf16 ->
    x [..., H, R, P] bf16 (allocated if not given)."""
    lib = load_library()
    *lead, H, P = u.shape
    if Wx.dim() != 3 or Wx.shape[0] != H or Wx.shape[2] != P or Wx.shape[1] % P:
        raise ValueError("Wx must be [H, R P, P]")
    R = Wx.shape[1] // P
    for name, t in (("u", u), ("Wx", Wx)):
        if not t.is_contiguous() or t.dtype not in _DTYPES:
            raise ValueError(f"{name} must be a contiguous float32 or bfloat16 tensor")
    if out is None:
        out = torch.empty((*lead, H, R, P), dtype=u.dtype, device=u.device)
    tokens = u.numel() // (H * P) if H * P else 0
    dims = Dims(1, tokens, H, P, 0, R, 0, _DTYPES[u.dtype], 0)
    _check(lib.mamba3_mimo_up(ctypes.byref(dims), _ptr(u), _ptr(Wx), _ptr(out), _stream(stream)), "mamba3_mimo_up")
    return out


def mamba3_mimo_down(y, Wy, z=None, w=None, eps: float = 1e-6, out=None, stream=None):
    """MIMO output projection per head: y [..., H, R, P] bf16, Wy [H, P, R P] bf16
    -> [..., H, P] bf16; with the gate z [..., H, P] the RMS norm over P (weight w
    [H, P] float32 or None) and silu(z) follow in the same kernel."""
    lib = load_library()
    *lead, H, R, P = y.shape
    if tuple(Wy.shape) != (H, P, R * P):
        raise ValueError("Wy must be [H, P, R P]")
    for name, t in (("y", y), ("Wy", Wy)):
        if not t.is_contiguous() or t.dtype not in _DTYPES:
            raise ValueError(f"{name} must be a contiguous float32 or bfloat16 tensor")
    if z is not None and (tuple(z.shape) != (*lead, H, P) or not z.is_contiguous() or z.dtype != y.dtype):
        raise ValueError("z must be contiguous [..., H, P] in the dtype of y")
    if w is not None and (w.dtype != torch.float32 or tuple(w.shape) != (H, P) or not w.is_contiguous()):
        raise ValueError("w must be a contiguous float32 tensor [H, P]")
    if out is None:
        out = torch.empty((*lead, H, P), dtype=y.dtype, device=y.device)
    tokens = y.numel() // (H * R * P) if H * R * P else 0
    dims = Dims(1, tokens, H, P, 0, R, 0, _DTYPES[y.dtype], 0)
    _check(lib.mamba3_mimo_down(ctypes.byref(dims), _ptr(y), _ptr(Wy), _ptr(z), _ptr(w), float(eps), _ptr(out),
                                _stream(stream)), "mamba3_mimo_down")
    return out


def mamba3_set_wait_limit(cycles: int) -> None:
    """Bound of every on-device wait in SM cycles (default 4e9, about 2 s)."""
    _check(load_library().mamba3_set_wait_limit(int(cycles)), "mamba3_set_wait_limit")


def mamba3_test_set_split(k: int, c1: int = 0) -> None:
    """Testing only: split units 0..k-1 after c1 chunks (k > 0), never split (k < 0),
    or restore the library's plan (k = 0)."""
    _check(load_library().mamba3_test_set_split(int(k), int(c1)), "mamba3_test_set_split")


def mamba3_test_set_segments(S: int) -> None:
    """Testing the segmented prefill only: S >= 2 segments whenever S divides the
    sequence length; 0 restores the library's choice."""
    _check(load_library().mamba3_test_set_segments(int(S)), "mamba3_test_set_segments")


def mamba3_test_withhold_loads(on: bool) -> None:
    """Testing the timeout path only: kernels launched while on issue no input
    copies, so their waits give up with MAMBA3_ERR_TIMEOUT."""
    _check(load_library().mamba3_test_withhold_loads(1 if on else 0), "mamba3_test_withhold_loads")


__all__ = [
    "Dims", "State", "BCNorm", "Mamba3Error", "load_library", "make_dims",
    "mamba3_scan_workspace_bytes", "mamba3_scan_segmented_workspace_bytes", "mamba3_scan_fwd_workspace_bytes", "mamba3_scan_fwd", "mamba3_scan_fwd_noalloc",
    "mamba3_scan_fwd_host_stage_bytes", "mamba3_scan_fwd_host", "mamba3_decode_step",
    "mamba3_scan_fwd_bcnorm", "mamba3_decode_step_bcnorm", "mamba3_scan_fwd_at", "mamba3_decode_step_at",
    "mamba3_scan_bwd_workspace_bytes", "mamba3_scan_bwd", "mamba3_scan_bwd_at", "mamba3_gated_norm",
    "mamba3_device_status", "mamba3_library_status", "mamba3_mimo_up", "mamba3_mimo_down", "mamba3_set_wait_limit", "mamba3_test_withhold_loads", "mamba3_test_set_segments", "mamba3_test_set_split",
    "mamba3_status_string",
]
