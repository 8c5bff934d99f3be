"""fp64 CPU oracle for the Mamba-3 selective recurrence.

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are the only
callers.  The product package never imports this module, and this module
imports nothing from the product package.

The arithmetic lives in ``mamba3_oracle.c`` (plain C, fp64, pthreads over the
independent (batch, head) units).  This file only compiles it with gcc,
loads it with ctypes and marshals numpy arrays.

Sources: the pages on the Mamba-3 paper -- "Mamba-3: 2x smaller state ..."
(MarkTechPost, Korean translation) sections 1.1 (exponential-trapezoidal
three-term update), 1.2 (complex state and the RoPE trick), 1.3 (MIMO rank-R
input and output shapes).  The readout ``y = C^T h + D x`` is the standard SSM
readout (the pages do not print it).

Parity status of each entry point (what pins it) is listed in
``tests/test_oracle_pins.py``; every function here is pinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mamba3_oracle.c")
_LIB = os.path.join(_HERE, "libmamba3_oracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-o", tmp, _SRC, "-lm", "-lpthread"]
        )
        os.replace(tmp, _LIB)
    return _LIB


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("batch", "seqlen", "nheads", "headdim", "dstate", "rank", "ngroups")]


_P = ctypes.POINTER(ctypes.c_double)


class _IO(ctypes.Structure):
    _fields_ = [
        (n, _P)
        for n in (
            "x", "B", "C", "theta", "dt", "lam", "A", "D",
            "h0", "bprev0", "xprev0", "angle0",
            "y", "h_out", "bprev_out", "xprev_out", "angle_out",
            "A_t",
        )
    ] + [("grad", ctypes.c_void_p)]


class _Grad(ctypes.Structure):
    _fields_ = [
        (n, _P)
        for n in (
            "dy", "dh_out", "dbprev_out", "dxprev_out", "dangle_out",
            "dx", "dB", "dC", "dtheta", "ddt", "dlam", "dA", "dD",
            "dh0", "dbprev0", "dxprev0", "dangle0",
        )
    ]


_lib = None


def _bind(lib):
    for name in ("m3o_scan_complex", "m3o_scan_rope"):
        f = getattr(lib, name)
        f.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_IO), ctypes.c_int,
                      ctypes.POINTER(ctypes.c_int), ctypes.c_int]
        f.restype = ctypes.c_int
    for name in ("m3o_scan_quadratic", "m3o_decode_step"):
        f = getattr(lib, name)
        f.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_IO), ctypes.c_int]
        f.restype = ctypes.c_int
    lib.m3o_scan_rope_bwd.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_IO), ctypes.c_int]
    lib.m3o_scan_rope_bwd.restype = ctypes.c_int
    lib.m3o_bc_norm.argtypes = [ctypes.POINTER(_Dims), _P, _P, _P, ctypes.c_double, _P]
    lib.m3o_gated_norm.argtypes = [ctypes.POINTER(_Dims), ctypes.c_int, _P, _P, _P, ctypes.c_double, _P]
    lib.m3o_gated_norm.restype = ctypes.c_int
    lib.m3o_bc_norm.restype = ctypes.c_int
    for name in ("m3o_mimo_up", "m3o_mimo_down"):
        f = getattr(lib, name)
        f.argtypes = [ctypes.POINTER(_Dims), _P, _P, _P]
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


@dataclass
class State:
    """Decode state in the real frame rotated by -Phi (float64 numpy arrays).

    h [b,H,N,P], b_prev [b,H,R,N], x_prev [b,H,R,P], angle [b,H,N/2].
    """
    h: np.ndarray
    b_prev: np.ndarray
    x_prev: np.ndarray
    angle: np.ndarray

    @staticmethod
    def zeros(batch, nheads, headdim, dstate, rank) -> "State":
        return State(
            np.zeros((batch, nheads, dstate, headdim)),
            np.zeros((batch, nheads, rank, dstate)),
            np.zeros((batch, nheads, rank, headdim)),
            np.zeros((batch, nheads, dstate // 2)),
        )


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    return a.ctypes.data_as(_P) if a is not None else None


def _prepare(x, B, C, theta, dt, lam, A, D):
    x, B, C, theta, dt, lam, A = map(_f64, (x, B, C, theta, dt, lam, A))
    D = _f64(D) if D is not None else None
    b, L, H, R, P = x.shape
    N = B.shape[-1]
    G = B.shape[2]
    assert B.shape == (b, L, G, R, N) and C.shape == B.shape and H % G == 0, \
        "B/C must be [b,L,H,R,N] or, grouped, [b,L,G,R,N] with H a multiple of G"
    assert theta.shape == (b, L, H, N // 2), "theta must be [b,L,H,N/2]"
    assert dt.shape == (b, L, H) and lam.shape == (b, L, H)
    assert A.shape == (H,) or A.shape == (b, L, H), "A must be [H] (per head) or [b,L,H] (per token)"
    dims = _Dims(b, L, H, P, N, R, 0 if G == H else G)
    return dims, (x, B, C, theta, dt, lam, A, D)


def _run(fn_name, x, B, C, theta, dt, lam, A, D=None, init: Optional[State] = None,
         want_state=True, nthreads: Optional[int] = None, units=None):
    lib = _load()
    dims, arrs = _prepare(x, B, C, theta, dt, lam, A, D)
    x, B, C, theta, dt, lam, A, D = arrs
    b, L, H, R, P = x.shape
    N = B.shape[-1]
    y = np.zeros_like(x)
    fin = State.zeros(b, H, P, N, R) if want_state else None
    A_t = None
    if A.ndim == 3:  # time-varying decay: A_t [b, L, H] replaces the per-head A
        A_t, A = A, np.zeros(H)
    keep = [x, B, C, theta, dt, lam, A, A_t, D, y]
    io = _IO()
    io.x, io.B, io.C, io.theta, io.dt, io.lam, io.A, io.D = map(_ptr, (x, B, C, theta, dt, lam, A, D))
    io.A_t = _ptr(A_t)
    if init is not None:
        ih, ib, ix, ia = (_f64(init.h), _f64(init.b_prev), _f64(init.x_prev), _f64(init.angle))
        keep += [ih, ib, ix, ia]
        io.h0, io.bprev0, io.xprev0, io.angle0 = map(_ptr, (ih, ib, ix, ia))
    io.y = _ptr(y)
    if fin is not None:
        io.h_out, io.bprev_out, io.xprev_out, io.angle_out = map(
            _ptr, (fin.h, fin.b_prev, fin.x_prev, fin.angle))
    nt = nthreads if nthreads is not None else (os.cpu_count() or 1)
    if fn_name in ("m3o_scan_complex", "m3o_scan_rope"):
        if units is not None:
            u = np.ascontiguousarray(np.asarray(units, dtype=np.int32))
            keep.append(u)
            rc = getattr(lib, fn_name)(ctypes.byref(dims), ctypes.byref(io), nt,
                                       u.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), len(u))
        else:
            rc = getattr(lib, fn_name)(ctypes.byref(dims), ctypes.byref(io), nt, None, 0)
    else:
        rc = getattr(lib, fn_name)(ctypes.byref(dims), ctypes.byref(io), nt)
    if rc != 0:
        raise ValueError(f"{fn_name} rejected its arguments (rc={rc})")
    return y, fin


def scan_complex(x, B, C, theta, dt, lam, A, D=None, init=None, nthreads=None, units=None):
    """The definition: explicit complex-diagonal state, sequential in t.
    A is [H] (one decay rate per head) or [b, L, H] (time-varying, one per token).
    B, C are [b, L, H, R, N] or, shared by groups of heads, [b, L, G, R, N]
    (head h reads group h // (H // G)).

    Returns (y [b,L,H,R,P], final State).  ``units`` optionally restricts the
    work to a list of flattened (b*H + h) indices (others stay zero).
    """
    return _run("m3o_scan_complex", x, B, C, theta, dt, lam, A, D, init, True, nthreads, units)


def scan_rope(x, B, C, theta, dt, lam, A, D=None, init=None, nthreads=None, units=None):
    """Real state with B, C rotated by -Phi_t (the RoPE form)."""
    return _run("m3o_scan_rope", x, B, C, theta, dt, lam, A, D, init, True, nthreads, units)


def scan_quadratic(x, B, C, theta, dt, lam, A, D=None, init=None, nthreads=None):
    """Materialised L x L masked-kernel form (brute force; tiny L only). Returns y."""
    y, _ = _run("m3o_scan_quadratic", x, B, C, theta, dt, lam, A, D, init, False, nthreads)
    return y


def decode_step(state: State, x, B, C, theta, dt, lam, A, D=None, nthreads=None):
    """One token continued from ``state``.

    Per-token inputs are shaped without the L axis: x [b,H,R,P], B/C [b,H,R,N],
    theta [b,H,N/2], dt/lam [b,H]; A is [H] or, time-varying, [b,H].
    Returns (y [b,H,R,P], new State).
    """
    add = lambda a: _f64(a)[:, None]
    A = _f64(A)
    y, fin = _run("m3o_decode_step", add(x), add(B), add(C), add(theta), add(dt), add(lam),
                  add(A) if A.ndim == 2 else A, D, state, True, nthreads)
    return y[:, 0], fin


def scan_bwd(x, B, C, theta, dt, lam, A, D, dy, init: Optional[State] = None,
             d_final: Optional[State] = None, nthreads=None) -> dict:
    """Gradients of the prefill (y and, with ``d_final``, the exported state) by
    reverse-mode differentiation of the RoPE form, token by token (the pages give
    no gradient formulas; the oracle's C source states the steps).

    dy is shaped like x; ``d_final`` holds the gradients of the exported state.
    Returns a dict: dx, dB, dC (shaped like x, B, C; grouped B, C get their
    heads' sums), dtheta, ddt, dlam (like theta, dt, lam), dA (like A: [H]
    summed over batch and tokens, or [b, L, H]), dD ([H]), and dh0, dbprev0,
    dxprev0, dangle0 (the initial state's, zero-state inputs included)."""
    dims, arrs = _prepare(x, B, C, theta, dt, lam, A, D)
    x, B, C, theta, dt, lam, A, D = arrs
    b, L, H, R, P = x.shape
    N = B.shape[-1]
    G = B.shape[2]
    dy = _f64(dy)
    assert dy.shape == x.shape, "dy must be shaped like x"
    A_t = None
    if A.ndim == 3:
        A_t, A = A, np.zeros(H)
    out = {
        "dx": np.zeros_like(x), "dB": np.zeros((b, L, H, R, N)), "dC": np.zeros((b, L, H, R, N)),
        "dtheta": np.zeros_like(theta), "ddt": np.zeros_like(dt), "dlam": np.zeros_like(lam),
        "dA": np.zeros((b, L, H)) if A_t is not None else np.zeros((b, H)), "dD": np.zeros((b, H)),
    }
    st0 = State.zeros(b, H, P, N, R)
    out.update(dh0=st0.h.copy(), dbprev0=st0.b_prev.copy(), dxprev0=st0.x_prev.copy(), dangle0=st0.angle.copy())
    keep = [x, B, C, theta, dt, lam, A, A_t, D, dy]
    io = _IO()
    io.x, io.B, io.C, io.theta, io.dt, io.lam, io.A, io.D = map(_ptr, (x, B, C, theta, dt, lam, A, D))
    io.A_t = _ptr(A_t)
    if init is not None:
        ih, ib, ix, ia = (_f64(init.h), _f64(init.b_prev), _f64(init.x_prev), _f64(init.angle))
        keep += [ih, ib, ix, ia]
        io.h0, io.bprev0, io.xprev0, io.angle0 = map(_ptr, (ih, ib, ix, ia))
    gr = _Grad()
    gr.dy = _ptr(dy)
    if d_final is not None:
        fh, fb, fx, fa = (_f64(d_final.h), _f64(d_final.b_prev), _f64(d_final.x_prev), _f64(d_final.angle))
        keep += [fh, fb, fx, fa]
        gr.dh_out, gr.dbprev_out, gr.dxprev_out, gr.dangle_out = map(_ptr, (fh, fb, fx, fa))
    for n in ("dx", "dB", "dC", "dtheta", "ddt", "dlam", "dA", "dD", "dh0", "dbprev0", "dxprev0", "dangle0"):
        setattr(gr, n, _ptr(out[n]))
    io.grad = ctypes.cast(ctypes.pointer(gr), ctypes.c_void_p)
    nt = nthreads if nthreads is not None else (os.cpu_count() or 1)
    rc = _load().m3o_scan_rope_bwd(ctypes.byref(dims), ctypes.byref(io), nt)
    if rc != 0:
        raise ValueError(f"m3o_scan_rope_bwd rejected its arguments (rc={rc})")
    if G != H:  # a shared row's gradient is the sum over the heads that read it
        out["dB"] = out["dB"].reshape(b, L, G, H // G, R, N).sum(axis=3)
        out["dC"] = out["dC"].reshape(b, L, G, H // G, R, N).sum(axis=3)
    if A_t is None:
        out["dA"] = out["dA"].sum(axis=0)
    out["dD"] = out["dD"].sum(axis=0)
    return out


def gated_norm(y, z, w=None, groups: Optional[int] = None, eps: float = 1e-6) -> np.ndarray:
    """Pre-gate grouped RMS norm and gate of the layer output: y, z [..., H, R, P]
    (leading axes flattened to tokens), w [H, R, P] or None, ``groups`` norm
    groups of H / groups consecutive heads (default H: one per head).  Source:
    "Mamba-3: 2x smaller state ..." (MarkTechPost, Korean translation), section 2
    (grouped RMS norm ahead of the gate); the gate is silu(z)."""
    y, z = _f64(y), _f64(z)
    assert y.shape == z.shape, "y and z must have the same shape"
    *lead, H, R, P = y.shape
    groups = H if groups is None else groups
    rows = int(np.prod(lead)) if lead else 1
    dims = _Dims(1, rows, H, P, 0, R, 0)
    w = _f64(w) if w is not None else None
    assert w is None or w.shape == (H, R, P), "w must be [H, R, P]"
    out = np.empty_like(y)
    rc = _load().m3o_gated_norm(ctypes.byref(dims), int(groups), _ptr(y), _ptr(z), _ptr(w), float(eps), _ptr(out))
    if rc != 0:
        raise ValueError("groups must divide the number of heads")
    return out


def mimo_up(u, Wx, rank: int) -> np.ndarray:
    """MIMO input projection (rank R) per head: u [..., H, P], Wx [H, R P, P]
    -> x [..., H, R, P] with x[.., h, r, p] = sum_q Wx[h, r P + p, q] u[.., h, q].
    Source: "Mamba-3: 2x smaller state ..." (MarkTechPost, Korean translation),
    section 1.3 (x_t is P x R); one dense matrix per head is this build's reading."""
    u, Wx = _f64(u), _f64(Wx)
    *lead, H, P = u.shape
    assert Wx.shape == (H, rank * P, P), "Wx must be [H, R P, P]"
    rows = int(np.prod(lead)) if lead else 1
    dims = _Dims(1, rows, H, P, 0, rank, 0)
    x = np.empty((*lead, H, rank, P))
    _load().m3o_mimo_up(ctypes.byref(dims), _ptr(u), _ptr(Wx), _ptr(x))
    return x


def mimo_down(y, Wy) -> np.ndarray:
    """MIMO output projection per head: y [..., H, R, P], Wy [H, P, R P] -> o
    [..., H, P] with o[.., h, p] = sum_{r, q} Wy[h, p, r P + q] y[.., h, r, q]
    (same page and reading as mimo_up)."""
    y, Wy = _f64(y), _f64(Wy)
    *lead, H, R, P = y.shape
    assert Wy.shape == (H, P, R * P), "Wy must be [H, P, R P]"
    rows = int(np.prod(lead)) if lead else 1
    dims = _Dims(1, rows, H, P, 0, R, 0)
    o = np.empty((*lead, H, P))
    _load().m3o_mimo_down(ctypes.byref(dims), _ptr(y), _ptr(Wy), _ptr(o))
    return o


__all__ = ["build", "State", "scan_complex", "scan_rope", "scan_quadratic", "decode_step", "bc_norm", "scan_bwd",
           "gated_norm", "mimo_up", "mimo_down"]


def bc_norm(z, w=None, bias=None, eps: float = 1e-6) -> np.ndarray:
    """RMS normalisation of raw B or C projections over the state dimension N,
    then a per-(head, rank) weight and bias: z [..., L, H, R, N] (leading batch
    dims flattened), w, bias [H, R, N] or None.  Source: "Mamba-3: 2x smaller
    state ..." (MarkTechPost, Korean translation), section 2 (B/C norm and
    head-specific bias)."""
    z = _f64(z)
    *lead, H, R, N = z.shape
    rows = int(np.prod(lead)) if lead else 1
    dims = _Dims(1, rows, H, 0, N, R, 0)
    w = _f64(w) if w is not None else None
    bias = _f64(bias) if bias is not None else None
    for a in (w, bias):
        assert a is None or a.shape == (H, R, N), "weight and bias must be [H, R, N]"
    out = np.empty_like(z)
    _load().m3o_bc_norm(ctypes.byref(dims), _ptr(z), _ptr(w), _ptr(bias), float(eps), _ptr(out))
    return out
