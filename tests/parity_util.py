"""Helpers shared by the GPU parity tests: run the CUDA path and the fp64
oracle on the same seeded inputs and compare with max|err| / max|ref|."""
from __future__ import annotations

import numpy as np
import torch

import linear_recurrent_scan_b200 as m3
import oracle
from linear_recurrent_scan_b200 import workloads as wl
from tests.conftest import rel_err

# Tolerances on max|err| / max|ref| (fp32 inputs; bf16 inputs with fp32 accumulation).
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}

NAMES = ("x", "B", "C", "theta", "dt", "lam")


def small_inputs(b, L, H, P, N, R, dtype, seed=wl.BASE_SEED, device="cuda"):
    w = wl.Workload("case", b, L, H, P, N, R, dtype)
    return wl.make_inputs(w, seed=seed, device=device)


def to_state_np(st: m3.State) -> oracle.State:
    f = lambda t: t.detach().to("cpu", torch.float64).numpy()
    return oracle.State(f(st.h), f(st.b_prev), f(st.x_prev), f(st.angle))


def gpu_scan(inp, init: m3.State = None, chunk=0, export=True):
    x = inp["x"]
    b, L, H, R, P = x.shape
    N = inp["B"].shape[-1]
    fin = m3.State.zeros(b, H, P, N, R, device=x.device) if export else None
    y = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], init=init, final_state=fin, chunk=chunk)
    torch.cuda.synchronize()
    return y, fin


def oracle_scan(inp, init: oracle.State = None, units=None):
    f = wl.to_f64({k: inp[k] for k in (*NAMES, "A", "D")})
    return oracle.scan_complex(**f, init=init, units=units)


def angle_err(a, b):
    d = np.asarray(a, np.float64) - np.asarray(b, np.float64)
    return float(np.max(np.abs(np.angle(np.exp(1j * d))))) if d.size else 0.0


def check_state(gpu: m3.State, ref: oracle.State, tol, units=None):
    g = to_state_np(gpu)
    sel = (lambda a: a) if units is None else (lambda a: a.reshape(-1, *a.shape[2:])[units])
    errs = {
        "h": rel_err(sel(g.h), sel(ref.h)),
        "b_prev": rel_err(sel(g.b_prev), sel(ref.b_prev)),
        "x_prev": rel_err(sel(g.x_prev), sel(ref.x_prev)),
        "angle": angle_err(sel(g.angle), sel(ref.angle)),
    }
    for k, e in errs.items():
        assert e <= (tol if k != "angle" else 1e-3), (k, e, errs)
    return errs


def unit_rows(y, units, nheads):
    """Select flattened (b*H + h) units from [b, L, H, ...] -> [n_units, L, ...]."""
    y = np.asarray(y)
    return np.stack([y[u // nheads, :, u % nheads] for u in units])
