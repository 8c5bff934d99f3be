"""Parity at the benchmark sizes, in the launch configuration bench.py times.

The GPU runs the whole workload; the fp64 oracle recomputes a fixed sample of
(batch, head) units (first, last and evenly spaced) over every token, and the
two are compared on those units' outputs and exported states.
"""
import numpy as np
import pytest
import torch

import linear_recurrent_scan_b200 as m3
import oracle
from linear_recurrent_scan_b200 import build as m3build
from linear_recurrent_scan_b200 import workloads as wl
from tests.conftest import rel_err
from tests.parity_util import NAMES, TOL, angle_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()


def sample_units(total, k):
    return sorted(set(int(round(i * (total - 1) / max(1, k - 1))) for i in range(k)))


def unit_inputs(inp, b, h):
    d = {n: inp[n][b:b + 1, :, h:h + 1] for n in NAMES}
    d["A"], d["D"] = inp["A"][h:h + 1], inp["D"][h:h + 1]
    return wl.to_f64(d)


def check_units(inp, y, fin, units, nheads, tol):
    for u in units:
        b, h = divmod(u, nheads)
        yr, fr = oracle.scan_complex(**unit_inputs(inp, b, h), nthreads=1)
        yg = y[b:b + 1, :, h:h + 1].float().cpu().double().numpy()
        assert rel_err(yg, yr) < tol, (u, rel_err(yg, yr))
        assert rel_err(fin.h[b, h].cpu().double().numpy(), fr.h[0, 0]) < tol, u
        assert rel_err(fin.b_prev[b, h].cpu().double().numpy(), fr.b_prev[0, 0]) < tol, u
        assert rel_err(fin.x_prev[b, h].cpu().double().numpy(), fr.x_prev[0, 0]) < tol, u
        assert angle_err(fin.angle[b, h].cpu().double().numpy(), fr.angle[0, 0]) < 1e-3, u


@pytest.mark.parametrize("name,k", [("siso_prefill_b8_l2048", 6), ("mimo4_prefill_b4_l8192", 3),
                                    ("mimo4_long_b1_l65536", 2)])
def test_prefill_full_size_sampled(name, k):
    w = wl.CONFIGS[name]
    inp = wl.make_inputs(w, device="cuda")
    fin = m3.State.zeros(w.batch, w.nheads, w.headdim, w.dstate, w.rank)
    y = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], final_state=fin)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    check_units(inp, y, fin, sample_units(w.batch * w.nheads, k), w.nheads, TOL[w.dtype])


@pytest.mark.parametrize("name", ["siso_decode_b128", "mimo4_decode_b128"])
def test_decode_full_batch_sampled(name):
    """Batch 128: a 512-token prefill seeds the state, then 16 decode steps; sampled units
    match the oracle's single 528-token prefill."""
    w = wl.CONFIGS[name]
    S = 16
    inp = wl.make_inputs(w.with_(seqlen=w.prefill_tokens + S), device="cuda")
    L0 = w.prefill_tokens
    st = m3.State.zeros(w.batch, w.nheads, w.headdim, w.dstate, w.rank)
    m3.mamba3_scan_fwd(*(inp[n][:, :L0].contiguous() for n in NAMES), inp["A"], inp["D"], final_state=st)
    ys = [m3.mamba3_decode_step(st, *(inp[n][:, t].contiguous() for n in NAMES), inp["A"], inp["D"])
          for t in range(L0, L0 + S)]
    torch.cuda.synchronize()
    ydec = torch.stack(ys, 1)
    for u in sample_units(w.batch * w.nheads, 4):
        b, h = divmod(u, w.nheads)
        yr, fr = oracle.scan_complex(**unit_inputs(inp, b, h), nthreads=1)
        assert rel_err(ydec[b:b + 1, :, h:h + 1].float().cpu().double().numpy(), yr[:, L0:]) < TOL[w.dtype], u
        assert rel_err(st.h[b, h].cpu().double().numpy(), fr.h[0, 0]) < TOL[w.dtype], u
