"""GPU vs fp64 oracle for grouped B/C: B and C [b, L, G, R, N] shared by groups
of H / G consecutive heads (head h reads group h // (H // G)).  The oracle takes
the grouped arrays as they are.  Bars: 1e-4 (fp32 inputs), 2e-2 (bf16 inputs);
grouped against the same rows repeated per head: bit for bit."""
import numpy as np
import pytest
import torch

import linear_recurrent_scan_b200 as m3
import oracle
from linear_recurrent_scan_b200 import build as m3build
from linear_recurrent_scan_b200 import workloads as wl
from tests.conftest import rel_err
from tests.parity_util import NAMES, TOL, check_state, gpu_scan, oracle_scan, small_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()


def grouped_inputs(b, L, H, P, N, R, G, dtype, seed):
    inp = small_inputs(b, L, H, P, N, R, dtype, seed=seed)
    inp.update(wl.grouped_bc(inp, G, seed=seed + 1))
    return inp


def per_head(inp, H):
    G = inp["B"].shape[-3]
    return dict(inp, B=inp["B"].repeat_interleave(H // G, dim=-3).contiguous(),
                C=inp["C"].repeat_interleave(H // G, dim=-3).contiguous())


@pytest.mark.parametrize("shape,G,dtype", [
    ((2, 200, 8, 64, 128, 1), 1, torch.bfloat16),   # tensor cores, all heads share one B/C row
    ((2, 200, 8, 64, 128, 1), 2, torch.bfloat16),
    ((1, 150, 16, 64, 64, 4), 4, torch.bfloat16),
    ((2, 97, 6, 64, 128, 2), 3, torch.bfloat16),    # H % 8 != 0
    ((1, 64, 8, 64, 128, 4), 8, torch.bfloat16),    # G = H: the per-head layout
    ((2, 130, 6, 16, 16, 2), 2, torch.float32),     # SIMT path
    ((1, 70, 4, 32, 8, 1), 1, torch.float32),
])
def test_prefill_grouped_matches_oracle(shape, G, dtype):
    b, L, H, P, N, R = shape
    inp = grouped_inputs(b, L, H, P, N, R, G, dtype, seed=1600 + L + G)
    y, fin = gpu_scan(inp)
    yr, fr = oracle_scan(inp)
    e = rel_err(y.float().cpu().double().numpy(), yr)
    assert e < TOL[dtype], e
    check_state(fin, fr, TOL[dtype])


@pytest.mark.parametrize("shape,G,dtype", [
    ((2, 300, 8, 64, 128, 1), 2, torch.bfloat16),
    ((1, 150, 16, 64, 64, 4), 4, torch.bfloat16),
    ((2, 130, 6, 16, 16, 2), 3, torch.float32),
])
def test_grouped_equals_per_head_repeat(shape, G, dtype):
    """The same rows given once per group or repeated per head: the kernels read
    identical values, so y and the state agree bit for bit."""
    b, L, H, P, N, R = shape
    inp = grouped_inputs(b, L, H, P, N, R, G, dtype, seed=1700 + L)
    y1, f1 = gpu_scan(inp)
    y2, f2 = gpu_scan(per_head(inp, H))
    assert torch.equal(y1, y2)
    for n in ("h", "b_prev", "x_prev", "angle"):
        assert torch.equal(getattr(f1, n), getattr(f2, n)), n


@pytest.mark.parametrize("P,R,dtype", [(64, 1, torch.bfloat16), (64, 4, torch.bfloat16), (16, 2, torch.float32)])
def test_decode_grouped_matches_oracle(P, R, dtype):
    """Grouped prefill of L0 tokens, then grouped decode steps, against the
    oracle's one longer prefill (P = 64: streaming decode; P = 16: per-unit decode)."""
    b, H, G, L0, S = 3, 8, 2, 60, 6
    N = 128 if P == 64 else 16
    inp = grouped_inputs(b, L0 + S, H, P, N, R, G, dtype, seed=1800 + P + R)
    pre = {n: inp[n][:, :L0].contiguous() for n in NAMES}
    st = m3.State.zeros(b, H, P, N, R)
    m3.mamba3_scan_fwd(*(pre[n] for n in NAMES), inp["A"], inp["D"], final_state=st)
    ys = []
    for t in range(L0, L0 + S):
        ys.append(m3.mamba3_decode_step(st, *(inp[n][:, t].contiguous() for n in NAMES), inp["A"], inp["D"]))
    torch.cuda.synchronize()
    yr, fr = oracle_scan(inp)
    yg = torch.stack(ys, 1).float().cpu().double().numpy()
    assert rel_err(yg, yr[:, L0:]) < TOL[dtype]
    check_state(st, fr, TOL[dtype])


def test_grouped_bcnorm_prefill_and_decode():
    """Grouped raw projections with the fused B/C norm: each head normalises the
    shared row and applies its own weight and bias (the oracle: the rows repeated
    per head, then oracle.bc_norm)."""
    b, L0, S, H, P, N, R, G = 2, 150, 4, 8, 64, 128, 2, 2
    inp = small_inputs(b, L0 + S, H, P, N, R, torch.bfloat16, seed=1900)
    raw = wl.raw_bc_inputs(inp, seed=1901)
    grp = wl.grouped_bc(inp, G, seed=1902)
    norm = m3.BCNorm(raw["w_B"], raw["w_C"], raw["bias_B"], raw["bias_C"], 1e-6)
    st = m3.State.zeros(b, H, P, N, R)
    m3.mamba3_scan_fwd_bcnorm(inp["x"][:, :L0].contiguous(), grp["B"][:, :L0].contiguous(),
                              grp["C"][:, :L0].contiguous(), *(inp[n][:, :L0].contiguous() for n in NAMES[3:]),
                              inp["A"], inp["D"], norm=norm, final_state=st)
    ys = []
    for t in range(L0, L0 + S):
        ys.append(m3.mamba3_decode_step_bcnorm(st, inp["x"][:, t].contiguous(), grp["B"][:, t].contiguous(),
                                               grp["C"][:, t].contiguous(),
                                               *(inp[n][:, t].contiguous() for n in NAMES[3:]),
                                               inp["A"], inp["D"], norm=norm))
    torch.cuda.synchronize()
    f = wl.to_f64({k: inp[k] for k in (*NAMES, "A", "D")})
    p = wl.to_f64({k: raw[k] for k in ("w_B", "w_C", "bias_B", "bias_C")})
    rep = wl.to_f64(per_head(grp, H))
    f["B"] = oracle.bc_norm(rep["B"], p["w_B"], p["bias_B"], 1e-6)
    f["C"] = oracle.bc_norm(rep["C"], p["w_C"], p["bias_C"], 1e-6)
    yr, fr = oracle.scan_complex(**f)
    yg = torch.stack(ys, 1).float().cpu().double().numpy()
    assert rel_err(yg, yr[:, L0:]) < TOL[torch.bfloat16]
    check_state(st, fr, TOL[torch.bfloat16])


def test_grouped_time_varying_decay():
    b, L, H, P, N, R, G = 2, 200, 8, 64, 128, 1, 4
    inp = grouped_inputs(b, L, H, P, N, R, G, torch.bfloat16, seed=2000)
    A_t = wl.decay_rates(inp["dt"], seed=2001)
    fin = m3.State.zeros(b, H, P, N, R)
    y = m3.mamba3_scan_fwd_at(*(inp[n] for n in NAMES), A_t, inp["D"], final_state=fin)
    torch.cuda.synchronize()
    f = wl.to_f64({k: inp[k] for k in (*NAMES, "D")})
    f["A"] = wl.to_f64({"A": A_t})["A"]
    yr, fr = oracle.scan_complex(**f)
    assert rel_err(y.float().cpu().double().numpy(), yr) < TOL[torch.bfloat16]
    check_state(fin, fr, TOL[torch.bfloat16])


def test_grouped_full_size_sampled_units():
    """The SISO prefill size (b8 L2048 H64 N128) with 8 groups of 8 heads: sampled
    units against the oracle (units restricts the oracle to those heads)."""
    b, L, H, P, N, R, G = 8, 2048, 64, 64, 128, 1, 8
    inp = grouped_inputs(b, L, H, P, N, R, G, torch.bfloat16, seed=2100)
    y, fin = gpu_scan(inp)
    units = [0, 7, 8, 63, 64 * 3 + 17, 64 * 8 - 1]
    yr, fr = oracle_scan(inp, units=units)
    yg = y.float().cpu().double().numpy()
    for u in units:
        bb, hh = divmod(u, H)
        assert rel_err(yg[bb, :, hh], yr[bb, :, hh]) < TOL[torch.bfloat16], u
    check_state(fin, fr, TOL[torch.bfloat16], units=units)
