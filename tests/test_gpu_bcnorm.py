"""GPU vs fp64 oracle for the fused B/C normalisation (raw B, C projections,
RMS norm over N with per-(head, rank) weight and bias, then the recurrence):
the oracle normalises with ``oracle.bc_norm`` and runs its scan / decode step
on the result.  Bar: max|err| / max|ref| <= 2e-2 (bf16 inputs)."""
import numpy as np
import pytest
import torch

import linear_recurrent_scan_b200 as m3
import oracle
from linear_recurrent_scan_b200 import build as m3build
from linear_recurrent_scan_b200 import workloads as wl
from tests.conftest import rel_err
from tests.parity_util import NAMES, TOL, check_state, small_inputs, to_state_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()


def normalised(raw, norm_params, with_weights, eps):
    """The oracle's B, C from the raw projections (fp64)."""
    f = wl.to_f64(raw)
    p = wl.to_f64(norm_params) if with_weights else {}
    B = oracle.bc_norm(f["B_raw"], p.get("w_B"), p.get("bias_B"), eps)
    C = oracle.bc_norm(f["C_raw"], p.get("w_C"), p.get("bias_C"), eps)
    return B, C


def norm_of(raw, with_weights, eps):
    if not with_weights:
        return m3.BCNorm(eps=eps)
    return m3.BCNorm(raw["w_B"], raw["w_C"], raw["bias_B"], raw["bias_C"], eps)


@pytest.mark.parametrize("shape", [(2, 200, 8, 64, 128, 1), (1, 150, 16, 64, 64, 4), (2, 97, 3, 64, 128, 2),
                                   (1, 64, 8, 64, 128, 4)])
@pytest.mark.parametrize("with_weights", [True, False])
def test_prefill_bcnorm_matches_oracle(shape, with_weights):
    b, L, H, P, N, R = shape
    eps = 1e-6
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=800 + L)
    raw = wl.raw_bc_inputs(inp, seed=900 + L)
    fin = m3.State.zeros(b, H, P, N, R)
    y = m3.mamba3_scan_fwd_bcnorm(inp["x"], raw["B_raw"], raw["C_raw"], inp["theta"], inp["dt"], inp["lam"],
                                  inp["A"], inp["D"], norm=norm_of(raw, with_weights, eps), final_state=fin)
    torch.cuda.synchronize()
    Bn, Cn = normalised(raw, raw, with_weights, eps)
    f = wl.to_f64({k: inp[k] for k in (*NAMES, "A", "D")})
    f["B"], f["C"] = Bn, Cn
    yr, fr = oracle.scan_complex(**f)
    e = rel_err(y.float().cpu().double().numpy(), yr)
    assert e < TOL[torch.bfloat16], e
    check_state(fin, fr, TOL[torch.bfloat16])


def test_prefill_bcnorm_scale_invariant_on_gpu():
    """Scaling the raw rows (by powers of two, exact in bf16) leaves the
    normalised B, C and hence y and the state unchanged (within the bf16 bar;
    a missing or misplaced norm changes them by the scale factors)."""
    b, L, H, P, N, R = 1, 100, 8, 64, 128, 2
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=811)
    raw = wl.raw_bc_inputs(inp, seed=812)
    norm = norm_of(raw, True, 0.0)
    args = (inp["theta"], inp["dt"], inp["lam"], inp["A"], inp["D"])
    f1, f2 = m3.State.zeros(b, H, P, N, R), m3.State.zeros(b, H, P, N, R)
    y1 = m3.mamba3_scan_fwd_bcnorm(inp["x"], raw["B_raw"], raw["C_raw"], *args, norm=norm, final_state=f1)
    y2 = m3.mamba3_scan_fwd_bcnorm(inp["x"], raw["B_raw"] * 8, raw["C_raw"] * 0.25, *args, norm=norm, final_state=f2)
    torch.cuda.synchronize()
    assert rel_err(y2.float().cpu().double().numpy(), y1.float().cpu().double().numpy()) < TOL[torch.bfloat16]
    assert rel_err(f2.h.cpu().double().numpy(), f1.h.cpu().double().numpy()) < TOL[torch.bfloat16]
    assert rel_err(f2.b_prev.cpu().double().numpy(), f1.b_prev.cpu().double().numpy()) < TOL[torch.bfloat16]


@pytest.mark.parametrize("R", [1, 4])
def test_decode_bcnorm_steps_match_oracle(R):
    """Fused prefill of L0 tokens, then fused decode steps == the oracle's longer
    prefill of the normalised inputs."""
    b, H, P, N, L0, S = 3, 8, 64, 128, 70, 7
    eps = 1e-6
    inp = small_inputs(b, L0 + S, H, P, N, R, torch.bfloat16, seed=820 + R)
    raw = wl.raw_bc_inputs(inp, seed=830 + R)
    norm = norm_of(raw, True, eps)
    pre = {n: inp[n][:, :L0].contiguous() for n in ("x", "theta", "dt", "lam")}
    st = m3.State.zeros(b, H, P, N, R)
    m3.mamba3_scan_fwd_bcnorm(pre["x"], raw["B_raw"][:, :L0].contiguous(), raw["C_raw"][:, :L0].contiguous(),
                              pre["theta"], pre["dt"], pre["lam"], inp["A"], inp["D"], norm=norm, final_state=st)
    ys = []
    for t in range(L0, L0 + S):
        ys.append(m3.mamba3_decode_step_bcnorm(st, inp["x"][:, t].contiguous(), raw["B_raw"][:, t].contiguous(),
                                               raw["C_raw"][:, t].contiguous(), inp["theta"][:, t].contiguous(),
                                               inp["dt"][:, t].contiguous(), inp["lam"][:, t].contiguous(),
                                               inp["A"], inp["D"], norm=norm))
    torch.cuda.synchronize()
    Bn, Cn = normalised(raw, raw, True, eps)
    f = wl.to_f64({k: inp[k] for k in (*NAMES, "A", "D")})
    f["B"], f["C"] = Bn, Cn
    yr, fr = oracle.scan_complex(**f)
    yg = torch.stack(ys, 1).float().cpu().double().numpy()
    assert rel_err(yg, yr[:, L0:]) < TOL[torch.bfloat16]
    check_state(st, fr, TOL[torch.bfloat16])


def test_plain_and_fused_agree_on_prenormalised_inputs():
    """The fused path with unit weight, zero bias and eps = 0 on raw rows that
    already have RMS 1 (within bf16) stays within the bf16 bar of the plain path."""
    b, L, H, P, N, R = 1, 130, 8, 64, 128, 1
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=840)
    Bf = inp["B"].float()
    Bu = (Bf / Bf.pow(2).mean(-1, keepdim=True).sqrt()).to(torch.bfloat16)
    Cf = inp["C"].float()
    Cu = (Cf / Cf.pow(2).mean(-1, keepdim=True).sqrt()).to(torch.bfloat16)
    y_plain = m3.mamba3_scan_fwd(inp["x"], Bu, Cu, inp["theta"], inp["dt"], inp["lam"], inp["A"], inp["D"])
    y_fused = m3.mamba3_scan_fwd_bcnorm(inp["x"], Bu, Cu, inp["theta"], inp["dt"], inp["lam"], inp["A"], inp["D"],
                                        norm=m3.BCNorm(eps=0.0))
    torch.cuda.synchronize()
    assert rel_err(y_fused.float().cpu().double().numpy(), y_plain.float().cpu().double().numpy()) < TOL[torch.bfloat16]
