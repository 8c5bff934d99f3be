"""GPU vs fp64 oracle for the time-varying decay: A_t per (batch, token, head) in
place of A per head (alpha_t = exp(dt_t A_t)).  The oracle takes A as [b, L, H].
Bars: 1e-4 (fp32 inputs), 2e-2 (bf16 inputs)."""
import pytest
import torch

import linear_recurrent_scan_b200 as m3
import oracle
from linear_recurrent_scan_b200 import build as m3build
from linear_recurrent_scan_b200 import workloads as wl
from tests.conftest import rel_err
from tests.parity_util import NAMES, TOL, check_state, small_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()


def oracle_at(inp, A_t):
    f = wl.to_f64({k: inp[k] for k in (*NAMES, "D")})
    f["A"] = wl.to_f64({"A": A_t})["A"]
    return oracle.scan_complex(**f)


@pytest.mark.parametrize("shape,dtype", [
    ((2, 200, 8, 64, 128, 1), torch.bfloat16),   # tensor cores, dt/lam/A_t tiles by TMA
    ((1, 150, 16, 64, 64, 4), torch.bfloat16),
    ((2, 97, 3, 64, 128, 2), torch.bfloat16),    # H % 8 != 0: global loads one chunk ahead
    ((1, 64, 8, 64, 128, 4), torch.bfloat16),
    ((2, 130, 3, 16, 16, 2), torch.float32),     # SIMT path
])
def test_prefill_time_varying_decay_matches_oracle(shape, dtype):
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, dtype, seed=1100 + L)
    A_t = wl.decay_rates(inp["dt"], seed=1200 + L)
    fin = m3.State.zeros(b, H, P, N, R)
    y = m3.mamba3_scan_fwd_at(*(inp[n] for n in NAMES), A_t, inp["D"], final_state=fin)
    torch.cuda.synchronize()
    yr, fr = oracle_at(inp, A_t)
    e = rel_err(y.float().cpu().double().numpy(), yr)
    assert e < TOL[dtype], e
    check_state(fin, fr, TOL[dtype])


@pytest.mark.parametrize("R", [1, 4])
def test_constant_rates_reproduce_the_per_head_path(R):
    """A_t[b, t, h] = A[h] with rates exact in bf16: the same arithmetic as the
    plain path, so y and the state agree bit for bit."""
    b, L, H, P, N = 2, 180, 8, 64, 128
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=1300 + R)
    inp["A"] = -torch.tensor([0.5, 1.0, 2.0, 3.0, 4.0, 6.0, 8.0, 16.0], device="cuda")
    A_t = inp["A"].to(torch.bfloat16).expand(b, L, H).contiguous()
    f1, f2 = m3.State.zeros(b, H, P, N, R), m3.State.zeros(b, H, P, N, R)
    y1 = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], final_state=f1)
    y2 = m3.mamba3_scan_fwd_at(*(inp[n] for n in NAMES), A_t, inp["D"], final_state=f2)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert torch.equal(f1.h, f2.h)


@pytest.mark.parametrize("P,dtype", [(64, torch.bfloat16), (16, torch.float32)])
def test_decode_time_varying_decay_matches_oracle(P, dtype):
    """Prefill L0 tokens, then decode steps, all with per-token rates, against the
    oracle's one longer prefill (P = 64: streaming decode; P = 16: per-unit decode)."""
    b, H, N, R, L0, S = 3, 8, 64 if P == 64 else 16, 2, 60, 6
    inp = small_inputs(b, L0 + S, H, P, N, R, dtype, seed=1400 + P)
    A_t = wl.decay_rates(inp["dt"], seed=1500 + P)
    pre = {n: inp[n][:, :L0].contiguous() for n in NAMES}
    st = m3.State.zeros(b, H, P, N, R)
    m3.mamba3_scan_fwd_at(*(pre[n] for n in NAMES), A_t[:, :L0].contiguous(), inp["D"], final_state=st)
    ys = []
    for t in range(L0, L0 + S):
        ys.append(m3.mamba3_decode_step_at(st, *(inp[n][:, t].contiguous() for n in NAMES),
                                           A_t[:, t].contiguous(), inp["D"]))
    torch.cuda.synchronize()
    yr, fr = oracle_at(inp, A_t)
    yg = torch.stack(ys, 1).float().cpu().double().numpy()
    assert rel_err(yg, yr[:, L0:]) < TOL[dtype]
    check_state(st, fr, TOL[dtype])
