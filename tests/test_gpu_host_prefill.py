"""The prefill from host buffers (mamba3_scan_fwd_host): sub-batches copied in,
computed and copied out on overlapping streams must give exactly the result of
the device call on the same inputs (every batch row is an independent set of
(b, h) units), and match the fp64 oracle at the bf16 / fp32 tolerances."""
import pytest
import torch

import linear_recurrent_scan_b200 as m3
from linear_recurrent_scan_b200 import build as m3build
from tests.conftest import rel_err
from tests.parity_util import NAMES, TOL, check_state, oracle_scan, small_inputs, to_state_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()


def rand_state(b, H, P, N, R, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g, device="cuda")
    return m3.State(r(b, H, N, P) * 0.5, r(b, H, R, N), r(b, H, R, P), r(b, H, N // 2) * 2.0)


@pytest.mark.parametrize("shape,dtype,with_init", [
    ((8, 300, 4, 64, 128, 1), torch.bfloat16, False),   # 8 sub-batches of one row
    ((5, 129, 2, 64, 64, 4), torch.bfloat16, True),      # 5 sub-batches, init state
    ((20, 70, 2, 64, 128, 2), torch.bfloat16, True),     # 8 sub-batches of 3 rows, the last of 2
    ((3, 100, 3, 16, 16, 2), torch.float32, False),      # the SIMT path
    ((1, 1, 2, 64, 128, 1), torch.bfloat16, True),       # one token
])
def test_host_prefill_equals_device_prefill(shape, dtype, with_init):
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, dtype, seed=8100 + b + L)
    init = rand_state(b, H, P, N, R, 8200 + L) if with_init else None
    fin_d = m3.State.zeros(b, H, P, N, R)
    y_d = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], init=init, final_state=fin_d)
    host = {n: inp[n].cpu().pin_memory() for n in NAMES}
    fin_h = m3.State.zeros(b, H, P, N, R)
    dims = m3.make_dims(inp["x"], inp["B"])
    stage = torch.zeros(m3.mamba3_scan_fwd_host_stage_bytes(dims), dtype=torch.uint8, device="cuda")
    y_h = m3.mamba3_scan_fwd_host(*(host[n] for n in NAMES), inp["A"], inp["D"], init=init, final_state=fin_h,
                                  stage=stage)
    torch.cuda.synchronize()
    assert m3.mamba3_device_status(stage) == m3.MAMBA3_OK
    assert torch.equal(y_h, y_d.cpu())
    for n in ("h", "b_prev", "x_prev", "angle"):
        assert torch.equal(getattr(fin_h, n), getattr(fin_d, n)), n
    yr, fr = oracle_scan(inp, init=to_state_np(init) if init is not None else None)
    assert rel_err(y_h.float().double().numpy(), yr) < TOL[dtype]
    check_state(fin_h, fr, TOL[dtype])


def test_host_prefill_back_to_back_reuses_the_stage():
    """Two calls in a row on the same stream and stage: the second must not
    overwrite slots the first is still reading, and both results must be exact."""
    b, L, H, P, N, R = 8, 200, 4, 64, 128, 1
    outs = []
    dims = None
    stage = None
    for k in range(2):
        inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=8300 + k)
        if stage is None:
            dims = m3.make_dims(inp["x"], inp["B"])
            stage = torch.zeros(m3.mamba3_scan_fwd_host_stage_bytes(dims), dtype=torch.uint8, device="cuda")
        host = {n: inp[n].cpu().pin_memory() for n in NAMES}
        y_h = m3.mamba3_scan_fwd_host(*(host[n] for n in NAMES), inp["A"], inp["D"], stage=stage)
        outs.append((inp, host, y_h))
    torch.cuda.synchronize()
    for inp, host, y_h in outs:
        y_d = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"])
        torch.cuda.synchronize()
        assert torch.equal(y_h, y_d.cpu())


def test_host_prefill_of_no_tokens_passes_the_state_through():
    """seqlen 0: nothing is copied; the final state is the initial one."""
    b, H, P, N, R = 2, 4, 64, 128, 1
    inp = small_inputs(b, 1, H, P, N, R, torch.bfloat16, seed=8400)
    host = {n: inp[n][:, :0].cpu().contiguous().pin_memory() for n in NAMES}
    init = rand_state(b, H, P, N, R, 8401)
    fin = m3.State.zeros(b, H, P, N, R)
    dims = m3.make_dims(host["x"], host["B"])
    stage = torch.zeros(m3.mamba3_scan_fwd_host_stage_bytes(dims), dtype=torch.uint8, device="cuda")
    y = m3.mamba3_scan_fwd_host(*(host[n] for n in NAMES), inp["A"], inp["D"], init=init, final_state=fin,
                                stage=stage)
    torch.cuda.synchronize()
    assert y.shape[1] == 0
    assert m3.mamba3_device_status(stage) == m3.MAMBA3_OK
    for n in ("h", "b_prev", "x_prev", "angle"):
        assert torch.equal(getattr(fin, n), getattr(init, n)), n
