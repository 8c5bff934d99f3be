"""Bounded device waits: a kernel whose waits cannot be met reports
MAMBA3_ERR_TIMEOUT and leaves the context usable.

The failure is made on the host: mamba3_test_withhold_loads makes the prefill's
producer and the decode step issue none of their input copies, so every wait on
those copies runs out after the (shortened) wait limit.  Nothing faults, traps
or hangs: the kernels give up, let whatever they issued complete, free their
tensor memory and return.  The next normal call on the same stream must succeed
and match the oracle."""
import pytest
import torch

import linear_recurrent_scan_b200 as m3
from linear_recurrent_scan_b200 import build as m3build
from tests.conftest import rel_err
from tests.parity_util import NAMES, TOL, oracle_scan, small_inputs

pytestmark = pytest.mark.gpu

SHORT = 2_000_000  # SM cycles (about 1 ms): each starved wait gives up after this


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()
    yield
    m3.mamba3_test_withhold_loads(False)
    m3.mamba3_set_wait_limit(4_000_000_000)


def _starved(fn):
    m3.mamba3_set_wait_limit(SHORT)
    m3.mamba3_test_withhold_loads(True)
    try:
        return fn()
    finally:
        m3.mamba3_test_withhold_loads(False)
        m3.mamba3_set_wait_limit(4_000_000_000)


@pytest.mark.parametrize("shape", [(1, 200, 3, 64, 128, 1), (2, 100, 2, 64, 64, 4)])
def test_prefill_timeout_is_reported_and_context_survives(shape):
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=5100 + L)
    dims = m3.make_dims(inp["x"], inp["B"])
    ws = torch.zeros(m3.mamba3_scan_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(inp["x"])
    _starved(lambda: m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], y=y, workspace=ws))
    assert m3.mamba3_device_status(ws) == m3.MAMBA3_ERR_TIMEOUT
    # the same stream, a normal call: status cleared, result correct
    y = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], y=y, workspace=ws)
    assert m3.mamba3_device_status(ws) == m3.MAMBA3_OK
    yr, _ = oracle_scan(inp)
    assert rel_err(y.float().cpu().double().numpy(), yr) < TOL[torch.bfloat16]


def test_decode_timeout_is_reported_and_context_survives():
    b, H, P, N, R = 4, 8, 64, 128, 1
    pre = small_inputs(b, 1, H, P, N, R, torch.bfloat16, seed=5200)
    st = m3.State.zeros(b, H, P, N, R, device="cuda")
    step = {n: pre[n][:, 0].contiguous() for n in NAMES}
    assert m3.mamba3_library_status() == m3.MAMBA3_OK
    _starved(lambda: m3.mamba3_decode_step(st, *(step[n] for n in NAMES), pre["A"], pre["D"]))
    assert m3.mamba3_library_status() == m3.MAMBA3_ERR_TIMEOUT
    assert m3.mamba3_library_status() == m3.MAMBA3_OK  # read and cleared
    # a normal step from a fresh zero state equals the one-token prefill
    st = m3.State.zeros(b, H, P, N, R, device="cuda")
    y = m3.mamba3_decode_step(st, *(step[n] for n in NAMES), pre["A"], pre["D"])
    assert m3.mamba3_library_status() == m3.MAMBA3_OK
    yr, _ = oracle_scan(pre)
    assert rel_err(y.float().cpu().double().numpy(), yr[:, 0]) < TOL[torch.bfloat16]


def test_segmented_prefill_timeout_is_reported_and_context_survives():
    """The segmented path (segment end states, their chaining, the prefill of the
    segments) with every input copy withheld: the segment-state pass and the prefill
    pass give up, the status says so, and the next call is correct."""
    b, L, H, P, N, R = 1, 512, 2, 64, 64, 4
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=5300)
    dims = m3.make_dims(inp["x"], inp["B"])
    m3.mamba3_test_set_segments(4)
    try:
        need = m3.mamba3_scan_segmented_workspace_bytes(dims)
        assert need > m3.mamba3_scan_workspace_bytes(dims)  # the segmented path is taken
        ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
        y = torch.empty_like(inp["x"])
        _starved(lambda: m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], y=y, workspace=ws))
        assert m3.mamba3_device_status(ws) == m3.MAMBA3_ERR_TIMEOUT
        y = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], y=y, workspace=ws)
        assert m3.mamba3_device_status(ws) == m3.MAMBA3_OK
    finally:
        m3.mamba3_test_set_segments(0)
    yr, _ = oracle_scan(inp)
    assert rel_err(y.float().cpu().double().numpy(), yr) < TOL[torch.bfloat16]
