"""The prefill entry point that allocates nothing (mamba3_scan_fwd_noalloc).

Some callers cannot call cudaMalloc themselves: code embedded in a host
framework whose pool owns all device memory, latency-critical serving loops
(an allocation may synchronise the device), runtimes with a budget fixed at
start-up.  For them the library keeps its scratch in a file-scope device array.
This test calls that entry point through the C ABI twice in a row and checks
each result against the workspace entry point on the same inputs.  It lives in
a file of its own so that it is collected after every other test.
"""
import pytest
import torch

import linear_recurrent_scan_b200 as m3
from linear_recurrent_scan_b200 import build as m3build
from tests.conftest import rel_err
from tests.parity_util import NAMES, TOL, small_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()


def _state_err(a: m3.State, b: m3.State):
    return max(rel_err(x.cpu().double().numpy(), y.cpu().double().numpy())
               for x, y in ((a.h, b.h), (a.b_prev, b.b_prev), (a.x_prev, b.x_prev), (a.angle, b.angle)))


@pytest.mark.parametrize("shape,dtype", [
    ((2, 300, 3, 64, 128, 1), torch.bfloat16),   # tensor-core kernel
    ((1, 150, 2, 64, 64, 4), torch.bfloat16),    # tensor-core kernel, MIMO
    ((2, 130, 2, 16, 16, 2), torch.float32),     # SIMT kernel
])
def test_noalloc_matches_workspace_entry_point(shape, dtype):
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, dtype, seed=1234 + L)
    args = [inp[n] for n in NAMES]
    ref_state = m3.State.zeros(b, H, P, N, R)
    y_ref = m3.mamba3_scan_fwd(*args, inp["A"], inp["D"], final_state=ref_state)
    torch.cuda.synchronize()
    for call in range(2):  # the shared scratch keeps the previous call's contents
        st = m3.State.zeros(b, H, P, N, R)
        y = torch.full_like(inp["x"], float("nan"))
        m3.mamba3_scan_fwd_noalloc(*args, inp["A"], inp["D"], y=y, final_state=st)
        torch.cuda.synchronize()
        assert rel_err(y.float().cpu().double().numpy(), y_ref.float().cpu().double().numpy()) < TOL[dtype], call
        assert _state_err(st, ref_state) < TOL[dtype], call
