"""The segmented prefill of long sequences over few (batch, head) units.

Each unit's sequence is cut into S segments: the segments' end states from a
zero state, their chaining in order (decay, rotation by the entering angle,
sum), then the prefill of all segments at once.  The split is exact up to
rounding, so y and the exported state must match the fp64 oracle at the bf16
tolerance (max|err| / max|ref| <= 2e-2) and the unsegmented GPU prefill.
mamba3_test_set_segments forces S on sizes the oracle finishes quickly; the
library's own choice is exercised at the long-context size (b1 L65536 H64,
sampled units) in test_gpu_fullsize.py and here through the workspace size."""
import pytest
import torch

import linear_recurrent_scan_b200 as m3
import oracle
from linear_recurrent_scan_b200 import build as m3build
from linear_recurrent_scan_b200 import workloads as wl
from tests.conftest import rel_err
from tests.parity_util import NAMES, TOL, check_state, oracle_scan, small_inputs, to_state_np

pytestmark = pytest.mark.gpu
TOLB = TOL[torch.bfloat16]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()
    yield
    m3.mamba3_test_set_segments(0)


def rand_state(b, H, P, N, R, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g, device="cuda")
    return m3.State(r(b, H, N, P) * 0.5, r(b, H, R, N), r(b, H, R, P), r(b, H, N // 2) * 2.0)


def run_segmented(inp, S, init=None, A_t=None):
    x = inp["x"]
    b, L, H, R, P = x.shape
    N = inp["B"].shape[-1]
    m3.mamba3_test_set_segments(S)
    try:
        dims = m3.make_dims(x, inp["B"])
        need = m3.mamba3_scan_segmented_workspace_bytes(dims)
        assert need > m3.mamba3_scan_workspace_bytes(dims)  # the segmented path is taken
        ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
        fin = m3.State.zeros(b, H, P, N, R)
        if A_t is None:
            y = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], init=init, final_state=fin,
                                   workspace=ws)
        else:
            y = m3.mamba3_scan_fwd_at(*(inp[n] for n in NAMES), A_t, inp["D"], init=init, final_state=fin,
                                      workspace=ws)
        assert m3.mamba3_device_status(ws) == m3.MAMBA3_OK
    finally:
        m3.mamba3_test_set_segments(0)
    return y, fin


@pytest.mark.parametrize("shape,S", [
    ((1, 1024, 3, 64, 128, 1), 4),
    ((2, 768, 2, 64, 64, 4), 3),
    ((1, 1000, 2, 64, 128, 2), 8),   # ragged segments: 125 tokens, not a whole chunk
    ((1, 512, 4, 64, 64, 4), 2),
])
@pytest.mark.parametrize("with_init", [False, True])
def test_segmented_prefill_matches_oracle(shape, S, with_init):
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=7100 + L + S)
    init = rand_state(b, H, P, N, R, 7200 + L) if with_init else None
    y, fin = run_segmented(inp, S, init)
    yr, fr = oracle_scan(inp, init=to_state_np(init) if init is not None else None)
    assert rel_err(y.float().cpu().double().numpy(), yr) < TOLB
    check_state(fin, fr, TOLB)
    # and the unsegmented prefill of the same inputs
    y1 = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], init=init)
    torch.cuda.synchronize()
    assert rel_err(y.float().cpu().double().numpy(), y1.float().cpu().double().numpy()) < TOLB


def test_segmented_time_varying_decay_and_grouped_bc():
    b, L, H, P, N, R = 1, 1024, 4, 64, 64, 4
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=7300)
    inp.update(wl.grouped_bc(inp, 2, seed=7301))
    A_t = wl.decay_rates(inp["dt"], seed=7302)
    y, fin = run_segmented(inp, 4, A_t=A_t)
    f = wl.to_f64({k: inp[k] for k in (*NAMES, "D")})
    f["A"] = A_t.float().cpu().double().numpy()
    yr, fr = oracle.scan_complex(**f)
    assert rel_err(y.float().cpu().double().numpy(), yr) < TOLB
    check_state(fin, fr, TOLB)


def test_library_segments_long_context_with_its_own_workspace_size():
    """The long-context shape (b1 L65536 H64 N64 R4) qualifies for segments with the
    library's choice: the segmented workspace exceeds the minimal one, and the
    final state of the segmented run equals the unsegmented run's."""
    w = wl.CONFIGS["mimo4_long_b1_l65536"]
    inp = wl.make_inputs(w, seed=7400, device="cuda")
    dims = m3.make_dims(inp["x"], inp["B"])
    seg = m3.mamba3_scan_segmented_workspace_bytes(dims)
    assert seg > m3.mamba3_scan_workspace_bytes(dims)
    fins = []
    ys = []
    for nbytes in (seg, m3.mamba3_scan_workspace_bytes(dims)):
        ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
        fin = m3.State.zeros(w.batch, w.nheads, w.headdim, w.dstate, w.rank)
        ys.append(m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], final_state=fin, workspace=ws))
        assert m3.mamba3_device_status(ws) == m3.MAMBA3_OK
        fins.append(fin)
    torch.cuda.synchronize()
    assert rel_err(ys[0].float().cpu().double().numpy(), ys[1].float().cpu().double().numpy()) < TOLB
    for n in ("h", "b_prev", "x_prev"):
        a, b = getattr(fins[0], n), getattr(fins[1], n)
        assert rel_err(a.cpu().double().numpy(), b.cpu().double().numpy()) < TOLB, n


def test_segmented_long_context_repeats_bit_identically():
    """The library's segmented prefill at the long-context shape, three times: the
    outputs must be bit-identical (a race between the combine's state copy and its
    update showed up as run-to-run differences in some segments' initial states)
    and match the unsegmented prefill."""
    w = wl.CONFIGS["mimo4_long_b1_l65536"]
    inp = wl.make_inputs(w, seed=7500, device="cuda")
    dims = m3.make_dims(inp["x"], inp["B"])
    ws = torch.zeros(m3.mamba3_scan_segmented_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    ys = []
    for _ in range(3):
        ys.append(m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], workspace=ws))
        assert m3.mamba3_device_status(ws) == m3.MAMBA3_OK
    y1 = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"],
                            workspace=torch.zeros(m3.mamba3_scan_workspace_bytes(dims), dtype=torch.uint8,
                                                  device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])
    assert rel_err(ys[0].float().cpu().double().numpy(), y1.float().cpu().double().numpy()) < TOLB
