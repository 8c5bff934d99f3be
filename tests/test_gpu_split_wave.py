"""The tensor-core prefill's split last wave: units that run in two CTAs (chunks
[0, c1) early, [c1, n) last, the second continuing from the carried state and
angle the first hands over through the workspace) must give the one-CTA result
bit for bit, for every variant of the kernel, and match the fp64 oracle.

mamba3_test_set_split forces a split on sizes the oracle finishes quickly; the
library's own plan is exercised on shapes with more units than SMs."""
import pytest
import torch

import linear_recurrent_scan_b200 as m3
from linear_recurrent_scan_b200 import build as m3build
from linear_recurrent_scan_b200 import workloads as wl
from tests.conftest import rel_err
from tests.parity_util import NAMES, TOL, check_state, oracle_scan, small_inputs, to_state_np, unit_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()
    yield
    m3.mamba3_test_set_split(0)


def rand_state(b, H, P, N, R, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g, device="cuda")
    return m3.State(r(b, H, N, P) * 0.5, r(b, H, R, N), r(b, H, R, P), r(b, H, N // 2) * 2.0)


def run(inp, split, init=None, variant="plain"):
    """(y, final state, status) of one prefill with the split plan `split`
    ((k, c1) forced, -1 never, 0 the library's plan), workspace as the binding sizes it."""
    if isinstance(split, tuple):
        m3.mamba3_test_set_split(*split)
    else:
        m3.mamba3_test_set_split(split)
    try:
        x = inp["x"]
        b, L, H, R, P = x.shape
        N = inp["B"].shape[-1]
        dims = m3.make_dims(x, inp["B"])
        ws = torch.full((m3.mamba3_scan_fwd_workspace_bytes(dims),), 0xAB, dtype=torch.uint8, device="cuda")
        fin = m3.State.zeros(b, H, P, N, R)
        args = [inp[n] for n in NAMES]
        if variant == "plain":
            y = m3.mamba3_scan_fwd(*args, inp["A"], inp["D"], init=init, final_state=fin, workspace=ws)
        elif variant == "at":
            y = m3.mamba3_scan_fwd_at(*args, inp["A_t"], inp["D"], init=init, final_state=fin, workspace=ws)
        else:
            y = m3.mamba3_scan_fwd_bcnorm(*args, inp["A"], inp["D"], norm=inp["norm"], init=init, final_state=fin,
                                          workspace=ws)
        torch.cuda.synchronize()
        return y, fin, m3.mamba3_device_status(ws)
    finally:
        m3.mamba3_test_set_split(0)


def assert_identical(r1, r2):
    y1, f1, s1 = r1
    y2, f2, s2 = r2
    assert s1 == m3.MAMBA3_OK and s2 == m3.MAMBA3_OK, (s1, s2)
    assert torch.equal(y1, y2)
    for n in ("h", "b_prev", "x_prev", "angle"):
        assert torch.equal(getattr(f1, n), getattr(f2, n)), n


@pytest.mark.parametrize("shape,split,with_init", [
    ((2, 300, 4, 64, 128, 1), (3, 1), False),    # 3 chunks, ragged tail, units 0..2 split after chunk 1
    ((2, 300, 4, 64, 128, 1), (8, 2), True),     # every unit split, from an initial state
    ((2, 100, 3, 64, 64, 4), (6, 2), True),      # R = 4: 32-token chunks, the last one ragged
    ((3, 257, 8, 64, 128, 2), (5, 3), False),    # dt, lam by TMA (8 heads); 5 chunks of 64 tokens
    ((1, 640, 8, 64, 64, 1), (4, 4), True),      # N = 64 (y by TMA stores); the split at a chunk of 5
    ((1, 129, 2, 64, 128, 1), (2, 1), True),     # second part of one token
])
def test_forced_split_is_bit_identical_and_matches_oracle(shape, split, with_init):
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=9100 + L + R)
    init = rand_state(b, H, P, N, R, 9200 + L) if with_init else None
    whole = run(inp, -1, init)
    parts = run(inp, split, init)
    assert_identical(whole, parts)
    yr, fr = oracle_scan(inp, init=to_state_np(init) if init is not None else None)
    assert rel_err(parts[0].float().cpu().double().numpy(), yr) < TOL[torch.bfloat16]
    check_state(parts[1], fr, TOL[torch.bfloat16])


def test_forced_split_that_does_not_fit_runs_whole():
    """k above the unit count or c1 past the last chunk: no split, same result."""
    inp = small_inputs(1, 200, 2, 64, 128, 1, torch.bfloat16, seed=9300)
    whole = run(inp, -1)
    assert_identical(whole, run(inp, (3, 1)))   # 2 units
    assert_identical(whole, run(inp, (1, 2)))   # 2 chunks


def test_split_variants_time_varying_decay_and_bc_norm():
    """The A_t and fused B/C norm kernels take the same hand-over."""
    b, L, H, P, N, R = 2, 300, 8, 64, 128, 1
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=9400)
    g = torch.Generator(device="cuda")
    g.manual_seed(9401)
    inp["A_t"] = (-torch.rand(b, L, H, generator=g, device="cuda") * 2.0 - 0.1).to(torch.bfloat16)
    init = rand_state(b, H, P, N, R, 9402)
    assert_identical(run(inp, -1, init, "at"), run(inp, (9, 1), init, "at"))
    inp["norm"] = m3.BCNorm(w_B=torch.rand(H, R, N, generator=g, device="cuda") + 0.5,
                            bias_B=torch.randn(H, R, N, generator=g, device="cuda") * 0.1,
                            w_C=torch.rand(H, R, N, generator=g, device="cuda") + 0.5,
                            bias_C=torch.randn(H, R, N, generator=g, device="cuda") * 0.1, eps=1e-5)
    assert_identical(run(inp, -1, init, "bcnorm"), run(inp, (5, 2), init, "bcnorm"))


@pytest.mark.parametrize("shape", [(3, 512, 64, 64, 128, 1), (5, 300, 64, 64, 64, 2)])
def test_library_plan_on_more_units_than_sms(shape):
    """192 and 320 units on 148 SMs: the library splits its last wave; the result is
    the whole-unit one bit for bit and matches the oracle on sampled units, split
    ones (the lowest unit indices) included."""
    b, L, H, P, N, R = shape
    dims = m3.Dims(b, L, H, P, N, R, 0, m3.MAMBA3_BF16, 0)
    assert m3.mamba3_scan_fwd_workspace_bytes(dims) > m3.mamba3_scan_workspace_bytes(dims)
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=9500 + L)
    init = rand_state(b, H, P, N, R, 9501)
    whole = run(inp, -1, init)
    auto = run(inp, 0, init)
    assert_identical(whole, auto)
    units = [0, 1, 17, b * H // 2, b * H - 1]
    yr, fr = oracle_scan(inp, init=to_state_np(init), units=units)
    yg = unit_rows(auto[0].float().cpu().double().numpy(), units, H)
    assert rel_err(yg, unit_rows(yr, units, H)) < TOL[torch.bfloat16]
    check_state(auto[1], fr, TOL[torch.bfloat16], units=units)


@pytest.mark.parametrize("name", ["siso_prefill_b8_l2048", "mimo4_prefill_b4_l8192"])
def test_full_size_split_is_bit_identical(name):
    """The bench's prefill shapes (512 and 256 units): the split plan's result equals
    the whole-unit launch bit for bit, repeatedly."""
    w = wl.CONFIGS[name]
    inp = wl.make_inputs(w, device="cuda")
    whole = run(inp, -1)
    for _ in range(3):
        assert_identical(whole, run(inp, 0))
