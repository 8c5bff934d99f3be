"""The backward pass's split last wave: a unit swept by two CTAs (the end of the
sequence first, then its start from the hand-over of the carried state's adjoint,
the running angle-gradient sum and one token's pending dt, lam share) must give the
one-CTA gradients: bit for bit for dx, dtheta, dB, dC and the initial state's;
within float32 summation order for ddt, dlam (each chunk's decay adjoint sums
per-warp shares with atomics, so they differ in the last bits between any two
runs), dA, dD and the grouped dB, dC; and the oracle's within the bf16 tolerance.
mamba3_test_set_split forces a split on small sizes (c1 counts the backward's
64-row chunks); the library's own plan runs on more units than SMs."""
import numpy as np
import pytest
import torch

import linear_recurrent_scan_b200 as m3
from linear_recurrent_scan_b200 import build as m3build
from tests.parity_util import NAMES, TOL, small_inputs
from tests.test_gpu_backward import STATE, check, dy_like, np64, rand_state, run_both

pytestmark = pytest.mark.gpu

EXACT = ("dx", "dtheta")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()
    yield
    m3.mamba3_test_set_split(0)


def bwd(inp, dy, split, init=None, d_final=None, A_t=None):
    if isinstance(split, tuple):
        m3.mamba3_test_set_split(*split)
    else:
        m3.mamba3_test_set_split(split)
    try:
        x = inp["x"]
        dims = m3.make_dims(x, inp["B"])
        ws = torch.full((m3.mamba3_scan_bwd_workspace_bytes(dims),), 0xCD, dtype=torch.uint8, device="cuda")
        args = [inp[n] for n in NAMES]
        if A_t is None:
            gr = m3.mamba3_scan_bwd(*args, inp["A"], inp["D"], dy, init=init, d_final=d_final, workspace=ws)
        else:
            gr = m3.mamba3_scan_bwd_at(*args, A_t, inp["D"], dy, init=init, d_final=d_final, workspace=ws)
        torch.cuda.synchronize()
        assert m3.mamba3_device_status(ws) == m3.MAMBA3_OK
        return gr
    finally:
        m3.mamba3_test_set_split(0)


def assert_same(g1, g2, grouped=False):
    exact = EXACT + (() if grouped else ("dB", "dC"))
    for n in exact:
        assert torch.equal(g1[n], g2[n]), n
    for n, _ in STATE:
        assert torch.equal(getattr(g1["d_init"], n), getattr(g2["d_init"], n)), n
    # (bf16 outputs: a last-bit difference of the fp32 sum can move one rounding step)
    for n in ("ddt", "dlam", "dA", "dD", "dA_t") + (("dB", "dC") if grouped else ()):
        if n in g1 and g1[n] is not None:
            a, b = np64(g1[n]), np64(g2[n])
            assert np.abs(a - b).max() <= 1e-2 * max(1e-6, np.abs(b).max()), n


@pytest.mark.parametrize("shape,split", [
    ((2, 300, 4, 64, 128, 1), (3, 2)),   # 5 chunks of 64 tokens, ragged tail; units 0..2 split after 2
    ((2, 300, 4, 64, 128, 1), (8, 4)),   # every unit, the second part one ragged chunk
    ((2, 100, 3, 64, 64, 4), (6, 3)),    # R = 4: 16-token chunks
    ((1, 200, 8, 64, 128, 2), (5, 1)),   # the start part a single chunk
])
def test_forced_backward_split_matches_unsplit_and_oracle(shape, split):
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=9700 + L + R)
    dy = dy_like(inp["x"], 9710 + L)
    init = rand_state(b, H, P, N, R, 9720 + L)
    d_final = rand_state(b, H, P, N, R, 9730 + L)
    whole = bwd(inp, dy, -1, init, d_final)
    parts = bwd(inp, dy, split, init, d_final)
    assert_same(whole, parts)
    _, ref = run_both(inp, dy, init, d_final)
    check(parts, ref, TOL[torch.bfloat16], dt=np64(inp["dt"]))


def test_forced_backward_split_time_varying_decay_and_grouped_bc():
    b, L, H, P, N, R = 2, 260, 8, 64, 128, 1
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=9800)
    dy = dy_like(inp["x"], 9801)
    g = torch.Generator(device="cuda")
    g.manual_seed(9802)
    A_t = (-torch.rand(b, L, H, generator=g, device="cuda") * 2.0 - 0.1).to(torch.bfloat16)
    init = rand_state(b, H, P, N, R, 9803)
    assert_same(bwd(inp, dy, -1, init, A_t=A_t), bwd(inp, dy, (7, 2), init, A_t=A_t))
    grp = dict(inp)
    grp["B"], grp["C"] = inp["B"][:, :, :2].contiguous(), inp["C"][:, :, :2].contiguous()  # G = 2
    assert_same(bwd(grp, dy, -1, init), bwd(grp, dy, (9, 3), init), grouped=True)


def test_library_backward_plan_on_more_units_than_sms():
    """192 units on 148 SMs: the library splits the reverse sweep's last wave; the
    gradients equal the one-CTA ones."""
    b, L, H, P, N, R = 3, 256, 64, 64, 128, 1
    dims = m3.Dims(b, L, H, P, N, R, 0, m3.MAMBA3_BF16, 0)
    m3.mamba3_test_set_split(-1)
    unsplit = m3.mamba3_scan_bwd_workspace_bytes(dims)
    m3.mamba3_test_set_split(0)
    assert m3.mamba3_scan_bwd_workspace_bytes(dims) > unsplit
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=9900)
    dy = dy_like(inp["x"], 9901)
    init = rand_state(b, H, P, N, R, 9902)
    assert_same(bwd(inp, dy, -1, init), bwd(inp, dy, 0, init))
