"""GPU backward pass (mamba3_scan_bwd) against the fp64 oracle's gradients
(oracle.scan_bwd, itself pinned to finite differences of the definition).

Every gradient tensor is compared by max|err| / max|ref|: 1e-4 for fp32 inputs,
2e-2 for bf16 inputs (the gradients are written in the input dtype)."""
import numpy as np
import pytest
import torch

import linear_recurrent_scan_b200 as m3
import oracle
from linear_recurrent_scan_b200 import build as m3build
from linear_recurrent_scan_b200 import workloads as wl
from tests.conftest import rel_err
from tests.parity_util import NAMES, TOL, small_inputs

pytestmark = pytest.mark.gpu

GRADS = ("dx", "dB", "dC", "dtheta", "ddt", "dlam", "dA", "dD")
STATE = (("h", "dh0"), ("b_prev", "dbprev0"), ("x_prev", "dxprev0"), ("angle", "dangle0"))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()


def rand_state(b, H, P, N, R, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g, device="cuda")
    return m3.State(r(b, H, N, P) * 0.5, r(b, H, R, N), r(b, H, R, P), r(b, H, N // 2) * 2.0)


def np64(t):
    return t.detach().float().cpu().double().numpy()


def run_both(inp, dy, init=None, d_final=None):
    gr = m3.mamba3_scan_bwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], dy, init=init, d_final=d_final)
    torch.cuda.synchronize()
    f = wl.to_f64({k: inp[k] for k in (*NAMES, "A", "D")})
    st = lambda s: oracle.State(*(np64(getattr(s, n)) for n, _ in STATE)) if s is not None else None
    ref = oracle.scan_bwd(**f, dy=np64(dy), init=st(init), d_final=st(d_final))
    return gr, ref


def check(gr, ref, tol, with_state=True, dt=None):
    errs = {n: rel_err(np64(gr[n]), ref[n]) for n in GRADS}
    if with_state:
        for n, gn in STATE:
            errs[gn] = rel_err(np64(getattr(gr["d_init"], n)), ref[gn])
        # From a zero state the initial angle's gradient vanishes (y sees only angle
        # differences), so measure it on the scale of the angle-gradient sums it is
        # one of: S_t = dtheta_t / dt_t (dtheta carries the factor dt, dangle0 none).
        d = np.abs(np64(gr["d_init"].angle) - ref["dangle0"]).max()
        sums = np.abs(ref["dtheta"] / dt[..., None]).max() if dt is not None else np.abs(ref["dtheta"]).max()
        errs["dangle0"] = float(d / max(np.abs(ref["dangle0"]).max(), sums))
    bad = {k: v for k, v in errs.items() if not v < tol}
    assert not bad, (bad, errs)


def dy_like(x, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return torch.randn(x.shape, generator=g, device="cuda").to(x.dtype)


@pytest.mark.parametrize("shape,dtype", [
    ((2, 100, 3, 16, 16, 1), torch.float32),   # 4 chunks of 32, ragged tail of 4
    ((1, 70, 2, 8, 8, 2), torch.float32),      # Q = 16
    ((2, 45, 2, 16, 32, 4), torch.float32),    # Q = 8
    ((1, 33, 2, 32, 16, 8), torch.float32),    # Q = 4
    ((1, 130, 4, 64, 128, 1), torch.bfloat16),
    ((1, 70, 4, 64, 128, 4), torch.bfloat16),
    ((2, 50, 3, 64, 64, 2), torch.bfloat16),
])
@pytest.mark.parametrize("with_state", [False, True])
def test_backward_matches_oracle(shape, dtype, with_state):
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, dtype, seed=2200 + L + R)
    dy = dy_like(inp["x"], 2300 + L)
    init = rand_state(b, H, P, N, R, 2400 + L) if with_state else None
    d_final = rand_state(b, H, P, N, R, 2500 + L) if with_state else None
    gr, ref = run_both(inp, dy, init, d_final)
    check(gr, ref, TOL[dtype], dt=np64(inp["dt"]))


@pytest.mark.parametrize("L", [1, 2, 31, 32, 33])
def test_backward_short_and_boundary_lengths(L):
    b, H, P, N, R = 2, 2, 16, 16, 1
    inp = small_inputs(b, L, H, P, N, R, torch.float32, seed=2600 + L)
    dy = dy_like(inp["x"], 2610 + L)
    gr, ref = run_both(inp, dy, rand_state(b, H, P, N, R, 2620 + L), rand_state(b, H, P, N, R, 2630 + L))
    check(gr, ref, TOL[torch.float32])


def test_backward_empty_sequence_passes_state_gradients_through():
    """L = 0: the exported state is the initial state, so its gradients pass
    through and every other gradient is zero."""
    b, H, P, N, R = 2, 3, 16, 16, 2
    inp = small_inputs(b, 0, H, P, N, R, torch.float32, seed=2700)
    dy = torch.zeros_like(inp["x"])
    d_final = rand_state(b, H, P, N, R, 2701)
    gr = m3.mamba3_scan_bwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], dy,
                            init=rand_state(b, H, P, N, R, 2702), d_final=d_final)
    torch.cuda.synchronize()
    for n, _ in STATE:
        assert torch.equal(getattr(gr["d_init"], n), getattr(d_final, n))
    assert torch.count_nonzero(gr["dA"]) == 0 and torch.count_nonzero(gr["dD"]) == 0


def test_backward_repeated_launches_identical():
    inp = small_inputs(2, 150, 4, 64, 128, 1, torch.bfloat16, seed=2800)
    dy = dy_like(inp["x"], 2801)
    outs = [m3.mamba3_scan_bwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], dy) for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        for n in ("dx", "dB", "dC", "dtheta", "ddt", "dlam"):
            assert torch.equal(o[n], outs[0][n]), n


def test_backward_full_size_sampled_units():
    """The SISO prefill size (b8 L2048 H64 P64 N128 bf16): sampled (batch, head)
    units against the oracle run on those units' slices (units are independent),
    and at every unit the identity of a loss linear in x: <dy, y> = <dx, x> (zero
    initial state, D included)."""
    b, L, H, P, N, R = 8, 2048, 64, 64, 128, 1
    w = wl.CONFIGS["siso_prefill_b8_l2048"]
    inp = wl.make_inputs(w, seed=2900, device="cuda")
    dy = dy_like(inp["x"], 2901)
    gr = m3.mamba3_scan_bwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], dy)
    y = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"])
    torch.cuda.synchronize()
    terms = dy.double() * y.double()
    lhs = terms.sum(dim=(1, 3, 4))
    rhs = (gr["dx"].double() * inp["x"].double()).sum(dim=(1, 3, 4))
    # y and dx are rounded to bf16 (relative 2^-8 per element), so the two sums may
    # differ by about 2^-8 of the terms' total magnitude, however much they cancel
    mass = terms.abs().sum(dim=(1, 3, 4))
    assert float(((lhs - rhs).abs() / mass).max()) < 1e-2
    for (bb, hh) in [(0, 0), (3, 17), (7, 63)]:
        sl = {n: inp[n][bb:bb + 1, :, hh:hh + 1].contiguous() for n in NAMES}
        f = wl.to_f64(sl)
        f["A"] = np64(inp["A"][hh:hh + 1])
        f["D"] = np64(inp["D"][hh:hh + 1])
        ref = oracle.scan_bwd(**f, dy=np64(dy[bb:bb + 1, :, hh:hh + 1]))
        for n in ("dx", "dB", "dC", "dtheta", "ddt", "dlam"):
            e = rel_err(np64(gr[n][bb:bb + 1, :, hh:hh + 1]), ref[n])
            assert e < TOL[torch.bfloat16], (n, bb, hh, e)


@pytest.mark.parametrize("shape,dtype", [
    ((2, 100, 3, 16, 16, 1), torch.float32),
    ((2, 45, 2, 16, 32, 4), torch.float32),
    ((1, 130, 4, 64, 128, 1), torch.bfloat16),
    ((1, 70, 4, 64, 128, 4), torch.bfloat16),
])
def test_backward_time_varying_decay_matches_oracle(shape, dtype):
    """mamba3_scan_bwd_at: a decay rate per token; its gradient dA_t is per token."""
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, dtype, seed=3300 + L + R)
    A_t = wl.decay_rates(inp["dt"], seed=3400 + L)
    dy = dy_like(inp["x"], 3500 + L)
    init, d_final = rand_state(b, H, P, N, R, 3600 + L), rand_state(b, H, P, N, R, 3700 + L)
    gr = m3.mamba3_scan_bwd_at(*(inp[n] for n in NAMES), A_t, inp["D"], dy, init=init, d_final=d_final)
    torch.cuda.synchronize()
    f = wl.to_f64({k: inp[k] for k in (*NAMES, "D")})
    f["A"] = np64(A_t)
    st = lambda s: oracle.State(*(np64(getattr(s, n)) for n, _ in STATE))
    ref = oracle.scan_bwd(**f, dy=np64(dy), init=st(init), d_final=st(d_final))
    gr["dA"] = gr["dA_t"]
    check(gr, ref, TOL[dtype])


@pytest.mark.parametrize("shape,G,dtype", [
    ((2, 100, 6, 16, 16, 1), 2, torch.float32),
    ((2, 45, 4, 16, 32, 4), 1, torch.float32),
    ((1, 130, 8, 64, 128, 1), 2, torch.bfloat16),
    ((1, 70, 8, 64, 128, 4), 4, torch.bfloat16),
])
def test_backward_grouped_bc_matches_oracle(shape, G, dtype):
    """B, C shared by groups of H / G heads: dB, dC are the sums of the group's
    heads' gradients (the oracle sums its per-head ones the same way)."""
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, dtype, seed=3800 + L + G)
    inp.update(wl.grouped_bc(inp, G, seed=3900 + L))
    dy = dy_like(inp["x"], 4000 + L)
    init, d_final = rand_state(b, H, P, N, R, 4100 + L), rand_state(b, H, P, N, R, 4200 + L)
    gr, ref = run_both(inp, dy, init, d_final)
    assert gr["dB"].shape == inp["B"].shape
    check(gr, ref, TOL[dtype])


@pytest.mark.parametrize("shape,G,dtype", [
    ((2, 45, 4, 16, 32, 4), 2, torch.float32),
    ((1, 130, 8, 64, 128, 1), 2, torch.bfloat16),
])
def test_backward_time_varying_decay_grouped_bc_matches_oracle(shape, G, dtype):
    """mamba3_scan_bwd_at with B, C shared by groups of heads: dB, dC summed over
    each group's heads and dA_t per token, against the oracle with A as [b, L, H]."""
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, dtype, seed=4300 + L + G)
    inp.update(wl.grouped_bc(inp, G, seed=4400 + L))
    A_t = wl.decay_rates(inp["dt"], seed=4500 + L)
    dy = dy_like(inp["x"], 4600 + L)
    init, d_final = rand_state(b, H, P, N, R, 4700 + L), rand_state(b, H, P, N, R, 4800 + L)
    gr = m3.mamba3_scan_bwd_at(*(inp[n] for n in NAMES), A_t, inp["D"], dy, init=init, d_final=d_final)
    torch.cuda.synchronize()
    f = wl.to_f64({k: inp[k] for k in (*NAMES, "D")})
    f["A"] = np64(A_t)
    st = lambda s: oracle.State(*(np64(getattr(s, n)) for n, _ in STATE))
    ref = oracle.scan_bwd(**f, dy=np64(dy), init=st(init), d_final=st(d_final))
    gr["dA"] = gr["dA_t"]
    assert gr["dB"].shape == inp["B"].shape
    check(gr, ref, TOL[dtype])
