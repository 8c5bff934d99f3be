"""Pins of the oracle's backward pass (oracle.scan_bwd), CPU only.

The pages give no gradient formulas; the oracle differentiates the RoPE form
token by token.  These pins tie it to things other than itself:

* central finite differences of the *complex-state* forward (oracle.scan_complex,
  the definition) for every input and every part of the initial state, with
  the exported state's gradients fed in too;
* exact identities of a function that is linear in a group of its inputs:
  the loss <dy, y> + <dh_out, h_out> + <dx_out, x_out> is linear in
  (x, h_0, x_prev0), so it equals <dx, x> + <dh0, h_0> + <dxprev0, x_prev0>;
  it is linear in C (y reads C~ once), and with h_0 = 0 linear in (B, b_prev0).
"""
import numpy as np
import pytest

import oracle

K_OF = lambda N: N // 2


def case(rng, b=1, L=9, H=2, P=3, N=4, R=2, G=None, time_varying=False):
    G = G or H
    inp = dict(x=rng.standard_normal((b, L, H, R, P)), B=rng.standard_normal((b, L, G, R, N)),
               C=rng.standard_normal((b, L, G, R, N)), theta=rng.uniform(0, np.pi, (b, L, H, K_OF(N))),
               dt=rng.uniform(0.05, 0.5, (b, L, H)), lam=rng.uniform(0, 1, (b, L, H)),
               A=-rng.uniform(0.2, 2, (b, L, H) if time_varying else (H,)), D=rng.standard_normal(H))
    st = oracle.State(rng.standard_normal((b, H, N, P)), rng.standard_normal((b, H, R, N)),
                      rng.standard_normal((b, H, R, P)), rng.uniform(-3, 3, (b, H, K_OF(N))))
    dy = rng.standard_normal((b, L, H, R, P))
    df = oracle.State(rng.standard_normal((b, H, N, P)), rng.standard_normal((b, H, R, N)),
                      rng.standard_normal((b, H, R, P)), rng.standard_normal((b, H, K_OF(N))))
    return inp, st, dy, df


STATE_GRADS = {"h": "dh0", "b_prev": "dbprev0", "x_prev": "dxprev0", "angle": "dangle0"}


def loss(inp, st, dy, df):
    y, f = oracle.scan_complex(**inp, init=st, nthreads=1)
    total = float((dy * y).sum())
    if df is not None:
        total += sum(float((getattr(df, n) * getattr(f, n)).sum()) for n in STATE_GRADS)
    return total


def fd_errors(inp, st, dy, df, eps=1e-6):
    """max |numeric - analytic| / max |numeric| per input."""
    g = oracle.scan_bwd(**inp, dy=dy, init=st, d_final=df, nthreads=1)
    errs = {}
    targets = [(n, inp[n], "d" + n) for n in inp] + [(n, getattr(st, n), gn) for n, gn in STATE_GRADS.items()]
    for name, arr, gname in targets:
        num = np.zeros_like(arr)
        for i in np.ndindex(arr.shape):
            old = arr[i]
            arr[i] = old + eps
            lp = loss(inp, st, dy, df)
            arr[i] = old - eps
            lm = loss(inp, st, dy, df)
            arr[i] = old
            num[i] = (lp - lm) / (2 * eps)
        errs[name] = float(np.max(np.abs(num - g[gname])) / max(1e-6, float(np.max(np.abs(num)))))
    return errs


@pytest.mark.parametrize("kw", [
    dict(),                                  # MIMO R = 2, A per head
    dict(R=1, L=11, H=3, N=6, P=2),           # SISO
    dict(time_varying=True),                 # A_t per token
    dict(G=1, H=2),                          # B, C shared by both heads
    dict(b=2, L=5, R=3, N=2, P=2),
])
def test_backward_matches_finite_differences_of_the_definition(kw):
    rng = np.random.default_rng(301 + len(kw) + 7 * kw.get("R", 2))
    inp, st, dy, df = case(rng, **kw)
    errs = fd_errors(inp, st, dy, df)
    assert max(errs.values()) < 1e-7, errs


def test_backward_without_initial_state_or_final_gradients():
    """Zero initial state and no exported-state gradient (the plain training
    call): still the finite-difference gradient, and dh0 is the gradient of a
    zero initial state."""
    rng = np.random.default_rng(311)
    inp, _, dy, _ = case(rng, L=13, R=1)
    g = oracle.scan_bwd(**inp, dy=dy, nthreads=1)
    zero = oracle.State.zeros(1, 2, 3, 4, 1)
    errs = fd_errors(inp, zero, dy, None)
    assert max(errs.values()) < 1e-7, errs
    assert np.abs(g["dh0"]).max() > 0
    # from a zero state y depends only on differences of angles, so shifting the
    # initial angle changes nothing: the per-token angle gradients cancel
    assert np.abs(g["dangle0"]).max() < 1e-12 * np.abs(g["dtheta"]).max()


def test_backward_linear_in_x_and_state():
    rng = np.random.default_rng(321)
    inp, st, dy, df = case(rng, L=15, R=2)
    df.b_prev[:] = 0.0
    df.angle[:] = 0.0
    g = oracle.scan_bwd(**inp, dy=dy, init=st, d_final=df)
    lhs = loss(inp, st, dy, df)
    rhs = (g["dx"] * inp["x"]).sum() + (g["dh0"] * st.h).sum() + (g["dxprev0"] * st.x_prev).sum()
    assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs))


def test_backward_linear_in_C_and_D():
    rng = np.random.default_rng(322)
    inp, st, dy, _ = case(rng, L=12, R=3, N=6)
    g = oracle.scan_bwd(**inp, dy=dy, init=st)
    y, _ = oracle.scan_complex(**inp, init=st)
    D = inp["D"][None, None, :, None, None]
    assert abs((dy * (y - D * inp["x"])).sum() - (g["dC"] * inp["C"]).sum()) <= 1e-11 * np.abs(y).sum()
    assert abs((dy * D * inp["x"]).sum() - (g["dD"] * inp["D"]).sum()) <= 1e-11 * np.abs(y).sum()


def test_backward_linear_in_B_with_zero_initial_h():
    rng = np.random.default_rng(323)
    inp, st, dy, _ = case(rng, L=10, R=2)
    st.h[:] = 0.0
    g = oracle.scan_bwd(**inp, dy=dy, init=st)
    y, _ = oracle.scan_complex(**inp, init=st)
    D = inp["D"][None, None, :, None, None]
    lhs = (dy * (y - D * inp["x"])).sum()
    rhs = (g["dB"] * inp["B"]).sum() + (g["dbprev0"] * st.b_prev).sum()
    assert abs(lhs - rhs) <= 1e-11 * np.abs(y).sum()


def test_grouped_gradient_is_sum_over_heads():
    """dB of a shared row equals the sum of the per-head gradients of the same
    rows repeated over the group's heads."""
    rng = np.random.default_rng(331)
    inp, st, dy, df = case(rng, L=8, H=4, G=2)
    g = oracle.scan_bwd(**inp, dy=dy, init=st, d_final=df)
    rep = dict(inp, B=np.repeat(inp["B"], 2, axis=2), C=np.repeat(inp["C"], 2, axis=2))
    gr = oracle.scan_bwd(**rep, dy=dy, init=st, d_final=df)
    for n in ("dB", "dC"):
        assert np.allclose(g[n], gr[n].reshape(1, 8, 2, 2, 2, 4).sum(axis=3), rtol=0, atol=1e-13)
    for n in ("dx", "dtheta", "ddt", "dlam", "dA", "dD", "dh0"):
        assert np.array_equal(g[n], gr[n]), n
