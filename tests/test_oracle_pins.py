"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test names the passage it follows.  Pages: "Mamba-3: 2x smaller state ..."
(MarkTechPost, Korean translation) sections 1.1 (exponential-trapezoidal
three-term update, exponential-Euler as the Mamba-1/2 predecessor, second-order
accuracy), 1.2 (complex state == real state with data-dependent RoPE on B and C,
parity task), 1.3 (MIMO rank-R shapes); the paper-review page (no1joon.github.io)
for the parity example and the constant state size.

What each pin catches (a plausible slip anywhere in the oracle fails one):
  * lfilter pins       -- the complex pole exp(dt(A + i theta)), both trapezoid
                          weights, the lag multiplied by the pole (library IIR filter)
  * impulse closed form-- the folded weight lam_s dt_s + (1 - lam_{s+1}) dt_{s+1}
                          and the index of lam/dt in the lag term
  * Euler / lag-only   -- lam = 1 and lam = 0 closed forms (geometric series)
  * ODE order          -- second order at lam = 1/2, first order at lam = 1
  * parity toy         -- rotation by the accumulated angle (golden fixture)
  * complex == RoPE == quadratic -- rotation sign, pairing, carry rotation,
                          chunk algebra (three independent formulations)
  * MIMO superposition -- all ranks of a token feed the state; readout per rank
  * composition        -- the exported decode state continues the sequence exactly
"""
import numpy as np
import pytest
import scipy.signal

import oracle
from tests.conftest import read_golden, rel_err

RNG = np.random.default_rng(1234)


def rand_inputs(b=2, L=23, H=3, P=5, N=8, R=1, rng=RNG, A_scale=1.0):
    K = N // 2
    return dict(
        x=rng.standard_normal((b, L, H, R, P)),
        B=rng.standard_normal((b, L, H, R, N)),
        C=rng.standard_normal((b, L, H, R, N)),
        theta=rng.uniform(0, np.pi, (b, L, H, K)),
        dt=rng.uniform(0.05, 0.5, (b, L, H)),
        lam=rng.uniform(0.0, 1.0, (b, L, H)),
        A=-A_scale * rng.uniform(0.2, 2.0, (H,)),
        D=rng.standard_normal((H,)),
    )


def rand_state(b, H, P, N, R, rng=RNG):
    return oracle.State(
        rng.standard_normal((b, H, N, P)),
        rng.standard_normal((b, H, R, N)),
        rng.standard_normal((b, H, R, P)),
        rng.uniform(-10, 10, (b, H, N // 2)),
    )


def slice_t(inp, lo, hi):
    return {k: (v[:, lo:hi] if v.ndim >= 3 else v) for k, v in inp.items()}


# --------------------------------------------------------------------------
# library IIR filter: the time-invariant complex SSM is a first-order filter
# --------------------------------------------------------------------------
@pytest.mark.parametrize("lam", [0.0, 0.3, 0.5, 1.0])
def test_time_invariant_equals_lfilter(lam):
    """Constant dt, lam, theta, B, C: pair k is the IIR filter
    H_k = b_k * lfilter([lam dt, (1 - lam) dt a_k], [1, -a_k], x), a_k = exp(dt (A + i theta_k)),
    y = sum_k Re(conj(c_k) H_k) + D x  (section 1.1 three-term update, section 1.2 complex pole)."""
    rng = np.random.default_rng(7)
    L, N = 64, 6
    K = N // 2
    dt, A, Dh = 0.3, -0.7, 0.4
    th = rng.uniform(0, np.pi, K)
    bvec = rng.standard_normal(N)
    cvec = rng.standard_normal(N)
    x = rng.standard_normal(L)
    inp = dict(
        x=x.reshape(1, L, 1, 1, 1),
        B=np.broadcast_to(bvec, (1, L, 1, 1, N)).copy(),
        C=np.broadcast_to(cvec, (1, L, 1, 1, N)).copy(),
        theta=np.broadcast_to(th, (1, L, 1, K)).copy(),
        dt=np.full((1, L, 1), dt),
        lam=np.full((1, L, 1), lam),
        A=np.array([A]),
        D=np.array([Dh]),
    )
    y, _ = oracle.scan_complex(**inp)
    ref = Dh * x
    for k in range(K):
        a = np.exp(dt * (A + 1j * th[k]))
        bk = bvec[2 * k] + 1j * bvec[2 * k + 1]
        ck = cvec[2 * k] + 1j * cvec[2 * k + 1]
        Hk = bk * scipy.signal.lfilter([lam * dt, (1 - lam) * dt * a], [1.0, -a], x.astype(complex))
        ref = ref + np.real(np.conj(ck) * Hk)
    assert rel_err(y.ravel(), ref) < 1e-12
    y2, _ = oracle.scan_rope(**inp)
    assert rel_err(y2.ravel(), ref) < 1e-12


# --------------------------------------------------------------------------
# single impulse: closed form of the folded trapezoid weight
# --------------------------------------------------------------------------
@pytest.mark.parametrize("fn", ["scan_complex", "scan_rope", "scan_quadratic"])
def test_impulse_closed_form(fn):
    """x != 0 only at token t0: H_t0 = lam_t0 dt_t0 u and for t > t0
    H_t = prod_{q=t0+1..t} exp(dt_q (A + i theta_q)) * (lam_t0 dt_t0 + (1 - lam_{t0+1}) dt_{t0+1}) u
    (unrolling the section 1.1 update: the lagged term of step t0+1 carries the same pole)."""
    rng = np.random.default_rng(11)
    L, N, P, R, t0 = 17, 6, 3, 2, 5
    K = N // 2
    inp = rand_inputs(1, L, 1, P, N, R, rng)
    inp["x"][:] = 0
    inp["x"][0, t0] = rng.standard_normal((1, R, P))
    inp["D"][:] = 0.0
    y = getattr(oracle, fn)(**inp)
    y = y[0] if isinstance(y, tuple) else y
    dt, lam, th, A = inp["dt"][0, :, 0], inp["lam"][0, :, 0], inp["theta"][0, :, 0], inp["A"][0]
    Bc = inp["B"][0, :, 0, :, 0::2] + 1j * inp["B"][0, :, 0, :, 1::2]  # [L,R,K]
    Cc = inp["C"][0, :, 0, :, 0::2] + 1j * inp["C"][0, :, 0, :, 1::2]
    u = np.einsum("rk,rp->kp", Bc[t0], inp["x"][0, t0, 0])  # [K,P]
    ref = np.zeros((L, R, P))
    w_hat = lam[t0] * dt[t0] + (1 - lam[t0 + 1]) * dt[t0 + 1]
    for t in range(t0, L):
        if t == t0:
            Ht = lam[t0] * dt[t0] * u
        else:
            logp = np.sum(dt[t0 + 1:t + 1, None] * (A + 1j * th[t0 + 1:t + 1]), axis=0)  # [K]
            Ht = np.exp(logp)[:, None] * w_hat * u
        ref[t] = np.real(np.einsum("rk,kp->rp", np.conj(Cc[t]), Ht))
    assert rel_err(y[0, :, 0], ref) < 1e-12


# --------------------------------------------------------------------------
# lam = 1: exponential-Euler (Mamba-2) and lam = 0: lag only
# --------------------------------------------------------------------------
def _scalar_case(lam, L=40, dt=0.2, A=-0.5, x0=1.3):
    return dict(
        x=np.full((1, L, 1, 1, 1), x0),
        B=np.tile(np.array([1.0, 0.0]), (1, L, 1, 1, 1)),
        C=np.tile(np.array([1.0, 0.0]), (1, L, 1, 1, 1)),
        theta=np.zeros((1, L, 1, 1)),
        dt=np.full((1, L, 1), dt),
        lam=np.full((1, L, 1), lam),
        A=np.array([A]),
        D=np.array([0.0]),
    )


def test_lambda_one_is_exponential_euler():
    """lam = 1 removes the lagged term: h_t = a h_{t-1} + dt x (section 1.1: exponential-Euler
    of Mamba-1/2 is the special case), so for constant input h_t = dt x (1 - a^t) / (1 - a)."""
    L, dt, A, x0 = 40, 0.2, -0.5, 1.3
    y, _ = oracle.scan_complex(**_scalar_case(1.0, L, dt, A, x0))
    a = np.exp(dt * A)
    t = np.arange(1, L + 1)
    assert rel_err(y.ravel(), dt * x0 * (1 - a ** t) / (1 - a)) < 1e-13


def test_lambda_one_ignores_carry():
    """With lam = 1 the carried B_{t-1} x_{t-1} has weight (1 - lam) dt a = 0."""
    rng = np.random.default_rng(3)
    inp = rand_inputs(1, 9, 2, 4, 6, 2, rng)
    inp["lam"][:] = 1.0
    s1 = rand_state(1, 2, 4, 6, 2, rng)
    s2 = oracle.State(s1.h, rng.standard_normal(s1.b_prev.shape), rng.standard_normal(s1.x_prev.shape), s1.angle)
    y1, _ = oracle.scan_complex(**inp, init=s1)
    y2, _ = oracle.scan_complex(**inp, init=s2)
    assert np.max(np.abs(y1 - y2)) < 1e-13


def test_lambda_zero_is_pure_lag():
    """lam = 0: h_t = a (h_{t-1} + dt u_{t-1}); constant input from a zero carry gives
    h_t = a dt x (1 - a^(t-1)) / (1 - a)."""
    L, dt, A, x0 = 40, 0.2, -0.5, 1.3
    y, _ = oracle.scan_complex(**_scalar_case(0.0, L, dt, A, x0))
    a = np.exp(dt * A)
    t = np.arange(1, L + 1)
    assert rel_err(y.ravel(), a * dt * x0 * (1 - a ** (t - 1)) / (1 - a)) < 1e-13


def test_theta_zero_is_real_ssm():
    """theta = 0: no rotation, the pairs are two independent real SSMs and the rotated frame
    is the identity (section 1.2: the rotation is what the complex part adds)."""
    rng = np.random.default_rng(5)
    inp = rand_inputs(1, 15, 1, 3, 4, 1, rng)
    inp["theta"][:] = 0.0
    y, fin = oracle.scan_complex(**inp)
    # real recurrence with unrotated B, C (typed as a dense loop over t)
    dt, lam, A = inp["dt"][0, :, 0], inp["lam"][0, :, 0], inp["A"][0]
    Bm, Cm, X = inp["B"][0, :, 0, 0], inp["C"][0, :, 0, 0], inp["x"][0, :, 0, 0]
    h = np.zeros((4, 3))
    uprev = np.zeros((4, 3))
    ref = []
    for t in range(15):
        u = np.outer(Bm[t], X[t])
        a = np.exp(dt[t] * A)
        h = a * h + (1 - lam[t]) * dt[t] * a * uprev + lam[t] * dt[t] * u
        ref.append(Cm[t] @ h + inp["D"][0] * X[t])
        uprev = u
    assert rel_err(y[0, :, 0, 0], np.array(ref)) < 1e-13
    assert rel_err(fin.h[0, 0], h) < 1e-13
    assert np.max(np.abs(fin.b_prev[0, 0, 0] - Bm[-1])) < 1e-15


# --------------------------------------------------------------------------
# second-order accuracy (golden: closed-form ODE solution)
# --------------------------------------------------------------------------
def _ode_error(step, lam, A, T, hT):
    n = int(round(T / step))
    tau = step * np.arange(1, n + 1)
    inp = dict(
        x=np.sin(tau).reshape(1, n, 1, 1, 1),
        B=np.tile(np.array([1.0, 0.0]), (1, n, 1, 1, 1)),
        C=np.tile(np.array([1.0, 0.0]), (1, n, 1, 1, 1)),
        theta=np.zeros((1, n, 1, 1)),
        dt=np.full((1, n, 1), step),
        lam=np.full((1, n, 1), lam),
        A=np.array([A]),
        D=np.array([0.0]),
    )
    y, _ = oracle.scan_complex(**inp)  # u_0 = sin(0) = 0 matches the zero carry
    return abs(y.ravel()[-1] - hT)


def test_second_order_accuracy():
    """Section 1.1: exponential-trapezoidal (lam = 1/2) is second-order accurate, the
    exponential-Euler rule (lam = 1) first order: halving the step divides the error by 4 / 2."""
    g = read_golden("trapezoid_ode.txt")
    A, T, hT = g["A"][0], g["T"][0], g["h_T"][0]
    steps = g["steps"]
    for lam, key in ((0.5, "ratio_trapezoid"), (1.0, "ratio_euler")):
        errs = [_ode_error(s, lam, A, T, hT) for s in steps]
        for e0, e1 in zip(errs, errs[1:]):
            assert abs(e0 / e1 - g[key][0]) < 0.15 * g[key][0], (lam, errs)


# --------------------------------------------------------------------------
# parity toy (golden)
# --------------------------------------------------------------------------
def test_parity_toy():
    """Section 1.2: rotation by pi per 1-bit flips the state's sign; y_t / y_1 = (-1)^(bits 2..t)."""
    g = read_golden("parity_toy.txt")
    bits = np.array(g["bits"])
    signs = np.array(g["signs"])
    L, N, P = len(bits), 4, 2
    rng = np.random.default_rng(9)
    x = np.zeros((1, L, 1, 1, P))
    x[0, 0, 0, 0] = rng.standard_normal(P)
    inp = dict(
        x=x,
        B=np.broadcast_to(rng.standard_normal(N), (1, L, 1, 1, N)).copy(),
        C=np.broadcast_to(rng.standard_normal(N), (1, L, 1, 1, N)).copy(),
        theta=np.pi * np.broadcast_to(bits[None, :, None, None], (1, L, 1, N // 2)).copy(),
        dt=np.ones((1, L, 1)),
        lam=np.ones((1, L, 1)),
        A=np.array([0.0]),
        D=np.array([0.0]),
    )
    for fn in (oracle.scan_complex, oracle.scan_rope):
        y, _ = fn(**inp)
        y = y[0, :, 0, 0]  # [L, P]
        assert np.all(np.abs(y[0]) > 1e-3)
        ratio = y / y[0]
        assert np.max(np.abs(ratio - signs[:, None])) < 1e-12


# --------------------------------------------------------------------------
# three formulations agree
# --------------------------------------------------------------------------
@pytest.mark.parametrize("R", [1, 3])
def test_complex_equals_rope(R):
    """Section 1.2: the complex-state SSM equals the real SSM with B, C rotated by the
    accumulated angle; checked on y and on the exported state, from a random init state."""
    rng = np.random.default_rng(21 + R)
    b, L, H, P, N = 2, 31, 3, 5, 8
    inp = rand_inputs(b, L, H, P, N, R, rng)
    s0 = rand_state(b, H, P, N, R, rng)
    y1, f1 = oracle.scan_complex(**inp, init=s0)
    y2, f2 = oracle.scan_rope(**inp, init=s0)
    assert rel_err(y2, y1) < 1e-12
    for a, c in ((f2.h, f1.h), (f2.b_prev, f1.b_prev), (f2.x_prev, f1.x_prev), (f2.angle, f1.angle)):
        assert rel_err(a, c) < 1e-12


@pytest.mark.parametrize("R", [1, 2])
def test_quadratic_equals_recurrence(R):
    """Brute-force L x L masked kernel (the unrolled update, with the block-causal R x R
    diagonal blocks of MIMO) equals the sequential recurrence."""
    rng = np.random.default_rng(31 + R)
    b, L, H, P, N = 1, 24, 2, 4, 6
    inp = rand_inputs(b, L, H, P, N, R, rng)
    s0 = rand_state(b, H, P, N, R, rng)
    yq = oracle.scan_quadratic(**inp, init=s0)
    yc, _ = oracle.scan_complex(**inp, init=s0)
    assert rel_err(yq, yc) < 1e-12


# --------------------------------------------------------------------------
# MIMO: superposition of rank-1 systems
# --------------------------------------------------------------------------
def test_mimo_is_superposition_of_siso():
    """Section 1.3: the rank-R input term sum_r B_t[:,r] x_t[:,r]^T; by linearity the MIMO
    state is the sum of R SISO states and output r reads that sum through C_t[:,r]."""
    rng = np.random.default_rng(41)
    b, L, H, P, N, R = 1, 19, 2, 3, 6, 3
    inp = rand_inputs(b, L, H, P, N, R, rng)
    inp["D"][:] = 0.0
    y, fin = oracle.scan_complex(**inp)
    for r in range(R):
        acc = np.zeros((b, L, H, 1, P))
        hsum = np.zeros_like(fin.h)
        for r2 in range(R):
            sub = dict(inp)
            sub["B"] = inp["B"][:, :, :, r2:r2 + 1]
            sub["x"] = inp["x"][:, :, :, r2:r2 + 1]
            sub["C"] = inp["C"][:, :, :, r:r + 1]
            ys, fs = oracle.scan_complex(**sub)
            acc += ys
            hsum += fs.h
        assert rel_err(y[:, :, :, r], acc[:, :, :, 0]) < 1e-12
        assert rel_err(fin.h, hsum) < 1e-12


# --------------------------------------------------------------------------
# composition: the exported state is a resume point
# --------------------------------------------------------------------------
@pytest.mark.parametrize("R", [1, 2])
def test_prefill_then_decode_equals_longer_prefill(R):
    rng = np.random.default_rng(51 + R)
    b, L, H, P, N, k = 2, 20, 2, 3, 8, 13
    inp = rand_inputs(b, L, H, P, N, R, rng)
    y_all, f_all = oracle.scan_complex(**inp)
    _, st = oracle.scan_complex(**slice_t(inp, 0, k))
    ys = []
    for t in range(k, L):
        yt, st = oracle.decode_step(st, *(inp[n][:, t] for n in ("x", "B", "C", "theta", "dt", "lam")),
                                    inp["A"], inp["D"])
        ys.append(yt)
    assert rel_err(np.stack(ys, 1), y_all[:, k:]) < 1e-12
    assert rel_err(st.h, f_all.h) < 1e-12
    assert rel_err(st.b_prev, f_all.b_prev) < 1e-12
    assert rel_err(st.x_prev, f_all.x_prev) < 1e-12


def test_split_prefill_equals_one_prefill():
    rng = np.random.default_rng(61)
    b, L, H, P, N, R, k = 1, 30, 3, 4, 6, 2, 11
    inp = rand_inputs(b, L, H, P, N, R, rng)
    s0 = rand_state(b, H, P, N, R, rng)
    y_all, f_all = oracle.scan_complex(**inp, init=s0)
    y1, s1 = oracle.scan_complex(**slice_t(inp, 0, k), init=s0)
    y2, s2 = oracle.scan_complex(**slice_t(inp, k, L), init=s1)
    assert rel_err(np.concatenate([y1, y2], 1), y_all) < 1e-12
    assert rel_err(s2.h, f_all.h) < 1e-12


def test_state_size_independent_of_length():
    """Constant-size state (paper-review page, cache-size table: 0.25 MiB at every length)."""
    rng = np.random.default_rng(71)
    sizes = set()
    for L in (1, 7, 40):
        _, f = oracle.scan_complex(**rand_inputs(1, L, 2, 3, 4, 2, rng))
        sizes.add(sum(a.nbytes for a in (f.h, f.b_prev, f.x_prev, f.angle)))
    assert len(sizes) == 1


def test_units_subset_matches_full():
    """The unit-subset option (used for sampled parity at full sizes) computes the same values."""
    rng = np.random.default_rng(81)
    inp = rand_inputs(2, 12, 3, 3, 4, 1, rng)
    y, f = oracle.scan_complex(**inp)
    ys, fs = oracle.scan_complex(**inp, units=[1, 4])
    for u in (1, 4):
        bb, hh = divmod(u, 3)
        assert np.array_equal(ys[bb, :, hh], y[bb, :, hh])
        assert np.array_equal(fs.h[bb, hh], f.h[bb, hh])


# ---------------------------------------------------------------- B/C normalisation
# "Mamba-3: 2x smaller state ..." (MarkTechPost, Korean translation), section 2:
# RMS norm of B and C over the state dimension, then a head-specific weight and bias.

def test_bc_norm_constant_row_closed_form():
    """A constant row c * 1_N gives c / sqrt(c^2 + eps) exactly: pins the mean (not
    the sum) over N and eps inside the square root (eps dominates here)."""
    N, c, eps = 16, 1e-3, 1e-4
    z = np.full((1, 1, 1, 1, N), c)
    out = oracle.bc_norm(z, eps=eps)
    assert np.allclose(out, c / np.sqrt(c * c + eps), rtol=1e-14, atol=0)
    assert abs(out[0, 0, 0, 0, 0] - 0.0995037190209989) < 1e-15


def test_bc_norm_unit_rms_per_row():
    """With eps = 0, unit weight and no bias every (b, t, h, r) row has RMS 1 over
    N, whatever the scale of the rows (pins the axis of the norm)."""
    rng = np.random.default_rng(91)
    z = rng.normal(size=(2, 5, 3, 2, 8)) * rng.uniform(0.01, 100.0, size=(2, 5, 3, 2, 1))
    out = oracle.bc_norm(z, eps=0.0)
    assert np.allclose(np.sqrt((out ** 2).mean(-1)), 1.0, rtol=1e-13)


def test_bc_norm_scale_invariant_and_odd():
    rng = np.random.default_rng(92)
    z = rng.normal(size=(1, 4, 2, 3, 8))
    base = oracle.bc_norm(z, eps=0.0)
    assert np.allclose(oracle.bc_norm(7.5 * z, eps=0.0), base, rtol=1e-13)
    assert np.allclose(oracle.bc_norm(-z, eps=0.0), -base, rtol=1e-13)


def test_bc_norm_weight_and_bias_per_head_and_rank():
    """Weight and bias index (head, rank, n): with H != R and distinct values per
    (h, r), a transposed or shared operand moves the rows' means away from the
    bias and their scale away from the weight."""
    rng = np.random.default_rng(93)
    H, R, N = 3, 2, 8
    z = rng.normal(size=(2, 6, H, R, N))
    w = rng.uniform(0.5, 2.0, size=(H, R, N))
    bias = rng.normal(size=(H, R, N)) * 3
    out = oracle.bc_norm(z, w, bias, eps=0.0)
    unit = oracle.bc_norm(z, eps=0.0)
    assert np.allclose((out - bias) / w, unit, rtol=1e-12, atol=1e-12)
    for h in range(H):
        for r in range(R):
            rows = (out[:, :, h, r, :] - bias[h, r]) / w[h, r]
            assert np.allclose(np.sqrt((rows ** 2).mean(-1)), 1.0, rtol=1e-12)


def test_bc_norm_zero_row_gives_bias():
    """Reading: an all-zero row with eps = 0 (0/0) normalises to 0, leaving the bias."""
    H, R, N = 2, 1, 8
    z = np.zeros((1, 1, H, R, N))
    bias = np.arange(H * R * N, dtype=np.float64).reshape(H, R, N)
    out = oracle.bc_norm(z, None, bias, eps=0.0)
    assert np.array_equal(out[0, 0], bias)


# ---------------------------------------------------------------- time-varying decay A_t
# "Mamba-3: 2x smaller state ..." (MarkTechPost, Korean translation), section 1.1
# writes the discretisation with a per-step A_t: each step's pole is exp(dt_t A_t).

@pytest.mark.parametrize("fn", ["scan_complex", "scan_rope", "scan_quadratic"])
def test_time_varying_decay_impulse_closed_form(fn):
    """Single impulse at t0 with a per-token A_t: the pole product runs over the
    per-token rates, H_t = prod_{q=t0+1..t} exp(dt_q (A_q + i theta_q)) * w_hat * u."""
    rng = np.random.default_rng(111)
    L, N, P, R, t0 = 15, 6, 3, 2, 4
    inp = rand_inputs(1, L, 1, P, N, R, rng)
    inp["x"][:] = 0
    inp["x"][0, t0] = rng.standard_normal((1, R, P))
    inp["D"][:] = 0.0
    At = -rng.uniform(0.1, 3.0, (1, L, 1))
    inp["A"] = At
    y = getattr(oracle, fn)(**inp)
    y = y[0] if isinstance(y, tuple) else y
    dt, lam, th = inp["dt"][0, :, 0], inp["lam"][0, :, 0], inp["theta"][0, :, 0]
    a_t = At[0, :, 0]
    Bc = inp["B"][0, :, 0, :, 0::2] + 1j * inp["B"][0, :, 0, :, 1::2]
    Cc = inp["C"][0, :, 0, :, 0::2] + 1j * inp["C"][0, :, 0, :, 1::2]
    u = np.einsum("rk,rp->kp", Bc[t0], inp["x"][0, t0, 0])
    ref = np.zeros((L, R, P))
    w_hat = lam[t0] * dt[t0] + (1 - lam[t0 + 1]) * dt[t0 + 1]
    for t in range(t0, L):
        if t == t0:
            Ht = lam[t0] * dt[t0] * u
        else:
            logp = np.sum(dt[t0 + 1:t + 1, None] * (a_t[t0 + 1:t + 1, None] + 1j * th[t0 + 1:t + 1]), axis=0)
            Ht = np.exp(logp)[:, None] * w_hat * u
        ref[t] = np.real(np.einsum("rk,kp->rp", np.conj(Cc[t]), Ht))
    assert rel_err(y[0, :, 0], ref) < 1e-12


def test_time_varying_decay_constant_in_time_is_per_head():
    """A_t[b, t, h] = A[h] for every token reproduces the per-head recurrence."""
    rng = np.random.default_rng(112)
    inp = rand_inputs(2, 19, 3, 4, 6, 2, rng)
    y, f = oracle.scan_complex(**inp)
    tv = dict(inp, A=np.broadcast_to(inp["A"], inp["dt"].shape).copy())
    y2, f2 = oracle.scan_complex(**tv)
    assert rel_err(y2, y) < 1e-14 and rel_err(f2.h, f.h) < 1e-14


@pytest.mark.parametrize("R", [1, 3])
def test_time_varying_decay_forms_agree(R):
    """Complex == RoPE == quadratic with a per-token decay (the chunk algebra of the
    quadratic form multiplies per-token poles)."""
    rng = np.random.default_rng(113 + R)
    inp = rand_inputs(1, 21, 2, 3, 6, R, rng)
    inp["A"] = -rng.uniform(0.05, 2.5, inp["dt"].shape)
    yc, _ = oracle.scan_complex(**inp)
    yr, _ = oracle.scan_rope(**inp)
    yq = oracle.scan_quadratic(**inp)
    assert rel_err(yr, yc) < 1e-12 and rel_err(yq, yc) < 1e-12


def test_time_varying_decay_prefill_then_decode():
    rng = np.random.default_rng(114)
    b, L, H, P, N, R, k = 2, 12, 2, 3, 4, 2, 8
    inp = rand_inputs(b, L, H, P, N, R, rng)
    inp["A"] = -rng.uniform(0.05, 2.5, (b, L, H))
    y_all, f_all = oracle.scan_complex(**inp)
    _, st = oracle.scan_complex(**slice_t(inp, 0, k))
    for t in range(k, L):
        step = {n: inp[n][:, t] for n in ("x", "B", "C", "theta", "dt", "lam", "A")}
        yt, st = oracle.decode_step(st, **step, D=inp["D"])
        assert rel_err(yt, y_all[:, t]) < 1e-12
    assert rel_err(st.h, f_all.h) < 1e-12


# ---------------------------------------------------------------- grouped B/C
# The pages give every head its own B and C.  The Mamba line also shares one B and
# C among a group of consecutive heads (ngroups G, head h reads group h // (H // G));
# the reading here: a grouped input is exactly the per-head input with each group's
# rows repeated over its heads.

@pytest.mark.parametrize("fn", ["scan_complex", "scan_rope", "scan_quadratic"])
@pytest.mark.parametrize("G,R", [(1, 1), (2, 2), (3, 1)])
def test_grouped_bc_equals_per_head_broadcast(fn, G, R):
    rng = np.random.default_rng(120 + 7 * G + R)
    b, L, H, P, N = 2, 17, 6, 3, 6
    inp = rand_inputs(b, L, H, P, N, R, rng)
    grp = dict(inp, B=rng.standard_normal((b, L, G, R, N)), C=rng.standard_normal((b, L, G, R, N)))
    rep = dict(inp, B=np.repeat(grp["B"], H // G, axis=2), C=np.repeat(grp["C"], H // G, axis=2))
    out_g = getattr(oracle, fn)(**grp)
    out_r = getattr(oracle, fn)(**rep)
    if isinstance(out_g, tuple):
        (yg, fg), (yr, fr) = out_g, out_r
        for n in ("h", "b_prev", "x_prev", "angle"):
            assert np.array_equal(getattr(fg, n), getattr(fr, n)), n
    else:
        yg, yr = out_g, out_r
    assert np.array_equal(yg, yr)


def test_grouped_bc_prefill_then_decode():
    rng = np.random.default_rng(131)
    b, L, H, P, N, R, G, k = 2, 12, 4, 3, 4, 2, 2, 7
    inp = rand_inputs(b, L, H, P, N, R, rng)
    inp["B"] = rng.standard_normal((b, L, G, R, N))
    inp["C"] = rng.standard_normal((b, L, G, R, N))
    y_all, f_all = oracle.scan_complex(**inp)
    _, st = oracle.scan_complex(**slice_t(inp, 0, k))
    for t in range(k, L):
        step = {n: inp[n][:, t] for n in ("x", "B", "C", "theta", "dt", "lam")}
        yt, st = oracle.decode_step(st, **step, A=inp["A"], D=inp["D"])
        assert rel_err(yt, y_all[:, t]) < 1e-12
    assert rel_err(st.h, f_all.h) < 1e-12


# ---------------------------------------------------------------- output side
# "Mamba-3: 2x smaller state ..." (MarkTechPost, Korean translation), section 2:
# a grouped RMS norm ahead of the output gate.  Pins: silu's exact values and its
# odd part, unit RMS of the normalised group, scale invariance, group locality,
# and the weight placed per (head, rank, channel).

def _gn_case(rng, b=2, L=5, H=6, R=2, P=4):
    return rng.standard_normal((b, L, H, R, P)), rng.standard_normal((b, L, H, R, P))


def test_gate_is_silu_at_exact_points():
    """z = 0 closes the gate; z = +-1 give +-1 / (1 + e^{-+1}) times the norm."""
    rng = np.random.default_rng(141)
    y, _ = _gn_case(rng)
    n1 = oracle.gated_norm(y, np.ones_like(y), eps=0.0)
    assert np.array_equal(oracle.gated_norm(y, np.zeros_like(y)), np.zeros_like(y))
    nm1 = oracle.gated_norm(y, -np.ones_like(y), eps=0.0)
    # silu(1) = 0.7310585786300049, silu(-1) = -0.2689414213699951
    assert np.allclose(nm1 / n1, -0.2689414213699951 / 0.7310585786300049, rtol=1e-13)


def test_gate_odd_part_is_the_identity():
    """silu(z) - silu(-z) = z, so out(z) - out(-z) = norm(y) w z exactly (no sigmoid)."""
    rng = np.random.default_rng(142)
    y, z = _gn_case(rng)
    w = rng.uniform(0.5, 1.5, (6, 2, 4))
    d = oracle.gated_norm(y, z, w, groups=3) - oracle.gated_norm(y, -z, w, groups=3)
    ones = oracle.gated_norm(y, np.ones_like(z), w, groups=3) - oracle.gated_norm(y, -np.ones_like(z), w, groups=3)
    assert np.allclose(d, ones * z, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("groups", [1, 2, 6])
def test_normalised_group_has_unit_rms(groups):
    """With the gate's odd part (out(z) - out(-z) = norm(y) z) at z = 1 and w = 1,
    every group of H / groups heads has unit RMS over its (h, r, p) channels."""
    rng = np.random.default_rng(143 + groups)
    y, _ = _gn_case(rng)
    one = np.ones_like(y)
    nrm = oracle.gated_norm(y, one, groups=groups, eps=0.0) - oracle.gated_norm(y, -one, groups=groups, eps=0.0)
    g = nrm.reshape(2, 5, groups, -1)
    assert np.allclose(np.sqrt((g ** 2).mean(axis=-1)), 1.0, rtol=1e-13)


def test_gated_norm_scale_invariant_and_group_local():
    rng = np.random.default_rng(145)
    y, z = _gn_case(rng)
    out = oracle.gated_norm(y, z, groups=3, eps=0.0)
    assert np.allclose(oracle.gated_norm(7.5 * y, z, groups=3, eps=0.0), out, rtol=1e-13)
    y2 = y.copy()
    y2[:, :, 2:4] *= rng.uniform(0.1, 10.0, y2[:, :, 2:4].shape)  # heads 2, 3 = group 1 of 3
    out2 = oracle.gated_norm(y2, z, groups=3, eps=0.0)
    assert np.array_equal(out2[:, :, :2], out[:, :, :2]) and np.array_equal(out2[:, :, 4:], out[:, :, 4:])
    assert not np.allclose(out2[:, :, 2:4], out[:, :, 2:4])


def test_gated_norm_weight_per_head_rank_channel_and_eps():
    rng = np.random.default_rng(146)
    y, z = _gn_case(rng)
    w = rng.uniform(0.5, 1.5, (6, 2, 4))
    assert np.allclose(oracle.gated_norm(y, z, w, groups=2), oracle.gated_norm(y, z, groups=2) * w, rtol=1e-14)
    # a constant group c: mean square c^2, so out = c / sqrt(c^2 + eps) silu(z)
    c, eps = 0.01, 1e-3
    yc = np.full_like(y, c)
    one = np.ones_like(y)
    nrm = oracle.gated_norm(yc, one, eps=eps) - oracle.gated_norm(yc, -one, eps=eps)
    assert np.allclose(nrm, c / np.sqrt(c * c + eps), rtol=1e-13)
