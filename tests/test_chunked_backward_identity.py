"""The chunked backward algebra that the GPU backward kernel follows, restated in
fp64 numpy and checked against the oracle's token-by-token adjoint
(oracle.scan_bwd, pinned to finite differences).  CPU only.

Per chunk (rows m = (token, rank), kernel K(t, t) = gamma_t, K(t, j < t) =
e^{cum_t - cum_j} w_j, P1 = C~ B~^T, P2 = dY X^T, G = dL/dhbar at the chunk end):
  dC~ = diag(e^cum) dY hbar_in^T + (K o P2) B~
  dB~ = diag(w e^{cum_end - cum}) X G^T + (K o P2)^T C~
  dX  = diag(w e^{cum_end - cum}) B~ G + (K o P1)^T dY + D dY
  dL/dhbar_in = e^{cum_end} G + C~^T diag(e^cum) dY
and the decay's gradient at token i sums every path that crosses it.  The lagged
weight of a chunk's first token sits in the previous chunk's last w, so its dt
and lam gradients complete one chunk later.  Agreement for chunk sizes 1, 3, 8
and the whole sequence, with ragged tails, checks that derivation exactly.
"""
import numpy as np
import pytest

import oracle


def rot(v0, v1, ph):
    c, s = np.cos(ph), np.sin(ph)
    return c * v0 + s * v1, -s * v0 + c * v1


def rotate_rows(Z, Phi):
    """Z [L, R, N] rotated pairwise by -Phi [L, K]."""
    out = np.empty_like(Z)
    a, b = rot(Z[..., 0::2], Z[..., 1::2], Phi[:, None, :])
    out[..., 0::2], out[..., 1::2] = a, b
    return out


def chunked_backward_unit(x, B, C, th, dt, lam, a_h, Dh, dy, st0, dfin, Q):
    """One (batch, head) unit: x [L,R,P], B, C [L,R,N], th [L,K], dt, lam [L];
    st0 / dfin: (h, b_prev, x_prev, angle) of the initial state and of the exported
    state's gradient, or None."""
    L, R, P = x.shape
    N = B.shape[-1]
    K = N // 2
    h0, bp0, xp0, ang0 = st0 if st0 is not None else (np.zeros((N, P)), np.zeros((R, N)), np.zeros((R, P)),
                                                        np.zeros(K))
    Phi = ang0 + np.cumsum(dt[:, None] * th, axis=0)
    Bt, Ct = rotate_rows(B, Phi), rotate_rows(C, Phi)
    dt_n = np.append(dt[1:], 0.0)
    lam_n = np.append(lam[1:], 1.0)
    gam = lam * dt
    w = gam + (1.0 - lam_n) * dt_n
    mu1 = (1.0 - lam[0]) * dt[0]
    u_init = np.einsum("rn,rp->np", bp0, xp0)
    chunks = [(t0, min(Q, L - t0)) for t0 in range(0, L, Q)]

    # pass 1: hbar at every chunk start
    hb = h0 + mu1 * u_init
    ck = []
    for t0, q in chunks:
        ck.append(hb.copy())
        cum = np.cumsum(dt[t0:t0 + q] * a_h)
        cend = cum[-1]
        U = np.einsum("jrn,jrp->jnp", Bt[t0:t0 + q], x[t0:t0 + q])
        hb = np.exp(cend) * hb + np.einsum("j,jnp->np", np.exp(cend - cum) * w[t0:t0 + q], U)

    # pass 2
    G = dfin[0].copy() if dfin is not None else np.zeros((N, P))
    S = dfin[3].copy() if dfin is not None else np.zeros(K)
    out = dict(dx=np.zeros_like(x), dB=np.zeros_like(B), dC=np.zeros_like(C), dtheta=np.zeros_like(th),
               ddt=np.zeros(L), dlam=np.zeros(L))
    dA = dD = 0.0
    pend = None  # (token, ddt without its lagged share, dlam without it)
    for ci in reversed(range(len(chunks))):
        t0, q = chunks[ci]
        M = q * R
        hbin = ck[ci]
        cum = np.cumsum(dt[t0:t0 + q] * a_h)
        cend = cum[-1]
        tok = np.arange(M) // R
        Cm, Bm = Ct[t0:t0 + q].reshape(M, N), Bt[t0:t0 + q].reshape(M, N)
        Xm, dYm = x[t0:t0 + q].reshape(M, P), dy[t0:t0 + q].reshape(M, P)
        wt, gt = w[t0:t0 + q], gam[t0:t0 + q]
        Km = np.zeros((M, M))
        for m in range(M):
            for j in range(M):
                if tok[j] == tok[m]:
                    Km[m, j] = gt[tok[m]]
                elif tok[j] < tok[m]:
                    Km[m, j] = np.exp(cum[tok[m]] - cum[tok[j]]) * wt[tok[j]]
        P1, P2 = Cm @ Bm.T, dYm @ Xm.T
        Sm, Wm = Km * P1, Km * P2
        Zs = (P1 * P2).reshape(q, R, q, R).sum(axis=(1, 3))  # token pairs
        dg = np.diag(Zs).copy()
        T = np.zeros((q, q))
        for t in range(q):
            for j in range(t):
                T[t, j] = np.exp(cum[t] - cum[j]) * Zs[t, j]
        ee = np.exp(cend - cum)
        yi, bg = Cm @ hbin, Bm @ G
        dX = (wt * ee)[tok][:, None] * bg + Sm.T @ dYm + Dh * dYm
        zin = np.bincount(tok, weights=np.exp(cum)[tok] * (dYm * yi).sum(1), minlength=q)
        zue = np.bincount(tok, weights=ee[tok] * (Xm * bg).sum(1), minlength=q)
        dD += (dYm * Xm).sum()
        c0 = np.exp(cend) * (hbin * G).sum()
        dCt = np.exp(cum)[tok][:, None] * (dYm @ hbin.T) + Wm @ Bm
        dBt = (wt * ee)[tok][:, None] * (Xm @ G.T) + Wm.T @ Cm
        if t0 + q == L and dfin is not None:  # the exported B~_{L-1}, x_{L-1}
            dBt[(q - 1) * R:] += dfin[1]
            dX[(q - 1) * R:] += dfin[2]
        G = np.exp(cend) * G + Cm.T @ (np.exp(cum)[tok][:, None] * dYm)
        out["dx"][t0:t0 + q] = dX.reshape(q, R, P)
        # rotation back and the angle's share
        dBr, dCr = dBt.reshape(q, R, N), dCt.reshape(q, R, N)
        ph = Phi[t0:t0 + q][:, None, :]
        c_, s_ = np.cos(ph), np.sin(ph)
        out["dB"][t0:t0 + q, :, 0::2] = c_ * dBr[..., 0::2] - s_ * dBr[..., 1::2]
        out["dB"][t0:t0 + q, :, 1::2] = s_ * dBr[..., 0::2] + c_ * dBr[..., 1::2]
        out["dC"][t0:t0 + q, :, 0::2] = c_ * dCr[..., 0::2] - s_ * dCr[..., 1::2]
        out["dC"][t0:t0 + q, :, 1::2] = s_ * dCr[..., 0::2] + c_ * dCr[..., 1::2]
        Bq, Cq = Bt[t0:t0 + q], Ct[t0:t0 + q]
        dphi = (dBr[..., 0::2] * Bq[..., 1::2] - dBr[..., 1::2] * Bq[..., 0::2]
                + dCr[..., 0::2] * Cq[..., 1::2] - dCr[..., 1::2] * Cq[..., 0::2]).sum(axis=1)
        dth = np.zeros(q)
        for i in reversed(range(q)):
            S = S + dphi[i]
            out["dtheta"][t0 + i] = dt[t0 + i] * S
            dth[i] = (th[t0 + i] * S).sum()
        # per-token scalars
        cZu = np.array([T[j + 1:, j].sum() for j in range(q)])
        cT = wt * cZu
        rT = np.array([(wt[:j] * T[j, :j]).sum() for j in range(q)])
        suf_zin, pre, F, dw_prev = zin.sum(), 0.0, 0.0, 0.0
        first = None
        for i in range(q):
            da = c0 + suf_zin + pre + F
            dw = zue[i] + cZu[i]
            dgt = dg[i] + dw
            ddt = da * a_h + dgt * lam[t0 + i] + dth[i]
            dlm = dgt * dt[t0 + i]
            dA += da * dt[t0 + i]
            if i > 0:
                out["ddt"][t0 + i] = ddt + dw_prev * (1.0 - lam[t0 + i])
                out["dlam"][t0 + i] = dlm - dw_prev * dt[t0 + i]
            else:
                first = (ddt, dlm)
            suf_zin -= zin[i]
            pre += wt[i] * zue[i]
            F += cT[i] - rT[i]
            dw_prev = dw
        if pend is not None:  # the later chunk's first token takes w_{q-1}'s lagged share
            tp, pd, pl = pend
            out["ddt"][tp] = pd + dw_prev * (1.0 - lam[tp])
            out["dlam"][tp] = pl - dw_prev * dt[tp]
        pend = (t0, first[0], first[1])
    dmu = (u_init * G).sum()
    out["ddt"][0] = pend[1] + dmu * (1.0 - lam[0])
    out["dlam"][0] = pend[2] - dmu * dt[0]
    out.update(dA=dA, dD=dD, dh0=G, dbprev0=mu1 * np.einsum("np,rp->rn", G, xp0),
               dxprev0=mu1 * np.einsum("np,rn->rp", G, bp0), dangle0=S)
    return out


@pytest.mark.parametrize("Q", [1, 3, 8, 64])
@pytest.mark.parametrize("R", [1, 2])
def test_chunked_backward_equals_token_adjoint(Q, R):
    rng = np.random.default_rng(500 + 10 * Q + R)
    b, L, H, P, N = 1, 21, 2, 3, 6
    K = N // 2
    inp = dict(x=rng.standard_normal((b, L, H, R, P)), B=rng.standard_normal((b, L, H, R, N)),
               C=rng.standard_normal((b, L, H, R, N)), theta=rng.uniform(0, np.pi, (b, L, H, K)),
               dt=rng.uniform(0.05, 0.5, (b, L, H)), lam=rng.uniform(0, 1, (b, L, H)),
               A=-rng.uniform(0.2, 2, (H,)), D=rng.standard_normal(H))
    st = oracle.State(rng.standard_normal((b, H, N, P)), rng.standard_normal((b, H, R, N)),
                      rng.standard_normal((b, H, R, P)), rng.uniform(-3, 3, (b, H, K)))
    df = oracle.State(rng.standard_normal((b, H, N, P)), rng.standard_normal((b, H, R, N)),
                      rng.standard_normal((b, H, R, P)), rng.standard_normal((b, H, K)))
    dy = rng.standard_normal((b, L, H, R, P))
    ref = oracle.scan_bwd(**inp, dy=dy, init=st, d_final=df)
    for h in range(H):
        u = (0, h)
        got = chunked_backward_unit(
            inp["x"][0, :, h], inp["B"][0, :, h], inp["C"][0, :, h], inp["theta"][0, :, h], inp["dt"][0, :, h],
            inp["lam"][0, :, h], inp["A"][h], inp["D"][h], dy[0, :, h],
            (st.h[u], st.b_prev[u], st.x_prev[u], st.angle[u]), (df.h[u], df.b_prev[u], df.x_prev[u], df.angle[u]),
            Q)
        for name in ("dx", "dB", "dC", "dtheta", "ddt", "dlam"):
            r = ref[name][0, :, h]
            assert np.allclose(got[name], r, rtol=1e-10, atol=1e-10 * np.abs(r).max()), (name, h)
        for name, rr in (("dh0", ref["dh0"][u]), ("dbprev0", ref["dbprev0"][u]), ("dxprev0", ref["dxprev0"][u]),
                         ("dangle0", ref["dangle0"][u])):
            assert np.allclose(got[name], rr, rtol=1e-10, atol=1e-10 * max(1.0, np.abs(rr).max())), name
    # dA, dD sum over the heads' units in the oracle; compare per head through single-head runs
    one = {k: (v[:, :, :1] if v.ndim >= 3 else v[:1]) for k, v in inp.items()}
    r1 = oracle.scan_bwd(**one, dy=dy[:, :, :1], init=oracle.State(st.h[:, :1], st.b_prev[:, :1], st.x_prev[:, :1],
                                                                     st.angle[:, :1]),
                         d_final=oracle.State(df.h[:, :1], df.b_prev[:, :1], df.x_prev[:, :1], df.angle[:, :1]))
    g0 = chunked_backward_unit(
        inp["x"][0, :, 0], inp["B"][0, :, 0], inp["C"][0, :, 0], inp["theta"][0, :, 0], inp["dt"][0, :, 0],
        inp["lam"][0, :, 0], inp["A"][0], inp["D"][0], dy[0, :, 0],
        (st.h[0, 0], st.b_prev[0, 0], st.x_prev[0, 0], st.angle[0, 0]),
        (df.h[0, 0], df.b_prev[0, 0], df.x_prev[0, 0], df.angle[0, 0]), Q)
    assert np.isclose(g0["dA"], r1["dA"][0], rtol=1e-10) and np.isclose(g0["dD"], r1["dD"][0], rtol=1e-10)
