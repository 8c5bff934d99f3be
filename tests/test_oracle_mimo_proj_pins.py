"""Pins of the oracle's MIMO rank-R projections (oracle.mimo_up, mimo_down).

"Mamba-3: 2x smaller state ..." (MarkTechPost, Korean translation), section 1.3:
MIMO raises the rank of the input and output projections so that x_t is P x R.
The reading: one dense matrix per head on each side, x[.., h, r, p] =
sum_q Wx[h, rP + p, q] u[.., h, q] and o[.., h, p] = sum_{r,q} Wy[h, p, rP + q]
y[.., h, r, q].  The pins: a library matrix product (numpy einsum) on random
inputs, identity weights (R = 1 is SISO), rank-1 weights in closed form, and
replicated / averaged ranks."""
import numpy as np
import pytest

import oracle


def rnd(*shape, seed=0):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("R", [1, 2, 4])
def test_up_and_down_equal_library_matrix_products(R):
    b, L, H, P = 2, 7, 3, 8
    u = rnd(b, L, H, P, seed=R)
    Wx = rnd(H, R * P, P, seed=10 + R)
    Wy = rnd(H, P, R * P, seed=20 + R)
    x = oracle.mimo_up(u, Wx, R)
    assert x.shape == (b, L, H, R, P)
    ref_x = np.einsum("hkq,blhq->blhk", Wx, u).reshape(b, L, H, R, P)
    assert np.abs(x - ref_x).max() < 1e-12
    o = oracle.mimo_down(x, Wy)
    ref_o = np.einsum("hpk,blhk->blhp", Wy, x.reshape(b, L, H, R * P))
    assert np.abs(o - ref_o).max() < 1e-12


def test_identity_weights_are_siso():
    b, L, H, P = 1, 5, 2, 6
    u = rnd(b, L, H, P, seed=3)
    eye = np.stack([np.eye(P)] * H)
    assert np.array_equal(oracle.mimo_up(u, eye, 1)[:, :, :, 0], u)
    y = rnd(b, L, H, 1, P, seed=4)
    assert np.array_equal(oracle.mimo_down(y, eye), y[:, :, :, 0])


def test_rank_one_weights_closed_form():
    """Wx[h] = a_h c_h^T gives x[.., h] = a_h <c_h, u[.., h]> (a scaled copy of a_h)."""
    b, L, H, P, R = 2, 4, 3, 5, 2
    a = rnd(H, R * P, seed=5)
    c = rnd(H, P, seed=6)
    Wx = a[:, :, None] * c[:, None, :]
    u = rnd(b, L, H, P, seed=7)
    x = oracle.mimo_up(u, Wx, R).reshape(b, L, H, R * P)
    dots = (u * c[None, None]).sum(-1)
    assert np.abs(x - dots[..., None] * a[None, None]).max() < 1e-12


def test_replicated_and_averaged_ranks():
    """Stacked identities copy u into every rank; [I/R ... I/R] averages the ranks."""
    b, L, H, P, R = 1, 3, 2, 4, 4
    u = rnd(b, L, H, P, seed=8)
    Wx = np.stack([np.vstack([np.eye(P)] * R)] * H)
    x = oracle.mimo_up(u, Wx, R)
    for r in range(R):
        assert np.array_equal(x[:, :, :, r], u)
    y = rnd(b, L, H, R, P, seed=9)
    Wy = np.stack([np.hstack([np.eye(P) / R] * R)] * H)
    assert np.abs(oracle.mimo_down(y, Wy) - y.mean(axis=3)).max() < 1e-12
