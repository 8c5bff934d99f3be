"""GPU MIMO rank-R projections (mamba3_mimo_up, mamba3_mimo_down with and without
the fused RMS norm and silu gate) against the fp64 oracle (oracle.mimo_up,
oracle.mimo_down, oracle.gated_norm) on the same bf16-rounded inputs.

Tolerance: max|err| / max|ref| <= 2e-2 (bf16 inputs and outputs, fp32
accumulation), the bound the recurrence's bf16 tests use."""
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
TOLB = TOL[torch.bfloat16]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()


def f64(t):
    return t.detach().float().cpu().double().numpy()


def weights(H, R, P, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    s = P ** -0.5
    Wx = (torch.randn(H, R * P, P, generator=g, device="cuda") * s).to(torch.bfloat16)
    Wy = (torch.randn(H, P, R * P, generator=g, device="cuda") * (R * P) ** -0.5).to(torch.bfloat16)
    return Wx, Wy


def randn(shape, seed, scale=1.0):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device="cuda") * scale).to(torch.bfloat16)


@pytest.mark.parametrize("R", [1, 2, 4])
@pytest.mark.parametrize("b,L,H", [(1, 1, 1), (2, 100, 3), (1, 300, 2)])
def test_up_matches_oracle(R, b, L, H):
    P = 64
    u = randn((b, L, H, P), 6100 + L + R)
    Wx, _ = weights(H, R, P, 6200 + R)
    x = m3.mamba3_mimo_up(u, Wx)
    torch.cuda.synchronize()
    assert x.shape == (b, L, H, R, P)
    assert rel_err(f64(x), oracle.mimo_up(f64(u), f64(Wx), R)) < TOLB


@pytest.mark.parametrize("R", [1, 2, 4])
@pytest.mark.parametrize("gate", [False, True])
@pytest.mark.parametrize("b,L,H", [(1, 1, 1), (2, 100, 3), (1, 300, 2)])
def test_down_matches_oracle(R, gate, b, L, H):
    P = 64
    y = randn((b, L, H, R, P), 6300 + L + R)
    _, Wy = weights(H, R, P, 6400 + R)
    z = randn((b, L, H, P), 6500 + L, scale=2.0) if gate else None
    w = (torch.rand(H, P, device="cuda") + 0.5) if gate else None
    o = m3.mamba3_mimo_down(y, Wy, z=z, w=w, eps=1e-6)
    torch.cuda.synchronize()
    assert o.shape == (b, L, H, P)
    ref = oracle.mimo_down(f64(y), f64(Wy))
    if gate:
        ref = oracle.gated_norm(ref[..., None, :], f64(z)[..., None, :], f64(w)[:, None, :], eps=1e-6)[..., 0, :]
    assert rel_err(f64(o), ref) < TOLB


def test_gate_with_zero_rows_and_no_weight():
    """Tokens whose projected row is zero give 0 with eps = 0 (no 0/0); w = None is weight 1."""
    b, L, H, R, P = 1, 130, 2, 2, 64
    y = randn((b, L, H, R, P), 6600)
    y[:, 5] = 0
    _, Wy = weights(H, R, P, 6601)
    z = randn((b, L, H, P), 6602)
    o = m3.mamba3_mimo_down(y, Wy, z=z, w=None, eps=0.0)
    torch.cuda.synchronize()
    assert torch.count_nonzero(o[:, 5]) == 0 and torch.isfinite(o.float()).all()
    ref = oracle.gated_norm(oracle.mimo_down(f64(y), f64(Wy))[..., None, :], f64(z)[..., None, :], None,
                            eps=0.0)[..., 0, :]
    assert rel_err(f64(o), np.nan_to_num(ref)) < TOLB


def test_mimo_layer_up_scan_down_matches_oracle():
    """The MIMO layer core end to end: u -> up (rank 4) -> chunked prefill -> down
    + gate, against the oracle's up -> complex-state scan -> down -> gated norm on
    the GPU's bf16-rounded intermediates (each stage is checked on its own input)."""
    b, L, H, P, N, R = 1, 200, 4, 64, 128, 4
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=6700)
    u = randn((b, L, H, P), 6701)
    Wx, Wy = weights(H, R, P, 6702)
    x = m3.mamba3_mimo_up(u, Wx)
    inp["x"] = x
    y = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"])
    z = randn((b, L, H, P), 6703)
    w = torch.rand(H, P, device="cuda") + 0.5
    o = m3.mamba3_mimo_down(y, Wy, z=z, w=w)
    torch.cuda.synchronize()
    assert rel_err(f64(x), oracle.mimo_up(f64(u), f64(Wx), R)) < TOLB
    f = wl.to_f64({k: inp[k] for k in (*NAMES, "A", "D")})
    yr, _ = oracle.scan_complex(**f)
    assert rel_err(f64(y), yr) < TOLB
    ref = oracle.gated_norm(oracle.mimo_down(f64(y), f64(Wy))[..., None, :], f64(z)[..., None, :],
                            f64(w)[:, None, :])[..., 0, :]
    assert rel_err(f64(o), ref) < TOLB


@pytest.mark.parametrize("R", [2, 4])
def test_head_switches_inside_persistent_ctas(R):
    """512 (head, tile) items on at most 296 persistent CTAs: most CTAs take two or
    more items and many cross a head boundary, so the weight buffers are reloaded
    mid-range (the gated R = 4 down projection has a single weight buffer).  Every
    output row is checked, and the library status stays clean."""
    b, L, H, P = 1, 8192, 8, 64
    u = randn((b, L, H, P), 6900 + R)
    Wx, Wy = weights(H, R, P, 6910 + R)
    z = randn((b, L, H, P), 6920 + R)
    w = torch.rand(H, P, device="cuda") + 0.5
    x = m3.mamba3_mimo_up(u, Wx)
    o = m3.mamba3_mimo_down(x, Wy)
    og = m3.mamba3_mimo_down(x, Wy, z=z, w=w)
    torch.cuda.synchronize()
    assert m3.mamba3_library_status() == m3.MAMBA3_OK
    assert rel_err(f64(x), oracle.mimo_up(f64(u), f64(Wx), R)) < TOLB
    ref = oracle.mimo_down(f64(x), f64(Wy))
    assert rel_err(f64(o), ref) < TOLB
    refg = oracle.gated_norm(ref[..., None, :], f64(z)[..., None, :], f64(w)[:, None, :])[..., 0, :]
    assert rel_err(f64(og), refg) < TOLB


def test_full_size_sampled_tokens():
    """MIMO R4 prefill size (b4 L8192 H64): sampled (token, head) rows against the oracle."""
    b, L, H, R, P = 4, 8192, 64, 4, 64
    u = randn((b, L, H, P), 6800)
    Wx, Wy = weights(H, R, P, 6801)
    x = m3.mamba3_mimo_up(u, Wx)
    z = randn((b, L, H, P), 6802)
    o = m3.mamba3_mimo_down(x, Wy, z=z)
    torch.cuda.synchronize()
    assert m3.mamba3_library_status() == m3.MAMBA3_OK
    rows = [(0, 0), (1, 4095), (2, 8191), (3, 77)]
    for bb, t in rows:
        xs = oracle.mimo_up(f64(u[bb, t]), f64(Wx), R)
        assert rel_err(f64(x[bb, t]), xs) < TOLB
        os_ = oracle.gated_norm(oracle.mimo_down(f64(x[bb, t]), f64(Wy))[:, None, :], f64(z[bb, t])[:, None, :],
                                None)[:, 0, :]
        assert rel_err(f64(o[bb, t]), os_) < TOLB
