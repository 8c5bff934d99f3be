"""GPU pre-gate grouped RMS norm and gate (mamba3_gated_norm) against the fp64
oracle (oracle.gated_norm).  Bars: 1e-4 (fp32), 2e-2 (bf16), max|err| / max|ref|."""
import pytest
import torch

import linear_recurrent_scan_b200 as m3
import oracle
from linear_recurrent_scan_b200 import build as m3build
from tests.conftest import rel_err
from tests.parity_util import TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()


def draw(shape, dtype, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    y = torch.randn(shape, generator=g, device="cuda") * torch.exp(torch.randn(shape[:-3] + (1, 1, 1), generator=g,
                                                                              device="cuda"))
    z = torch.randn(shape, generator=g, device="cuda") * 2.0
    w = torch.rand(shape[-3:], generator=g, device="cuda") + 0.5
    return y.to(dtype).contiguous(), z.to(dtype).contiguous(), w


def f64(t):
    return t.detach().double().cpu().numpy()


# (shape [..., H, R, P], groups): group size S = H / groups * R * P covers the
# team kernel (S / 8 or S / 4 lanes in {1, ..., 32}), the vector row kernel and
# the element-wise row kernel
CASES = [
    ((2, 50, 8, 1, 8), 8),        # bf16 S = 8: one lane per group
    ((2, 50, 8, 1, 64), 8),       # S = 64 (one SISO head)
    ((2, 50, 8, 1, 64), 2),       # S = 256: 32 lanes
    ((2, 30, 8, 2, 64), 2),       # S = 512: row kernel, 16-byte accesses
    ((1, 40, 6, 3, 4), 6),        # S = 12: row kernel, element-wise (bf16)
    ((1, 40, 6, 3, 4), 2),        # S = 36
    ((1, 10, 8, 4, 64), 2),       # S = 1024: 32 lanes x 4 vectors (bf16)
    ((1, 10, 8, 4, 64), 1),       # S = 2048: row kernel, 256 threads
    ((3, 17, 64, 4, 64), 64),     # MIMO R = 4 heads
    ((128, 64, 1, 64), 64),       # one decode step's output [b, H, R, P]
]


@pytest.mark.parametrize("shape,groups", CASES)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("with_w", [True, False])
def test_gated_norm_matches_oracle(shape, groups, dtype, with_w):
    y, z, w = draw(shape, dtype, seed=3000 + sum(shape) + groups)
    w = w if with_w else None
    out = m3.mamba3_gated_norm(y, z, w, groups=groups, eps=1e-6)
    torch.cuda.synchronize()
    ref = oracle.gated_norm(f64(y), f64(z), f64(w) if w is not None else None, groups=groups, eps=1e-6)
    assert rel_err(f64(out), ref) < TOL[dtype]


def test_gated_norm_in_place_and_zero_groups():
    y, z, w = draw((2, 33, 8, 1, 64), torch.bfloat16, seed=3100)
    y[0, 3] = 0.0  # all-zero groups with eps = 0 give 0
    ref = oracle.gated_norm(f64(y), f64(z), f64(w), groups=4, eps=0.0)
    out = m3.mamba3_gated_norm(y, z, w, groups=4, eps=0.0, out=y)
    torch.cuda.synchronize()
    assert out.data_ptr() == y.data_ptr()
    assert rel_err(f64(y), ref) < TOL[torch.bfloat16]
    assert torch.count_nonzero(y[0, 3]) == 0 and not torch.isnan(y).any()


def test_gated_norm_after_the_prefill():
    """The output side on the prefill's y (SISO b2 L300 H8): the same as the oracle
    applied to the oracle's own y."""
    from tests.parity_util import NAMES, oracle_scan, small_inputs
    inp = small_inputs(2, 300, 8, 64, 128, 1, torch.bfloat16, seed=3200)
    y = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"])
    _, z, w = draw(tuple(y.shape), torch.bfloat16, seed=3201)
    out = m3.mamba3_gated_norm(y, z, w, groups=8)
    torch.cuda.synchronize()
    yr, _ = oracle_scan(inp)
    ref = oracle.gated_norm(yr, f64(z), f64(w), groups=8)
    assert rel_err(f64(out), ref) < TOL[torch.bfloat16]
