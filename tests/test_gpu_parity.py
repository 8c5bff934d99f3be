"""GPU vs fp64 oracle parity for the prefill (chunked scan) and the decode step.

All calls go through the C ABI (ctypes binding).  Metric: max|err| / max|ref|
over the whole output; bar 1e-4 for fp32 inputs, 2e-2 for bf16 inputs with
fp32 accumulation.  Sizes span several chunks and a ragged tail.
"""
import numpy as np
import pytest
import torch

import linear_recurrent_scan_b200 as m3
import oracle
from linear_recurrent_scan_b200 import build as m3build
from linear_recurrent_scan_b200 import workloads as wl
from tests.conftest import rel_err
from tests.parity_util import (NAMES, TOL, check_state, gpu_scan, oracle_scan, small_inputs, to_state_np,
                               unit_rows)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    m3build.build()
    m3.load_library()


# ---------------------------------------------------------------- prefill
def test_tiny_siso_fp32_config():
    """The tiny fp32 configuration (b1 L256 H2 P16 N16 R1, chunk 64) at 1e-4."""
    w = wl.CONFIGS["tiny_siso_fp32"]
    inp = wl.make_inputs(w, device="cuda")
    y, fin = gpu_scan(inp, chunk=w.chunk)
    yr, fr = oracle_scan(inp)
    assert rel_err(y.cpu().double().numpy(), yr) < 1e-4
    check_state(fin, fr, 1e-4)


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 129, 257])
@pytest.mark.parametrize("R", [1, 2, 4])
def test_ragged_lengths_fp32(L, R):
    inp = small_inputs(2, L, 3, 16, 16, R, torch.float32, seed=100 + L + R)
    y, fin = gpu_scan(inp)
    yr, fr = oracle_scan(inp)
    assert rel_err(y.cpu().double().numpy(), yr) < 1e-4
    check_state(fin, fr, 1e-4)


@pytest.mark.parametrize("shape", [
    (2, 200, 3, 64, 128, 1), (1, 300, 2, 64, 128, 4), (2, 150, 2, 64, 64, 4), (1, 97, 2, 64, 128, 2),
    (1, 130, 2, 32, 64, 1), (1, 70, 3, 16, 32, 8),
    # heads a multiple of 8: dt and lam are staged by TMA (ragged tails included)
    (2, 333, 8, 64, 128, 2), (1, 200, 16, 64, 64, 4), (1, 129, 8, 64, 128, 1), (1, 31, 8, 64, 128, 4),
])
def test_bf16_shapes(shape):
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=200 + L)
    y, fin = gpu_scan(inp)
    yr, fr = oracle_scan(inp)
    e = rel_err(y.float().cpu().double().numpy(), yr)
    assert e < TOL[torch.bfloat16], e
    check_state(fin, fr, TOL[torch.bfloat16])


@pytest.mark.parametrize("shape", [(2, 200, 148, 64, 128, 2), (5, 200, 40, 64, 128, 2), (2, 300, 100, 64, 128, 1),
                                   # y written through the epilogue warps' TMA stores (N = 64; N = 128 with R = 4)
                                   (2, 300, 100, 64, 128, 4), (3, 250, 64, 64, 64, 1)])
def test_repeated_launches_are_identical_and_match(shape):
    """Many units in flight, launched repeatedly: every launch must match the
    oracle and reproduce the first launch bit for bit (a race between a shared
    tile's refill and its last readers shows up as a rare per-launch error)."""
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=1000 + L)
    yr, fr = oracle_scan(inp)
    first = None
    for rep in range(8):
        y, fin = gpu_scan(inp)
        if first is None:
            e = rel_err(y.float().cpu().double().numpy(), yr)
            assert e < TOL[torch.bfloat16], e
            check_state(fin, fr, TOL[torch.bfloat16])
            first = (y.clone(), fin.h.clone(), fin.angle.clone())
        else:
            assert torch.equal(y, first[0]), f"launch {rep}: y differs from the first launch"
            assert torch.equal(fin.h, first[1]), f"launch {rep}: h differs from the first launch"
            assert torch.equal(fin.angle, first[2]), f"launch {rep}: angle differs from the first launch"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_init_state_and_in_place_continuation(dtype):
    """Split prefill with the exported state == one prefill; final_state may alias init."""
    b, L, H, P, N, R, k = 2, 300, 2, 64, 128, 1, 131
    inp = small_inputs(b, L, H, P, N, R, dtype, seed=300)
    first = {n: inp[n][:, :k].contiguous() for n in NAMES}
    second = {n: inp[n][:, k:].contiguous() for n in NAMES}
    for d in (first, second):
        d["A"], d["D"] = inp["A"], inp["D"]
    _, st = gpu_scan(first)
    y2 = m3.mamba3_scan_fwd(*(second[n] for n in NAMES), inp["A"], inp["D"], init=st, final_state=st)
    torch.cuda.synchronize()
    yr, fr = oracle_scan(inp)
    assert rel_err(y2.float().cpu().double().numpy(), yr[:, k:]) < TOL[dtype]
    check_state(st, fr, TOL[dtype])


@pytest.mark.parametrize("shape", [(2, 150, 100, 64, 64, 2), (3, 97, 64, 64, 128, 1)])
def test_random_init_state_many_units_bf16(shape):
    """More (batch, head) units than SMs, each starting from its own random
    state: every CTA initialises the carried state and angle per unit."""
    b, L, H, P, N, R = shape
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=320 + L)
    g = torch.Generator().manual_seed(7)
    st = m3.State(*(torch.randn(*s, generator=g).cuda() for s in
                    ((b, H, N, P), (b, H, R, N), (b, H, R, P))), torch.rand(b, H, N // 2, generator=g).cuda() * 6 - 3)
    ref_init = to_state_np(st)
    y, fin = gpu_scan(inp, init=st)
    yr, fr = oracle_scan(inp, init=ref_init)
    e = rel_err(y.float().cpu().double().numpy(), yr)
    assert e < TOL[torch.bfloat16], e
    check_state(fin, fr, TOL[torch.bfloat16])


def test_random_init_state_fp32():
    b, L, H, P, N, R = 1, 100, 2, 16, 16, 2
    inp = small_inputs(b, L, H, P, N, R, torch.float32, seed=310)
    g = torch.Generator().manual_seed(5)
    st = m3.State(*(torch.randn(*s, generator=g).cuda() for s in
                    ((b, H, N, P), (b, H, R, N), (b, H, R, P))), torch.rand(b, H, N // 2, generator=g).cuda() * 6 - 3)
    ref_init = to_state_np(st)
    y, fin = gpu_scan(inp, init=st)
    yr, fr = oracle_scan(inp, init=ref_init)
    assert rel_err(y.cpu().double().numpy(), yr) < 1e-4
    check_state(fin, fr, 1e-4)


@pytest.mark.parametrize("case", ["lam_one", "theta_zero", "A_zero", "no_D"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_special_inputs(case, dtype):
    """The degenerate cases of the method: exponential-Euler (lam = 1), no rotation
    (theta = 0), no decay (A = 0), no skip term (D = None)."""
    inp = small_inputs(1, 190, 2, 64, 64, 1, dtype, seed=400)
    if case == "lam_one":
        inp["lam"] = torch.ones_like(inp["lam"])
    elif case == "theta_zero":
        inp["theta"] = torch.zeros_like(inp["theta"])
    elif case == "A_zero":
        inp["A"] = torch.zeros_like(inp["A"])
    D = None if case == "no_D" else inp["D"]
    fin = m3.State.zeros(1, 2, 64, 64, 1)
    y = m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], D, final_state=fin)
    torch.cuda.synchronize()
    f = wl.to_f64({k: inp[k] for k in (*NAMES, "A")})
    yr, fr = oracle.scan_complex(**f, D=None if D is None else wl.to_f64({"D": D})["D"])
    assert rel_err(y.float().cpu().double().numpy(), yr) < TOL[dtype]
    check_state(fin, fr, TOL[dtype])


def test_empty_sequence_passes_state_through():
    b, H, P, N, R = 1, 2, 16, 16, 1
    x = torch.zeros(b, 0, H, R, P, device="cuda")
    B = torch.zeros(b, 0, H, R, N, device="cuda")
    th = torch.zeros(b, 0, H, N // 2, device="cuda")
    dt = torch.zeros(b, 0, H, device="cuda")
    A = torch.full((H,), -1.0, device="cuda")
    init = m3.State(*(torch.randn(*s, device="cuda") for s in ((b, H, N, P), (b, H, R, N), (b, H, R, P), (b, H, N // 2))))
    fin = m3.State.zeros(b, H, P, N, R)
    m3.mamba3_scan_fwd(x, B, B, th, dt, dt, A, init=init, final_state=fin)
    torch.cuda.synchronize()
    for a, c in zip((fin.h, fin.b_prev, fin.x_prev, fin.angle), (init.h, init.b_prev, init.x_prev, init.angle)):
        assert torch.equal(a, c)


def test_guard_bands_untouched():
    """Outputs written exactly in bounds: sentinels around y and the state survive."""
    b, L, H, P, N, R = 1, 77, 2, 64, 128, 1
    inp = small_inputs(b, L, H, P, N, R, torch.bfloat16, seed=500)
    pad = 4096
    ybuf = torch.full((pad + inp["x"].numel() + pad,), 12345.0, dtype=torch.bfloat16, device="cuda")
    y = ybuf[pad:pad + inp["x"].numel()].view_as(inp["x"])
    hbuf = torch.full((pad + b * H * N * P + pad,), -777.0, device="cuda")
    fin = m3.State(hbuf[pad:pad + b * H * N * P].view(b, H, N, P), torch.zeros(b, H, R, N, device="cuda"),
                   torch.zeros(b, H, R, P, device="cuda"), torch.zeros(b, H, N // 2, device="cuda"))
    m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], y=y, final_state=fin)
    torch.cuda.synchronize()
    assert torch.all(ybuf[:pad] == 12345.0) and torch.all(ybuf[-pad:] == 12345.0)
    assert torch.all(hbuf[:pad] == -777.0) and torch.all(hbuf[-pad:] == -777.0)
    yr, _ = oracle_scan(inp)
    assert rel_err(y.float().cpu().double().numpy(), yr) < 2e-2


def test_device_status_ok_after_scan():
    inp = small_inputs(1, 64, 2, 64, 128, 1, torch.bfloat16, seed=600)
    dims = m3.make_dims(inp["x"], inp["B"])
    ws = torch.empty(m3.mamba3_scan_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], workspace=ws)
    assert m3.mamba3_device_status(ws) == m3.MAMBA3_OK


# ---------------------------------------------------------------- decode
@pytest.mark.parametrize("R", [1, 2, 4])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_steps_match_oracle(R, dtype):
    """Prefill (GPU) then decode steps (GPU) == the oracle's one longer prefill."""
    b, H, P, N, L0, S = 3, 2, 64, 128, 70, 9
    inp = small_inputs(b, L0 + S, H, P, N, R, dtype, seed=700 + R)
    pre = {n: inp[n][:, :L0].contiguous() for n in NAMES}
    pre["A"], pre["D"] = inp["A"], inp["D"]
    _, st = gpu_scan(pre)
    ys = []
    for t in range(L0, L0 + S):
        ys.append(m3.mamba3_decode_step(st, *(inp[n][:, t].contiguous() for n in NAMES), inp["A"], inp["D"]))
    torch.cuda.synchronize()
    yr, fr = oracle_scan(inp)
    yg = torch.stack(ys, 1).float().cpu().double().numpy()
    assert rel_err(yg, yr[:, L0:]) < TOL[dtype]
    check_state(st, fr, TOL[dtype])


@pytest.mark.parametrize("R", [1, 4])
def test_decode_single_step_vs_oracle_step(R):
    """One step from a random state against the oracle's decode step (fp32: 1e-4)."""
    b, H, P, N = 4, 3, 64, 128
    g = torch.Generator().manual_seed(17 + R)
    st = m3.State(torch.randn(b, H, N, P, generator=g).cuda(), torch.randn(b, H, R, N, generator=g).cuda(),
                  torch.randn(b, H, R, P, generator=g).cuda(), (torch.rand(b, H, N // 2, generator=g) * 6 - 3).cuda())
    ref0 = to_state_np(st)
    tok = small_inputs(b, 1, H, P, N, R, torch.float32, seed=800 + R)
    step = {n: tok[n][:, 0].contiguous() for n in NAMES}
    y = m3.mamba3_decode_step(st, *(step[n] for n in NAMES), tok["A"], tok["D"])
    torch.cuda.synchronize()
    f = wl.to_f64({**step, "A": tok["A"], "D": tok["D"]})
    yr, fr = oracle.decode_step(ref0, *(f[n] for n in NAMES), f["A"], f["D"])
    assert rel_err(y.cpu().double().numpy(), yr) < 1e-4
    check_state(st, fr, 1e-4)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_chunk_size_invariance(dtype):
    """The chunk length is a blocking choice only: chunks of 1, 8, 32, 64 tokens (SIMT path)
    and the tensor-core default (128 rows) all match the oracle."""
    b, L, H, P, N, R = 1, 300, 2, 64, 128, 1
    inp = small_inputs(b, L, H, P, N, R, dtype, seed=900)
    yr, fr = oracle_scan(inp)
    for chunk in (1, 8, 32, 64, 0):
        y, fin = gpu_scan(inp, chunk=chunk)
        assert rel_err(y.float().cpu().double().numpy(), yr) < TOL[dtype], chunk
        check_state(fin, fr, TOL[dtype])
