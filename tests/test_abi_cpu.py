"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any CUDA call.

Every call below either fails host validation (so nothing is ever enqueued,
even on a machine with a GPU) or is skipped when a CUDA device is present.
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import linear_recurrent_scan_b200 as m3
from linear_recurrent_scan_b200 import build as m3build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    m3build.build()
    return m3.load_library()


def declared_symbols():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"MAMBA3_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_entry_points():
    names = declared_symbols()
    for n in ("mamba3_scan_fwd", "mamba3_decode_step", "mamba3_scan_workspace_bytes",
              "mamba3_device_status", "mamba3_status_string", "mamba3_version"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", m3.LIB_PATH]).decode()
    exported = set(re.findall(r"\sT\s(\w+)$", out, re.M))
    missing = [n for n in declared_symbols() if n not in exported]
    assert not missing, missing
    for n in declared_symbols():
        assert hasattr(lib, n)


def test_no_driver_or_oracle_dependency(lib):
    """The library links CUDA's runtime statically and never the oracle."""
    out = subprocess.check_output(["ldd", m3.LIB_PATH]).decode()
    assert "libcuda.so" not in out and "oracle" not in out


def test_status_strings(lib):
    assert m3.mamba3_status_string(0) == "ok"
    for c in (-1, -2, -3, -4, -5):
        assert m3.mamba3_status_string(c) != "unknown status"
    assert m3.mamba3_status_string(17) == "unknown status"
    assert lib.mamba3_version() // 100 == m3.ABI_MAJOR == 2


def dims(**kw):
    d = dict(batch=2, seqlen=64, nheads=3, headdim=16, dstate=16, rank=1, chunk=0, in_dtype=m3.MAMBA3_BF16)
    d.update(kw)
    return m3.Dims(**d)


@pytest.mark.parametrize("bad", [
    dict(batch=0), dict(nheads=0), dict(headdim=6), dict(headdim=0), dict(dstate=15), dict(dstate=0),
    dict(rank=3), dict(rank=0), dict(in_dtype=7), dict(seqlen=-1), dict(chunk=-2),
    dict(ngroups=-1), dict(ngroups=2), dict(ngroups=6),
])
def test_workspace_bytes_rejects_bad_dims(lib, bad):
    assert lib.mamba3_scan_workspace_bytes(ctypes.byref(dims(**bad))) == 0


def test_workspace_bytes_valid(lib):
    assert lib.mamba3_scan_workspace_bytes(ctypes.byref(dims())) >= 256
    assert lib.mamba3_scan_workspace_bytes(None) == 0


FAKE = 0x10000  # never dereferenced: every call using it fails validation first


def scan(lib, d, ptrs=None, init=None, final=None, ws=FAKE, ws_bytes=1 << 20):
    p = dict(x=FAKE, B=FAKE, C=FAKE, theta=FAKE, dt=FAKE, lam=FAKE, A=FAKE, D=None, y=FAKE)
    p.update(ptrs or {})
    return lib.mamba3_scan_fwd(ctypes.byref(d) if d is not None else None, p["x"], p["B"], p["C"], p["theta"],
                               p["dt"], p["lam"], p["A"], p["D"], init, p["y"], final, ws, ws_bytes, None)


@pytest.mark.parametrize("name", ["x", "B", "C", "theta", "dt", "lam", "A", "y"])
def test_scan_rejects_null_pointer(lib, name):
    assert scan(lib, dims(), {name: None}) == m3.MAMBA3_ERR_INVALID


@pytest.mark.parametrize("name", ["x", "B", "C", "theta", "y"])
def test_scan_rejects_misaligned_pointer(lib, name):
    assert scan(lib, dims(), {name: FAKE + 8}) == m3.MAMBA3_ERR_INVALID


def test_scan_rejects_bad_dims_and_state(lib):
    assert scan(lib, None) == m3.MAMBA3_ERR_INVALID
    assert scan(lib, dims(rank=5)) == m3.MAMBA3_ERR_INVALID
    half = m3._CState(FAKE, None, FAKE, FAKE)
    assert scan(lib, dims(), init=ctypes.byref(half)) == m3.MAMBA3_ERR_INVALID
    assert scan(lib, dims(), final=ctypes.byref(half)) == m3.MAMBA3_ERR_INVALID
    mis = m3._CState(FAKE + 4, FAKE, FAKE, FAKE)
    assert scan(lib, dims(), init=ctypes.byref(mis)) == m3.MAMBA3_ERR_INVALID


def test_scan_rejects_workspace(lib):
    assert scan(lib, dims(), ws=None) == m3.MAMBA3_ERR_WORKSPACE
    assert scan(lib, dims(), ws_bytes=16) == m3.MAMBA3_ERR_WORKSPACE
    assert scan(lib, dims(), ws=FAKE + 4) == m3.MAMBA3_ERR_WORKSPACE


def test_scan_rejects_unsupported_shape(lib):
    # a chunk whose rows do not fit the SIMT kernel and no tensor-core shape
    assert scan(lib, dims(chunk=4096, in_dtype=m3.MAMBA3_F32)) == m3.MAMBA3_ERR_UNSUPPORTED
    assert scan(lib, dims(dstate=4096)) == m3.MAMBA3_ERR_UNSUPPORTED


def decode(lib, d, st=True, ptrs=None):
    p = dict(x=FAKE, B=FAKE, C=FAKE, theta=FAKE, dt=FAKE, lam=FAKE, A=FAKE, D=None, y=FAKE)
    p.update(ptrs or {})
    cs = m3._CState(FAKE, FAKE, FAKE, FAKE) if st else None
    return lib.mamba3_decode_step(ctypes.byref(d), ctypes.byref(cs) if cs is not None else None, p["x"], p["B"],
                                  p["C"], p["theta"], p["dt"], p["lam"], p["A"], p["D"], p["y"], None)


def test_decode_rejects(lib):
    assert decode(lib, dims(), st=False) == m3.MAMBA3_ERR_INVALID
    assert decode(lib, dims(), ptrs={"x": None}) == m3.MAMBA3_ERR_INVALID
    assert decode(lib, dims(), ptrs={"B": FAKE + 2}) == m3.MAMBA3_ERR_INVALID
    assert decode(lib, dims(headdim=12)) == m3.MAMBA3_ERR_UNSUPPORTED  # 128 % (P/4) != 0
    assert decode(lib, dims(headdim=64, dstate=512)) == m3.MAMBA3_ERR_UNSUPPORTED


def test_device_status_null(lib):
    assert lib.mamba3_device_status(None, None) == m3.MAMBA3_ERR_INVALID


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_is_a_cuda_error(lib):
    """No CPU fallback: with valid host arguments and no GPU the call fails in CUDA."""
    assert scan(lib, dims()) == m3.MAMBA3_ERR_CUDA
    assert decode(lib, dims()) == m3.MAMBA3_ERR_CUDA


def test_python_binding_validates_shapes(lib):
    x = torch.zeros(1, 4, 2, 1, 8, dtype=torch.bfloat16)
    B = torch.zeros(1, 4, 2, 1, 16, dtype=torch.bfloat16)
    th = torch.zeros(1, 4, 2, 7, dtype=torch.bfloat16)  # wrong: N/2 = 8
    dt = torch.zeros(1, 4, 2, dtype=torch.bfloat16)
    A = torch.zeros(2)
    with pytest.raises(ValueError):
        m3.mamba3_scan_fwd(x, B, B, th, dt, dt, A)


def scan_bcn(lib, d, norm, ptrs=None):
    p = dict(x=FAKE, B=FAKE, C=FAKE, theta=FAKE, dt=FAKE, lam=FAKE, A=FAKE, D=None, y=FAKE)
    p.update(ptrs or {})
    return lib.mamba3_scan_fwd_bcnorm(ctypes.byref(d), p["x"], p["B"], p["C"], p["theta"], p["dt"], p["lam"],
                                      p["A"], p["D"], ctypes.byref(norm) if norm is not None else None, None, p["y"],
                                      None, FAKE, 1 << 20, None)


def decode_bcn(lib, d, norm):
    cs = m3._CState(FAKE, FAKE, FAKE, FAKE)
    return lib.mamba3_decode_step_bcnorm(ctypes.byref(d), ctypes.byref(cs), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                         FAKE, None, ctypes.byref(norm) if norm is not None else None, FAKE, None)


def test_bcnorm_entry_points_validate_on_host(lib):
    ok = m3._CNorm(None, None, None, None, 1e-6)
    assert scan_bcn(lib, dims(), None) == m3.MAMBA3_ERR_INVALID                         # norm is required
    assert scan_bcn(lib, dims(), m3._CNorm(None, None, None, None, -1.0)) == m3.MAMBA3_ERR_INVALID
    assert scan_bcn(lib, dims(), m3._CNorm(FAKE + 2, None, None, None, 1e-6)) == m3.MAMBA3_ERR_INVALID
    assert scan_bcn(lib, dims(), ok, {"B": None}) == m3.MAMBA3_ERR_INVALID
    # the fused form runs on the tensor-core path only (bf16, P = 64, N in {64, 128})
    assert scan_bcn(lib, dims(in_dtype=m3.MAMBA3_F32), ok) == m3.MAMBA3_ERR_UNSUPPORTED
    assert decode_bcn(lib, dims(), None) == m3.MAMBA3_ERR_INVALID
    assert scan_bcn(lib, dims(ngroups=2), ok) == m3.MAMBA3_ERR_INVALID                 # 2 groups, 3 heads
    assert decode_bcn(lib, dims(ngroups=2), ok) == m3.MAMBA3_ERR_INVALID
    assert decode_bcn(lib, dims(headdim=32), ok) == m3.MAMBA3_ERR_UNSUPPORTED            # streaming kernel: P = 64


def test_time_varying_decay_entry_points_validate_on_host(lib):
    p = dict(x=FAKE, B=FAKE, C=FAKE, theta=FAKE, dt=FAKE, lam=FAKE, y=FAKE)
    rc = lib.mamba3_scan_fwd_at(ctypes.byref(dims()), p["x"], p["B"], p["C"], p["theta"], p["dt"], p["lam"], None,
                                None, None, p["y"], None, FAKE, 1 << 20, None)
    assert rc == m3.MAMBA3_ERR_INVALID                                   # A_t is required
    rc = lib.mamba3_scan_fwd_at(ctypes.byref(dims()), p["x"], p["B"], p["C"], p["theta"], p["dt"], p["lam"], FAKE + 2,
                                None, None, p["y"], None, FAKE, 1 << 20, None)
    assert rc == m3.MAMBA3_ERR_INVALID                                   # misaligned A_t
    cs = m3._CState(FAKE, FAKE, FAKE, FAKE)
    rc = lib.mamba3_decode_step_at(ctypes.byref(dims()), ctypes.byref(cs), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                   None, FAKE, None)
    assert rc == m3.MAMBA3_ERR_INVALID


def test_grouped_bc_dims_rejected(lib):
    """ngroups must be 0 (one B/C row per head) or a divisor of nheads."""
    for g in (0, 1, 3):
        assert lib.mamba3_scan_workspace_bytes(ctypes.byref(dims(ngroups=g))) >= 256
    assert scan(lib, dims(ngroups=2)) == m3.MAMBA3_ERR_INVALID
    assert decode(lib, dims(ngroups=2)) == m3.MAMBA3_ERR_INVALID


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_grouped_bc_dims_accepted(lib):
    """The valid group counts pass the host checks and, with no GPU, fail in CUDA."""
    for g in (0, 1, 3):
        assert scan(lib, dims(ngroups=g)) == m3.MAMBA3_ERR_CUDA
        assert decode(lib, dims(ngroups=g)) == m3.MAMBA3_ERR_CUDA


def test_python_binding_infers_groups(lib):
    x = torch.zeros(1, 4, 6, 1, 8, dtype=torch.bfloat16)
    th = torch.zeros(1, 4, 6, 8, dtype=torch.bfloat16)
    dt = torch.zeros(1, 4, 6, dtype=torch.bfloat16)
    for G in (1, 2, 3, 6):
        B = torch.zeros(1, 4, G, 1, 16, dtype=torch.bfloat16)
        assert m3.make_dims(x, B).ngroups == G
    with pytest.raises(ValueError):  # 4 groups do not divide 6 heads
        m3.mamba3_scan_fwd(x, *(2 * [torch.zeros(1, 4, 4, 1, 16, dtype=torch.bfloat16)]), th, dt, dt,
                           torch.zeros(6))
    with pytest.raises(ValueError):  # grouped B with a per-head C
        m3.mamba3_scan_fwd(x, torch.zeros(1, 4, 2, 1, 16, dtype=torch.bfloat16),
                           torch.zeros(1, 4, 6, 1, 16, dtype=torch.bfloat16), th, dt, dt, torch.zeros(6))


def bwd(lib, d, ptrs=None, ws=FAKE, ws_bytes=1 << 40):
    p = dict(x=FAKE, B=FAKE, C=FAKE, theta=FAKE, dt=FAKE, lam=FAKE, A=FAKE, D=None, dy=FAKE, dx=FAKE, dB=FAKE,
             dC=FAKE, dtheta=FAKE, ddt=FAKE, dlam=FAKE, dA=FAKE, dD=None)
    p.update(ptrs or {})
    return lib.mamba3_scan_bwd(ctypes.byref(d), p["x"], p["B"], p["C"], p["theta"], p["dt"], p["lam"], p["A"],
                               p["D"], None, p["dy"], None, p["dx"], p["dB"], p["dC"], p["dtheta"], p["ddt"],
                               p["dlam"], p["dA"], p["dD"], None, ws, ws_bytes, None)


@pytest.mark.parametrize("name", ["x", "B", "dy", "dx", "dB", "dC", "dtheta", "ddt", "dlam", "dA", "A"])
def test_backward_rejects_null_pointer(lib, name):
    assert bwd(lib, dims(), {name: None}) == m3.MAMBA3_ERR_INVALID


def test_backward_host_validation(lib):
    d = dims()
    need = lib.mamba3_scan_bwd_workspace_bytes(ctypes.byref(d))
    # 2 x 3 units, 64 tokens in chunks of 32: the state (16 x 16) and angle (8) at each chunk start
    assert need == 256 + 2 * 3 * 2 * (16 * 16 + 8) * 4
    assert bwd(lib, d, ws_bytes=need - 1) == m3.MAMBA3_ERR_WORKSPACE
    assert bwd(lib, d, ws=FAKE + 8) == m3.MAMBA3_ERR_WORKSPACE
    assert bwd(lib, d, {"dB": FAKE + 4}) == m3.MAMBA3_ERR_INVALID
    # grouped B/C: the groups' fp32 sums of dB, dC (2 x b L G R N, here G = 1) come on top of the checkpoints
    dg = dims(ngroups=1)
    assert lib.mamba3_scan_bwd_workspace_bytes(ctypes.byref(dg)) == need + 2 * 2 * 64 * 1 * 1 * 16 * 4
    assert bwd(lib, dg, ws_bytes=need) == m3.MAMBA3_ERR_WORKSPACE
    assert bwd(lib, dims(dstate=256, headdim=128)) == m3.MAMBA3_ERR_UNSUPPORTED  # tiles beyond shared memory
    assert lib.mamba3_scan_bwd_workspace_bytes(ctypes.byref(dims(rank=3))) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_backward_valid_call_without_device_is_a_cuda_error(lib):
    assert bwd(lib, dims()) == m3.MAMBA3_ERR_CUDA
    assert bwd(lib, dims(ngroups=1)) == m3.MAMBA3_ERR_CUDA  # grouped B/C


def gnorm(lib, d, groups, y=FAKE, z=FAKE, w=None, eps=1e-6, out=FAKE):
    return lib.mamba3_gated_norm(ctypes.byref(d), groups, y, z, w, eps, out, None)


def test_gated_norm_host_validation(lib):
    d = dims(nheads=4)
    assert gnorm(lib, d, 3) == m3.MAMBA3_ERR_INVALID          # 3 groups, 4 heads
    assert gnorm(lib, d, 0) == m3.MAMBA3_ERR_INVALID
    assert gnorm(lib, d, 2, eps=-1.0) == m3.MAMBA3_ERR_INVALID
    assert gnorm(lib, d, 2, y=None) == m3.MAMBA3_ERR_INVALID
    assert gnorm(lib, d, 2, out=FAKE + 8) == m3.MAMBA3_ERR_INVALID
    assert gnorm(lib, d, 2, w=FAKE + 4) == m3.MAMBA3_ERR_INVALID  # w: 16-byte aligned
    assert gnorm(lib, dims(nheads=4, seqlen=0), 2, y=None, z=None, out=None) == m3.MAMBA3_OK  # nothing to do


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_gated_norm_valid_call_without_device_is_a_cuda_error(lib):
    assert gnorm(lib, dims(nheads=4), 2) == m3.MAMBA3_ERR_CUDA


def bwd_at(lib, d, ptrs=None):
    p = dict(A_t=FAKE, dA_t=FAKE)
    p.update(ptrs or {})
    return lib.mamba3_scan_bwd_at(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, p["A_t"], None, None, FAKE,
                                  None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, p["dA_t"], None, None, FAKE, 1 << 40, None)


def test_backward_time_varying_decay_host_validation(lib):
    assert bwd_at(lib, dims(), {"A_t": None}) == m3.MAMBA3_ERR_INVALID
    assert bwd_at(lib, dims(), {"dA_t": None}) == m3.MAMBA3_ERR_INVALID
    assert bwd_at(lib, dims(), {"A_t": FAKE + 2}) == m3.MAMBA3_ERR_INVALID


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_backward_time_varying_decay_valid_call_without_device(lib):
    assert bwd_at(lib, dims()) == m3.MAMBA3_ERR_CUDA


def proj_up(lib, d, u=FAKE, W=FAKE, x=FAKE):
    return lib.mamba3_mimo_up(ctypes.byref(d), u, W, x, None)


def proj_down(lib, d, y=FAKE, W=FAKE, z=None, w=None, eps=1e-6, out=FAKE):
    return lib.mamba3_mimo_down(ctypes.byref(d), y, W, z, w, eps, out, None)


def test_mimo_projection_host_validation(lib):
    d = dims(rank=4, headdim=64)
    assert proj_up(lib, d, u=None) == m3.MAMBA3_ERR_INVALID
    assert proj_up(lib, d, x=FAKE + 8) == m3.MAMBA3_ERR_INVALID
    assert proj_down(lib, d, W=None) == m3.MAMBA3_ERR_INVALID
    assert proj_down(lib, d, z=FAKE + 8) == m3.MAMBA3_ERR_INVALID
    assert proj_down(lib, d, w=FAKE + 2, z=FAKE) == m3.MAMBA3_ERR_INVALID
    assert proj_down(lib, d, eps=-1.0) == m3.MAMBA3_ERR_INVALID
    assert proj_up(lib, dims(rank=3, headdim=64)) == m3.MAMBA3_ERR_INVALID
    assert proj_up(lib, dims(rank=4, headdim=32)) == m3.MAMBA3_ERR_UNSUPPORTED
    assert proj_up(lib, dims(rank=8, headdim=64)) == m3.MAMBA3_ERR_UNSUPPORTED
    assert proj_down(lib, dims(rank=4, headdim=64, in_dtype=m3.MAMBA3_F32)) == m3.MAMBA3_ERR_UNSUPPORTED
    assert proj_up(lib, dims(rank=4, headdim=64, seqlen=0), u=None, W=None, x=None) == m3.MAMBA3_OK  # nothing to do


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_mimo_projection_valid_call_without_device_is_a_cuda_error(lib):
    assert proj_up(lib, dims(rank=4, headdim=64)) == m3.MAMBA3_ERR_CUDA
    assert proj_down(lib, dims(rank=2, headdim=64), z=FAKE, w=FAKE) == m3.MAMBA3_ERR_CUDA


def host_scan(lib, d, ptrs=None, init=None, final=None, stage=FAKE, stage_bytes=1 << 30):
    p = dict(x=FAKE, B=FAKE, C=FAKE, theta=FAKE, dt=FAKE, lam=FAKE, A=FAKE, D=None, y=FAKE)
    p.update(ptrs or {})
    return lib.mamba3_scan_fwd_host(ctypes.byref(d) if d is not None else None, p["x"], p["B"], p["C"], p["theta"],
                                    p["dt"], p["lam"], p["A"], p["D"], init, p["y"], final, stage, stage_bytes,
                                    None)


def test_host_stage_bytes(lib):
    """The status word, then two slots of one sub-batch (here one batch row of two)
    of x, y, B, C, theta, dt and lam, each 256-byte aligned."""
    es, L, H, R, P, N = 2, 64, 3, 1, 16, 16
    al = lambda v: (v + 255) // 256 * 256
    slot = 2 * al(L * H * R * P * es) + 2 * al(L * H * R * N * es) + al(L * H * (N // 2) * es) + 2 * al(L * H * es)
    assert lib.mamba3_scan_fwd_host_stage_bytes(ctypes.byref(dims())) == 256 + 2 * slot
    # batch 20: 8 sub-batches of 3 rows (the last one 2), slots sized for 3 rows
    slot3 = 2 * al(3 * L * H * R * P * es) + 2 * al(3 * L * H * R * N * es) + al(3 * L * H * (N // 2) * es) + \
        2 * al(3 * L * H * es)
    assert lib.mamba3_scan_fwd_host_stage_bytes(ctypes.byref(dims(batch=20))) == 256 + 2 * slot3
    assert lib.mamba3_scan_fwd_host_stage_bytes(ctypes.byref(dims(batch=0))) == 0


@pytest.mark.parametrize("name", ["x", "B", "C", "theta", "dt", "lam", "A", "y"])
def test_host_scan_rejects_null_pointer(lib, name):
    assert host_scan(lib, dims(), {name: None}) == m3.MAMBA3_ERR_INVALID


def test_host_scan_rejects_stage_and_dims(lib):
    d = dims()
    need = lib.mamba3_scan_fwd_host_stage_bytes(ctypes.byref(d))
    assert host_scan(lib, d, stage_bytes=need - 1) == m3.MAMBA3_ERR_WORKSPACE
    assert host_scan(lib, d, stage=FAKE + 8) == m3.MAMBA3_ERR_WORKSPACE
    assert host_scan(lib, d, stage=None) == m3.MAMBA3_ERR_WORKSPACE
    assert host_scan(lib, dims(rank=3)) == m3.MAMBA3_ERR_INVALID
    assert host_scan(lib, None) == m3.MAMBA3_ERR_INVALID
