"""The bench's algorithmic byte counts (the roofline numerators) against the
per-unit figures they are defined by, and its traffic table's staleness rule.
CPU only: nothing here launches a kernel."""
import bench
from linear_recurrent_scan_b200 import workloads as wl

SISO = wl.CONFIGS["siso_prefill_b8_l2048"]
DEC = wl.CONFIGS["siso_decode_b128"]
MIMO_DEC = wl.CONFIGS["mimo4_decode_b128"]


def test_prefill_bytes_siso():
    # 900 B per token-head (x 128, y 128, B 256, C 256, theta 128, dt 2, lam 2) + the fp32
    # final state per (b, h): 4 (N P + R N + R P + N/2) = 33,792 B + A, D
    assert bench.prefill_bytes(SISO) == 900 * 8 * 2048 * 64 + 33792 * 8 * 64 + 8 * 64
    assert bench.prefill_bytes(SISO, export_state=False) == 900 * 8 * 2048 * 64 + 8 * 64


def test_prefill_bytes_grouped():
    # one B and C row per token instead of one per head: 512 B per token-head become 512 B per token
    per_head_bc = 2 * 2 * 128 * 8 * 2048 * 64
    per_group_bc = 2 * 2 * 128 * 8 * 2048
    assert bench.prefill_bytes(SISO, groups=1) == bench.prefill_bytes(SISO) - per_head_bc + per_group_bc
    assert bench.prefill_bytes(SISO, groups=64) == bench.prefill_bytes(SISO)


def test_decode_bytes():
    # per (b, h): the fp32 state read and written (2 x 33,792 B) + 900 B of token inputs and y
    assert bench.decode_bytes(DEC) == 128 * 64 * 68484 + 8 * 64
    # MIMO R4: state 2 x 4 (8192 + 512 + 256 + 64) = 72,192 B, io 2 (512 + 1024 + 64 + 2) = 3,204 B
    assert bench.decode_bytes(MIMO_DEC) == 128 * 64 * (72192 + 3204) + 8 * 64


def test_backward_bytes():
    # inputs (772 B) and their gradients (772 B) once, dy (128 B) once: 1672 B per token-head
    assert bench.backward_bytes(SISO) == 1672 * 8 * 2048 * 64 + 16 * 64


def test_traffic_is_null_when_sources_change(monkeypatch):
    key = "prefill"
    files, sha, nbytes, cite = bench.TRAFFIC[key]
    monkeypatch.setitem(bench.TRAFFIC, key, (files, "0" * 64, nbytes, cite))
    assert bench.traffic(key) is None
    monkeypatch.setitem(bench.TRAFFIC, key, (files, bench.sources_sha(files), nbytes, cite))
    assert bench.traffic(key) == nbytes


def test_mimo_proj_bytes():
    w = wl.CONFIGS["mimo4_prefill_b4_l8192"]
    th = 4 * 8192 * 64
    wts = 2 * 64 * 4 * 64 * 64
    # up: u (128 B) read, x (512 B) written per token-head; down: y (512 B), z (128 B) read, out (128 B) written
    assert bench.mimo_proj_bytes(w) == {"up": th * 640 + wts, "down_gated": th * 768 + wts + 4 * 64 * 64}
