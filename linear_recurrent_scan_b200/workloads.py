"""Seeded synthetic inputs for the Mamba-3 recurrence.

This module only draws random numbers with the distributions of the layer's
inputs; it contains none of the recurrence's arithmetic.  Both the CUDA path
(tests, bench) and the fp64 oracle read the tensors it returns, so the two
sides always see the same (already rounded) values.

Distributions (the pages run trained 1.5B-class models on FineWeb-Edu; no
weights or data exist here, so these synthetic draws stand in for the
projections that feed the layer):

* x ~ N(0, 1)
* B, C ~ N(0, 1), RMS-normalised over N per (b, t, h, r) (eps 1e-6, unit
  weight; the "BC norm" of the Mamba-3 block) plus a head-specific
  channel-wise bias [H, R, N] ~ N(0, 0.1^2); grouped B, C (shared by several
  heads) the same without the bias
* dt = clamp(softplus(z + b_h), 1e-3, 0.1), z ~ N(0, 1), with
  b_h = softplus^-1(dt0_h) and dt0_h log-uniform in [1e-3, 0.1]
* A_h = -exp(U(0, log 16))  (one real scalar per head, in [-16, -1])
* lam = sigmoid(N(0, 1))
* theta ~ U(0, pi), one angle per (token, head, B/C pair)
* D ~ N(0, 1)

Sources: "Mamba-3: 2x smaller state ..." (MarkTechPost, Korean translation)
section 2 (RMS normalisation of B and C, head-specific B/C bias) and the
workload table of the benchmark configurations (sizes below).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int  # P
    dstate: int  # N
    rank: int  # R
    dtype: torch.dtype  # dtype of the per-token inputs and of y
    chunk: int = 0  # 0 = library default
    decode_steps: int = 0
    prefill_tokens: int = 0  # decode workloads: prompt length that seeds the state

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def token_heads(self) -> int:
        return self.batch * self.seqlen * self.nheads


# The five benchmark configurations (sizes as in the benchmark table).
CONFIGS: Dict[str, Workload] = {
    "tiny_siso_fp32": Workload("tiny_siso_fp32", 1, 256, 2, 16, 16, 1, torch.float32, chunk=64),
    "siso_prefill_b8_l2048": Workload("siso_prefill_b8_l2048", 8, 2048, 64, 64, 128, 1, torch.bfloat16),
    "mimo4_prefill_b4_l8192": Workload("mimo4_prefill_b4_l8192", 4, 8192, 64, 64, 128, 4, torch.bfloat16),
    "siso_decode_b128": Workload("siso_decode_b128", 128, 1, 64, 64, 128, 1, torch.bfloat16,
                                 decode_steps=1024, prefill_tokens=512),
    "mimo4_decode_b128": Workload("mimo4_decode_b128", 128, 1, 64, 64, 128, 4, torch.bfloat16,
                                  decode_steps=1024, prefill_tokens=512),
    "mimo4_long_b1_l65536": Workload("mimo4_long_b1_l65536", 1, 65536, 64, 64, 64, 4, torch.bfloat16,
                                     decode_steps=1024),
}

BASE_SEED = 20260316


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _rand(shape, g, device):
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32)


def head_params(nheads: int, rank: int, dstate: int, seed: int, device="cpu") -> Dict[str, torch.Tensor]:
    """Per-head parameters: A [H], D [H] (fp32), dt bias [H], B/C bias [H,R,N]."""
    g = _gen(device, seed * 7 + 1)
    A = -torch.exp(_rand((nheads,), g, device) * math.log(16.0))
    D = _randn((nheads,), g, device)
    lo, hi = math.log(1e-3), math.log(0.1)
    dt0 = torch.exp(lo + (hi - lo) * _rand((nheads,), g, device))
    dt_bias = dt0 + torch.log(-torch.expm1(-dt0))  # softplus^-1(dt0)
    b_bias = 0.1 * _randn((nheads, rank, dstate), g, device)
    c_bias = 0.1 * _randn((nheads, rank, dstate), g, device)
    return {"A": A, "D": D, "dt_bias": dt_bias, "b_bias": b_bias, "c_bias": c_bias}


def _bc(shape, bias, g, device, eps=1e-6):
    v = _randn(shape, g, device)
    v = v * torch.rsqrt(v.pow(2).mean(dim=-1, keepdim=True) + eps)
    return v + bias


def token_inputs(batch: int, seqlen: int, nheads: int, headdim: int, dstate: int, rank: int,
                 dtype: torch.dtype, seed: int, device="cpu",
                 params: Optional[Dict[str, torch.Tensor]] = None) -> Dict[str, torch.Tensor]:
    """Per-token inputs x, B, C, theta, dt, lam (rounded to ``dtype``).

    Shapes: x [b,L,H,R,P], B/C [b,L,H,R,N], theta [b,L,H,N/2], dt/lam [b,L,H].
    """
    if params is None:
        params = head_params(nheads, rank, dstate, seed, device)
    g = _gen(device, seed)
    b, L, H, R, P, N = batch, seqlen, nheads, rank, headdim, dstate
    out = {}
    out["x"] = _randn((b, L, H, R, P), g, device).to(dtype)
    out["B"] = _bc((b, L, H, R, N), params["b_bias"].to(device), g, device).to(dtype)
    out["C"] = _bc((b, L, H, R, N), params["c_bias"].to(device), g, device).to(dtype)
    out["theta"] = (math.pi * _rand((b, L, H, N // 2), g, device)).to(dtype)
    z = _randn((b, L, H), g, device)
    out["dt"] = torch.nn.functional.softplus(z + params["dt_bias"].to(device)).clamp(1e-3, 0.1).to(dtype)
    out["lam"] = torch.sigmoid(_randn((b, L, H), g, device)).to(dtype)
    return out


def make_inputs(w: Workload, seed: int = BASE_SEED, device="cpu", seqlen: Optional[int] = None,
                batch: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """All inputs of one workload: per-token tensors plus A, D (fp32, [H])."""
    params = head_params(w.nheads, w.rank, w.dstate, seed, device)
    d = token_inputs(batch or w.batch, seqlen if seqlen is not None else w.seqlen, w.nheads, w.headdim,
                     w.dstate, w.rank, w.dtype, seed, device, params)
    d["A"] = params["A"].float().contiguous()
    d["D"] = params["D"].float().contiguous()
    return d


def decode_inputs(w: Workload, steps: int, seed: int = BASE_SEED + 1, device="cpu") -> Dict[str, torch.Tensor]:
    """Per-step decode inputs with a leading step axis: x [S,b,H,R,P], ...

    Drawn as one sequence of ``steps`` tokens and moved to step-major layout so
    that each step's slice is contiguous.
    """
    d = token_inputs(w.batch, steps, w.nheads, w.headdim, w.dstate, w.rank, w.dtype, seed, device,
                     head_params(w.nheads, w.rank, w.dstate, BASE_SEED, device))
    return {k: v.transpose(0, 1).contiguous() for k, v in d.items()}


def raw_bc_inputs(inp: Dict[str, torch.Tensor], seed: int = BASE_SEED + 2) -> Dict[str, torch.Tensor]:
    """Raw (not yet normalised) B and C projections with the shapes, dtype and
    device of inp["B"], inp["C"]: N(0, 1) rows times a per-row scale drawn
    log-uniform in [0.1, 10]; and the B/C norm parameters of the heads, float32
    [H, R, N]: weights U(0.5, 1.5), biases N(0, 0.1^2)."""
    B = inp["B"]
    dev = B.device
    *lead, H, R, N = B.shape
    g = _gen(dev, seed)
    out = {}
    for name in ("B_raw", "C_raw"):
        z = torch.randn(B.shape, generator=g, device=dev, dtype=torch.float32)
        scale = torch.exp(torch.empty(*lead, H, R, 1, device=dev).uniform_(math.log(0.1), math.log(10.0), generator=g))
        out[name] = (z * scale).to(B.dtype).contiguous()
    for name in ("w_B", "w_C"):
        out[name] = torch.empty(H, R, N, device=dev).uniform_(0.5, 1.5, generator=g)
    for name in ("bias_B", "bias_C"):
        out[name] = torch.randn(H, R, N, generator=g, device=dev) * 0.1
    return out


def grouped_bc(inp: Dict[str, torch.Tensor], ngroups: int, seed: int = BASE_SEED + 5) -> Dict[str, torch.Tensor]:
    """B and C shared by ``ngroups`` groups of heads: [..., G, R, N] in place of
    inp["B"], inp["C"] [..., H, R, N] (dtype and device kept), drawn like the
    per-head rows but without the head-specific bias, which a row shared by
    several heads cannot carry."""
    B = inp["B"]
    *lead, H, R, N = B.shape
    assert H % ngroups == 0
    g = _gen(B.device, seed)
    shape = (*lead, ngroups, R, N)
    return {name: _bc(shape, 0.0, g, B.device).to(B.dtype).contiguous() for name in ("B", "C")}


def decay_rates(like: torch.Tensor, seed: int = BASE_SEED + 4) -> torch.Tensor:
    """A time-varying decay rate per token and head, shaped, typed and placed like
    `like` (dt): A_t = -exp(U(log 0.5, log 16))."""
    g = _gen(like.device, seed)
    u = torch.empty(like.shape, device=like.device).uniform_(math.log(0.5), math.log(16.0), generator=g)
    return (-torch.exp(u)).to(like.dtype).contiguous()


def to_f64(d: Dict[str, torch.Tensor]):
    """Widen every tensor to a float64 numpy array (exact for bf16/fp32)."""
    return {k: v.detach().to("cpu", torch.float64).numpy() for k, v in d.items()}
