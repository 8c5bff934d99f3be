"""Benchmark tool beside bench.py: run a few prefills (or decode steps, backward
passes, output-side norms) of one workload, for profilers.

    python profile_case.py --workload siso_prefill_b8_l2048 --batch 2 --reps 3
    python profile_case.py --workload siso_decode_b128 --decode --reps 3
    python profile_case.py --workload siso_prefill_b8_l2048 --groups 1 --reps 3
    python profile_case.py --workload siso_prefill_b8_l2048 --backward --reps 3
    python profile_case.py --workload siso_prefill_b8_l2048 --gated-norm 64 --reps 3
    python profile_case.py --workload mimo4_prefill_b4_l8192 --mimo-proj --reps 3

Inputs are seeded synthetic tensors on cuda:0.  Prints the CUDA-event time
of each call; under a profiler those times are not benchmark numbers.
"""
from __future__ import annotations

import argparse

import torch

import linear_recurrent_scan_b200 as m3
from linear_recurrent_scan_b200 import workloads as wl

NAMES = ("x", "B", "C", "theta", "dt", "lam")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="siso_prefill_b8_l2048", choices=sorted(wl.CONFIGS))
    ap.add_argument("--batch", type=int, default=0, help="override the batch size (0 = workload's)")
    ap.add_argument("--seqlen", type=int, default=0, help="override the sequence length (0 = workload's)")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--decode", action="store_true", help="time decode steps instead of the prefill")
    ap.add_argument("--groups", type=int, default=0, help="B, C shared by this many groups of heads (0 = per head)")
    ap.add_argument("--backward", action="store_true", help="time the prefill's backward pass")
    ap.add_argument("--gated-norm", type=int, default=0, metavar="G",
                    help="time the output side (grouped RMS norm + gate, G norm groups) on a prefill-sized y")
    ap.add_argument("--mimo-proj", action="store_true",
                    help="time the rank-R up projection and the gated down projection on the workload's tokens")
    args = ap.parse_args()
    w = wl.CONFIGS[args.workload]
    if args.batch:
        w = w.with_(batch=args.batch)
    if args.seqlen:
        w = w.with_(seqlen=args.seqlen)
    dev = torch.device("cuda", 0)
    m3.load_library()
    st = m3.State.zeros(w.batch, w.nheads, w.headdim, w.dstate, w.rank, device=dev)
    if args.decode:
        pre = wl.make_inputs(w.with_(seqlen=max(1, w.prefill_tokens)), device=dev)
        m3.mamba3_scan_fwd(*(pre[n] for n in NAMES), pre["A"], pre["D"], final_state=st)
        steps = wl.decode_inputs(w, args.reps, device=dev)
        if args.groups:
            steps.update(wl.grouped_bc(steps, args.groups))
        for i in range(args.reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            m3.mamba3_decode_step(st, *(steps[n][i] for n in NAMES), pre["A"], pre["D"])
            e1.record()
            torch.cuda.synchronize()
            print(f"decode step {i}: {e0.elapsed_time(e1) * 1000:.1f} us")
        return
    if args.gated_norm:
        g = torch.Generator(device=dev)
        g.manual_seed(wl.BASE_SEED + 10)
        shape = (w.batch, w.seqlen, w.nheads, w.rank, w.headdim)
        y = torch.randn(shape, generator=g, device=dev).to(w.dtype)
        z = torch.randn(shape, generator=g, device=dev).to(w.dtype)
        wt = torch.rand((w.nheads, w.rank, w.headdim), generator=g, device=dev) + 0.5
        out = torch.empty_like(y)
        for i in range(args.reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            m3.mamba3_gated_norm(y, z, wt, groups=args.gated_norm, out=out)
            e1.record()
            torch.cuda.synchronize()
            print(f"gated norm {w.name} groups {args.gated_norm} rep {i}: {e0.elapsed_time(e1) * 1000:.1f} us")
        return
    if args.mimo_proj:
        g = torch.Generator(device=dev)
        g.manual_seed(wl.BASE_SEED + 11)
        P, R, H = w.headdim, w.rank, w.nheads
        u = torch.randn((w.batch, w.seqlen, H, P), generator=g, device=dev).to(w.dtype)
        Wx = (torch.randn((H, R * P, P), generator=g, device=dev) * P ** -0.5).to(w.dtype)
        Wy = (torch.randn((H, P, R * P), generator=g, device=dev) * (R * P) ** -0.5).to(w.dtype)
        z = torch.randn((w.batch, w.seqlen, H, P), generator=g, device=dev).to(w.dtype)
        wn = torch.rand((H, P), generator=g, device=dev) + 0.5
        x = torch.empty((w.batch, w.seqlen, H, R, P), device=dev, dtype=w.dtype)
        o = torch.empty_like(u)
        for i in range(args.reps):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            ev[0].record()
            m3.mamba3_mimo_up(u, Wx, out=x)
            ev[1].record()
            m3.mamba3_mimo_down(x, Wy, z=z, w=wn, out=o)
            ev[2].record()
            torch.cuda.synchronize()
            print(f"mimo up {w.name} rep {i}: {ev[0].elapsed_time(ev[1]):.4f} ms; "
                  f"down (gated) {ev[1].elapsed_time(ev[2]):.4f} ms")
        if m3.mamba3_library_status() != m3.MAMBA3_OK:
            raise RuntimeError("library status after the projections is not OK")
        return
    inp = wl.make_inputs(w, device=dev)
    if args.groups:
        inp.update(wl.grouped_bc(inp, args.groups))
    y = torch.empty_like(inp["x"])
    if args.backward:
        g = torch.Generator(device=dev)
        g.manual_seed(wl.BASE_SEED + 9)
        dy = torch.randn(inp["x"].shape, generator=g, device=dev).to(inp["x"].dtype)
        dims = m3.make_dims(inp["x"], inp["B"])
        ws = torch.empty(m3.mamba3_scan_bwd_workspace_bytes(dims), dtype=torch.uint8, device=dev)
        grads = None
        flush = torch.ones(256 << 20, dtype=torch.uint8, device=dev)  # read before each pass: L2 cold
        for i in range(args.reps):
            flush.sum()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            grads = m3.mamba3_scan_bwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], dy, grads=grads, workspace=ws)
            e1.record()
            torch.cuda.synchronize()
            print(f"backward {w.name} b{w.batch} L{w.seqlen} rep {i}: {e0.elapsed_time(e1):.3f} ms")
        return
    for i in range(args.reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        m3.mamba3_scan_fwd(*(inp[n] for n in NAMES), inp["A"], inp["D"], y=y, final_state=st)
        e1.record()
        torch.cuda.synchronize()
        print(f"prefill {w.name} b{w.batch} L{w.seqlen} rep {i}: {e0.elapsed_time(e1):.3f} ms")


if __name__ == "__main__":
    main()
