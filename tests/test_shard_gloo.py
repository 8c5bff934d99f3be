"""Multi-rank host logic on CPU (gloo, world size 2): the batch partition covers every
(batch, head) unit exactly once, per-shard results (fp64 oracle) gathered from the
ranks equal the unsharded result, and timings reduce to the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from linear_recurrent_scan_b200.shard import all_reduce_sum_, batch_range, max_over_ranks, sum_over_ranks


@pytest.mark.parametrize("gb,world", [(8, 2), (7, 2), (1, 3), (128, 8), (5, 5), (0, 2)])
def test_batch_range_partitions(gb, world):
    seen = []
    for r in range(world):
        a, b = batch_range(gb, world, r)
        assert 0 <= a <= b <= gb
        seen += list(range(a, b))
    assert seen == list(range(gb))
    sizes = [batch_range(gb, world, r)[1] - batch_range(gb, world, r)[0] for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def test_batch_range_rejects():
    with pytest.raises(ValueError):
        batch_range(4, 0, 0)
    with pytest.raises(ValueError):
        batch_range(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from tests.test_oracle_pins import rand_inputs

        inp = rand_inputs(b=5, L=17, H=2, P=3, N=4, R=2, rng=np.random.default_rng(99))
        a, b = batch_range(5, world, rank)
        part = {k: (v[a:b] if v.ndim >= 3 else v) for k, v in inp.items()}
        y, _ = oracle.scan_complex(**part, nthreads=1)
        ys = [None] * world
        dist.all_gather_object(ys, (a, b, y))
        t = max_over_ranks(float(rank + 1))
        s = sum_over_ranks(1.0)
        if rank == 0:
            y_full, _ = oracle.scan_complex(**inp, nthreads=1)
            got = np.concatenate([blk for _, _, blk in sorted(ys, key=lambda e: e[0])], 0)
            q.put((float(np.max(np.abs(got - y_full))), t, s))
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_match_unsharded():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    err, tmax, tsum = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert err == 0.0
    assert tmax == 2.0 and tsum == 2.0


def _bwd_worker(rank, world, port, q):
    """Data-parallel backward: each rank differentiates its batch shard; dA and dD
    (sums over the batch) are summed over the ranks, everything else stays local."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from tests.test_oracle_pins import rand_inputs

        rng = np.random.default_rng(77)
        inp = rand_inputs(b=5, L=13, H=3, P=3, N=4, R=2, rng=rng)
        dy = rng.standard_normal(inp["x"].shape)
        a, b = batch_range(5, world, rank)
        part = {k: (v[a:b] if v.ndim >= 3 else v) for k, v in inp.items()}
        g = oracle.scan_bwd(**part, dy=dy[a:b], nthreads=1)
        params = [torch.from_numpy(g["dA"].copy()), torch.from_numpy(g["dD"].copy())]
        all_reduce_sum_(params)
        dxs = [None] * world
        dist.all_gather_object(dxs, (a, g["dx"]))
        if rank == 0:
            full = oracle.scan_bwd(**inp, dy=dy, nthreads=1)
            dx = np.concatenate([blk for _, blk in sorted(dxs, key=lambda e: e[0])], 0)
            q.put((float(np.max(np.abs(params[0].numpy() - full["dA"]))),
                   float(np.max(np.abs(params[1].numpy() - full["dD"]))),
                   float(np.max(np.abs(dx - full["dx"])))))
    finally:
        dist.destroy_process_group()


def test_two_rank_backward_reduces_parameter_gradients():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_bwd_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    e_a, e_d, e_x = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert e_a < 1e-12 and e_d < 1e-12 and e_x == 0.0
