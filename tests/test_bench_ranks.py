"""bench.py's multi-rank plumbing on the CPU: world-size-2 gloo process group, each rank
reports its own time and every rank gets the maximum (the only collective the benchmark
uses; ranks run independent replicas with no data-path exchange)."""
import os
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank
        q.put((rank, bench.max_over_ranks(local_ms, world)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}


def test_single_rank_passthrough():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_weak_scaling_replicas_draw_different_inputs():
    """Each rank runs its own sequences: same shapes, different seeded inputs."""
    sys.path.insert(0, ROOT)
    import bench
    from layer_wise_mixed_b200 import configs, inputs
    w = configs.tiny()
    assert bench.rank_workload(w, 0, 1) is w
    ws = [bench.rank_workload(w, r, 4) for r in range(4)]
    assert len({x.name for x in ws}) == 4
    assert all((x.batch, x.n_kv_heads, x.layer_bits) == (w.batch, w.n_kv_heads, w.layer_bits) for x in ws)
    k0, _ = inputs.layer_kv(ws[0], 0, 32)
    k1, _ = inputs.layer_kv(ws[1], 0, 32)
    assert k0.shape == k1.shape and not (k0 == k1).all()
