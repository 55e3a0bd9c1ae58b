"""The N > 1 path of bench.py on CPU with the gloo backend (world size 2):
each rank draws its own sequence (weak scaling, no data-path collective),
the step time is reduced as the max over ranks, and the whole-job value
counts the units of every rank."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from cross_layer_top_b200 import synth
    cfg = bench.rank_config(synth.CONFIGS["tiny"], rank)
    lay = synth.prefill_layer(cfg, 0, "cpu")
    my_ms = 10.0 + 5.0 * rank  # a stand-in per-rank step time
    bench.dist_barrier(world)
    mx = bench.dist_max(my_ms, world, device="cpu")
    q.put((rank, cfg.seed, float(lay["qI"].float().sum()), mx))
    dist.destroy_process_group()


def test_two_rank_gloo_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, sum0, mx0), (r1, s1, sum1, mx1) = res
    assert s0 != s1 and sum0 != sum1          # independent sequences per rank
    assert mx0 == mx1 == 15.0                 # max over ranks, seen by every rank
    import sys
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 100 units x 3 steps in 15 ms (the slowest rank) -> 40000 units/s
    assert bench.weak_scaling_value(100, 3, 2, 15.0) == pytest.approx(40000.0)
