"""The prefill split across ranks (host logic and the all-gather), on CPU:

  * ic_prefill_partition covers [0, L) with disjoint ranges, and balances the
    F-layer work (scored pairs, rows t >= k cost t + 1) far better than a
    contiguous split;
  * with 2 gloo ranks on the tiny workload, each rank's all-gather of k_I, K
    and V reassembles the whole tensors exactly, and the rows each rank then
    computes (here with the oracle, the only CPU compute path) put together
    equal the one-rank oracle stack bit for bit.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _pairs(ranges, k):
    return sum(t + 1 for a, b in ranges for t in range(max(a, k), b))


@pytest.mark.parametrize("L,W", [(16384, 2), (16384, 4), (16384, 8), (512, 4), (131072, 8),
                                 (1000, 3), (7, 4), (5, 1), (0, 2)])
def test_partition_covers_rows_once(L, W):
    from cross_layer_top_b200 import sharding
    parts = sharding.partition(L, W)
    assert len(parts) == W
    seen = np.zeros(L, np.int32)
    for rr in parts:
        assert len(rr) == 2
        for a, b in rr:
            assert 0 <= a <= b <= L
            seen[a:b] += 1
    assert np.all(seen == 1)
    sizes = sorted(b - a for rr in parts for a, b in rr)
    assert not sizes or sizes[-1] - sizes[0] <= 1


@pytest.mark.parametrize("L,W", [(16384, 2), (16384, 4), (16384, 8), (131072, 8)])
def test_partition_balances_indexer_work(L, W):
    from cross_layer_top_b200 import sharding
    k = 2048
    work = [_pairs(rr, k) for rr in sharding.partition(L, W)]
    contiguous = [_pairs([(r * L // W, (r + 1) * L // W)], k) for r in range(W)]
    assert sum(work) == sum(contiguous)
    assert max(work) / np.mean(work) < 1.15
    assert max(contiguous) / np.mean(contiguous) > 1.5


def test_partition_rejects_bad_arguments():
    from cross_layer_top_b200 import indexcache as ic
    for args in [(16, 0, 0), (16, 2, 2), (16, 2, -1), (-1, 2, 0)]:
        with pytest.raises(ic.ICError) as e:
            ic.ic_prefill_partition(*args)
        assert e.value.code == ic.IC_ERR_INVALID_ARG


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
    import oracle
    from cross_layer_top_b200 import sharding, synth
    cfg = synth.CONFIGS["tiny"]
    L, k = cfg.L, cfg.k
    parts = sharding.partition(L, world)
    mine = parts[rank]
    rows = np.concatenate([np.arange(a, b) for a, b in mine]).astype(np.int32)
    idx_layers, out_layers, gathered_ok = [], [], True
    cache = None
    for l in range(cfg.n_layers):
        full = synth.prefill_layer(cfg, l, "cpu")  # every rank draws the same layer
        local = {n: sharding.rows_of(t, mine) for n, t in full.items()}
        g = {}
        for n in ("kI", "K", "V"):
            if n in local:
                g[n] = sharding.allgather_rows(local[n], parts, L)
                gathered_ok &= torch.equal(g[n], full[n])
        f = lambda t: synth.bf16_to_f32_numpy(t)
        if cfg.pattern[l] == "F":
            # the rank's rows only: its q_I / w rows at their positions
            qI = np.zeros((L,) + tuple(full["qI"].shape[1:]), np.float32)
            w = np.zeros((L, cfg.H_I), np.float32)
            qI[rows] = f(local["qI"])
            w[rows] = f(local["w"])
            cache = oracle.index_topk(qI, f(g["kI"]), w, k, rows=rows)
        Q = np.zeros((L, cfg.Hq, cfg.d), np.float32)
        Q[rows] = f(local["Q"])
        out = oracle.sparse_attn(Q, f(g["K"]), f(g["V"]), cache, rows=rows)
        idx_layers.append(cache)
        out_layers.append(out)
    q.put((rank, rows, idx_layers, out_layers, gathered_ok))
    dist.destroy_process_group()


def test_two_rank_gloo_split_equals_one_rank_oracle():
    import oracle
    from cross_layer_top_b200 import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = synth.CONFIGS["tiny"]
    layers = [{n: synth.bf16_to_f32_numpy(t) for n, t in synth.prefill_layer(cfg, l, "cpu").items()}
              for l in range(cfg.n_layers)]
    ref_idx, ref_out = oracle.run_stack(cfg.pattern, layers, cfg.k)
    covered = np.zeros(cfg.L, bool)
    for rank, rows, idx_layers, out_layers, gathered_ok in res:
        assert gathered_ok, "rank %d: the all-gather did not reassemble k_I, K, V" % rank
        covered[rows] = True
        for l in range(cfg.n_layers):
            assert np.array_equal(idx_layers[l], ref_idx[l][rows]), (rank, l)
            assert np.array_equal(out_layers[l], ref_out[l][rows]), (rank, l)
    assert covered.all()
