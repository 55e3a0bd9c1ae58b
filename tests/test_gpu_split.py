"""The prefill split across ranks on the GPU, with the ranks run one after
another on one device (they never wait on one another: after the
all-gather each rank's work is local).

Every rank's rows of the index tensors must equal the same rows of the
one-rank stack bit for bit: the indexer and the top-k compute each row from
the same inputs in the same order, whichever rows share the launch.  The
same holds for the attention outputs while both launches keep one CTA per
row.  A launch of few rows (under about three CTAs per SM) spreads each
row's key slots over a cluster of CTAs, which rounds differently.  A rank's
output rows are then checked against the oracle with the attention bars
instead.

The all-gather itself is the host-side plumbing checked with gloo ranks in
tests/test_prefill_split.py.  Here each rank's k_I/K/V are the whole
tensors it would receive."""
import numpy as np
import pytest
import torch

from cross_layer_top_b200 import synth
from tests import attn_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ic():
    from cross_layer_top_b200 import indexcache
    return indexcache


def _full_stack(ic, ctx, cfg, layers):
    L, k = cfg.L, cfg.k
    for lay in layers:
        lay["out"] = torch.empty((L, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        lay["idx_snapshot"] = torch.empty((L, k), dtype=torch.int32, device="cuda")
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, L=L)
    cache = torch.empty((L, k), dtype=torch.int32, device="cuda")
    ic.ic_run_stack(ctx, ic.ic_create_pattern(cfg.pattern), layers, dims, cache)
    ctx.sync_status()
    return dims


@pytest.mark.parametrize("name,world", [("tiny", 2), ("tiny", 3), ("prefill", 4), ("prefill", 8)])
def test_split_ranks_equal_one_rank_stack(ic, name, world):
    from cross_layer_top_b200 import sharding
    cfg = synth.CONFIGS[name]
    L, k = cfg.L, cfg.k
    ctx = ic.Context(0)
    layers = [synth.prefill_layer(cfg, l, "cuda") for l in range(cfg.n_layers)]
    dims = _full_stack(ic, ctx, cfg, layers)
    pat = ic.ic_create_pattern(cfg.pattern)
    covered = torch.zeros(L, dtype=torch.bool)
    for rank, mine in enumerate(sharding.partition(L, world)):
        n = sum(b - a for a, b in mine)
        local = []
        for lay in layers:
            loc = {m: sharding.rows_of(lay[m], mine) for m in ("qI", "w", "Q") if m in lay}
            loc.update({m: lay[m] for m in ("kI", "K", "V") if m in lay})  # gathered: all rows
            loc["out"] = torch.empty((n, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
            loc["idx_snapshot"] = torch.empty((n, k), dtype=torch.int32, device="cuda")
            local.append(loc)
        cache = torch.empty((n, k), dtype=torch.int32, device="cuda")
        ic.ic_run_stack_rows(ctx, pat, local, dims, mine, cache)
        ctx.sync_status()
        rows = np.concatenate([np.arange(a, b) for a, b in mine]).astype(np.int32)
        for l in range(cfg.n_layers):
            idx_l = local[l]["idx_snapshot"]
            assert torch.equal(idx_l, sharding.rows_of(layers[l]["idx_snapshot"], mine)), (rank, l)
            if torch.equal(local[l]["out"], sharding.rows_of(layers[l]["out"], mine)):
                continue
            assert n < 3 * torch.cuda.get_device_properties(0).multi_processor_count, (rank, l)
            sel = np.arange(n) if n <= 256 else np.linspace(0, n - 1, 64).astype(np.int64)
            f = synth.bf16_to_f32_numpy
            attn_check.check(local[l]["out"].float().cpu().numpy()[sel],
                             f(layers[l]["Q"]), f(layers[l]["K"]), f(layers[l]["V"]),
                             idx_l.cpu().numpy()[sel], rows=rows[sel],
                             what="rank %d layer %d" % (rank, l))
        for a, b in mine:
            covered[a:b] = True
    assert covered.all()
    ctx.close()


def test_index_fp_rows_ranges_across_k(ic):
    """ic_index_fp_rows on ranges below k, across k and past k (compact q_I /
    w rows) equals the same rows of ic_index_fp."""
    cfg = synth.CONFIGS["tiny"]
    L, k = cfg.L, cfg.k
    ctx = ic.Context(0)
    lay = synth.prefill_layer(cfg, 0, "cuda")
    full = torch.empty((L, k), dtype=torch.int32, device="cuda")
    ic.ic_index_fp(ctx, lay["qI"], lay["kI"], lay["w"], k, full)
    for a, b in [(0, 10), (10, 64), (30, 200), (64, 65), (300, 512), (511, 512), (100, 100)]:
        got = torch.full((b - a, k), -7, dtype=torch.int32, device="cuda")
        ic.ic_index_fp_rows(ctx, lay["qI"][a:b].contiguous(), lay["w"][a:b].contiguous(), lay["kI"],
                            a, b, k, got)
        ctx.sync_status()
        assert torch.equal(got, full[a:b]), (a, b)
    ctx.close()
