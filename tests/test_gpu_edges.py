"""Edge cases of the path on the GPU against the oracle: degenerate stacks
(L <= k, where every row keeps all of its causal keys and sparse attention
is ordinary causal attention; L = 1; k = 1; a single F layer), empty launches,
one-candidate decode rows, the longest decode rows, whose top-k leaves
the cluster form for the single-CTA kernel's general path (rows past its
shared selection bitmap), and decode stacks of ragged sequence lengths."""
import numpy as np
import pytest
import torch

import oracle
from cross_layer_top_b200 import synth
from tests import attn_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ic():
    from cross_layer_top_b200 import indexcache
    return indexcache


@pytest.fixture(scope="module")
def ctx(ic):
    c = ic.Context(0)
    yield c
    c.close()


def f32(t):
    return synth.bf16_to_f32_numpy(t)


def _stack(ic, ctx, cfg, pattern):
    layers = [synth.prefill_layer(cfg, l, "cpu", indexer=(c == "F")) for l, c in enumerate(pattern)]
    g = []
    for lay in layers:
        d = {n: v.cuda() for n, v in lay.items()}
        d["out"] = torch.empty((cfg.L, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        d["idx_snapshot"] = torch.empty((cfg.L, cfg.k), dtype=torch.int32, device="cuda")
        g.append(d)
    cache = torch.empty((cfg.L, cfg.k), dtype=torch.int32, device="cuda")
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, cfg.k, cfg.Hq, cfg.d, L=cfg.L)
    ic.ic_run_stack(ctx, ic.ic_create_pattern(pattern), g, dims, cache)
    ctx.sync_status()
    return layers, g


@pytest.mark.parametrize("L,k,pattern", [(100, 2048, "FSS"), (1, 64, "F"), (300, 1, "FSF"),
                                         (129, 128, "FS")])
def test_degenerate_prefill_stacks(ic, ctx, L, k, pattern):
    """Integer indexer inputs: indices bit-exact.  L <= k: every row keeps
    0..t, and the attention equals dense causal attention (torch SDPA in
    fp64 on the CPU).  k = 1: the single best key per row."""
    import dataclasses
    cfg = dataclasses.replace(synth.CONFIGS["tiny"], L=L, k=k, pattern=pattern, seed=11)
    layers, g = _stack(ic, ctx, cfg, pattern)
    olayers = [{n: f32(v) for n, v in lay.items()} for lay in layers]
    oidx, _ = oracle.run_stack(pattern, olayers, k)
    for l in range(len(pattern)):
        snap = g[l]["idx_snapshot"].cpu().numpy()
        assert np.array_equal(snap, oidx[l]), l
        got = g[l]["out"].float().cpu().numpy()
        attn_check.check(got, olayers[l]["Q"], olayers[l]["K"], olayers[l]["V"], snap,
                         what="L=%d k=%d layer %d" % (L, k, l))
        if L <= k:
            assert np.array_equal(snap[:, :L], np.where(np.tril(np.ones((L, L), bool)),
                                                        np.arange(L)[None, :], -1))
            q = torch.from_numpy(olayers[l]["Q"]).double().transpose(0, 1)  # [Hq, L, d]
            kk = torch.from_numpy(olayers[l]["K"]).double()[None].expand(cfg.Hq, L, cfg.d)
            vv = torch.from_numpy(olayers[l]["V"]).double()[None].expand(cfg.Hq, L, cfg.d)
            dense = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, is_causal=True)
            ref = dense.transpose(0, 1).numpy()
            assert np.abs(got - ref).max() <= 2e-2


def test_empty_launches_do_nothing(ic, ctx):
    """Zero rows of attention or overlap and an empty row range of the
    indexer enqueue nothing and leave the outputs untouched."""
    Q = torch.zeros((0, 16, 128), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((10, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((0, 64), dtype=torch.int32, device="cuda")
    out = torch.zeros((0, 16, 128), dtype=torch.bfloat16, device="cuda")
    ic.ic_sparse_attn(ctx, Q, K, K, idx, out)
    n0 = ctx.launch_count()
    cfg = synth.CONFIGS["tiny"]
    lay = synth.prefill_layer(cfg, 0, "cuda")
    sc = torch.full((4, 512), 7.0, device="cuda")
    ic.ic_index_score(ctx, lay["qI"], lay["kI"], lay["w"], 100, 100, sc, 512)
    ctx.sync_status()
    assert ctx.launch_count() == n0 and bool((sc == 7.0).all())


def test_decode_one_candidate_and_full_rows(ic, ctx):
    """Decode rows of 1, 2 and k candidates next to long rows: the short
    ones keep every candidate, the long ones match the oracle bit for bit
    (integer inputs)."""
    from tests.test_gpu_decode import _decode_inputs
    B, S_max, k = 5, 40000, 2048
    lens = [1, 2, 2048, 40000, 39999]
    q, w, k8, sc, lt = _decode_inputs(B, S_max, 64, 5, lens=lens, integer=True)
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    ic.ic_index_fp_decode(ctx, q.cuda(), w.cuda(), k8.cuda(), sc.cuda(), lt.cuda(), k, idx)
    ctx.sync_status()
    got = idx.cpu().numpy()
    for b in range(B):
        ref = oracle.decode_scores(f32(q[b]), f32(w[b]), k8[b].numpy(), sc[b].numpy(), S=lens[b])
        assert got[b].tolist() == oracle.topk_row(ref, k).tolist(), b


def test_decode_rows_past_the_cluster_form(ic, ctx):
    """Rows of 400001 candidates (longer than 8 CTAs' segments hold): the
    top-k takes the single-CTA kernel's general path (rows past its shared
    selection bitmap).  Integer inputs: bit-exact against the oracle."""
    from tests.test_gpu_decode import _decode_inputs
    B, S_max, k = 2, 400001, 2048
    q, w, k8, sc, lt = _decode_inputs(B, S_max, 64, 6, lens=[400001, 300000], integer=True)
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    ic.ic_index_fp_decode(ctx, q.cuda(), w.cuda(), k8.cuda(), sc.cuda(), lt.cuda(), k, idx)
    ctx.sync_status()
    got = idx.cpu().numpy()
    for b in range(B):
        n = int(lt[b])
        ref = oracle.decode_scores(f32(q[b]), f32(w[b]), k8[b].numpy(), sc[b].numpy(), S=n)
        assert got[b].tolist() == oracle.topk_row(ref, k).tolist(), b


@pytest.mark.parametrize("S_max", [9000, 40001])
def test_decode_stack_ragged_lengths(ic, ctx, S_max):
    """A decode stack whose sequences hold different numbers of candidates
    (1, k + 1, a middle length and the full capacity), with the single-CTA
    top-k (9000) and the cluster top-k (40001): F-layer selections within
    the oracle's bar (rows of at most k candidates take all of them), the
    reuse invariant, and every layer's attention against the oracle."""
    import dataclasses
    k = 2048
    cfg = dataclasses.replace(synth.CONFIGS["decode"], B=4, ctx=S_max - 1, pattern="FSFS", k=k,
                              seed=17)
    B, S = cfg.B, cfg.S
    lens = [S, 1, k + 1, S // 2]
    seq_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.decode_layer(cfg, l, "cuda")
        lay["seq_len"] = seq_len
        lay["out"] = torch.empty((B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        lay["idx_snapshot"] = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
        layers.append(lay)
    dims = ic.stack_dims(ic.IC_DECODE, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, B=B, S_max=S,
                         seq_len=seq_len)
    cache = torch.empty((B, k), dtype=torch.int32, device="cuda")
    ic.ic_run_stack(ctx, ic.ic_create_pattern(cfg.pattern), layers, dims, cache)
    ctx.sync_status()
    src = oracle.pattern_src(cfg.pattern)
    snaps = [lay["idx_snapshot"].cpu().numpy() for lay in layers]
    for l, c in enumerate(cfg.pattern):
        assert np.array_equal(snaps[l], snaps[src[l]]), l
        lay = layers[l]
        if c == "F":
            for b in range(B):
                n = lens[b]
                ref = oracle.decode_scores(f32(lay["q"][b]), f32(lay["w"][b]),
                                           lay["kI8"][b].cpu().numpy(),
                                           lay["kI_scale"][b].cpu().numpy(), S=n)
                row = snaps[l][b]
                m = min(n, k)
                assert np.all(row[m:] == -1) and np.all(np.diff(row[:m]) > 0)
                assert row[:m].min() >= 0 and row[:m].max() < n
                if n <= k:
                    assert row[:m].tolist() == list(range(n))
                else:
                    kth = oracle.kth_score(ref, k)
                    assert ref[row[:m]].min() >= kth - 1e-3 * abs(kth)
        got = lay["out"].float().cpu().numpy().astype(np.float64)
        attn_check.check(got, f32(lay["Q"]), f32(lay["K"]), f32(lay["V"]), snaps[l],
                         rows_per_seq=1, what="ragged decode S_max=%d layer %d" % (S_max, l))
