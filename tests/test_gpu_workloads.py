"""GPU parity at the full sizes of the workloads, in the launch
configuration the benchmark times, on sampled outputs the oracle computes
one by one:

  * long prefill: L = 131072, H_I = 64, d_I = 128, k = 2048: one F layer
    with its score scratch processed in row chunks; the FSSS stack (an S
    layer's attention rows checked) and the all-F stack (every F layer's
    selections on sampled rows);
  * batched decode: the whole 16-layer FSSS x4 stack at 32 sequences x
    65537 candidates: every F layer's selections for 4 sequences and the
    attention of 4 layers (S layers among them);
  * 200K-context decode: 8 sequences x 200001 candidates, 47-layer stacks at
    uniform retention 1/1, 1/2, 1/4 and 1/8 and under the searched 1/4
    pattern (F layers checked against the oracle, S layers must carry their
    F layer's index tensor), FP8 indexer keys.

Same bars as tests/test_gpu_parity.py: selected sets within 1e-3 of the
oracle's k-th score, attention within 2e-2 + 1e-2 |o| and the bf16 rounding
bound of tests/attn_check.py.
"""
import numpy as np
import pytest
import torch

import oracle
from cross_layer_top_b200 import synth
from tests import attn_check

pytestmark = pytest.mark.gpu

SEL_RTOL = 1e-3


@pytest.fixture(scope="module")
def ic():
    from cross_layer_top_b200 import indexcache
    return indexcache


def f32(t):
    return synth.bf16_to_f32_numpy(t)


def check_selection(idx_row, score_row, k):
    n = len(score_row)
    m = min(n, k)
    sel = idx_row[:m]
    assert np.all(idx_row[m:] == -1) and np.all(np.diff(sel) > 0)
    assert sel.min() >= 0 and sel.max() < n
    if n <= k:
        assert sel.tolist() == list(range(n))
        return
    kth = oracle.kth_score(score_row, k)
    assert score_row[sel].min() >= kth - SEL_RTOL * abs(kth)


def test_long_prefill_sampled(ic):
    cfg = synth.CONFIGS["long_prefill"]
    L, k = cfg.L, cfg.k
    # a 1 GiB score scratch forces several row chunks
    ctx = ic.Context(0, scratch_bytes=1 << 30)
    lay = synth.prefill_layer(cfg, 0, "cuda")
    idx = torch.empty((L, k), dtype=torch.int32, device="cuda")
    ic.ic_index_fp(ctx, lay["qI"], lay["kI"], lay["w"], k, idx)
    out = torch.empty((L, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
    ic.ic_sparse_attn(ctx, lay["Q"], lay["K"], lay["V"], idx, out)
    ctx.sync_status()
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([[0, k - 1, k, 2049, 65535, 65536, L - 1],
                                     rng.integers(k, L, 9)])).astype(np.int32)
    rt = torch.from_numpy(rows).long().cuda()
    sc = oracle.index_scores_at(f32(lay["qI"][rt]), f32(lay["w"][rt]), f32(lay["kI"]), rows)
    got = idx[rt].cpu().numpy()
    for r, t in enumerate(rows):
        check_selection(got[r], sc[r, :t + 1], k)
    o = out[rt].float().cpu().numpy().astype(np.float64)
    attn_check.check(o, f32(lay["Q"][rt]), f32(lay["K"]), f32(lay["V"]), got, rows=rows,
                     q_is_rows=True, what="long prefill")
    ctx.close()


def _prefill_stack(ic, ctx, cfg, pattern, snap_layers):
    """Runs the prefill stack of `cfg` under `pattern` (every layer drawn with
    indexer inputs); snapshots the index tensors of snap_layers."""
    L, k = cfg.L, cfg.k
    layers = []
    for l in range(len(pattern)):
        lay = synth.prefill_layer(cfg, l, "cuda", indexer=True)
        lay["out"] = torch.empty((L, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        if l in snap_layers:
            lay["idx_snapshot"] = torch.empty((L, k), dtype=torch.int32, device="cuda")
        layers.append(lay)
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, L=L)
    cache = torch.empty((L, k), dtype=torch.int32, device="cuda")
    ic.ic_run_stack(ctx, ic.ic_create_pattern(pattern), layers, dims, cache)
    ctx.sync_status()
    return layers


def _check_prefill_rows(lay, idx_rows, rows, k, what, selection=True):
    rt = torch.from_numpy(rows).long().cuda()
    if selection:
        sc = oracle.index_scores_at(f32(lay["qI"][rt]), f32(lay["w"][rt]), f32(lay["kI"]), rows)
        for r, t in enumerate(rows):
            check_selection(idx_rows[r], sc[r, :t + 1], k)
    o = lay["out"][rt].float().cpu().numpy().astype(np.float64)
    attn_check.check(o, f32(lay["Q"][rt]), f32(lay["K"]), f32(lay["V"]), idx_rows, rows=rows,
                     q_is_rows=True, what=what)


def test_long_prefill_fsss_stack(ic):
    """The long-prefill FSSS stack: layer 0's selections and attention on
    sampled rows, and the attention of S layer 2 on the same rows with the
    reused indices (which must equal layer 0's)."""
    cfg = synth.CONFIGS["long_prefill"]
    L, k = cfg.L, cfg.k
    ctx = ic.Context(0)
    layers = _prefill_stack(ic, ctx, cfg, "FSSS", (0, 2))
    rows = np.array([1, k - 1, k, 40000, 99999, L - 1], np.int32)
    rt = torch.from_numpy(rows).long().cuda()
    assert torch.equal(layers[0]["idx_snapshot"], layers[2]["idx_snapshot"])
    idx_rows = layers[0]["idx_snapshot"][rt].cpu().numpy()
    _check_prefill_rows(layers[0], idx_rows, rows, k, "long prefill layer 0")
    _check_prefill_rows(layers[2], idx_rows, rows, k, "long prefill S layer 2", selection=False)
    ctx.close()


def test_long_prefill_all_f_stack(ic):
    """The long-prefill all-F stack (the indexer-share run): every F layer
    selects from its own scores; sampled rows of layers 1 and 3."""
    cfg = synth.CONFIGS["long_prefill_allF"]
    L, k = cfg.L, cfg.k
    ctx = ic.Context(0)
    layers = _prefill_stack(ic, ctx, cfg, "FFFF", (1, 3))
    for l, rows in ((1, [k, 77777, L - 1]), (3, [k - 1, 5000, 131000])):
        rows = np.array(rows, np.int32)
        rt = torch.from_numpy(rows).long().cuda()
        idx_rows = layers[l]["idx_snapshot"][rt].cpu().numpy()
        _check_prefill_rows(layers[l], idx_rows, rows, k, "all-F layer %d" % l)
    ctx.close()


def _decode_stack_layers(cfg, all_indexer):
    B, k = cfg.B, cfg.k
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.decode_layer(cfg, l, "cuda", indexer=True if all_indexer else None)
        lay["out"] = torch.empty((B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        lay["idx_snapshot"] = torch.empty((B, k), dtype=torch.int32, device="cuda")
        layers.append(lay)
    return layers


def _run_and_check_decode(ic, ctx, cfg, layers, pattern, f_checks, seqs, attn_layers):
    """One decode step of the stack under `pattern`: the reuse invariant on
    every layer, the selections of the first f_checks F layers (and the
    last) for `seqs`, and the attention of attn_layers."""
    B, S, k = cfg.B, cfg.S, cfg.k
    dims = ic.stack_dims(ic.IC_DECODE, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, B=B, S_max=S,
                         seq_len=layers[0]["seq_len"])
    cache = torch.empty((B, k), dtype=torch.int32, device="cuda")
    for lay in layers:
        lay["idx_snapshot"].fill_(-7)
    ic.ic_run_stack(ctx, ic.ic_create_pattern(pattern), layers, dims, cache)
    ctx.sync_status()
    src = oracle.pattern_src(pattern)
    snaps = [lay["idx_snapshot"].cpu().numpy() for lay in layers]
    f_layers = [l for l, c in enumerate(pattern) if c == "F"]
    checked = 0
    for l in sorted(set(f_layers[:f_checks] + f_layers[-1:])):
        lay = layers[l]
        for b in seqs:
            sc = oracle.decode_scores(f32(lay["q"][b]), f32(lay["w"][b]),
                                      lay["kI8"][b].cpu().numpy(), lay["kI_scale"][b].cpu().numpy())
            check_selection(snaps[l][b], sc, k)
            checked += 1
    for l in range(len(pattern)):
        assert np.array_equal(snaps[l], snaps[src[l]]), (pattern, l)
    for l in attn_layers:
        lay = layers[l]
        o = lay["out"].float().cpu().numpy().astype(np.float64)
        attn_check.check(o, f32(lay["Q"]), f32(lay["K"]), f32(lay["V"]), snaps[l],
                         rows_per_seq=1, what="%s decode layer %d" % (pattern, l))
    return checked


def test_batched_decode_full_stack(ic):
    """The whole batched-decode stack (32 x 65537, 16 layers FSSS x4): every
    F layer's selections for 4 sequences, attention of layers 0, 1, 6 and
    15 (S layers 1, 6 and 15 attend with reused indices)."""
    cfg = synth.CONFIGS["decode"]
    ctx = ic.Context(0)
    layers = _decode_stack_layers(cfg, all_indexer=False)
    n = _run_and_check_decode(ic, ctx, cfg, layers, cfg.pattern, 4, (0, 7, 20, 31), (0, 1, 6, 15))
    assert n == 16
    ctx.close()


@pytest.fixture(scope="module")
def sweep_layers():
    cfg = synth.CONFIGS["decode_sweep_r1"]
    layers = _decode_stack_layers(cfg, all_indexer=True)
    yield cfg, layers
    del layers[:]
    torch.cuda.empty_cache()


@pytest.mark.parametrize("which", ["r1", "r2", "r4", "r8", "searched_1/4"])
def test_decode_200k_retention_stacks(ic, sweep_layers, which):
    """47-layer decode stacks over 8 x 200001 candidates, the same layer
    tensors under each pattern of the retention sweep (uniform 1/1, 1/2,
    1/4, 1/8; the searched 1/4 string of the summary page's Appendix B)."""
    cfg, layers = sweep_layers
    if which.startswith("searched"):
        pattern = synth.SEARCHED_PATTERNS_47[which.split("_")[1]]
        assert pattern.count("F") == 12
    else:
        r = int(which[1:])
        pattern = synth.uniform_pattern(cfg.n_layers, r)
        assert pattern.count("F") == {1: 47, 2: 24, 4: 12, 8: 6}[r]
    ctx = ic.Context(0)
    n = _run_and_check_decode(ic, ctx, cfg, layers, pattern, 2, (0, cfg.B - 1), (0, 1, 23, 46))
    assert n == 6
    ctx.close()
