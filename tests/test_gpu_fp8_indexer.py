"""GPU parity of the FP8 prefill indexer (e4m3 q_I / k_I with fp32 scales,
tcgen05 kind::f8f6f4) against the oracle's scores on the dequantised inputs.

Bars: bit-exact on integer inputs (every product and sum exact in fp32);
Gaussian inputs within 1e-4 of the row's largest score; selected sets within
1e-3 of the oracle's k-th score, as for the bf16 indexer."""
import numpy as np
import pytest
import torch

import oracle
from cross_layer_top_b200 import synth

pytestmark = pytest.mark.gpu

SEL_RTOL = 1e-3


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


def _e4m3_table():
    """e4m3 bytes of the integers -6..6 (index v + 6)."""
    out = []
    for v in range(-6, 7):
        if v == 0:
            out.append(0)
            continue
        a = abs(v)
        e = a.bit_length() - 1
        m = (a - (1 << e)) * 8 >> e
        out.append((0x80 if v < 0 else 0) | ((e + 7) << 3) | m)
    return torch.tensor(out, dtype=torch.uint8)


def _integer_inputs(L, H, seed):
    gen = torch.Generator().manual_seed(seed)
    tab = _e4m3_table()
    qI8 = tab[torch.randint(0, 13, (L, H, 128), generator=gen)]
    kI8 = tab[torch.randint(0, 13, (L, 128), generator=gen)]
    q_scale = torch.tensor([0.5, 1.0, 2.0])[torch.randint(0, 3, (L, H), generator=gen)]
    k_scale = torch.tensor([0.25, 1.0, 4.0])[torch.randint(0, 3, (L,), generator=gen)]
    w = torch.tensor([-1.0, -0.5, 0.5, 1.0])[torch.randint(0, 4, (L, H), generator=gen)].bfloat16()
    return qI8, q_scale.float(), kI8, k_scale.float(), w


@pytest.mark.parametrize("H_I", [64, 32, 16])
def test_fp8_scores_integer_bit_exact(ic, ctx, H_I):
    L = 700  # several 128-key tiles and a ragged tail
    qI8, qs, kI8, ks, w = _integer_inputs(L, H_I, H_I)
    ld = 704
    out = torch.full((L, ld), float("nan"), device="cuda")
    ic.ic_index_score_fp8(ctx, qI8.cuda(), qs.cuda(), kI8.cuda(), ks.cuda(), w.cuda(), 0, L, out)
    ctx.sync_status()
    ref = oracle.index_scores_fp8(qI8.numpy(), qs.numpy(), kI8.numpy(), ks.numpy(), f32(w))
    got = out.cpu().numpy().astype(np.float64)
    tri = np.tril(np.ones((L, L), bool))
    assert np.array_equal(got[:, :L][tri], ref[tri])
    assert np.all(np.isnan(got[:, :L][~tri]))  # s > t never written


def test_fp8_scores_row_window(ic, ctx):
    """A row window [row_begin, row_end) writes rows t - row_begin only."""
    L, H_I = 600, 64
    qI8, qs, kI8, ks, w = _integer_inputs(L, H_I, 5)
    rb, re = 130, 517
    out = torch.full((re - rb, 520), float("nan"), device="cuda")
    ic.ic_index_score_fp8(ctx, qI8.cuda(), qs.cuda(), kI8.cuda(), ks.cuda(), w.cuda(), rb, re, out)
    ctx.sync_status()
    rows = np.arange(rb, re, dtype=np.int32)
    ref = oracle.index_scores_fp8(qI8.numpy(), qs.numpy(), kI8.numpy(), ks.numpy(), f32(w), rows=rows)
    got = out.cpu().numpy().astype(np.float64)
    for i, t in enumerate(rows):
        assert np.array_equal(got[i, :t + 1], ref[i, :t + 1])


def test_fp8_scores_gaussian_close(ic, ctx):
    cfg = synth.PrefillConfig("fp8_small", 3000, "F", 64, 128, 2048, 16, 128, 9)
    lay = synth.prefill_indexer_fp8(cfg, 0, "cuda")
    L = cfg.L
    out = torch.zeros((L, 3008), device="cuda")
    ic.ic_index_score_fp8(ctx, lay["qI8"], lay["q_scale"], lay["kI8"], lay["k_scale"], lay["w"], 0,
                          L, out)
    ctx.sync_status()
    rows = np.array([0, 1, 127, 128, 999, 2047, 2048, L - 1], np.int32)
    ref = oracle.index_scores_fp8(lay["qI8"].cpu().numpy(), lay["q_scale"].cpu().numpy(),
                                  lay["kI8"].cpu().numpy(), lay["k_scale"].cpu().numpy(),
                                  f32(lay["w"]), rows=rows)
    got = out.cpu().numpy()[rows].astype(np.float64)
    for i, t in enumerate(rows):
        r = ref[i, :t + 1]
        assert np.all(np.abs(got[i, :t + 1] - r) <= 1e-4 * np.abs(r).max() + 1e-6)


def test_fp8_index_fp_prefill_workload_sampled(ic, ctx):
    """The prefill workload's sizes (L=16384, H_I=64, d_I=128, k=2048) with
    its indexer inputs quantised: F-layer selections on sampled rows."""
    cfg = synth.CONFIGS["prefill"]
    lay = synth.prefill_indexer_fp8(cfg, 0, "cuda")
    L, k = cfg.L, cfg.k
    idx = torch.empty((L, k), dtype=torch.int32, device="cuda")
    ic.ic_index_fp_fp8(ctx, lay["qI8"], lay["q_scale"], lay["kI8"], lay["k_scale"], lay["w"], k, idx)
    ctx.sync_status()
    rows = np.array([0, k - 1, k, k + 1, 9000, L - 1], np.int32)
    ref = oracle.index_scores_fp8(lay["qI8"].cpu().numpy(), lay["q_scale"].cpu().numpy(),
                                  lay["kI8"].cpu().numpy(), lay["k_scale"].cpu().numpy(),
                                  f32(lay["w"]), rows=rows)
    got = idx.cpu().numpy()[rows]
    for i, t in enumerate(rows):
        sel = got[i, :min(t + 1, k)]
        assert np.all(np.diff(sel) > 0) and sel.min() >= 0 and sel.max() <= t
        assert np.all(got[i, min(t + 1, k):] == -1)
        if t + 1 <= k:
            assert sel.tolist() == list(range(t + 1))
        else:
            kth = oracle.kth_score(ref[i, :t + 1], k)
            assert ref[i, sel].min() >= kth - SEL_RTOL * abs(kth)


def test_fp8_argument_errors(ic, ctx):
    L = 256
    qI8 = torch.zeros((L, 4, 128), dtype=torch.uint8, device="cuda")
    qs = torch.ones((L, 4), device="cuda")
    kI8 = torch.zeros((L, 128), dtype=torch.uint8, device="cuda")
    ks = torch.ones(L, device="cuda")
    w = torch.zeros((L, 4), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((L, L), device="cuda")
    with pytest.raises(ic.ICError) as e:
        ic.ic_index_score_fp8(ctx, qI8, qs, kI8, ks, w, 0, L, out)  # H_I = 4
    assert e.value.code == ic.IC_ERR_UNSUPPORTED
    qI8 = torch.zeros((L, 64, 64), dtype=torch.uint8, device="cuda")
    qs = torch.ones((L, 64), device="cuda")
    kI8 = torch.zeros((L, 64), dtype=torch.uint8, device="cuda")
    w = torch.zeros((L, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ic.ICError) as e:
        ic.ic_index_score_fp8(ctx, qI8, qs, kI8, ks, w, 0, L, out)  # d_I = 64
    assert e.value.code == ic.IC_ERR_UNSUPPORTED
