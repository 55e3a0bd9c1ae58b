"""GPU parity of the decode path (FP8 indexer-key scan, top-k over whole
sequences, split attention) against the CPU oracle."""
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


@pytest.fixture(scope="module")
def ctx(ic):
    c = ic.Context(0)
    yield c
    c.close()


def f32(t):
    return synth.bf16_to_f32_numpy(t)


def _decode_inputs(B, S_max, H_I, seed, lens=None, integer=False):
    gen = torch.Generator().manual_seed(seed)
    if integer:
        q = torch.randint(-3, 4, (B, H_I, 128), generator=gen).bfloat16()
        w = torch.tensor([-1.0, -0.5, 0.5, 1.0])[torch.randint(0, 4, (B, H_I), generator=gen)].bfloat16()
        # e4m3 bytes of small integers and halves: 0, +-0.5, +-1, +-1.5, +-2, +-3
        table = torch.tensor([0x00, 0x30, 0xB0, 0x38, 0xB8, 0x3C, 0xBC, 0x40, 0xC0, 0x44, 0xC4],
                             dtype=torch.uint8)
        k8 = table[torch.randint(0, len(table), (B, S_max, 128), generator=gen)]
        sc = torch.tensor([1.0, 0.5, 2.0, 0.25])[torch.randint(0, 4, (B, S_max), generator=gen)]
    else:
        q = torch.randn((B, H_I, 128), generator=gen).bfloat16()
        w = (torch.randn((B, H_I), generator=gen) / 8).bfloat16()
        k8, sc = synth.fp8_e4m3_quantize_per_token(torch.randn((B, S_max, 128), generator=gen))
    if lens is None:
        lens = [S_max] * B
    return q, w, k8.contiguous(), sc.float().contiguous(), torch.tensor(lens, dtype=torch.int32)


@pytest.mark.parametrize("H_I", [64, 32])
def test_decode_scores_integer_bit_exact(ic, ctx, H_I):
    B, S_max = 3, 1000
    q, w, k8, sc, lens = _decode_inputs(B, S_max, H_I, 1, lens=[1000, 129, 1], integer=True)
    ld = 1024
    out = torch.full((B, ld), float("nan"), device="cuda")
    ic.ic_index_score_decode(ctx, q.cuda(), w.cuda(), k8.cuda(), sc.cuda(), lens.cuda(), out)
    ctx.sync_status()
    got = out.cpu().numpy()
    for b in range(B):
        n = int(lens[b])
        ref = oracle.decode_scores(f32(q[b]), f32(w[b]), k8[b].numpy(), sc[b].numpy(), S=n)
        assert np.array_equal(got[b, :n].astype(np.float64), ref)
        assert np.all(np.isnan(got[b, n:]))


def _e4m3_byte_of_int(v):
    """e4m3 encoding of an integer with |v| <= 16 (1 sign, 4 exponent bits
    with bias 7, 3 mantissa bits)."""
    if v == 0:
        return 0
    a = abs(v)
    e = a.bit_length() - 1
    m = (a - (1 << e)) * 8 >> e
    assert (((1 << e) + (m << e >> 3)) == a), v
    return (0x80 if v < 0 else 0) | ((e + 7) << 3) | m


@pytest.mark.parametrize("H_I", [64, 32])
def test_decode_scores_wide_integer_exact(ic, ctx, H_I):
    """Integer q in [-31, 31] and integer keys in [-16, 16]: a dot product
    reaches 6.3e4 (well past 2^14) and every product, dot product and head
    sum is an integer multiple of 0.5 small enough to be exact in fp32, so
    the scores must equal the oracle's bit for bit.  This pins the split of
    q into two e4m3 terms and full fp32 accumulation in the tensor core."""
    B, S_max = 2, 777
    gen = torch.Generator().manual_seed(11)
    q = torch.randint(-31, 32, (B, H_I, 128), generator=gen).float()
    q[:, 0, 0] = 31.0  # fixes max|q|, hence the power-of-two rescaling
    q[:, 1, :] = torch.where(q[:, 1, :] >= 0, 31.0, -31.0)  # a head with large dot products
    table = torch.tensor([_e4m3_byte_of_int(v) for v in range(-16, 17)], dtype=torch.uint8)
    k8 = table[torch.randint(0, 33, (B, S_max, 128), generator=gen)]
    for b in range(B):  # rows 0..4: keys 16 sign(q[b,1,:]), so head 1's dot product is 31*16*128
        k8[b, :5, :] = torch.where(q[b, 1, :] >= 0, table[32], table[0])
    w = torch.tensor([-1.0, -0.5, 0.5, 1.0])[torch.randint(0, 4, (B, H_I), generator=gen)]
    sc = torch.tensor([1.0, 0.5, 2.0, 0.25])[torch.randint(0, 4, (B, S_max), generator=gen)]
    lens = torch.tensor([S_max, 300], dtype=torch.int32)
    q, w = q.bfloat16(), w.bfloat16()
    out = torch.full((B, 780), float("nan"), device="cuda")  # ld: a multiple of 4
    ic.ic_index_score_decode(ctx, q.cuda(), w.cuda(), k8.cuda(), sc.float().cuda(), lens.cuda(), out)
    ctx.sync_status()
    got = out.cpu().numpy()
    for b in range(B):
        n = int(lens[b])
        ref = oracle.decode_scores(f32(q[b]), f32(w[b]), k8[b].numpy(), sc[b].float().numpy(), S=n)
        assert np.array_equal(got[b, :n].astype(np.float64), ref)


def test_decode_scores_gaussian_close(ic, ctx):
    B, S_max = 4, 6000
    q, w, k8, sc, lens = _decode_inputs(B, S_max, 64, 2, lens=[6000, 5999, 4097, 3])
    out = torch.zeros((B, 6016), device="cuda")
    ic.ic_index_score_decode(ctx, q.cuda(), w.cuda(), k8.cuda(), sc.cuda(), lens.cuda(), out)
    ctx.sync_status()
    got = out.cpu().numpy()
    for b in range(B):
        n = int(lens[b])
        ref = oracle.decode_scores(f32(q[b]), f32(w[b]), k8[b].numpy(), sc[b].numpy(), S=n)
        assert np.all(np.abs(got[b, :n] - ref) <= 1e-4 * np.abs(ref).max() + 1e-6)


def test_decode_index_selected_set(ic, ctx):
    B, S_max, k = 4, 70001, 2048
    q, w, k8, sc, lens = _decode_inputs(B, S_max, 64, 3, lens=[70001, 2048, 2049, 33333])
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    ic.ic_index_fp_decode(ctx, q.cuda(), w.cuda(), k8.cuda(), sc.cuda(), lens.cuda(), k, idx)
    ctx.sync_status()
    got = idx.cpu().numpy()
    for b in range(B):
        n = int(lens[b])
        ref = oracle.decode_scores(f32(q[b]), f32(w[b]), k8[b].numpy(), sc[b].numpy(), S=n)
        m = min(n, k)
        sel = got[b, :m]
        assert np.all(got[b, m:] == -1) and np.all(np.diff(sel) > 0) and sel.max() < n
        if n > k:
            kth = oracle.kth_score(ref, k)
            assert ref[sel].min() >= kth - SEL_RTOL * abs(kth)


def _first_digit_bin_count(score64, k):
    """How many of a row's fp32 scores share the top 11 bits of the order key
    (sign-adjusted bits, -0.0 as +0.0) with its k-th largest score: the
    size of the top-k's threshold bin on the first radix digit."""
    x = (score64.astype(np.float32) + np.float32(0.0)).view(np.uint32)
    key = np.where(x >> 31 == 1, ~x, x | np.uint32(0x80000000)).astype(np.uint32)
    kth = np.sort(key)[::-1][k - 1]
    return int(np.sum((key >> 21) == (kth >> 21)))


def test_decode_index_histogram_paths_bit_exact(ic, ctx):
    """The decode F layer with the scan's first-digit histograms (cluster
    top-k): rows whose threshold bin fits the candidate list, rows whose bin
    overflows it (massive ties: a zero query gives all-zero scores), rows of
    at most k candidates, in one launch and again in a second call with the
    roles swapped (the histograms must be clear between calls).  Integer
    inputs make the scores exact, so every row must equal the oracle's
    top-k bit for bit (ties to the lower index)."""
    B, S_max, k = 6, 70001, 2048
    lens = [70001, 2048, 60000, 70001, 1, 50001]
    q, w, k8, sc, lens_t = _decode_inputs(B, S_max, 64, 21, lens=lens, integer=True)
    calls = []
    q1 = q.clone()
    q1[3] = 0  # row 3: every score 0
    calls.append(q1)
    q2 = q.clone()
    q2[0] = 0  # second call: row 0 tied instead, row 3 spread out
    calls.append(q2)
    kinds = set()
    for qc in calls:
        idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
        ic.ic_index_fp_decode(ctx, qc.cuda(), w.cuda(), k8.cuda(), sc.cuda(), lens_t.cuda(), k, idx)
        ctx.sync_status()
        got = idx.cpu().numpy()
        for b in range(B):
            n = lens[b]
            ref = oracle.decode_scores(f32(qc[b]), f32(w[b]), k8[b].numpy(), sc[b].numpy(), S=n)
            assert got[b].tolist() == oracle.topk_row(ref, k).tolist(), b
            if n > k:
                kinds.add("fits" if _first_digit_bin_count(ref, k) <= 4096 else "overflows")
    assert kinds == {"fits", "overflows"}


def test_decode_index_few_ties_bit_exact(ic, ctx):
    """The decode F layer (scan with first-digit histograms, cluster top-k)
    on wide integer inputs (q in [-31, 31], keys in [-16, 16]): every score
    is exact in fp32 (as in test_decode_scores_wide_integer_exact) and the
    scores are spread widely, so the k-th largest is mostly unique.  Rows
    whose keys equal to the threshold are all taken select through the
    top-k's bitmap output; every row must equal the oracle's top-k bit for
    bit, and most rows must be of that kind."""
    B, S_max, k, H_I = 4, 70001, 2048, 64
    gen = torch.Generator().manual_seed(29)
    q = torch.randint(-31, 32, (B, H_I, 128), generator=gen).float()
    q[:, 0, 0] = 31.0
    table = torch.tensor([_e4m3_byte_of_int(v) for v in range(-16, 17)], dtype=torch.uint8)
    k8 = table[torch.randint(0, 33, (B, S_max, 128), generator=gen)]
    w = torch.tensor([-1.0, -0.5, 0.5, 1.0])[torch.randint(0, 4, (B, H_I), generator=gen)]
    sc = torch.tensor([1.0, 0.5, 2.0, 0.25])[torch.randint(0, 4, (B, S_max), generator=gen)]
    lens = [S_max, 65537, 40000, 2049]
    q, w = q.bfloat16(), w.bfloat16()
    idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    ic.ic_index_fp_decode(ctx, q.cuda(), w.cuda(), k8.cuda(), sc.float().cuda(),
                          torch.tensor(lens, dtype=torch.int32).cuda(), k, idx)
    ctx.sync_status()
    got = idx.cpu().numpy()
    unique_kth = 0
    for b in range(B):
        n = lens[b]
        ref = oracle.decode_scores(f32(q[b]), f32(w[b]), k8[b].numpy(), sc[b].float().numpy(), S=n)
        assert got[b].tolist() == oracle.topk_row(ref, k).tolist(), b
        kth = np.sort(ref)[::-1][k - 1]
        unique_kth += int(np.sum(ref == kth) == 1)
    assert unique_kth >= 3


def test_decode_workload_sampled(ic, ctx):
    """Decode workload shapes (32 sequences x 65537 candidates, H_I=64,
    k=2048): one F layer, 6 sequences checked against the oracle."""
    cfg = synth.CONFIGS["decode"]
    lay = synth.decode_layer(cfg, 0, "cuda")
    B, k = cfg.B, cfg.k
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    ic.ic_index_fp_decode(ctx, lay["q"], lay["w"], lay["kI8"], lay["kI_scale"], lay["seq_len"], k,
                          idx)
    ctx.sync_status()
    got = idx.cpu().numpy()
    for b in [0, 1, 15, 30, 31]:
        ref = oracle.decode_scores(f32(lay["q"][b]), f32(lay["w"][b]), lay["kI8"][b].cpu().numpy(),
                                   lay["kI_scale"][b].cpu().numpy())
        kth = oracle.kth_score(ref, k)
        sel = got[b]
        assert np.all(np.diff(sel) > 0)
        assert ref[sel].min() >= kth - SEL_RTOL * abs(kth)


def test_decode_stack(ic, ctx):
    """Decode F/S stack through ic_run_stack: snapshots obey the reuse rule,
    F-layer selections and every layer's attention match the oracle."""
    cfg = synth.DecodeConfig("small_decode", 3, 4999, "FSSFS", 64, 128, 256, 16, 128, 9)
    B, S, k = cfg.B, cfg.S, cfg.k
    layers, olay = [], []
    for l in range(cfg.n_layers):
        lay = synth.decode_layer(cfg, l, "cuda")
        lay["out"] = torch.empty((B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        lay["idx_snapshot"] = torch.empty((B, k), dtype=torch.int32, device="cuda")
        layers.append(lay)
    seq_len = layers[0]["seq_len"]
    pat = ic.ic_create_pattern(cfg.pattern)
    dims = ic.stack_dims(ic.IC_DECODE, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, B=B, S_max=S,
                         seq_len=seq_len)
    cache = torch.empty((B, k), dtype=torch.int32, device="cuda")
    ic.ic_run_stack(ctx, pat, layers, dims, cache)
    ctx.sync_status()
    src = oracle.pattern_src(cfg.pattern)
    snaps = [lay["idx_snapshot"].cpu().numpy() for lay in layers]
    for l in range(cfg.n_layers):
        assert np.array_equal(snaps[l], snaps[src[l]])
        lay = layers[l]
        if cfg.pattern[l] == "F":
            for b in range(B):
                ref = oracle.decode_scores(f32(lay["q"][b]), f32(lay["w"][b]),
                                           lay["kI8"][b].cpu().numpy(),
                                           lay["kI_scale"][b].cpu().numpy())
                kth = oracle.kth_score(ref, k)
                assert ref[snaps[l][b]].min() >= kth - SEL_RTOL * abs(kth)
        got = lay["out"].float().cpu().numpy().astype(np.float64)
        attn_check.check(got, f32(lay["Q"]), f32(lay["K"]), f32(lay["V"]), snaps[l],
                                     rows_per_seq=1)


def test_decode_every_e4m3_byte_exact(ic, ctx):
    """Each key row holds one nonzero e4m3 byte b at position j < 32; heads
    0..31 read +k[j] (q = e_j, w = 1) and heads 32..63 read -k[j] (q = -e_j,
    w = 0.5), so the score is k[j] for k[j] > 0 and 0.5*|k[j]| otherwise —
    exact in fp32.  Rows cover all 254 finite byte values (subnormals and
    both signs) at every position: the widening to bf16 must be exact."""
    B, S = 1, 254 * 32
    vals = [b for b in range(256) if b not in (0x7F, 0xFF)]
    k8 = torch.zeros((B, S, 128), dtype=torch.uint8)
    s = 0
    for j in range(32):
        for b in vals:
            k8[0, s, j] = b
            s += 1
    q = torch.zeros((B, 64, 128))
    for h in range(32):
        q[0, h, h] = 1.0
        q[0, 32 + h, h] = -1.0
    w = torch.tensor([[1.0] * 32 + [0.5] * 32])
    sc = torch.full((B, S), 2.0)
    lens = torch.tensor([S], dtype=torch.int32)
    q, w = q.bfloat16(), w.bfloat16()
    out = torch.zeros((B, S), device="cuda")
    ic.ic_index_score_decode(ctx, q.cuda(), w.cuda(), k8.cuda(), sc.cuda(), lens.cuda(), out)
    ctx.sync_status()
    ref = oracle.decode_scores(f32(q[0]), f32(w[0]), k8[0].numpy(), sc[0].numpy())
    assert np.array_equal(out.cpu().numpy()[0].astype(np.float64), ref)


def test_decode_stack_programmatic_launch_matches(ic, ctx):
    """A small-batch decode stack launches its kernels as programmatic
    dependents (an S layer's attention reads the index cache and prefetches
    its K/V rows before waiting for the previous kernel).  Index snapshots
    put a copy between kernels and so break those overlaps: the same stack
    run without snapshots, back to back, must produce bit-identical outputs
    to the run with them, and its S-layer attention must match the oracle."""
    cfg = synth.DecodeConfig("pdl_decode", 4, 6000, "FSSSFSSS", 64, 128, 512, 16, 128, 31)
    B, S, k = cfg.B, cfg.S, cfg.k
    assert B * 8 <= 148  # the stack uses programmatic launches at this batch
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.decode_layer(cfg, l, "cuda")
        lay["out"] = torch.empty((B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        layers.append(lay)
    seq_len = layers[0]["seq_len"]
    seq_len.copy_(torch.tensor([6001, 4097, 513, 2], dtype=torch.int32))
    pat = ic.ic_create_pattern(cfg.pattern)
    dims = ic.stack_dims(ic.IC_DECODE, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, B=B, S_max=S,
                         seq_len=seq_len)
    cache = torch.empty((B, k), dtype=torch.int32, device="cuda")
    snaps = [torch.empty((B, k), dtype=torch.int32, device="cuda") for _ in range(cfg.n_layers)]
    for lay, sn in zip(layers, snaps):
        lay["idx_snapshot"] = sn
    ic.ic_run_stack(ctx, pat, layers, dims, cache)
    ctx.sync_status()
    with_snap = [lay["out"].clone() for lay in layers]
    for lay in layers:
        del lay["idx_snapshot"]
    for _ in range(3):
        for lay in layers:
            lay["out"].zero_()
        ic.ic_run_stack(ctx, pat, layers, dims, cache)
        ctx.sync_status()
        for l in range(cfg.n_layers):
            assert torch.equal(layers[l]["out"], with_snap[l]), l
    s_idx = snaps[7].cpu().numpy()  # layer 7 (S) attends with layer 4's indices
    lay = layers[7]
    got = lay["out"].float().cpu().numpy().astype(np.float64)
    attn_check.check(got, f32(lay["Q"]), f32(lay["K"]), f32(lay["V"]), s_idx, rows_per_seq=1)


def test_decode_stack_cross_layer_prefetch_matches(ic, ctx):
    """A decode stack of a batch too large for programmatic launches
    (B * 8 > SMs): an attention layer followed by an S layer warms L2 with
    that layer's K/V rows at the shared index slots.  A prefetch changes no
    value, so every layer's output must equal a standalone ic_sparse_attn call
    on the same indices bit for bit, and an S layer must match the oracle."""
    cfg = synth.DecodeConfig("wide_decode", 24, 3000, "FSSSFS", 64, 128, 512, 16, 128, 37)
    B, S, k = cfg.B, cfg.S, cfg.k
    assert B * 8 > 148  # no programmatic launches: the cross-layer prefetch runs
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.decode_layer(cfg, l, "cuda")
        lay["out"] = torch.empty((B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        layers.append(lay)
    seq_len = layers[0]["seq_len"]
    pat = ic.ic_create_pattern(cfg.pattern)
    dims = ic.stack_dims(ic.IC_DECODE, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, B=B, S_max=S,
                         seq_len=seq_len)
    cache = torch.empty((B, k), dtype=torch.int32, device="cuda")
    snaps = [torch.empty((B, k), dtype=torch.int32, device="cuda") for _ in range(cfg.n_layers)]
    for lay, sn in zip(layers, snaps):
        lay["idx_snapshot"] = sn
    ic.ic_run_stack(ctx, pat, layers, dims, cache)
    ctx.sync_status()
    for l in range(cfg.n_layers):
        lay = layers[l]
        alone = torch.empty_like(lay["out"])
        ic.ic_sparse_attn(ctx, lay["Q"], lay["K"], lay["V"], snaps[l], alone, rows_per_seq=1,
                          kv_seq_stride=S * cfg.d, kv_len=S)
        ctx.sync_status()
        assert torch.equal(lay["out"], alone), l
    lay = layers[3]  # an S layer after an S layer: both had their rows prefetched
    got = lay["out"].float().cpu().numpy().astype(np.float64)
    attn_check.check(got, f32(lay["Q"]), f32(lay["K"]), f32(lay["V"]),
                                 snaps[3].cpu().numpy(), rows_per_seq=1)
