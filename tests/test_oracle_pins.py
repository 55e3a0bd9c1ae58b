"""Pins of the CPU oracle against values and facts fixed outside it.

Each test ties one oracle function to something other than its own code:
values the pages print (tests/golden), hand-worked examples, closed forms,
library routines (torch SDPA, numpy stable sort, torch's FP8 cast),
exhaustive search on tiny inputs, and invariants of the definitions.  A
plausible slip in the oracle (dropped ReLU, transposed q/k, wrong head of w,
wrong tie rule, sign error, unsorted output) fails at least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle


# ----------------------------------------------------------------- pattern
def test_fs_walkthrough(golden):
    g = golden["fs_walkthrough"]
    assert oracle.pattern_src(g["pattern"]).tolist() == g["src"]
    # layers 1..5 (1-based) of the walk-through
    assert [s + 1 for s in oracle.pattern_src(g["pattern"])[:5]] == g["src_1based_for_layers_1_to_5"]


def test_uniform_pattern(golden):
    g = golden["uniform_r4"]
    assert oracle.pattern_uniform(g["n"], g["r"]) == g["pattern"]
    assert oracle.pattern_uniform(47, 1) == "F" * 47
    assert oracle.pattern_uniform(47, 8).count("F") == 6


def test_appendix_b_patterns(golden):
    for p in golden["appendix_b_patterns"]["patterns"]:
        c = p["c"]
        assert len(c) == p["layers"]
        src = oracle.pattern_src(c)
        num, den = map(int, p["retention"].split("/"))
        # retention r keeps about N*r indexers (the searched 78-layer 1/4
        # pattern has 22 F layers against 19.5)
        assert abs(c.count("F") - len(c) * num / den) <= 3
        for l, ch in enumerate(c):
            assert c[src[l]] == "F"
            assert src[l] <= l
            assert "F" not in c[src[l] + 1:l + 1] if ch == "S" else src[l] == l


def test_searched_patterns_in_the_sweep_match_the_pages(golden):
    """The decode sweep's searched patterns are the printed 47-layer ones."""
    from cross_layer_top_b200 import synth
    printed = {p["retention"]: p["c"] for p in golden["appendix_b_patterns"]["patterns"]
               if p["layers"] == 47}
    assert synth.SEARCHED_PATTERNS_47 == printed
    assert [c.count("F") for c in synth.SEARCHED_PATTERNS_47.values()] == [24, 12, 7]


@pytest.mark.parametrize("bad", ["", "SFFF", "FSXS", "fsss", "S"])
def test_pattern_rejects(bad):
    with pytest.raises(ValueError):
        oracle.pattern_src(bad)


# ------------------------------------------------------------------ scores
def test_hand_scores(golden):
    g = golden["hand_scores"]
    I = oracle.index_scores(np.array(g["q"]), np.array(g["k"]), np.array(g["w"]))
    for t, row in enumerate(g["I"]):
        assert I[t, :t + 1].tolist() == row
        assert np.all(np.isnan(I[t, t + 1:]))
    for t in range(3):
        assert oracle.topk_row(I[t, :t + 1], 2).tolist() == g["top2"][t]
        assert oracle.topk_row(I[t, :t + 1], 1).tolist() == g["top1"][t]


def test_scores_single_head_closed_form():
    # H = 1, d = 1, w = 1: I[t,s] = max(q_t * k_s, 0) -- an outer product
    rng = np.random.default_rng(1)
    L = 17
    q = rng.integers(-5, 6, (L, 1, 1)).astype(np.float32)
    k = rng.integers(-5, 6, (L, 1)).astype(np.float32)
    w = np.ones((L, 1), np.float32)
    I = oracle.index_scores(q, k, w)
    ref = np.maximum(np.outer(q[:, 0, 0], k[:, 0]), 0.0)
    tri = np.tril(np.ones((L, L), bool))
    assert np.array_equal(I[tri], ref[tri])
    assert not np.array_equal(ref, ref.T)  # the case distinguishes q_t k_s from q_s k_t


def test_scores_unit_vector_heads():
    # q[t, j] = a_t * e_j  =>  q[t,j].k_s = a_t * k_s[j]
    rng = np.random.default_rng(2)
    L, H = 9, 4
    a = rng.integers(1, 4, L).astype(np.float32)
    q = np.zeros((L, H, H), np.float32)
    for t in range(L):
        q[t] = a[t] * np.eye(H)
    k = rng.integers(-3, 4, (L, H)).astype(np.float32)
    w = rng.choice([-1.0, -0.5, 0.5, 1.0], (L, H)).astype(np.float32)
    I = oracle.index_scores(q, k, w)
    for t in range(L):
        for s in range(t + 1):
            expect = sum(w[t, j] * max(a[t] * k[s, j], 0.0) for j in range(H))
            assert I[t, s] == expect


def test_scores_invariants():
    rng = np.random.default_rng(3)
    L, H, d = 33, 6, 8
    q = rng.standard_normal((L, H, d)).astype(np.float32)
    k = rng.standard_normal((L, d)).astype(np.float32)
    w1 = rng.standard_normal((L, H)).astype(np.float32)
    w2 = rng.standard_normal((L, H)).astype(np.float32)
    tri = np.tril(np.ones((L, L), bool))
    I1 = oracle.index_scores(q, k, w1)[tri]
    I2 = oracle.index_scores(q, k, w2)[tri]
    I12 = oracle.index_scores(q, k, (w1.astype(np.float64) + w2).astype(np.float32))[tri]
    # linear in w (w1+w2 is not exact in float32, so compare with tolerance)
    assert np.allclose(I12, I1 + I2, rtol=1e-6, atol=1e-5)
    # positively homogeneous in q (power-of-two scale keeps float32 exact)
    assert np.array_equal(oracle.index_scores(4 * q, k, w1)[tri], 4 * I1)
    # permuting heads of q and w together changes nothing
    perm = rng.permutation(H)
    Ip = oracle.index_scores(q[:, perm], k, w1[:, perm])[tri]
    assert np.allclose(Ip, I1, rtol=1e-12, atol=1e-12)
    # permuting only w's heads does change the scores (w is per head)
    assert not np.allclose(oracle.index_scores(q, k, w1[:, perm])[tri], I1)
    # ReLU: flipping q flips which heads are active; with w = 1, I(q) - I(-q) = sum_j q_j.k
    ones = np.ones((L, H), np.float32)
    Ipos = oracle.index_scores(q, k, ones)
    Ineg = oracle.index_scores(-q, k, ones)
    lin = np.einsum("thd,sd->ts", q.astype(np.float64), k.astype(np.float64))
    assert np.allclose((Ipos - Ineg)[tri], lin[tri], rtol=1e-9, atol=1e-9)
    # and I(q) + I(-q) = sum_j |q_j.k|
    absd = np.einsum("thd,sd->tsh", q.astype(np.float64), k.astype(np.float64))
    assert np.allclose((Ipos + Ineg)[tri], np.abs(absd).sum(-1)[tri], rtol=1e-9, atol=1e-9)


def test_scores_orthogonal_and_negative_weights():
    L, H, d = 8, 2, 4
    q = np.zeros((L, H, d), np.float32)
    q[:, :, 0] = 1.0
    k = np.zeros((L, d), np.float32)
    k[:, 1] = 3.0  # orthogonal to every q
    w = np.ones((L, H), np.float32)
    I = oracle.index_scores(q, k, w)
    tri = np.tril(np.ones((L, L), bool))
    assert np.all(I[tri] == 0.0)
    # all-negative weights: every score <= 0; top-k keeps the zero scores,
    # lowest indices first
    rng = np.random.default_rng(4)
    q = rng.integers(-2, 3, (L, H, d)).astype(np.float32)
    k = rng.integers(-2, 3, (L, d)).astype(np.float32)
    w = -np.ones((L, H), np.float32)
    I = oracle.index_scores(q, k, w)
    assert np.all(I[tri] <= 0)
    row = I[L - 1]
    zeros = [s for s in range(L) if row[s] == 0.0]
    assert oracle.topk_row(row, len(zeros)).tolist() == zeros


def test_scores_at_equals_scores_of_full_tensors():
    """index_scores_at (sampled rows given compactly) against index_scores on
    the whole tensors, bit for bit: Gaussian and integer inputs, unsorted
    and repeated positions.  A wrong row stride or pos[r] mixed up with r
    fails here."""
    rng = np.random.default_rng(17)
    L, H, d = 90, 3, 5
    for integer in (False, True):
        if integer:
            q = rng.integers(-3, 4, (L, H, d)).astype(np.float32)
            k = rng.integers(-3, 4, (L, d)).astype(np.float32)
            w = rng.choice([-1.0, -0.5, 0.5, 1.0], (L, H)).astype(np.float32)
        else:
            q = rng.standard_normal((L, H, d)).astype(np.float32)
            k = rng.standard_normal((L, d)).astype(np.float32)
            w = rng.standard_normal((L, H)).astype(np.float32)
        pos = np.array([57, 3, 89, 0, 57, 12, 44, 3], np.int32)  # unsorted, repeated
        full = oracle.index_scores(q, k, w, rows=pos)
        at = oracle.index_scores_at(q[pos], w[pos], k, pos)
        assert at.shape == (len(pos), 90)
        for r, t in enumerate(pos):
            assert np.array_equal(at[r, :t + 1], full[r, :t + 1])
            assert np.all(np.isnan(at[r, t + 1:]))


def test_scores_at_hand_case():
    """Two compact rows at positions 2 and 0 (H = 1, d = 2, w = [2] and
    [-1]) over keys k0 = (1, 0), k1 = (0, 1), k2 = (1, 1):
      row at t = 2, q = (1, -2): dots 1, -2, -1 -> 2*ReLU = 2, 0, 0
      row at t = 0, q = (3, 1):  dot 3            -> -1*3 = -3."""
    q_rows = np.array([[[1.0, -2.0]], [[3.0, 1.0]]], np.float32)
    w_rows = np.array([[2.0], [-1.0]], np.float32)
    k = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]], np.float32)
    out = oracle.index_scores_at(q_rows, w_rows, k, np.array([2, 0], np.int32))
    assert out[0].tolist() == [2.0, 0.0, 0.0]
    assert out[1, 0] == -3.0 and np.all(np.isnan(out[1, 1:]))


def test_integer_scores_are_exact_multiples_of_half():
    rng = np.random.default_rng(5)
    L, H, d = 64, 4, 32
    q = rng.integers(-3, 4, (L, H, d)).astype(np.float32)
    k = rng.integers(-3, 4, (L, d)).astype(np.float32)
    w = rng.choice([-1.0, -0.5, 0.5, 1.0], (L, H)).astype(np.float32)
    I = oracle.index_scores(q, k, w)
    tri = np.tril(np.ones((L, L), bool))
    v = I[tri]
    assert np.all(v * 2 == np.round(v * 2))
    assert np.max(np.abs(v)) <= H * d * 9


def _e4m3_int(v):
    """e4m3 byte of an integer with |v| <= 16."""
    v = int(v)
    if v == 0:
        return 0
    a = abs(v)
    e = a.bit_length() - 1
    m = (a - (1 << e)) * 8 >> e
    return (0x80 if v < 0 else 0) | ((e + 7) << 3) | m


def test_fp8_scores_hand_example():
    # q = [1.5, -2] * 2 = [3, -4]; k0 = [2, 0.5] * 0.5 = [1, 0.25]; k1 = [-2, 1] * 1
    q8 = np.array([[[0x3C, 0xC0]], [[0x3C, 0xC0]]], np.uint8)
    q_scale = np.array([[2.0], [2.0]], np.float32)
    k8 = np.array([[0x40, 0x30], [0xC0, 0x38]], np.uint8)
    k_scale = np.array([0.5, 1.0], np.float32)
    w = np.array([[0.5], [0.5]], np.float32)
    I = oracle.index_scores_fp8(q8, q_scale, k8, k_scale, w)
    assert I[0, 0] == 0.5 * (3 * 1 - 4 * 0.25)      # 1.0
    assert I[1, 0] == 1.0
    assert I[1, 1] == 0.0                          # 3*-2 - 4*1 < 0: ReLU
    assert np.isnan(I[0, 1])


def test_fp8_scores_equal_bf16_scores_on_integer_values():
    rng = np.random.default_rng(12)
    L, H, d = 21, 4, 16
    qi = rng.integers(-16, 17, (L, H, d))
    ki = rng.integers(-16, 17, (L, d))
    w = rng.choice([-1.0, -0.5, 0.5, 1.0], (L, H)).astype(np.float32)
    enc = np.vectorize(_e4m3_int)
    I8 = oracle.index_scores_fp8(enc(qi).astype(np.uint8), np.ones((L, H), np.float32),
                                 enc(ki).astype(np.uint8), np.ones(L, np.float32), w)
    I16 = oracle.index_scores(qi.astype(np.float32), ki.astype(np.float32), w)
    tri = np.tril(np.ones((L, L), bool))
    assert np.array_equal(I8[tri], I16[tri])


def test_fp8_scores_scale_laws():
    rng = np.random.default_rng(13)
    L, H, d = 17, 3, 8
    q8 = rng.integers(0, 0x7E, (L, H, d)).astype(np.uint8) | (rng.integers(0, 2, (L, H, d)) << 7).astype(np.uint8)
    k8 = rng.integers(0, 0x7E, (L, d)).astype(np.uint8)
    qs = rng.uniform(0.5, 2.0, (L, H)).astype(np.float32)
    ks = rng.uniform(0.5, 2.0, L).astype(np.float32)
    w = rng.standard_normal((L, H)).astype(np.float32)
    I = oracle.index_scores_fp8(q8, qs, k8, ks, w)
    tri = np.tril(np.ones((L, L), bool))
    # a key's scale multiplies its column (power of two: exact)
    ks2 = ks.copy()
    ks2[5] *= 4
    I2 = oracle.index_scores_fp8(q8, qs, k8, ks2, w)
    assert np.array_equal(I2[5:, 5], 4 * I[5:, 5])
    assert np.array_equal(np.delete(I2, 5, axis=1)[np.delete(tri, 5, axis=1)],
                          np.delete(I, 5, axis=1)[np.delete(tri, 5, axis=1)])
    # a query head's scale and its weight are interchangeable (both > 0 factors)
    qs3, w3 = qs.copy(), w.copy()
    qs3[:, 1] *= 2
    w3[:, 1] *= 2
    A = oracle.index_scores_fp8(q8, qs3, k8, ks, w)
    B = oracle.index_scores_fp8(q8, qs, k8, ks, w3)
    assert np.allclose(A[tri], B[tri], rtol=1e-12, atol=1e-12)
    assert not np.allclose(A[tri], I[tri])


# ------------------------------------------------------------------- top-k
def test_topk_page_toy(golden):
    g = golden["topk_average_toy"]
    assert oracle.topk_row(g["scores"], 1).tolist() == g["top1"]
    assert oracle.topk_row(g["scores"], 2).tolist() == g["top2"]


def _brute_topk(score, k):
    """Exhaustive search: the unique k-subset S such that every member beats
    every non-member under (score desc, index asc)."""
    n = len(score)
    m = min(n, k)
    found = []
    for sub in itertools.combinations(range(n), m):
        rest = [b for b in range(n) if b not in sub]
        if all(score[a] > score[b] or (score[a] == score[b] and a < b) for a in sub for b in rest):
            found.append(list(sub))
    assert len(found) == 1
    return found[0] + [-1] * (k - m)


def test_topk_bruteforce_tiny():
    rng = np.random.default_rng(6)
    for trial in range(300):
        n = int(rng.integers(1, 9))
        k = int(rng.integers(1, 10))
        score = rng.integers(-2, 3, n).astype(np.float64)  # many ties
        if trial % 3 == 0:
            score = rng.standard_normal(n)
        assert oracle.topk_row(score, k).tolist() == _brute_topk(score.tolist(), k)


def test_topk_matches_stable_argsort():
    rng = np.random.default_rng(7)
    for n, k in [(100, 10), (5000, 2048), (2048, 2048), (3000, 64), (10, 64)]:
        score = np.round(rng.standard_normal(n) * 4) / 4  # ties
        ref = np.sort(np.argsort(-score, kind="stable")[:k])
        got = oracle.topk_row(score, k)
        m = min(n, k)
        assert got[:m].tolist() == ref.tolist()
        assert np.all(got[m:] == -1)


def test_topk_invariants_and_degenerate():
    rng = np.random.default_rng(8)
    n, k = 777, 64
    score = rng.integers(-3, 4, n).astype(np.float64)
    T = oracle.topk_row(score, k)
    assert len(set(T.tolist())) == k and np.all(np.diff(T) > 0) and T.max() < n
    sel = set(T.tolist())
    mn = min(score[s] for s in sel)
    last_tied = max(s for s in sel if score[s] == mn)
    for s in range(n):
        if s not in sel:
            assert score[s] < mn or (score[s] == mn and s > last_tied)
    # all equal -> first k indices; k >= n -> everything then -1
    assert oracle.topk_row(np.zeros(100), 7).tolist() == list(range(7))
    assert oracle.topk_row(np.ones(5), 8).tolist() == [0, 1, 2, 3, 4, -1, -1, -1]
    assert oracle.kth_score(np.array([3.0, 1.0, 2.0]), 2) == 2.0


# -------------------------------------------------------------------- FP8
def test_e4m3_decode_matches_torch_cast(golden):
    allb = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_to_float64(allb)
    ref = torch.from_numpy(allb).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2
    assert np.array_equal(mine[~nan], ref[~nan])
    for hexs, val in golden["e4m3_bytes"]["pairs"]:
        assert oracle.e4m3_to_float64(np.array([int(hexs, 16)]))[0] == val


def test_decode_scores_closed_form():
    # H = 1, d = 1, w = 1: I[s] = max(q * e4m3(b_s) * scale_s, 0)
    kq = np.array([[0x38], [0x40], [0xB8], [0x01], [0x7E]], np.uint8)
    sc = np.array([1.0, 0.5, 2.0, 4.0, 0.25], np.float32)
    q = np.array([[3.0]], np.float32)
    w = np.array([1.0], np.float32)
    got = oracle.decode_scores(q, w, kq, sc)
    assert got.tolist() == [3.0, 3.0, 0.0, 3.0 * 2 ** -9 * 4, 3.0 * 448 * 0.25]
    # two heads with opposite q: w=(1,1) gives |q.k|
    q2 = np.array([[1.5], [-1.5]], np.float32)
    got2 = oracle.decode_scores(q2, np.array([1.0, 1.0], np.float32), kq, sc)
    vals = [1.0 * 1.0, 2.0 * 0.5, -1.0 * 2.0, 2 ** -9 * 4.0, 448 * 0.25]
    assert np.allclose(got2, [1.5 * abs(v) for v in vals], rtol=0, atol=0)


# --------------------------------------------------------------- attention
def test_hand_attention(golden):
    g = golden["hand_attention"]
    for case in g["cases"]:
        out = oracle.sparse_attn(np.array(g["Q"]), np.array(g["K"]), np.array(g["V"]),
                                 np.array([case["idx"]]), rows=[0], scale=1.0)
        assert np.allclose(out[0, 0], case["out"], rtol=0, atol=1e-13)


def test_attention_full_set_equals_sdpa_causal():
    # with k >= t+1 every causal position is selected: sparse attention is
    # ordinary causal softmax attention (torch SDPA in fp64, a library routine)
    rng = np.random.default_rng(9)
    L, Hq, d, k = 40, 3, 16, 64
    Q = rng.standard_normal((L, Hq, d)).astype(np.float32)
    K = rng.standard_normal((L, d)).astype(np.float32)
    V = rng.standard_normal((L, d)).astype(np.float32)
    idx = np.full((L, k), -1, np.int32)
    for t in range(L):
        idx[t, :t + 1] = np.arange(t + 1)
    got = oracle.sparse_attn(Q, K, V, idx)
    q = torch.from_numpy(Q.astype(np.float64)).permute(1, 0, 2)       # [Hq, L, d]
    kk = torch.from_numpy(K.astype(np.float64))[None].expand(Hq, L, d)
    vv = torch.from_numpy(V.astype(np.float64))[None].expand(Hq, L, d)
    ref = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, is_causal=True)
    assert np.allclose(got, ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


def test_attention_invariants():
    rng = np.random.default_rng(10)
    S, Hq, d = 50, 4, 8
    Q = rng.standard_normal((1, Hq, d)).astype(np.float32)
    K = rng.standard_normal((S, d)).astype(np.float32)
    V = rng.standard_normal((S, d)).astype(np.float32)
    idx = np.array([[3, 7, 11, 20, 49, -1, 5]], np.int32)
    base = oracle.sparse_attn(Q, K, V, idx)
    # order of the index list and -1 entries do not matter
    perm = np.array([[49, -1, 5, 11, 3, 20, 7]], np.int32)
    assert np.allclose(oracle.sparse_attn(Q, K, V, perm), base, rtol=1e-13, atol=1e-14)
    # uniform V rows -> output equals that row
    Vu = np.tile(V[:1], (S, 1))
    assert np.allclose(oracle.sparse_attn(Q, K, Vu, idx)[0], np.tile(V[0], (Hq, 1)), atol=1e-14)
    # a single selected key -> its V row
    one = np.array([[-1, 17, -1]], np.int32)
    assert np.allclose(oracle.sparse_attn(Q, K, V, one)[0], np.tile(V[17], (Hq, 1)), atol=0)
    # scaling Q by c and the softmax scale by 1/c changes nothing
    a = oracle.sparse_attn(Q, K, V, idx, scale=0.25)
    b = oracle.sparse_attn(4 * Q, K, V, idx, scale=1 / 16)
    assert np.allclose(a, b, rtol=1e-13, atol=1e-14)
    # the result is a convex combination of the selected V rows
    sel = V[[3, 7, 11, 20, 49, 5]]
    assert np.all(base[0] <= sel.max(0) + 1e-12) and np.all(base[0] >= sel.min(0) - 1e-12)


def test_attention_batched_sequences():
    # rows_per_seq = 1 with [B, S, d] K/V: row b attends to sequence b only
    rng = np.random.default_rng(11)
    B, S, Hq, d = 3, 20, 2, 8
    Q = rng.standard_normal((B, Hq, d)).astype(np.float32)
    K = rng.standard_normal((B, S, d)).astype(np.float32)
    V = rng.standard_normal((B, S, d)).astype(np.float32)
    idx = np.array([[0, 5, 19], [1, 2, -1], [7, 8, 9]], np.int32)
    got = oracle.sparse_attn(Q, K, V, idx, rows_per_seq=1)
    for b in range(B):
        one = oracle.sparse_attn(Q[b:b + 1], K[b], V[b], idx[b:b + 1])
        assert np.array_equal(got[b], one[0])


# ------------------------------------------------------------ stack / misc
def test_attn_weight_spread_closed_forms():
    """sqrt(sum_s p_s^2 V[s]^2) with the softmax weights of sparse_attn:
      * equal logits (Q = 0) give p_s = 1/n: sqrt(sum_s V[s]^2) / n;
      * one key gives |V[s]|;
      * two keys with logits 0 and -g (scale 1): p = (1, e^-g)/(1 + e^-g),
        so sqrt(V_a^2 + e^-2g V_b^2) / (1 + e^-g)."""
    rng = np.random.default_rng(3)
    K = rng.standard_normal((20, 4)).astype(np.float32)
    V = rng.standard_normal((20, 4)).astype(np.float32)
    sel = np.array([[4, 9, -1, 13, 2, -1]], np.int32)
    sp = oracle.attn_weight_spread(np.zeros((1, 2, 4), np.float32), K, V, sel)
    want = np.sqrt((V[[4, 9, 13, 2]].astype(np.float64) ** 2).sum(0)) / 4
    assert np.allclose(sp[0, 0], want, rtol=1e-12) and np.allclose(sp[0, 1], want, rtol=1e-12)
    one = oracle.attn_weight_spread(rng.standard_normal((1, 3, 4)).astype(np.float32), K, V,
                                    np.array([[-1, 7, -1]], np.int32))
    assert np.allclose(one[0], np.abs(V[7].astype(np.float64))[None, :], rtol=1e-12)
    # two keys: K rows e0 and e1, Q = (0, -g): logits 0 and -g
    g = 1.5
    K2 = np.eye(4, dtype=np.float32)
    Q2 = np.array([[[0.0, -g, 0.0, 0.0]]], np.float32)
    V2 = rng.standard_normal((4, 4)).astype(np.float32)
    sp2 = oracle.attn_weight_spread(Q2, K2, V2, np.array([[0, 1]], np.int32), scale=1.0)
    e = math.exp(-g)
    want2 = np.sqrt(V2[0].astype(np.float64) ** 2 + e * e * V2[1].astype(np.float64) ** 2) / (1 + e)
    assert np.allclose(sp2[0, 0], want2, rtol=1e-12)


def test_overlap_page_toy(golden):
    g = golden["overlap_toy"]
    assert oracle.overlap(g["a"], g["b"]) == g["overlap"]


def test_overlap_against_set_intersection():
    """The pairwise search equals a hash-set intersection on rows without
    repeats; a row against itself counts its selected entries, disjoint rows
    count nothing."""
    rng = np.random.default_rng(4)
    k = 97
    for _ in range(20):
        na, nb = rng.integers(0, k + 1, 2)
        pool = rng.permutation(150)
        a = np.full(k, -1, np.int32)
        b = np.full(k, -1, np.int32)
        a[rng.permutation(k)[:na]] = pool[:na]
        b[rng.permutation(k)[:nb]] = rng.permutation(pool[:120])[:nb]
        expect = len(set(a[a >= 0].tolist()) & set(b[b >= 0].tolist()))
        assert round(oracle.overlap(a, b) * k) == expect  # the ratio, scaled back to a count
        assert round(oracle.overlap(a, a) * k) == na
    assert oracle.overlap(np.arange(10), np.arange(10, 20)) == 0.0


def test_stack_reuse_invariant():
    rng = np.random.default_rng(12)
    L, H, d, Hq, dv, k = 48, 2, 8, 2, 8, 8
    pattern = "FSSFS"
    layers = []
    for c in pattern:
        lay = {"Q": rng.standard_normal((L, Hq, dv)).astype(np.float32),
               "K": rng.standard_normal((L, dv)).astype(np.float32),
               "V": rng.standard_normal((L, dv)).astype(np.float32)}
        if c == "F":
            lay.update(qI=rng.integers(-3, 4, (L, H, d)).astype(np.float32),
                       kI=rng.integers(-3, 4, (L, d)).astype(np.float32),
                       w=rng.choice([-1.0, 1.0], (L, H)).astype(np.float32))
        layers.append(lay)
    idx, outs = oracle.run_stack(pattern, layers, k)
    src = oracle.pattern_src(pattern)
    for l in range(len(pattern)):
        assert np.array_equal(idx[l], idx[src[l]])
    assert not np.array_equal(idx[0], idx[3])  # layer 3 ran its own indexer
    # rows t < k select everything up to t
    for t in range(k):
        assert idx[0][t].tolist() == list(range(t + 1)) + [-1] * (k - t - 1)
    # S layers attend with their own Q/K/V: outputs differ across layers
    assert not np.allclose(outs[1], outs[2])
