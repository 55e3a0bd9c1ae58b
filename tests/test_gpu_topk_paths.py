"""The top-k kernels' branches, each forced by a constructed row and
checked bit-exact against the oracle's top-k (positions of the k largest,
ascending, ties to the lower position).

The row kernel comes in two shapes, chosen by the longest row of a launch
(16 warps and 4096 candidate slots above 32768 keys, 8 warps and 2048 slots
up to it); a launch of few long rows with given lengths takes the cluster
form instead.  Each set of rows runs in the launch shape that reaches the
intended kernel, padded with Gaussian rows of assorted lengths where the
row kernel needs more rows than the cluster form takes (every row checked):
  - the bitmap path on Gaussian rows, including one at the bitmap's
    capacity (131072 keys) and one at the short shape's limit (32768), and
    one tie at T taken whole;
  - the general path: a row longer than the bitmap holds, a candidate bin
    larger than the candidate list, a warp slice that overflows, and a tie
    at T that is split by position;
  - rows of at most k keys (all taken, -1 padding);
  - rows whose threshold lies among signed zeros and denormals (the first
    digit's bins 1023 and 1024)."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

K = 2048


@pytest.fixture(scope="module")
def ic():
    from cross_layer_top_b200 import indexcache
    return indexcache


def _long_rows():
    """Rows for the long-row shape (and the cluster form): 4096 slots, and
    a warp's slice of 256 slots over segments of n / 16 keys."""
    rng = np.random.default_rng(2024)
    rows = {}
    rows["gauss_20000"] = rng.standard_normal(20000)
    rows.update(_zero_threshold_rows(rng, 40000))
    rows["gauss_at_bitmap_cap"] = rng.standard_normal(131072)
    rows["longer_than_bitmap"] = rng.standard_normal(140000)
    # 1000 keys far above, then 5000 keys in [1.0, 1.25) (one 11-bit bin), the rest below:
    # the threshold bin holds more keys than the candidate list
    r = np.full(20000, -1.0) - rng.random(20000)
    r[rng.permutation(20000)[:1000]] = 100.0 + rng.random(1000)
    free = np.flatnonzero(r < 0)
    r[rng.permutation(free)[:5000]] = 1.0 + 0.25 * rng.random(5000)
    rows["bin_over_list"] = r
    # the same, 3000 threshold-bin keys packed at the start (first warp's segment)
    r = np.full(20000, -1.0) - rng.random(20000)
    r[:3000] = 1.0 + 0.25 * rng.random(3000)
    r[3000 + rng.permutation(17000)[:1000]] = 100.0 + rng.random(1000)
    rows["slice_overflow"] = r
    # 2045 keys above 10, the k-th value 5.0 three times (all taken), the rest below
    r = -rng.random(9000)
    pos = rng.permutation(9000)
    r[pos[:2045]] = 10.0 + rng.random(2045)
    r[pos[2045:2048]] = 5.0
    rows["tie_taken_whole"] = r
    # the same with 5.0 six times: three taken, the lowest positions
    r = -rng.random(9000)
    pos = rng.permutation(9000)
    r[pos[:2045]] = 10.0 + rng.random(2045)
    r[pos[2045:2051]] = 5.0
    rows["tie_split"] = r
    return {n: v.astype(np.float32) for n, v in rows.items()}


def _zero_threshold_rows(rng, n):
    """Rows whose k-th largest score lies in the bins around zero (key bins
    1023 and 1024): signed zeros and denormals, where the first digit counted
    on raw float bits differs from the order keys (-0.0) and the kernel
    counts again."""
    tiny = np.float32(1e-42)  # a denormal
    # the k-th largest is 0: 1000 positives, 3000 zeros of both signs, negatives
    r = np.concatenate([rng.random(1000) + 1.0, np.zeros(3000), -(rng.random(n - 4000) + 1.0)])
    r = rng.permutation(r).astype(np.float32)
    r[rng.permutation(np.flatnonzero(r == 0))[:1500]] = np.float32(-0.0)
    rows = {"threshold_at_zero": r}
    # the k-th largest is a negative denormal: 1000 positives, 500 zeros, 2000
    # negative denormals, negatives
    r = np.concatenate([rng.random(1000) + 1.0, np.zeros(500),
                        -tiny * (1 + rng.integers(0, 50, 2000)), -(rng.random(n - 3500) + 1.0)])
    rows["threshold_negative_denormal"] = rng.permutation(r).astype(np.float32)
    # the k-th largest is a positive denormal, next to -0.0 keys
    r = np.concatenate([rng.random(1000) + 1.0, tiny * (1 + rng.integers(0, 50, 2000)),
                        np.full(1000, -0.0), -(rng.random(n - 4000) + 1.0)])
    rows["threshold_positive_denormal"] = rng.permutation(r).astype(np.float32)
    return rows


def _short_rows():
    """Rows for the short-row shape: 2048 slots, and a warp's slice of 256
    slots over segments of n / 8 keys (2560 keys at n = 20000)."""
    rng = np.random.default_rng(2025)
    rows = {}
    rows["gauss_16384"] = rng.standard_normal(16384)
    rows.update(_zero_threshold_rows(rng, 9000))
    rows["gauss_at_short_limit"] = rng.standard_normal(32768)
    rows["gauss_2049"] = rng.standard_normal(2049)
    rows["few_keys"] = rng.standard_normal(700)
    # 1000 keys far above, 2500 keys in [1.0, 1.25) (one 11-bit bin): more
    # than the list's 2048 slots
    r = np.full(20000, -1.0) - rng.random(20000)
    r[rng.permutation(20000)[:1000]] = 100.0 + rng.random(1000)
    free = np.flatnonzero(r < 0)
    r[rng.permutation(free)[:2500]] = 1.0 + 0.25 * rng.random(2500)
    rows["bin_over_list"] = r
    # 1500 keys far above, 1000 threshold-bin keys packed at the start: they
    # fit the list but not the first warp's slice
    r = np.full(20000, -1.0) - rng.random(20000)
    r[:1000] = 1.0 + 0.25 * rng.random(1000)
    r[1000 + rng.permutation(19000)[:1500]] = 100.0 + rng.random(1500)
    rows["slice_overflow"] = r
    # 2045 keys above 10, then the k-th value 5.0 three times (all taken) or
    # six times (three taken, the lowest positions)
    for name, ties in (("tie_taken_whole", 3), ("tie_split", 6)):
        r = -rng.random(9000)
        pos = rng.permutation(9000)
        r[pos[:2045]] = 10.0 + rng.random(2045)
        r[pos[2045:2045 + ties]] = 5.0
        rows[name] = r
    return {n: v.astype(np.float32) for n, v in rows.items()}


def _check_launch(ic, rows, min_rows, filler_max, seed):
    """One ic_topk launch over `rows` (padded to min_rows with Gaussian
    rows of up to filler_max keys), every row compared with the oracle."""
    rng = np.random.default_rng(seed)
    rows = dict(rows)
    i = 0
    while len(rows) < min_rows:
        rows["filler_%d" % i] = rng.standard_normal(int(rng.integers(1, filler_max + 1))).astype(np.float32)
        i += 1
    names = list(rows)
    ld = (max(len(v) for v in rows.values()) + 3) // 4 * 4
    sc = torch.full((len(names), ld), -1e30, dtype=torch.float32)
    for i, n in enumerate(names):
        sc[i, :len(rows[n])] = torch.from_numpy(rows[n])
    lens = torch.tensor([len(rows[n]) for n in names], dtype=torch.int32)
    ctx = ic.Context(0)
    idx = torch.empty((len(names), K), dtype=torch.int32, device="cuda")
    ic.ic_topk(ctx, sc.cuda(), K, idx, row_len=lens.cuda(), ld=ld)
    ctx.sync_status()
    got = idx.cpu().numpy()
    for i, n in enumerate(names):
        want = oracle.topk_row(rows[n].astype(np.float64), K)
        assert got[i].tolist() == want.tolist(), n
    ctx.close()
    return ld


# rows * 8 CTAs above 4 per SM of a 148-SM part (and of any up to 192 SMs):
# the launch cannot take the cluster form
ROW_KERNEL_ROWS = 97


def test_topk_cluster_form_every_path_bit_exact(ic):
    """The constructed long rows alone: seven rows of up to 140000 keys
    with given lengths take the cluster form."""
    _check_launch(ic, _long_rows(), 0, 0, 0)


def test_topk_long_row_kernel_every_path_bit_exact(ic):
    """The same rows among 97: the row kernel's long-row shape."""
    ld = _check_launch(ic, _long_rows(), ROW_KERNEL_ROWS, 140000, 1)
    assert ld > 32768


def test_topk_short_row_kernel_every_path_bit_exact(ic):
    """Rows of at most 32768 keys among 97: the short-row shape, at its
    limit."""
    ld = _check_launch(ic, _short_rows(), ROW_KERNEL_ROWS, 32768, 2)
    assert ld == 32768
