"""The top-k kernel's branches, each forced by a constructed row and
checked bit-exact against the oracle's top-k (positions of the k largest,
ascending, ties to the lower position):
  - the bitmap path on Gaussian rows, including one at the bitmap's
    capacity (131072 keys), and one tie at T taken whole;
  - the general path: a row longer than the bitmap holds, a candidate bin
    larger than the candidate list, a warp slice that overflows, and a tie
    at T that is split by position."""
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


def _rows():
    rng = np.random.default_rng(2024)
    rows = {}
    rows["gauss_20000"] = rng.standard_normal(20000)
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


def test_topk_every_path_bit_exact(ic):
    ctx = ic.Context(0)
    rows = _rows()
    names = list(rows)
    ld = (max(len(v) for v in rows.values()) + 3) // 4 * 4
    sc = torch.full((len(names), ld), -1e30, dtype=torch.float32)
    for i, n in enumerate(names):
        sc[i, :len(rows[n])] = torch.from_numpy(rows[n])
    lens = torch.tensor([len(rows[n]) for n in names], dtype=torch.int32)
    idx = torch.empty((len(names), K), dtype=torch.int32, device="cuda")
    ic.ic_topk(ctx, sc.cuda(), K, idx, row_len=lens.cuda(), ld=ld)
    ctx.sync_status()
    got = idx.cpu().numpy()
    for i, n in enumerate(names):
        want = oracle.topk_row(rows[n].astype(np.float64), K)
        assert got[i].tolist() == want.tolist(), n
    ctx.close()
