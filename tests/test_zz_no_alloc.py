"""The allocation-free decode indexer entry point.

ic_index_fp_decode_noalloc serves callers that cannot allocate device memory
on their decode path (an engine that owns all free HBM for its KV-cache
pool, or a decode step replayed from a captured stream).  It keeps its score
rows in a fixed array inside the library instead of context scratch.  This
file is collected last on purpose: it must pass both alone in a fresh
process and after every other test.  The checks, on calls in a row:
  * its index rows equal those of ic_index_fp_decode on the same inputs (the
    same kernels run, so the comparison is exact); one batch of short rows
    takes the single-CTA top-k, the others the cluster top-k;
  * on sampled sequences its selections meet the oracle's bar (every
    selected score at least the oracle's k-th score minus 1e-3 of it);
  * the allocation-free status query reports no device error afterwards.
"""
import numpy as np
import pytest
import torch

import oracle
from cross_layer_top_b200 import synth

SEL_RTOL = 1e-3

pytestmark = pytest.mark.gpu


def _inputs(B, S_max, seed):
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn((B, 64, 128), generator=gen).bfloat16().cuda()
    w = (torch.randn((B, 64), generator=gen) / 8).bfloat16().cuda()
    k8, sc = synth.fp8_e4m3_quantize_per_token(torch.randn((B, S_max, 128), generator=gen))
    lens = torch.randint(1, S_max + 1, (B,), generator=gen, dtype=torch.int32)
    lens[0] = S_max
    return q, w, k8.contiguous().cuda(), sc.float().contiguous().cuda(), lens.cuda()


def _check_against_oracle(got, q, w, k8, sc, lens, b, k):
    n = int(lens[b])
    score = oracle.decode_scores(synth.bf16_to_f32_numpy(q[b]), synth.bf16_to_f32_numpy(w[b]),
                                 k8[b, :n].cpu().numpy(), sc[b, :n].cpu().numpy())
    row = got[b].cpu().numpy()
    m = min(n, k)
    sel = row[:m]
    assert np.all(row[m:] == -1) and np.all(np.diff(sel) > 0)
    assert sel.min() >= 0 and sel.max() < n
    if n <= k:
        assert sel.tolist() == list(range(n))
        return
    kth = oracle.kth_score(score, k)
    assert score[sel].min() >= kth - SEL_RTOL * abs(kth)


def test_noalloc_matches_regular_entry_point_and_oracle():
    from cross_layer_top_b200 import indexcache as ic
    ctx = ic.Context(0)
    k = 2048
    # 8 x 30001 and 5 x 65537 take the cluster top-k; 32 x 9000 the single-CTA one
    for call, (B, S_max, seed) in enumerate([(8, 30001, 1), (5, 65537, 2), (32, 9000, 3)]):
        q, w, k8, sc, lens = _inputs(B, S_max, seed)
        ref = torch.empty((B, k), dtype=torch.int32, device="cuda")
        ic.ic_index_fp_decode(ctx, q, w, k8, sc, lens, k, ref)
        got = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
        ic.ic_index_fp_decode_noalloc(q, w, k8, sc, lens, k, got)
        ic.ic_noalloc_sync_status()
        ctx.sync_status()
        assert torch.equal(got, ref), "call %d differs from ic_index_fp_decode" % call
        for b in (0, B - 1):
            _check_against_oracle(got, q, w, k8, sc, lens, b, k)
    ctx.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from cross_layer_top_b200 import indexcache as ic
    B, S_max = 128, 40000  # 128 * 40000 scores > 4 Mi
    q = torch.zeros((B, 64, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((B, 64), dtype=torch.bfloat16, device="cuda")
    k8 = torch.zeros((B, S_max, 128), dtype=torch.uint8, device="cuda")
    sc = torch.ones((B, S_max), dtype=torch.float32, device="cuda")
    lens = torch.full((B,), S_max, dtype=torch.int32, device="cuda")
    idx = torch.empty((B, 64), dtype=torch.int32, device="cuda")
    with pytest.raises(ic.ICError) as e:
        ic.ic_index_fp_decode_noalloc(q, w, k8, sc, lens, 64, idx)
    assert e.value.code == ic.IC_ERR_UNSUPPORTED
    assert "exceeds" in str(e.value)
