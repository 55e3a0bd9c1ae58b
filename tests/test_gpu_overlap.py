"""GPU parity of the cross-layer overlap |T_a ∩ T_b| (IndexCache paper,
Appendix A) against the oracle: bit-exact hit counts per row."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from cross_layer_top_b200 import synth

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "pages_examples.json")


@pytest.fixture(scope="module")
def ic():
    from cross_layer_top_b200 import indexcache
    return indexcache


@pytest.fixture(scope="module")
def ctx(ic):
    c = ic.Context(0)
    yield c
    c.close()


def gpu_hits(ic, ctx, a, b, n_keys):
    a_d = torch.as_tensor(a, dtype=torch.int32).cuda()
    b_d = torch.as_tensor(b, dtype=torch.int32).cuda()
    hits = torch.full((a_d.shape[0],), -7, dtype=torch.int32, device="cuda")
    ic.ic_index_overlap(ctx, a_d, b_d, hits, n_keys)
    ctx.sync_status()
    return hits.cpu().numpy()


def oracle_hits(a, b):
    k = a.shape[1]
    return np.array([round(oracle.overlap(a[r], b[r]) * k) for r in range(a.shape[0])])


def test_overlap_page_example(ic, ctx):
    g = json.load(open(GOLDEN))["overlap_toy"]
    a, b = np.array([g["a"]]), np.array([g["b"]])
    h = gpu_hits(ic, ctx, a, b, 16)
    assert h.tolist() == [3] and h[0] / a.shape[1] == g["overlap"]


@pytest.mark.parametrize("n_keys,k", [(5000, 2048), (200001, 2048), (500000, 300), (64, 64)])
def test_overlap_random_rows(ic, ctx, n_keys, k):
    rng = np.random.default_rng(n_keys + k)
    rows = 37
    a = np.full((rows, k), -1, np.int32)
    b = np.full((rows, k), -1, np.int32)
    for r in range(rows):
        na = int(rng.integers(0, k + 1)) if r % 4 else k
        nb = int(rng.integers(0, k + 1)) if r % 3 else k
        pool = rng.permutation(min(n_keys, 3 * k))[: max(na, nb)]  # shared pool: real overlaps
        a[r, :na] = rng.permutation(pool[:na]) if r % 2 else np.sort(pool[:na])
        b[r, :nb] = rng.permutation(pool[:nb])
        if r % 5 == 0 and na > 3:  # a repeated entry in a counts once per occurrence
            a[r, 1] = a[r, 0]
        if r % 7 == 0:  # -1 gaps scattered inside the row
            a[r, ::3] = -1
    got = gpu_hits(ic, ctx, a, b, n_keys)
    assert np.array_equal(got, oracle_hits(a, b))


def test_overlap_invariants_on_a_stack(ic, ctx):
    """Top-k sets from the GPU indexer on two layers' tensors: a set against
    itself gives its number of selected entries, the relation is symmetric,
    sampled rows match the oracle, and rows t < k overlap fully."""
    cfg = synth.CONFIGS["tiny"]
    lays = [synth.prefill_layer(cfg, l, "cuda", indexer=True) for l in range(2)]
    L, k = cfg.L, cfg.k
    idx = []
    for lay in lays:
        t = torch.empty((L, k), dtype=torch.int32, device="cuda")
        ic.ic_index_fp(ctx, lay["qI"], lay["kI"], lay["w"], k, t)
        idx.append(t)
    ctx.sync_status()
    valid = (idx[0] >= 0).sum(1).cpu().numpy()
    hits_self = torch.empty(L, dtype=torch.int32, device="cuda")
    ic.ic_index_overlap(ctx, idx[0], idx[0], hits_self, L)
    hab = torch.empty(L, dtype=torch.int32, device="cuda")
    hba = torch.empty(L, dtype=torch.int32, device="cuda")
    ic.ic_index_overlap(ctx, idx[0], idx[1], hab, L)
    ic.ic_index_overlap(ctx, idx[1], idx[0], hba, L)
    ctx.sync_status()
    assert np.array_equal(hits_self.cpu().numpy(), valid)
    assert np.array_equal(hab.cpu().numpy(), hba.cpu().numpy())
    rows = np.array([0, 1, 63, 64, 65, 300, L - 1])
    a, b = idx[0].cpu().numpy()[rows], idx[1].cpu().numpy()[rows]
    assert np.array_equal(hab.cpu().numpy()[rows], oracle_hits(a, b))
    # rows t < k select all of 0..t in both layers: full overlap
    assert np.array_equal(hab.cpu().numpy()[:k], np.arange(1, k + 1))


def test_overlap_bad_index_is_reported(ic, ctx):
    a = np.array([[0, 1, 2, 99], [3, -4, 5, 6]], np.int32)
    b = np.array([[0, 1, 2, 3], [3, 4, 5, 6]], np.int32)
    a_d, b_d = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    hits = torch.empty(2, dtype=torch.int32, device="cuda")
    ic.ic_index_overlap(ctx, a_d, b_d, hits, 10)
    with pytest.raises(ic.ICError) as e:
        ctx.sync_status()
    assert e.value.code == ic.IC_ERR_DEVICE
    ctx.sync_status()
    assert hits.cpu().numpy().tolist() == [3, 3]  # the bad entries were skipped
