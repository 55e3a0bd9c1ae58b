"""The attention check (tests/attn_check.py) can fail: on the CPU, the
oracle's own output with one plausible kernel mistake planted, then rounded
to bf16 as a kernel's output is, must be rejected, and the correct output
rounded to bf16 must be accepted.  Both at the prefill workloads' scale
(Q, K, V ~ N(0,1)/sqrt(128): near-uniform softmax over 2048 keys, |o| about
2e-3) and with peaked logits (Q scaled by 8 at unit scale, as in the
decode workloads), 16 query heads, d = 128."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import attn_check

Hq, D, KSEL, S = 16, 128, 2048, 6000


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).bfloat16().float().numpy().astype(np.float64)


def _case(kind, seed):
    rng = np.random.default_rng(seed)
    if kind == "uniform":
        std_q = std_kv = 1.0 / math.sqrt(D)
    else:
        std_q, std_kv = 8.0, 1.0
    Q = _bf16(rng.standard_normal((3, Hq, D)) * std_q).astype(np.float32)
    K = _bf16(rng.standard_normal((S, D)) * std_kv).astype(np.float32)
    V = _bf16(rng.standard_normal((S, D)) * std_kv).astype(np.float32)
    idx = np.stack([np.sort(rng.choice(S, KSEL, replace=False)) for _ in range(3)]).astype(np.int32)
    return Q, K, V, idx


def _attn(Q, K, V, idx):
    return oracle.sparse_attn(Q, K, V, idx)


def _mutations(Q, K, V, idx, rng):
    """(name, index rows, V) pairs, each one kernel mistake."""
    out = []
    # the selected key with the largest weight for head 0 of row 0 is the
    # one whose loss matters most in a peaked row; in a uniform row any is
    logits = (Q[0, 0].astype(np.float64) @ K[idx[0]].T.astype(np.float64))
    j = int(np.argmax(logits))
    drop = idx.copy()
    drop[0, j] = -1
    out.append(("one key dropped", drop, V))
    sel = set(idx[0].tolist())
    shift = idx.copy()
    jj = next(x for x in [j] + list(range(KSEL)) if idx[0, x] + 1 not in sel and idx[0, x] + 1 < S)
    shift[0, jj] += 1
    out.append(("one index shifted by one", shift, V))
    outside = next(u for u in rng.permutation(S) if u not in sel)
    wrongv = V.copy()
    wrongv[idx[0, j]] = V[outside]
    out.append(("one V row read from the wrong position", idx, wrongv))
    half = idx.copy()
    half[:, KSEL // 2:] = -1
    out.append(("second half of the keys dropped", half, V))
    return out


@pytest.mark.parametrize("kind", ["uniform", "peaked"])
def test_checker_accepts_rounded_truth_and_rejects_mutations(kind):
    Q, K, V, idx = _case(kind, 5 if kind == "uniform" else 6)
    ref = _attn(Q, K, V, idx)
    spread = oracle.attn_weight_spread(Q, K, V, idx)
    assert attn_check.passes(_bf16(ref), ref, spread)
    if kind == "uniform":
        # the scale that makes the stated tolerance alone empty: |o| ~ 2e-3,
        # so an all-zero output meets 2e-2 + 1e-2 |o| but not the bound
        assert np.abs(ref).mean() < 5e-3
        b1, b2 = attn_check.bars(np.zeros_like(ref), ref, spread)
        assert b1.all() and not b2.all()
    rng = np.random.default_rng(1)
    for name, midx, mV in _mutations(Q, K, V, idx, rng):
        bad = _bf16(_attn(Q, K, mV, midx))
        assert not attn_check.passes(bad, ref, spread), "%s (%s) was accepted" % (name, kind)

