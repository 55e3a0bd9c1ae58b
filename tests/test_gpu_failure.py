"""Failure detection on the GPU without a fault: a device wait that nothing
ever satisfies runs out after its bound, the kernel returns, the host reads
IC_ERR_TIMEOUT from ic_sync_status, and the context keeps working."""
import numpy as np
import pytest
import torch

import oracle
from cross_layer_top_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ic():
    from cross_layer_top_b200 import indexcache
    return indexcache


def test_bounded_wait_reports_timeout_and_context_survives(ic):
    from cross_layer_top_b200 import probe
    ctx = ic.Context(0)
    probe.ic_probe_wait_timeout(ctx)
    with pytest.raises(ic.ICError) as e:
        ctx.sync_status()
    assert e.value.code == ic.IC_ERR_TIMEOUT
    ctx.sync_status()  # reported once, then cleared
    # the same context still computes: tiny integer scores, bit-exact
    cfg = synth.CONFIGS["tiny"]
    lay = synth.prefill_layer(cfg, 0, "cuda")
    L = cfg.L
    out = torch.full((L, L), float("nan"), device="cuda")
    ic.ic_index_score(ctx, lay["qI"], lay["kI"], lay["w"], 0, L, out)
    ctx.sync_status()
    rows = np.array([0, 1, 200, L - 1], np.int32)
    ref = oracle.index_scores(synth.bf16_to_f32_numpy(lay["qI"]), synth.bf16_to_f32_numpy(lay["kI"]),
                              synth.bf16_to_f32_numpy(lay["w"]), rows=rows)
    got = out.cpu().numpy()[rows].astype(np.float64)
    for i, t in enumerate(rows):
        assert np.array_equal(got[i, :t + 1], ref[i, :t + 1])
    ctx.close()
