"""ic_run_stack_ahead: the layer stack with every F layer's indexer issued
ahead on a second stream (the multi-layer indexer page's scheduling), run
eagerly and as a captured graph (ic_stack_graph_create_ahead).  The order
of the kernels changes, not their inputs, so every index tensor and output
must equal ic_run_stack's bit for bit; on the integer tiny workload
the indices are also checked against the oracle's stack and the attention
against the oracle within the attention bars of tests/attn_check.py.

Patterns with F layers back to back (FSFFSSFS) make the two index buffers
alternate with no S layer between two writes."""
import numpy as np
import pytest
import torch

import oracle
from cross_layer_top_b200 import synth
from tests import attn_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ic():
    from cross_layer_top_b200 import indexcache
    return indexcache


def f32(t):
    return synth.bf16_to_f32_numpy(t)


def _prefill_layers(cfg, pattern, device):
    layers = []
    for l, c in enumerate(pattern):
        lay = synth.prefill_layer(cfg, l, device, indexer=c == "F")
        layers.append(lay)
    return layers


def _with_outputs(layers, rows, cfg):
    out = []
    for lay in layers:
        g = {n: v.cuda() for n, v in lay.items()}
        g["out"] = torch.full((rows, cfg.Hq, cfg.d), float("nan"), dtype=torch.bfloat16,
                              device="cuda")
        g["idx_snapshot"] = torch.full((rows, cfg.k), -7, dtype=torch.int32, device="cuda")
        out.append(g)
    return out


def _run_both(ic, ctx, pattern, glayers_a, glayers_b, dims, rows, k, graph=False):
    """ic_run_stack into glayers_a, ic_run_stack_ahead into glayers_b (with
    graph=True: its captured graph, replayed twice with the outputs and
    buffers reset in between), then every output and index tensor compared."""
    pat = ic.ic_create_pattern(pattern)
    cache = torch.empty((rows, k), dtype=torch.int32, device="cuda")
    ic.ic_run_stack(ctx, pat, glayers_a, dims, cache)
    c0 = torch.full((rows, k), -9, dtype=torch.int32, device="cuda")
    c1 = torch.full((rows, k), -9, dtype=torch.int32, device="cuda")
    if graph:
        g = ic.ic_stack_graph_create_ahead(ctx, pat, glayers_b, dims, c0, c1)
        for _ in range(2):
            for lay in glayers_b:
                lay["out"].fill_(float("nan"))
                lay["idx_snapshot"].fill_(-7)
            c0.fill_(-9)
            c1.fill_(-9)
            g.launch()
        ctx.sync_status()
        g.close()
    else:
        ic.ic_run_stack_ahead(ctx, pat, glayers_b, dims, c0, c1)
    ctx.sync_status()
    for l in range(len(pattern)):
        assert torch.equal(glayers_a[l]["idx_snapshot"], glayers_b[l]["idx_snapshot"]), l
        assert torch.equal(glayers_a[l]["out"], glayers_b[l]["out"]), l
    # the last index tensors of the even and odd F layers stay in their buffers
    f = [l for l, c in enumerate(pattern) if c == "F"]
    for parity, buf in ((0, c0), (1, c1)):
        mine = [l for j, l in enumerate(f) if j % 2 == parity]
        if mine:
            assert torch.equal(buf, glayers_b[mine[-1]]["idx_snapshot"])
        else:
            assert torch.all(buf == -9)


@pytest.mark.parametrize("graph", [False, True])
def test_stack_ahead_tiny_against_oracle(ic, graph):
    cfg = synth.CONFIGS["tiny"]
    pattern = "FSFFSSFS"
    L, k = cfg.L, cfg.k
    layers = _prefill_layers(cfg, pattern, "cpu")
    ctx = ic.Context(0)
    ga = _with_outputs(layers, L, cfg)
    gb = _with_outputs(layers, L, cfg)
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, L=L)
    _run_both(ic, ctx, pattern, ga, gb, dims, L, k, graph=graph)
    olayers = [{n: f32(v) for n, v in lay.items()} for lay in layers]
    oidx, oout = oracle.run_stack(pattern, olayers, k)
    for l in range(len(pattern)):
        assert np.array_equal(gb[l]["idx_snapshot"].cpu().numpy(), oidx[l]), l
        got = gb[l]["out"].float().cpu().numpy()
        attn_check.check(got, olayers[l]["Q"], olayers[l]["K"], olayers[l]["V"], oidx[l],
                         what="ahead tiny layer %d" % l)
    ctx.close()


def test_stack_ahead_prefill_equals_stack(ic):
    """The prefill workload (L = 16384, FSSSFSSS) and a pattern with F
    layers back to back, both at full size."""
    cfg = synth.CONFIGS["prefill"]
    L, k = cfg.L, cfg.k
    ctx = ic.Context(0)
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, L=L)
    for pattern in (cfg.pattern, "FFSFSSFF"):
        layers = _prefill_layers(cfg, pattern, "cuda")
        _run_both(ic, ctx, pattern, _with_outputs(layers, L, cfg), _with_outputs(layers, L, cfg),
                  dims, L, k)
        del layers
        torch.cuda.empty_cache()
    ctx.close()


@pytest.mark.parametrize("graph", [False, True])
def test_stack_ahead_decode_equals_stack(ic, graph):
    """The batched-decode stack (32 x 65537, 16 layers FSSS x4), eagerly and
    as a captured graph."""
    cfg = synth.CONFIGS["decode"]
    B, S, k = cfg.B, cfg.S, cfg.k
    ctx = ic.Context(0)
    layers = [synth.decode_layer(cfg, l, "cuda") for l in range(cfg.n_layers)]
    dims = ic.stack_dims(ic.IC_DECODE, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, B=B, S_max=S,
                         seq_len=layers[0]["seq_len"])

    def outputs():
        out = []
        for lay in layers:
            g = dict(lay)
            g["out"] = torch.full((B, cfg.Hq, cfg.d), float("nan"), dtype=torch.bfloat16,
                                  device="cuda")
            g["idx_snapshot"] = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
            out.append(g)
        return out

    _run_both(ic, ctx, cfg.pattern, outputs(), outputs(), dims, B, k, graph=graph)
    ctx.close()


def test_stack_ahead_needs_two_buffers(ic):
    """Both the eager call and the graph capture refuse one buffer twice."""
    cfg = synth.CONFIGS["tiny"]
    L, k = cfg.L, cfg.k
    ctx = ic.Context(0)
    layers = _with_outputs(_prefill_layers(cfg, cfg.pattern, "cpu"), L, cfg)
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, L=L)
    cache = torch.empty((L, k), dtype=torch.int32, device="cuda")
    with pytest.raises(ic.ICError) as e:
        ic.ic_run_stack_ahead(ctx, ic.ic_create_pattern(cfg.pattern), layers, dims, cache, cache)
    assert e.value.code == ic.IC_ERR_INVALID_ARG
    with pytest.raises(ic.ICError) as e:
        ic.ic_stack_graph_create_ahead(ctx, ic.ic_create_pattern(cfg.pattern), layers, dims,
                                       cache, cache)
    assert e.value.code == ic.IC_ERR_INVALID_ARG
    ctx.close()


def test_stack_ahead_error_leaves_context_usable(ic):
    """A layer that fails its argument checks (no Q) after F layers' indexers
    were issued on the side stream: the call returns IC_ERR_INVALID_ARG, the
    caller's stream covers the side stream's work, and the next call on the
    same context is bit-identical to ic_run_stack."""
    cfg = synth.CONFIGS["tiny"]
    pattern = "FSFS"
    L, k = cfg.L, cfg.k
    layers = _prefill_layers(cfg, pattern, "cpu")
    ctx = ic.Context(0)
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, L=L)
    bad = _with_outputs(layers, L, cfg)
    bad[3]["Q"] = None
    c0 = torch.empty((L, k), dtype=torch.int32, device="cuda")
    c1 = torch.empty((L, k), dtype=torch.int32, device="cuda")
    with pytest.raises(ic.ICError) as e:
        ic.ic_run_stack_ahead(ctx, ic.ic_create_pattern(pattern), bad, dims, c0, c1)
    assert e.value.code == ic.IC_ERR_INVALID_ARG
    torch.cuda.current_stream().synchronize()
    ctx.sync_status()
    _run_both(ic, ctx, pattern, _with_outputs(layers, L, cfg), _with_outputs(layers, L, cfg), dims,
              L, k)
    ctx.close()
