"""ic_stack_graph_*: the layer stack captured once as a CUDA graph and
replayed.  A replay runs the same kernels on the same buffers as
ic_run_stack, so every output and index snapshot must be bit-identical to
the eager stack's, also after the inputs change in place; each replay adds
the captured kernel count to the launch counter; and while a graph exists
the context refuses to regrow the scratch the graph uses."""
import pytest
import torch

from cross_layer_top_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ic():
    from cross_layer_top_b200 import indexcache
    return indexcache


def _decode_stack(ic, cfg):
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.decode_layer(cfg, l, "cuda")
        lay["out"] = torch.empty((cfg.B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        lay["idx_snapshot"] = torch.empty((cfg.B, cfg.k), dtype=torch.int32, device="cuda")
        layers.append(lay)
    dims = ic.stack_dims(ic.IC_DECODE, cfg.H_I, cfg.d_I, cfg.k, cfg.Hq, cfg.d, B=cfg.B,
                         S_max=cfg.S, seq_len=layers[0]["seq_len"])
    return layers, dims


def _prefill_stack(ic, cfg):
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.prefill_layer(cfg, l, "cuda")
        lay["out"] = torch.empty((cfg.L, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        lay["idx_snapshot"] = torch.empty((cfg.L, cfg.k), dtype=torch.int32, device="cuda")
        layers.append(lay)
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, cfg.k, cfg.Hq, cfg.d, L=cfg.L)
    return layers, dims


def _snap(layers):
    return [(lay["out"].clone(), lay["idx_snapshot"].clone()) for lay in layers]


def _replay_matches_eager(ic, ctx, pattern, layers, dims, rows, k, perturb):
    cache = torch.empty((rows, k), dtype=torch.int32, device="cuda")
    g = ic.ic_stack_graph_create(ctx, ic.ic_create_pattern(pattern), layers, dims, cache)
    n = g.kernels()
    assert n >= len(pattern)  # at least one attention launch per layer
    results = []
    for step in range(3):
        if step:
            perturb(layers, step)
        before = ctx.launch_count()
        g.launch()
        torch.cuda.synchronize()
        ctx.sync_status()
        assert ctx.launch_count() - before == n
        got = _snap(layers)
        ic.ic_run_stack(ctx, ic.ic_create_pattern(pattern), layers, dims, cache)
        torch.cuda.synchronize()
        ctx.sync_status()
        for (o, s), lay in zip(got, layers):
            assert torch.equal(o, lay["out"])
            assert torch.equal(s, lay["idx_snapshot"])
        results.append(got)
    # the perturbations reached the replays
    assert not torch.equal(results[0][0][0], results[1][0][0])
    return g


def test_graph_decode_matches_eager(ic):
    ctx = ic.Context(0)
    cfg = synth.DecodeConfig("graph_decode", 3, 4999, "FSSFS", 64, 128, 256, 16, 128, 21)
    layers, dims = _decode_stack(ic, cfg)

    def perturb(layers, step):
        for lay in layers:
            lay["Q"].mul_(-1)
            if "q" in lay:
                lay["q"].copy_(lay["q"].roll(step, dims=-1))

    g = _replay_matches_eager(ic, ctx, cfg.pattern, layers, dims, cfg.B, cfg.k, perturb)
    g.close()
    ctx.close()


def test_graph_decode_lengths_change_in_place(ic):
    """seq_len is read by the kernels at run time: shortening rows in place
    between replays is seen by the graph."""
    ctx = ic.Context(0)
    cfg = synth.DecodeConfig("graph_decode_len", 4, 3000, "FSFS", 64, 128, 256, 16, 128, 22)
    layers, dims = _decode_stack(ic, cfg)
    seq_len = layers[0]["seq_len"]

    def perturb(layers, step):
        seq_len.copy_(torch.tensor([3000, 1, 2048 - step, 700 * step], dtype=torch.int32))

    g = _replay_matches_eager(ic, ctx, cfg.pattern, layers, dims, cfg.B, cfg.k, perturb)
    snap = layers[0]["idx_snapshot"].cpu()
    assert (snap[1, 1:] == -1).all() and snap[1, 0] == 0
    g.close()
    ctx.close()


def test_graph_prefill_matches_eager(ic):
    ctx = ic.Context(0)
    cfg = synth.PrefillConfig("graph_prefill", 1500, "FSSFSS", 64, 128, 256, 16, 128, 23)
    layers, dims = _prefill_stack(ic, cfg)

    def perturb(layers, step):
        for lay in layers:
            lay["V"].mul_(0.5)
            if "qI" in lay:
                lay["qI"].mul_(-1)

    g = _replay_matches_eager(ic, ctx, cfg.pattern, layers, dims, cfg.L, cfg.k, perturb)
    g.close()
    ctx.close()


def test_graph_pins_scratch(ic):
    """While a graph exists, a call needing larger scratch fails with
    IC_ERR_NOMEM instead of freeing the graph's buffer; after the graph is
    destroyed the same call succeeds."""
    ctx = ic.Context(0)
    cfg = synth.DecodeConfig("graph_pin", 2, 2500, "FS", 64, 128, 256, 16, 128, 24)
    layers, dims = _decode_stack(ic, cfg)
    cache = torch.empty((cfg.B, cfg.k), dtype=torch.int32, device="cuda")
    g = ic.ic_stack_graph_create(ctx, ic.ic_create_pattern(cfg.pattern), layers, dims, cache)
    L = 4096
    gen = torch.Generator().manual_seed(5)
    qI = torch.randn((L, 64, 128), generator=gen).to(torch.bfloat16).cuda()
    kI = torch.randn((L, 128), generator=gen).to(torch.bfloat16).cuda()
    w = torch.randn((L, 64), generator=gen).to(torch.bfloat16).cuda()
    idx = torch.empty((L, 256), dtype=torch.int32, device="cuda")
    with pytest.raises(ic.ICError) as ei:
        ic.ic_index_fp(ctx, qI, kI, w, 256, idx)
    assert ei.value.code == ic.IC_ERR_NOMEM
    # the graph still replays
    g.launch()
    torch.cuda.synchronize()
    ctx.sync_status()
    g.close()
    ic.ic_index_fp(ctx, qI, kI, w, 256, idx)
    torch.cuda.synchronize()
    ctx.sync_status()
    ctx.close()


def test_graph_context_close_releases_graphs(ic):
    ctx = ic.Context(0)
    cfg = synth.DecodeConfig("graph_close", 2, 2500, "FS", 64, 128, 256, 16, 128, 25)
    layers, dims = _decode_stack(ic, cfg)
    cache = torch.empty((cfg.B, cfg.k), dtype=torch.int32, device="cuda")
    g = ic.ic_stack_graph_create(ctx, ic.ic_create_pattern(cfg.pattern), layers, dims, cache)
    ctx.close()
    assert not g.handle
