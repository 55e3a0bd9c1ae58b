"""ic_run_stack_host (inputs and outputs in pinned host memory, copies
overlapped with the compute) against ic_run_stack on the same inputs in
device memory: the same kernels run on the same values, so every output and
index snapshot must be bit-identical, across repeated calls."""
import pytest
import torch

from cross_layer_top_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ic():
    from cross_layer_top_b200 import indexcache
    return indexcache


def _pinned(t):
    h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
    h.copy_(t)
    return h


def _host_layers(layers):
    out = []
    for lay in layers:
        h = {n: _pinned(t) for n, t in lay.items() if n not in ("out", "idx_snapshot", "seq_len")}
        h["out"] = torch.empty(lay["out"].shape, dtype=lay["out"].dtype, pin_memory=True)
        h["idx_snapshot"] = torch.empty_like(lay["idx_snapshot"])  # device, as documented
        out.append(h)
    return out


def _run_both(ic, ctx, pattern, layers, dims, rows, k):
    cache = torch.empty((rows, k), dtype=torch.int32, device="cuda")
    ic.ic_run_stack(ctx, ic.ic_create_pattern(pattern), layers, dims, cache)
    host = _host_layers(layers)
    cache_h = torch.empty((rows, k), dtype=torch.int32, device="cuda")
    ic.ic_run_stack_host(ctx, ic.ic_create_pattern(pattern), host, dims, cache_h)
    torch.cuda.synchronize()
    ctx.sync_status()
    return host


def _check_equal(layers, host):
    for lay, h in zip(layers, host):
        assert torch.equal(lay["out"].cpu(), h["out"])
        assert torch.equal(lay["idx_snapshot"], h["idx_snapshot"])


def test_host_stack_prefill_matches_device_stack(ic):
    ctx = ic.Context(0)
    cfg = synth.PrefillConfig("host_prefill", 1500, "FSSFSS", 64, 128, 256, 16, 128, 13)
    L, k = cfg.L, cfg.k
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.prefill_layer(cfg, l, "cuda")
        lay["out"] = torch.empty((L, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        lay["idx_snapshot"] = torch.empty((L, k), dtype=torch.int32, device="cuda")
        layers.append(lay)
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, L=L)
    host = _run_both(ic, ctx, cfg.pattern, layers, dims, L, k)
    _check_equal(layers, host)
    # a second call on changed inputs reuses the slots and the events
    for lay in layers:
        lay["Q"].mul_(-1)
    host2 = _run_both(ic, ctx, cfg.pattern, layers, dims, L, k)
    _check_equal(layers, host2)
    assert not torch.equal(host[0]["out"], host2[0]["out"])
    ctx.close()


def test_host_stack_decode_matches_device_stack(ic):
    ctx = ic.Context(0)
    cfg = synth.DecodeConfig("host_decode", 3, 4999, "FSSFS", 64, 128, 256, 16, 128, 14)
    B, S, k = cfg.B, cfg.S, cfg.k
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.decode_layer(cfg, l, "cuda")
        lay["out"] = torch.empty((B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        lay["idx_snapshot"] = torch.empty((B, k), dtype=torch.int32, device="cuda")
        layers.append(lay)
    seq_len = layers[0]["seq_len"]
    dims = ic.stack_dims(ic.IC_DECODE, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, B=B, S_max=S,
                         seq_len=seq_len)
    for _ in range(2):
        host = _run_both(ic, ctx, cfg.pattern, layers, dims, B, k)
        _check_equal(layers, host)
    ctx.close()


def test_host_stack_prefill_workload(ic):
    """The prefill workload (L=16384, 8 layers FSSSFSSS): every output equal
    to the device-memory stack's."""
    ctx = ic.Context(0)
    cfg = synth.CONFIGS["prefill"]
    L, k = cfg.L, cfg.k
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.prefill_layer(cfg, l, "cuda")
        lay["out"] = torch.empty((L, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        lay["idx_snapshot"] = torch.empty((L, k), dtype=torch.int32, device="cuda")
        layers.append(lay)
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, L=L)
    host = _run_both(ic, ctx, cfg.pattern, layers, dims, L, k)
    _check_equal(layers, host)
    ctx.close()


def test_host_stack_error_leaves_context_usable(ic):
    """A layer without an output buffer fails its checks after earlier layers'
    copies were issued: the call returns IC_ERR_INVALID_ARG, the caller's
    stream covers the copies already issued, and the next call on the same
    context matches ic_run_stack bit for bit."""
    ctx = ic.Context(0)
    cfg = synth.PrefillConfig("host_prefill_err", 1500, "FSSF", 64, 128, 256, 16, 128, 14)
    L, k = cfg.L, cfg.k
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.prefill_layer(cfg, l, "cuda")
        lay["out"] = torch.empty((L, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
        lay["idx_snapshot"] = torch.empty((L, k), dtype=torch.int32, device="cuda")
        layers.append(lay)
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, L=L)
    bad = _host_layers(layers)
    bad[2]["out"] = None
    cache = torch.empty((L, k), dtype=torch.int32, device="cuda")
    with pytest.raises(ic.ICError) as e:
        ic.ic_run_stack_host(ctx, ic.ic_create_pattern(cfg.pattern), bad, dims, cache)
    assert e.value.code == ic.IC_ERR_INVALID_ARG
    torch.cuda.current_stream().synchronize()
    ctx.sync_status()
    host = _run_both(ic, ctx, cfg.pattern, layers, dims, L, k)
    _check_equal(layers, host)
    ctx.close()
