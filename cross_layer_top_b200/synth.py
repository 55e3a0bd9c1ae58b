"""Seeded synthetic inputs for the IndexCache hot path.

This module holds none of the method's arithmetic: it only draws the tensors
that both the CUDA path and the CPU oracle consume.  Five workloads mirror
the shapes the pages measure (200K-class contexts, k = 2048, 47-layer
stacks); no dataset or trained weight is involved.

Distributions per workload (all tensors bf16 unless stated):
  tiny          L=512, pattern FSSS, H_I=4, d_I=32, k=64; q_I/k_I integers
                uniform in [-3, 3]; w uniform over {-1,-0.5,0.5,1}; attention
                4 query heads, 1 KV head, d=64, Q/K/V ~ N(0,1); seed 0
  prefill       L=16384, FSSSFSSS, H_I=64, d_I=128, k=2048; q_I/k_I ~ N(0,1),
                w ~ N(0,1)/sqrt(64); 16 query heads, d=128, Q/K/V ~
                N(0,1)/sqrt(128); seed 1
  long_prefill  as prefill with L=131072, pattern FSSS (or FFFF); seed 2
  decode        32 sequences x (65536 cached + 1 new) tokens, 16 layers
                FSSS x4; FP8 e4m3 indexer-key cache with a per-token fp32
                scale (amax/448 of the N(0,1) key); main K/V ~ N(0,1);
                16 query heads, d=128, k=2048; seed 3
  decode_sweep  8 sequences x (200000 + 1) tokens, 47 layers, uniform
                retention 1/r (or the searched patterns below); otherwise as
                decode; seed 4
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class PrefillConfig:
    name: str
    L: int
    pattern: str
    H_I: int
    d_I: int
    k: int
    Hq: int
    d: int
    seed: int
    integer_indexer: bool = False

    @property
    def n_layers(self) -> int:
        return len(self.pattern)


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    ctx: int
    pattern: str
    H_I: int
    d_I: int
    k: int
    Hq: int
    d: int
    seed: int

    @property
    def n_layers(self) -> int:
        return len(self.pattern)

    @property
    def S(self) -> int:
        # cached context plus the new token, whose keys are appended first
        return self.ctx + 1


def uniform_pattern(n: int, r: int) -> str:
    return "".join("F" if l % r == 0 else "S" for l in range(n))


CONFIGS = {
    "tiny": PrefillConfig("tiny", 512, "FSSS", 4, 32, 64, 4, 64, 0, integer_indexer=True),
    "prefill": PrefillConfig("prefill", 16384, "FSSSFSSS", 64, 128, 2048, 16, 128, 1),
    "long_prefill": PrefillConfig("long_prefill", 131072, "FSSS", 64, 128, 2048, 16, 128, 2),
    "long_prefill_allF": PrefillConfig("long_prefill_allF", 131072, "FFFF", 64, 128, 2048, 16,
                                       128, 2),
    "decode": DecodeConfig("decode", 32, 65536, uniform_pattern(16, 4), 64, 128, 2048, 16, 128, 3),
}
for _r in (1, 2, 4, 8):
    CONFIGS["decode_sweep_r%d" % _r] = DecodeConfig(
        "decode_sweep_r%d" % _r, 8, 200000, uniform_pattern(47, _r), 64, 128, 2048, 16, 128, 4)

# The F/S patterns searched for the 47-layer model at retention 1/2, 1/4 and
# 1/8 ("IndexCache: Accelerating Sparse Attention via Cross-Layer Index
# Reuse", Appendix B): 24, 12 and 7 F layers.  Run on the 200K decode sweep's
# layer tensors in place of the uniform patterns.
SEARCHED_PATTERNS_47 = {
    "1/2": "FSFSFSSSSFSFFFFSFFSSFFSFFFSSFFSSFSSSSFSFFFSFSSF",
    "1/4": "FSFSFSSSSFSSSFSSFFSSFSSFSSSSFSSSFSSSSFSSSSSSSSS",
    "1/8": "FSSSFSSSSSSSSFSSSFSSSSSFSSSSFSSSSSSSSFSSSSSSSSS",
}


def _gen(device, seed: int, layer: int, slot: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + layer * 1009 + slot * 17 + 12345) % (2 ** 63))
    return g


def _normal(shape, std, device, seed, layer, slot):
    x = torch.randn(shape, generator=_gen(device, seed, layer, slot), device=device,
                    dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def prefill_layer(cfg: PrefillConfig, layer: int, device="cpu", indexer: bool | None = None):
    """Tensors of one prefill layer.  'qI','kI','w' only on F layers."""
    if indexer is None:
        indexer = cfg.pattern[layer] == "F"
    L, out = cfg.L, {}
    if indexer:
        if cfg.integer_indexer:
            g = _gen(device, cfg.seed, layer, 0)
            out["qI"] = torch.randint(-3, 4, (L, cfg.H_I, cfg.d_I), generator=g,
                                      device=device).to(torch.bfloat16)
            g = _gen(device, cfg.seed, layer, 1)
            out["kI"] = torch.randint(-3, 4, (L, cfg.d_I), generator=g,
                                      device=device).to(torch.bfloat16)
            g = _gen(device, cfg.seed, layer, 2)
            choice = torch.randint(0, 4, (L, cfg.H_I), generator=g, device=device)
            table = torch.tensor([-1.0, -0.5, 0.5, 1.0], device=device)
            out["w"] = table[choice].to(torch.bfloat16)
        else:
            out["qI"] = _normal((L, cfg.H_I, cfg.d_I), 1.0, device, cfg.seed, layer, 0)
            out["kI"] = _normal((L, cfg.d_I), 1.0, device, cfg.seed, layer, 1)
            out["w"] = _normal((L, cfg.H_I), 1.0 / math.sqrt(cfg.H_I), device, cfg.seed, layer, 2)
    std = 1.0 if cfg.integer_indexer else 1.0 / math.sqrt(cfg.d)
    out["Q"] = _normal((L, cfg.Hq, cfg.d), std, device, cfg.seed, layer, 3)
    out["K"] = _normal((L, cfg.d), std, device, cfg.seed, layer, 4)
    out["V"] = _normal((L, cfg.d), std, device, cfg.seed, layer, 5)
    return out


def fp8_e4m3_quantize_per_token(x: torch.Tensor):
    """Input preparation for the FP8 indexer-key cache: per-token scale =
    amax(|x|)/448 (the e4m3 maximum), bytes = e4m3(x / scale) via torch's
    float8_e4m3fn cast.  Returns (uint8 bytes, fp32 scale)."""
    amax = x.abs().amax(dim=-1).clamp_min(1e-12)
    scale = (amax / 448.0).to(torch.float32)
    q = (x / scale.unsqueeze(-1)).to(torch.float8_e4m3fn)
    return q.view(torch.uint8), scale


def prefill_indexer_fp8(cfg: PrefillConfig, layer: int, device="cpu"):
    """The indexer inputs of ``prefill_layer`` (same draw) prepared for the
    FP8 indexer: q_I in e4m3 with one fp32 scale per (token, head), k_I in
    e4m3 with one per token (amax/448 each), w unchanged."""
    lay = prefill_layer(cfg, layer, device, indexer=True)
    qI8, q_scale = fp8_e4m3_quantize_per_token(lay["qI"].float())
    kI8, k_scale = fp8_e4m3_quantize_per_token(lay["kI"].float())
    return {"qI8": qI8.contiguous(), "q_scale": q_scale.contiguous(), "kI8": kI8.contiguous(),
            "k_scale": k_scale.contiguous(), "w": lay["w"]}


def decode_layer(cfg: DecodeConfig, layer: int, device="cpu", indexer: bool | None = None,
                 batch=None):
    """Tensors of one decode layer (one step).  'q','w','kI8','kI_scale' only
    on F layers.  ``batch`` optionally restricts to a slice of sequences
    (same values as the full draw is NOT guaranteed; use for small tests)."""
    if indexer is None:
        indexer = cfg.pattern[layer] == "F"
    B = cfg.B if batch is None else batch
    S = cfg.S
    out = {}
    if indexer:
        out["q"] = _normal((B, cfg.H_I, cfg.d_I), 1.0, device, cfg.seed, layer, 0)
        out["w"] = _normal((B, cfg.H_I), 1.0 / math.sqrt(cfg.H_I), device, cfg.seed, layer, 2)
        k32 = torch.randn((B, S, cfg.d_I), generator=_gen(device, cfg.seed, layer, 1),
                          device=device, dtype=torch.float32)
        out["kI8"], out["kI_scale"] = fp8_e4m3_quantize_per_token(k32)
        del k32
    out["Q"] = _normal((B, cfg.Hq, cfg.d), 1.0, device, cfg.seed, layer, 3)
    out["K"] = _normal((B, S, cfg.d), 1.0, device, cfg.seed, layer, 4)
    out["V"] = _normal((B, S, cfg.d), 1.0, device, cfg.seed, layer, 5)
    out["seq_len"] = torch.full((B,), S, dtype=torch.int32, device=device)
    return out


def bf16_to_f32_numpy(t: torch.Tensor):
    """Exact widening of a bf16 tensor to a host float32 numpy array."""
    return t.detach().to("cpu", torch.float32).numpy()
