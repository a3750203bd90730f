"""Seeded synthetic workloads for the fused MoE layer.

This module only draws random numbers with the shapes and distributions of
the benchmark workloads; it holds none of the layer's arithmetic (no routing,
no alignment, no quantisation).  Both the CUDA path and the CPU oracle take
their inputs from here, so the two sides always see the same bytes.

Every tensor comes from its own ``torch.Generator`` seeded from
``(seed, tensor name, expert)``, so one expert's weights can be regenerated
alone.  The stream depends on the device the generator runs on (CPU and CUDA
use different generators); parity tests draw on one device and copy to the
other.
"""

from __future__ import annotations

import dataclasses
import zlib

import torch


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    """Shape and input recipe of one workload family."""

    name: str
    E: int
    topk: int
    H: int
    I: int
    fp8: bool             # 8-bit E4M3 weights (with mx: MXFP8 scales, else 128x128 fp32 block scales)
    routing: str          # "logits" | "biased_logits" | "uniform_ids" | "zipf"
    tokens: tuple         # the batch sizes T of the family
    zipf_s: float = 1.2
    bias_std: float = 0.5
    w_std: float = 0.02
    x_scale: float = 0.1
    mx: bool = False


CONFIGS = {
    # tiny layer: T=16, E=8, top-2, H=256, I=128, bf16 weights, logits routing
    "tiny": MoEConfig("tiny", E=8, topk=2, H=256, I=128, fp8=False,
                      routing="logits", tokens=(16,)),
    # Qwen3-235B-shaped MoE layer at decode batch sizes, bf16 weights
    "decode_bf16": MoEConfig("decode_bf16", E=128, topk=8, H=4096, I=1536, fp8=False,
                             routing="logits", tokens=(1, 4, 16, 64)),
    # same layer, FP8 128x128 block-scaled weights, uniformly random expert ids
    "fp8_uniform": MoEConfig("fp8_uniform", E=128, topk=8, H=4096, I=1536, fp8=True,
                             routing="uniform_ids", tokens=(256, 1024, 4096)),
    # prefill: 16384 tokens, logits plus a per-expert bias for moderate imbalance
    "prefill_fp8": MoEConfig("prefill_fp8", E=128, topk=8, H=4096, I=1536, fp8=True,
                             routing="biased_logits", tokens=(16384,)),
    # the prefill and decode layers with MXFP8 weights (E4M3, one E8M0 scale per 32 elements)
    "prefill_mxfp8": MoEConfig("prefill_mxfp8", E=128, topk=8, H=4096, I=1536, fp8=True,
                               routing="biased_logits", tokens=(16384,), mx=True),
    "decode_mxfp8": MoEConfig("decode_mxfp8", E=128, topk=8, H=4096, I=1536, fp8=True,
                              routing="logits", tokens=(1, 4, 16, 64), mx=True),
    # large experts with Zipf(1.2)-skewed choice without replacement
    "skewed_fp8": MoEConfig("skewed_fp8", E=256, topk=8, H=7168, I=2048, fp8=True,
                            routing="zipf", tokens=(1, 32, 512, 8192)),
}


def _gen(device, seed: int, *tags) -> torch.Generator:
    key = zlib.crc32(repr((int(seed),) + tuple(tags)).encode())
    g = torch.Generator(device=device)
    g.manual_seed(key)
    return g


def make_expert_weights(cfg: MoEConfig, e: int, seed: int = 0, device="cpu"):
    """bf16 draw of expert ``e``: w13 [2I, H] and w2 [H, I], both ~ N(0, w_std)."""
    g13 = _gen(device, seed, "w13", e)
    w13 = torch.randn((2 * cfg.I, cfg.H), generator=g13, device=device, dtype=torch.float32)
    w13 = (w13 * cfg.w_std).to(torch.bfloat16)
    g2 = _gen(device, seed, "w2", e)
    w2 = torch.randn((cfg.H, cfg.I), generator=g2, device=device, dtype=torch.float32)
    w2 = (w2 * cfg.w_std).to(torch.bfloat16)
    return w13, w2


def make_weights(cfg: MoEConfig, seed: int = 0, device="cpu"):
    """bf16 weights of all experts: w13 [E, 2I, H], w2 [E, H, I]."""
    w13 = torch.empty((cfg.E, 2 * cfg.I, cfg.H), dtype=torch.bfloat16, device=device)
    w2 = torch.empty((cfg.E, cfg.H, cfg.I), dtype=torch.bfloat16, device=device)
    for e in range(cfg.E):
        a, b = make_expert_weights(cfg, e, seed, device)
        w13[e].copy_(a)
        w2[e].copy_(b)
    return w13, w2


def make_tokens(cfg: MoEConfig, T: int, seed: int = 0, device="cpu"):
    """x [T, H] bf16 ~ N(0, 1) * x_scale."""
    g = _gen(device, seed, "x", T)
    x = torch.randn((T, cfg.H), generator=g, device=device, dtype=torch.float32)
    return (x * cfg.x_scale).to(torch.bfloat16)


def _choice_weights(cfg: MoEConfig, T: int, g, device):
    """Weights of pre-chosen experts: softmax of N(0, 1) draws over the k slots.

    The softmax here only shapes the input distribution (a Dirichlet-like draw
    that sums to one); it is not the layer's router.
    """
    z = torch.randn((T, cfg.topk), generator=g, device=device, dtype=torch.float32)
    return torch.softmax(z, dim=-1)


def make_routing(cfg: MoEConfig, T: int, seed: int = 0, device="cpu"):
    """Routing input of the workload.

    Returns ``{"logits": [T, E] fp32}`` for the router-driven workloads, or
    ``{"topk_ids": [T, k] int32, "topk_weights": [T, k] fp32}`` where the
    recipe fixes the choice directly (uniform ids with replacement, so a row
    may repeat an expert; or Zipf(s) without replacement, expert e having
    rank e+1, drawn as the k largest of log p + Gumbel noise, which samples
    sequentially without replacement).
    """
    g = _gen(device, seed, "route", cfg.routing, T)
    if cfg.routing == "logits":
        return {"logits": torch.randn((T, cfg.E), generator=g, device=device, dtype=torch.float32)}
    if cfg.routing == "biased_logits":
        gb = _gen(device, seed, "expert_bias")
        bias = torch.randn((cfg.E,), generator=gb, device=device, dtype=torch.float32) * cfg.bias_std
        z = torch.randn((T, cfg.E), generator=g, device=device, dtype=torch.float32)
        return {"logits": z + bias}
    if cfg.routing == "uniform_ids":
        ids = torch.randint(0, cfg.E, (T, cfg.topk), generator=g, device=device, dtype=torch.int64)
        return {"topk_ids": ids.to(torch.int32), "topk_weights": _choice_weights(cfg, T, g, device)}
    if cfg.routing == "zipf":
        rank = torch.arange(1, cfg.E + 1, device=device, dtype=torch.float64)
        logp = -cfg.zipf_s * torch.log(rank)
        u = torch.rand((T, cfg.E), generator=g, device=device, dtype=torch.float64)
        u = u.clamp(1e-300, 1.0 - 1e-16)
        gumbel = -torch.log(-torch.log(u))
        ids = torch.topk(logp + gumbel, cfg.topk, dim=-1).indices
        return {"topk_ids": ids.to(torch.int32), "topk_weights": _choice_weights(cfg, T, g, device)}
    raise ValueError(f"unknown routing recipe {cfg.routing!r}")


def make_custom_config(name="custom", **kw) -> MoEConfig:
    base = dict(E=8, topk=2, H=256, I=128, fp8=False, routing="logits", tokens=(16,))
    base.update(kw)
    return MoEConfig(name, **base)
