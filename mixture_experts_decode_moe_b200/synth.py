"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers and lays them out in the library's
storage formats; it contains none of the MoE arithmetic. Both the tests'
oracle side and the CUDA side take their inputs from here. Streams are a
function of (seed, device): weights use seed 1000*workload + layer,
activations and scores use that seed + 500.

Workloads (the pages' shapes; weights are random, no trained checkpoint):
  tiny          H=512, E=16, k=2, I=256, bf16 N(0, 0.02), router N(0, 0.02),
                64 tokens x ~ N(0, 1), seed 0.
  a3b_bf16      40 layers, H=2048, E=256, k=8, I=512 + shared I=512, bf16
                N(0, 0.02) per layer, router N(0, 0.02) * 0.1 (near-uniform
                routing), 256 tokens x ~ N(0, 1).  (Table 3 "Qwen3.5" row of
                the arXiv:2610.37386 review; "256, 8 (+1 shared)" in "Mixture
                of Experts Changes the Arithmetic".)
  batch_sweep   E=64 LINEAR experts, each one 8192x8192 bf16 N(0, 0.02); k=3
                distinct ids uniform per token; B in {1,4,16,64,256}.
                ("5,010억 개 중 230억 개만 켠다", §3 [A]/[B].)
  a3b_int4      a3b shapes, expert codes int4 q = clamp(rint(w0/s), -8, 7),
                w0 ~ N(0, 0.02), s ~ U(0.005, 0.03) as bf16, groups of 64
                along the input dim; shared, router bf16; B in {1, 8}.
  channel_topk  48 layers, H=2048, E=128, k=8, I=768 channel-major bf16
                N(0, 0.02); router N(0, 0.02); scores |N(0,1)| x a
                Pareto(alpha=1.5, x_m=1) scale per (layer, expert, channel);
                keep 13% or 18% of 6144 candidates. (Table 3 "Qwen3-Thinking".)
"""

from __future__ import annotations

import math

import torch

WORKLOADS = {
    "tiny": dict(cfg=1, H=512, E=16, k=2, I=256, I_shared=0, layers=1, tokens=64, router_scale=1.0),
    "a3b_bf16": dict(cfg=2, H=2048, E=256, k=8, I=512, I_shared=512, layers=40, tokens=256, router_scale=0.1),
    "batch_sweep": dict(cfg=3, H=8192, E=64, k=3, batches=(1, 4, 16, 64, 256)),
    "a3b_int4": dict(cfg=4, H=2048, E=256, k=8, I=512, I_shared=512, layers=40, batches=(1, 8),
                     router_scale=0.1),
    "channel_topk": dict(cfg=5, H=2048, E=128, k=8, I=768, layers=48, keep_frac=(0.13, 0.18)),
}

W_STD = 0.02


def weight_seed(cfg: int, layer: int) -> int:
    return 1000 * cfg + layer


def act_seed(cfg: int, layer: int = 0) -> int:
    return 1000 * cfg + layer + 500


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_bf16(shape, std: float, g: torch.Generator, device) -> torch.Tensor:
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return t.mul_(std).to(torch.bfloat16)


def tokens(B: int, H: int, seed: int, device="cpu") -> torch.Tensor:
    """x ~ N(0, 1) rounded to bf16, [B, H]."""
    return normal_bf16((B, H), 1.0, _gen(seed, device), device)


def uniform_ids(B: int, E: int, k: int, seed: int, device="cpu") -> torch.Tensor:
    """k distinct expert ids per token, uniform over E, int32 [B, k]."""
    g = _gen(seed, device)
    u = torch.rand((B, E), generator=g, device=device)
    return u.argsort(dim=1)[:, :k].to(torch.int32).contiguous()


def _chunked_normal(shape, std, g, device):
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(shape[0], -1)
    for i in range(shape[0]):
        flat[i].copy_(torch.randn(flat.shape[1], generator=g, device=device).mul_(std))
    return out


def swiglu_layer_bf16(H, E, I, I_shared, seed, device="cpu", router_scale=1.0):
    """Planar bf16 SwiGLU layer: router [E,H], gate/up/down_t [E,I,H], shared [I_sh,H]."""
    g = _gen(seed, device)
    L = {"router": normal_bf16((E, H), W_STD * router_scale, g, device)}
    for name in ("gate", "up", "down_t"):
        L[name] = _chunked_normal((E, I, H), W_STD, g, device)
    if I_shared:
        for name in ("sh_gate", "sh_up", "sh_down_t"):
            L[name] = normal_bf16((I_shared, H), W_STD, g, device)
    return L


def _pack_int4(q: torch.Tensor) -> torch.Tensor:
    """Two's-complement nibbles, element 2i low, 2i+1 high -> uint8 [..., n/2]."""
    q = (q.to(torch.int16) & 0xF).to(torch.uint8)
    return (q[..., 0::2] | (q[..., 1::2] << 4)).contiguous()


def _int4_codes(w0: torch.Tensor, s: torch.Tensor) -> torch.Tensor:
    return torch.clamp(torch.round(w0 / s), -8, 7)


def swiglu_layer_int4(H, E, I, I_shared, seed, device="cpu", router_scale=1.0):
    """int4 group-64 experts (codes + bf16 scales), bf16 router and shared expert."""
    g = _gen(seed, device)
    L = {"router": normal_bf16((E, H), W_STD * router_scale, g, device)}
    for name in ("gate", "up"):
        codes = torch.empty((E, I, H // 2), dtype=torch.uint8, device=device)
        scales = torch.empty((E, I, H // 64), dtype=torch.bfloat16, device=device)
        for e in range(E):
            w0 = torch.randn((I, H), generator=g, device=device).mul_(W_STD)
            s = torch.empty((I, H // 64), device=device).uniform_(0.005, 0.03, generator=g).to(torch.bfloat16)
            codes[e] = _pack_int4(_int4_codes(w0, s.float().repeat_interleave(64, dim=1)))
            scales[e] = s
        L[name], L[name + "_s"] = codes, scales
    codes = torch.empty((E, I, H // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((E, I // 64, H), dtype=torch.bfloat16, device=device)
    for e in range(E):
        w0 = torch.randn((I, H), generator=g, device=device).mul_(W_STD)
        s = torch.empty((I // 64, H), device=device).uniform_(0.005, 0.03, generator=g).to(torch.bfloat16)
        codes[e] = _pack_int4(_int4_codes(w0, s.float().repeat_interleave(64, dim=0)))
        scales[e] = s
    L["down_t"], L["down_s"] = codes, scales
    if I_shared:
        for name in ("sh_gate", "sh_up", "sh_down_t"):
            L[name] = normal_bf16((I_shared, H), W_STD, g, device)
    return L


def channel_major_layer(H, E, I, seed, device="cpu", router_scale=1.0):
    """Channel-major bf16 experts [E, I, 3, H] (gate row, up row, down column) + router."""
    g = _gen(seed, device)
    router = normal_bf16((E, H), W_STD * router_scale, g, device)
    return {"router": router, "cm": _chunked_normal((E, I, 3, H), W_STD, g, device)}


def channel_major_layer_lowrank(H, E, I, seed, rank=32, noise=0.3, device="cpu", router_scale=1.0):
    """Channel-major layer like channel_major_layer, except that the down
    columns share a planted rank-`rank` subspace: d = W_STD (sqrt(1 - noise^2)
    B z + noise eps), B [H, rank] with orthonormal columns scaled by
    sqrt(H / rank), z ~ N(0, I_rank), eps ~ N(0, I_H) per channel, so each
    coordinate still has standard deviation W_STD and a fraction of about
    1 - noise^2 of each column's energy lies in span(B). Stands in for trained
    down projections, whose columns concentrate in few directions."""
    g = _gen(seed, device)
    router = normal_bf16((E, H), W_STD * router_scale, g, device)
    gu = _chunked_normal((E, I, 2, H), W_STD, g, device)
    q, _ = torch.linalg.qr(torch.randn((H, rank), generator=g, device=device, dtype=torch.float32))
    basis = q * (H / rank) ** 0.5
    z = torch.randn((E * I, rank), generator=g, device=device)
    eps = torch.randn((E * I, H), generator=g, device=device)
    d = W_STD * ((1.0 - noise * noise) ** 0.5 * (z @ basis.T) + noise * eps)
    cm = torch.cat([gu, d.to(torch.bfloat16).view(E, I, 1, H)], dim=2).contiguous()
    return {"router": router, "cm": cm, "basis": basis}


def channel_scale(E, I, seed, device="cpu") -> torch.Tensor:
    """Per-channel Pareto(alpha=1.5, x_m=1) scale: U^(-1/1.5), U ~ U(0, 1]."""
    g = _gen(seed, device)
    u = 1.0 - torch.rand((E, I), generator=g, device=device)  # (0, 1]
    return u.pow(-1.0 / 1.5)


def channel_scores(B, E, I, scale: torch.Tensor, seed, device="cpu") -> torch.Tensor:
    """scores[b, e, c] = |N(0, 1)| * scale[e, c], fp32 [B, E, I]."""
    g = _gen(seed, device)
    z = torch.randn((B, E, I), generator=g, device=device).abs_()
    return (z * scale.to(device)).contiguous()


def reader_signs(H: int, seed: int, device="cpu") -> torch.Tensor:
    """The channel screen's random rotation signs: H values of +-1, int8."""
    g = _gen(seed, device)
    return (torch.randint(0, 2, (H,), generator=g, device=device, dtype=torch.int8) * 2 - 1).to(torch.int8)


def router_weights(B: int, k: int, seed: int, device="cpu") -> torch.Tensor:
    """Positive per-slot expert weights U(0.05, 1), fp32 [B, k] (an input
    of the screen; the screen does not require them to sum to 1)."""
    g = _gen(seed, device)
    return (0.05 + 0.95 * torch.rand((B, k), generator=g, device=device)).contiguous()


def linear_experts(E, H, seed, device="cpu") -> torch.Tensor:
    """E expert matrices [E, H, H] bf16 N(0, 0.02)."""
    return _chunked_normal((E, H, H), W_STD, _gen(seed, device), device)


def keep_count(frac: float, k: int, I: int) -> int:
    """Kept channels for a budget fraction of the k*I candidates (nearest)."""
    return int(math.floor(frac * k * I + 0.5))
