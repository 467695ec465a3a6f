"""Seeded synthetic inputs for the CONF-KV decode step.

Draws the tensors a model would hand the cache manager: prompt K/V, the new
token's q/k/v each step, next-token logits and (fixed-budget mode) static
priorities. It holds none of the method's arithmetic; tests feed the same
bytes to the CUDA library and to the CPU oracle.

Recipe (the pages give no workload data, so these stand in for it):

* q, k, v: fp16 samples of N(0, 1).
* heavy hitters: each key (per layer, sequence, KV head and token, prompt and
  decode alike) is scaled by 4 with probability 0.01, independently; values
  are not scaled.
* logits: fp32 N(0, 1) times a per-(sequence, step) scale that is 8
  ("confident" regime) with probability 0.7 and 0.5 otherwise.
* priorities: fp32 U(0, 1) per token and KV head.

Every draw comes from a torch.Generator seeded by the caller, so the bytes are
reproducible on one device type.
"""
from __future__ import annotations

import torch

HEAVY_FRACTION = 0.01
HEAVY_SCALE = 4.0
CONFIDENT_SCALE = 8.0
UNCERTAIN_SCALE = 0.5
CONFIDENT_PROB = 0.7


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_fp16(shape, gen, device="cpu") -> torch.Tensor:
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.float16)


def keys_with_heavy_hitters(shape, gen, device="cpu") -> torch.Tensor:
    """fp16 N(0,1) keys of shape [..., T, D]; each row scaled x4 w.p. 0.01."""
    k = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    heavy = torch.rand(shape[:-1], generator=gen, device=device) < HEAVY_FRACTION
    k = torch.where(heavy[..., None], k * HEAVY_SCALE, k)
    return k.to(torch.float16)


def prefill_kv(B, Hkv, T, D, gen, device="cpu"):
    """Prompt K and V for one layer, [B, Hkv, T, D] fp16."""
    k = keys_with_heavy_hitters((B, Hkv, T, D), gen, device)
    v = normal_fp16((B, Hkv, T, D), gen, device)
    return k, v


def step_qkv(lead, Hq, Hkv, D, gen, device="cpu"):
    """New-token q [*lead, Hq, D], k/v [*lead, Hkv, D] fp16 (lead = (B,) or (L, B))."""
    lead = tuple(lead)
    q = normal_fp16(lead + (Hq, D), gen, device)
    k = keys_with_heavy_hitters(lead + (Hkv, 1, D), gen, device).reshape(lead + (Hkv, D))
    v = normal_fp16(lead + (Hkv, D), gen, device)
    return q, k, v


def bursty_logits(B, V, gen, device="cpu") -> torch.Tensor:
    """fp32 logits [B, V]: N(0,1) times 8 (p = 0.7) or 0.5 per row."""
    confident = torch.rand((B, 1), generator=gen, device=device) < CONFIDENT_PROB
    scale = torch.where(confident, torch.tensor(CONFIDENT_SCALE, device=device),
                        torch.tensor(UNCERTAIN_SCALE, device=device))
    return torch.randn((B, V), generator=gen, device=device, dtype=torch.float32) * scale


def priorities(shape, gen, device="cpu") -> torch.Tensor:
    """fp32 U(0, 1) static priorities."""
    return torch.rand(shape, generator=gen, device=device, dtype=torch.float32)
