"""Seeded synthetic inputs shaped like the workloads the SageAttention2 / 2++ pages
measure (LLM prefill, image and video diffusion transformers).

This module holds no arithmetic of the attention method: it only draws random
tensors.  Both the CUDA path (tests, benchmark) and the oracle side of the tests
use it, so that the two sides see identical inputs.

Variance reading: "N(0, s)" in a workload description is read as variance s
(standard deviation sqrt(s)).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

SEED_BASE = 1234


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N_q: int
    N_kv: int
    d: int
    causal: bool
    dtype: torch.dtype
    seed: int
    recipe: str
    H_kv: int = 0   # key/value heads (grouped-query attention); 0 means H (multi-head)
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def Hk(self) -> int:
        return self.H_kv or self.H

    def ops(self) -> float:
        """Algorithmic tensor ops 4 B H Nq Nkv d (QK^T and PV, 2 ops per MAC), halved if causal."""
        o = 4.0 * self.B * self.H * self.N_q * self.N_kv * self.d
        return o / 2.0 if self.causal else o

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "H_kv": self.Hk, "N_q": self.N_q,
                "N_kv": self.N_kv, "d": self.d, "causal": self.causal, "dtype": str(self.dtype).replace("torch.", ""),
                "seed": self.seed, "recipe": self.recipe}


# The five workload families, in a fixed order that also fixes their seeds.
TINY = Workload("tiny", 1, 2, 256, 256, 64, False, torch.float16, SEED_BASE + 0, "tiny")
IMAGE_DIT = Workload("image_dit", 2, 16, 4096, 4096, 128, False, torch.bfloat16, SEED_BASE + 1, "image_dit")
LLM_PREFILL = Workload("llm_prefill", 1, 32, 32768, 32768, 128, True, torch.bfloat16, SEED_BASE + 2, "llm")
VIDEO_DIT = Workload("video_dit", 2, 48, 17776, 17776, 64, False, torch.bfloat16, SEED_BASE + 3, "video_dit")
# LLM prefill with grouped-query attention: 32 query heads over 8 key/value heads
LLM_PREFILL_GQA = Workload("llm_prefill_gqa", 1, 32, 32768, 32768, 128, True, torch.bfloat16, SEED_BASE + 5, "llm",
                           H_kv=8)

WORKLOADS = {w.name: w for w in (TINY, IMAGE_DIT, LLM_PREFILL, VIDEO_DIT, LLM_PREFILL_GQA)}

SWEEP_N = (1024, 2048, 4096, 8192, 16384, 32768, 65536)


def sweep_point(n: int, d: int, causal: bool) -> Workload:
    idx = SWEEP_N.index(n) * 4 + (0 if d == 64 else 2) + (1 if causal else 0)
    return Workload("sweep_n%d_d%d_%s" % (n, d, "causal" if causal else "full"), 1, 32, n, n, d, causal,
                    torch.bfloat16, SEED_BASE + 4 + 1000 * (idx + 1), "sweep")


def by_name(name: str) -> Workload:
    """A named workload: one of WORKLOADS, or a sweep point 'sweep_n<N>_d<d>_<causal|full>'."""
    if name in WORKLOADS:
        return WORKLOADS[name]
    if name.startswith("sweep_"):
        parts = name.split("_")
        n, d, kind = int(parts[1][1:]), int(parts[2][1:]), parts[3]
        if n in SWEEP_N and d in (64, 128) and kind in ("causal", "full"):
            return sweep_point(n, d, kind == "causal")
    raise KeyError("unknown workload %r" % name)


def custom(name, B, H, N_q, N_kv, d, causal, dtype=torch.bfloat16, seed=SEED_BASE + 99, recipe="image_dit", H_kv=0):
    """A workload with the value recipe of one of the families but other sizes (tests)."""
    return Workload(name, B, H, N_q, N_kv, d, causal, dtype, seed, recipe, H_kv=H_kv)


def _rope(x: torch.Tensor, base: float = 10000.0) -> torch.Tensor:
    """Rotate-half rotary position rotation by token position along dim -2 ([B, H, N, d])."""
    n, d = x.shape[-2], x.shape[-1]
    half = d // 2
    inv = base ** (-torch.arange(0, half, dtype=torch.float64) * 2.0 / d)
    ang = torch.arange(n, dtype=torch.float64)[:, None] * inv[None, :]
    cos, sin = torch.cos(ang).float(), torch.sin(ang).float()
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1)


def generate(w: Workload):
    """Q [B,H,Nq,d], K, V [B,H_kv,Nkv,d] on the CPU, head-major, in the workload dtype."""
    g = torch.Generator().manual_seed(w.seed)
    B, H, Hk, nq, nk, d = w.B, w.H, w.Hk, w.N_q, w.N_kv, w.d
    q = torch.randn((B, H, nq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, Hk, nk, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hk, nk, d), generator=g, dtype=torch.float32)
    if w.recipe == "tiny":
        # per-channel K offset, variance 4, shared across tokens
        k += math.sqrt(4.0) * torch.randn((B, Hk, 1, d), generator=g)
    elif w.recipe == "image_dit":
        k += math.sqrt(8.0) * torch.randn((B, Hk, 1, d), generator=g)
        mask = torch.rand((B, H, nq, d), generator=g) < 0.01
        q = torch.where(mask, q * 20.0, q)
    elif w.recipe == "llm":
        k += math.sqrt(5.0) * torch.randn((B, Hk, 1, d), generator=g)
        q = _rope(q)
        k = _rope(k)
    elif w.recipe == "video_dit":
        k += math.sqrt(10.0) * torch.randn((B, Hk, 1, d), generator=g)
        log_std = torch.rand((B, Hk, 1, d), generator=g) * 3.0 - 2.0     # U(-2, 1)
        v = v * torch.pow(10.0, log_std)
    elif w.recipe == "sweep":
        k += math.sqrt(5.0) * torch.randn((B, Hk, 1, d), generator=g)
        mask = torch.rand((B, H, nq, d), generator=g) < 0.01
        q = torch.where(mask, q * 20.0, q)
    else:
        raise ValueError("unknown recipe %r" % w.recipe)
    return q.to(w.dtype), k.to(w.dtype), v.to(w.dtype)


def to_nhd(x: torch.Tensor) -> torch.Tensor:
    """[B, H, N, d] -> contiguous token-major [B, N, H, d]."""
    return x.permute(0, 2, 1, 3).contiguous()
