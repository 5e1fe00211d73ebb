"""Seeded synthetic inputs for zigzag context-parallel attention.

This module holds no attention arithmetic: it only draws the inputs that both
the oracle and the CUDA library consume, so the two sides see identical data.

Workloads (sequence lengths, head counts, cp sizes, orders and the packed
document mix) follow the long-context settings of the Accelerate "Context
Parallel" concept guide (128k tokens, cp 8, all-gather or ring rotation) and a
Llama-3-8B-shaped GQA attention (32 query / 8 KV heads, head dim 128).

Draw recipe (one torch CPU generator per call, seeded):
  Q, K, V, dO drawn in that order with ``torch.randn`` in fp32, shape
  [B, H, S, D] in ORIGINAL token order, multiplied by ``amp`` and rounded to
  bf16 (round-to-nearest-even by ``Tensor.to``).
Document lengths: numpy ``default_rng(seed).lognormal(ln(median), sigma)``,
rounded with ``rint``, clipped to [lo, hi], then (for per-document sharding,
whose chunks must be whole 128-row tiles) rounded to the nearest multiple of
``quantum`` (at least one quantum), drawn one at a time until their sum reaches
S; the last document is cut so the lengths sum to exactly S.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seq_len: int
    cp: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    rotate: str                      # "allgather" | "ring"
    amp: float = 1.0                 # multiplier on the N(0,1) draw
    docs: bool = False               # packed-document mask
    backward: bool = True
    seed: int = 0
    doc_median: float = 2048.0
    doc_sigma: float = 1.0
    doc_clip: tuple = (128, 32768)
    shard: str = "sequence"          # "sequence" | "doc" (per-document zigzag)
    doc_quantum: int = 1             # document lengths a multiple of this
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 512, 2, 2, 2, 64, "allgather", backward=False, seed=0),
    "fb8k": Workload("fb8k", 1, 8192, 4, 8, 8, 128, "allgather", seed=1),
    "gqa32k": Workload("gqa32k", 1, 32768, 8, 32, 8, 128, "ring", amp=0.5, seed=2),
    "docs64k": Workload("docs64k", 1, 65536, 8, 32, 8, 128, "ring", docs=True, seed=3),
    "long128k": Workload("long128k", 1, 131072, 8, 32, 8, 128, "allgather", seed=4),
    # gqa32k at head_dim 256
    "gqa32k_d256": Workload("gqa32k_d256", 1, 32768, 8, 32, 8, 256, "ring", amp=0.5, seed=5),
    # the docs64k mix with every document cut into 2cp chunks of whole 128-row tiles
    "docs64k_perdoc": Workload("docs64k_perdoc", 1, 65536, 8, 32, 8, 128, "ring", docs=True,
                               seed=3, shard="doc", doc_quantum=2048),
}


def doc_lengths(seq_len: int, seed: int, median: float = 2048.0, sigma: float = 1.0,
                clip: tuple = (128, 32768), quantum: int = 1) -> list[int]:
    """Seeded lognormal document lengths summing to exactly ``seq_len``, each a
    multiple of ``quantum`` (``seq_len`` must then be one too)."""
    if quantum < 1 or seq_len % quantum:
        raise ValueError(f"seq_len {seq_len} is not a multiple of quantum {quantum}")
    rng = np.random.default_rng(seed)
    lens: list[int] = []
    total = 0
    while total < seq_len:
        x = float(rng.lognormal(mean=math.log(median), sigma=sigma))
        n = int(np.clip(np.rint(x), clip[0], clip[1]))
        if quantum > 1:
            n = max(quantum, int(np.rint(n / quantum)) * quantum)
        lens.append(n)
        total += n
    lens[-1] -= total - seq_len
    if lens[-1] == 0:
        lens.pop()
    return lens


def cu_seqlens(lengths) -> np.ndarray:
    """Offsets [0, l0, l0+l1, ...] as int32."""
    out = np.zeros(len(lengths) + 1, dtype=np.int64)
    out[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return out.astype(np.int32)


def attn_inputs(batch: int, num_heads: int, num_kv_heads: int, seq_len: int, head_dim: int,
                seed: int, amp: float = 1.0, with_dout: bool = True,
                device: str | torch.device = "cpu") -> dict:
    """Q [B,Hq,S,D], K/V [B,Hkv,S,D] and optionally dO [B,Hq,S,D], bf16, original order.

    On a CUDA device the draw uses a CUDA generator (same recipe, different stream
    of numbers); parity tests draw on the CPU so the oracle sees identical values.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)

    def draw(h):
        x = torch.randn((batch, h, seq_len, head_dim), generator=gen, dtype=torch.float32,
                        device=device)
        if amp != 1.0:
            x.mul_(amp)
        return x.to(torch.bfloat16)

    out = {"q": draw(num_heads), "k": draw(num_kv_heads), "v": draw(num_kv_heads)}
    if with_dout:
        out["do"] = draw(num_heads)
    return out


def workload_inputs(w: Workload, device="cpu", with_dout=None) -> dict:
    """Inputs of a named workload plus its cu_seqlens (None for the plain causal mask)."""
    wd = w.backward if with_dout is None else with_dout
    t = attn_inputs(w.batch, w.num_heads, w.num_kv_heads, w.seq_len, w.head_dim, w.seed,
                    amp=w.amp, with_dout=wd, device=device)
    t["cu_seqlens"] = (cu_seqlens(doc_lengths(w.seq_len, w.seed, w.doc_median, w.doc_sigma,
                                              w.doc_clip, w.doc_quantum)) if w.docs else None)
    return t
