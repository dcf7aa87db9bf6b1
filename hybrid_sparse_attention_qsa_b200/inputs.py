"""Seeded synthetic inputs for the QSA hot path.

This module is shared by the tests, the benchmark and the oracle checks.  It holds none of the
method's arithmetic (no pooling, scoring, selection or attention): it only draws tensors.

Recipe (the same for every workload):
  * one ``torch.Generator`` on the target device, seeded with the workload's seed;
  * tensors are drawn in the order q, k, v, qi, ki as fp32 N(0, 1), divided by sqrt(last dim)
    (128 for q/k/v, 64 for the indexer tensors) and rounded to bf16;
  * the long-prefill workload then picks floor(boost_frac * T) token positions without
    replacement (``randperm`` from the same generator) and multiplies the k and ki rows at those
    positions by ``boost`` (x4 is exact in bf16), which gives peaked indexer scores;
  * large tensors are drawn in chunks of at most ``_CHUNK`` elements so that the fp32 staging
    buffer stays small; the chunking is part of the recipe, so a given (workload, device) pair
    always yields the same bytes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np
import torch

_CHUNK = 1 << 26


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" or "decode"
    B: int
    T: int               # prefill length, or cache length L for decode
    Hq: int
    Hkv: int
    D: int
    Hi: int
    Di: int
    blk: int
    k: int
    seed: int
    boost_frac: float = 0.0
    boost: float = 1.0

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", "prefill", B=1, T=2048, Hq=1, Hkv=1, D=128, Hi=1, Di=64, blk=4, k=64, seed=0),
    "prefill_32k": Workload("prefill_32k", "prefill", B=1, T=32768, Hq=16, Hkv=2, D=128, Hi=4, Di=64, blk=4,
                            k=512, seed=1),
    "prefill_128k": Workload("prefill_128k", "prefill", B=1, T=131072, Hq=16, Hkv=2, D=128, Hi=4, Di=64, blk=4,
                             k=512, seed=2, boost_frac=0.05, boost=4.0),
    "decode_256k": Workload("decode_256k", "decode", B=32, T=262144, Hq=16, Hkv=2, D=128, Hi=4, Di=64, blk=4,
                            k=512, seed=3),
    "prefill_1m": Workload("prefill_1m", "prefill", B=1, T=1048576, Hq=16, Hkv=2, D=128, Hi=4, Di=64, blk=4,
                           k=1024, seed=4),
    "decode_1m": Workload("decode_1m", "decode", B=8, T=1048576, Hq=16, Hkv=2, D=128, Hi=4, Di=64, blk=4,
                          k=1024, seed=6),
    # a small decode batch (4 sequences x 64K, caches of 268 MB: larger than L2) for profiling runs
    "decode_64k_b4": Workload("decode_64k_b4", "decode", B=4, T=65536, Hq=16, Hkv=2, D=128, Hi=4, Di=64, blk=4,
                              k=512, seed=8),
    # the attention shape of the model on the pages (24 query heads over 2 KV heads at head
    # dimension 256) with the 128K recipe otherwise
    "prefill_128k_model": Workload("prefill_128k_model", "prefill", B=1, T=131072, Hq=24, Hkv=2, D=256, Hi=4, Di=64,
                                   blk=4, k=512, seed=5, boost_frac=0.05, boost=4.0),
    "prefill_32k_model": Workload("prefill_32k_model", "prefill", B=1, T=32768, Hq=24, Hkv=2, D=256, Hi=4, Di=64,
                                  blk=4, k=512, seed=7, boost_frac=0.05, boost=4.0),
}


def _randn_bf16(gen: torch.Generator, shape, device) -> torch.Tensor:
    """N(0,1)/sqrt(shape[-1]) in fp32, rounded to bf16, drawn in fixed-size chunks."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    inv = 1.0 / math.sqrt(shape[-1])
    for s in range(0, flat.numel(), _CHUNK):
        e = min(s + _CHUNK, flat.numel())
        tmp = torch.randn(e - s, generator=gen, dtype=torch.float32, device=device)
        tmp.mul_(inv)
        flat[s:e].copy_(tmp)
        del tmp
    return out


def make_prefill(w: Workload, device="cpu") -> dict:
    """q [B,T,Hq,D], k/v [B,T,Hkv,D], qi [B,T,Hi,Di], ki [B,T,Di], all bf16."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    q = _randn_bf16(g, (w.B, w.T, w.Hq, w.D), device)
    k = _randn_bf16(g, (w.B, w.T, w.Hkv, w.D), device)
    v = _randn_bf16(g, (w.B, w.T, w.Hkv, w.D), device)
    qi = _randn_bf16(g, (w.B, w.T, w.Hi, w.Di), device)
    ki = _randn_bf16(g, (w.B, w.T, w.Di), device)
    if w.boost_frac > 0:
        nboost = int(math.floor(w.boost_frac * w.T))
        for b in range(w.B):
            pos = torch.randperm(w.T, generator=g, device=device)[:nboost]
            k[b, pos] *= w.boost
            ki[b, pos] *= w.boost
    return dict(q=q, k=k, v=v, qi=qi, ki=ki)


def make_decode(w: Workload, device="cpu", seqlens=None) -> dict:
    """One decode step: q [B,Hq,D], caches k/v [B,L,Hkv,D], qi [B,Hi,Di], ki cache [B,L,Di],
    seqlens [B] int32 (the new token included; all equal to L unless given)."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    q = _randn_bf16(g, (w.B, w.Hq, w.D), device)
    k = _randn_bf16(g, (w.B, w.T, w.Hkv, w.D), device)
    v = _randn_bf16(g, (w.B, w.T, w.Hkv, w.D), device)
    qi = _randn_bf16(g, (w.B, w.Hi, w.Di), device)
    ki = _randn_bf16(g, (w.B, w.T, w.Di), device)
    if seqlens is None:
        seqlens = torch.full((w.B,), w.T, dtype=torch.int32, device=device)
    else:
        seqlens = torch.as_tensor(seqlens, dtype=torch.int32, device=device)
    return dict(q=q, k=k, v=v, qi=qi, ki=ki, seqlens=seqlens)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> its uint16 bit patterns as a host numpy array (copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(a: np.ndarray, device="cpu") -> torch.Tensor:
    """uint16 bit patterns -> bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
