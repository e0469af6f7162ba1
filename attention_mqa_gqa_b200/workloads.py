"""Seeded synthetic inputs for the attention workloads.

This module only draws random numbers and lays them out; it holds none of
the attention arithmetic.  It is the one module shared by the CUDA path's
tests/bench and the CPU oracle: both receive the same tensors.

Recipe (every workload): a CPU ``torch.Generator`` seeded with the
workload's seed draws, in this order, the per-sequence KV lengths
(``randint(lo, hi + 1)``), then Q, then K (or the latent cache), then V, each
as N(0, 1) float32 rounded once to the workload's element type.  The KV
tensors hold ``max(lengths)`` rows per sequence; rows past a sequence's
length are ordinary finite draws that the attention ignores.

Layouts follow [B, H, S, d] with the innermost dimension contiguous.  In the
MLA-absorbed workload the cache is one tensor [B, S, 576] (rows
[c_kv (512) | k_pe (64)]), exposed as ``k`` = cache[:, None] and ``v`` = the
first 512 columns of the same storage (a strided view, no copy).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    skv_lo: int
    skv_hi: int
    d_k: int
    d_v: int
    dtype: torch.dtype
    causal: bool
    scale: float
    mla: bool
    seed: int
    topk: int = 0  # > 0: attention over at most topk selected positions per sequence

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def is_decode(self) -> bool:
        """Runs on the split-KV decode path and is bound by reading the KV
        cache: one query per sequence, or a few (a power of two up to 16 at
        head dim 128 or 512: extend / speculative-decoding verification)."""
        if self.Sq == 1 or self.topk:
            return True
        return (self.d_k in (128, 512) and self.d_k == self.d_v and self.Sq <= 16
                and self.Sq & (self.Sq - 1) == 0)

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


# The workloads: MQA d=512 prefill (tiny, fp16) and decode, MQA d=512
# prefill, GQA 64/8 d=128 decode and prefill, absorbed-MLA decode, and
# expanded-MLA prefill (d_k = 192, d_v = 128).
WORKLOADS = {
    "mqa_prefill_tiny": Workload("mqa_prefill_tiny", 1, 16, 1, 128, 128, 128, 512, 512,
                                 torch.float16, True, 1 / math.sqrt(512), False, 0),
    "mqa_decode": Workload("mqa_decode", 32, 16, 1, 1, 1024, 8192, 512, 512,
                           torch.bfloat16, True, 1 / math.sqrt(512), False, 1),
    "mqa_prefill": Workload("mqa_prefill", 2, 16, 1, 4096, 4096, 4096, 512, 512,
                            torch.bfloat16, True, 1 / math.sqrt(512), False, 2),
    "gqa_decode": Workload("gqa_decode", 64, 64, 8, 1, 4096, 4096, 128, 128,
                           torch.bfloat16, True, 1 / math.sqrt(128), False, 3),
    "gqa_prefill": Workload("gqa_prefill", 1, 64, 8, 8192, 8192, 8192, 128, 128,
                            torch.bfloat16, True, 1 / math.sqrt(128), False, 3),
    "mla_decode": Workload("mla_decode", 64, 128, 1, 1, 4096, 16384, 576, 512,
                           torch.bfloat16, True, 1 / math.sqrt(192), True, 4),
    # speculative-decoding verify step: 4 queries per sequence against the cache
    "gqa_extend": Workload("gqa_extend", 64, 64, 8, 4, 4096, 4096, 128, 128,
                           torch.bfloat16, True, 1 / math.sqrt(128), False, 6),
    # DSA-style sparse decode over the absorbed-MLA cache: per sequence 2048
    # of 16K-48K cached positions are selected (the selection is an input)
    "mla_topk_decode": Workload("mla_topk_decode", 64, 128, 1, 1, 16384, 49152, 576, 512,
                                torch.bfloat16, True, 1 / math.sqrt(192), True, 7, topk=2048),
    # MLA prefill in the expanded (MHA) form: 128 heads, q/k head dim 192
    # (128 nope + 64 rope columns, already rotated), v head dim 128
    "mla_prefill": Workload("mla_prefill", 1, 128, 128, 4096, 4096, 4096, 192, 128,
                            torch.bfloat16, True, 1 / math.sqrt(192), False, 5),
}


def _randn_into(t: torch.Tensor, g: torch.Generator, rows_per_chunk: int = 1 << 22) -> None:
    """Fill ``t`` (any float dtype, contiguous) with N(0,1) float32 draws
    rounded once to t.dtype, drawn in row-major order in bounded chunks."""
    flat = t.view(-1)
    n = flat.numel()
    step = rows_per_chunk
    for s in range(0, n, step):
        e = min(n, s + step)
        flat[s:e].copy_(torch.randn(e - s, generator=g, dtype=torch.float32))


def make_selection(skv, topk: int, g: torch.Generator):
    """Stand-in for an indexer's top-k choice: per sequence, min(topk, skv[b])
    distinct positions of [0, skv[b]) drawn uniformly, in ascending order.
    Returns (idx int32 [B, topk] -- unused slots 0 --, n_sel int32 [B])."""
    B = len(skv)
    idx = torch.zeros(B, topk, dtype=torch.int32)
    n_sel = torch.zeros(B, dtype=torch.int32)
    for b in range(B):
        L = int(skv[b])
        n = min(topk, L)
        if n:
            idx[b, :n] = torch.randperm(L, generator=g)[:n].sort().values.to(torch.int32)
        n_sel[b] = n
    return idx, n_sel


def make_inputs(w: Workload, skv_override=None) -> dict:
    """Draw the inputs of workload ``w`` on the CPU.

    Returns a dict with q, k, v (CPU tensors of w.dtype), skv (int32 [B]),
    max_skv, for MLA the backing ``cache`` tensor, and for a top-k workload
    the selection ``idx`` (int32 [B, topk]) and ``n_sel`` (int32 [B])."""
    g = torch.Generator().manual_seed(w.seed)
    skv = torch.randint(w.skv_lo, w.skv_hi + 1, (w.B,), generator=g, dtype=torch.int64)
    if skv_override is not None:
        skv = torch.as_tensor(skv_override, dtype=torch.int64)
    skv = skv.to(torch.int32)
    S = max(int(skv.max()), 1)
    q = torch.empty(w.B, w.Hq, w.Sq, w.d_k, dtype=w.dtype)
    _randn_into(q, g)
    out = {"skv": skv, "max_skv": S, "q": q}
    if w.mla:
        cache = torch.empty(w.B, S, w.d_k, dtype=w.dtype)
        _randn_into(cache, g)
        out["cache"] = cache
        out["k"] = cache.view(w.B, 1, S, w.d_k)
        out["v"] = cache.view(w.B, 1, S, w.d_k)[..., : w.d_v]
    else:
        k = torch.empty(w.B, w.Hkv, S, w.d_k, dtype=w.dtype)
        _randn_into(k, g)
        v = torch.empty(w.B, w.Hkv, S, w.d_v, dtype=w.dtype)
        _randn_into(v, g)
        out["k"], out["v"] = k, v
    if w.topk:
        out["idx"], out["n_sel"] = make_selection(skv.tolist(), w.topk, g)
    return out


def make_case(B, Hq, Hkv, Sq, skv, d_k, d_v, dtype=torch.bfloat16, causal=True,
              scale=None, mla=False, seed=0, max_skv=None) -> tuple[Workload, dict]:
    """A small ad-hoc case with explicit per-sequence lengths ``skv`` (list)."""
    skv = list(skv)
    w = Workload(f"case_{B}x{Hq}x{Hkv}x{Sq}", B, Hq, Hkv, Sq, min(skv), max(skv), d_k, d_v,
                 dtype, causal, scale if scale is not None else 1 / math.sqrt(d_k), mla, seed)
    g = torch.Generator().manual_seed(seed)
    S = max(max(skv), 1) if max_skv is None else max_skv
    q = torch.empty(B, Hq, Sq, d_k, dtype=dtype)
    _randn_into(q, g)
    out = {"skv": torch.tensor(skv, dtype=torch.int32), "max_skv": S, "q": q}
    if mla:
        cache = torch.empty(B, S, d_k, dtype=dtype)
        _randn_into(cache, g)
        out["cache"] = cache
        out["k"] = cache.view(B, 1, S, d_k)
        out["v"] = cache.view(B, 1, S, d_k)[..., :d_v]
    else:
        k = torch.empty(B, Hkv, S, d_k, dtype=dtype)
        _randn_into(k, g)
        v = torch.empty(B, Hkv, S, d_v, dtype=dtype)
        _randn_into(v, g)
        out["k"], out["v"] = k, v
    return w, out
