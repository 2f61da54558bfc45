"""Seeded synthetic workloads for paired-head attention.

This module only draws inputs: shapes, seeds, document lengths and rotary positions. It holds no
part of the attention or rotary arithmetic, so both the CUDA path and the float64 oracle can take
their inputs from here without sharing any computation.

Workloads (shapes follow the Paired Head Attention record page: narrow 64-wide heads, window 128
on the interleaved sequence, varlen packed documents; plus GPT-2-124M and long-context GQA shapes):

* ``tiny``          B=1, T=64, H=2, hd=16, fp32, causal, no window, standard and paired.
* ``gpt2``          B=8 x T=1024, H=12, hd=64, bf16, causal, scale 1/8.
* ``paired_varlen`` 65,536 packed tokens, document lengths geometric(mean 512) capped at 2048 with
                    the last document cut to fill; H=6 (3 pairs), hd=128, bf16, causal, window 128
                    slots, paired, staggered rotary, global packed positions.
* ``mixed_window``  B=4 x T=8192, H=12, hd=64, bf16, causal, window in {128, 1024, 0}, paired or not.
* ``gqa_long``      B=2 x T=16384, 32 query heads over 8 kv heads, hd=128, bf16, causal, no window.

All Q/K/V values are N(0, 1). ``tiny`` draws q, k, v in that order from one generator seeded 0;
the others draw q, k, v from generators seeded 1, 2, 3.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    doc_lens: tuple          # tokens per document
    n_heads: int
    n_kv_heads: int
    head_dim: int
    dtype: str               # "bf16" or "f32"
    causal: bool = True
    window: int = 0          # key slots incl. the query's own; 0 = none
    paired: bool = False
    stagger: bool = False    # paired only: odd heads take phase 2p+1
    scale: float = 0.0       # 0 = 1/sqrt(head_dim)
    positions: str = "per_doc"   # "per_doc" (restart at each document) or "global" (packed index)
    seeds: tuple = (1, 2, 3)
    single_stream: bool = False  # draw q, k, v from one generator (seeds[0]) in that order
    rope_base: float = 10000.0

    @property
    def total(self) -> int:
        return int(sum(self.doc_lens))

    @property
    def batch(self) -> int:
        return len(self.doc_lens)

    @property
    def max_len(self) -> int:
        return int(max(self.doc_lens)) if self.doc_lens else 0

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def geometric_doc_lengths(total: int, mean: float, cap: int, seed: int) -> tuple:
    """Document lengths drawn from geometric(1/mean), capped at ``cap``; drawing stops once the
    running sum reaches ``total`` and the last document is cut so that the lengths sum to it."""
    rng = np.random.default_rng(seed)
    lens = []
    acc = 0
    while acc < total:
        n = int(min(rng.geometric(1.0 / mean), cap))
        n = min(n, total - acc)
        lens.append(n)
        acc += n
    return tuple(lens)


def workload(name: str, **overrides) -> Workload:
    """The named workload, optionally with fields replaced."""
    if name == "tiny":
        w = Workload("tiny", (64,), 2, 2, 16, "f32", seeds=(0,), single_stream=True)
    elif name == "gpt2":
        w = Workload("gpt2", (1024,) * 8, 12, 12, 64, "bf16", scale=0.125)
    elif name == "paired_varlen":
        w = Workload("paired_varlen", geometric_doc_lengths(65536, 512.0, 2048, 0), 6, 6, 128,
                     "bf16", window=128, paired=True, stagger=True, positions="global")
    elif name == "mixed_window":
        w = Workload("mixed_window", (8192,) * 4, 12, 12, 64, "bf16", window=128)
    elif name == "gqa_long":
        w = Workload("gqa_long", (16384,) * 2, 32, 8, 128, "bf16")
    else:
        raise KeyError(name)
    return w.with_(**overrides) if overrides else w


WORKLOADS = ("tiny", "gpt2", "paired_varlen", "mixed_window", "gqa_long")


def cu_seqlens(w: Workload) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(np.asarray(w.doc_lens, dtype=np.int64))]).astype(np.int32)


def positions(w: Workload) -> np.ndarray:
    """Rotary position of every packed token: its index in the packed row ("global") or its index
    inside its own document ("per_doc")."""
    if w.positions == "global":
        return np.arange(w.total, dtype=np.int32)
    return np.concatenate([np.arange(n, dtype=np.int32) for n in w.doc_lens]) if w.doc_lens \
        else np.zeros((0,), dtype=np.int32)


def qkv_float32(w: Workload, rank: int = 0):
    """q[T][H][hd], k[T][Hkv][hd], v[T][Hkv][hd] as float32 N(0,1) draws. ``rank`` shifts the
    seeds so that data-parallel ranks get different documents of the same shape."""
    T = w.total
    shapes = [(T, w.n_heads, w.head_dim), (T, w.n_kv_heads, w.head_dim),
              (T, w.n_kv_heads, w.head_dim)]
    if w.single_stream:
        rng = np.random.default_rng(w.seeds[0] + 1000 * rank)
        # draw in float64 (numpy's default stream), then narrow: the same numbers as
        # rng.standard_normal(shape) in q, k, v order
        return tuple(rng.standard_normal(s).astype(np.float32) for s in shapes)
    return tuple(np.random.default_rng(seed + 1000 * rank).standard_normal(s, dtype=np.float32)
                 for seed, s in zip(w.seeds, shapes))


def make_inputs(w: Workload, rank: int = 0, device: Optional[str] = None):
    """Inputs as torch tensors in the workload's dtype (bf16 by round-to-nearest-even from the
    float32 draws), plus int32 cu_seqlens and positions. Returns a dict."""
    import torch

    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q, k, v = (torch.from_numpy(a).to(dt) for a in qkv_float32(w, rank))
    out = dict(q=q, k=k, v=v, cu_seqlens=torch.from_numpy(cu_seqlens(w)),
               positions=torch.from_numpy(positions(w)))
    if device is not None:
        out = {key: t.to(device) for key, t in out.items()}
    return out


def make_fp8_inputs(w: Workload, rank: int = 0, device: Optional[str] = None):
    """FP8 versions of make_inputs' q, k, v: each float32 draw divided by its tensor's scale
    s = max|x| / 448 (rounded to float32, so that the largest magnitude lands on e4m3's largest
    finite value) and cast to torch.float8_e4m3fn. Returns a dict with q8, k8, v8 (float8 tensors),
    q_scale, k_scale, v_scale (floats; x ~ scale * value(code)), cu_seqlens and positions."""
    import torch

    out = {}
    for name, a in zip(("q", "k", "v"), qkv_float32(w, rank)):
        amax = float(np.abs(a).max()) if a.size else 1.0
        sc = float(np.float32(amax / 448.0)) if amax > 0 else 1.0
        t = torch.from_numpy(a) / sc
        out[name + "8"] = t.to(torch.float8_e4m3fn)
        out[name + "_scale"] = sc
    out["cu_seqlens"] = torch.from_numpy(cu_seqlens(w))
    out["positions"] = torch.from_numpy(positions(w))
    if device is not None:
        out = {key: (t.to(device) if hasattr(t, "to") else t) for key, t in out.items()}
    return out


def to_f64(t) -> np.ndarray:
    """Exact float64 copy of a (bf16 / f32) torch tensor -- what the oracle receives."""
    import torch

    return t.detach().to("cpu", torch.float64).numpy()
