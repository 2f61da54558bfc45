"""One forward step -- RoPE on q and k, then varlen attention -- over a fixed problem shape.

``AttentionStep`` owns the device buffers the C ABI expects the caller to provide (rotary tables,
workspace, O and LSE), allocated once through torch, and issues the two library calls. It is
plumbing only: all arithmetic runs in libpha's kernels.
"""
from __future__ import annotations

import dataclasses

import torch

from . import pha


@dataclasses.dataclass
class StepShape:
    n_heads: int
    n_kv_heads: int
    head_dim: int
    dtype: str                 # "bf16" | "f32"
    batch: int
    max_len: int
    total_tokens: int
    tab_rows: int              # rows of the rotary tables (max position + 1)
    paired: bool = False
    stagger: bool = False
    causal: bool = True
    window: int = 0
    scale: float = 0.0
    rope_base: float = 10000.0

    @classmethod
    def of(cls, w, tab_rows: int) -> "StepShape":
        """Shape of a synth.Workload."""
        return cls(w.n_heads, w.n_kv_heads, w.head_dim, w.dtype, w.batch, w.max_len, w.total,
                   tab_rows, w.paired, w.stagger, w.causal, w.window, w.scale, w.rope_base)


class AttentionStep:
    """rope_tables: "stored" -- float32 cos / sin rows per position (pha_rope_tables, pha_rope);
    "factored" -- the compact float64 factor tables (pha_rope_factor_tables, pha_rope_factored)."""

    def __init__(self, shape: StepShape, device="cuda", rope_tables: str = "stored"):
        if rope_tables not in ("stored", "factored"):
            raise ValueError(f"rope_tables: {rope_tables!r}")
        self.s = shape
        self.rope_tables = rope_tables
        dev = torch.device(device)
        width = (2 if shape.paired else 1) * shape.head_dim
        self.cos_tab = self.sin_tab = self.factors = None
        if rope_tables == "stored":
            self.cos_tab = torch.empty(max(shape.tab_rows, 1), width, device=dev)
            self.sin_tab = torch.empty_like(self.cos_tab)
            pha.pha_rope_tables(self.cos_tab, self.sin_tab, shape.tab_rows, shape.head_dim,
                                shape.paired, shape.rope_base)
        else:
            nbytes = pha.pha_rope_factor_bytes(shape.tab_rows, shape.head_dim, shape.paired)
            self.factors = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
            pha.pha_rope_factor_tables(self.factors, shape.tab_rows, shape.head_dim,
                                       shape.paired, shape.rope_base)
        dt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
        self.o = torch.empty(shape.total_tokens, shape.n_heads, shape.head_dim, dtype=dt, device=dev)
        self.lse = torch.empty(shape.total_tokens, shape.n_heads, dtype=torch.float32, device=dev)
        nbytes = pha.pha_attn_workspace_bytes(shape.batch, shape.max_len, shape.n_heads,
                                              shape.head_dim, shape.paired)
        self.workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
        self.stagger_offset = shape.head_dim if (shape.paired and shape.stagger) else 0

    def rope(self, q, k, positions, stream=None):
        if self.factors is not None:
            pha.pha_rope_factored(q, k, self.factors, self.s.tab_rows, positions,
                                  paired=self.s.paired, stagger_offset=self.stagger_offset,
                                  stream=stream)
            return
        pha.pha_rope(q, k, self.cos_tab, self.sin_tab, positions, paired=self.s.paired,
                     stagger_offset=self.stagger_offset, stream=stream)

    def norm_rope(self, q, k, positions, q_weight=None, k_weight=None, eps=1e-6, stream=None):
        """QK RMS-norm of every head row, then RoPE, in place (one kernel)."""
        if self.factors is not None:
            pha.pha_qk_norm_rope_factored(q, k, self.factors, self.s.tab_rows, positions,
                                          q_weight, k_weight, eps, paired=self.s.paired,
                                          stagger_offset=self.stagger_offset, stream=stream)
            return
        pha.pha_qk_norm_rope(q, k, self.cos_tab, self.sin_tab, positions, q_weight, k_weight, eps,
                             paired=self.s.paired, stagger_offset=self.stagger_offset,
                             stream=stream)

    def attn(self, q, k, v, cu_seqlens, stream=None):
        pha.pha_attn_fwd(q, k, v, cu_seqlens, self.s.max_len, self.o, self.lse, self.workspace,
                         causal=self.s.causal, window=self.s.window, paired=self.s.paired,
                         scale=self.s.scale, stream=stream)
        return self.o, self.lse

    @property
    def aux_v_supported(self) -> bool:
        """Whether pha_attn_fwd_aux_v covers this shape (the bf16 tensor-core kernels: head_dim
        64 or 128)."""
        s = self.s
        return s.dtype == "bf16" and s.head_dim in (64, 128)

    def attn_aux_v(self, q, k, v, aux_v, cu_seqlens, stream=None):
        """Attention over (q, k, v + aux_v); v and aux_v are left unchanged."""
        pha.pha_attn_fwd_aux_v(q, k, v, aux_v, cu_seqlens, self.s.max_len, self.o, self.lse,
                               self.workspace, causal=self.s.causal, window=self.s.window,
                               paired=self.s.paired, scale=self.s.scale, stream=stream)
        return self.o, self.lse

    def rope_bwd(self, dq, dk, positions, stream=None):
        """In place: gradients w.r.t. the rotated q, k -> w.r.t. the unrotated q, k."""
        if self.factors is not None:
            pha.pha_rope_bwd_factored(dq, dk, self.factors, self.s.tab_rows, positions,
                                      paired=self.s.paired, stagger_offset=self.stagger_offset,
                                      stream=stream)
            return
        pha.pha_rope_bwd(dq, dk, self.cos_tab, self.sin_tab, positions, paired=self.s.paired,
                         stagger_offset=self.stagger_offset, stream=stream)

    def attn_bwd(self, q, k, v, dout, cu_seqlens, dq, dk, dv, stream=None):
        """Backward of the last attention call (same q, k, v; its o and lse are used): dq, dk, dv
        for dout. Returns (dq, dk, dv)."""
        s = self.s
        if getattr(self, "bwd_workspace", None) is None:
            nbytes = pha.pha_attn_bwd_workspace_bytes(s.batch, s.max_len, s.total_tokens,
                                                      s.n_heads, s.head_dim, s.paired)
            self.bwd_workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
        pha.pha_attn_bwd(q, k, v, self.o, self.lse, dout, cu_seqlens, s.max_len, dq, dk, dv,
                         self.bwd_workspace, causal=s.causal, window=s.window, paired=s.paired,
                         scale=s.scale, stream=stream)
        return dq, dk, dv

    def __call__(self, q, k, v, cu_seqlens, positions, stream=None):
        """RoPE q and k in place, then attention. Returns (o, lse) (buffers owned by the step)."""
        self.rope(q, k, positions, stream)
        return self.attn(q, k, v, cu_seqlens, stream)

    def status(self):
        """(device status, scheduled work items) of the last attention call; synchronises."""
        return pha.pha_attn_status(self.workspace)
