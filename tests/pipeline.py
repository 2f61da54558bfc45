"""Shared test helpers: run the CUDA path through the C-ABI binding, run the oracle on the same
seeded inputs, compare. Tolerances (stated by the task's parity bar):
  bf16 inputs, fp32 accumulation: max |O - O_ref| <= 2e-2, mean |O - O_ref| <= 2e-3
  f32 inputs:  |O - O_ref| <= 1e-5 * max_d |O_ref[row, :]|   (row-normwise relative)
  LSE:         |lse - lse_ref| <= 1e-3
"""
import numpy as np
import torch

import oracle
from paired_heads_b200 import synth

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
F32_REL = 1e-5
LSE_ABS = 1e-3


def run_gpu(w, rope=True, rank=0, inputs=None, rope_tables="stored"):
    """Inputs (CPU tensors) and the GPU outputs (CPU tensors) of one forward over workload w
    (RoPE with the stored float32 tables or the factored ones, as bench.py's step)."""
    from paired_heads_b200.runner import AttentionStep, StepShape

    inp = inputs if inputs is not None else synth.make_inputs(w, rank=rank)
    dev = torch.device("cuda:0")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    cu, pos = inp["cu_seqlens"].to(dev), inp["positions"].to(dev)
    tab_rows = int(inp["positions"].max()) + 1 if w.total else 1
    step = AttentionStep(StepShape.of(w, tab_rows), dev, rope_tables=rope_tables)
    if rope:
        step.rope(q, k, pos)
    o, lse = step.attn(q, k, v, cu)
    torch.cuda.synchronize()
    status = step.status()
    return inp, dict(q=q.cpu(), k=k.cpu(), o=o.cpu(), lse=lse.cpu(), status=status)


def oracle_inputs(w, inp, rope=True):
    """float64 q, k (rotated and stored in the workload's dtype when rope), v."""
    q, k, v = (synth.to_f64(inp[n]) for n in ("q", "k", "v"))
    if rope:
        pos = inp["positions"].numpy()
        q = oracle.rope_stored(q, pos, w.dtype, w.paired, w.stagger, w.rope_base)
        k = oracle.rope_stored(k, pos, w.dtype, w.paired, w.stagger, w.rope_base)
    return q, k, v


def run_oracle(w, inp, rope=True, rows=None):
    q, k, v = oracle_inputs(w, inp, rope)
    cu = inp["cu_seqlens"].numpy()
    if rows is None:
        return oracle.attn_fwd(q, k, v, cu, w.causal, w.window, w.paired, w.scale)
    return oracle.attn_rows(q, k, v, cu, rows, w.causal, w.window, w.paired, w.scale)


def check(w, o_gpu, lse_gpu, o_ref, lse_ref):
    """Assert the parity bar; returns the error summary."""
    o = o_gpu.to(torch.float64).numpy().reshape(o_ref.shape)
    lse = lse_gpu.to(torch.float64).numpy().reshape(lse_ref.shape)
    err = np.abs(o - o_ref)
    lerr = np.abs(lse - lse_ref)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    summary = dict(max_abs=float(err.max(initial=0)), mean_abs=float(err.mean()) if err.size else 0.0,
                   lse_max=float(lerr.max(initial=0)))
    if w.dtype == "bf16":
        assert summary["max_abs"] <= BF16_MAX_ABS, summary
        assert summary["mean_abs"] <= BF16_MEAN_ABS, summary
    else:
        rowmax = np.abs(o_ref).max(axis=-1, keepdims=True)
        assert np.all(err <= F32_REL * rowmax), float((err / np.maximum(rowmax, 1e-300)).max())
    assert summary["lse_max"] <= LSE_ABS, summary
    return summary


def sample_rows(w, n, seed=0):
    """Rows (t*H + h) to check at full size: the first and last tokens of every document, tokens
    on both sides of every 64-token tile edge near the window, and random tokens; all heads."""
    rng = np.random.default_rng(seed)
    cu = synth.cu_seqlens(w)
    toks = set()
    for b in range(w.batch):
        a, e = int(cu[b]), int(cu[b + 1])
        if e > a:
            toks.update({a, e - 1, min(a + 63, e - 1), min(a + 64, e - 1)})
            if w.window:
                toks.update({min(a + w.window // 2, e - 1), min(a + w.window, e - 1)})
    toks = sorted(toks)
    if len(toks) > n // 2:
        toks = sorted(rng.choice(toks, n // 2, replace=False).tolist())
    extra = rng.choice(w.total, max(n - len(toks), 0), replace=w.total < n)
    toks = np.unique(np.concatenate([np.asarray(toks, dtype=np.int64), extra]))
    heads = np.arange(w.n_heads)
    return (toks[:, None] * w.n_heads + heads[None, :]).reshape(-1)
