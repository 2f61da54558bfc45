"""Backward on the GPU (pha_rope_bwd, pha_attn_bwd) against the float64 oracle's gradients, which
recompute the softmax from q and k. Needs a B200.

Tolerances: the kernels compute in float32 from the bf16 (or f32) inputs and the forward's float32
lse, and store in the input dtype. bf16 storage rounds each gradient to 8 significant bits
(relative error <= 2^-9); the float32 sums add ~1e-6 of the largest terms. So bf16 gradients are
compared with rtol 8e-3 plus an absolute 2e-3 of the tensor's largest value (sums that cancel),
f32 gradients with rtol 1e-4 plus 1e-5 of the largest value."""
import numpy as np
import pytest
import torch

import oracle
from paired_heads_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paired_heads_b200 import build

    build.build()
    import paired_heads_b200.pha  # noqa: F401


def _close(got, ref, dt, what):
    g = got.to(torch.float64).cpu().numpy().reshape(ref.shape)
    scale = float(np.abs(ref).max()) or 1.0
    rtol, atol = (8e-3, 2e-3 * scale) if dt == "bf16" else (1e-4, 1e-5 * scale)
    err = np.abs(g - ref) - rtol * np.abs(ref)
    assert np.all(err <= atol), (what, float(np.abs(g - ref).max()), scale)
    assert np.all(np.isfinite(g)), what


def _ulp_bf16(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


@pytest.mark.parametrize("paired,stagger,dt", [(True, True, "bf16"), (False, False, "bf16"),
                                               (True, True, "f32")])
def test_rope_bwd_parity(paired, stagger, dt):
    H, Hkv, hd, T = (6, 6, 128, 700) if dt == "bf16" else (4, 2, 16, 64)
    w = synth.Workload("rb", (T,), H, Hkv, hd, dt, paired=paired, stagger=stagger,
                       positions="global")
    inp = synth.make_inputs(w)
    rng = np.random.default_rng(T)
    pos = rng.integers(0, 3000, T).astype(np.int32)
    pos[5] = -1                                     # outside the table: unchanged
    from paired_heads_b200.runner import AttentionStep, StepShape

    step = AttentionStep(StepShape.of(w, 3000), "cuda")
    gq, gk = inp["q"].cuda(), inp["k"].cuda()      # stand-ins for upstream gradients
    step.rope_bwd(gq, gk, torch.from_numpy(pos).cuda())
    for x, got in ((inp["q"], gq), (inp["k"], gk)):
        ref = oracle.rope_bwd(synth.to_f64(x), np.clip(pos, 0, None), paired, stagger,
                              table_f32=True)
        ref[5] = synth.to_f64(x)[5]
        ref = oracle.round_bf16(ref) if dt == "bf16" else ref.astype(np.float32).astype(np.float64)
        g = got.to(torch.float64).cpu().numpy()
        diff = np.abs(g - ref)
        ulp = _ulp_bf16(ref) if dt == "bf16" else np.spacing(np.abs(ref).astype(np.float32))
        assert np.all(diff <= ulp * 1.0001)
        assert np.mean(diff == 0) > 0.9999


CASES = [
    # doc lens, H, Hkv, hd, dtype, causal, window, paired
    ((300, 5, 190), 6, 6, 128, "bf16", True, 128, True),
    ((257, 130), 4, 2, 64, "bf16", True, 37, False),
    ((200, 64), 8, 2, 128, "bf16", True, 0, False),
    ((150, 90), 4, 4, 64, "bf16", False, 0, True),
    ((64,), 2, 2, 16, "f32", True, 0, True),
    ((80, 20), 4, 2, 32, "f32", True, 9, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{len(c[0])}docs-H{c[1]}/{c[2]}-hd{c[3]}-{c[4]}-c{int(c[5])}-w{c[6]}-p{int(c[7])}")
def test_attn_bwd_parity(case):
    lens, H, Hkv, hd, dt, causal, window, paired = case
    w = synth.Workload("bwd", lens, H, Hkv, hd, dt, causal=causal, window=window, paired=paired,
                       stagger=paired)
    inp = synth.make_inputs(w)
    rng = np.random.default_rng(sum(lens) + H)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    g_up = torch.from_numpy(rng.standard_normal(tuple(inp["q"].shape)).astype(np.float32)).to(tdt)
    from paired_heads_b200.runner import AttentionStep, StepShape

    step = AttentionStep(StepShape.of(w, 1), "cuda")
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    cu = inp["cu_seqlens"].cuda()
    step.attn(q, k, v, cu)                          # the forward's lse
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    step.attn_bwd(q, k, v, g_up.cuda(), cu, dq, dk, dv)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.attn_bwd(synth.to_f64(inp["q"]), synth.to_f64(inp["k"]),
                                 synth.to_f64(inp["v"]), synth.to_f64(g_up),
                                 inp["cu_seqlens"].numpy(), causal, window, paired, w.scale)
    _close(dq, rq, dt, "dq")
    _close(dk, rk, dt, "dk")
    _close(dv, rv, dt, "dv")


def test_backward_through_rope_and_attention():
    # the whole chain: the forward on rotated q, k, then dq, dk back through pha_rope_bwd
    w = synth.workload("paired_varlen", doc_lens=synth.geometric_doc_lengths(1500, 512.0, 2048, 0))
    inp = synth.make_inputs(w)
    from paired_heads_b200.runner import AttentionStep, StepShape

    tab_rows = int(inp["positions"].max()) + 1
    step = AttentionStep(StepShape.of(w, tab_rows), "cuda")
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    cu, pos = inp["cu_seqlens"].cuda(), inp["positions"].cuda()
    step.rope(q, k, pos)
    step.attn(q, k, v, cu)
    g_up = torch.from_numpy(np.random.default_rng(3).standard_normal(tuple(q.shape)).astype(np.float32)).to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    step.attn_bwd(q, k, v, g_up.cuda(), cu, dq, dk, dv)
    step.rope_bwd(dq, dk, pos)
    torch.cuda.synchronize()
    pnp = inp["positions"].numpy()
    qr = oracle.rope_stored(synth.to_f64(inp["q"]), pnp, "bf16", True, True)
    kr = oracle.rope_stored(synth.to_f64(inp["k"]), pnp, "bf16", True, True)
    rq, rk, rv = oracle.attn_bwd(qr, kr, synth.to_f64(inp["v"]), synth.to_f64(g_up),
                                 inp["cu_seqlens"].numpy(), True, w.window, True, w.scale)
    rq = oracle.rope_bwd(rq, pnp, True, True, table_f32=True)
    rk = oracle.rope_bwd(rk, pnp, True, True, table_f32=True)
    _close(dq, rq, "bf16", "dq")
    _close(dk, rk, "bf16", "dk")
    _close(dv, rv, "bf16", "dv")
