"""Backward on the GPU (pha_rope_bwd, pha_attn_bwd) against the float64 oracle's gradients, which
recompute the softmax from q and k. Needs a B200.

Tolerances. Both backward paths take D_i = dO_i . O_i from the forward's stored O; the
tensor-core path (bf16, head_dim 64 / 128, every window: band work lists or per-tile ones)
follows FlashAttention's backward arithmetic ("Training an LLM from scratch (part 2)", section
"4. GQA & FlashAttention"): P and dS rounded to bf16 as MMA operands, float32 accumulation; the
CUDA-core path (every other shape) keeps P and dS in float32. Near a document start a row sees few keys, P is large and dq is
a difference of large terms, so a tolerance scaled by the tensor's maximum does not describe the
error. bf16 gradients are therefore bounded per element, from the rounding steps of the
tensor-core path (u = 2^-8, the unit roundoff of bf16's 8 significant bits); the CUDA-core path's
rounding steps are a subset of these:
(err(x) is the error of the computed x; dO, dP, dS are gradients)
  O (stored bf16, from bf16 P):  err(O_ie) <= 2u sum_j P_ij |v_je|
  so D = dO . O:                 err(D_i) <= 2u A_i,  A_i = sum_j P_ij (|dO_i| . |v_j|)
  dS (bf16 of P (dP - D)):       err(dS_ij) <= u |dS_ij| + P_ij err(D_i)
  dq = scale dS K, dk = scale dS^T Q:  scale sum err(dS) |k| (|q|), + u |result| (stored bf16)
  dv = P^T dO with P in bf16:    u sum_i P_ij |dO_ie| + u |dv|
each evaluated in float64 from the inputs and the exact P, dS, and allowed 1.25 times (the float32
sums, the exponentials and the lse add relative errors near 1e-6 of the same terms). f32
gradients (CUDA cores, float32 throughout) are compared with rtol 1e-4 plus 1e-5 of the tensor's
largest value."""
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


def _bf16_bounds(Q, K, V, G, cu, causal, window, paired, scale, hd):
    """Per-element error bounds of the bf16 backward (module docstring), token layout."""
    u = 2.0 ** -8
    T = Q.shape[0]
    m = 2 if paired else 1
    sv = lambda x: x.reshape(T * m, x.shape[1] // m, hd)
    Qs, Ks, Vs, Gs = sv(Q), sv(K), sv(V), sv(G)
    grp = Qs.shape[1] // Ks.shape[1]
    bq, bk, bv = np.zeros_like(Qs), np.zeros_like(Ks), np.zeros_like(Vs)
    cus = np.asarray(cu, dtype=np.int64) * m
    for a, b in zip(cus[:-1], cus[1:]):
        n = b - a
        if n == 0:
            continue
        i, j = np.arange(n)[:, None], np.arange(n)[None, :]
        vis = np.ones((n, n), dtype=bool)
        if causal:
            vis &= j <= i
            if window > 0:
                vis &= i - j < window
        for h in range(Qs.shape[1]):
            g = h // grp
            q, k, v, go = Qs[a:b, h], Ks[a:b, g], Vs[a:b, g], Gs[a:b, h]
            S = np.where(vis, q @ k.T * scale, -np.inf)
            P = np.exp(S - S.max(1, keepdims=True))
            P /= P.sum(1, keepdims=True)
            dP = go @ v.T
            dS = P * (dP - (P * dP).sum(1, keepdims=True))
            dD = 2 * u * (P * (np.abs(go) @ np.abs(v).T)).sum(1)
            bq[a:b, h] += scale * (u * np.abs(dS) @ np.abs(k) + dD[:, None] * (P @ np.abs(k)))
            bk[a:b, g] += scale * (u * np.abs(dS).T @ np.abs(q) + (P * dD[:, None]).T @ np.abs(q))
            bv[a:b, g] += u * P.T @ np.abs(go)
    return (bq.reshape(Q.shape), bk.reshape(K.shape), bv.reshape(V.shape))


def _close_bound(got, ref, bound, what):
    g = got.to(torch.float64).cpu().numpy().reshape(ref.shape)
    lim = 1.25 * (bound + 2.0 ** -8 * np.abs(ref)) + 1e-6 * float(np.abs(ref).max())
    err = np.abs(g - ref)
    worst = np.unravel_index(np.argmax(err / lim), err.shape)
    assert np.all(err <= lim), (what, worst, float(err[worst]), float(lim[worst]))
    assert np.all(np.isfinite(g)), what


def _ulp_bf16(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


@pytest.mark.parametrize("tables", ["stored", "factored"])
@pytest.mark.parametrize("paired,stagger,dt,H,Hkv,T", [
    (True, True, "bf16", 6, 6, 700), (False, False, "bf16", 6, 6, 700), (True, True, "f32", 4, 2, 64),
    (False, False, "bf16", 32, 8, 700),  # 640 chunks a token: the factored kernel splits tokens
    (True, True, "bf16", 6, 6, 5000),    # more tokens than the factored kernel's warps
])
def test_rope_bwd_parity(paired, stagger, dt, H, Hkv, T, tables):
    hd = 128 if dt == "bf16" else 16
    w = synth.Workload("rb", (T,), H, Hkv, hd, dt, paired=paired, stagger=stagger,
                       positions="global")
    inp = synth.make_inputs(w)
    rng = np.random.default_rng(T)
    pos = rng.integers(0, 3000, T).astype(np.int32)
    pos[5] = -1                                     # outside the table: unchanged
    from paired_heads_b200.runner import AttentionStep, StepShape

    step = AttentionStep(StepShape.of(w, 3000), "cuda", rope_tables=tables)
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
    # tensor cores, band work lists (bf16, causal, window <= 128, hd 64 / 128)
    ((300, 5, 190), 6, 6, 128, "bf16", True, 128, True),
    ((257, 130), 4, 2, 64, "bf16", True, 37, False),
    ((1100, 37, 600), 6, 6, 128, "bf16", True, 128, True),   # runs split into items (has-prev)
    ((700, 129), 8, 2, 128, "bf16", True, 100, False),      # group of 4 query heads per kv head
    ((64, 1, 130), 2, 2, 64, "bf16", True, 1, True),        # window 1, a one-token document
    # tensor cores, tile work lists (bf16, hd 64 / 128, no window or one longer than a tile)
    ((200, 64), 8, 2, 128, "bf16", True, 0, False),
    ((150, 90), 4, 4, 64, "bf16", False, 0, True),          # non-causal, paired
    ((700, 1, 1300), 4, 4, 64, "bf16", True, 0, False),     # full causal over ~10 key tiles
    ((2000,), 4, 4, 64, "bf16", True, 1024, False),         # window 1024
    ((900, 37), 8, 4, 128, "bf16", True, 300, True),        # window 300, paired, GQA
    ((600,), 32, 8, 128, "bf16", True, 0, False),           # GQA 32 / 8 (groups of 4)
    ((129, 257), 4, 2, 128, "bf16", False, 0, False),       # non-causal, GQA
    # CUDA cores (f32; a bf16 forward exists only for head_dim 64 / 128)
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
    args = (synth.to_f64(inp["q"]), synth.to_f64(inp["k"]), synth.to_f64(inp["v"]),
            synth.to_f64(g_up))
    rq, rk, rv = oracle.attn_bwd(*args, inp["cu_seqlens"].numpy(), causal, window, paired, w.scale)
    if dt == "bf16":
        scale = w.scale if w.scale > 0 else 1.0 / np.sqrt(hd)
        bq, bk, bv = _bf16_bounds(*args, inp["cu_seqlens"].numpy(), causal, window, paired,
                                  scale, hd)
        _close_bound(dq, rq, bq, "dq")
        _close_bound(dk, rk, bk, "dk")
        _close_bound(dv, rv, bv, "dv")
    else:
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
    args = (qr, kr, synth.to_f64(inp["v"]), synth.to_f64(g_up))
    rq0, rk0, rv = oracle.attn_bwd(*args, inp["cu_seqlens"].numpy(), True, w.window, True, w.scale)
    rq = oracle.rope_bwd(rq0, pnp, True, True, table_f32=True)
    rk = oracle.rope_bwd(rk0, pnp, True, True, table_f32=True)
    # bounds of the tensor-core backward, plus the bf16 rounding of its stored dq, dk, carried
    # through the rotation of each adjacent pair (|cos|, |sin| <= 1: element e of the output
    # mixes elements e and e ^ 1 of its input)
    scale = w.scale if w.scale > 0 else 1.0 / np.sqrt(w.head_dim)
    bq, bk, bv = _bf16_bounds(*args, inp["cu_seqlens"].numpy(), True, w.window, True, scale,
                              w.head_dim)
    swap = np.arange(w.head_dim) ^ 1
    for b, r0 in ((bq, rq0), (bk, rk0)):
        b += 2.0 ** -8 * np.abs(r0)
        b += b[..., swap].copy()
    _close_bound(dq, rq, bq, "dq")
    _close_bound(dk, rk, bk, "dk")
    _close_bound(dv, rv, bv, "dv")
