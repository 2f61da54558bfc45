"""GPU parity: the CUDA path (through the C-ABI binding) against the float64 oracle on the same
seeded inputs, element by element. Needs a B200."""
import numpy as np
import pytest
import torch

import oracle
from paired_heads_b200 import synth
from pipeline import (check, oracle_inputs, run_gpu, run_oracle, sample_rows)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paired_heads_b200 import build

    build.build()
    import paired_heads_b200.pha  # noqa: F401


def _pha():
    from paired_heads_b200 import pha

    return pha


# ------------------------------------------------------------------------------------ rotary

@pytest.mark.parametrize("paired", [False, True])
@pytest.mark.parametrize("hd", [16, 64, 128])
def test_rope_tables(paired, hd):
    pha = _pha()
    rows = 5000
    width = (2 if paired else 1) * hd
    ct = torch.empty(rows, width, device="cuda")
    st = torch.empty_like(ct)
    pha.pha_rope_tables(ct, st, rows, hd, paired, 10000.0)
    p = np.arange(rows, dtype=np.float64)[:, None]
    j = np.arange(width)[None, :]
    phase = (2 * p + (j // hd)) if paired else p
    ang = phase * 10000.0 ** (-2.0 * ((j % hd) // 2) / hd)
    # float64 angles rounded once to float32: within one float32 ulp of numpy's values
    np.testing.assert_allclose(ct.cpu().numpy(), np.cos(ang), rtol=0, atol=6e-8)
    np.testing.assert_allclose(st.cpu().numpy(), np.sin(ang), rtol=0, atol=6e-8)


@pytest.mark.parametrize("paired", [False, True])
@pytest.mark.parametrize("hd", [16, 128])
def test_rope_factor_tables(paired, hd):
    pha = _pha()
    rows = 5000
    nb = pha.pha_rope_factor_bytes(rows, hd, paired)
    fac = torch.empty(nb, dtype=torch.uint8, device="cuda")
    pha.pha_rope_factor_tables(fac, rows, hd, paired, 10000.0)
    f = fac.view(torch.float64).cpu().numpy().reshape(-1, 2)
    half = hd // 2
    a_width = hd if paired else half
    n_lo = 16 * a_width
    inv = 10000.0 ** (-2.0 * np.arange(half) / hd)
    # the documented layout: fine rows (position l, or 2l + half) then coarse rows (16 r, or 32 r)
    a = np.arange(a_width)
    lo_pos = (2 * np.arange(16)[:, None] + a[None, :] // half) if paired else \
        np.broadcast_to(np.arange(16)[:, None], (16, a_width))
    lo_ang = lo_pos * inv[a % half][None, :]
    n_hi = -(-rows // 16)
    hi_ang = (np.arange(n_hi)[:, None] * 16 * (2 if paired else 1)) * inv[None, :]
    ang = np.concatenate([lo_ang.reshape(-1), hi_ang.reshape(-1)])
    assert f.shape[0] == n_lo + n_hi * half
    # float64 sincos of float64 angles (up to 1e4 rad here): the C library and CUDA agree to a
    # few units of 1e-16 per angle unit
    np.testing.assert_allclose(f[:, 0], np.cos(ang), rtol=0, atol=1e-12)
    np.testing.assert_allclose(f[:, 1], np.sin(ang), rtol=0, atol=1e-12)
    # recombined by angle addition and rounded to float32 they are the stored tables' values,
    # except in the last bit next to float32 rounding midpoints, or, very close to zero, by the
    # difference of the two forms' float64 angles (the stored one rounds p * f once, the factored
    # one rounds its two parts: at most 1.5 float64 ulp of the largest angle, 1e4 rad here)
    width = (2 if paired else 1) * hd
    ct = torch.empty(rows, width, device="cuda")
    st = torch.empty_like(ct)
    pha.pha_rope_tables(ct, st, rows, hd, paired, 10000.0)
    p = np.arange(rows)
    j = np.arange(width)
    lo_idx = (p % 16)[:, None] * a_width + ((j // hd) * half if paired else 0) + (j % hd) // 2
    hi_idx = n_lo + (p // 16)[:, None] * half + ((j % hd) // 2)[None, :]
    fl, fh = f[lo_idx], f[hi_idx]
    c = (fh[..., 0] * fl[..., 0] - fh[..., 1] * fl[..., 1]).astype(np.float32)
    s_ = (fh[..., 1] * fl[..., 0] + fh[..., 0] * fl[..., 1]).astype(np.float32)
    for got, ref in ((c, ct.cpu().numpy()), (s_, st.cpu().numpy())):
        d = np.abs(got.astype(np.float64) - ref)
        assert np.all(d <= np.spacing(np.abs(ref)) * 1.0001 + 1.5 * 2.0 ** -39 + 1e-15)
        assert np.mean(d == 0) > 0.99, float(np.mean(d == 0))


def test_rope_factored_matches_stored():
    # the headline shape on a slice of tokens at positions up to 131,072: both paths are correctly
    # rounded, so they differ only where a last-bit difference of a cosine or sine moves a rounding
    # (expected about 1e-8 of the elements)
    from paired_heads_b200.runner import AttentionStep, StepShape

    w = synth.Workload("rope", (4096,), 6, 6, 128, "bf16", paired=True, stagger=True,
                       positions="global")
    inp = synth.make_inputs(w)
    rng = np.random.default_rng(5)
    pos = torch.from_numpy(rng.integers(0, 131072, 4096).astype(np.int32)).cuda()
    outs = []
    for tables in ("stored", "factored"):
        step = AttentionStep(StepShape.of(w, 131072), "cuda", rope_tables=tables)
        q, k = inp["q"].cuda(), inp["k"].cuda()
        step.rope(q, k, pos)
        outs.append((q, k))
    for a, b in zip(outs[0], outs[1]):
        same = (a.view(torch.int16) == b.view(torch.int16)).double().mean().item()
        assert same > 0.99999, same
        d = (a.double() - b.double()).abs()
        assert torch.all(d <= a.double().abs() * 2.0 ** -7 + 1e-30)


def _ulp_bf16(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


ROPE_CASES = [
    # dtype, paired, stagger, hd, H, Hkv, T
    ("bf16", False, False, 64, 12, 12, 777),
    ("bf16", True, True, 128, 6, 6, 1000),
    ("bf16", True, False, 64, 12, 4, 300),
    ("bf16", False, False, 16, 3, 1, 50),
    ("f32", False, False, 16, 2, 2, 64),
    ("f32", True, True, 16, 2, 2, 64),
    ("f32", True, True, 128, 4, 2, 100),
    # wider tokens than one ring slot of the factored kernel (288 chunks of 16 bytes): 640, 416
    # and 384 chunks, split into segments of 224 + 224 + 192, 224 + 192 and 2 x 192 chunks
    ("bf16", False, False, 128, 32, 8, 500),
    ("bf16", True, True, 128, 20, 6, 300),
    ("f32", True, True, 128, 6, 6, 200),
    # more tokens than the factored kernel's warps (148 SMs x 24): several rounds, the last one
    # partly filled
    ("bf16", True, True, 128, 6, 6, 5000),
    ("bf16", False, False, 64, 12, 4, 4001),
]


@pytest.mark.parametrize("tables", ["stored", "factored"])
@pytest.mark.parametrize("case", ROPE_CASES)
def test_rope_parity(case, tables):
    dt, paired, stagger, hd, H, Hkv, T = case
    w = synth.Workload("rope", (T,), H, Hkv, hd, dt, paired=paired, stagger=stagger,
                       positions="global")
    inp = synth.make_inputs(w)
    # positions: random rows of a 70,000-row table, plus two outside it (left unchanged)
    rng = np.random.default_rng(T)
    pos = rng.integers(0, 70000, T).astype(np.int32)
    pos[3], pos[7] = -1, 70000
    inp["positions"] = torch.from_numpy(pos)
    from paired_heads_b200.runner import AttentionStep, StepShape

    step = AttentionStep(StepShape.of(w, 70000), "cuda", rope_tables=tables)
    q, k = inp["q"].cuda(), inp["k"].cuda()
    step.rope(q, k, inp["positions"].cuda())
    pos_ok = np.clip(pos, 0, None)
    for name, got in (("q", q), ("k", k)):
        x = synth.to_f64(inp[name])
        ref = oracle.rope_stored(x, pos_ok, dt, paired, stagger)
        ref[3], ref[7] = x[3], x[7]
        g = got.to(torch.float64).cpu().numpy()
        # Both sides round the float64 rotation of the float32 table values once to the dtype,
        # so they agree bit for bit except where the two float32 tables differ in a last bit
        # (CUDA's and the C library's float64 sin / cos / pow; with factored tables also the
        # float64 angle addition), which may move a result by one unit in the last place.
        diff = np.abs(g - ref)
        ulp = _ulp_bf16(ref) if dt == "bf16" else np.spacing(np.abs(ref).astype(np.float32))
        assert np.all(diff <= ulp * 1.0001), float((diff / ulp).max())
        assert np.mean(diff == 0) > 0.9999, float(np.mean(diff == 0))


# ------------------------------------------------------------------------------------ fp32 path

@pytest.mark.parametrize("paired", [False, True])
def test_tiny_f32_end_to_end(paired):
    w = synth.workload("tiny", paired=paired, stagger=paired)
    inp, g = run_gpu(w)
    o_ref, lse_ref = run_oracle(w, inp)
    check(w, g["o"], g["lse"], o_ref, lse_ref)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_pages_mask_example(dt):
    # Paired, one pair (page's example, 1-based position 4): K = 0 and V one-hot over
    # (head, position), so each output row is uniform over the keys the row sees.
    T, H = 4, 2
    hd = 16 if dt == "f32" else 64
    rng = np.random.default_rng(1)
    q = rng.standard_normal((T, H, hd)).astype(np.float32)
    k = np.zeros((T, H, hd), np.float32)
    v = np.zeros((T, H, hd), np.float32)
    for h in range(H):
        for t in range(T):
            v[t, h, h * T + t] = 1.0
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    w = synth.Workload("mask", (T,), H, H, hd, dt, paired=True)
    inp = dict(q=torch.from_numpy(q).to(tdt), k=torch.from_numpy(k).to(tdt),
               v=torch.from_numpy(v).to(tdt), cu_seqlens=torch.tensor([0, T], dtype=torch.int32),
               positions=torch.arange(T, dtype=torch.int32))
    _, g = run_gpu(w, rope=False, inputs=inp)
    o = g["o"].float().numpy()
    # head 1 @4 sees head-1 keys 1-4 and head-2 keys 1-3; head 2 @4 sees all eight
    e1 = np.zeros(hd)
    e1[[0, 1, 2, 3, 4, 5, 6]] = 1 / 7
    e2 = np.zeros(hd)
    e2[:8] = 1 / 8
    tol = 1e-7 if dt == "f32" else 2e-3
    np.testing.assert_allclose(o[3, 0], e1, atol=tol)
    np.testing.assert_allclose(o[3, 1], e2, atol=tol)


# ------------------------------------------------------------------------------------ bf16 path

ATTN_CASES = [
    # doc lens, H, Hkv, hd, causal, window, paired
    ((1, 127, 128, 129, 300, 513), 4, 4, 64, True, 0, False),
    ((1, 127, 128, 129, 300, 513), 4, 4, 128, True, 0, False),
    ((700, 5, 260), 6, 6, 128, True, 128, True),
    ((700, 5, 260), 6, 6, 64, True, 1, True),
    ((1000,), 4, 2, 64, True, 200, False),
    ((333, 64), 8, 2, 128, True, 0, False),
    ((333, 64), 8, 4, 64, True, 37, True),
    ((250, 130), 2, 2, 64, False, 0, False),
    ((250, 130), 4, 2, 128, False, 0, True),
    ((2000,), 2, 2, 128, True, 300, True),
    ((0, 77, 0, 0, 190), 2, 1, 64, True, 0, False),
    # windows around the 32-column chunk boundaries of the masked-tile path
    ((600, 257), 4, 4, 128, True, 31, False),
    ((600, 257), 4, 4, 64, True, 33, True),
    ((500, 3), 2, 2, 128, True, 63, True),
    ((500, 3), 2, 2, 64, True, 65, False),
    ((900,), 4, 2, 128, True, 96, True),
    ((900,), 4, 2, 64, True, 129, False),
    ((1100, 130), 6, 6, 128, True, 257, True),
    # band kernel (causal, window <= 128): runs of 8 query tiles (1024 slots) with exact and
    # one-row-over chunk boundaries, single-tile documents, the smallest windows, GQA
    ((512, 513, 64, 1, 2049), 4, 2, 128, True, 128, True),
    ((1024, 1025, 127, 129, 1), 2, 2, 64, True, 2, False),
    ((3000, 7), 8, 2, 128, True, 100, False),
    ((128, 256, 2176), 2, 2, 128, True, 128, False),
]


@pytest.mark.parametrize("case", ATTN_CASES)
def test_attention_bf16_parity(case):
    lens, H, Hkv, hd, causal, window, paired = case
    w = synth.Workload("case", lens, H, Hkv, hd, "bf16", causal=causal, window=window,
                       paired=paired, stagger=paired)
    inp, g = run_gpu(w, rope=False)
    assert g["status"] == (0, g["status"][1])
    o_ref, lse_ref = run_oracle(w, inp, rope=False)
    check(w, g["o"], g["lse"], o_ref, lse_ref)


SCALED = [
    synth.workload("gpt2", doc_lens=(1024,) * 2),
    synth.workload("paired_varlen", doc_lens=synth.geometric_doc_lengths(6000, 512.0, 2048, 0)),
    synth.workload("mixed_window", doc_lens=(1500,), window=128),
    synth.workload("mixed_window", doc_lens=(1500,), window=1024, paired=True, stagger=True),
    synth.workload("mixed_window", doc_lens=(1500,), window=0, paired=True, stagger=True),
    synth.workload("gqa_long", doc_lens=(1200, 700)),
]


@pytest.mark.parametrize("w", SCALED, ids=lambda w: f"{w.name}-w{w.window}-p{int(w.paired)}")
def test_end_to_end_scaled(w):
    inp = synth.make_inputs(w)
    o_ref, lse_ref = run_oracle(w, inp)
    for tables in ("stored", "factored"):  # the two RoPE table forms, then attention
        _, g = run_gpu(w, inputs=inp, rope_tables=tables)
        check(w, g["o"], g["lse"], o_ref, lse_ref)


FULL = [
    synth.workload("gpt2"),
    synth.workload("paired_varlen"),
    synth.workload("mixed_window", window=128),
    synth.workload("mixed_window", window=128, paired=True, stagger=True),
    synth.workload("mixed_window", window=1024),
    synth.workload("mixed_window", window=1024, paired=True, stagger=True),
    synth.workload("mixed_window", window=0),
    synth.workload("mixed_window", window=0, paired=True, stagger=True),
    synth.workload("gqa_long"),
]


@pytest.mark.parametrize("w", FULL, ids=lambda w: f"{w.name}-w{w.window}-p{int(w.paired)}")
def test_full_size_sampled_rows(w):
    # the launch configuration bench.py times: factored RoPE, then attention
    inp, g = run_gpu(w, rope_tables="factored")
    rows = sample_rows(w, 400)
    o_ref, lse_ref = run_oracle(w, inp, rows=rows)
    o = g["o"].reshape(-1, w.head_dim)[torch.from_numpy(rows)]
    lse = g["lse"].reshape(-1)[torch.from_numpy(rows)]
    check(w, o, lse, o_ref, lse_ref)
    # every output finite
    assert torch.isfinite(g["o"].float()).all() and torch.isfinite(g["lse"]).all()


# ------------------------------------------------------------------------------------ edge cases

def test_window_one_returns_own_value_exactly():
    w = synth.Workload("w1", (300, 1, 40), 4, 2, 128, "bf16", window=1)
    inp, g = run_gpu(w, rope=False)
    v = inp["v"].repeat_interleave(2, dim=1)
    assert torch.equal(g["o"], v)


def test_malformed_seqlens_write_nothing():
    pha = _pha()
    from paired_heads_b200.runner import AttentionStep, StepShape

    w = synth.Workload("bad", (100, 200), 2, 2, 64, "bf16")
    inp = synth.make_inputs(w)
    # claim max_len 150 while a document is 200 tokens long
    step = AttentionStep(StepShape(n_heads=2, n_kv_heads=2, head_dim=64, dtype="bf16", batch=2,
                                   max_len=150, total_tokens=300, tab_rows=300), "cuda")
    step.o.fill_(float("nan"))
    step.attn(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), inp["cu_seqlens"].cuda())
    status, n = step.status()
    assert (status, n) == (1, 0)
    assert torch.isnan(step.o.float()).all()
    # decreasing boundaries
    cu = torch.tensor([0, 200, 100], dtype=torch.int32, device="cuda")
    step.attn(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), cu)
    assert step.status() == (1, 0)
    assert pha.pha_status_string(0) == "ok"


def test_no_writes_outside_outputs():
    pha = _pha()
    w = synth.Workload("canary", (129, 300), 6, 6, 128, "bf16", window=128, paired=True,
                       stagger=True)
    inp = synth.make_inputs(w)
    T, H, D, pad = w.total, w.n_heads, w.head_dim, 64
    o_big = torch.full((T + 2 * pad, H, D), 7.0, dtype=torch.bfloat16, device="cuda")
    l_big = torch.full((T + 2 * pad, H), 7.0, device="cuda")
    o, lse = o_big[pad:pad + T], l_big[pad:pad + T]
    ws = torch.empty(pha.pha_attn_workspace_bytes(w.batch, w.max_len, H, D, True),
                     dtype=torch.uint8, device="cuda")
    pha.pha_attn_fwd(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), inp["cu_seqlens"].cuda(),
                     w.max_len, o, lse, ws, window=w.window, paired=True)
    torch.cuda.synchronize()
    assert (o_big[:pad] == 7).all() and (o_big[pad + T:] == 7).all()
    assert (l_big[:pad] == 7).all() and (l_big[pad + T:] == 7).all()
    o_ref, lse_ref = run_oracle(w, inp, rope=False)
    check(w, o.cpu(), lse.cpu(), o_ref, lse_ref)


def test_empty_input_is_a_no_op():
    pha = _pha()
    q = torch.empty(0, 2, 64, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    ws = torch.empty(pha.pha_attn_workspace_bytes(1, 0, 2, 64, False), dtype=torch.uint8,
                     device="cuda")
    pha.pha_attn_fwd(q, q, q, torch.zeros(2, dtype=torch.int32, device="cuda"), 0, o, None, ws)
    torch.cuda.synchronize()
    assert pha.pha_attn_status(ws) == (0, 0)


def test_repeatable_bit_for_bit():
    w = synth.workload("paired_varlen", doc_lens=synth.geometric_doc_lengths(4000, 512.0, 2048, 3))
    inp = synth.make_inputs(w)
    _, a = run_gpu(w, inputs=inp)
    _, b = run_gpu(w, inputs=inp)
    assert torch.equal(a["o"], b["o"]) and torch.equal(a["lse"], b["lse"])
