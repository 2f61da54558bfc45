"""QK RMS-norm + RoPE (pha_qk_norm_rope) on the GPU against the float64 oracle: the oracle normalises
and rotates in float64 and rounds once to the buffer dtype; the kernel normalises in float32 and
rounds the exactly rounded rotation of those values. Needs a B200."""
import numpy as np
import pytest
import torch

import oracle
from paired_heads_b200 import synth
from pipeline import check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paired_heads_b200 import build

    build.build()
    import paired_heads_b200.pha  # noqa: F401


def _ulp(ref, dt):
    if dt == "bf16":
        e = np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126)))
        return 2.0 ** (e - 7)
    return np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)


CASES = [
    # dtype, paired, stagger, hd, H, Hkv, T, weights, eps
    ("bf16", True, True, 128, 6, 6, 1000, False, 1e-6),
    ("bf16", True, True, 128, 6, 6, 1000, True, 1e-6),
    ("bf16", False, False, 64, 12, 4, 777, True, 1e-5),
    ("bf16", True, False, 64, 8, 4, 300, False, 0.0),
    ("bf16", False, False, 256, 4, 2, 200, True, 1e-6),
    ("f32", False, False, 16, 2, 2, 64, True, 1e-6),
    ("f32", True, True, 128, 4, 2, 100, False, 1e-6),
    # wider tokens than one ring slot of the factored kernel with the norm (192 chunks of 16
    # bytes): 640, 416 and 384 chunks, split into segments of 4 x 160, 160 + 160 + 96 and 2 x 192
    ("bf16", False, False, 128, 32, 8, 300, True, 1e-6),
    ("bf16", True, True, 128, 20, 6, 200, True, 1e-6),
    ("f32", True, True, 128, 6, 6, 100, True, 1e-6),
    # more tokens than the factored kernel's warps: several rounds, the last one partly filled
    ("bf16", True, True, 128, 6, 6, 5000, True, 1e-6),
]


@pytest.mark.parametrize("tables", ["stored", "factored"])
@pytest.mark.parametrize("case", CASES)
def test_norm_rope_parity(case, tables):
    dt, paired, stagger, hd, H, Hkv, T, weights, eps = case
    w = synth.Workload("norm", (T,), H, Hkv, hd, dt, paired=paired, stagger=stagger,
                       positions="global")
    inp = synth.make_inputs(w)
    rng = np.random.default_rng(T + hd)
    pos = rng.integers(0, 5000, T).astype(np.int32)
    pos[3], pos[7] = -1, 5000           # outside the table: normalised, not rotated
    # rows of very different scales, so the norm does real work
    scale = torch.from_numpy(rng.uniform(0.05, 20.0, (T, 1, 1)).astype(np.float32))
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    qh = (inp["q"].float() * scale).to(tdt)
    kh = (inp["k"].float() * scale).to(tdt)
    qw = torch.from_numpy(rng.uniform(0.5, 1.5, hd).astype(np.float32)) if weights else None
    kw = torch.from_numpy(rng.uniform(0.5, 1.5, hd).astype(np.float32)) if weights else None
    from paired_heads_b200.runner import AttentionStep, StepShape

    step = AttentionStep(StepShape.of(w, 5000), "cuda", rope_tables=tables)
    q, k = qh.cuda(), kh.cuda()
    step.norm_rope(q, k, torch.from_numpy(pos).cuda(), None if qw is None else qw.cuda(),
                   None if kw is None else kw.cuda(), eps)
    for name, x, got, gw in (("q", qh, q, qw), ("k", kh, k, kw)):
        ref = oracle.norm_rope_stored(synth.to_f64(x), pos, dt, paired, stagger,
                                      gamma=None if gw is None else gw.numpy(), eps=eps,
                                      tab_rows=5000)
        g = got.to(torch.float64).cpu().numpy()
        diff = np.abs(g - ref)
        # The kernel normalises in float32: its normalised values carry a relative error of a few
        # 2^-24 (x * inv, * weight, and inv itself). The rotation then moves each output by at most
        # that error times |c x0| + |s x1| <= 2 max|x_n| (about 1e-5 here, normalised values are
        # below ~20), and rounding adds at most one unit in the last place of the stored value.
        # Away from cancellation and rounding boundaries the stored values are equal.
        if dt == "bf16":
            assert np.all(diff <= _ulp(ref, dt) * 1.0001 + 1e-5), (name, float(diff.max()))
            assert np.mean(diff == 0) > 0.999, (name, float(np.mean(diff == 0)))
        else:
            np.testing.assert_allclose(g, ref, rtol=2e-6, atol=2e-6)


@pytest.mark.parametrize("wname", ["paired_varlen_small", "gqa_small"])
def test_norm_rope_then_attention_end_to_end(wname):
    if wname == "paired_varlen_small":
        w = synth.workload("paired_varlen", doc_lens=synth.geometric_doc_lengths(5000, 512.0, 2048, 0))
    else:
        w = synth.workload("gqa_long", doc_lens=(900, 300))
    inp = synth.make_inputs(w)
    from paired_heads_b200.runner import AttentionStep, StepShape

    tab_rows = int(inp["positions"].max()) + 1
    step = AttentionStep(StepShape.of(w, tab_rows), "cuda")
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    cu, pos = inp["cu_seqlens"].cuda(), inp["positions"].cuda()
    gw = torch.linspace(0.75, 1.25, w.head_dim)
    step.norm_rope(q, k, pos, gw.cuda(), gw.flip(0).cuda(), 1e-6)
    o, lse = step.attn(q, k, v, cu)
    torch.cuda.synchronize()
    qr = oracle.norm_rope_stored(synth.to_f64(inp["q"]), inp["positions"].numpy(), w.dtype,
                                 w.paired, w.stagger, gamma=gw.numpy(), eps=1e-6)
    kr = oracle.norm_rope_stored(synth.to_f64(inp["k"]), inp["positions"].numpy(), w.dtype,
                                 w.paired, w.stagger, gamma=gw.flip(0).numpy(), eps=1e-6)
    o_ref, lse_ref = oracle.attn_fwd(qr, kr, synth.to_f64(inp["v"]), inp["cu_seqlens"].numpy(),
                                     w.causal, w.window, w.paired, w.scale)
    check(w, o.cpu(), lse.cpu(), o_ref, lse_ref)
