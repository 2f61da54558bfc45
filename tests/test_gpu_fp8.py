"""FP8 attention (pha_attn_fwd_fp8) against the oracle on the same e4m3 codes and scales
("modded-nanogpt Paired Head Attention record", section "5. interactions with other mechanisms":
the packed FP8 QKV path).

Tolerance: that of the bf16 path (max |O - O_ref| <= 2e-2, mean <= 2e-3; LSE within 1e-3). The
inputs are exact in the kernel's arithmetic (e4m3 x e4m3 products are exact in the float32
accumulator; V widens exactly to f16), so the only roundings are the float32 sums, P rounded to
f16 (10 fraction bits, finer than the bf16 path's 7) and the bf16 output, each bounded as on the
bf16 path. The oracle runs in float64 on the decoded codes times their scales."""
import numpy as np
import pytest
import torch

import oracle
from paired_heads_b200 import synth

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS, LSE_ABS = 2e-2, 2e-3, 1e-3

CASES = [
    # name, doc lengths, H, Hkv, hd, causal, window, paired
    ("gpt2_hd64", (300, 129, 1, 700), 4, 4, 64, True, 0, False),
    ("paired_varlen_w128", synth.geometric_doc_lengths(3000, 512.0, 2048, 3), 6, 6, 128, True, 128, True),
    ("mixed_w300_paired_hd64", (1500, 37), 4, 4, 64, True, 300, True),
    ("gqa_8_2_hd128", (1100, 260), 8, 2, 128, True, 0, False),
    ("noncausal_hd64", (257, 64), 2, 2, 64, False, 0, False),
    ("window1_hd128", (400,), 2, 2, 128, True, 1, False),
    ("paired_gqa_hd128", (513,), 8, 4, 128, True, 0, True),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_fp8_matches_oracle(case):
    from paired_heads_b200 import build, pha

    build.build()
    name, lens, H, Hkv, hd, causal, window, paired = case
    w = synth.Workload(name, tuple(lens), H, Hkv, hd, "bf16", causal=causal, window=window,
                       paired=paired)
    inp = synth.make_fp8_inputs(w)
    q8, k8, v8 = (inp[n].cuda() for n in ("q8", "k8", "v8"))
    cu = inp["cu_seqlens"].cuda()
    o = torch.full((w.total, H, hd), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.total, H), float("nan"), device="cuda")
    ws = torch.empty(pha.pha_attn_workspace_bytes(w.batch, w.max_len, H, hd, paired),
                     dtype=torch.uint8, device="cuda")
    pha.pha_attn_fwd_fp8(q8, k8, v8, inp["q_scale"], inp["k_scale"], inp["v_scale"], cu,
                         w.max_len, o, lse, ws, causal=causal, window=window, paired=paired)
    status, _ = pha.pha_attn_status(ws)
    assert status == 0

    codes = {n: inp[n].view(torch.uint8).numpy() for n in ("q8", "k8", "v8")}
    o_ref, lse_ref = oracle.attn_fwd_fp8(codes["q8"], codes["k8"], codes["v8"], inp["q_scale"],
                                         inp["k_scale"], inp["v_scale"], inp["cu_seqlens"].numpy(),
                                         causal, window, paired)
    err = np.abs(o.float().cpu().numpy() - o_ref)
    assert np.isfinite(err).all()
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    assert np.abs(lse.cpu().numpy() - lse_ref).max() <= LSE_ABS


def test_fp8_v_scale_is_exact_in_the_epilogue():
    """Doubling v_scale doubles every output element exactly (a power of two: bf16 rounding
    commutes with it)."""
    from paired_heads_b200 import pha

    w = synth.Workload("t", (300, 77), 4, 4, 128, "bf16")
    inp = synth.make_fp8_inputs(w)
    q8, k8, v8 = (inp[n].cuda() for n in ("q8", "k8", "v8"))
    cu = inp["cu_seqlens"].cuda()
    ws = torch.empty(pha.pha_attn_workspace_bytes(w.batch, w.max_len, 4, 128, False),
                     dtype=torch.uint8, device="cuda")
    outs = []
    for sv in (inp["v_scale"], 2 * inp["v_scale"]):
        o = torch.empty(w.total, 4, 128, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(w.total, 4, device="cuda")
        pha.pha_attn_fwd_fp8(q8, k8, v8, inp["q_scale"], inp["k_scale"], sv, cu, w.max_len, o, lse,
                             ws)
        outs.append((o, lse))
    assert torch.equal(outs[1][0].float(), 2 * outs[0][0].float())
    assert torch.equal(outs[1][1], outs[0][1])
