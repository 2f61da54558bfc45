"""Value embedding added to v inside the attention kernels (pha_attn_fwd_aux_v) on the GPU: bit for
bit the O and LSE of pha_attn_fwd on v + aux_v formed by a bf16 tensor addition, v and aux_v left
unchanged, and within the parity bar of the oracle, on the band kernel (causal windows <= 128)
and the block kernel (no window, longer windows). Needs a B200."""
import numpy as np
import pytest
import torch

import oracle
from paired_heads_b200 import synth
from pipeline import check, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paired_heads_b200 import build

    build.build()
    import paired_heads_b200.pha  # noqa: F401


def _both(w, inp, aux):
    from paired_heads_b200.runner import AttentionStep, StepShape

    dev = torch.device("cuda:0")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    a = aux.to(dev)
    cu = inp["cu_seqlens"].to(dev)
    step = AttentionStep(StepShape.of(w, 1), dev)
    assert step.aux_v_supported
    v0, a0 = v.clone(), a.clone()
    o, lse = step.attn_aux_v(q, k, v, a, cu)
    o_f, lse_f = o.clone(), lse.clone()
    torch.cuda.synchronize()
    assert step.status()[0] == 0
    assert torch.equal(v, v0) and torch.equal(a, a0)
    o_s, lse_s = step.attn(q, k, v + a, cu)   # the bf16 tensor addition
    torch.cuda.synchronize()
    return o_f.cpu(), lse_f.cpu(), o_s.cpu(), lse_s.cpu()


CASES = [
    # doc lens, H, Hkv, hd, window, paired -- windows <= 128 run on the band kernel, the others
    # (0 = no window) on the block kernel
    ((700, 5, 260), 6, 6, 128, 128, True),
    ((512, 513, 64, 1, 2049), 4, 2, 128, 128, True),
    ((1024, 1025, 127, 129, 1), 4, 2, 64, 2, False),
    ((3000, 7), 8, 2, 128, 100, False),
    ((333, 64), 8, 4, 64, 37, True),
    ((1500, 257, 1), 4, 4, 64, 0, False),
    ((900, 300), 8, 2, 128, 0, True),
    ((2100, 33), 4, 2, 64, 300, True),
    ((1030,), 4, 4, 128, 1024, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{len(c[0])}docs-H{c[1]}-hd{c[3]}-w{c[4]}-p{int(c[5])}")
def test_aux_v_matches_separate_add_and_oracle(case):
    lens, H, Hkv, hd, window, paired = case
    w = synth.Workload("auxv", lens, H, Hkv, hd, "bf16", causal=True, window=window,
                       paired=paired, stagger=paired)
    inp = synth.make_inputs(w)
    rng = np.random.default_rng(sum(lens))
    aux = torch.from_numpy(rng.standard_normal(tuple(inp["v"].shape)).astype(np.float32)).to(torch.bfloat16)
    o_f, lse_f, o_s, lse_s = _both(w, inp, aux)
    assert torch.equal(o_f.view(torch.int16), o_s.view(torch.int16))
    assert torch.equal(lse_f.view(torch.int32), lse_s.view(torch.int32))
    vs = oracle.add_stored(synth.to_f64(inp["v"]), synth.to_f64(aux), "bf16")
    o_ref, lse_ref = oracle.attn_fwd(synth.to_f64(inp["q"]), synth.to_f64(inp["k"]), vs,
                                     inp["cu_seqlens"].numpy(), True, window, paired, w.scale)
    check(w, o_f, lse_f, o_ref, lse_ref)


def test_aux_v_full_size_paired_varlen():
    w = synth.workload("paired_varlen")
    inp = synth.make_inputs(w)
    rng = np.random.default_rng(5)
    aux = torch.from_numpy(rng.standard_normal(tuple(inp["v"].shape)).astype(np.float32)).to(torch.bfloat16)
    o_f, lse_f, o_s, lse_s = _both(w, inp, aux)
    assert torch.equal(o_f.view(torch.int16), o_s.view(torch.int16))
    assert torch.equal(lse_f.view(torch.int32), lse_s.view(torch.int32))
    rows = sample_rows(w, 200)
    vs = oracle.add_stored(synth.to_f64(inp["v"]), synth.to_f64(aux), "bf16")
    o_ref, lse_ref = oracle.attn_rows(synth.to_f64(inp["q"]), synth.to_f64(inp["k"]), vs,
                                      inp["cu_seqlens"].numpy(), rows, True, w.window, True, w.scale)
    idx = torch.from_numpy(np.asarray(rows))
    check(w, o_f.reshape(-1, w.head_dim)[idx], lse_f.reshape(-1)[idx], o_ref, lse_ref)
