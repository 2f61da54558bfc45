"""The scheduler's work-list cache (GPU): a workspace reused across calls keeps its list only while
everything the list was built from is unchanged -- the shape key, cu_seqlens and the items
themselves -- and every call matches the oracle."""
import numpy as np
import pytest
import torch

from paired_heads_b200 import synth
from pipeline import check, run_oracle

pytestmark = pytest.mark.gpu

HEADER_REUSED = 14   # int32 index of the header's "reused" field (kernels.cuh, WorkspaceHeader)
HEADER_BYTES = 256


def _reused(step) -> int:
    torch.cuda.synchronize()
    return int(step.workspace[:HEADER_BYTES].view(torch.int32)[HEADER_REUSED].item())


def _workload(lens, window):
    return synth.Workload("cache", tuple(lens), 4, 4, 128, "bf16", window=window, paired=True,
                          stagger=True)


@pytest.mark.parametrize("window", [128, 0, 300])   # band list, block lists
def test_alternating_cu_seqlens_on_one_workspace(window):
    from paired_heads_b200.runner import AttentionStep, StepShape

    # two document mixes with the same count, longest document and total: the shape key is the
    # same, only cu_seqlens tells them apart
    wa = _workload((300, 500, 224), window)
    wb = _workload((224, 500, 300), window)
    ia, ib = synth.make_inputs(wa), synth.make_inputs(wb)
    refs = {id(ia): run_oracle(wa, ia, rope=False), id(ib): run_oracle(wb, ib, rope=False)}
    step = AttentionStep(StepShape.of(wa, 1), "cuda")
    dev = torch.device("cuda")
    expect_reused = [0, 1, 0, 1, 0, 0]
    for n, (w, inp) in enumerate([(wa, ia), (wa, ia), (wb, ib), (wb, ib), (wa, ia), (wb, ib)]):
        q, k, v, cu = (inp[x].to(dev) for x in ("q", "k", "v", "cu_seqlens"))
        o, lse = step.attn(q, k, v, cu)
        assert _reused(step) == expect_reused[n], n
        assert step.status()[0] == 0
        check(w, o.cpu(), lse.cpu(), *refs[id(inp)])


def test_changed_items_are_rebuilt():
    from paired_heads_b200.runner import AttentionStep, StepShape

    w = _workload((300, 500, 224), 128)
    inp = synth.make_inputs(w)
    ref = run_oracle(w, inp, rope=False)
    step = AttentionStep(StepShape.of(w, 1), "cuda")
    dev = torch.device("cuda")
    q, k, v, cu = (inp[x].to(dev) for x in ("q", "k", "v", "cu_seqlens"))
    step.attn(q, k, v, cu)
    o1 = step.o.clone()
    step.attn(q, k, v, cu)
    assert _reused(step) == 1
    # overwrite one work item (the caller may use the workspace as scratch between calls)
    doc_bytes = (4 * (w.batch + 1) + 15) // 16 * 16
    item0 = HEADER_BYTES + doc_bytes
    step.workspace[item0:item0 + 16] = torch.arange(16, dtype=torch.uint8, device=dev)
    o, lse = step.attn(q, k, v, cu)
    assert _reused(step) == 0
    assert torch.equal(o, o1)
    check(w, o.cpu(), lse.cpu(), *ref)
    # and a changed shape (another window) is not taken for the same list
    step.s.window = 64
    step.attn(q, k, v, cu)
    assert _reused(step) == 0
    check(w.with_(window=64), step.o.cpu(), step.lse.cpu(), *run_oracle(w.with_(window=64), inp,
                                                                         rope=False))
