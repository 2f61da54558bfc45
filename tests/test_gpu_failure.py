"""A kernel wait that gives up, on the GPU, without faulting or hanging it: the band kernel's
failure-detection hook makes its softmax warps wait on a barrier that nothing signals, with a
short limit. The wait runs out, the kernel records device status 3, every role winds down (copies
and MMAs in flight drained, tensor memory freed) and no output row is written. A normal call on
the same stream and workspace then runs and matches the oracle: the context is still usable."""
import numpy as np
import pytest
import torch

import oracle
from paired_heads_b200 import synth

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_reports_status_3_and_leaves_the_context_usable():
    from paired_heads_b200 import build, pha

    build.build()
    w = synth.workload("paired_varlen", doc_lens=(300, 1, 129, 70))
    inp = synth.make_inputs(w)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    cu = inp["cu_seqlens"].cuda()
    ws = torch.empty(pha.pha_attn_workspace_bytes(w.batch, w.max_len, w.n_heads, w.head_dim, True),
                     dtype=torch.uint8, device="cuda")
    kw = dict(causal=True, window=w.window, paired=True)

    o = torch.full_like(q, float("nan"))
    lse = torch.full((w.total, w.n_heads), float("nan"), device="cuda")
    pha.pha_test_attn_fwd_stalled(q, k, v, cu, w.max_len, o, lse, ws, 2000, **kw)
    status, n_items = pha.pha_attn_status(ws)
    assert status == 3 and n_items > 0
    assert torch.isnan(o.float()).all() and torch.isnan(lse).all()   # nothing written

    pha.pha_attn_fwd(q, k, v, cu, w.max_len, o, lse, ws, **kw)
    status, _ = pha.pha_attn_status(ws)
    assert status == 0
    o_ref, lse_ref = oracle.attn_fwd(synth.to_f64(inp["q"]), synth.to_f64(inp["k"]),
                                     synth.to_f64(inp["v"]), inp["cu_seqlens"].numpy(), True,
                                     w.window, True)
    err = np.abs(o.float().cpu().numpy() - o_ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    assert np.abs(lse.cpu().numpy() - lse_ref).max() <= 1e-3
