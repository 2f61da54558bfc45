"""World-size-2 data-parallel plumbing on CPU (gloo): each rank draws its own documents of the
same shape, runs the oracle on them, and the timing reduce returns the maximum over ranks."""
import multiprocessing as mp
import os
import socket

import numpy as np


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    try:
        import torch

        import oracle
        from paired_heads_b200 import dist as pdist
        from paired_heads_b200 import synth

        d = pdist.init("gloo", timeout_s=60)
        w = synth.workload("paired_varlen", doc_lens=(100, 37, 200))
        inp = synth.make_inputs(w, rank=rank)
        o, lse = oracle.attn_fwd(synth.to_f64(inp["q"]), synth.to_f64(inp["k"]),
                                 synth.to_f64(inp["v"]), inp["cu_seqlens"].numpy(), True,
                                 w.window, True)
        # each rank's documents differ; gather a checksum of the inputs and of the outputs
        cs = torch.tensor([float(inp["q"].float().sum()), float(np.sum(o))], dtype=torch.float64)
        allcs = [torch.zeros_like(cs) for _ in range(world)]
        d.all_gather(allcs, cs)
        elapsed = 1.0 + rank * 0.25
        mx = pdist.max_over_ranks(d, elapsed)
        pdist.finalize(d)
        q.put((rank, [c.tolist() for c in allcs], mx, bool(np.all(np.isfinite(lse)))))
    except Exception as e:  # report, never hang the parent
        q.put((rank, "error", repr(e), False))


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r = q.get(timeout=120)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        assert res[r][1] != "error", res[r]
        assert res[r][2] == 1.25            # max over ranks
        assert res[r][3]
    gathered = res[0][1]
    assert gathered == res[1][1]
    assert gathered[0] != gathered[1]       # distinct documents per rank


def test_single_process_is_a_no_op():
    from paired_heads_b200 import dist as pdist

    assert pdist.init("gloo") is None
    assert pdist.max_over_ranks(None, 3.5) == 3.5
