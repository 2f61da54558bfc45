"""Host logic of bench.py (no GPU): the algorithmic counters against brute force, the e2e leg's
partition of documents into chunks, and the validity check of the committed ncu traffic."""
import importlib.util
import json
import os

import numpy as np
import pytest

from paired_heads_b200 import build, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("lens,H,causal,window,paired", [
    ((5, 1, 12), 4, True, 0, False),
    ((5, 1, 12), 4, True, 3, False),
    ((7, 9), 2, False, 0, False),
    ((7, 9, 1), 6, True, 4, True),
    ((130,), 2, True, 128, True),
])
def test_visible_pairs_brute_force(bench, lens, H, causal, window, paired):
    w = synth.Workload("t", lens, H, H, 16, "bf16", causal=causal, window=window, paired=paired)
    m = 2 if paired else 1
    want = 0
    for n in lens:
        L = n * m
        i, j = np.arange(L)[:, None], np.arange(L)[None, :]
        vis = np.ones((L, L), dtype=bool)
        if causal:
            vis &= j <= i
            if window > 0:
                vis &= i - j < window
        want += int(vis.sum())
    want *= H // m
    assert bench.visible_pairs(w) == want
    assert bench.attn_flops(w) == 4.0 * 16 * want


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("n_chunks", [1, 2, 4, 8])
def test_doc_chunks_partition(bench, seed, n_chunks):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, 300, rng.integers(1, 40))   # zero-length documents included
    cu = [0] + np.cumsum(lens).tolist()
    chunks = bench.doc_chunks(cu, n_chunks)
    assert 1 <= len(chunks) <= n_chunks
    assert chunks[0][0] == 0 and chunks[-1][1] == len(lens)
    for (a0, a1), (b0, _) in zip(chunks, chunks[1:]):
        assert a1 == b0                                 # contiguous, each document once
    assert all(a1 > a0 for a0, a1 in chunks)            # no empty group


def test_load_traffic_follows_the_sources(bench, tmp_path, monkeypatch):
    w = synth.workload("paired_varlen")
    srcs = ["paired_heads_b200/csrc/rope.cu", "paired_heads_b200/csrc/ptx.cuh"]
    key = f"{w.name}:w{w.window}:p{int(w.paired)}:rope"
    (tmp_path / "profiles").mkdir()

    def write(entry):
        (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({key: entry}))

    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    write({"bytes_per_launch": 123, "sources": srcs, "sources_sha": build.files_sha(srcs)})
    assert bench.load_traffic(w, "rope") == 123
    write({"bytes_per_launch": 123, "sources": srcs, "sources_sha": "0" * 16})
    assert bench.load_traffic(w, "rope") is None       # a kernel source changed since the capture
    assert bench.load_traffic(w, "attention") is None  # no entry
    assert bench.load_traffic(synth.workload("gpt2"), "rope") is None


def test_committed_traffic_entries_name_existing_sources():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    for key, ent in d.items():
        if key.startswith("_"):
            continue
        assert ent["bytes_per_launch"] == ent["read"] + ent["write"]
        for rel in ent["sources"]:
            assert os.path.exists(os.path.join(ROOT, rel)), rel


def test_gpus_two_starts_two_ranks():
    """`bench.py --gpus 2` run without a launcher re-runs itself as two processes under
    torch.distributed.run; --launch-check makes each rank join a gloo group and report its id."""
    import socket
    import subprocess
    import sys

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env["MASTER_PORT"] = str(port)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--launch-check"], capture_output=True, text=True, timeout=240, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["world"] == 2 and d["ranks"] == [0, 1]


def test_rope_bytes_by_table_form(bench):
    # stored tables: q and k read and written, plus a cos and a sin row per token; factored tables:
    # q and k read and written, plus the factor tables once (16 fine rows, one coarse row per 16)
    w = synth.workload("paired_varlen")
    qk = 2 * w.total * (w.n_heads + w.n_kv_heads) * w.head_dim * 2
    assert bench.rope_bytes(w, "stored") == qk + 2 * 4 * w.total * 2 * w.head_dim
    rows = 131072
    fac = (16 * w.head_dim + (rows // 16) * (w.head_dim // 2)) * 16
    assert bench.rope_bytes(w, "factored", rows) == qk + fac
    g = synth.workload("gpt2")  # unpaired: fine rows hold head_dim / 2 angles
    qk_g = 2 * g.total * (g.n_heads + g.n_kv_heads) * g.head_dim * 2
    assert bench.rope_bytes(g, "factored", 1000) == qk_g + (16 * (g.head_dim // 2) + 63 * (g.head_dim // 2)) * 16
