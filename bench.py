"""Benchmark: one step = RoPE on q and k + varlen (paired-head) attention forward, on synthetic
inputs resident in HBM. Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--window W]
                    [--paired 0|1] [--qk-norm] [--aux-v] [--backward] [--impl reference]
                    [--rope-tables factored|stored]

--rope-tables picks the rotary tables of the step's RoPE: the compact float64 factor tables
(pha_rope_factored, default) or the stored float32 cos / sin rows (pha_rope); the other form is
timed after the step on the same inputs and reported beside it.

--qk-norm replaces pha_rope with pha_qk_norm_rope (the QK RMS-norm of every head row, then RoPE,
in one kernel). --aux-v adds a value embedding (a second v-shaped tensor) to v inside the
attention kernel (pha_attn_fwd_aux_v). --backward also times the backward (pha_attn_bwd +
pha_rope_bwd) after the forward step and reports it under "backward" (not in `value`).

Default workload: the paired-head varlen packed batch (65,536 tokens, documents ~ geometric(512)
capped at 2048, 6 heads -> 3 pairs, head_dim 128, bf16, causal, window 128 slots, staggered
rotary). N > 1 runs under torchrun, one process per GPU, each rank with its own documents of the
same shape (weak scaling; the forward needs no collective, so only the timing reduce crosses
ranks).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paired_heads_b200 import synth  # noqa: E402

METRIC = "attention fwd TFLOP/s (causal-counted) and % of bf16 tensor peak on 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- workload algebra

def visible_pairs(w) -> int:
    """Number of (query slot, head, visible key) triples of the attention (the causal count)."""
    mult = 2 if w.paired else 1
    heads = w.n_heads // mult
    total = 0
    for n in w.doc_lens:
        L = n * mult
        i = np.arange(L, dtype=np.int64)
        vis = (i + 1) if w.causal else np.full(L, L, dtype=np.int64)
        if w.window > 0:
            vis = np.minimum(vis, w.window)
        total += int(vis.sum())
    return total * heads


def doc_chunks(cu, n_chunks: int):
    """Split documents 0 .. len(cu) - 2 (token offsets cu) into at most n_chunks contiguous groups
    of about equal token counts: a list of (first doc, last doc + 1), covering every document once,
    each group holding at least one document."""
    batch = len(cu) - 1
    chunks = []
    d0 = 0
    for c in range(n_chunks):
        target = cu[-1] * (c + 1) / n_chunks
        d1 = d0 + 1
        while d1 < batch and (cu[d1] < target or d1 == d0) and c < n_chunks - 1:
            d1 += 1
        if c == n_chunks - 1:
            d1 = batch
        if d1 > d0:
            chunks.append((d0, d1))
        d0 = d1
        if d0 >= batch:
            break
    return chunks


def attn_flops(w) -> float:
    return 4.0 * w.head_dim * visible_pairs(w)


def attn_bytes(w) -> float:
    esz = 2 if w.dtype == "bf16" else 4
    return float(w.total * w.head_dim * esz * (2 * w.n_heads + 2 * w.n_kv_heads) + 4 * w.total * w.n_heads)


def rope_bytes(w, tables: str = "stored", tab_rows: int = 0) -> float:
    """Algorithmic HBM bytes of one RoPE call: q and k read and written, plus the tables: a cos
    and a sin row per token (stored), or the factor tables read once (factored, L1 / L2-resident
    after that)."""
    esz = 2 if w.dtype == "bf16" else 4
    qk = 2 * w.total * (w.n_heads + w.n_kv_heads) * w.head_dim * esz
    if tables == "stored":
        return float(qk + 2 * 4 * w.total * (2 if w.paired else 1) * w.head_dim)
    a_width = w.head_dim if w.paired else w.head_dim // 2
    fac = (16 * a_width + -(-tab_rows // 16) * (w.head_dim // 2)) * 16
    return float(qk + fac)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def pick_workload(args):
    kw = {}
    if args.window is not None:
        kw["window"] = args.window
    if args.paired is not None:
        kw["paired"] = bool(args.paired)
        kw["stagger"] = bool(args.paired)
    return synth.workload(args.workload, **kw)


def workload_config(w) -> dict:
    return {"workload": w.name, "tokens": w.total, "docs": w.batch, "max_doc_len": w.max_len,
            "n_heads": w.n_heads, "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
            "causal": w.causal, "window": w.window, "paired": w.paired, "stagger": w.stagger,
            "rope_positions": w.positions}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- oracle timing

def oracle_sample(w, budget_tokens: int):
    """The leading documents of the workload, up to ~budget_tokens tokens (at least one)."""
    lens, acc = [], 0
    for n in w.doc_lens:
        if acc and acc + n > budget_tokens:
            break
        lens.append(n)
        acc += n
    return w.with_(doc_lens=tuple(lens))


def time_oracle(w, budget_tokens: int, qk_norm: bool = False):
    """Oracle (float64 C) run of one step (RoPE stored in the buffer dtype + attention) on a
    bounded sample of the workload. Returns (TFLOP/s, seconds, sample workload, threads)."""
    import oracle

    s = oracle_sample(w, budget_tokens)
    inp = synth.make_inputs(s)
    q, k, v = (synth.to_f64(inp[n]) for n in ("q", "k", "v"))
    pos = inp["positions"].numpy()
    t0 = time.perf_counter()
    if qk_norm:
        qr = oracle.norm_rope_stored(q, pos, w.dtype, w.paired, w.stagger, w.rope_base)
        kr = oracle.norm_rope_stored(k, pos, w.dtype, w.paired, w.stagger, w.rope_base)
    else:
        qr = oracle.rope_stored(q, pos, w.dtype, w.paired, w.stagger, w.rope_base)
        kr = oracle.rope_stored(k, pos, w.dtype, w.paired, w.stagger, w.rope_base)
    oracle.attn_fwd(qr, kr, v, inp["cu_seqlens"].numpy(), w.causal, w.window, w.paired, w.scale)
    dt = time.perf_counter() - t0
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return attn_flops(s) / dt / 1e12, dt, s, threads


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="paired_varlen", choices=synth.WORKLOADS)
    ap.add_argument("--window", type=int, default=None)
    ap.add_argument("--paired", type=int, default=None)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--qk-norm", action="store_true",
                    help="QK RMS-norm + RoPE (pha_qk_norm_rope) instead of RoPE alone")
    ap.add_argument("--backward", action="store_true",
                    help="also time the backward (pha_attn_bwd + pha_rope_bwd)")
    ap.add_argument("--aux-v", action="store_true",
                    help="add a value embedding to v inside attention (pha_attn_fwd_aux_v)")
    ap.add_argument("--rope-tables", default="factored", choices=["factored", "stored"],
                    help="RoPE with the factored float64 tables (pha_rope_factored) or the stored "
                         "float32 rows (pha_rope)")
    ap.add_argument("--oracle-tokens", type=int, default=16384)
    ap.add_argument("--no-suite", action="store_true",
                    help="skip the per-workload timings of the other page-shaped workloads")
    ap.add_argument("--launch-check", action="store_true",
                    help="start the ranks, join a gloo group, print each rank's id and exit "
                         "(tests the multi-process launch without a GPU)")
    args = ap.parse_args()
    w = pick_workload(args)

    from paired_heads_b200 import dist as pdist

    rank, world, local_rank = pdist.env()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        raise SystemExit(launch_ranks(args.gpus))
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but {world} ranks were launched")

    if args.launch_check:
        d = pdist.init("gloo", timeout_s=60)
        ranks = pdist.gather_ints(d, rank)
        if rank == 0:
            print(json.dumps({"launch_check": True, "world": world, "ranks": ranks}))
        pdist.finalize(d)
        return

    if args.impl == "reference":
        return run_reference(args, w, rank, world)

    import torch

    from paired_heads_b200.runner import AttentionStep, StepShape

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = pdist.init("nccl", device=dev)

    inp = synth.make_inputs(w, rank=rank)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    cu, pos = inp["cu_seqlens"].to(dev), inp["positions"].to(dev)
    tab_rows = int(inp["positions"].max()) + 1
    step = AttentionStep(StepShape.of(w, tab_rows), dev, rope_tables=args.rope_tables)
    stream = torch.cuda.current_stream(dev)

    def rotary(qq, kk, pp):
        if args.qk_norm:
            step.norm_rope(qq, kk, pp)
        else:
            step.rope(qq, kk, pp)

    aux = None
    if args.aux_v:
        if not step.aux_v_supported:
            raise SystemExit("--aux-v needs the bf16 tensor-core path (head_dim 64 or 128)")
        g = torch.Generator().manual_seed(7 + 1000 * rank)
        aux = torch.randn(tuple(v.shape), generator=g).to(v.dtype).to(dev)

    def attention(qq, kk, vv, cc, aa):
        if args.aux_v:
            return step.attn_aux_v(qq, kk, vv, aa, cc)
        return step.attn(qq, kk, vv, cc)

    def run_step():
        rotary(q, k, pos)
        attention(q, k, v, cu, aux)

    for _ in range(max(args.warmup, 3)):
        run_step()
    torch.cuda.synchronize(dev)
    status, n_items = step.status()
    if status != 0:
        raise SystemExit(f"device status {status} after warm-up")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.get_device_properties(dev).index if hasattr(
        torch.cuda.get_device_properties(dev), "index") else local_rank)
    clocks.start()
    time.sleep(0.3)
    pdist.barrier(dist)
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        ev[s][0].record(stream)
        rotary(q, k, pos)
        ev[s][1].record(stream)
        attention(q, k, v, cu, aux)
        ev[s][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    pdist.barrier(dist)
    clk = clocks.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    rope_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    attn_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    status, _ = step.status()
    if status != 0:
        raise SystemExit(f"device status {status} after timing")

    elapsed_ms = pdist.max_over_ranks(dist, elapsed_ms, dev)
    ms_per_step = elapsed_ms / args.steps

    # ---- backward (optional): gradients of the step for a fixed upstream gradient
    bwd = None
    if args.backward:
        g_up = torch.randn(tuple(q.shape), generator=torch.Generator().manual_seed(11)).to(q.dtype).to(dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        for _ in range(3):
            step.attn_bwd(q, k, v, g_up, cu, dq, dk, dv)
            step.rope_bwd(dq, dk, pos)
        torch.cuda.synchronize(dev)
        nb = max(3, min(args.steps, 20))
        bev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(nb)]
        pdist.barrier(dist)
        for e in bev:
            e[0].record(stream)
            step.attn_bwd(q, k, v, g_up, cu, dq, dk, dv)
            e[1].record(stream)
            step.rope_bwd(dq, dk, pos)
            e[2].record(stream)
        torch.cuda.synchronize(dev)
        b_ms = pdist.max_over_ranks(dist, bev[0][0].elapsed_time(bev[-1][2]) / nb, dev)
        ab_ms = sum(e[0].elapsed_time(e[1]) for e in bev) / nb
        rb_ms = sum(e[1].elapsed_time(e[2]) for e in bev) / nb
        bwd_flops = 2.5 * attn_flops(w)
        tc_bwd = w.dtype == "bf16" and w.head_dim in (64, 128)
        bwd = {"ms": b_ms, "steps": nb, "flops": bwd_flops,
               "tflops": bwd_flops * world / (b_ms * 1e-3) / 1e12,
               "attn_bwd_ms": ab_ms, "rope_bwd_ms": rb_ms,
               "attn_bwd_tflops": bwd_flops / (ab_ms * 1e-3) / 1e12,
               "attn_bwd_frac_of_bf16_peak": bwd_flops / (ab_ms * 1e-3) / 1e12 / load_peaks()[0]["bf16_tflops"],
               "kernels": ("pha_attn_bwd: D = dO.O, then the dQ and dK/dV kernels on the tensor cores "
                           "(tcgen05)" if tc_bwd else
                           "pha_attn_bwd: D = dO.O, then dq and dk/dv on CUDA cores") +
                          "; then pha_rope_bwd",
               "flop_count": "2.5 x the forward's causal-counted FLOPs (S, dP, dV, dK, dQ)",
               "traffic_per_launch": {"dq_kernel": load_traffic(w, "attn_bwd_dq"),
                                      "dkdv_kernel": load_traffic(w, "attn_bwd_dkdv")}
               if tc_bwd else None}

    # ---- end to end through the public API with host buffers. Documents are independent, so the
    # step is issued in chunks of whole documents on three streams, one a stage: host->device
    # copies, kernels, device->host copies, chained per chunk by events. The copy-in stream thus
    # never waits for a kernel or a copy-out (the host->device link is the bound), and the
    # copy-out of one chunk runs beside the copy-in of the next. Every input byte is copied in and
    # every output byte copied out within each timed step. Steps follow each other as a stream of
    # batches would: a chunk's buffers are refilled once the previous step's kernels on that chunk
    # are done, and its outputs rewritten once the previous step's copy-out of them is done.
    host = {n: inp[n].pin_memory() for n in ("q", "k", "v", "cu_seqlens", "positions")}
    if args.aux_v:
        host["aux_v"] = aux.cpu().pin_memory()
    o_host = torch.empty(step.o.shape, dtype=step.o.dtype).pin_memory()
    lse_host = torch.empty(step.lse.shape, dtype=torch.float32).pin_memory()
    cu_h = host["cu_seqlens"].tolist()
    chunks = doc_chunks(cu_h, max(1, min(8, w.batch)))
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    parts = []
    for (a0, a1) in chunks:
        t0, t1 = cu_h[a0], cu_h[a1]
        sub = w.with_(doc_lens=tuple(w.doc_lens[a0:a1]))
        st_ = AttentionStep(StepShape.of(sub, tab_rows), dev, rope_tables=args.rope_tables)
        bufs = {n: torch.empty((t1 - t0,) + tuple(host[n].shape[1:]), dtype=host[n].dtype, device=dev)
                for n in host if n not in ("cu_seqlens", "positions")}
        bufs["cu_seqlens"] = torch.empty(a1 - a0 + 1, dtype=torch.int32, device=dev)
        bufs["positions"] = torch.empty(t1 - t0, dtype=torch.int32, device=dev)
        hsrc = {n: host[n][t0:t1] for n in host if n not in ("cu_seqlens",)}
        hsrc["cu_seqlens"] = (host["cu_seqlens"][a0:a1 + 1] - t0).pin_memory()
        parts.append((st_, bufs, hsrc, t0, t1))

    ev_in = [torch.cuda.Event() for _ in parts]
    ev_k = [torch.cuda.Event() for _ in parts]
    ev_out = [torch.cuda.Event() for _ in parts]

    def e2e_step():
        for c, (st_, bufs, hsrc, t0, t1) in enumerate(parts):
            s_in.wait_event(ev_k[c])  # the previous step's kernels on this chunk are done
            with torch.cuda.stream(s_in):
                for n, t in bufs.items():
                    t.copy_(hsrc[n], non_blocking=True)
                ev_in[c].record(s_in)
            s_comp.wait_event(ev_in[c])
            s_comp.wait_event(ev_out[c])  # the previous step's outputs of this chunk are out
            with torch.cuda.stream(s_comp):
                if args.qk_norm:
                    st_.norm_rope(bufs["q"], bufs["k"], bufs["positions"])
                else:
                    st_.rope(bufs["q"], bufs["k"], bufs["positions"])
                if args.aux_v:
                    o, lse = st_.attn_aux_v(bufs["q"], bufs["k"], bufs["v"], bufs["aux_v"], bufs["cu_seqlens"])
                else:
                    o, lse = st_.attn(bufs["q"], bufs["k"], bufs["v"], bufs["cu_seqlens"])
                ev_k[c].record(s_comp)
            s_out.wait_event(ev_k[c])
            with torch.cuda.stream(s_out):
                o_host[t0:t1].copy_(o, non_blocking=True)
                lse_host[t0:t1].copy_(lse, non_blocking=True)
                ev_out[c].record(s_out)

    def e2e_run(n_steps, start_event):
        for sc in (s_in, s_comp, s_out):
            sc.wait_event(start_event)
        for _ in range(n_steps):
            e2e_step()
        for sc in (s_in, s_comp, s_out):
            stream.wait_stream(sc)

    ev0 = torch.cuda.Event()
    ev0.record(stream)
    e2e_run(3, ev0)
    torch.cuda.synchronize(dev)
    e_steps = max(5, min(args.steps, 20))
    pdist.barrier(dist)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    e2e_run(e_steps, a)
    b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = pdist.max_over_ranks(dist, a.elapsed_time(b) / e_steps, dev)
    h2d = sum(host[n].numel() * host[n].element_size() for n in host)
    d2h = o_host.numel() * o_host.element_size() + lse_host.numel() * 4

    # the other RoPE table form on the same inputs, for comparison (not part of `value`)
    alt_tables = "stored" if args.rope_tables == "factored" else "factored"
    alt = AttentionStep(StepShape.of(w, tab_rows), dev, rope_tables=alt_tables)
    alt_rope = alt.norm_rope if args.qk_norm else alt.rope
    for _ in range(3):
        alt_rope(q, k, pos)
    alt_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)]
              for _ in range(max(5, min(args.steps, 50)))]
    for e in alt_ev:
        e[0].record(stream)
        alt_rope(q, k, pos)
        e[1].record(stream)
    torch.cuda.synchronize(dev)
    alt_ms = sum(e[0].elapsed_time(e[1]) for e in alt_ev) / len(alt_ev)
    del alt

    flops = attn_flops(w)
    peaks, peak_src = load_peaks()
    value = flops * world / (ms_per_step * 1e-3) / 1e12
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    rname = "qk_norm_rope" if args.qk_norm else "rope"
    rb = rope_bytes(w, args.rope_tables, tab_rows)
    # the value embedding is one more v-shaped read of the attention kernel
    ab = attn_bytes(w) + (float(w.total * w.n_kv_heads * w.head_dim * 2) if args.aux_v else 0.0)
    kernels = {
        rname: {"ms": rope_ms, "tables": args.rope_tables, "bytes": rb,
                 "gbs": rb / (rope_ms * 1e-3) / 1e9,
                 "frac_of_hbm": rb / (rope_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                 "traffic": load_traffic(w, rname + ("_factored" if args.rope_tables == "factored"
                                                     else ""))},
        f"{rname}_{alt_tables}": {
            "ms": alt_ms, "tables": alt_tables, "bytes": rope_bytes(w, alt_tables, tab_rows),
            "gbs": rope_bytes(w, alt_tables, tab_rows) / (alt_ms * 1e-3) / 1e9,
            "note": "the other table form, timed after the step on the same inputs; not in value"},
        "attention": {"ms": attn_ms, "flops": flops, "bytes": ab,
                      "tflops": attn_tflops,
                      "gbs": ab / (attn_ms * 1e-3) / 1e9,
                      "frac_of_hbm": ab / (attn_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                      "frac_of_bf16_peak": attn_tflops / peaks["bf16_tflops"],
                      "traffic": load_traffic(w, "attention")},
    }
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    attn_bound = "hbm" if flops / ab < ridge else "tensor"
    dominant = "attention" if attn_ms >= rope_ms else rname
    if dominant == rname or attn_bound == "hbm":
        kname = dominant
        achieved = kernels[kname]["gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
    else:
        kname = "attention"
        roof = {"bound": "tensor", "achieved": attn_tflops, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": attn_tflops / peaks["bf16_tflops"]}
    roof["kernel"] = kname
    roof["peak_source"] = f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'})"
    roof["traffic"] = kernels[kname]["traffic"]
    roof["timing"] = ("CUDA events on the launching stream around each library call in the timed "
                      "region; the attention call includes its scheduler kernel")

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded N(0,1) q/k/v; geometric document lengths)",
        "config": {**workload_config(w), "qk_norm": bool(args.qk_norm), "aux_v": bool(args.aux_v),
                   "rope_tables": args.rope_tables,
                   "parallelism": f"dp{world} (independent documents per rank)",
                   "l2": (f"inputs larger than L2 (q, k, v {attn_bytes(w) / 1e6:.0f} MB > 126 MB); "
                          "no flush")},
        "pct_of_bf16_peak": 100.0 * value / world / peaks["bf16_tflops"],
        "attention_only_tflops": attn_tflops,
        "tokens_per_s": w.total * world / (ms_per_step * 1e-3),
        "kernels": kernels,
        "roofline": roof,
        "e2e": {"value": flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "chunks": len(parts),
                "how": "public API from pinned host buffers, whole-document chunks on three "
                       "streams (copy-in, kernels, copy-out, chained by events: a chunk's copy-in "
                       "overlaps the previous chunks' kernels and copy-out, and the next step's "
                       "copy-in the end of this one)"},
        "gpu_launches": 3 * args.steps,
        "work_items": n_items,
        "clocks": clk,
    }
    if bwd is not None:
        line["backward"] = bwd
    if not args.no_suite and args.workload == "paired_varlen" and not (args.qk_norm or args.aux_v):
        line["configs"] = time_suite(max(3, min(args.steps, 20)), args.warmup, dev, peaks, rank,
                                     args.rope_tables)
        line["fp8"] = time_fp8(max(3, min(args.steps, 20)), args.warmup, dev, peaks, rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, secs, s, thr = time_oracle(w, args.oracle_tokens, args.qk_norm)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                                "seconds": secs,
                                "sample": f"first {s.batch} documents ({s.total} tokens) of the "
                                          f"workload: float64 {'QK RMS-norm + ' if args.qk_norm else ''}"
                                          f"RoPE + attention, full rows"}
    if rank == 0:
        print(json.dumps(line))
    pdist.finalize(dist)


# The other workloads of the page-shaped suite, timed after the headline in the default run:
# (label, workload, overrides). The mixed-window workload runs at each window, paired or not.
SUITE = (
    ("gpt2", "gpt2", {}),
    ("mixed_window_w128", "mixed_window", {"window": 128}),
    ("mixed_window_w128_paired", "mixed_window", {"window": 128, "paired": True, "stagger": True}),
    ("mixed_window_w1024", "mixed_window", {"window": 1024}),
    ("mixed_window_w1024_paired", "mixed_window", {"window": 1024, "paired": True, "stagger": True}),
    ("mixed_window_full", "mixed_window", {"window": 0}),
    ("mixed_window_full_paired", "mixed_window", {"window": 0, "paired": True, "stagger": True}),
    ("gqa_long", "gqa_long", {}),
)
L2_BYTES = 126 * 1024 * 1024


def time_suite(steps: int, warmup: int, dev, peaks, rank: int = 0, rope_tables: str = "factored"):
    """RoPE + attention on each workload of SUITE, timed per call with CUDA events on the launching
    stream. Workloads whose inputs fit in L2 get a 256 MiB buffer written before every step (outside
    the events). Returns {label: {...}}."""
    import torch

    from paired_heads_b200.runner import AttentionStep, StepShape

    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    out = {}
    for label, name, kw in SUITE:
        w = synth.workload(name, **kw)
        inp = synth.make_inputs(w, rank=rank)
        q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
        cu, pos = inp["cu_seqlens"].to(dev), inp["positions"].to(dev)
        rows = int(inp["positions"].max()) + 1
        step = AttentionStep(StepShape.of(w, rows), dev, rope_tables=rope_tables)
        rb = rope_bytes(w, rope_tables, rows)
        in_l2 = attn_bytes(w) + rb < L2_BYTES
        for _ in range(max(warmup, 3)):
            step.rope(q, k, pos)
            step.attn(q, k, v, cu)
        torch.cuda.synchronize(dev)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        sampler = ClockSampler(dev.index if dev.index is not None else 0)
        sampler.start()
        time.sleep(0.2)
        for s in range(steps):
            if in_l2:
                flush.fill_(s & 0xFF)
            ev[s][0].record(stream)
            step.rope(q, k, pos)
            ev[s][1].record(stream)
            step.attn(q, k, v, cu)
            ev[s][2].record(stream)
        torch.cuda.synchronize(dev)
        clk = sampler.stop()
        status, _ = step.status()
        if status != 0:
            raise SystemExit(f"{label}: device status {status}")
        rope_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
        attn_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / steps
        flops, ab = attn_flops(w), attn_bytes(w)
        tflops = flops / (attn_ms * 1e-3) / 1e12
        ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
        bound = "hbm" if flops / ab < ridge else "tensor"
        roof_tflops = min(peaks["bf16_tflops"], flops / ab * peaks["hbm_gbs"] * 1e9 / 1e12)
        out[label] = {
            "tokens": w.total, "n_heads": w.n_heads, "n_kv_heads": w.n_kv_heads,
            "head_dim": w.head_dim, "window": w.window, "paired": w.paired,
            "kernel": "band" if (w.causal and 1 <= w.window <= 128) else "block",
            "attn_ms": attn_ms, "attn_tflops": tflops,
            "frac_of_bf16_peak": tflops / peaks["bf16_tflops"],
            "bound": bound, "frac_of_roofline": tflops / roof_tflops,
            "attn_gbs": ab / (attn_ms * 1e-3) / 1e9,
            "rope_ms": rope_ms, "rope_gbs": rb / (rope_ms * 1e-3) / 1e9,
            "step_ms": rope_ms + attn_ms,
            "tokens_per_s": w.total / ((rope_ms + attn_ms) * 1e-3),
            "l2": "flushed (256 MiB write) before each step" if in_l2 else "inputs larger than L2",
            "steps": steps, "sm_mhz": clk.get("sm_mhz"), "clock_reasons": clk.get("reasons"),
        }
        del q, k, v, cu, pos, step, inp
        torch.cuda.empty_cache()
    return out


FP8_SUITE = (("paired_varlen", "paired_varlen", {}),
             ("mixed_window_full", "mixed_window", {"window": 0}),
             ("gqa_long", "gqa_long", {}))


def time_fp8(steps: int, warmup: int, dev, peaks, rank: int = 0):
    """pha_attn_fwd_fp8 on e4m3 copies of the workloads' q, k, v (per-tensor scales), timed per
    call with CUDA events. S = Q K^T runs in kind::f8f6f4 (twice the bf16 rate, nominally), P V in
    kind::f16, so the applicable tensor peak is 4/3 of the bf16 one (half the FLOPs at each rate)."""
    import torch

    from paired_heads_b200 import pha

    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    out = {}
    for label, name, kw in FP8_SUITE:
        w = synth.workload(name, **kw)
        inp = synth.make_fp8_inputs(w, rank=rank)
        q8, k8, v8 = (inp[n].to(dev) for n in ("q8", "k8", "v8"))
        cu = inp["cu_seqlens"].to(dev)
        o = torch.empty(w.total, w.n_heads, w.head_dim, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(w.total, w.n_heads, device=dev)
        ws = torch.empty(pha.pha_attn_workspace_bytes(w.batch, w.max_len, w.n_heads, w.head_dim,
                                                      w.paired), dtype=torch.uint8, device=dev)
        sc = (inp["q_scale"], inp["k_scale"], inp["v_scale"])

        def call():
            pha.pha_attn_fwd_fp8(q8, k8, v8, *sc, cu, w.max_len, o, lse, ws, causal=w.causal,
                                 window=w.window, paired=w.paired, scale=w.scale)

        for _ in range(max(warmup, 3)):
            call()
        torch.cuda.synchronize(dev)
        fbytes = float(w.total * w.head_dim * (w.n_heads + 2 * w.n_kv_heads)
                       + 2 * w.total * w.n_heads * w.head_dim + 4 * w.total * w.n_heads)
        in_l2 = fbytes < L2_BYTES
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for s_ in range(steps):
            if in_l2:
                flush.fill_(s_ & 0xFF)
            ev[s_][0].record(stream)
            call()
            ev[s_][1].record(stream)
        torch.cuda.synchronize(dev)
        status, _ = pha.pha_attn_status(ws)
        if status != 0:
            raise SystemExit(f"fp8 {label}: device status {status}")
        ms = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
        flops = attn_flops(w)
        tf = flops / (ms * 1e-3) / 1e12
        out[label] = {"attn_ms": ms, "attn_tflops": tf,
                      "frac_of_bf16_peak": tf / peaks["bf16_tflops"],
                      "frac_of_mixed_peak": tf / (peaks["bf16_tflops"] * 4.0 / 3.0),
                      "bytes": fbytes, "gbs": fbytes / (ms * 1e-3) / 1e9,
                      "frac_of_hbm": fbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "steps": steps}
        del q8, k8, v8, o, lse, ws, inp
        torch.cuda.empty_cache()
    return out


def launch_ranks(n: int) -> int:
    """Re-run this command as n processes on one node (one per GPU) under torch.distributed.run.
    Returns the launcher's exit code."""
    port = int(os.environ.get("MASTER_PORT", "29517"))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__),
           *sys.argv[1:]]
    return subprocess.call(cmd)


def load_traffic(w, kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it matches this workload and
    the kernel's current sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    key = f"{w.name}:w{w.window}:p{int(w.paired)}:{kernel}"
    ent = d.get(key)
    if not ent:
        return None
    from paired_heads_b200 import build as b

    # valid while the files that define this kernel's device code are those that were captured
    now = b.files_sha(ent["sources"]) if "sources" in ent else b.sources_sha()
    if ent.get("sources_sha") != now:
        return None
    return ent.get("bytes_per_launch")


def run_reference(args, w, rank, world):
    """The oracle, as it stands, timed on the host cores on a bounded sample per step."""
    if rank != 0:
        return
    for _ in range(max(args.warmup, 0)):
        pass  # the oracle has no warm-up state; each step is timed from cold
    vals, secs = [], []
    tokens = max(2048, args.oracle_tokens // 4)
    s = None
    thr = 1
    for _ in range(args.steps):
        tf, dt, s, thr = time_oracle(w, tokens)
        vals.append(tf)
        secs.append(dt)
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(secs),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": {**workload_config(w), "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                         "sample": f"first {s.batch} documents ({s.total} tokens) per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
