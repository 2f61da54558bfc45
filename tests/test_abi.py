"""The C-ABI library loads, exports every entry point include/pha.h declares, and rejects bad
arguments before touching the GPU (these calls never reach a CUDA call, so they run on CPU)."""
import ctypes
import os
import re
import subprocess

import pytest

from paired_heads_b200 import build as pha_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pha():
    pha_build.build()
    from paired_heads_b200 import pha as mod

    return mod


def _declared():
    text = open(os.path.join(ROOT, "include", "pha.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pha_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    assert _declared() == ["pha_attn_bwd", "pha_attn_bwd_workspace_bytes", "pha_attn_fwd",
                           "pha_attn_fwd_aux_v", "pha_attn_fwd_fp8", "pha_attn_fwd_noalloc",
                           "pha_attn_status",
                           "pha_attn_workspace_bytes", "pha_qk_norm_rope",
                           "pha_qk_norm_rope_factored", "pha_rope", "pha_rope_bwd",
                           "pha_rope_bwd_factored", "pha_rope_factor_bytes",
                           "pha_rope_factor_tables", "pha_rope_factored", "pha_rope_tables",
                           "pha_status_string", "pha_test_attn_fwd_stalled"]


def test_library_exports_every_declared_symbol(pha):
    lib = ctypes.CDLL(pha.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", pha.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(_declared()) <= exported


def test_status_strings(pha):
    assert pha.pha_status_string(0) == "ok"
    assert pha.pha_status_string(-3).startswith("workspace")
    assert pha.pha_status_string(7) == "unknown status"


def test_workspace_bytes_closed_form(pha):
    # 256-byte header + int32[batch+1] padded to 16 bytes + 16 bytes per (block of 256 query
    # slots, head) work item
    def pad(n):
        return (4 * (n + 1) + 15) // 16 * 16
    assert pha.pha_attn_workspace_bytes(8, 1024, 12, 64, False) == 256 + pad(8) + 16 * 8 * 4 * 12
    assert pha.pha_attn_workspace_bytes(113, 2048, 6, 128, True) == 256 + pad(113) + 16 * 113 * 16 * 3
    assert pha.pha_attn_workspace_bytes(1, 1, 2, 64, True) == 256 + pad(1) + 16 * 1 * 1 * 1
    assert pha.pha_attn_workspace_bytes(0, 10, 2, 64, False) == 0
    assert pha.pha_attn_workspace_bytes(1, 10, 3, 64, True) == 0   # odd heads cannot pair


A = 0x10000          # an aligned fake device address (never dereferenced: calls fail first)
MIS = 0x10004        # misaligned


def _attn(pha, **kw):
    args = dict(q=A, k=A, v=A, cu=A, batch=1, max_len=128, total=128, H=4, Hkv=4, hd=64,
                dtype=pha.PHA_BF16, causal=1, window=0, paired=0, scale=0.0, o=A, lse=A, ws=A,
                ws_bytes=1 << 20)
    args.update(kw)
    lib = pha.library()
    return lib.pha_attn_fwd(args["q"], args["k"], args["v"], args["cu"], args["batch"],
                            args["max_len"], args["total"], args["H"], args["Hkv"], args["hd"],
                            args["dtype"], args["causal"], args["window"], args["paired"],
                            ctypes.c_float(args["scale"]), args["o"], args["lse"], args["ws"],
                            args["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(H=6, Hkv=4), -1),                    # heads not a multiple of kv heads
    (dict(H=6, Hkv=6, paired=1), 0),           # (valid shape; see below)
    (dict(H=6, Hkv=3, paired=1), -1),          # odd kv heads cannot pair
    (dict(H=5, Hkv=5, paired=1), -1),          # odd heads cannot pair
    (dict(causal=0, window=16), -2),           # windowed non-causal attention
    (dict(hd=96), -2),                         # bf16 tensor-core path: head_dim 64 / 128 only
    (dict(dtype=1, hd=160), -2),               # f32 path: head_dim <= 128
    (dict(q=MIS), -1),
    (dict(o=MIS), -1),
    (dict(lse=A + 2), -1),
    (dict(q=None), -1),
    (dict(batch=0), -1),
    (dict(total=-1), -1),
    (dict(dtype=7), -1),
    (dict(ws=None), -3),
    (dict(ws_bytes=100), -3),
    (dict(ws=MIS), -3),
])
def test_attn_argument_errors(pha, kw, code):
    if code == 0:
        # a valid problem would launch; only check that the workspace bound is what gates it
        assert _attn(pha, ws_bytes=10, **kw) == -3
        return
    assert _attn(pha, **kw) == code


def _stalled(pha, stall_us, **kw):
    args = dict(q=A, k=A, v=A, cu=A, batch=1, max_len=128, total=128, H=4, Hkv=4, hd=64,
                dtype=pha.PHA_BF16, causal=1, window=128, paired=0, scale=0.0, o=A, lse=A, ws=A,
                ws_bytes=10)
    args.update(kw)
    return pha.library().pha_test_attn_fwd_stalled(
        args["q"], args["k"], args["v"], args["cu"], args["batch"], args["max_len"], args["total"],
        args["H"], args["Hkv"], args["hd"], args["dtype"], args["causal"], args["window"],
        args["paired"], ctypes.c_float(args["scale"]), args["o"], args["lse"], args["ws"],
        args["ws_bytes"], stall_us, None)


@pytest.mark.parametrize("stall_us,kw,code", [
    (0, {}, -1),                               # the hook needs a stall
    (-5, {}, -1),
    (100001, {}, -1),
    (1000, dict(window=0), -2),                # only the band kernel has the hook
    (1000, dict(window=256), -2),
    (1000, dict(dtype=1, hd=16), -2),
    (1000, {}, -3),                            # otherwise the checks of pha_attn_fwd apply
])
def test_stall_hook_argument_errors(pha, stall_us, kw, code):
    assert _stalled(pha, stall_us, **kw) == code


def _fp8(pha, **kw):
    args = dict(q=A, k=A, v=A, sq=1.0, sk=1.0, sv=1.0, cu=A, batch=1, max_len=128, total=128, H=4,
                Hkv=4, hd=64, causal=1, window=0, paired=0, scale=0.0, o=A, lse=A, ws=A,
                ws_bytes=1 << 20)
    args.update(kw)
    f = ctypes.c_float
    return pha.library().pha_attn_fwd_fp8(
        args["q"], args["k"], args["v"], f(args["sq"]), f(args["sk"]), f(args["sv"]), args["cu"],
        args["batch"], args["max_len"], args["total"], args["H"], args["Hkv"], args["hd"],
        args["causal"], args["window"], args["paired"], f(args["scale"]), args["o"], args["lse"],
        args["ws"], args["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(sq=0.0), -1),                        # scales must be positive and finite
    (dict(sk=-1.0), -1),
    (dict(sv=float("inf")), -1),
    (dict(sq=float("nan")), -1),
    (dict(H=6, Hkv=4), -1),
    (dict(H=5, Hkv=5, paired=1), -1),
    (dict(causal=0, window=16), -2),
    (dict(hd=96), -2),                         # head_dim 64 / 128 only
    (dict(q=MIS), -1),
    (dict(v=None), -1),
    (dict(ws=None), -3),
    (dict(ws_bytes=100), -3),
])
def test_fp8_argument_errors(pha, kw, code):
    assert _fp8(pha, **kw) == code


def _rope(pha, **kw):
    args = dict(q=A, k=A, cos=A, sin=A, rows=16, width=64, pos=A, total=4, H=2, Hkv=2, hd=64,
                dtype=pha.PHA_BF16, paired=0, stagger=0)
    args.update(kw)
    return pha.library().pha_rope(args["q"], args["k"], args["cos"], args["sin"], args["rows"],
                                  args["width"], args["pos"], args["total"], args["H"],
                                  args["Hkv"], args["hd"], args["dtype"], args["paired"],
                                  args["stagger"], None)


@pytest.mark.parametrize("kw", [
    dict(width=128),                           # standard table must be head_dim wide
    dict(stagger=64),                          # stagger only on the paired path
    dict(paired=1, width=64),                  # paired table must be 2*head_dim wide
    dict(paired=1, width=128, stagger=32),     # stagger offset 0 or head_dim
    dict(hd=40, width=40),                     # bf16 spans of 16 elements
    dict(dtype=1, hd=12, width=12),            # f32 spans of 8 elements
    dict(q=MIS),
    dict(cos=MIS),
    dict(k=None),
    dict(H=0),
    dict(total=-2),
])
def test_rope_argument_errors(pha, kw):
    assert _rope(pha, **kw) == -1


def test_rope_empty_is_a_no_op(pha):
    assert _rope(pha, total=0) == 0
    assert _rope(pha, total=0, paired=1, width=128, stagger=64) == 0


def test_rope_tables_argument_errors(pha):
    lib = pha.library()
    assert lib.pha_rope_tables(MIS, A, 4, 64, 0, ctypes.c_double(1e4), None) == -1
    assert lib.pha_rope_tables(A, A, 4, 63, 0, ctypes.c_double(1e4), None) == -1
    assert lib.pha_rope_tables(A, A, 4, 64, 0, ctypes.c_double(0.0), None) == -1
    assert lib.pha_rope_tables(A, A, -1, 64, 1, ctypes.c_double(1e4), None) == -1


def _norm_rope(pha, **kw):
    args = dict(q=A, k=A, qw=None, kw=None, eps=1e-6, cos=A, sin=A, rows=16, width=64, pos=A,
                total=4, H=2, Hkv=2, hd=64, dtype=pha.PHA_BF16, paired=0, stagger=0)
    args.update(kw)
    return pha.library().pha_qk_norm_rope(
        args["q"], args["k"], args["qw"], args["kw"], ctypes.c_float(args["eps"]), args["cos"],
        args["sin"], args["rows"], args["width"], args["pos"], args["total"], args["H"],
        args["Hkv"], args["hd"], args["dtype"], args["paired"], args["stagger"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(eps=-1.0), -1),                      # eps >= 0
    (dict(eps=float("inf")), -1),
    (dict(eps=float("nan")), -1),
    (dict(qw=MIS), -1),                        # weights 16-byte aligned
    (dict(kw=MIS), -1),
    (dict(width=128), -1),                     # table checks as pha_rope
    (dict(paired=1, width=128, stagger=32), -1),
    (dict(q=MIS), -1),
    (dict(hd=48, width=48), -2),               # 6 chunks per head row: not a divisor of 32
    (dict(dtype=1, hd=24, width=24), -2),
])
def test_norm_rope_argument_errors(pha, kw, code):
    assert _norm_rope(pha, **kw) == code


def test_norm_rope_empty_is_a_no_op(pha):
    assert _norm_rope(pha, total=0) == 0


def _attn_aux(pha, **kw):
    args = dict(q=A, k=A, v=A, aux=A, cu=A, batch=1, max_len=128, total=128, H=4, Hkv=4, hd=64,
                dtype=pha.PHA_BF16, causal=1, window=128, paired=0, scale=0.0, o=A, lse=A, ws=A,
                ws_bytes=10)
    args.update(kw)
    return pha.library().pha_attn_fwd_aux_v(
        args["q"], args["k"], args["v"], args["aux"], args["cu"], args["batch"], args["max_len"],
        args["total"], args["H"], args["Hkv"], args["hd"], args["dtype"], args["causal"],
        args["window"], args["paired"], ctypes.c_float(args["scale"]), args["o"], args["lse"],
        args["ws"], args["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(), -3),                              # valid: only the (too small) workspace stops it
    (dict(aux=None), -1),
    (dict(aux=MIS), -1),
    (dict(window=0), -3),                      # the block kernel has it too: valid
    (dict(window=129), -3),
    (dict(dtype=1), -2),
    (dict(hd=96), -2),
    (dict(H=6, Hkv=4), -1),
])
def test_attn_aux_v_argument_errors(pha, kw, code):
    assert _attn_aux(pha, **kw) == code


def _attn_bwd(pha, **kw):
    args = dict(q=A, k=A, v=A, o=A, lse=A, g=A, cu=A, batch=1, max_len=128, total=128, H=4, Hkv=4,
                hd=64, dtype=pha.PHA_BF16, causal=1, window=0, paired=0, scale=0.0, dq=A, dk=A,
                dv=A, ws=A, ws_bytes=10)
    args.update(kw)
    return pha.library().pha_attn_bwd(
        args["q"], args["k"], args["v"], args["o"], args["lse"], args["g"], args["cu"], args["batch"],
        args["max_len"], args["total"], args["H"], args["Hkv"], args["hd"], args["dtype"],
        args["causal"], args["window"], args["paired"], ctypes.c_float(args["scale"]), args["dq"],
        args["dk"], args["dv"], args["ws"], args["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(), -3),                              # valid: only the (too small) workspace stops it
    (dict(lse=None), -1),
    (dict(lse=A + 2), -1),
    (dict(o=None), -1),
    (dict(o=MIS), -1),
    (dict(g=None), -1),
    (dict(dk=MIS), -1),
    (dict(H=6, Hkv=4), -1),
    (dict(H=6, Hkv=3, paired=1), -1),
    (dict(causal=0, window=16), -2),
    (dict(hd=160), -2),
    (dict(dtype=7), -1),
    (dict(total=0, ws=None), 0),               # nothing to do
])
def test_attn_bwd_argument_errors(pha, kw, code):
    assert _attn_bwd(pha, **kw) == code


def test_attn_bwd_workspace_bytes(pha):
    def up(n):
        return (n + 255) // 256 * 256

    def pad(n):
        return (4 * (n + 1) + 15) // 16 * 16
    for batch, max_len, total, H, hd, paired in [(113, 2048, 65536, 6, 128, True),
                                                 (3, 700, 1000, 4, 64, False), (1, 0, 0, 2, 16, True)]:
        fwd = pha.pha_attn_workspace_bytes(batch, max_len, H, hd, paired)
        assert fwd > 0
        m = 2 if paired else 1
        tiles = -(-max_len * m // 128)                  # 128-slot tiles per document
        sched = 256 + pad(batch) + 16 * batch * tiles * (H // m)
        assert sched >= fwd                             # holds every work list of the forward
        assert pha.pha_attn_bwd_workspace_bytes(batch, max_len, total, H, hd, paired) == \
            up(sched) + up(total * H * 4)
    assert pha.pha_attn_bwd_workspace_bytes(1, 16, -1, 2, 16, False) == 0
    assert pha.pha_attn_bwd_workspace_bytes(0, 16, 16, 2, 16, False) == 0
    assert pha.pha_attn_bwd_workspace_bytes(1, 16, 16, 3, 16, True) == 0


def test_rope_bwd_argument_errors(pha):
    lib = pha.library()
    args = [A, A, A, A, 16, 64, A, 4, 2, 2, 64, pha.PHA_BF16, 0, 0, None]
    assert lib.pha_rope_bwd(*args[:5], 128, *args[6:]) == -1        # table width
    assert lib.pha_rope_bwd(MIS, *args[1:]) == -1
    assert lib.pha_rope_bwd(*args[:7], 0, *args[8:]) == 0           # no tokens


def test_rope_factor_bytes_closed_form(pha):
    # 16 fine rows of head_dim/2 (standard) or head_dim (paired) (cos, sin) float64 pairs, then
    # ceil(rows/16) coarse rows of head_dim/2 pairs
    for rows, hd, paired in [(0, 64, 0), (1, 64, 1), (16, 128, 0), (17, 128, 1), (131072, 128, 1)]:
        a = hd if paired else hd // 2
        assert pha.pha_rope_factor_bytes(rows, hd, paired) == (16 * a + -(-rows // 16) * (hd // 2)) * 16
    assert pha.pha_rope_factor_bytes(-1, 64, 0) == 0
    assert pha.pha_rope_factor_bytes(4, 63, 0) == 0
    assert pha.pha_rope_factor_bytes(4, 64, 2) == 0


def test_rope_factor_tables_argument_errors(pha):
    lib = pha.library()
    need = pha.pha_rope_factor_bytes(64, 64, 1)
    d = ctypes.c_double(1e4)
    assert lib.pha_rope_factor_tables(None, need, 64, 64, 1, d, None) == -1
    assert lib.pha_rope_factor_tables(MIS, need, 64, 64, 1, d, None) == -1
    assert lib.pha_rope_factor_tables(A, need - 16, 64, 64, 1, d, None) == -1   # too small
    assert lib.pha_rope_factor_tables(A, need, 64, 63, 1, d, None) == -1
    assert lib.pha_rope_factor_tables(A, need, 64, 64, 1, ctypes.c_double(-1.0), None) == -1
    assert lib.pha_rope_factor_tables(A, need, -1, 64, 1, d, None) == -1


def _rope_factored(pha, fn="pha_rope_factored", **kw):
    args = dict(q=A, k=A, fac=A, rows=16, pos=A, total=4, H=2, Hkv=2, hd=64,
                dtype=pha.PHA_BF16, paired=0, stagger=0)
    args.update(kw)
    tail = (args["fac"], args["rows"], args["pos"], args["total"], args["H"], args["Hkv"],
            args["hd"], args["dtype"], args["paired"], args["stagger"], None)
    lib = pha.library()
    if fn == "pha_qk_norm_rope_factored":
        return lib.pha_qk_norm_rope_factored(args["q"], args["k"], None, None, ctypes.c_float(1e-6),
                                             *tail)
    return getattr(lib, fn)(args["q"], args["k"], *tail)


@pytest.mark.parametrize("fn", ["pha_rope_factored", "pha_rope_bwd_factored",
                                "pha_qk_norm_rope_factored"])
@pytest.mark.parametrize("kw", [
    dict(stagger=64),                          # stagger only on the paired path
    dict(paired=1, stagger=32),                # stagger offset 0 or head_dim
    dict(hd=40),                               # bf16 spans of 16 elements
    dict(dtype=1, hd=12),                      # f32 spans of 8 elements
    dict(q=MIS),
    dict(fac=MIS),
    dict(fac=None),
    dict(k=None),
    dict(pos=None),
    dict(H=0),
    dict(rows=-1),
    dict(total=-2),
])
def test_rope_factored_argument_errors(pha, fn, kw):
    assert _rope_factored(pha, fn, **kw) == -1


@pytest.mark.parametrize("fn", ["pha_rope_factored", "pha_rope_bwd_factored",
                                "pha_qk_norm_rope_factored"])
def test_rope_factored_empty_is_a_no_op(pha, fn):
    assert _rope_factored(pha, fn, total=0) == 0
    assert _rope_factored(pha, fn, total=0, paired=1, stagger=64, q=None, k=None, fac=None,
                          pos=None) == 0


def test_norm_rope_factored_unsupported_head_dim(pha):
    # 6 chunks per head row: not a divisor of 32
    assert _rope_factored(pha, "pha_qk_norm_rope_factored", hd=48) == -2
