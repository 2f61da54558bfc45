"""float64 CPU oracle for RoPE and causal / windowed varlen attention (standard and paired-head).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its
``cpu_baseline`` leg and ``--impl reference``) may import this package. The product package
``paired_heads_b200`` never imports it, and it never imports the product package: the two share
no code. The arithmetic lives in ``oracle.c`` (plain C, float64, explicit loops); this module only
marshals numpy arrays into it.

Sources: the "modded-nanogpt Paired Head Attention record" page (sections "core idea",
"interleave semantics under the causal mask", "staggered rotary", "sequence length and window
handling", "4. interleave index in the Triton kernel"); the "Training an LLM from scratch (part
2)" page, sections "2. RoPE" and "4. GQA & FlashAttention"; the "ChatGPT" source notes, section
"SingleHeadAttention"; the "mHC module" page (max-subtracted softmax).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_c = ctypes.c_int
_l = ctypes.c_int64
_d = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP, no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_rope.argtypes = [_f64p, _i32p, _l, _c, _c, _c, _c, _d, _c]
        lib.oracle_round_bf16.argtypes = [_f64p, _l]
        lib.oracle_interleave.argtypes = [_f64p, _f64p, _l, _c, _c]
        lib.oracle_deinterleave.argtypes = [_f64p, _f64p, _l, _c, _c]
        lib.oracle_attention.argtypes = [_f64p, _f64p, _f64p, _i64p, _c, _c, _c, _c, _c, _c, _d,
                                         _f64p, _f64p]
        lib.oracle_attention_rows.argtypes = [_f64p, _f64p, _f64p, _i64p, _c, _c, _c, _c, _c, _c,
                                              _d, _i64p, _l, _f64p, _f64p]
        lib.oracle_attn_fwd.argtypes = [_f64p, _f64p, _f64p, _i32p, _c, _c, _c, _c, _c, _c, _c,
                                        _d, _f64p, _f64p]
        lib.oracle_rms_norm.argtypes = [_f64p, _l, _c, ctypes.c_void_p, _d]
        lib.oracle_attn_bwd.argtypes = [_f64p, _f64p, _f64p, _f64p, _i32p, _c, _c, _c, _c, _c, _c,
                                        _c, _d, _f64p, _f64p, _f64p]
        lib.oracle_rope_bwd.argtypes = [_f64p, _i32p, _l, _c, _c, _c, _c, _d, _c]
        lib.oracle_decode_e4m3.argtypes = [_u8p, _f64p, _l]
        lib.oracle_encode_e4m3.argtypes = [_f64p, _u8p, _l]
        lib.oracle_decode_e4m3.restype = ctypes.c_int
        lib.oracle_encode_e4m3.restype = ctypes.c_int
        lib.oracle_attn_bwd.restype = ctypes.c_int
        lib.oracle_rope_bwd.restype = ctypes.c_int
        for f in ("oracle_rms_norm", "oracle_rope", "oracle_round_bf16", "oracle_interleave", "oracle_deinterleave", "oracle_attention",
                  "oracle_attention_rows", "oracle_attn_fwd"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"{what}: oracle rejected the arguments (rc={rc})")


def rope(x, positions, paired: bool = False, stagger: bool = False, base: float = 10000.0,
         table_f32: bool = False):
    """Rotate x[T][H][hd] (returns a new float64 array). Phase of token t, head h is
    positions[t] (standard) or 2*positions[t] + (h % 2 if stagger) (paired). table_f32 rounds
    the cosines and sines to float32 first (the values a float32 rotary table holds)."""
    y = _f64(x).copy()
    T, H, hd = y.shape
    pos = np.ascontiguousarray(positions, dtype=np.int32)
    assert pos.shape == (T,)
    _check(_load().oracle_rope(y, pos, T, H, hd, int(paired), int(stagger), float(base),
                               int(table_f32)), "rope")
    return y


def round_bf16(x):
    """Nearest bfloat16 value of every element (ties to even), as float64 (new array)."""
    y = _f64(x).copy()
    _check(_load().oracle_round_bf16(y.reshape(-1), y.size), "round_bf16")
    return y


def rope_stored(x, positions, dtype: str, paired: bool = False, stagger: bool = False,
                base: float = 10000.0):
    """RoPE as the pipeline stores it: cosines and sines taken from float32 tables, rotation in
    float64, result rounded to the buffer's dtype ("bf16": nearest bfloat16; "f32": nearest
    float32)."""
    y = rope(x, positions, paired, stagger, base, table_f32=True)
    if dtype == "bf16":
        return round_bf16(y)
    return y.astype(np.float32).astype(np.float64)


def rms_norm(x, gamma=None, eps: float = 1e-6):
    """RMS normalisation over the last axis of x (returns a new float64 array); gamma: per-element
    weights of that axis, or None for ones ("Training an LLM from scratch (part 2)", section
    "1. RMSNorm")."""
    y = _f64(x).copy()
    d = y.shape[-1]
    g = None if gamma is None else _f64(gamma).reshape(d).copy()
    _check(_load().oracle_rms_norm(y.reshape(-1), y.size // d, d,
                                   None if g is None else g.ctypes.data, float(eps)), "rms_norm")
    return y


def norm_rope_stored(x, positions, dtype: str, paired: bool = False, stagger: bool = False,
                     base: float = 10000.0, gamma=None, eps: float = 1e-6, tab_rows=None):
    """QK RMS-norm of each head row, then RoPE with float32 table values, rounded once to the
    buffer's dtype. Tokens whose position lies outside [0, tab_rows) are normalised but not
    rotated."""
    n = rms_norm(x, gamma, eps)
    pos = np.ascontiguousarray(positions, dtype=np.int64)
    safe = np.clip(pos, 0, None).astype(np.int32)
    y = rope(n, safe, paired, stagger, base, table_f32=True)
    if tab_rows is not None:
        out = (pos < 0) | (pos >= tab_rows)
        y[out] = n[out]
    if dtype == "bf16":
        return round_bf16(y)
    return y.astype(np.float32).astype(np.float64)


def add_stored(v, aux, dtype: str):
    """v + aux (the value embedding added to v before attention: "modded-nanogpt Paired Head
    Attention record" page, section "3. the paired branch of the forward pass"), as the pipeline
    stores it in the buffer's dtype. Both operands are exact in float64, so the sum is exact and
    is rounded once."""
    y = _f64(v) + _f64(aux)
    if dtype == "bf16":
        return round_bf16(y)
    return y.astype(np.float32).astype(np.float64)


def interleave(x):
    """Explicit paired interleave [T][H][d] -> [2T][H/2][d] (copy loop in C)."""
    x = _f64(x)
    T, H, d = x.shape
    y = np.empty((2 * T, H // 2, d), dtype=np.float64)
    _check(_load().oracle_interleave(x, y, T, H, d), "interleave")
    return y


def deinterleave(y):
    """Inverse of :func:`interleave`: [2T][H/2][d] -> [T][H][d]."""
    y = _f64(y)
    S, Hp, d = y.shape
    x = np.empty((S // 2, 2 * Hp, d), dtype=np.float64)
    _check(_load().oracle_deinterleave(y, x, S // 2, 2 * Hp, d), "deinterleave")
    return x


def attention_slots(q, k, v, cu_slots, causal=True, window=0, scale=None):
    """Attention over slot-major buffers (no pairing): q[S][H][hd], k,v[S][Hkv][hd]; documents
    are the slot ranges of cu_slots. Returns (o[S][H][hd], lse[S][H])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    S, H, hd = q.shape
    Hkv = k.shape[1]
    cu = np.ascontiguousarray(cu_slots, dtype=np.int64)
    scale = 1.0 / np.sqrt(hd) if scale is None or scale <= 0 else float(scale)
    o = np.zeros_like(q)
    lse = np.zeros((S, H), dtype=np.float64)
    _check(_load().oracle_attention(q, k, v, cu, len(cu) - 1, H, Hkv, hd, int(causal),
                                    int(window), scale, o, lse), "attention")
    return o, lse


def attn_fwd(q, k, v, cu_seqlens, causal=True, window=0, paired=False, scale=None):
    """Full forward in token layout: q[T][H][hd], k,v[T][Hkv][hd], cu_seqlens in tokens.
    Paired: explicit interleave, doubled cu_seqlens, H/2 heads, window unchanged, de-interleave.
    Returns (o[T][H][hd], lse[T][H])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, H, hd = q.shape
    Hkv = k.shape[1]
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    scale = 1.0 / np.sqrt(hd) if scale is None or scale <= 0 else float(scale)
    o = np.zeros_like(q)
    lse = np.zeros((T, H), dtype=np.float64)
    _check(_load().oracle_attn_fwd(q, k, v, cu, len(cu) - 1, H, Hkv, hd, int(causal),
                                   int(window), int(paired), scale, o, lse), "attn_fwd")
    return o, lse


def decode_e4m3(codes):
    """float64 value of every e4m3 code (uint8 array of the same shape); see oracle.c."""
    b = np.ascontiguousarray(codes, dtype=np.uint8)
    y = np.empty(b.shape, dtype=np.float64)
    _check(_load().oracle_decode_e4m3(b.reshape(-1), y.reshape(-1), b.size), "decode_e4m3")
    return y


def encode_e4m3(x):
    """Nearest e4m3 code of every element (ties to even; NaN past 448), as uint8."""
    y = _f64(x)
    b = np.empty(y.shape, dtype=np.uint8)
    _check(_load().oracle_encode_e4m3(y.reshape(-1), b.reshape(-1), y.size), "encode_e4m3")
    return b


def attn_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, cu_seqlens, causal=True, window=0,
                 paired=False, scale=None):
    """Attention over FP8 inputs: q = q_scale * value(q8), k = k_scale * value(k8),
    v = v_scale * value(v8) (e4m3 codes, per-tensor float32 scales), then attn_fwd on those
    exact float64 values. Returns (o, lse) like attn_fwd; the softmax scale defaults to
    1/sqrt(head_dim)."""
    q = decode_e4m3(q8) * float(np.float32(q_scale))
    k = decode_e4m3(k8) * float(np.float32(k_scale))
    v = decode_e4m3(v8) * float(np.float32(v_scale))
    return attn_fwd(q, k, v, cu_seqlens, causal, window, paired, scale)


def attn_rows(q, k, v, cu_seqlens, rows, causal=True, window=0, paired=False, scale=None):
    """Selected output rows of :func:`attn_fwd`, computed one by one.

    ``rows`` index the caller's [T][H] row space as t*H + h. For the paired case the rows are
    computed on the interleaved sequence addressed as a view of the same buffers -- slot s, head
    h' lives at flat offset (s*(H/2) + h')*hd, the identity that the tests pin against the
    explicit interleave bit for bit -- so no 2T copies are made. Returns (o[n][hd], lse[n])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, H, hd = q.shape
    Hkv = k.shape[1]
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    scale = 1.0 / np.sqrt(hd) if scale is None or scale <= 0 else float(scale)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    if paired:
        # token t, head h  ->  slot 2t + h//(H/2), head h % (H/2)
        t, h = rows // H, rows % H
        Hp = H // 2
        slot_rows = (2 * t + h // Hp) * Hp + (h % Hp)
        qs = q.reshape(2 * T, Hp, hd)
        ks = k.reshape(2 * T, Hkv // 2, hd)
        vs = v.reshape(2 * T, Hkv // 2, hd)
        cu_s = np.ascontiguousarray(2 * cu)
        Hs, Hkvs = Hp, Hkv // 2
    else:
        slot_rows, qs, ks, vs, cu_s, Hs, Hkvs = rows, q, k, v, np.ascontiguousarray(cu), H, Hkv
    slot_rows = np.ascontiguousarray(slot_rows, dtype=np.int64)
    n = len(slot_rows)
    o = np.zeros((n, hd), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    _check(_load().oracle_attention_rows(np.ascontiguousarray(qs), np.ascontiguousarray(ks),
                                         np.ascontiguousarray(vs), cu_s, len(cu_s) - 1, Hs, Hkvs,
                                         hd, int(causal), int(window), scale, slot_rows, n, o,
                                         lse), "attn_rows")
    return o, lse


def attn_bwd(q, k, v, dout, cu_seqlens, causal=True, window=0, paired=False, scale=None):
    """Gradients (dq, dk, dv) of attn_fwd's O with respect to q, k, v for the upstream gradient
    dout (float64; token-major like attn_fwd). P is recomputed from q and k."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    T, H, hd = q.shape
    Hkv = k.shape[1]
    scale = 1.0 / np.sqrt(hd) if scale is None or scale <= 0 else float(scale)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    _check(_load().oracle_attn_bwd(q, k, v, dout, cu, len(cu) - 1, H, Hkv, hd, int(causal),
                                   int(window), int(paired), scale, dq, dk, dv), "attn_bwd")
    return dq, dk, dv


def rope_bwd(dy, positions, paired: bool = False, stagger: bool = False, base: float = 10000.0,
             table_f32: bool = False):
    """Gradient of rope() with respect to its input for the upstream gradient dy: the transposed
    rotation of every pair (returns a new float64 array)."""
    y = _f64(dy).copy()
    T, H, hd = y.shape
    pos = np.ascontiguousarray(positions, dtype=np.int32)
    _check(_load().oracle_rope_bwd(y, pos, T, H, hd, int(paired), int(stagger), float(base),
                                   int(table_f32)), "rope_bwd")
    return y
