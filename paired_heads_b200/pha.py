"""ctypes binding of libpha (include/pha.h). Argument marshalling only: every step runs in the
library's CUDA kernels. Importing this module loads libpha.so and raises if it is missing -- there
is no fallback.

Functions keep the C names. Tensor arguments may be torch tensors (their device pointer is
passed) or plain integers (raw device addresses). ``stream`` defaults to torch's current stream
on the tensors' device. A negative status raises :class:`PhaError`.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpha.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "pha.h")

PHA_BF16 = 0
PHA_F32 = 1
STATUS = {0: "PHA_OK", -1: "PHA_ERR_INVALID", -2: "PHA_ERR_UNSUPPORTED", -3: "PHA_ERR_WORKSPACE",
          -4: "PHA_ERR_CUDA"}
DEVICE_STATUS = {0: "ok", 1: "malformed cu_seqlens", 2: "work list overflow", 3: "wait timeout"}


class PhaError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn}: {STATUS.get(code, code)} ({msg})")
        self.code = code


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libpha.so is not built ({LIB_PATH}); run `python -m paired_heads_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)
_p = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t

_lib.pha_status_string.argtypes = [_i]
_lib.pha_status_string.restype = ctypes.c_char_p
_lib.pha_rope_tables.argtypes = [_p, _p, _i, _i, _i, ctypes.c_double, _p]
_lib.pha_rope.argtypes = [_p, _p, _p, _p, _i, _i, _p, _i, _i, _i, _i, _i, _i, _i, _p]
_lib.pha_attn_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
_lib.pha_attn_workspace_bytes.restype = _sz
_lib.pha_attn_fwd.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                              ctypes.c_float, _p, _p, _p, _sz, _p]
_lib.pha_attn_status.argtypes = [_p, ctypes.POINTER(_i), ctypes.POINTER(_i), _p]
_lib.pha_attn_fwd_noalloc.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                      ctypes.c_float, _p, _p, _p]
_lib.pha_attn_fwd_fp8.argtypes = [_p, _p, _p, ctypes.c_float, ctypes.c_float, ctypes.c_float, _p,
                                  _i, _i, _i, _i, _i, _i, _i, _i, _i, ctypes.c_float, _p, _p, _p,
                                  _sz, _p]
_lib.pha_test_attn_fwd_stalled.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                           _i, ctypes.c_float, _p, _p, _p, _sz, _i, _p]
_lib.pha_attn_fwd_aux_v.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                    ctypes.c_float, _p, _p, _p, _sz, _p]
_lib.pha_rope_bwd.argtypes = [_p, _p, _p, _p, _i, _i, _p, _i, _i, _i, _i, _i, _i, _i, _p]
_lib.pha_attn_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i]
_lib.pha_attn_bwd_workspace_bytes.restype = _sz
_lib.pha_attn_bwd.argtypes = [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                              _i, ctypes.c_float, _p, _p, _p, _p, _sz, _p]
_lib.pha_qk_norm_rope.argtypes = [_p, _p, _p, _p, ctypes.c_float, _p, _p, _i, _i, _p, _i, _i, _i,
                                  _i, _i, _i, _i, _p]
_lib.pha_rope_factor_bytes.argtypes = [_i, _i, _i]
_lib.pha_rope_factor_bytes.restype = _sz
_lib.pha_rope_factor_tables.argtypes = [_p, _sz, _i, _i, _i, ctypes.c_double, _p]
_lib.pha_rope_factored.argtypes = [_p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i, _i, _p]
_lib.pha_rope_bwd_factored.argtypes = [_p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i, _i, _p]
_lib.pha_qk_norm_rope_factored.argtypes = [_p, _p, _p, _p, ctypes.c_float, _p, _i, _p, _i, _i, _i,
                                           _i, _i, _i, _i, _p]
for _f in ("pha_rope_tables", "pha_rope", "pha_attn_fwd", "pha_attn_status",
           "pha_attn_fwd_noalloc", "pha_test_attn_fwd_stalled", "pha_attn_fwd_fp8", "pha_qk_norm_rope", "pha_attn_fwd_aux_v", "pha_rope_bwd",
           "pha_attn_bwd", "pha_rope_factor_tables", "pha_rope_factored", "pha_rope_bwd_factored",
           "pha_qk_norm_rope_factored"):
    getattr(_lib, _f).restype = _i


def exported_symbols() -> list:
    """Names of the functions include/pha.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(pha_\w+)\s*\(", text, re.M)))


def library():
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream, *tensors):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch

    for t in tensors:
        if t is not None and not isinstance(t, int) and t.is_cuda:
            return torch.cuda.current_stream(t.device).cuda_stream
    return torch.cuda.current_stream().cuda_stream


def _check(fn: str, rc: int):
    if rc != 0:
        raise PhaError(fn, rc, _lib.pha_status_string(rc).decode())


def _dtype_code(t) -> int:
    import torch

    if t.dtype == torch.bfloat16:
        return PHA_BF16
    if t.dtype == torch.float32:
        return PHA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def pha_status_string(code: int) -> str:
    return _lib.pha_status_string(code).decode()


def pha_rope_tables(cos_tab, sin_tab, rows: int, head_dim: int, paired: bool, base: float = 10000.0,
                    stream=None):
    _check("pha_rope_tables", _lib.pha_rope_tables(_ptr(cos_tab), _ptr(sin_tab), rows, head_dim,
                                                   int(paired), float(base),
                                                   _stream(stream, cos_tab)))


def pha_rope(q, k, cos_tab, sin_tab, positions, paired: bool = False, stagger_offset: int = 0,
             stream=None, *, tab_rows=None, tab_width=None, total_tokens=None, n_heads=None,
             n_kv_heads=None, head_dim=None, dtype=None):
    """In-place RoPE of q [T][H][hd] and k [T][Hkv][hd]. Shapes are taken from the tensors unless
    given explicitly (needed when raw addresses are passed)."""
    if total_tokens is None:
        total_tokens, n_heads, head_dim = q.shape
        n_kv_heads = 0 if k is None else k.shape[1]
        tab_rows, tab_width = cos_tab.shape
        dtype = _dtype_code(q)
    _check("pha_rope", _lib.pha_rope(_ptr(q), _ptr(k), _ptr(cos_tab), _ptr(sin_tab), tab_rows,
                                     tab_width, _ptr(positions), total_tokens, n_heads, n_kv_heads,
                                     head_dim, dtype, int(paired), stagger_offset,
                                     _stream(stream, q)))


def pha_qk_norm_rope(q, k, cos_tab, sin_tab, positions, q_weight=None, k_weight=None,
                     eps: float = 1e-6, paired: bool = False, stagger_offset: int = 0, stream=None,
                     *, tab_rows=None, tab_width=None, total_tokens=None, n_heads=None,
                     n_kv_heads=None, head_dim=None, dtype=None):
    """In-place QK RMS-norm (per head row, optional float32 weights of length head_dim) followed
    by RoPE of q [T][H][hd] and k [T][Hkv][hd]."""
    if total_tokens is None:
        total_tokens, n_heads, head_dim = q.shape
        n_kv_heads = 0 if k is None else k.shape[1]
        tab_rows, tab_width = cos_tab.shape
        dtype = _dtype_code(q)
    _check("pha_qk_norm_rope",
           _lib.pha_qk_norm_rope(_ptr(q), _ptr(k), _ptr(q_weight), _ptr(k_weight), float(eps),
                                 _ptr(cos_tab), _ptr(sin_tab), tab_rows, tab_width, _ptr(positions),
                                 total_tokens, n_heads, n_kv_heads, head_dim, dtype, int(paired),
                                 stagger_offset, _stream(stream, q)))


def pha_rope_bwd(dq, dk, cos_tab, sin_tab, positions, paired: bool = False, stagger_offset: int = 0,
                 stream=None, *, tab_rows=None, tab_width=None, total_tokens=None, n_heads=None,
                 n_kv_heads=None, head_dim=None, dtype=None):
    """In place: gradients with respect to the rotated q, k -> with respect to the unrotated ones."""
    if total_tokens is None:
        total_tokens, n_heads, head_dim = dq.shape
        n_kv_heads = 0 if dk is None else dk.shape[1]
        tab_rows, tab_width = cos_tab.shape
        dtype = _dtype_code(dq)
    _check("pha_rope_bwd", _lib.pha_rope_bwd(_ptr(dq), _ptr(dk), _ptr(cos_tab), _ptr(sin_tab),
                                             tab_rows, tab_width, _ptr(positions), total_tokens,
                                             n_heads, n_kv_heads, head_dim, dtype, int(paired),
                                             stagger_offset, _stream(stream, dq)))


def pha_rope_factor_bytes(rows: int, head_dim: int, paired: bool) -> int:
    return int(_lib.pha_rope_factor_bytes(rows, head_dim, int(paired)))


def pha_rope_factor_tables(factors, rows: int, head_dim: int, paired: bool,
                           base: float = 10000.0, stream=None, *, nbytes=None):
    """Factored rotary tables for table rows [0, rows) into the device buffer `factors`."""
    if nbytes is None:
        nbytes = factors.numel() * factors.element_size()
    _check("pha_rope_factor_tables",
           _lib.pha_rope_factor_tables(_ptr(factors), nbytes, rows, head_dim, int(paired),
                                       float(base), _stream(stream, factors)))


def _rope_shape(q, k):
    total_tokens, n_heads, head_dim = q.shape
    return total_tokens, n_heads, 0 if k is None else k.shape[1], head_dim, _dtype_code(q)


def pha_rope_factored(q, k, factors, rows: int, positions, paired: bool = False,
                      stagger_offset: int = 0, stream=None):
    """pha_rope with factored tables (pha_rope_factor_tables for `rows` rows)."""
    t, h, hkv, hd, dt = _rope_shape(q, k)
    _check("pha_rope_factored",
           _lib.pha_rope_factored(_ptr(q), _ptr(k), _ptr(factors), rows, _ptr(positions), t, h,
                                  hkv, hd, dt, int(paired), stagger_offset, _stream(stream, q)))


def pha_qk_norm_rope_factored(q, k, factors, rows: int, positions, q_weight=None, k_weight=None,
                              eps: float = 1e-6, paired: bool = False, stagger_offset: int = 0,
                              stream=None):
    """pha_qk_norm_rope with factored tables."""
    t, h, hkv, hd, dt = _rope_shape(q, k)
    _check("pha_qk_norm_rope_factored",
           _lib.pha_qk_norm_rope_factored(_ptr(q), _ptr(k), _ptr(q_weight), _ptr(k_weight),
                                          float(eps), _ptr(factors), rows, _ptr(positions), t, h,
                                          hkv, hd, dt, int(paired), stagger_offset,
                                          _stream(stream, q)))


def pha_rope_bwd_factored(dq, dk, factors, rows: int, positions, paired: bool = False,
                          stagger_offset: int = 0, stream=None):
    """pha_rope_bwd with factored tables."""
    t, h, hkv, hd, dt = _rope_shape(dq, dk)
    _check("pha_rope_bwd_factored",
           _lib.pha_rope_bwd_factored(_ptr(dq), _ptr(dk), _ptr(factors), rows, _ptr(positions), t,
                                      h, hkv, hd, dt, int(paired), stagger_offset,
                                      _stream(stream, dq)))


def pha_attn_bwd_workspace_bytes(batch: int, max_len: int, total_tokens: int, n_heads: int,
                                 head_dim: int, paired: bool) -> int:
    return int(_lib.pha_attn_bwd_workspace_bytes(batch, max_len, total_tokens, n_heads, head_dim,
                                                 int(paired)))


def pha_attn_bwd(q, k, v, o, lse, dout, cu_seqlens, max_len: int, dq, dk, dv, workspace, *,
                 causal: bool = True, window: int = 0, paired: bool = False, scale: float = 0.0,
                 stream=None, batch=None, total_tokens=None, n_heads=None, n_kv_heads=None,
                 head_dim=None, dtype=None, workspace_bytes=None):
    """Backward of pha_attn_fwd (o, lse: its outputs): writes dq, dk, dv for the upstream
    gradient dout."""
    if total_tokens is None:
        total_tokens, n_heads, head_dim = q.shape
        n_kv_heads = k.shape[1]
        batch = cu_seqlens.shape[0] - 1
        dtype = _dtype_code(q)
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pha_attn_bwd",
           _lib.pha_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                             _ptr(cu_seqlens), batch, max_len, total_tokens, n_heads, n_kv_heads,
                             head_dim, dtype, int(causal), int(window), int(paired), float(scale),
                             _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), workspace_bytes,
                             _stream(stream, q)))


def pha_attn_workspace_bytes(batch: int, max_len: int, n_heads: int, head_dim: int,
                             paired: bool) -> int:
    return int(_lib.pha_attn_workspace_bytes(batch, max_len, n_heads, head_dim, int(paired)))


def pha_attn_fwd(q, k, v, cu_seqlens, max_len: int, o, lse, workspace, *, causal: bool = True,
                 window: int = 0, paired: bool = False, scale: float = 0.0, stream=None,
                 batch=None, total_tokens=None, n_heads=None, n_kv_heads=None, head_dim=None,
                 dtype=None, workspace_bytes=None):
    """Varlen attention forward into o (like q) and lse [T][H] float32 (or None)."""
    if total_tokens is None:
        total_tokens, n_heads, head_dim = q.shape
        n_kv_heads = k.shape[1]
        batch = cu_seqlens.shape[0] - 1
        dtype = _dtype_code(q)
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pha_attn_fwd", _lib.pha_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), batch,
                                             max_len, total_tokens, n_heads, n_kv_heads, head_dim,
                                             dtype, int(causal), int(window), int(paired),
                                             float(scale), _ptr(o), _ptr(lse), _ptr(workspace),
                                             workspace_bytes, _stream(stream, q)))


def pha_attn_fwd_aux_v(q, k, v, aux_v, cu_seqlens, max_len: int, o, lse, workspace, *,
                       causal: bool = True, window: int = 0, paired: bool = False,
                       scale: float = 0.0, stream=None, batch=None, total_tokens=None,
                       n_heads=None, n_kv_heads=None, head_dim=None, dtype=None,
                       workspace_bytes=None):
    """Varlen attention forward over (q, k, v + aux_v) into o and lse (v, aux_v unchanged)."""
    if total_tokens is None:
        total_tokens, n_heads, head_dim = q.shape
        n_kv_heads = k.shape[1]
        batch = cu_seqlens.shape[0] - 1
        dtype = _dtype_code(q)
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pha_attn_fwd_aux_v",
           _lib.pha_attn_fwd_aux_v(_ptr(q), _ptr(k), _ptr(v), _ptr(aux_v), _ptr(cu_seqlens), batch,
                                   max_len, total_tokens, n_heads, n_kv_heads, head_dim, dtype,
                                   int(causal), int(window), int(paired), float(scale), _ptr(o),
                                   _ptr(lse), _ptr(workspace), workspace_bytes, _stream(stream, q)))


def pha_attn_fwd_noalloc(q, k, v, cu_seqlens, max_len: int, o, lse, *, causal: bool = True,
                         window: int = 0, paired: bool = False, scale: float = 0.0, stream=None,
                         batch=None, total_tokens=None, n_heads=None, n_kv_heads=None,
                         head_dim=None, dtype=None):
    """pha_attn_fwd with the library's built-in 1 MiB scratch instead of a workspace (for callers
    that cannot allocate device memory; calls that can overlap on the GPU must be ordered)."""
    if total_tokens is None:
        total_tokens, n_heads, head_dim = q.shape
        n_kv_heads = k.shape[1]
        batch = cu_seqlens.shape[0] - 1
        dtype = _dtype_code(q)
    _check("pha_attn_fwd_noalloc",
           _lib.pha_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), batch, max_len,
                                     total_tokens, n_heads, n_kv_heads, head_dim, dtype,
                                     int(causal), int(window), int(paired), float(scale), _ptr(o),
                                     _ptr(lse), _stream(stream, q)))


def pha_attn_fwd_fp8(q8, k8, v8, q_scale: float, k_scale: float, v_scale: float, cu_seqlens,
                     max_len: int, o, lse, workspace, *, causal: bool = True, window: int = 0,
                     paired: bool = False, scale: float = 0.0, stream=None):
    """Attention forward over e4m3 q8, k8, v8 (torch.float8_e4m3fn or uint8 tensors) with
    per-tensor scales, into o (bf16, q's shape) and lse [T][H] float32 (or None)."""
    total_tokens, n_heads, head_dim = q8.shape
    _check("pha_attn_fwd_fp8",
           _lib.pha_attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), float(q_scale), float(k_scale),
                                 float(v_scale), _ptr(cu_seqlens), cu_seqlens.shape[0] - 1,
                                 max_len, total_tokens, n_heads, k8.shape[1], head_dim,
                                 int(causal), int(window), int(paired), float(scale), _ptr(o),
                                 _ptr(lse), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream, q8)))


def pha_test_attn_fwd_stalled(q, k, v, cu_seqlens, max_len: int, o, lse, workspace, stall_us: int,
                              *, causal: bool = True, window: int = 0, paired: bool = False,
                              scale: float = 0.0, stream=None):
    """Failure-detection test hook: pha_attn_fwd whose band-kernel softmax first waits stall_us
    microseconds on a barrier nothing signals (device status 3 afterwards, no output written)."""
    total_tokens, n_heads, head_dim = q.shape
    _check("pha_test_attn_fwd_stalled",
           _lib.pha_test_attn_fwd_stalled(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens),
                                          cu_seqlens.shape[0] - 1, max_len, total_tokens, n_heads,
                                          k.shape[1], head_dim, _dtype_code(q), int(causal),
                                          int(window), int(paired), float(scale), _ptr(o),
                                          _ptr(lse), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(),
                                          int(stall_us), _stream(stream, q)))


def pha_attn_status(workspace, stream=None):
    """(device status, scheduled work items) recorded in the workspace; synchronises."""
    st, n = _i(0), _i(0)
    _check("pha_attn_status", _lib.pha_attn_status(_ptr(workspace), ctypes.byref(st),
                                                   ctypes.byref(n), _stream(stream, workspace)))
    return st.value, n.value
