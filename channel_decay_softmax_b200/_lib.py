"""ctypes binding of libwall.so: one Python function per C-ABI entry point,
same names, argument marshalling only (torch tensors in, device pointers
out).  Every computation runs in the library's CUDA kernels; there is no
fallback.  If the library or a CUDA device is missing, the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwall.so")

(WALL_OK, WALL_ERR_INVALID_ARG, WALL_ERR_UNSUPPORTED, WALL_ERR_CUDA, WALL_ERR_TIMEOUT,
 WALL_ERR_RANGE) = range(6)
WALL_BF16, WALL_FP32 = 0, 1

EXPORTS = ["wall_version", "wall_error_string", "wall_prefix_cumsum", "wall_attn_fwd_workspace",
           "wall_attn_fwd", "wall_attn_bwd_workspace", "wall_attn_bwd", "wall_build_kv_cache",
           "wall_attn_decode_workspace", "wall_attn_decode", "wall_get_status",
           "wall_selftest_wait_timeout", "wall_attn_decode_noalloc", "wall_timing_enable",
           "wall_timing_read", "wall_decode_step_workspace", "wall_decode_step",
           "wall_attn_decode_chunk_workspace", "wall_attn_decode_chunk",
           "wall_attn_fwd_gate_workspace", "wall_attn_fwd_gate", "wall_timing_enable_slots",
           "wall_attn_bwd_workspace_min"]

_lib = None


class WallError(RuntimeError):
    def __init__(self, call: str, code: int):
        msg = lib().wall_error_string(code).decode() if _lib is not None else str(code)
        super().__init__(f"{call} failed: {msg} (status {code})")
        self.code = code


def lib():
    """Loads libwall.so (built by ``python -m channel_decay_softmax_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m channel_decay_softmax_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, fp, ip, i, f, sz = (ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                ctypes.c_float, ctypes.c_size_t)
        L.wall_version.restype = i
        L.wall_error_string.restype = ctypes.c_char_p
        L.wall_error_string.argtypes = [i]
        L.wall_prefix_cumsum.restype = i
        L.wall_prefix_cumsum.argtypes = [vp, i, fp, i, i, i, i, ip, i, fp, fp, vp]
        L.wall_attn_fwd_workspace.restype = sz
        L.wall_attn_fwd_workspace.argtypes = [i, i, i, i, i, i, i, i, i]
        L.wall_attn_fwd.restype = i
        L.wall_attn_fwd.argtypes = [vp, vp, vp, fp, i, i, i, i, i, i, i, f, fp, fp, i, ip, i, vp,
                                    fp, vp, sz, vp]
        L.wall_attn_bwd_workspace.restype = sz
        L.wall_attn_bwd_workspace.argtypes = [i, i, i, i, i, i, i, i, i, i]
        L.wall_attn_bwd_workspace_min.restype = sz
        L.wall_attn_bwd_workspace_min.argtypes = [i, i, i, i, i, i, i, i, i]
        L.wall_attn_bwd.restype = i
        L.wall_attn_bwd.argtypes = [vp, vp, vp, vp, fp, vp, fp, i, i, i, i, i, i, i, f, fp, fp,
                                    i, ip, i, vp, vp, vp, vp, fp, fp, vp, sz, vp, vp]
        L.wall_build_kv_cache.restype = i
        L.wall_build_kv_cache.argtypes = [vp, fp, i, i, i, i, i, i, i, i, vp, fp, i, vp]
        L.wall_attn_decode_workspace.restype = sz
        L.wall_attn_decode_workspace.argtypes = [i, i, i, i, i, i]
        L.wall_attn_decode.restype = i
        L.wall_attn_decode.argtypes = [vp, vp, fp, vp, fp, fp, f, i, i, i, i, i, i, i, i, i, vp,
                                       fp, vp, sz, vp]
        L.wall_get_status.restype = i
        L.wall_get_status.argtypes = [vp]
        L.wall_selftest_wait_timeout.restype = i
        L.wall_selftest_wait_timeout.argtypes = [i, vp]
        L.wall_attn_decode_noalloc.restype = i
        L.wall_attn_decode_noalloc.argtypes = [vp, vp, fp, vp, fp, fp, f, i, i, i, i, i, i, i, i,
                                               i, vp, fp, vp]
        L.wall_timing_enable.restype = i
        L.wall_timing_enable.argtypes = [i]
        L.wall_timing_enable_slots.restype = i
        L.wall_timing_enable_slots.argtypes = [ctypes.c_uint]
        L.wall_timing_read.restype = i
        L.wall_timing_read.argtypes = [i, ctypes.POINTER(ctypes.c_char_p),
                                       ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double)]
        L.wall_decode_step_workspace.restype = sz
        L.wall_decode_step_workspace.argtypes = [i, i, i, i, i, i]
        L.wall_decode_step.restype = i
        L.wall_decode_step.argtypes = [vp, vp, vp, vp, i, fp, vp, vp, fp, fp, f, i, i, i, i, i,
                                       i, i, i, vp, fp, vp, sz, vp]
        L.wall_attn_fwd_gate_workspace.restype = sz
        L.wall_attn_fwd_gate_workspace.argtypes = [i, i, i, i, i, i, i, i, i]
        L.wall_attn_fwd_gate.restype = i
        L.wall_attn_fwd_gate.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, f, fp, fp, i, ip,
                                         i, fp, vp, fp, vp, sz, vp]
        L.wall_attn_decode_chunk_workspace.restype = sz
        L.wall_attn_decode_chunk_workspace.argtypes = [i, i, i, i, i, i, i, i, i]
        L.wall_attn_decode_chunk.restype = i
        L.wall_attn_decode_chunk.argtypes = [vp, vp, fp, vp, fp, fp, f, i, i, i, i, i, i, i, i,
                                             i, i, vp, fp, vp, sz, vp]
        _lib = L
    return _lib


def _check(name, code):
    if code != WALL_OK:
        raise WallError(name, code)


def dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return WALL_BF16
    if t == torch.float32:
        return WALL_FP32
    raise TypeError(f"unsupported dtype {t}; use bfloat16 or float32")


def _p(t):
    """Device pointer of a tensor (None -> NULL); requires contiguous CUDA memory."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libwall takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libwall takes contiguous tensors")
    return t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


# ---------------------------------------------------------------------------
# one wrapper per entry point (argument order of include/wall.h)

def wall_version() -> int:
    return lib().wall_version()


def wall_get_status(stream=None) -> int:
    return lib().wall_get_status(_stream(stream))


def wall_selftest_wait_timeout(limit_us: int, stream=None):
    _check("wall_selftest_wait_timeout", lib().wall_selftest_wait_timeout(int(limit_us),
                                                                          _stream(stream)))


def wall_prefix_cumsum(g, P, B, T, HQ, K, cu_seqlens=None, n_seq=0, carry_in=None,
                       carry_out=None, stream=None):
    _check("wall_prefix_cumsum", lib().wall_prefix_cumsum(
        _p(g), dtype_code(g.dtype), _p(P), B, T, HQ, K, _p(cu_seqlens), n_seq, _p(carry_in),
        _p(carry_out), _stream(stream)))


def wall_attn_fwd_workspace(dtype, B, T, H, HQ, K, V, has_g_scalar, n_seq=0) -> int:
    return lib().wall_attn_fwd_workspace(dtype_code(dtype), B, T, H, HQ, K, V,
                                         int(bool(has_g_scalar)), n_seq)


def wall_attn_fwd(q, k, v, P, B, T, H, HQ, K, V, scale, g_scalar, sink_bias, window_size,
                  cu_seqlens, n_seq, o, lse, workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("wall_attn_fwd", lib().wall_attn_fwd(
        _p(q), _p(k), _p(v), _p(P), dtype_code(q.dtype), B, T, H, HQ, K, V, float(scale),
        _p(g_scalar), _p(sink_bias), int(window_size), _p(cu_seqlens), n_seq, _p(o), _p(lse),
        _p(workspace), ws_bytes, _stream(stream)))


def wall_attn_bwd_workspace(dtype, B, T, H, HQ, K, V, has_g_scalar, n_seq=0,
                            window_size=0) -> int:
    return lib().wall_attn_bwd_workspace(dtype_code(dtype), B, T, H, HQ, K, V,
                                         int(bool(has_g_scalar)), n_seq, int(window_size or 0))


def wall_attn_bwd_workspace_min(dtype, B, T, H, HQ, K, V, has_g_scalar, n_seq=0) -> int:
    return lib().wall_attn_bwd_workspace_min(dtype_code(dtype), B, T, H, HQ, K, V,
                                             int(bool(has_g_scalar)), n_seq)


def wall_attn_bwd(dO, q, k, v, P, o, lse, B, T, H, HQ, K, V, scale, g_scalar, sink_bias,
                  window_size, cu_seqlens, n_seq, dq, dk, dv, dg, dg_scalar, dsink, workspace,
                  fwd_workspace=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("wall_attn_bwd", lib().wall_attn_bwd(
        _p(dO), _p(q), _p(k), _p(v), _p(P), _p(o), _p(lse), dtype_code(q.dtype), B, T, H, HQ, K,
        V, float(scale), _p(g_scalar), _p(sink_bias), int(window_size), _p(cu_seqlens), n_seq,
        _p(dq), _p(dk), _p(dv), _p(dg), _p(dg_scalar), _p(dsink), _p(workspace), ws_bytes,
        _p(fwd_workspace), _stream(stream)))


def wall_build_kv_cache(k, P, B, Tn, H, HQ, K, C, t0, k_tilde, r_cache, Tcap, stream=None):
    _check("wall_build_kv_cache", lib().wall_build_kv_cache(
        _p(k), _p(P), dtype_code(k.dtype), B, Tn, H, HQ, K, C, t0, _p(k_tilde), _p(r_cache),
        Tcap, _stream(stream)))


def wall_attn_decode_workspace(B, T_kv, H, HQ, V, C) -> int:
    return lib().wall_attn_decode_workspace(B, T_kv, H, HQ, V, C)


def wall_attn_decode(q, v, p_curr, k_tilde, r_cache, sink_bias, scale, C, B, T_kv, Tcap, H, HQ,
                     K, V, o, lse, workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("wall_attn_decode", lib().wall_attn_decode(
        _p(q), _p(v), _p(p_curr), _p(k_tilde), _p(r_cache), _p(sink_bias), float(scale), C,
        dtype_code(q.dtype), B, T_kv, Tcap, H, HQ, K, V, _p(o), _p(lse), _p(workspace), ws_bytes,
        _stream(stream)))


def wall_attn_decode_noalloc(q, v, p_curr, k_tilde, r_cache, sink_bias, scale, C, B, T_kv, Tcap,
                             H, HQ, K, V, o, lse, stream=None):
    """wall_attn_decode without a workspace (fixed scratch inside the library)."""
    _check("wall_attn_decode_noalloc", lib().wall_attn_decode_noalloc(
        _p(q), _p(v), _p(p_curr), _p(k_tilde), _p(r_cache), _p(sink_bias), float(scale), C,
        dtype_code(q.dtype), B, T_kv, Tcap, H, HQ, K, V, _p(o), _p(lse), _stream(stream)))


def wall_decode_step_workspace(B, Tcap, H, HQ, V, C) -> int:
    return lib().wall_decode_step_workspace(B, Tcap, H, HQ, V, C)


def wall_decode_step(q, k, v, g, carry, k_tilde, v_cache, r_cache, sink_bias, scale, C, t, B,
                     Tcap, H, HQ, K, V, o, lse, workspace, stream=None):
    """One streaming token: prefix update, cache append and decode in one launch."""
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("wall_decode_step", lib().wall_decode_step(
        _p(q), _p(k), _p(v), _p(g), dtype_code(q.dtype), _p(carry), _p(k_tilde), _p(v_cache),
        _p(r_cache), _p(sink_bias), float(scale), C, t, B, Tcap, H, HQ, K, V, _p(o), _p(lse),
        _p(workspace), ws_bytes, _stream(stream)))


def wall_attn_decode_chunk_workspace(dtype, B, Tq, T_kv, H, HQ, K, V, C) -> int:
    return lib().wall_attn_decode_chunk_workspace(dtype, B, Tq, T_kv, H, HQ, K, V, C)


def wall_attn_decode_chunk(q, v, p, k_tilde, r_cache, sink_bias, scale, C, B, Tq, T_kv, Tcap, H,
                           HQ, K, V, o, lse, workspace, stream=None):
    """Tq queries per batch row at the last Tq cached positions, one call."""
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("wall_attn_decode_chunk", lib().wall_attn_decode_chunk(
        _p(q), _p(v), _p(p), _p(k_tilde), _p(r_cache), _p(sink_bias), float(scale), C,
        dtype_code(q.dtype), B, Tq, T_kv, Tcap, H, HQ, K, V, _p(o), _p(lse), _p(workspace),
        ws_bytes, _stream(stream)))


def wall_attn_fwd_gate_workspace(dtype, B, T, H, HQ, K, V, has_g_scalar, n_seq=0) -> int:
    return lib().wall_attn_fwd_gate_workspace(dtype_code(dtype), B, T, H, HQ, K, V,
                                              int(bool(has_g_scalar)), n_seq)


def wall_attn_fwd_gate(q, k, v, g, B, T, H, HQ, K, V, scale, g_scalar, sink_bias, window_size,
                       cu_seqlens, n_seq, P, o, lse, workspace, stream=None):
    """Prefix scan and forward in one call; P is written for the backward."""
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("wall_attn_fwd_gate", lib().wall_attn_fwd_gate(
        _p(q), _p(k), _p(v), _p(g), dtype_code(q.dtype), B, T, H, HQ, K, V, float(scale),
        _p(g_scalar), _p(sink_bias), int(window_size), _p(cu_seqlens), n_seq, _p(P), _p(o),
        _p(lse), _p(workspace), ws_bytes, _stream(stream)))
