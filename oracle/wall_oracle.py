"""fp64 CPU oracle for Wall Attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It shares no code with the CUDA path
(``channel_decay_softmax_b200``) and imports nothing from it.

The arithmetic lives in ``wall_oracle.c`` (plain C, fp64).  This wrapper only
marshals numpy arrays and does two plain steps in numpy that need no loops:
the GQA group sum of per-query-head key/value gradients, and the decode-cache
layout (``kv_cache``).

Pages followed (cited by page title and section):
  * Tilde blog "Wall Attention", "Definition: Wall Attention": the score
    sum_n (prod_{r=j+1..i} g_{r,n}) q_{i,n} k_{j,n}, softmax over j, times v_j,
    and the factorised form with P_t = sum_{u<=t} log g_u.
  * wall-attention-release README, "Usage": shapes q [B,T,HQ,K],
    k [B,T,H,K], v [B,T,H,V], g [B,T,HQ,K]; scale K**-0.5; optional
    g_scalar [B,T,HQ], sink_bias [HQ], window_size, cu_seqlens (B == 1).
  * README "Decode": P is the cumulative sum of g scaled by 1/ln 2;
    k_tilde[j] = k[j] * exp2(R_c - P[j]) with a per-chunk anchor R_c;
    r_cache [B, ceil(T_kv/C), HQ, K].

Readings where the pages are silent (each also recorded in the design notes):
``g`` is the natural-log gate; the product runs over r = j+1..i inclusive;
causal only; scale multiplies the decayed dot product and the g_scalar bias
is added unscaled; the sink is one extra logit with a zero value row; a key
is inside the window iff 0 <= i - j < window; query head h reads kv head
h // (HQ // H); R_c is P at the chunk's first row.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wall_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libwall_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_lp = ctypes.POINTER(ctypes.c_long)
_ip = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile the oracle's C source into ``oracle/libwall_oracle.so``."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.wo_forward.restype = ctypes.c_int
        lib.wo_forward.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_long, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                   ctypes.c_long, _lp, ctypes.c_int, ctypes.c_int, _ip,
                                   ctypes.c_int, ctypes.c_long, ctypes.c_long, ctypes.c_long,
                                   _dp, _dp, ctypes.c_int]
        lib.wo_backward.restype = ctypes.c_int
        lib.wo_backward.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_long,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_double, ctypes.c_long, _lp, ctypes.c_int,
                                    ctypes.c_int, _ip, ctypes.c_int, _dp, _dp, _dp, _dp, _dp,
                                    _dp, _dp, _dp, ctypes.c_int]
        lib.wo_prefix_log2.restype = ctypes.c_int
        lib.wo_prefix_log2.argtypes = [_dp, ctypes.c_long, ctypes.c_int, ctypes.c_int, _lp,
                                       ctypes.c_int, _dp, _dp]
        lib.wo_set_mutation.argtypes = [ctypes.c_int]
        lib.wo_get_mutation.restype = ctypes.c_int
        _lib = lib
    return _lib


def set_mutation(m: int) -> None:
    """Plant a deliberate mistake in the oracle (tests of the pins only)."""
    _load().wo_set_mutation(int(m))


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor -> numpy without importing torch here
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, ct=_dp):
    return None if a is None else a.ctypes.data_as(ct)


def _seqs(B, T, cu_seqlens):
    if cu_seqlens is None:
        return np.arange(B + 1, dtype=np.int64) * T
    if B != 1:
        raise ValueError("cu_seqlens requires B == 1")
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    if cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0, end at T and not decrease")
    return cu


def _units(units, nseq, HQ):
    if units is None:
        return None, 0
    u = np.ascontiguousarray(np.asarray(units, dtype=np.int32))
    if u.size and (u.min() < 0 or u.max() >= nseq * HQ):
        raise ValueError("unit out of range")
    return u, int(u.size)


def prefix_log2(g, cu_seqlens=None, carry_in=None):
    """P[b,t,h,n] = carry + sum_{u=s(t)..t} g[b,u,h,n] / ln 2 (inclusive, per
    sequence).  README "Decode": the prefix is the cumulative sum of g with
    scale 1/ln 2; Tilde blog: P_t = sum_{u<=t} log g_u."""
    g = _f64(g)
    B, T, HQ, K = g.shape
    cu = _seqs(B, T, cu_seqlens)
    nseq = len(cu) - 1
    c = _f64(carry_in)
    if c is not None:
        c = c.reshape(nseq, HQ, K)
    P = np.zeros_like(g)
    rc = _load().wo_prefix_log2(_ptr(g), B * T, HQ, K, _ptr(cu, _lp), nseq, _ptr(c), _ptr(P))
    if rc:
        raise ValueError("oracle prefix: bad arguments")
    return P


def forward(q, k, v, g, scale=None, g_scalar=None, sink_bias=None, window_size=0,
            cu_seqlens=None, form="product", units=None, rows=None, nthreads=None,
            q_rows_only=False):
    """Wall forward in fp64: returns (o [B,T,HQ,V], lse [B,T,HQ]).

    form="product" evaluates prod_{r=j+1..i} exp(g_r) directly (blog,
    "Definition: Wall Attention"); form="prefix" evaluates exp(L_i - L_j)
    with L the natural-log prefix (blog, factorised form).  ``units`` lists
    (sequence * HQ + head) pairs to compute and ``rows`` = (lo, hi) limits
    the rows (relative to each sequence start); entries not computed are NaN.
    With ``q_rows_only`` q holds only the queries of those rows,
    [B, hi - lo, HQ, K] (dense batches only).
    """
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    B, T, HQ, K = g.shape
    H, V = k.shape[2], v.shape[3]
    q_rows = 0
    if q_rows_only:
        if rows is None or cu_seqlens is not None:
            raise ValueError("q_rows_only needs rows=(lo, hi) and dense batches")
        q_rows = rows[1] - rows[0]
        if q.shape != (B, q_rows, HQ, K):
            raise ValueError("q must be [B, hi - lo, HQ, K]")
    if scale is None:
        scale = K ** -0.5
    cu = _seqs(B, T, cu_seqlens)
    nseq = len(cu) - 1
    gs, sk = _f64(g_scalar), _f64(sink_bias)
    u, nu = _units(units, nseq, HQ)
    lo, hi = (-1, -1) if rows is None else rows
    o = np.full((B, T, HQ, V), np.nan)
    lse = np.full((B, T, HQ), np.nan)
    rc = _load().wo_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(gs), _ptr(sk), B * T, H,
                            HQ, K, V, float(scale), int(window_size or 0), _ptr(cu, _lp), nseq,
                            0 if form == "product" else 1, _ptr(u, _ip), nu, int(lo), int(hi),
                            int(q_rows), _ptr(o), _ptr(lse), int(nthreads or default_threads()))
    if rc:
        raise ValueError("oracle forward: bad arguments")
    return o, lse


def backward(q, k, v, g, dO, scale=None, g_scalar=None, sink_bias=None, window_size=0,
             cu_seqlens=None, form="product", units=None, nthreads=None):
    """Analytic gradients of sum(o * dO), fp64.

    Returns a dict: o, lse, dq [B,T,HQ,K], dk_h [B,T,HQ,K] and dv_h
    [B,T,HQ,V] (per query head, before the GQA sum), dk [B,T,H,K] and
    dv [B,T,H,V] (group sums; NaN when a group is only partly computed),
    dg [B,T,HQ,K], dg_scalar [B,T,HQ] or None, dsink [HQ] or None.
    """
    q, k, v, g, dO = _f64(q), _f64(k), _f64(v), _f64(g), _f64(dO)
    B, T, HQ, K = q.shape
    H, V = k.shape[2], v.shape[3]
    G = HQ // H
    if scale is None:
        scale = K ** -0.5
    cu = _seqs(B, T, cu_seqlens)
    nseq = len(cu) - 1
    gs, sk = _f64(g_scalar), _f64(sink_bias)
    u, nu = _units(units, nseq, HQ)
    o = np.full((B, T, HQ, V), np.nan)
    lse = np.full((B, T, HQ), np.nan)
    dq = np.zeros((B, T, HQ, K))
    dkh = np.zeros((B, T, HQ, K))
    dvh = np.zeros((B, T, HQ, V))
    dg = np.full((B, T, HQ, K), np.nan)
    dgs = np.full((B, T, HQ), np.nan) if gs is not None else None
    dsk = np.full((nseq, HQ), np.nan) if sk is not None else None
    rc = _load().wo_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(gs), _ptr(sk), _ptr(dO),
                             B * T, H, HQ, K, V, float(scale), int(window_size or 0),
                             _ptr(cu, _lp), nseq, 0 if form == "product" else 1, _ptr(u, _ip),
                             nu, _ptr(o), _ptr(lse), _ptr(dq), _ptr(dkh), _ptr(dvh), _ptr(dg),
                             _ptr(dgs), _ptr(dsk), int(nthreads or default_threads()))
    if rc:
        raise ValueError("oracle backward: bad arguments")
    if u is not None:
        done = np.zeros((nseq, HQ), dtype=bool)
        done.reshape(-1)[u] = True
        # rows of heads that were not computed are unknown, not zero
        rows_seq = np.repeat(np.arange(nseq), np.diff(cu)).reshape(B, T) if nseq else None
        mask = done[rows_seq] if nseq else np.zeros((B, T, HQ), bool)
        for a in (dq, dkh):
            a[~mask] = np.nan
        dvh[~mask] = np.nan
    # GQA: query head h reads kv head h // G, so its key/value gradient
    # lands on that kv head (sum over the group).
    dk = dkh.reshape(B, T, H, G, K).sum(axis=3)
    dv = dvh.reshape(B, T, H, G, V).sum(axis=3)
    dsink = None if dsk is None else dsk.sum(axis=0)
    return dict(o=o, lse=lse, dq=dq, dk_h=dkh, dv_h=dvh, dk=dk, dv=dv, dg=dg,
                dg_scalar=dgs, dsink=dsink)


def kv_cache(k, g, chunk_size, HQ=None):
    """Pre-rescaled decode cache, fp64 (README "Decode").

    k_tilde[b,t,h,:] = k[b,t,h // G,:] * 2**(R_c - P[b,t,h,:]) for c = t // C,
    r_cache[b,c,h,:] = R_c, with P the base-2 prefix and R_c = P at the
    chunk's first row.  Shapes: k_tilde [B,T,HQ,K], r_cache [B,ceil(T/C),HQ,K].
    """
    k, g = _f64(k), _f64(g)
    B, T, H, K = k.shape
    HQ = g.shape[2]
    G = HQ // H
    C = int(chunk_size)
    P = prefix_log2(g)
    nc = -(-T // C)
    r_cache = P[:, ::C]                                  # rows c*C
    R = np.repeat(r_cache, C, axis=1)[:, :T]             # anchor of each row
    k_exp = np.repeat(k, G, axis=2)                      # kv head h // G
    k_tilde = k_exp * np.exp2(R - P)
    assert r_cache.shape == (B, nc, HQ, K)
    return k_tilde, r_cache
