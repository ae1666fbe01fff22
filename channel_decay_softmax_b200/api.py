"""User-facing Wall Attention API over the C ABI (wall-attention-release
README "Usage" and "Decode": wall_attn, build_wall_kv_cache,
wall_attn_decode, plus the prefix P = cumsum(g) / ln 2).

torch provides device memory, streams and autograd bookkeeping; every step
of the computation runs in libwall.so's CUDA kernels.
"""
from __future__ import annotations

import torch

from . import _lib as L


def _shape_checks(q, k, v, g):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4 or g.dim() != 4:
        raise ValueError("q, k, v, g must be [B, T, heads, dim]")
    B, T, HQ, K = q.shape
    if k.shape[:2] != (B, T) or v.shape[:2] != (B, T) or g.shape != q.shape:
        raise ValueError("q, k, v, g disagree on B, T (or g is not shaped like q)")
    H = k.shape[2]
    if v.shape[2] != H or k.shape[3] != K or HQ % H != 0:
        raise ValueError("need k [B,T,H,K], v [B,T,H,V] with HQ % H == 0")
    return B, T, H, HQ, K, v.shape[3]


def _n_seq(cu_seqlens, B):
    if cu_seqlens is None:
        return 0
    if B != 1:
        raise ValueError("cu_seqlens requires B == 1")
    if cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    return cu_seqlens.numel() - 1


def _ws(nbytes, device):
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def prefix_cumsum(g, cu_seqlens=None, carry_in=None, return_carry=False):
    """P = cumsum_t(g) / ln 2 per sequence (fp32), with an optional carried-in
    prefix [n_seq or B, HQ, K]; README "Decode" builds P this way."""
    g = g.contiguous()
    B, T, HQ, K = g.shape
    P = torch.empty(g.shape, dtype=torch.float32, device=g.device)
    nseq = _n_seq(cu_seqlens, B)
    ns = nseq if cu_seqlens is not None else B
    carry_out = torch.empty((ns, HQ, K), dtype=torch.float32, device=g.device) \
        if return_carry else None
    cin = carry_in.contiguous().float() if carry_in is not None else None
    L.wall_prefix_cumsum(g, P, B, T, HQ, K, cu_seqlens, nseq, cin, carry_out)
    return (P, carry_out) if return_carry else P


def wall_attn_fwd(q, k, v, P, scale=None, g_scalar=None, sink_bias=None, window_size=None,
                  cu_seqlens=None, return_workspace=False):
    """Forward from a precomputed prefix P; returns (o, lse), or (o, lse,
    workspace) with return_workspace: the workspace holds the anchored
    operands, which wall_attn_bwd can reuse (its fwd_workspace)."""
    B, T, H, HQ, K, V = _shape_checks(q, k, v, P)
    nseq = _n_seq(cu_seqlens, B)
    o = torch.empty((B, T, HQ, V), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, T, HQ), dtype=torch.float32, device=q.device)
    ws = _ws(L.wall_attn_fwd_workspace(q.dtype, B, T, H, HQ, K, V, g_scalar is not None, nseq),
             q.device)
    L.wall_attn_fwd(q, k, v, P, B, T, H, HQ, K, V, scale or 0.0, g_scalar, sink_bias,
                    window_size or 0, cu_seqlens, nseq, o, lse, ws)
    return (o, lse, ws) if return_workspace else (o, lse)


def wall_attn_fwd_gate(q, k, v, g, scale=None, g_scalar=None, sink_bias=None, window_size=None,
                       cu_seqlens=None, return_workspace=False):
    """Prefix scan and forward in one call, the prefix fused into the
    forward's operand pass; returns (o, lse, P), or (o, lse, P, workspace)
    with return_workspace (the workspace serves wall_attn_bwd as its
    fwd_workspace).  P and o are bit for bit those of prefix_cumsum followed
    by wall_attn_fwd."""
    g = g.contiguous()
    B, T, H, HQ, K, V = _shape_checks(q, k, v, g)
    nseq = _n_seq(cu_seqlens, B)
    o = torch.empty((B, T, HQ, V), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, T, HQ), dtype=torch.float32, device=q.device)
    P = torch.empty((B, T, HQ, K), dtype=torch.float32, device=q.device)
    ws = _ws(L.wall_attn_fwd_gate_workspace(q.dtype, B, T, H, HQ, K, V, g_scalar is not None,
                                            nseq), q.device)
    L.wall_attn_fwd_gate(q, k, v, g, B, T, H, HQ, K, V, scale or 0.0, g_scalar, sink_bias,
                         window_size or 0, cu_seqlens, nseq, P, o, lse, ws)
    return (o, lse, P, ws) if return_workspace else (o, lse, P)


def wall_attn_bwd(dO, q, k, v, P, o, lse, scale=None, g_scalar=None, sink_bias=None,
                  window_size=None, cu_seqlens=None, want_dsink=False, fwd_workspace=None):
    """Backward; returns dq, dk, dv, dg, dg_scalar (or None), dsink (or None).
    fwd_workspace: the workspace returned by wall_attn_fwd(..., return_workspace=True)
    for the same inputs, whose anchored operands are then reused."""
    B, T, H, HQ, K, V = _shape_checks(q, k, v, P)
    nseq = _n_seq(cu_seqlens, B)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    dg = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    dgs = torch.empty_like(g_scalar) if g_scalar is not None else None
    dsink = torch.empty((HQ,), dtype=torch.float32, device=q.device) \
        if (want_dsink and sink_bias is not None) else None
    ws = _ws(L.wall_attn_bwd_workspace(q.dtype, B, T, H, HQ, K, V, g_scalar is not None, nseq),
             q.device)
    L.wall_attn_bwd(dO.contiguous(), q, k, v, P, o, lse, B, T, H, HQ, K, V, scale or 0.0,
                    g_scalar, sink_bias, window_size or 0, cu_seqlens, nseq, dq, dk, dv, dg, dgs,
                    dsink, ws, fwd_workspace)
    return dq, dk, dv, dg, dgs, dsink


class WallAttnFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, g, scale, g_scalar, sink_bias, window_size, cu_seqlens):
        q, k, v, g = (t.contiguous() for t in (q, k, v, g))
        if g.dtype != q.dtype or k.dtype != q.dtype or v.dtype != q.dtype:
            raise TypeError("q, k, v and g must share one dtype")
        gs = g_scalar.contiguous().float() if g_scalar is not None else None
        sk = sink_bias.contiguous().float() if sink_bias is not None else None
        o, lse, P, fws = wall_attn_fwd_gate(q, k, v, g, scale, gs, sk, window_size, cu_seqlens,
                                            return_workspace=True)
        ctx.save_for_backward(q, k, v, P, o, lse, gs, sk, cu_seqlens, fws)
        ctx.scale, ctx.window_size = scale, window_size
        ctx.gs_dtype = g_scalar.dtype if g_scalar is not None else None
        ctx.sk_dtype = sink_bias.dtype if sink_bias is not None else None
        return o

    @staticmethod
    def backward(ctx, dO):
        q, k, v, P, o, lse, gs, sk, cu, fws = ctx.saved_tensors
        want_dsink = sk is not None and ctx.needs_input_grad[6]
        dq, dk, dv, dg, dgs, dsink = wall_attn_bwd(dO, q, k, v, P, o, lse, ctx.scale, gs, sk,
                                                   ctx.window_size, cu, want_dsink, fws)
        if dgs is not None and ctx.gs_dtype is not None:
            dgs = dgs.to(ctx.gs_dtype)
        if dsink is not None:
            dsink = dsink.to(ctx.sk_dtype)
        return dq, dk, dv, dg, None, dgs, dsink, None, None


def wall_attn(q, k, v, g, scale=None, g_scalar=None, sink_bias=None, window_size=None,
              cu_seqlens=None):
    """Wall Attention o [B,T,HQ,V] (README "Usage"), differentiable in q, k,
    v, g, g_scalar and sink_bias.  g is the per-channel log-gate; g = 0 is
    vanilla causal softmax attention."""
    return WallAttnFunction.apply(q, k, v, g, scale, g_scalar, sink_bias, window_size, cu_seqlens)


def build_wall_kv_cache(k, P, chunk_size=64, capacity=None, HQ=None):
    """Pre-rescaled decode cache (README "Decode"): k_tilde [B,Tcap,HQ,K] in
    k's dtype and r_cache [B,ceil(Tcap/C),HQ,K] fp32, Tcap = capacity or T."""
    k = k.contiguous()
    P = P.contiguous()
    B, T, H, K = k.shape
    HQ = P.shape[2]
    Tcap = capacity or T
    C = int(chunk_size)
    k_tilde = torch.empty((B, Tcap, HQ, K), dtype=k.dtype, device=k.device)
    r_cache = torch.empty((B, -(-Tcap // C), HQ, K), dtype=torch.float32, device=k.device)
    L.wall_build_kv_cache(k, P, B, T, H, HQ, K, C, 0, k_tilde, r_cache, Tcap)
    return k_tilde, r_cache


def wall_attn_decode(q, v, p_curr, k_tilde, r_cache, sink_bias=None, scale=None,
                     cache_chunk_size=64, T_kv=None):
    """One decode step (README "Decode"); returns (o [B,1,HQ,V], lse
    [B,1,HQ]).  The first T_kv cache positions are read (default: all)."""
    B, Tcap, HQ, K = k_tilde.shape
    H, V = v.shape[2], v.shape[3]
    T_kv = Tcap if T_kv is None else int(T_kv)
    if v.shape[1] != Tcap:
        raise ValueError("v and k_tilde must have the same capacity")
    o = torch.empty((B, 1, HQ, V), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, 1, HQ), dtype=torch.float32, device=q.device)
    C = int(cache_chunk_size)
    ws = _ws(L.wall_attn_decode_workspace(B, T_kv, H, HQ, V, C), q.device)
    sk = sink_bias.contiguous().float() if sink_bias is not None else None
    L.wall_attn_decode(q.contiguous(), v, p_curr.contiguous(), k_tilde, r_cache, sk, scale or 0.0,
                       C, B, T_kv, Tcap, H, HQ, K, V, o, lse, ws)
    return o, lse


def wall_attn_decode_chunk(q, v, p, k_tilde, r_cache, sink_bias=None, scale=None,
                           cache_chunk_size=64, T_kv=None):
    """Multi-token decode / chunked prefill against the pre-rescaled cache:
    q [B,Tq,HQ,K] and p [B,Tq,HQ,K] (P at their positions) are the queries of
    the last Tq of the first T_kv cached positions (default: all), each
    attending causally to the cache up to its own position.  Returns
    (o [B,Tq,HQ,V], lse [B,Tq,HQ])."""
    B, Tcap, HQ, K = k_tilde.shape
    H, V = v.shape[2], v.shape[3]
    Tq = q.shape[1]
    T_kv = Tcap if T_kv is None else int(T_kv)
    if v.shape[1] != Tcap:
        raise ValueError("v and k_tilde must have the same capacity")
    o = torch.empty((B, Tq, HQ, V), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, Tq, HQ), dtype=torch.float32, device=q.device)
    C = int(cache_chunk_size)
    ws = _ws(L.wall_attn_decode_chunk_workspace(L.dtype_code(q.dtype), B, Tq, T_kv, H, HQ, K, V,
                                                C), q.device)
    sk = sink_bias.contiguous().float() if sink_bias is not None else None
    L.wall_attn_decode_chunk(q.contiguous(), v, p.contiguous(), k_tilde, r_cache, sk,
                             scale or 0.0, C, B, Tq, T_kv, Tcap, H, HQ, K, V, o, lse, ws)
    return o, lse


class WallDecodeCache:
    """Append-as-you-go decode state (README "Decode": the streaming serving
    loop): cache buffers of a fixed capacity plus the running prefix.

    ``append(k, v, g)`` fills the next positions (prefill); each ``step(q,
    k, v, g)`` appends one token (prefix update, new chunk anchor when a
    chunk starts, k_tilde and v rows) and decodes it.  Inside the fused
    step's domain (bf16, K and V in {64, 128}, HQ/H <= 8, chunk a multiple
    of 32) a step is one launch of wall_decode_step; elsewhere it is the
    prefix scan, the cache build and wall_attn_decode in turn.
    """

    def __init__(self, B, H, HQ, K, V, capacity, chunk_size=64, dtype=torch.bfloat16,
                 device="cuda", scale=None, sink_bias=None):
        self.B, self.H, self.HQ, self.K, self.V = B, H, HQ, K, V
        self.cap, self.C, self.scale, self.dtype = capacity, chunk_size, scale, dtype
        self.k_tilde = torch.empty((B, capacity, HQ, K), dtype=dtype, device=device)
        self.v = torch.empty((B, capacity, H, V), dtype=dtype, device=device)
        self.r_cache = torch.empty((B, -(-capacity // chunk_size), HQ, K), dtype=torch.float32,
                                   device=device)
        self.carry = torch.zeros((B, HQ, K), dtype=torch.float32, device=device)
        self.sink = sink_bias.contiguous().float() if sink_bias is not None else None
        self.length = 0
        self.ws = _ws(L.wall_attn_decode_workspace(B, capacity, H, HQ, V, chunk_size), device)
        self.fused = (dtype == torch.bfloat16 and K in (64, 128) and V in (64, 128)
                      and HQ // H <= 8 and chunk_size % 32 == 0)
        if self.fused:
            # the fused step's arrival counters must start at zero
            self.step_ws = torch.zeros(
                max(int(L.wall_decode_step_workspace(B, capacity, H, HQ, V, chunk_size)), 1),
                dtype=torch.uint8, device=device)

    def append(self, k, v, g):
        """Appends Tn tokens: k [B,Tn,H,K], v [B,Tn,H,V], g [B,Tn,HQ,K];
        returns their prefix P [B,Tn,HQ,K]."""
        k, v, g = k.contiguous(), v.contiguous(), g.contiguous()
        B, Tn = k.shape[:2]
        t0 = self.length
        if t0 + Tn > self.cap:
            raise ValueError("decode cache capacity exceeded")
        P = torch.empty((B, Tn, self.HQ, self.K), dtype=torch.float32, device=k.device)
        carry_out = torch.empty_like(self.carry)
        L.wall_prefix_cumsum(g, P, B, Tn, self.HQ, self.K, None, 0, self.carry, carry_out)
        self.carry = carry_out
        L.wall_build_kv_cache(k, P, B, Tn, self.H, self.HQ, self.K, self.C, t0, self.k_tilde,
                              self.r_cache, self.cap)
        self.v[:, t0:t0 + Tn].copy_(v)
        self.length = t0 + Tn
        return P

    def decode(self, q, p_curr):
        return wall_attn_decode(q, self.v, p_curr, self.k_tilde, self.r_cache, self.sink,
                                self.scale, self.C, T_kv=self.length)

    def extend(self, q, k, v, g):
        """Appends Tn tokens and attends all their queries at once (chunked
        prefill / multi-token decode): q [B,Tn,HQ,K], k [B,Tn,H,K],
        v [B,Tn,H,V], g [B,Tn,HQ,K]; returns (o [B,Tn,HQ,V], lse [B,Tn,HQ])."""
        P = self.append(k, v, g)
        return wall_attn_decode_chunk(q, self.v, P, self.k_tilde, self.r_cache, self.sink,
                                      self.scale, self.C, T_kv=self.length)

    def step(self, q, k, v, g, fused=None):
        """Appends one token and decodes its query; returns (o, lse).
        q [B,1,HQ,K], k [B,1,H,K], v [B,1,H,V], g [B,1,HQ,K].  ``fused=False``
        takes the three-call path even where the fused step applies."""
        if fused is None:
            fused = self.fused
        if not fused:
            P = self.append(k, v, g)
            return self.decode(q, P[:, -1:])
        if not self.fused:
            raise ValueError("the fused decode step does not cover this cache's shapes or dtype")
        t = self.length
        if t + 1 > self.cap:
            raise ValueError("decode cache capacity exceeded")
        B, HQ, V = self.B, self.HQ, self.V
        o = torch.empty((B, 1, HQ, V), dtype=q.dtype, device=q.device)
        lse = torch.empty((B, 1, HQ), dtype=torch.float32, device=q.device)
        L.wall_decode_step(q.contiguous(), k.contiguous(), v.contiguous(), g.contiguous(),
                           self.carry, self.k_tilde, self.v, self.r_cache, self.sink,
                           self.scale or 0.0, self.C, t, B, self.cap, self.H, HQ, self.K, V,
                           o, lse, self.step_ws)
        self.length = t + 1
        return o, lse


def timing_enable(on=True):
    """Starts (clears) or stops the library's per-stage device timing: each
    timed stage records CUDA events on the stream it runs on (wall.h,
    wall_timing_enable)."""
    L._check("wall_timing_enable", L.lib().wall_timing_enable(1 if on else 0))


TIMING_SLOTS = ("prefix_scan", "operands", "fwd_tc", "bwd_pre", "bwd_keyblock", "bwd_dq",
                "bwd_finalize", "reverse_scan", "decode", "cache_build", "decode_step",
                "decode_chunk")


def timing_enable_slots(names):
    """Times only the named stages (see TIMING_SLOTS); an empty list stops."""
    mask = 0
    for n in names:
        mask |= 1 << TIMING_SLOTS.index(n)
    L._check("wall_timing_enable_slots", L.lib().wall_timing_enable_slots(mask))


def timing_read():
    """Per-stage {name: (launches, total_ms)} since the last read or enable;
    synchronizes on the recorded events and clears the totals."""
    import ctypes
    n = len(TIMING_SLOTS)
    names = (ctypes.c_char_p * n)()
    launches = (ctypes.c_int * n)()
    ms = (ctypes.c_double * n)()
    L._check("wall_timing_read", L.lib().wall_timing_read(n, names, launches, ms))
    return {names[i].decode(): (launches[i], ms[i]) for i in range(n)}
