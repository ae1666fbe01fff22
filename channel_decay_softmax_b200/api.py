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
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be 1-D [n_seq + 1]")
    return cu_seqlens.numel() - 1


# The library receives bare pointers and sizes: a tensor of the wrong dtype
# or shape would make a kernel read or write past its buffer.  These checks
# run before any call into the library.

def _io_dtype(q, *others):
    """q's dtype (bf16 or fp32), shared by every tensor in ``others``."""
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError(f"unsupported dtype {q.dtype}; use bfloat16 or float32")
    for t in others:
        if t is not None and t.dtype != q.dtype:
            raise TypeError(f"inputs must share one dtype: {q.dtype} and {t.dtype}")
    return q.dtype


def _expect(name, t, shape, dtype=None):
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _opt_f32(name, t, shape):
    """An optional fp32 argument (g_scalar, sink_bias): shape-checked, then
    made contiguous fp32."""
    if t is None:
        return None
    _expect(name, t, shape)
    return t.contiguous().float()


def _same_device(ref, *ts):
    for t in ts:
        if t is not None and t.device != ref.device:
            raise ValueError(f"all tensors must be on {ref.device}, got one on {t.device}")


def _check_cache(q, v, p, k_tilde, r_cache, C, T_kv, Tq):
    """Shapes of a decode call against the cache: q and p [B,Tq,HQ,K],
    v [B,Tcap,H,V], r_cache [B,ceil(Tcap/C),HQ,K] fp32, 1 <= Tq <= T_kv <= Tcap."""
    if k_tilde.dim() != 4 or v.dim() != 4:
        raise ValueError("k_tilde must be [B,Tcap,HQ,K] and v [B,Tcap,H,V]")
    B, Tcap, HQ, K = k_tilde.shape
    _io_dtype(k_tilde, q, v)
    if v.shape[0] != B or v.shape[1] != Tcap or HQ % v.shape[2] != 0:
        raise ValueError("v must be [B,Tcap,H,V] with the cache's B, Tcap and HQ % H == 0")
    if C < 1:
        raise ValueError("cache_chunk_size must be positive")
    if not 1 <= Tq <= T_kv <= Tcap:
        raise ValueError(f"need 1 <= Tq ({Tq}) <= T_kv ({T_kv}) <= capacity ({Tcap})")
    _expect("q", q, (B, Tq, HQ, K))
    _expect("p", p, (B, Tq, HQ, K), torch.float32)
    _expect("r_cache", r_cache, (B, -(-Tcap // C), HQ, K), torch.float32)
    _same_device(k_tilde, q, v, p, r_cache)


def _ws(nbytes, device):
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def prefix_cumsum(g, cu_seqlens=None, carry_in=None, return_carry=False):
    """P = cumsum_t(g) / ln 2 per sequence (fp32), with an optional carried-in
    prefix [n_seq or B, HQ, K]; README "Decode" builds P this way."""
    if g.dim() != 4:
        raise ValueError("g must be [B, T, HQ, K]")
    _io_dtype(g)
    g = g.contiguous()
    B, T, HQ, K = g.shape
    nseq = _n_seq(cu_seqlens, B)
    ns = nseq if cu_seqlens is not None else B
    cin = _opt_f32("carry_in", carry_in, (ns, HQ, K))
    _same_device(g, cu_seqlens, cin)
    P = torch.empty(g.shape, dtype=torch.float32, device=g.device)
    carry_out = torch.empty((ns, HQ, K), dtype=torch.float32, device=g.device) \
        if return_carry else None
    L.wall_prefix_cumsum(g, P, B, T, HQ, K, cu_seqlens, nseq, cin, carry_out)
    return (P, carry_out) if return_carry else P


def wall_attn_fwd(q, k, v, P, scale=None, g_scalar=None, sink_bias=None, window_size=None,
                  cu_seqlens=None, return_workspace=False):
    """Forward from a precomputed prefix P; returns (o, lse), or (o, lse,
    workspace) with return_workspace: the workspace holds the anchored
    operands, which wall_attn_bwd can reuse (its fwd_workspace)."""
    B, T, H, HQ, K, V = _shape_checks(q, k, v, P)
    nseq = _n_seq(cu_seqlens, B)
    _io_dtype(q, k, v)
    _expect("P", P, q.shape, torch.float32)
    g_scalar = _opt_f32("g_scalar", g_scalar, (B, T, HQ))
    sink_bias = _opt_f32("sink_bias", sink_bias, (HQ,))
    _same_device(q, k, v, P, g_scalar, sink_bias, cu_seqlens)
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
    _io_dtype(q, k, v, g)
    g_scalar = _opt_f32("g_scalar", g_scalar, (B, T, HQ))
    sink_bias = _opt_f32("sink_bias", sink_bias, (HQ,))
    _same_device(q, k, v, g, g_scalar, sink_bias, cu_seqlens)
    o = torch.empty((B, T, HQ, V), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, T, HQ), dtype=torch.float32, device=q.device)
    P = torch.empty((B, T, HQ, K), dtype=torch.float32, device=q.device)
    ws = _ws(L.wall_attn_fwd_gate_workspace(q.dtype, B, T, H, HQ, K, V, g_scalar is not None,
                                            nseq), q.device)
    L.wall_attn_fwd_gate(q, k, v, g, B, T, H, HQ, K, V, scale or 0.0, g_scalar, sink_bias,
                         window_size or 0, cu_seqlens, nseq, P, o, lse, ws)
    return (o, lse, P, ws) if return_workspace else (o, lse, P)


def wall_attn_bwd(dO, q, k, v, P, o, lse, scale=None, g_scalar=None, sink_bias=None,
                  window_size=None, cu_seqlens=None, want_dsink=False, fwd_workspace=None,
                  store_ds=True):
    """Backward; returns dq, dk, dv, dg, dg_scalar (or None), dsink (or None).
    fwd_workspace: the workspace returned by wall_attn_fwd(..., return_workspace=True)
    for the same inputs, whose anchored operands are then reused.  store_ds=False
    gives the library the smaller workspace without the dS tiles: its dq pass
    then recomputes them (less memory, more time)."""
    B, T, H, HQ, K, V = _shape_checks(q, k, v, P)
    nseq = _n_seq(cu_seqlens, B)
    _io_dtype(q, k, v, dO, o)
    _expect("P", P, q.shape, torch.float32)
    _expect("dO", dO, (B, T, HQ, V))
    _expect("o", o, (B, T, HQ, V))
    _expect("lse", lse, (B, T, HQ), torch.float32)
    g_scalar = _opt_f32("g_scalar", g_scalar, (B, T, HQ))
    sink_bias = _opt_f32("sink_bias", sink_bias, (HQ,))
    _same_device(q, k, v, P, dO, o, lse, g_scalar, sink_bias, cu_seqlens, fwd_workspace)
    if fwd_workspace is not None:
        # the forward's operands are read from it: it must hold at least the
        # forward workspace of this problem
        need = L.wall_attn_fwd_workspace(q.dtype, B, T, H, HQ, K, V, g_scalar is not None, nseq)
        have = fwd_workspace.numel() * fwd_workspace.element_size()
        if not fwd_workspace.is_contiguous() or have < need:
            raise ValueError(f"fwd_workspace holds {have} bytes; this problem's forward "
                             f"workspace needs {need}")
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    dg = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    dgs = torch.empty_like(g_scalar) if g_scalar is not None else None
    dsink = torch.empty((HQ,), dtype=torch.float32, device=q.device) \
        if (want_dsink and sink_bias is not None) else None
    if store_ds:
        nbytes = L.wall_attn_bwd_workspace(q.dtype, B, T, H, HQ, K, V, g_scalar is not None,
                                           nseq, window_size or 0)
    else:
        nbytes = L.wall_attn_bwd_workspace_min(q.dtype, B, T, H, HQ, K, V, g_scalar is not None,
                                               nseq)
    ws = _ws(nbytes, q.device)
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


class WallAttnStepGraph:
    """One training step -- the fused prefix + forward and the backward
    reusing its operands -- captured once in a CUDA graph for fixed shapes
    and options, then replayed.  Small problems are bound by the host's
    issue of the step's launches; a replay is one graph launch.

    The inputs are copied into buffers the graph owns (``inputs``); replay()
    copies any new inputs in, replays, and returns the graph's output
    tensors (o, lse, dq, dk, dv, dg, dg_scalar, dsink), which the next replay
    overwrites.
    """

    def __init__(self, q, k, v, g, dO, scale=None, g_scalar=None, sink_bias=None,
                 window_size=None, cu_seqlens=None, want_dsink=False, warmup=2):
        self.inputs = {n: t.detach().contiguous().clone()
                       for n, t in (("q", q), ("k", k), ("v", v), ("g", g), ("dO", dO))}
        self.scale, self.window, self.want_dsink = scale, window_size, want_dsink
        self.gs = g_scalar.detach().contiguous().float().clone() if g_scalar is not None else None
        self.sk = sink_bias.detach().contiguous().float().clone() if sink_bias is not None else None
        self.cu = cu_seqlens.clone() if cu_seqlens is not None else None
        # warm-up on a side stream (first-call setup happens outside the capture)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(max(1, warmup)):
                self._step()
        torch.cuda.current_stream().wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.outputs = self._step()

    def _step(self):
        x = self.inputs
        o, lse, P, fws = wall_attn_fwd_gate(x["q"], x["k"], x["v"], x["g"], self.scale, self.gs,
                                            self.sk, self.window, self.cu, return_workspace=True)
        dq, dk, dv, dg, dgs, dsink = wall_attn_bwd(
            x["dO"], x["q"], x["k"], x["v"], P, o, lse, self.scale, self.gs, self.sk,
            self.window, self.cu, self.want_dsink and self.sk is not None, fws)
        return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv, dg=dg, dg_scalar=dgs, dsink=dsink)

    def replay(self, **new_inputs):
        """Copies the given inputs (any of q, k, v, g, dO) in and replays."""
        for n, t in new_inputs.items():
            if n not in self.inputs:
                raise KeyError(f"unknown input {n}")
            _expect(n, t, self.inputs[n].shape, self.inputs[n].dtype)
            self.inputs[n].copy_(t)
        self.graph.replay()
        return self.outputs


def build_wall_kv_cache(k, P, chunk_size=64, capacity=None, HQ=None):
    """Pre-rescaled decode cache (README "Decode"): k_tilde [B,Tcap,HQ,K] in
    k's dtype and r_cache [B,ceil(Tcap/C),HQ,K] fp32, Tcap = capacity or T."""
    if k.dim() != 4 or P.dim() != 4:
        raise ValueError("k must be [B,T,H,K] and P [B,T,HQ,K]")
    _io_dtype(k)
    k = k.contiguous()
    P = P.contiguous()
    B, T, H, K = k.shape
    HQ = P.shape[2]
    _expect("P", P, (B, T, HQ, K), torch.float32)
    if HQ % H != 0:
        raise ValueError("HQ must be a multiple of H")
    _same_device(k, P)
    Tcap = capacity or T
    C = int(chunk_size)
    if Tcap < T or C < 1:
        raise ValueError("need capacity >= T and chunk_size >= 1")
    k_tilde = torch.empty((B, Tcap, HQ, K), dtype=k.dtype, device=k.device)
    r_cache = torch.empty((B, -(-Tcap // C), HQ, K), dtype=torch.float32, device=k.device)
    L.wall_build_kv_cache(k, P, B, T, H, HQ, K, C, 0, k_tilde, r_cache, Tcap)
    return k_tilde, r_cache


def wall_attn_decode(q, v, p_curr, k_tilde, r_cache, sink_bias=None, scale=None,
                     cache_chunk_size=64, T_kv=None):
    """One decode step (README "Decode"); returns (o [B,1,HQ,V], lse
    [B,1,HQ]).  The first T_kv cache positions are read (default: all)."""
    C = int(cache_chunk_size)
    T_kv = k_tilde.shape[1] if T_kv is None else int(T_kv)
    _check_cache(q, v, p_curr, k_tilde, r_cache, C, T_kv, 1)
    B, Tcap, HQ, K = k_tilde.shape
    H, V = v.shape[2], v.shape[3]
    sk = _opt_f32("sink_bias", sink_bias, (HQ,))
    _same_device(k_tilde, sk)
    o = torch.empty((B, 1, HQ, V), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, 1, HQ), dtype=torch.float32, device=q.device)
    ws = _ws(L.wall_attn_decode_workspace(B, T_kv, H, HQ, V, C), q.device)
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
    C = int(cache_chunk_size)
    T_kv = k_tilde.shape[1] if T_kv is None else int(T_kv)
    if q.dim() != 4:
        raise ValueError("q must be [B, Tq, HQ, K]")
    Tq = q.shape[1]
    _check_cache(q, v, p, k_tilde, r_cache, C, T_kv, Tq)
    B, Tcap, HQ, K = k_tilde.shape
    H, V = v.shape[2], v.shape[3]
    sk = _opt_f32("sink_bias", sink_bias, (HQ,))
    _same_device(k_tilde, sk)
    o = torch.empty((B, Tq, HQ, V), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, Tq, HQ), dtype=torch.float32, device=q.device)
    ws = _ws(L.wall_attn_decode_chunk_workspace(L.dtype_code(q.dtype), B, Tq, T_kv, H, HQ, K, V,
                                                C), q.device)
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
        if HQ % H != 0 or capacity < 1 or chunk_size < 1:
            raise ValueError("need HQ % H == 0, capacity >= 1 and chunk_size >= 1")
        self.B, self.H, self.HQ, self.K, self.V = B, H, HQ, K, V
        self.cap, self.C, self.scale, self.dtype = capacity, chunk_size, scale, dtype
        self.k_tilde = torch.empty((B, capacity, HQ, K), dtype=dtype, device=device)
        self.v = torch.empty((B, capacity, H, V), dtype=dtype, device=device)
        self.r_cache = torch.empty((B, -(-capacity // chunk_size), HQ, K), dtype=torch.float32,
                                   device=device)
        self.carry = torch.zeros((B, HQ, K), dtype=torch.float32, device=device)
        self.sink = _opt_f32("sink_bias", sink_bias, (HQ,))
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
        Tn = self._check_tokens(k, v, g)
        k, v, g = k.contiguous(), v.contiguous(), g.contiguous()
        B = self.B
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

    def _check_tokens(self, k, v, g, q=None):
        """Shapes and dtype of Tn new tokens for this cache; returns Tn."""
        if k.dim() != 4:
            raise ValueError("k must be [B, Tn, H, K]")
        Tn = k.shape[1]
        B, H, HQ = self.B, self.H, self.HQ
        _expect("k", k, (B, Tn, H, self.K), self.dtype)
        _expect("v", v, (B, Tn, H, self.V), self.dtype)
        _expect("g", g, (B, Tn, HQ, self.K), self.dtype)
        _expect("q", q, (B, Tn, HQ, self.K), self.dtype)
        _same_device(self.k_tilde, k, v, g, q)
        return Tn

    def decode(self, q, p_curr):
        return wall_attn_decode(q, self.v, p_curr, self.k_tilde, self.r_cache, self.sink,
                                self.scale, self.C, T_kv=self.length)

    def extend(self, q, k, v, g):
        """Appends Tn tokens and attends all their queries at once (chunked
        prefill / multi-token decode): q [B,Tn,HQ,K], k [B,Tn,H,K],
        v [B,Tn,H,V], g [B,Tn,HQ,K]; returns (o [B,Tn,HQ,V], lse [B,Tn,HQ])."""
        self._check_tokens(k, v, g, q)
        P = self.append(k, v, g)
        return wall_attn_decode_chunk(q, self.v, P, self.k_tilde, self.r_cache, self.sink,
                                      self.scale, self.C, T_kv=self.length)

    def step(self, q, k, v, g, fused=None):
        """Appends one token and decodes its query; returns (o, lse).
        q [B,1,HQ,K], k [B,1,H,K], v [B,1,H,V], g [B,1,HQ,K].  ``fused=False``
        takes the three-call path even where the fused step applies."""
        if fused is None:
            fused = self.fused
        if self._check_tokens(k, v, g, q) != 1:
            raise ValueError("step takes one token; use extend for several")
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
                "decode_chunk", "exact_units")


def timing_enable_slots(names):
    """Times only the named stages (see TIMING_SLOTS); an empty list stops."""
    mask = 0
    for n in names:
        if n not in TIMING_SLOTS:
            raise ValueError(f"unknown stage {n!r}; the stages are {', '.join(TIMING_SLOTS)}")
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
