"""GPU parity of the decode path: the pre-rescaled cache (layout bit-exact,
values against the oracle), single-step decode and the streaming append
loop, against the fp64 oracle's forward rows and the GPU prefill forward."""
import numpy as np
import pytest
import torch

from channel_decay_softmax_b200 import api
from channel_decay_softmax_b200 import inputs as I
from oracle import wall_oracle as wo
from tests.helpers import assert_fwd, max_abs, np64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _small_decode_spec(**over):
    base = dict(B=2, T=1000, HQ=8, H=2)
    base.update(over)
    return I.spec(5, **base)


def _batch(s, b, n_rows=64, device="cpu"):
    return I.decode_batch_inputs(s, b, device=device, n_query_rows=n_rows)


def _stack(s, n_rows=64):
    xs = [_batch(s, b, n_rows) for b in range(s.B)]
    return {k: torch.stack([x[k] for x in xs]) for k in xs[0]}


def test_cache_layout_and_values():
    s = _small_decode_spec(T=1000)  # 1000 = 15 full chunks of 64 + a ragged one
    x = _stack(s)
    k, g = x["k"].to(DEV), x["g"].to(DEV)
    P = api.prefix_cumsum(g)
    kt, rc = api.build_wall_kv_cache(k, P, chunk_size=s.chunk)
    torch.cuda.synchronize()
    C = s.chunk
    nc = -(-s.T // C)
    assert kt.shape == (s.B, s.T, s.HQ, s.K) and rc.shape == (s.B, nc, s.HQ, s.K)
    # r_cache holds P at each chunk's first row, bit for bit
    assert torch.equal(rc, P[:, ::C])
    # at chunk starts the factor is exp2(0) = 1: k_tilde is k itself, bit for bit
    kx = k.repeat_interleave(s.G, dim=2)
    assert torch.equal(kt[:, ::C], kx[:, ::C])
    # everywhere: the oracle's fp64 k * 2^(R_c - P) within bf16 rounding
    kt_ref, rc_ref = wo.kv_cache(x["k"], x["g"], C)
    rel = np.abs(np64(kt) - kt_ref) / np.maximum(np.abs(kt_ref), 1e-3)
    assert float(rel.max()) < 2 ** -7, float(rel.max())
    assert max_abs(rc, rc_ref) / max(1.0, float(np.abs(rc_ref).max())) < 2e-6


def test_cache_append_keeps_started_anchor():
    """Appending rows inside a started chunk keeps that chunk's anchor: after
    appends that split chunks, r_cache holds the streamed P at each chunk's
    first row bit for bit, and k_tilde matches the one-shot build (the
    streamed prefix differs from the one-shot one only by fp32 rounding)."""
    s = _small_decode_spec(B=1, T=200)
    x = _stack(s)
    k, g = x["k"].to(DEV), x["g"].to(DEV)
    P = api.prefix_cumsum(g)
    kt_full, rc_full = api.build_wall_kv_cache(k, P, chunk_size=64)
    cache = api.WallDecodeCache(s.B, s.H, s.HQ, s.K, s.V, capacity=200, chunk_size=64,
                                dtype=s.dtype, device=DEV)
    v = x["v"].to(DEV)
    parts = []
    for a, b in ((0, 70), (70, 71), (71, 128), (128, 200)):
        parts.append(cache.append(k[:, a:b], v[:, a:b], g[:, a:b]))
    torch.cuda.synchronize()
    P_stream = torch.cat(parts, 1)
    assert torch.equal(cache.r_cache, P_stream[:, ::64])
    assert max_abs(P_stream, P) <= 1e-5 * max(1.0, float(P.abs().max()))
    assert torch.equal(cache.v, v)
    kx = k.repeat_interleave(s.G, dim=2)
    assert torch.equal(cache.k_tilde[:, ::64], kx[:, ::64])
    assert max_abs(cache.k_tilde, kt_full) <= 2 ** -6 * float(kt_full.float().abs().max())


def _decode_vs_oracle(s, bs, rows_from_end=1):
    """Single-step decode of the last row of sampled batch rows."""
    for b in bs:
        x = _batch(s, b, n_rows=1, device=DEV)
        k, v, g, q = x["k"][None], x["v"][None], x["g"][None], x["q"][None]
        P = api.prefix_cumsum(g)
        kt, rc = api.build_wall_kv_cache(k, P, chunk_size=s.chunk)
        o, lse = api.wall_attn_decode(q, v, P[:, -1:], kt, rc, scale=s.scale,
                                      cache_chunk_size=s.chunk)
        torch.cuda.synchronize()
        # the oracle's forward row T-1 with this query in that row
        o_ref, l_ref = wo.forward(q.cpu(), k.cpu(), v.cpu(), g.cpu(), scale=s.scale,
                                  rows=(s.T - 1, s.T), q_rows_only=True)
        assert_fwd(s.dtype, o[0, 0], o_ref[0, -1], lse[0, 0], l_ref[0, -1], what=f"b={b}")


def test_decode_single_step_small():
    _decode_vs_oracle(_small_decode_spec(T=1000), [0, 1])


def test_decode_fp32_small():
    s = _small_decode_spec(T=333, dtype=torch.float32)
    _decode_vs_oracle(s, [0])


@pytest.mark.slow
def test_decode_single_step_full_size_sampled():
    """Config 5 (B=32, T_kv=32768, HQ=32, H=8) at full size, in the launch
    configuration of the benchmark: every batch row decoded on the GPU,
    sampled rows checked against the oracle."""
    s = I.spec(5)
    d = I.decode_inputs(s, device=DEV, n_query_rows=1)
    P = api.prefix_cumsum(d["g"])
    kt, rc = api.build_wall_kv_cache(d["k"], P, chunk_size=s.chunk)
    o, lse = api.wall_attn_decode(d["q_tail"], d["v"], P[:, -1:].contiguous(), kt, rc,
                                  scale=s.scale, cache_chunk_size=s.chunk)
    torch.cuda.synchronize()
    del kt, rc, P
    for b in (0, 17, 31):
        o_ref, l_ref = wo.forward(d["q_tail"][b:b + 1].cpu(), d["k"][b:b + 1].cpu(),
                                  d["v"][b:b + 1].cpu(), d["g"][b:b + 1].cpu(), scale=s.scale,
                                  rows=(s.T - 1, s.T), q_rows_only=True)
        assert_fwd(s.dtype, o[b, 0], o_ref[0, -1], lse[b, 0], l_ref[0, -1], what=f"b={b}")


def _streaming(s, n_stream, check_prefill, fused=None):
    """Build the cache from [0, T - n) then append n tokens one by one; each
    decoded row must equal the oracle's forward row (and the GPU prefill
    forward row).  ``fused`` picks the one-launch step or the three-call
    append + decode (default: the fused step where it applies)."""
    x = _stack(s, n_rows=n_stream)
    k, v, g = x["k"].to(DEV), x["v"].to(DEV), x["g"].to(DEV)
    q_tail = x["q"].to(DEV)
    T0 = s.T - n_stream
    cache = api.WallDecodeCache(s.B, s.H, s.HQ, s.K, s.V, capacity=s.T, chunk_size=s.chunk,
                                dtype=s.dtype, device=DEV, scale=s.scale)
    cache.append(k[:, :T0], v[:, :T0], g[:, :T0])
    outs, lses = [], []
    for t in range(T0, s.T):
        o, lse = cache.step(q_tail[:, t - T0:t - T0 + 1], k[:, t:t + 1], v[:, t:t + 1],
                            g[:, t:t + 1], fused=fused)
        outs.append(o)
        lses.append(lse)
    torch.cuda.synchronize()
    o_stream = torch.cat(outs, 1)
    l_stream = torch.cat(lses, 1)
    for b in range(s.B):
        o_ref, l_ref = wo.forward(x["q"][b:b + 1], x["k"][b:b + 1], x["v"][b:b + 1],
                                  x["g"][b:b + 1], scale=s.scale, rows=(T0, s.T),
                                  q_rows_only=True)
        assert_fwd(s.dtype, o_stream[b], o_ref[0, T0:], l_stream[b], l_ref[0, T0:],
                   what=f"stream b={b}")
    if check_prefill:
        qfull = torch.zeros((s.B, s.T, s.HQ, s.K), dtype=s.dtype)
        qfull[:, T0:] = x["q"]
        o_pf = api.wall_attn(qfull.to(DEV), k, v, g, scale=s.scale)
        assert_fwd(s.dtype, o_stream, o_pf[:, T0:], what="stream vs prefill")


@pytest.mark.parametrize("fused", [True, False], ids=["fused_step", "three_call"])
def test_streaming_loop_small(fused):
    _streaming(_small_decode_spec(T=700), 64, check_prefill=True, fused=fused)


def _step_cache(s, x, T0, fused, sink=None):
    """Cache of capacity T with positions [0, T0) appended at once, then
    T - T0 single-token steps; returns the cache and the decoded rows."""
    k, v, g, q = (x[n].to(DEV) for n in ("k", "v", "g", "q"))
    cache = api.WallDecodeCache(s.B, s.H, s.HQ, s.K, s.V, capacity=s.T, chunk_size=s.chunk,
                                dtype=s.dtype, device=DEV, scale=s.scale, sink_bias=sink)
    if T0 > 0:
        cache.append(k[:, :T0], v[:, :T0], g[:, :T0])
    outs, lses = [], []
    for t in range(T0, s.T):
        o, lse = cache.step(q[:, t - T0:t - T0 + 1], k[:, t:t + 1], v[:, t:t + 1],
                            g[:, t:t + 1], fused=fused)
        outs.append(o)
        lses.append(lse)
    torch.cuda.synchronize()
    return cache, torch.cat(outs, 1), torch.cat(lses, 1)


def test_decode_step_matches_three_call_path():
    """The fused step leaves the carry, k_tilde, v and r_cache bit for bit as
    the prefix scan + cache build + value copy do (the same fp32 operations:
    P_t = carry + g / ln 2 in one fused rounding, k * exp2(R - P_t) rounded
    to bf16), across chunk starts at 128 and 192.  Its decoded rows agree to
    bf16 rounding: the new token's own score comes from k itself (factor
    exp2(0) = 1), not from its rounded k_tilde row.  Every call leaves the
    per-head arrival counters at zero."""
    s = _small_decode_spec(B=2, T=300, HQ=8, H=2)
    T0 = 100
    x = _stack(s, n_rows=s.T - T0)
    cf, of, lf = _step_cache(s, x, T0, fused=True)
    c3, o3, l3 = _step_cache(s, x, T0, fused=False)
    assert torch.equal(cf.carry, c3.carry)
    assert torch.equal(cf.k_tilde, c3.k_tilde)
    assert torch.equal(cf.v, c3.v)
    assert torch.equal(cf.r_cache, c3.r_cache)
    assert_fwd(s.dtype, of, o3, lf, l3, what="fused vs three-call")
    al = lambda n: (n + 255) // 256 * 256
    counters = cf.step_ws[-al(4 * s.B * s.HQ):]
    assert int(counters.count_nonzero()) == 0


@pytest.mark.parametrize("HQ,H,K,V,C,sink", [
    (8, 1, 64, 64, 32, True),     # 8 heads per kv head (one warp per head), sink
    (4, 2, 128, 64, 64, False),   # K != V
    (2, 2, 64, 128, 96, True),    # no grouping, a chunk that is not a power of two
])
def test_decode_step_from_empty_cache(HQ, H, K, V, C, sink):
    """Streaming from an empty cache (t = 0 decodes the token against itself
    only): every row equals the oracle's forward row, with the sink logit."""
    s = _small_decode_spec(B=2, T=200, HQ=HQ, H=H, K=K, V=V, chunk=C)
    x = _stack(s, n_rows=s.T)
    sk = None
    if sink:
        gen = torch.Generator().manual_seed(77)
        sk = torch.randn((HQ,), generator=gen, dtype=torch.float32)
    cache, o, lse = _step_cache(s, x, 0, fused=True,
                                sink=sk.to(DEV) if sk is not None else None)
    assert cache.fused
    for b in range(s.B):
        o_ref, l_ref = wo.forward(x["q"][b:b + 1], x["k"][b:b + 1], x["v"][b:b + 1],
                                  x["g"][b:b + 1], scale=s.scale, sink_bias=sk,
                                  rows=(0, s.T), q_rows_only=True)
        assert_fwd(s.dtype, o[b], o_ref[0], lse[b], l_ref[0], what=f"step b={b}")


@pytest.mark.slow
def test_streaming_loop_full_size_sampled():
    """Config 5's 64-token append loop on sampled batch rows at T_kv=32768."""
    s = I.spec(5, B=2)
    _streaming(s, 64, check_prefill=False)
