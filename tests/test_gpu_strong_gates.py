"""GPU parity with strongly decaying gate channels: per-step log-gates of
-0.5, -1 and -3 (a gate of 0.61, 0.37 and 0.05) next to the pages' mild ones.

The per-block anchor keeps every exponent bounded by one block's accumulated
gate (blog "Wall Attention", fast training section 1).  A -3 channel sums to
about -554 in base 2 over a 128-row block, far outside bf16 and fp32.  The
training path detects such (sequence, head) units while it forms the anchored
operands and recomputes them exactly on CUDA cores.  The decode cache keeps
one anchor per chunk (README "Decode"), so a chunk past the range cannot be
stored; building or appending one records WALL_ERR_RANGE.  Every case is
compared with the fp64 oracle at the benchmark spec's tolerances."""
import pytest
import torch

from channel_decay_softmax_b200 import _lib as L
from channel_decay_softmax_b200 import api
from channel_decay_softmax_b200 import inputs as I
from oracle import wall_oracle as wo
from tests.helpers import assert_fwd, assert_grad
from tests.test_gpu_training import _check_all, _to

pytestmark = pytest.mark.gpu

DEV = "cuda"
MIX = (0.5, 1.0, 3.0)


def _clear_status():
    L.wall_get_status()


@pytest.mark.parametrize("cfg,T", [(2, 300), (2, 1024), (3, 300), (3, 1024)])
def test_training_strong_gates(cfg, T):
    """Prefix scan, forward and backward on config 2's and config 3's shapes
    with a third of the channels strongly decaying: every head has such
    channels, so every unit takes the exact path."""
    _clear_status()
    s = I.spec(cfg, T=T, B=1, g_strong=MIX)
    _check_all(s, I.training_inputs(s), what=f"strong cfg{cfg} T={T}")
    assert L.wall_get_status() == L.WALL_OK


def test_training_strong_gates_within_anchor_range():
    """Channels at -0.5 per step sum to about -92 in base 2 over a block,
    inside the anchored operands' range: the tensor-core path itself."""
    _clear_status()
    s = I.spec(3, T=1024, B=1, g_strong=(0.5, 0.5, 0.5))
    _check_all(s, I.training_inputs(s), what="strong -0.5")
    assert L.wall_get_status() == L.WALL_OK


def test_training_strong_gates_mixed_units_varlen_options():
    """Strong channels in the first 4 of a GQA group's 8 query heads of a
    varlen problem with every option (g_scalar, sink, window): recomputed
    and tensor-core units side by side, summed into one kv head's dk and
    dv, and the per-sequence unit flags."""
    _clear_status()
    s = I.spec(4, len_lo=64, len_hi=600, window=128, g_strong=MIX, strong_heads=4)
    _check_all(s, I.training_inputs(s), what="strong varlen options")
    assert L.wall_get_status() == L.WALL_OK


def test_training_strong_gates_fp32():
    """The fp32 CUDA-core path: blocks wider than its anchor range take
    their diagonal tile pair by pair.  T = 130 keeps |P| under about 600, so
    that P's own fp32 rounding stays inside the 1e-5 bound."""
    _clear_status()
    s = I.spec(1, T=130, g_strong=MIX)
    _check_all(s, I.training_inputs(s), what="strong fp32")
    assert L.wall_get_status() == L.WALL_OK


def test_strong_gates_bench_sequence_and_autograd():
    """The benchmark's call sequence (wall_attn_fwd_gate, then wall_attn_bwd
    given the gate call's workspace) and the autograd function, with strong
    channels in the first 6 of 16 heads (kv head 1 sums a recomputed and a
    tensor-core pair of heads)."""
    _clear_status()
    s = I.spec(3, T=700, B=1, g_strong=MIX, strong_heads=6)
    xc = I.training_inputs(s)
    x = _to(xc)
    ref = wo.backward(xc["q"], xc["k"], xc["v"], xc["g"], xc["dO"], scale=s.scale)
    o, lse, P, ws = api.wall_attn_fwd_gate(x["q"], x["k"], x["v"], x["g"], s.scale,
                                           return_workspace=True)
    dq, dk, dv, dg, _, _ = api.wall_attn_bwd(x["dO"], x["q"], x["k"], x["v"], P, o, lse,
                                             s.scale, fwd_workspace=ws)
    torch.cuda.synchronize()
    assert_fwd(s.dtype, o, ref["o"], lse, ref["lse"], what="gate call")
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv), ("dg", dg)):
        assert_grad(s.dtype, name, got, ref[name], what="bwd with gate workspace")
    q, k, v, g = (x[n].clone().requires_grad_(True) for n in ("q", "k", "v", "g"))
    oa = api.wall_attn(q, k, v, g, scale=s.scale)
    oa.backward(x["dO"])
    torch.cuda.synchronize()
    assert_fwd(s.dtype, oa, ref["o"], what="autograd")
    for name, got in (("dq", q.grad), ("dk", k.grad), ("dv", v.grad), ("dg", g.grad)):
        assert_grad(s.dtype, name, got, ref[name], what="autograd")
    assert L.wall_get_status() == L.WALL_OK


@pytest.mark.slow
def test_strong_gates_long_context_sampled():
    """Config 3 at T = 8192 with strong channels, one GQA group (4 query
    heads) against the oracle, element by element."""
    _clear_status()
    s = I.spec(3, g_strong=MIX)
    _check_all(s, I.training_inputs(s), units=[4, 5, 6, 7], what="strong cfg3 full")
    assert L.wall_get_status() == L.WALL_OK


def _decode_spec(**over):
    base = dict(B=2, T=1000, HQ=8, H=2)
    base.update(over)
    return I.spec(5, **base)


def _stack(s, n_rows):
    xs = [I.decode_batch_inputs(s, b, device="cpu", n_query_rows=n_rows) for b in range(s.B)]
    return {k: torch.stack([x[k] for x in xs]) for k in xs[0]}


def _oracle_rows(s, x, b, T0):
    return wo.forward(x["q"][b:b + 1], x["k"][b:b + 1], x["v"][b:b + 1], x["g"][b:b + 1],
                      scale=s.scale, rows=(T0, s.T), q_rows_only=True)


@pytest.mark.parametrize("fused", [True, False], ids=["fused_step", "three_call"])
def test_decode_and_streaming_strong_within_range(fused):
    """C = 64 with channels at -0.5 and -1 per step (a chunk sums to about
    -46 and -92 in base 2): cache build, 16 streamed tokens and their
    decodes match the oracle rows, with no status."""
    _clear_status()
    s = _decode_spec(g_strong=(0.5, 1.0))
    n = 16
    x = _stack(s, n)
    k, v, g, q = (x[name].to(DEV) for name in ("k", "v", "g", "q"))
    T0 = s.T - n
    cache = api.WallDecodeCache(s.B, s.H, s.HQ, s.K, s.V, capacity=s.T, chunk_size=s.chunk,
                                dtype=s.dtype, device=DEV, scale=s.scale)
    cache.append(k[:, :T0], v[:, :T0], g[:, :T0])
    outs, lses = [], []
    for t in range(T0, s.T):
        o, lse = cache.step(q[:, t - T0:t - T0 + 1], k[:, t:t + 1], v[:, t:t + 1],
                            g[:, t:t + 1], fused=fused)
        outs.append(o)
        lses.append(lse)
    torch.cuda.synchronize()
    o_s, l_s = torch.cat(outs, 1), torch.cat(lses, 1)
    for b in range(s.B):
        o_ref, l_ref = _oracle_rows(s, x, b, T0)
        assert_fwd(s.dtype, o_s[b], o_ref[0, T0:], l_s[b], l_ref[0, T0:], what=f"b={b}")
    assert L.wall_get_status() == L.WALL_OK


def test_decode_chunk_strong_within_range():
    """The chunk call (two 128-row query blocks) with channels at -0.5 per
    step: a query block sums to about -92, inside the range."""
    _clear_status()
    s = _decode_spec(g_strong=(0.5,))
    Tq = 130
    x = _stack(s, Tq)
    k, v, g, q = (x[name].to(DEV) for name in ("k", "v", "g", "q"))
    P = api.prefix_cumsum(g)
    kt, rc = api.build_wall_kv_cache(k, P, chunk_size=s.chunk)
    o, lse = api.wall_attn_decode_chunk(q, v, P[:, -Tq:], kt, rc, scale=s.scale,
                                        cache_chunk_size=s.chunk)
    torch.cuda.synchronize()
    T0 = s.T - Tq
    for b in range(s.B):
        o_ref, l_ref = _oracle_rows(s, x, b, T0)
        assert_fwd(s.dtype, o[b], o_ref[0, T0:], lse[b], l_ref[0, T0:], what=f"chunk b={b}")
    assert L.wall_get_status() == L.WALL_OK


def test_decode_out_of_range_reported():
    """Channels at -3 per step: a 64-row cache chunk sums to about -277 in
    base 2, beyond the range k_tilde can hold.  The cache build, a streamed
    append and a chunk call whose 128-row query block spans more than the
    range (-1 per step) each record WALL_ERR_RANGE instead of returning
    silent overflow; the status reads once and clears."""
    _clear_status()
    s = _decode_spec(T=300, g_strong=(3.0,))
    x = _stack(s, 1)
    k, v, g = (x[name].to(DEV) for name in ("k", "v", "g"))
    P = api.prefix_cumsum(g)
    api.build_wall_kv_cache(k, P, chunk_size=s.chunk)
    assert L.wall_get_status() == L.WALL_ERR_RANGE
    assert L.wall_get_status() == L.WALL_OK
    cache = api.WallDecodeCache(s.B, s.H, s.HQ, s.K, s.V, capacity=s.T, chunk_size=s.chunk,
                                dtype=s.dtype, device=DEV, scale=s.scale)
    qs = torch.zeros((s.B, 1, s.HQ, s.K), dtype=s.dtype, device=DEV)
    for t in range(0, 80):  # one chunk start (t = 64) and its first rows
        cache.step(qs, k[:, t:t + 1], v[:, t:t + 1], g[:, t:t + 1])
    assert L.wall_get_status() == L.WALL_ERR_RANGE
    s1 = _decode_spec(T=300, g_strong=(1.0,))
    Tq = 130
    x1 = _stack(s1, Tq)
    k1, v1, g1, q1 = (x1[name].to(DEV) for name in ("k", "v", "g", "q"))
    P1 = api.prefix_cumsum(g1)
    kt1, rc1 = api.build_wall_kv_cache(k1, P1, chunk_size=s1.chunk)
    assert L.wall_get_status() == L.WALL_OK  # the cache itself is in range
    api.wall_attn_decode_chunk(q1, v1, P1[:, -Tq:], kt1, rc1, scale=s1.scale,
                               cache_chunk_size=s1.chunk)
    assert L.wall_get_status() == L.WALL_ERR_RANGE
    assert L.wall_get_status() == L.WALL_OK
