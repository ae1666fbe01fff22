"""GPU parity of wall_attn_decode_chunk: Tq queries at the last Tq cached
positions attend to the pre-rescaled cache at once (multi-token decode and
chunked prefill, bottom-right aligned causal mask).  Every row must equal the
fp64 oracle's forward row at its position, on both paths (tensor cores for
bf16 with K == V in {64, 128}; the split-KV decode elsewhere)."""
import numpy as np
import pytest
import torch

from channel_decay_softmax_b200 import _lib as L
from channel_decay_softmax_b200 import api
from channel_decay_softmax_b200 import inputs as I
from oracle import wall_oracle as wo
from tests.helpers import assert_fwd

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _inputs(s, Tq):
    xs = [I.decode_batch_inputs(s, b, device="cpu", n_query_rows=Tq) for b in range(s.B)]
    return {k: torch.stack([x[k] for x in xs]) for k in xs[0]}


def _sink(HQ, seed=77):
    gen = torch.Generator().manual_seed(seed)
    return torch.randn((HQ,), generator=gen, dtype=torch.float32)


def _cache(s, x, Tcap, fill_nan=False):
    """The whole sequence appended at once into a cache of capacity Tcap;
    positions past T (and, with fill_nan, their value rows) hold NaN."""
    k, v, g = x["k"].to(DEV), x["v"].to(DEV), x["g"].to(DEV)
    P = api.prefix_cumsum(g)
    kt, rc = api.build_wall_kv_cache(k, P, chunk_size=s.chunk, capacity=Tcap)
    vc = torch.empty((s.B, Tcap, s.H, s.V), dtype=s.dtype, device=DEV)
    if fill_nan:
        kt[:, s.T:] = float("nan")
        vc[:, s.T:] = float("nan")
    vc[:, :s.T] = v
    return P, kt, rc, vc


def _check_rows(s, x, o, lse, Tq, sink=None, what=""):
    T0 = s.T - Tq
    for b in range(s.B):
        o_ref, l_ref = wo.forward(x["q"][b:b + 1], x["k"][b:b + 1], x["v"][b:b + 1],
                                  x["g"][b:b + 1], scale=s.scale, sink_bias=sink,
                                  rows=(T0, s.T), q_rows_only=True)
        assert_fwd(s.dtype, o[b], o_ref[0, T0:], lse[b], l_ref[0, T0:], what=f"{what} b={b}")


@pytest.mark.parametrize("Tq", [1, 5, 64, 130, 1000])
def test_chunk_tensor_core_path(Tq):
    """bf16, K = V = 128, C = 64: one query row, a few, a 64-row chunk, two
    query blocks with a ragged tail, and the whole sequence (the chunk is
    then a full prefill of the cache, every row its own causal limit)."""
    s = I.spec(5, B=2, T=1000, HQ=8, H=2)
    assert L.lib() and s.dtype == torch.bfloat16
    x = _inputs(s, Tq)
    P, kt, rc, vc = _cache(s, x, Tcap=s.T)
    o, lse = api.wall_attn_decode_chunk(x["q"].to(DEV), vc, P[:, s.T - Tq:], kt, rc,
                                        scale=s.scale, cache_chunk_size=s.chunk)
    torch.cuda.synchronize()
    assert L.wall_get_status() == L.WALL_OK
    _check_rows(s, x, o, lse, Tq, what=f"Tq={Tq}")


@pytest.mark.parametrize("K,C,sink", [(64, 32, True), (128, 128, False), (128, 256, True)])
def test_chunk_tensor_core_shapes(K, C, sink):
    """K = V = 64, chunk sizes 32 (four chunks per key tile), 128 and 256 (a
    chunk spans tiles), with and without the sink logit; GQA 4:1."""
    s = I.spec(5, B=2, T=777, HQ=8, H=2, K=K, V=K, chunk=C)
    Tq = 100
    x = _inputs(s, Tq)
    sk = _sink(s.HQ) if sink else None
    P, kt, rc, vc = _cache(s, x, Tcap=s.T)
    o, lse = api.wall_attn_decode_chunk(x["q"].to(DEV), vc, P[:, s.T - Tq:], kt, rc,
                                        sink_bias=sk.to(DEV) if sink else None, scale=s.scale,
                                        cache_chunk_size=C)
    torch.cuda.synchronize()
    _check_rows(s, x, o, lse, Tq, sink=sk, what=f"K={K} C={C}")


def test_chunk_ignores_cache_past_T_kv():
    """A cache of larger capacity whose positions past T_kv hold NaN: the
    tensor-core path reads keys and values through maps that end at T_kv,
    the split path never reads past T_kv; neither output may see them."""
    s = I.spec(5, B=2, T=300, HQ=8, H=2)
    Tq = 37
    x = _inputs(s, Tq)
    P, kt, rc, vc = _cache(s, x, Tcap=450, fill_nan=True)
    for chunk_c, what in ((s.chunk, "tensor cores"), (48, "split")):
        if chunk_c != s.chunk:  # rebuild with a chunk size outside the tensor-core domain
            kt, rc = api.build_wall_kv_cache(x["k"].to(DEV), P, chunk_size=chunk_c, capacity=450)
            kt[:, s.T:] = float("nan")
        o, lse = api.wall_attn_decode_chunk(x["q"].to(DEV), vc, P[:, s.T - Tq:], kt, rc,
                                            scale=s.scale, cache_chunk_size=chunk_c, T_kv=s.T)
        torch.cuda.synchronize()
        assert bool(torch.isfinite(o.float()).all()), what
        _check_rows(s, x, o, lse, Tq, what=what)


@pytest.mark.parametrize("dtype,K,V,C", [
    (torch.float32, 64, 64, 64),    # fp32: split path, 1e-5
    (torch.bfloat16, 128, 64, 64),  # K != V: split path
    (torch.bfloat16, 128, 128, 48),  # chunk outside the tensor-core domain
])
def test_chunk_split_path(dtype, K, V, C):
    s = I.spec(5, B=2, T=333, HQ=4, H=2, K=K, V=V, chunk=C, dtype=dtype)
    Tq = 7
    x = _inputs(s, Tq)
    sk = _sink(s.HQ, seed=5)
    P, kt, rc, vc = _cache(s, x, Tcap=s.T)
    o, lse = api.wall_attn_decode_chunk(x["q"].to(DEV), vc, P[:, s.T - Tq:], kt, rc,
                                        sink_bias=sk.to(DEV), scale=s.scale, cache_chunk_size=C)
    torch.cuda.synchronize()
    _check_rows(s, x, o, lse, Tq, sink=sk, what=f"{dtype} K={K} V={V} C={C}")


def test_chunk_one_row_equals_decode():
    """Tq = 1 is one decode step: the split path gives wall_attn_decode's
    result, the tensor-core path agrees with it to bf16 rounding."""
    s = I.spec(5, B=2, T=1000, HQ=8, H=2)
    x = _inputs(s, 1)
    P, kt, rc, vc = _cache(s, x, Tcap=s.T)
    q, p = x["q"].to(DEV), P[:, -1:].contiguous()
    o_d, l_d = api.wall_attn_decode(q, vc, p, kt, rc, scale=s.scale, cache_chunk_size=s.chunk)
    o_c, l_c = api.wall_attn_decode_chunk(q, vc, p, kt, rc, scale=s.scale,
                                          cache_chunk_size=s.chunk)
    torch.cuda.synchronize()
    assert_fwd(s.dtype, o_c, o_d, l_c, l_d, what="chunk vs decode")


def test_chunked_prefill_through_the_cache():
    """A sequence prefilled in uneven chunks (crossing cache-chunk starts, one
    single token among them) with WallDecodeCache.extend: prefix carry,
    cache append and chunk attention together reproduce every forward row."""
    s = I.spec(5, B=2, T=1000, HQ=8, H=2)
    x = _inputs(s, s.T)
    k, v, g, q = (x[n].to(DEV) for n in ("k", "v", "g", "q"))
    cache = api.WallDecodeCache(s.B, s.H, s.HQ, s.K, s.V, capacity=1024, chunk_size=s.chunk,
                                dtype=s.dtype, device=DEV, scale=s.scale)
    outs, lses = [], []
    t = 0
    for n in (300, 1, 199, 500):
        o, lse = cache.extend(q[:, t:t + n], k[:, t:t + n], v[:, t:t + n], g[:, t:t + n])
        outs.append(o)
        lses.append(lse)
        t += n
    torch.cuda.synchronize()
    o = torch.cat(outs, 1)
    lse = torch.cat(lses, 1)
    _check_rows(s, x, o, lse, s.T, what="chunked prefill")


def test_chunk_argument_checks():
    s = I.spec(5, B=1, T=64, HQ=2, H=1)
    x = _inputs(s, 8)
    P, kt, rc, vc = _cache(s, x, Tcap=s.T)
    q = x["q"].to(DEV)
    with pytest.raises(L.WallError):  # more queries than cached positions
        o = torch.empty((1, 8, 2, 128), dtype=s.dtype, device=DEV)
        L.wall_attn_decode_chunk(q, vc, P[:, -8:].contiguous(), kt, rc, None, s.scale, 64, 1, 8,
                                 4, s.T, 1, 2, 128, 128, o, None,
                                 torch.empty(1 << 20, dtype=torch.uint8, device=DEV))
    with pytest.raises(L.WallError):  # workspace too small
        o = torch.empty((1, 8, 2, 128), dtype=s.dtype, device=DEV)
        L.wall_attn_decode_chunk(q, vc, P[:, -8:].contiguous(), kt, rc, None, s.scale, 64, 1, 8,
                                 s.T, s.T, 1, 2, 128, 128, o, None,
                                 torch.empty(16, dtype=torch.uint8, device=DEV))


@pytest.mark.slow
def test_chunk_full_size_sampled():
    """The decode workload at full size (B=32, T_kv=32768, HQ=32, H=8,
    K=V=128, C=64) with its last 64 positions as one chunk, in the launch
    configuration of the benchmark; sampled batch rows against the oracle."""
    s = I.spec(5)
    Tq = 64
    d = I.decode_inputs(s, device=DEV, n_query_rows=Tq)
    P = api.prefix_cumsum(d["g"])
    kt, rc = api.build_wall_kv_cache(d["k"], P, chunk_size=s.chunk)
    p_tail = P[:, s.T - Tq:].contiguous()
    del P
    o, lse = api.wall_attn_decode_chunk(d["q_tail"], d["v"], p_tail, kt, rc, scale=s.scale,
                                        cache_chunk_size=s.chunk)
    torch.cuda.synchronize()
    assert L.wall_get_status() == L.WALL_OK
    del kt, rc
    assert bool(torch.isfinite(o.float()).all())
    for b in (0, 31):
        o_ref, l_ref = wo.forward(d["q_tail"][b:b + 1].cpu(), d["k"][b:b + 1].cpu(),
                                  d["v"][b:b + 1].cpu(), d["g"][b:b + 1].cpu(), scale=s.scale,
                                  rows=(s.T - Tq, s.T), q_rows_only=True)
        assert np.isfinite(o_ref[0, s.T - Tq:]).all()
        assert_fwd(s.dtype, o[b], o_ref[0, s.T - Tq:], lse[b], l_ref[0, s.T - Tq:],
                   what=f"b={b}")
