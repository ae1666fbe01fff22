"""The decode entry point that allocates nothing (wall_attn_decode_noalloc).

Callers that cannot allocate device memory -- code running under CUDA graph
capture that must not allocate, serving loops with memory planned up front,
bindings without a device allocator -- get the same decode with its split
partials in a fixed scratch array inside the library.  This file is collected
last so a failure here leaves every other test already run.
"""
import pytest
import torch

from channel_decay_softmax_b200 import _lib as L
from channel_decay_softmax_b200 import api
from channel_decay_softmax_b200 import inputs as I
from oracle import wall_oracle as wo
from tests.helpers import assert_fwd


def _cache(s, T, dev="cuda"):
    xs = [I.decode_batch_inputs(s, b, device="cpu", n_query_rows=1) for b in range(s.B)]
    k = torch.stack([x["k"][:T] for x in xs])
    v = torch.stack([x["v"][:T] for x in xs])
    g = torch.stack([x["g"][:T] for x in xs])
    q = torch.stack([x["q"] for x in xs])
    P = api.prefix_cumsum(g.to(dev))
    kt, rc = api.build_wall_kv_cache(k.to(dev), P, chunk_size=s.chunk)
    host = dict(q=q, k=k, v=v, g=g)
    return q.to(dev), v.to(dev), P[:, -1:].contiguous(), kt, rc, host


def _two_calls(s):
    """Two calls in a row with different lengths (so different split
    counts): each must equal wall_attn_decode on the same cache and the fp64
    oracle's forward row at the last position."""
    for T in (s.T, s.T - 300):
        q, v, pc, kt, rc, host = _cache(s, T)
        o_ref, lse_ref = api.wall_attn_decode(q, v, pc, kt, rc, scale=s.scale,
                                              cache_chunk_size=s.chunk)
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        L.wall_attn_decode_noalloc(q, v, pc, kt, rc, None, s.scale, s.chunk, s.B, T, T, s.H,
                                   s.HQ, s.K, s.V, o, lse)
        torch.cuda.synchronize()
        assert_fwd(s.dtype, o, o_ref, lse, lse_ref, what=f"noalloc vs decode T={T}")
        for b in range(s.B):
            o_or, l_or = wo.forward(host["q"][b:b + 1], host["k"][b:b + 1], host["v"][b:b + 1],
                                    host["g"][b:b + 1], scale=s.scale, rows=(T - 1, T),
                                    q_rows_only=True)
            assert_fwd(s.dtype, o[b, 0], o_or[0, -1], lse[b, 0], l_or[0, -1],
                       what=f"noalloc vs oracle T={T} b={b}")
    assert L.wall_get_status() == L.WALL_OK


@pytest.mark.gpu
def test_noalloc_decode_matches_decode_on_two_calls_in_a_row():
    """bf16, K = V = 128, C = 64: the persistent TMA decode kernel."""
    _two_calls(I.spec(5, B=2, T=1000, HQ=8, H=2))


@pytest.mark.gpu
def test_noalloc_decode_split_kernel_fp32():
    """fp32 with a chunk of 48 (not a multiple of 32): the general split
    kernel writes its partials into the fixed scratch."""
    _two_calls(I.spec(5, B=2, T=1000, HQ=8, H=2, dtype=torch.float32, chunk=48))


def test_noalloc_rejects_problems_beyond_its_scratch():
    # B * HQ * splits * (V + 2) floats must fit in 2^20; this needs far more
    # (checked on the host before any CUDA call)
    FAKE = 4096
    rc = L.lib().wall_attn_decode_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, 0.0, 64, 0, 4096,
                                          65536, 65536, 32, 32, 128, 128, FAKE, FAKE, None)
    assert rc == L.WALL_ERR_UNSUPPORTED
