"""Anchor invariance of the GPU path (Tilde blog "Wall Attention", fast
training section 1: the per-block anchor cancels between the query and key
operands, so the result does not depend on where it sits).

The kernels' anchors are R = floor(P at a 128-row block's first row) for the
training operands and the chunk-call queries, and R_c = P at a chunk's first
row for the decode cache.  Adding an integer c_n to every P of a channel
moves each of them by exactly c_n.  With P on a grid of 2^-10 (so that every
sum and difference below is exact in fp32), the anchored operands, the
per-tile factors 2^(R_I - R_J) and therefore every output must be bit for
bit the same, even for |c| near 1000, where 2^P itself lies far outside the
fp32 range: a kernel that formed 2^P or 2^-P anywhere would return inf, 0 or
NaN.  A fractional shift moves the floor's rounding points instead, so the
training outputs may then differ by bf16 rounding only; the decode cache,
whose anchor is P itself, stays bit-identical under any exact shift."""
import pytest
import torch

from channel_decay_softmax_b200 import api
from channel_decay_softmax_b200 import inputs as I
from tests.helpers import assert_fwd, assert_grad

pytestmark = pytest.mark.gpu

DEV = "cuda"
GRID = 1024.0     # P on multiples of 2^-10
FRAC = 0.6875     # 11/16: a fractional shift that keeps every sum exact


def _grid_prefix(g):
    P = api.prefix_cumsum(g)
    return torch.round(P * GRID) / GRID


def _shift(P, seed, frac=0.0):
    """P + c with c an integer in [-1000, 1000] (+ frac) per (batch row,
    head, channel); returns the shifted prefix and c."""
    gen = torch.Generator().manual_seed(seed)
    B, _, HQ, K = P.shape
    c = (torch.randint(-1000, 1001, (B, 1, HQ, K), generator=gen).float() + frac).to(P.device)
    Ps = P + c
    # the shift is exact: it is undone bit for bit
    assert torch.equal(Ps - c, P)
    return Ps, c


def _train(x, P, window):
    q, k, v = x["q"], x["k"], x["v"]
    o, lse = api.wall_attn_fwd(q, k, v, P, x["scale"], window_size=window)
    dq, dk, dv, dg, _, _ = api.wall_attn_bwd(x["dO"], q, k, v, P, o, lse, x["scale"],
                                             window_size=window)
    torch.cuda.synchronize()
    return o, lse, (dq, dk, dv, dg)


@pytest.mark.parametrize("K,window", [(64, 0), (128, 0), (64, 300)],
                         ids=["K64_stored_dS", "K128_stored_dS", "K64_window_recompute"])
def test_training_invariant_to_shift_of_P(K, window):
    s = I.spec(2, T=700, K=K, V=K)
    x = {n: (t.to(DEV) if isinstance(t, torch.Tensor) else t)
         for n, t in I.training_inputs(s).items()}
    P = _grid_prefix(x["g"])
    o, lse, grads = _train(x, P, window)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()

    Pi, _ = _shift(P, seed=11)
    assert float(Pi.abs().max()) > 900.0  # 2^P overflows fp32 here
    oi, lsei, gi = _train(x, Pi, window)
    assert torch.equal(oi, o) and torch.equal(lsei, lse)
    for name, a, b in zip(("dq", "dk", "dv", "dg"), gi, grads):
        assert torch.equal(a, b), f"integer shift changed {name}"

    Pf, _ = _shift(P, seed=12, frac=FRAC)
    of, lsef, gf = _train(x, Pf, window)
    assert_fwd(s.dtype, of, o, lsef, lse, None, "fractional shift")
    for name, a, b in zip(("dq", "dk", "dv", "dg"), gf, grads):
        assert_grad(s.dtype, name, a, b, None, "fractional shift")


def test_decode_cache_invariant_to_shift_of_P():
    s = I.spec(2, T=700)  # B=2 HQ=8 H=4 K=V=64, cache chunks of 64
    x = {n: (t.to(DEV) if isinstance(t, torch.Tensor) else t)
         for n, t in I.training_inputs(s).items()}
    q, k, v = x["q"], x["k"], x["v"]
    C, Tq = 64, 64
    P = _grid_prefix(x["g"])

    def run(PP):
        kt, rc = api.build_wall_kv_cache(k, PP, chunk_size=C)
        o1, l1 = api.wall_attn_decode(q[:, -1:], v, PP[:, -1:], kt, rc, scale=s.scale,
                                      cache_chunk_size=C)
        oc, lc = api.wall_attn_decode_chunk(q[:, -Tq:], v, PP[:, -Tq:], kt, rc, scale=s.scale,
                                            cache_chunk_size=C)
        torch.cuda.synchronize()
        return kt, rc, o1, l1, oc, lc

    kt, rc, o1, l1, oc, lc = run(P)
    assert torch.isfinite(o1.float()).all() and torch.isfinite(oc.float()).all()
    for frac in (0.0, FRAC):
        Ps, c = _shift(P, seed=13, frac=frac)
        kts, rcs, o1s, l1s, ocs, lcs = run(Ps)
        what = f"shift + {frac}"
        # the cache anchor is P itself: k_tilde and the one-row decode are
        # unchanged by any exact shift, r_cache moves with it
        assert torch.equal(kts, kt), what
        assert torch.equal(rcs - c, rc), what
        assert torch.equal(o1s, o1) and torch.equal(l1s, l1), what
        # the chunk's query blocks use floor anchors: bit-identical under an
        # integer shift, equal to bf16 rounding under a fractional one
        if frac == 0.0:
            assert torch.equal(ocs, oc) and torch.equal(lcs, lc), what
        else:
            assert_fwd(s.dtype, ocs, oc, lcs, lc, None, what)
