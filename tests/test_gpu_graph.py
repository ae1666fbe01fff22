"""The training step captured in a CUDA graph (api.WallAttnStepGraph)
replays exactly the direct calls: the same kernels on the same inputs give
the same bits, both on the inputs it was captured with and on new inputs
copied in before a replay."""
import pytest
import torch

from channel_decay_softmax_b200 import _lib as L
from channel_decay_softmax_b200 import api
from channel_decay_softmax_b200 import inputs as I
from tests.test_gpu_training import _to

pytestmark = pytest.mark.gpu


def _direct(x, s, kw, want_dsink):
    o, lse, P, fws = api.wall_attn_fwd_gate(x["q"], x["k"], x["v"], x["g"], s.scale,
                                            return_workspace=True, **kw)
    dq, dk, dv, dg, dgs, dsink = api.wall_attn_bwd(x["dO"], x["q"], x["k"], x["v"], P, o, lse,
                                                   s.scale, want_dsink=want_dsink,
                                                   fwd_workspace=fws, **kw)
    torch.cuda.synchronize()
    return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv, dg=dg, dg_scalar=dgs, dsink=dsink)


def _same(got, want, what):
    for n, w in want.items():
        if w is None:
            assert got[n] is None, (what, n)
        else:  # every output, dsink included, is summed in a fixed order
            assert torch.equal(got[n], w), (what, n)


@pytest.mark.parametrize("case", ["cfg2", "varlen_options"])
def test_step_graph_replays_the_direct_calls(case):
    if case == "cfg2":
        s = I.spec(2)
    else:
        s = I.spec(4, len_lo=64, len_hi=600, window=128)
    x = _to(I.training_inputs(s))
    kw = dict(g_scalar=x["g_scalar"], sink_bias=x["sink_bias"], window_size=x["window_size"],
              cu_seqlens=x["cu_seqlens"])
    want_dsink = x["sink_bias"] is not None
    G = api.WallAttnStepGraph(x["q"], x["k"], x["v"], x["g"], x["dO"], s.scale,
                              want_dsink=want_dsink, **kw)
    out = G.replay()
    torch.cuda.synchronize()
    _same(out, _direct(x, s, kw, want_dsink), f"{case} capture inputs")
    # other inputs of the same shapes, copied in before the replay
    y = _to(I.training_inputs(I.spec(2, seed=5) if case == "cfg2"
                              else I.spec(4, len_lo=64, len_hi=600, window=128, seed=5)))
    out = G.replay(q=y["q"], k=y["k"], v=y["v"], g=y["g"], dO=y["dO"])
    torch.cuda.synchronize()
    y.update(cu_seqlens=x["cu_seqlens"])
    _same(out, _direct(y, s, kw, want_dsink), f"{case} new inputs")
    assert L.wall_get_status() == L.WALL_OK
