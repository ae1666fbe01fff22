"""GPU parity of the training path on degenerate shapes: GQA groups of one
and of every query head, a sequence of exactly one 128-row tile and ones a
row short of or past it, an odd batch, and a window of one key, where
attention reduces to copying the row's own value (the only visible key gets
weight 1, so o = v and the score gradients vanish)."""
import pytest
import torch

from channel_decay_softmax_b200 import api
from channel_decay_softmax_b200 import inputs as I
from tests.test_gpu_training import _check_all, _to

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,T,HQ,H,K", [
    (1, 128, 2, 2, 128),   # G = 1, exactly one tile
    (1, 129, 16, 1, 64),   # G = 16 (every query head on one kv head), ragged second tile
    (3, 127, 4, 1, 64),    # odd batch, one row short of a tile
    (2, 256, 4, 4, 64),    # G = 1, two whole tiles (stored dS tiles J <= I)
], ids=["G1_T128", "G16_T129", "B3_T127", "G1_T256"])
def test_gqa_and_tile_boundaries(B, T, HQ, H, K):
    s = I.spec(2, B=B, T=T, HQ=HQ, H=H, K=K, V=K)
    _check_all(s, I.training_inputs(s), what=f"B={B} T={T} HQ={HQ} H={H} K={K}")


@pytest.mark.parametrize("K", [64, 128])
def test_window_of_one_key_copies_the_value(K):
    s = I.spec(2, T=300, K=K, V=K, window=1)
    x_cpu = I.training_inputs(s)
    _check_all(s, x_cpu, what=f"window 1 K={K}")
    x = _to(x_cpu)
    P = api.prefix_cumsum(x["g"])
    o, _ = api.wall_attn_fwd(x["q"], x["k"], x["v"], P, s.scale, window_size=1)
    torch.cuda.synchronize()
    v_rep = x["v"].repeat_interleave(s.G, dim=2).float()
    # o is v up to the final rounding of a weight within one ulp of 1
    assert bool(((o.float() - v_rep).abs() <= 2.0 ** -8 * v_rep.abs()).all())
