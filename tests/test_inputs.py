"""The seeded synthetic inputs (the recipe the design notes state): shapes,
dtypes and value distributions of every configuration, determinism under a
seed, the varlen length mix, and the per-batch-row decode generator."""
import math

import pytest
import torch

from channel_decay_softmax_b200 import inputs as I


def test_configs_match_the_stated_workloads():
    want = {1: (1, 256, 2, 1, 64, 64, torch.float32), 2: (2, 1024, 8, 4, 64, 64, torch.bfloat16),
            3: (1, 8192, 16, 4, 128, 128, torch.bfloat16),
            5: (32, 32768, 32, 8, 128, 128, torch.bfloat16)}
    for cfg, (B, T, HQ, H, K, V, dt) in want.items():
        s = I.spec(cfg)
        assert (s.B, s.T, s.HQ, s.H, s.K, s.V, s.dtype) == (B, T, HQ, H, K, V, dt), cfg
        assert s.seed == 1000 + cfg
    s4 = I.spec(4)
    assert (s4.n_seq, s4.len_lo, s4.len_hi, s4.window, s4.g_scalar, s4.sink) == \
        (8, 512, 4096, 1024, True, True)
    assert I.spec(5).chunk == 64


def test_training_inputs_shapes_dtypes_and_determinism():
    s = I.spec(2, T=96)
    a, b = I.training_inputs(s), I.training_inputs(s)
    for n in ("q", "k", "v", "g", "dO"):
        assert torch.equal(a[n], b[n]), n
        assert a[n].dtype == s.dtype
    assert a["q"].shape == (2, 96, 8, 64) and a["k"].shape == (2, 96, 4, 64)
    assert a["g"].shape == a["q"].shape and a["dO"].shape == (2, 96, 8, 64)
    c = I.training_inputs(I.spec(2, T=96, seed=7))
    assert not torch.equal(a["q"], c["q"])


def test_gate_distributions():
    # config 3: decaying gate g = -0.05 |N(0,1)|
    g = I.training_inputs(I.spec(3, T=2048))["g"].float()
    assert float(g.max()) <= 0.0
    mean = 0.05 * math.sqrt(2 / math.pi)
    assert abs(float(g.mean()) + mean) < 0.02 * mean
    # config 2: g = 0.02 N(0,1), both signs
    g2 = I.training_inputs(I.spec(2))["g"].float()
    assert abs(float(g2.std()) - 0.02) < 0.001 and float(g2.min()) < 0 < float(g2.max())


def test_varlen_mix_and_options():
    s = I.spec(4)
    lengths = I.varlen_lengths(s)
    assert len(lengths) == 8 and all(512 <= n <= 4096 for n in lengths)
    assert lengths == I.varlen_lengths(I.spec(4, seed=99))  # lengths have their own seed
    x = I.training_inputs(I.spec(4, len_lo=5, len_hi=40))
    cu = x["cu_seqlens"]
    assert cu.dtype == torch.int32 and int(cu[0]) == 0 and int(cu[-1]) == x["T"]
    assert bool((cu[1:] >= cu[:-1]).all())
    assert x["g_scalar"].dtype == torch.float32 and x["g_scalar"].shape == (1, x["T"], 16)
    assert float(x["g_scalar"].max()) < 0.0           # logsigmoid
    assert x["sink_bias"].shape == (16,) and x["window_size"] == 1024


def test_decode_rows_regenerate_alone():
    s = I.spec(5, B=3, T=200)
    d = I.decode_inputs(s, n_query_rows=4)
    assert d["k"].shape == (3, 200, 8, 128) and d["q_tail"].shape == (3, 4, 32, 128)
    one = I.decode_batch_inputs(s, 2, n_query_rows=4)
    for n, m in (("k", "k"), ("v", "v"), ("g", "g"), ("q", "q_tail")):
        assert torch.equal(one[n], d[m][2]), n
    assert float(d["g"].float().max()) <= 0.0          # g = -0.02 |N|


@pytest.mark.parametrize("T,W", [(10, 0), (10, 3), (4, 10), (1, 1), (0, 5), (300, 128)])
def test_causal_pair_counts(T, W):
    # brute force over (i, j): visible iff j <= i and (no window or i - j < W)
    want = sum(1 for i in range(T) for j in range(i + 1) if W <= 0 or i - j < W)
    assert I.causal_pairs(T, W) == want
