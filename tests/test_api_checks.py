"""CPU tests of the Python API's argument checks.  The library takes bare
pointers, so a tensor of the wrong dtype or shape must be refused before any
call into it; the well-formed calls below get past every check and stop only
at the binding's refusal of host tensors (no GPU here)."""
import pytest
import torch

from channel_decay_softmax_b200 import api

BF, F32 = torch.bfloat16, torch.float32
B, T, HQ, H, K, V = 2, 40, 4, 2, 64, 64
HOST = "libwall takes CUDA tensors"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from channel_decay_softmax_b200 import build
    build.build()


def _train(dtype=BF):
    return dict(q=torch.zeros(B, T, HQ, K, dtype=dtype), k=torch.zeros(B, T, H, K, dtype=dtype),
                v=torch.zeros(B, T, H, V, dtype=dtype), g=torch.zeros(B, T, HQ, K, dtype=dtype),
                P=torch.zeros(B, T, HQ, K, dtype=F32), dO=torch.zeros(B, T, HQ, V, dtype=dtype),
                o=torch.zeros(B, T, HQ, V, dtype=dtype), lse=torch.zeros(B, T, HQ, dtype=F32))


def _passes_checks(fn, *a, **kw):
    with pytest.raises(ValueError, match=HOST):
        fn(*a, **kw)


def test_well_formed_training_calls_pass_the_checks():
    x = _train()
    _passes_checks(api.prefix_cumsum, x["g"], carry_in=torch.zeros(B, HQ, K))
    _passes_checks(api.wall_attn_fwd, x["q"], x["k"], x["v"], x["P"],
                   g_scalar=torch.zeros(B, T, HQ, dtype=BF), sink_bias=torch.zeros(HQ))
    _passes_checks(api.wall_attn_fwd_gate, x["q"], x["k"], x["v"], x["g"])
    _passes_checks(api.wall_attn_bwd, x["dO"], x["q"], x["k"], x["v"], x["P"], x["o"],
                   x["lse"], g_scalar=torch.zeros(B, T, HQ))
    # an expanded upstream gradient (o.sum().backward()) has o's shape
    _passes_checks(api.wall_attn_bwd, torch.ones(1, dtype=BF).expand(B, T, HQ, V), x["q"],
                   x["k"], x["v"], x["P"], x["o"], x["lse"])
    cu = torch.tensor([0, 10, T], dtype=torch.int32)
    y = {n: t[:1] for n, t in x.items()}
    _passes_checks(api.prefix_cumsum, y["g"], cu, torch.zeros(2, HQ, K))
    _passes_checks(api.wall_attn_fwd, y["q"], y["k"], y["v"], y["P"], cu_seqlens=cu)


@pytest.mark.parametrize("case", ["P_bf16", "k_fp32", "g_fp32", "lse_bf16", "o_shape", "dO_dtype",
                                  "g_scalar_shape", "sink_shape", "cu_2d", "carry_shape",
                                  "fp16"])
def test_training_calls_refuse_bad_tensors(case):
    x = _train()
    q, k, v, g, P, dO, o, lse = (x[n] for n in ("q", "k", "v", "g", "P", "dO", "o", "lse"))
    if case == "P_bf16":
        call = lambda: api.wall_attn_fwd(q, k, v, P.to(BF))
    elif case == "k_fp32":
        call = lambda: api.wall_attn_fwd(q, k.float(), v, P)
    elif case == "g_fp32":
        call = lambda: api.wall_attn_fwd_gate(q, k, v, g.float())
    elif case == "lse_bf16":
        call = lambda: api.wall_attn_bwd(dO, q, k, v, P, o, lse.to(BF))
    elif case == "o_shape":
        call = lambda: api.wall_attn_bwd(dO, q, k, v, P, o[:, :-1], lse)
    elif case == "dO_dtype":
        call = lambda: api.wall_attn_bwd(dO.float(), q, k, v, P, o, lse)
    elif case == "g_scalar_shape":
        call = lambda: api.wall_attn_fwd(q, k, v, P, g_scalar=torch.zeros(B, T, HQ, 1))
    elif case == "sink_shape":
        call = lambda: api.wall_attn_fwd(q, k, v, P, sink_bias=torch.zeros(HQ + 1))
    elif case == "cu_2d":
        call = lambda: api.wall_attn_fwd(q[:1], k[:1], v[:1], P[:1],
                                         cu_seqlens=torch.zeros(1, 3, dtype=torch.int32))
    elif case == "carry_shape":
        call = lambda: api.prefix_cumsum(g, carry_in=torch.zeros(B + 1, HQ, K))
    else:
        call = lambda: api.prefix_cumsum(g.half())
    with pytest.raises((TypeError, ValueError)) as e:
        call()
    assert HOST not in str(e.value)


def test_backward_refuses_a_smaller_forward_workspace():
    x = _train()
    small = torch.empty(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="fwd_workspace"):
        api.wall_attn_bwd(x["dO"], x["q"], x["k"], x["v"], x["P"], x["o"], x["lse"],
                          fwd_workspace=small)


def _cache(C=16, Tcap=T, dtype=BF):
    k_tilde = torch.zeros(B, Tcap, HQ, K, dtype=dtype)
    v = torch.zeros(B, Tcap, H, V, dtype=dtype)
    r_cache = torch.zeros(B, -(-Tcap // C), HQ, K, dtype=F32)
    return k_tilde, v, r_cache


def test_well_formed_decode_calls_pass_the_checks():
    kt, v, rc = _cache()
    q1 = torch.zeros(B, 1, HQ, K, dtype=BF)
    p1 = torch.zeros(B, 1, HQ, K)
    _passes_checks(api.build_wall_kv_cache, torch.zeros(B, T, H, K, dtype=BF),
                   torch.zeros(B, T, HQ, K), chunk_size=16, capacity=T + 8)
    _passes_checks(api.wall_attn_decode, q1, v, p1, kt, rc, cache_chunk_size=16)
    _passes_checks(api.wall_attn_decode, q1, v, p1, kt, rc, sink_bias=torch.zeros(HQ),
                   cache_chunk_size=16, T_kv=5)
    qc = torch.zeros(B, 7, HQ, K, dtype=BF)
    _passes_checks(api.wall_attn_decode_chunk, qc, v, torch.zeros(B, 7, HQ, K), kt, rc,
                   cache_chunk_size=16, T_kv=30)


@pytest.mark.parametrize("case", ["r_cache_other_chunk", "p_bf16", "q_rows", "v_capacity",
                                  "T_kv_beyond", "Tq_beyond_T_kv", "q_dtype", "P_cache_shape",
                                  "capacity_short"])
def test_decode_calls_refuse_bad_tensors(case):
    kt, v, rc = _cache()
    q1 = torch.zeros(B, 1, HQ, K, dtype=BF)
    p1 = torch.zeros(B, 1, HQ, K)
    if case == "r_cache_other_chunk":  # built with chunks of 16, decoded with 8
        call = lambda: api.wall_attn_decode(q1, v, p1, kt, rc, cache_chunk_size=8)
    elif case == "p_bf16":
        call = lambda: api.wall_attn_decode(q1, v, p1.to(BF), kt, rc, cache_chunk_size=16)
    elif case == "q_rows":
        call = lambda: api.wall_attn_decode(torch.zeros(B, 2, HQ, K, dtype=BF), v, p1, kt, rc,
                                            cache_chunk_size=16)
    elif case == "v_capacity":
        call = lambda: api.wall_attn_decode(q1, v[:, :-1], p1, kt, rc, cache_chunk_size=16)
    elif case == "T_kv_beyond":
        call = lambda: api.wall_attn_decode(q1, v, p1, kt, rc, cache_chunk_size=16, T_kv=T + 1)
    elif case == "Tq_beyond_T_kv":
        call = lambda: api.wall_attn_decode_chunk(torch.zeros(B, 9, HQ, K, dtype=BF), v,
                                                  torch.zeros(B, 9, HQ, K), kt, rc,
                                                  cache_chunk_size=16, T_kv=8)
    elif case == "q_dtype":
        call = lambda: api.wall_attn_decode(q1.float(), v, p1, kt, rc, cache_chunk_size=16)
    elif case == "P_cache_shape":
        call = lambda: api.build_wall_kv_cache(torch.zeros(B, T, H, K, dtype=BF),
                                               torch.zeros(B, T - 1, HQ, K), chunk_size=16)
    else:
        call = lambda: api.build_wall_kv_cache(torch.zeros(B, T, H, K, dtype=BF),
                                               torch.zeros(B, T, HQ, K), chunk_size=16,
                                               capacity=T - 1)
    with pytest.raises((TypeError, ValueError)) as e:
        call()
    assert HOST not in str(e.value)


def test_decode_cache_checks_new_tokens():
    cache = api.WallDecodeCache(B, H, HQ, K, V, capacity=64, chunk_size=32, device="cpu")
    k = torch.zeros(B, 3, H, K, dtype=BF)
    v = torch.zeros(B, 3, H, V, dtype=BF)
    g = torch.zeros(B, 3, HQ, K, dtype=BF)
    q = torch.zeros(B, 3, HQ, K, dtype=BF)
    _passes_checks(cache.append, k, v, g)
    _passes_checks(cache.extend, q, k, v, g)
    _passes_checks(cache.step, q[:, :1], k[:, :1], v[:, :1], g[:, :1])
    bad = [
        lambda: cache.append(k.float(), v, g),                   # dtype other than the cache's
        lambda: cache.append(k, v[:, :2], g),                    # token counts disagree
        lambda: cache.append(k[:1], v[:1], g[:1]),               # batch other than the cache's
        lambda: cache.extend(q[..., :32], k, v, g),              # head size
        lambda: cache.step(q, k, v, g),                          # three tokens in one step
        lambda: cache.step(q[:, :1], k[:, :1], v[:, :1], g[:, :1, :2]),
    ]
    for call in bad:
        with pytest.raises((TypeError, ValueError)) as e:
            call()
        assert HOST not in str(e.value)
    assert cache.length == 0
    with pytest.raises(ValueError):
        api.WallDecodeCache(B, 3, HQ, K, V, capacity=64, device="cpu")  # HQ % H != 0
    with pytest.raises(ValueError):
        api.WallDecodeCache(B, H, HQ, K, V, capacity=64, device="cpu",
                            sink_bias=torch.zeros(HQ + 1))


def test_readme_call_pattern_passes_the_checks():
    """The calls exactly as the wall-attention-release README writes them
    ("Usage", "Decode": positional and keyword names, a non-leaf g, an
    expanded upstream gradient later) get through every check."""
    import channel_decay_softmax_b200 as wa
    B, T, H, HQ, K, V, C = 2, 64, 4, 8, 64, 64, 16
    q = torch.randn(B, T, HQ, K, dtype=BF, requires_grad=True)
    k = torch.randn(B, T, H, K, dtype=BF, requires_grad=True)
    v = torch.randn(B, T, H, V, dtype=BF, requires_grad=True)
    g = torch.randn(B, T, HQ, K, dtype=BF, requires_grad=True) * 0.02
    _passes_checks(wa.wall_attn, q, k, v, g, scale=K ** -0.5)
    P = torch.zeros(B, T, HQ, K)
    _passes_checks(wa.build_wall_kv_cache, k.detach(), P, chunk_size=C)
    k_tilde = torch.zeros(B, T, HQ, K, dtype=BF)
    r_cache = torch.zeros(B, T // C, HQ, K)
    _passes_checks(wa.wall_attn_decode, q=q.detach()[:, -1:], v=v.detach(), p_curr=P[:, -1:],
                   k_tilde=k_tilde, r_cache=r_cache, sink_bias=None, scale=K ** -0.5,
                   cache_chunk_size=C)


def test_timing_slots_by_name():
    api.timing_enable_slots(["bwd_keyblock", "fwd_tc"])
    api.timing_enable_slots([])
    with pytest.raises(ValueError, match="unknown stage 'bwd'"):
        api.timing_enable_slots(["bwd"])


def test_step_graph_replay_checks_new_inputs():
    """WallAttnStepGraph.replay copies new inputs into the graph's buffers
    only when they match them (the capture itself needs a GPU)."""
    g = object.__new__(api.WallAttnStepGraph)
    g.inputs = {"q": torch.zeros(1, 4, 2, 8, dtype=BF)}
    replays = []
    g.graph = type("G", (), {"replay": lambda self: replays.append(1)})()
    g.outputs = {"o": None}
    with pytest.raises(KeyError):
        g.replay(x=torch.zeros(1))
    with pytest.raises(ValueError):
        g.replay(q=torch.zeros(1, 5, 2, 8, dtype=BF))
    with pytest.raises(TypeError):
        g.replay(q=torch.zeros(1, 4, 2, 8))
    assert not replays
    assert g.replay(q=torch.ones(1, 4, 2, 8, dtype=BF)) == {"o": None}
    assert replays == [1] and float(g.inputs["q"].float().sum()) == 64.0
