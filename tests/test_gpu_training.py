"""GPU parity of the training path (prefix scan, forward, backward) against
the fp64 oracle, through the C ABI, on the pages' workload configurations."""
import numpy as np
import pytest
import torch

from channel_decay_softmax_b200 import api
from channel_decay_softmax_b200 import inputs as I
from oracle import wall_oracle as wo
from tests.helpers import assert_fwd, assert_grad, max_abs, np64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _to(x, dev=DEV):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _run_gpu(x, want_dsink=False):
    q, k, v, g = x["q"], x["k"], x["v"], x["g"]
    cu = x["cu_seqlens"]
    P = api.prefix_cumsum(g, cu)
    o, lse = api.wall_attn_fwd(q, k, v, P, x["scale"], x["g_scalar"], x["sink_bias"],
                               x["window_size"], cu)
    grads = api.wall_attn_bwd(x["dO"], q, k, v, P, o, lse, x["scale"], x["g_scalar"],
                              x["sink_bias"], x["window_size"], cu, want_dsink=want_dsink)
    torch.cuda.synchronize()
    return P, o, lse, grads


def _oracle_kw(x):
    return dict(scale=x["scale"], g_scalar=x["g_scalar"], sink_bias=x["sink_bias"],
                window_size=x["window_size"],
                cu_seqlens=None if x["cu_seqlens"] is None else x["cu_seqlens"].cpu().numpy())


def _check_all(s, x_cpu, units=None, what=""):
    x = _to(x_cpu)
    want_dsink = x["sink_bias"] is not None
    P, o, lse, (dq, dk, dv, dg, dgs, dsink) = _run_gpu(x, want_dsink)
    ref = wo.backward(x_cpu["q"], x_cpu["k"], x_cpu["v"], x_cpu["g"], x_cpu["dO"],
                      units=units, **_oracle_kw(x_cpu))
    mask = None
    kmask = None
    if units is not None:
        heads = sorted({u % s.HQ for u in units})
        mask = np.zeros(o.shape[:3], dtype=bool)
        mask[:, :, heads] = True
        kvh = sorted({h // s.G for h in heads})
        kmask = np.zeros(dk.shape[:3], dtype=bool)
        kmask[:, :, kvh] = True
    assert_fwd(s.dtype, o, ref["o"], lse, ref["lse"], mask, what)
    assert_grad(s.dtype, "dq", dq, ref["dq"], mask, what)
    assert_grad(s.dtype, "dk", dk, ref["dk"], kmask, what)
    assert_grad(s.dtype, "dv", dv, ref["dv"], kmask, what)
    assert_grad(s.dtype, "dg", dg, ref["dg"], mask, what)
    if dgs is not None:
        assert_grad(s.dtype, "dg_scalar", dgs, ref["dg_scalar"], mask, what,
                    relative_to_max=True)
    if dsink is not None and units is None:
        assert_grad(s.dtype, "dsink", dsink, ref["dsink"], None, what, relative_to_max=True)
    return P


def test_prefix_cumsum_matches_oracle():
    for cfg in (1, 2, 3):
        s = I.spec(cfg)
        x = I.training_inputs(s)
        P = api.prefix_cumsum(x["g"].to(DEV))
        ref = wo.prefix_log2(x["g"])
        err = max_abs(P, ref) / max(1.0, float(np.abs(ref).max()))
        assert err < 2e-6, (cfg, err)


def test_prefix_cumsum_varlen_and_carry():
    s = I.spec(4, len_lo=1, len_hi=3000, n_seq=6, K=64)
    x = I.training_inputs(s, lengths=[1, 2999, 0, 2048, 7, 2049])
    cu = x["cu_seqlens"]
    carry = torch.randn((6, s.HQ, s.K), generator=torch.Generator().manual_seed(5))
    P, cout = api.prefix_cumsum(x["g"].to(DEV), cu.to(DEV), carry.to(DEV), return_carry=True)
    ref = wo.prefix_log2(x["g"], cu_seqlens=cu.numpy(), carry_in=carry)
    scale = max(1.0, float(np.abs(ref).max()))
    assert max_abs(P, ref) / scale < 2e-6
    # carry_out = last P of each sequence, carry_in for the empty one
    cu_np = cu.numpy()
    for i in range(6):
        a, b = cu_np[i], cu_np[i + 1]
        want = ref[0, b - 1] if b > a else carry[i].double().numpy()
        assert max_abs(cout[i], want) / scale < 2e-6


def test_prefix_streaming_equals_one_shot():
    """Scanning a sequence piece by piece with the carry gives the one-shot P."""
    s = I.spec(2)
    g = I.training_inputs(s)["g"].to(DEV)
    P_full = api.prefix_cumsum(g)
    carry = torch.zeros((s.B, s.HQ, s.K), device=DEV)
    parts = []
    for a, b in ((0, 1), (1, 300), (300, 301), (301, 1024)):
        P, carry = api.prefix_cumsum(g[:, a:b].contiguous(), carry_in=carry, return_carry=True)
        parts.append(P)
    assert max_abs(torch.cat(parts, 1), P_full) < 1e-4


def test_cfg1_tiny_fp32_full():
    """Config 1 (fp32, B=1 T=256 HQ=2 H=1 K=V=64): every output within 1e-5."""
    s = I.spec(1)
    _check_all(s, I.training_inputs(s), what="cfg1")


def test_cfg1_fp32_with_all_options():
    s = I.spec(4, dtype=torch.float32, K=64, V=64, HQ=4, H=2, window=100, len_lo=1,
               len_hi=300, n_seq=4)
    x = I.training_inputs(s, lengths=[1, 173, 64, 300])
    _check_all(s, x, what="fp32 options")


def test_cfg2_training_bf16_full():
    """Config 2 (bf16, B=2 T=1024 HQ=8 H=4 K=V=64), element by element."""
    s = I.spec(2)
    _check_all(s, I.training_inputs(s), what="cfg2")


def test_cfg3_long_context_reduced():
    """Config 3's shapes and gate with T=700: several tiles and a ragged tail."""
    s = I.spec(3, T=700)
    _check_all(s, I.training_inputs(s), what="cfg3/T=700")


@pytest.mark.slow
def test_cfg3_long_context_full_size_sampled():
    """Config 3 at T=8192 (|P| > 160): one GQA group (4 query heads) against
    the oracle, element by element."""
    s = I.spec(3)
    _check_all(s, I.training_inputs(s), units=[4, 5, 6, 7], what="cfg3 full")


def test_cfg4_varlen_options_reduced():
    """Config 4's options (varlen, g_scalar, sink, window) at reduced lengths."""
    s = I.spec(4, len_lo=64, len_hi=600, window=128)
    _check_all(s, I.training_inputs(s), what="cfg4 reduced")


@pytest.mark.slow
def test_cfg4_varlen_options_full_size_sampled():
    s = I.spec(4)
    x = I.training_inputs(s)
    nseq = s.n_seq
    units = [seq * s.HQ + h for seq in range(nseq) for h in (0, 1, 2, 3, 4, 5, 6, 7)]
    _check_all(s, x, units=units, what="cfg4 full")


def test_g_zero_matches_torch_sdpa():
    """g = 0 is plain causal attention: compare with torch's own kernel."""
    s = I.spec(2, T=300)
    x = _to(I.training_inputs(s))
    g0 = torch.zeros_like(x["g"])
    o = api.wall_attn(x["q"], x["k"], x["v"], g0, scale=s.scale)
    qt = x["q"].float().permute(0, 2, 1, 3)
    kt = x["k"].float().permute(0, 2, 1, 3).repeat_interleave(s.G, 1)
    vt = x["v"].float().permute(0, 2, 1, 3).repeat_interleave(s.G, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    assert max_abs(o, ref.permute(0, 2, 1, 3)) < 2e-2


def test_autograd_function_matches_direct_calls():
    s = I.spec(2, T=200)
    x = _to(I.training_inputs(s))
    q, k, v, g = (x[n].clone().requires_grad_(True) for n in ("q", "k", "v", "g"))
    o = api.wall_attn(q, k, v, g, scale=s.scale)
    o.backward(x["dO"])
    P, o2, lse, (dq, dk, dv, dg, _, _) = _run_gpu(x)
    assert torch.equal(o, o2)
    for a, b in ((q.grad, dq), (k.grad, dk), (v.grad, dv), (g.grad, dg)):
        assert torch.equal(a, b)


def test_empty_and_single_row():
    for T in (0, 1):
        s = I.spec(2, T=T, B=1)
        x = _to(I.training_inputs(s))
        P, o, lse, grads = _run_gpu(x)
        # the fused prefix forward (autograd path) on the same rows
        og, lg, Pg = api.wall_attn_fwd_gate(x["q"], x["k"], x["v"], x["g"], x["scale"])
        assert torch.equal(og, o) and torch.equal(Pg, P)
        assert o.shape == (1, T, s.HQ, s.V)
        if T == 1:
            # one visible key: o = v of the same row, dq = dk = dg = 0
            assert max_abs(o[0, 0], x["v"][0, 0].repeat_interleave(s.G, 0)) == 0.0
            assert float(grads[0].float().abs().max()) < 1e-5


def test_backward_reuses_forward_operands_bit_exactly():
    """wall_attn_bwd with the forward's workspace reads the anchored operands
    that call prepared instead of recomputing them: the same deterministic
    values, so every gradient must match the recomputing call bit for bit
    (config 2 shape, no sink: no atomics on the path)."""
    s = I.spec(2)
    x = _to(I.training_inputs(s))
    q, k, v = x["q"], x["k"], x["v"]
    P = api.prefix_cumsum(x["g"])
    o, lse, fws = api.wall_attn_fwd(q, k, v, P, x["scale"], return_workspace=True)
    a = api.wall_attn_bwd(x["dO"], q, k, v, P, o, lse, x["scale"])
    b = api.wall_attn_bwd(x["dO"], q, k, v, P, o, lse, x["scale"], fwd_workspace=fws)
    torch.cuda.synchronize()
    for name, ta, tb in zip(("dq", "dk", "dv", "dg"), a[:4], b[:4]):
        assert torch.equal(ta, tb), name


def test_backward_reuses_forward_operands_bit_exactly_with_options():
    """The same with every option (varlen, window, g_scalar, sink): given
    the forward's workspace, the backward also reads the forward's prefix of
    g_scalar instead of scanning it again, and dsink is a fixed-order sum, so
    all six gradients match the recomputing call bit for bit."""
    s = I.spec(4, len_lo=64, len_hi=600, window=128)
    x = _to(I.training_inputs(s))
    q, k, v, g = x["q"], x["k"], x["v"], x["g"]
    kw = dict(g_scalar=x["g_scalar"], sink_bias=x["sink_bias"], window_size=x["window_size"],
              cu_seqlens=x["cu_seqlens"])
    o, lse, P, fws = api.wall_attn_fwd_gate(q, k, v, g, x["scale"], return_workspace=True, **kw)
    a = api.wall_attn_bwd(x["dO"], q, k, v, P, o, lse, x["scale"], want_dsink=True, **kw)
    b = api.wall_attn_bwd(x["dO"], q, k, v, P, o, lse, x["scale"], fwd_workspace=fws,
                          want_dsink=True, **kw)
    torch.cuda.synchronize()
    for name, ta, tb in zip(("dq", "dk", "dv", "dg", "dg_scalar", "dsink"), a, b):
        assert ta is not None and tb is not None, name
        assert torch.equal(ta, tb), name


@pytest.mark.parametrize("case", ["cfg3_block", "options"])
def test_repeated_calls_bit_identical(case):
    """Two identical forward + backward calls give identical bits in every
    output, dsink and dg_scalar included: the library has no float atomics
    and fixes every summation order."""
    if case == "cfg3_block":
        s = I.spec(3, T=1024)
    else:
        s = I.spec(4, len_lo=64, len_hi=600, window=128)
    x = _to(I.training_inputs(s))
    q, k, v, g = x["q"], x["k"], x["v"], x["g"]
    kw = dict(g_scalar=x["g_scalar"], sink_bias=x["sink_bias"], window_size=x["window_size"],
              cu_seqlens=x["cu_seqlens"])
    want_dsink = x["sink_bias"] is not None
    runs = []
    for _ in range(2):
        o, lse, P, fws = api.wall_attn_fwd_gate(q, k, v, g, x["scale"], return_workspace=True,
                                                **kw)
        grads = api.wall_attn_bwd(x["dO"], q, k, v, P, o, lse, x["scale"], fwd_workspace=fws,
                                  want_dsink=want_dsink, **kw)
        runs.append((o, lse, P) + tuple(grads))
    torch.cuda.synchronize()
    names = ("o", "lse", "P", "dq", "dk", "dv", "dg", "dg_scalar", "dsink")
    for name, a, b in zip(names, runs[0], runs[1]):
        if a is None:
            assert b is None, name
            continue
        assert torch.equal(a, b), name


def _run_gpu_recompute(x):
    """_run_gpu with the smaller backward workspace: no dS tiles, so the dq
    pass recomputes S, P, dP and dS"""
    q, k, v, g = x["q"], x["k"], x["v"], x["g"]
    cu = x["cu_seqlens"]
    P = api.prefix_cumsum(g, cu)
    o, lse = api.wall_attn_fwd(q, k, v, P, x["scale"], x["g_scalar"], x["sink_bias"],
                               x["window_size"], cu)
    grads = api.wall_attn_bwd(x["dO"], q, k, v, P, o, lse, x["scale"], x["g_scalar"],
                              x["sink_bias"], x["window_size"], cu, store_ds=False)
    torch.cuda.synchronize()
    return P, o, lse, grads


@pytest.mark.parametrize("case", ["dense_K64", "dense_K128", "varlen_window_K128"])
def test_dq_from_stored_ds_matches_recompute(case):
    """The key-block kernel stores its dS tiles (banded per (sequence, head)
    for varlen packing and windows) and dq is one contraction per tile; the
    smaller workspace without the tiles sends dq through the recomputing
    query-block kernel instead.  Both match the oracle, with the scalar gate
    and sink, and agree with each other to bf16 rounding."""
    if case.startswith("dense"):
        K = 64 if case.endswith("64") else 128
        s = I.spec(2, T=700, K=K, V=K, g_scalar=True, sink=True)
        lengths = None
    else:
        s = I.spec(4, K=128, V=128, HQ=8, H=2, n_seq=5, window=300)
        lengths = [700, 1, 130, 0, 517]
    x_cpu = I.training_inputs(s, lengths=lengths)
    _check_all(s, x_cpu, what=f"stored dS {case}")
    x = _to(x_cpu)
    _, _, _, ga = _run_gpu(x)
    _, _, _, gb = _run_gpu_recompute(x)
    for name, ta, tb in zip(("dq", "dk", "dv", "dg"), ga[:4], gb[:4]):
        e = float((ta.float() - tb.float()).norm() / tb.float().norm())
        assert e < 1e-2, (name, e)


@pytest.mark.parametrize("case", ["cfg2", "cfg4_reduced", "fp32_options", "varlen_ragged"])
def test_fwd_gate_equals_prefix_then_forward(case):
    """wall_attn_fwd_gate fuses the prefix scan into the forward's operand
    pass: P must be bit for bit wall_prefix_cumsum's, o and lse bit for bit
    wall_attn_fwd's from that P, and its workspace must serve the backward as
    the forward's does (dense, varlen with every option, fp32)."""
    if case == "cfg2":
        s = I.spec(2)
    elif case == "cfg4_reduced":
        s = I.spec(4, len_lo=64, len_hi=600, window=128)
    elif case == "fp32_options":
        s = I.spec(4, dtype=torch.float32, K=64, V=64, HQ=4, H=2, window=100, len_lo=1,
                   len_hi=300)
    else:
        # empty and one-row sequences, chunk (32) and anchor-block (128)
        # boundaries falling inside sequences
        s = I.spec(4, K=64, V=64, HQ=4, H=2, n_seq=6, g_scalar=False, sink=False, window=0)
    lengths = [0, 1, 33, 0, 130, 257] if case == "varlen_ragged" else None
    x = _to(I.training_inputs(s, lengths=lengths))
    q, k, v, g, cu = x["q"], x["k"], x["v"], x["g"], x["cu_seqlens"]
    kw = dict(g_scalar=x["g_scalar"], sink_bias=x["sink_bias"], window_size=x["window_size"],
              cu_seqlens=cu)
    P = api.prefix_cumsum(g, cu)
    o, lse, fws = api.wall_attn_fwd(q, k, v, P, x["scale"], return_workspace=True, **kw)
    o2, lse2, P2, gws = api.wall_attn_fwd_gate(q, k, v, g, x["scale"], return_workspace=True,
                                               **kw)
    torch.cuda.synchronize()
    assert torch.equal(P2, P)
    assert torch.equal(o2, o)
    assert torch.equal(lse2, lse)
    a = api.wall_attn_bwd(x["dO"], q, k, v, P, o, lse, x["scale"], fwd_workspace=fws, **kw)
    b = api.wall_attn_bwd(x["dO"], q, k, v, P2, o2, lse2, x["scale"], fwd_workspace=gws, **kw)
    torch.cuda.synchronize()
    for name, ta, tb in zip(("dq", "dk", "dv", "dg"), a[:4], b[:4]):
        assert torch.equal(ta, tb), name


def _compare_units(s, xc, o, lse, grads, units, what):
    """o, lse and the gradients of the given (sequence * HQ + head) units
    against the oracle, element by element."""
    ref = wo.backward(xc["q"], xc["k"], xc["v"], xc["g"], xc["dO"], units=units,
                      **_oracle_kw(xc))
    heads = sorted({u % s.HQ for u in units})
    mask = np.zeros(o.shape[:3], dtype=bool)
    mask[:, :, heads] = True
    dq, dk, dv, dg, dgs, dsink = grads
    kmask = np.zeros(dk.shape[:3], dtype=bool)
    kmask[:, :, sorted({h // s.G for h in heads})] = True
    assert_fwd(s.dtype, o, ref["o"], lse, ref["lse"], mask, what)
    assert_grad(s.dtype, "dq", dq, ref["dq"], mask, what)
    assert_grad(s.dtype, "dk", dk, ref["dk"], kmask, what)
    assert_grad(s.dtype, "dv", dv, ref["dv"], kmask, what)
    assert_grad(s.dtype, "dg", dg, ref["dg"], mask, what)
    if dgs is not None:
        assert_grad(s.dtype, "dg_scalar", dgs, ref["dg_scalar"], mask, what,
                    relative_to_max=True)


@pytest.mark.slow
def test_cfg3_headline_call_sequence_full_size_sampled():
    """The benchmark's own call sequence at T = 8192 on its inputs:
    wall_attn_fwd_gate (prefix scan fused into the operand pass), then
    wall_attn_bwd given the gate call's workspace.  One GQA group (4 query
    heads) against the oracle, element by element."""
    s = I.spec(3)
    xc = I.training_inputs(s)
    x = _to(xc)
    o, lse, P, ws = api.wall_attn_fwd_gate(x["q"], x["k"], x["v"], x["g"], s.scale,
                                           return_workspace=True)
    grads = api.wall_attn_bwd(x["dO"], x["q"], x["k"], x["v"], P, o, lse, s.scale,
                              fwd_workspace=ws)
    torch.cuda.synchronize()
    _compare_units(s, xc, o, lse, grads, [4, 5, 6, 7], "headline sequence T=8192")


def _autograd_cfg4(s, xc, units, what):
    x = _to(xc)
    q, k, v, g = (x[n].clone().requires_grad_(True) for n in ("q", "k", "v", "g"))
    gs = x["g_scalar"].clone().requires_grad_(True)
    sk = x["sink_bias"].clone().requires_grad_(True)
    o = api.wall_attn(q, k, v, g, scale=s.scale, g_scalar=gs, sink_bias=sk,
                      window_size=x["window_size"], cu_seqlens=x["cu_seqlens"])
    o.backward(x["dO"])
    torch.cuda.synchronize()
    # lse is not an autograd output: compare it from a forward call
    _, lse = api.wall_attn_fwd(x["q"], x["k"], x["v"], api.prefix_cumsum(x["g"], x["cu_seqlens"]),
                               s.scale, x["g_scalar"], x["sink_bias"], x["window_size"],
                               x["cu_seqlens"])
    _compare_units(s, xc, o.detach(), lse,
                   (q.grad, k.grad, v.grad, g.grad, gs.grad, None), units, what)
    if units is None or len(units) == s.HQ * s.n_seq:
        ref = wo.backward(xc["q"], xc["k"], xc["v"], xc["g"], xc["dO"], **_oracle_kw(xc))
        assert_grad(s.dtype, "dsink", sk.grad, ref["dsink"], None, what, relative_to_max=True)


def test_cfg4_through_autograd_reduced():
    """Config 4's options through the autograd function (the README's call
    pattern), every unit, dsink included."""
    s = I.spec(4, len_lo=64, len_hi=600, window=128)
    units = [seq * s.HQ + h for seq in range(s.n_seq) for h in range(s.HQ)]
    _autograd_cfg4(s, I.training_inputs(s), units, "cfg4 autograd reduced")


@pytest.mark.slow
def test_cfg4_through_autograd_full_size_sampled():
    s = I.spec(4)
    units = [seq * s.HQ + h for seq in range(s.n_seq) for h in (0, 1, 2, 3, 4, 5, 6, 7)]
    _autograd_cfg4(s, I.training_inputs(s), units, "cfg4 autograd full")
