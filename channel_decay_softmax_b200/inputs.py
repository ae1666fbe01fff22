"""Seeded synthetic inputs shaped like the Wall Attention pages' workloads.

This module holds no Wall Attention arithmetic: only shapes, seeds and
value distributions.  It is the one module that both the CUDA path's tests
and the oracle's tests draw their inputs from.

Workloads (shapes and distributions follow the wall-attention-release
README "Usage" example -- q, k, v ~ N(0, 1), g = 0.02 * N(0, 1) -- and the
Tilde blog's remark that |P| passes 160 by T = 8192):

  1  tiny fp32:          B=1, T=256,  HQ=2,  H=1, K=V=64,  g = 0.02 N
  2  training, bf16:     B=2, T=1024, HQ=8,  H=4, K=V=64,  g = 0.02 N
  3  long context, bf16: B=1, T=8192, HQ=16, H=4, K=V=128, g = -0.05 |N|
  4  varlen + options:   B=1, 8 sequences of length U[512, 4096] (seed 2000),
                         HQ=16, H=2, K=V=128, g = 0.02 N,
                         g_scalar = logsigmoid(N(4, 1)) [1,T,HQ],
                         sink_bias ~ N(0, 1) [HQ], window 1024
  5  decode, bf16:       B=32, T_kv=32768, HQ=32, H=8, K=V=128,
                         g = -0.02 |N|, cache chunk C = 64

Values are drawn in fp32 from a torch Generator seeded 1000 + config and
then cast to the config's dtype; both the CUDA path and the oracle consume
the cast values.  The upstream gradient dO is N(0, 1) (the README example
back-propagates o.sum(), i.e. dO = 1; a random dO is the stronger test).

Strongly decaying channels (``g_strong``, any config): a fast-forgetting
channel of a trained gate, the blog's "dynamic" channels, is not in the
pages' workloads; this recipe adds it.  For query head h and channel n the
channel class is (h * K + n) % 8; class c < len(g_strong) gets the per-step
log-gate -g_strong[c] * |1 + 0.1 N| (so -3 forgets 95 % per step), the
others keep the config's distribution.  ``strong_heads`` > 0 limits the
strong channels to the first that many query heads.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Spec:
    name: str
    B: int
    T: int
    HQ: int
    H: int
    K: int
    V: int
    dtype: torch.dtype
    g_kind: str                 # "normal" (g = amp*N) or "decay" (g = -amp*|N|)
    g_amp: float
    n_seq: int = 0              # > 0: varlen packing with this many sequences
    len_lo: int = 0
    len_hi: int = 0
    g_scalar: bool = False
    sink: bool = False
    window: int = 0
    chunk: int = 64             # decode-cache chunk size
    seed: int = 0
    g_strong: tuple = ()        # per-step decay of the strong channel classes
    strong_heads: int = 0       # > 0: strong channels in heads [0, strong_heads) only

    @property
    def G(self) -> int:
        return self.HQ // self.H

    @property
    def scale(self) -> float:
        return self.K ** -0.5


CONFIGS = {
    1: Spec("tiny_fp32", 1, 256, 2, 1, 64, 64, torch.float32, "normal", 0.02, seed=1001),
    2: Spec("train_bf16", 2, 1024, 8, 4, 64, 64, torch.bfloat16, "normal", 0.02, seed=1002),
    3: Spec("long_bf16", 1, 8192, 16, 4, 128, 128, torch.bfloat16, "decay", 0.05, seed=1003),
    4: Spec("varlen_opts_bf16", 1, 0, 16, 2, 128, 128, torch.bfloat16, "normal", 0.02,
            n_seq=8, len_lo=512, len_hi=4096, g_scalar=True, sink=True, window=1024,
            seed=1004),
    5: Spec("decode_bf16", 32, 32768, 32, 8, 128, 128, torch.bfloat16, "decay", 0.02,
            chunk=64, seed=1005),
}

LENGTHS_SEED = 2000


def spec(cfg: int, **over) -> Spec:
    """The workload spec of config ``cfg``, with optional field overrides
    (smaller T or B for element-by-element parity)."""
    s = CONFIGS[cfg]
    return replace(s, **over) if over else s


def varlen_lengths(s: Spec) -> list[int]:
    """Sequence lengths for a varlen spec, uniform integers in [lo, hi]."""
    gen = torch.Generator().manual_seed(LENGTHS_SEED)
    return torch.randint(s.len_lo, s.len_hi + 1, (s.n_seq,), generator=gen).tolist()


def cu_seqlens_of(lengths) -> torch.Tensor:
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32)


def _gate(gen, shape, s: Spec, device) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    g = -s.g_amp * x.abs() if s.g_kind == "decay" else s.g_amp * x
    if s.g_strong:
        HQ, K = shape[-2], shape[-1]
        cls = (torch.arange(HQ, device=device)[:, None] * K +
               torch.arange(K, device=device)[None, :]) % 8
        if s.strong_heads > 0:
            cls[s.strong_heads:] = 8
        jitter = (1.0 + 0.1 * torch.randn(shape, generator=gen, device=device,
                                          dtype=torch.float32)).abs()
        for c, a in enumerate(s.g_strong):
            g = torch.where(cls == c, -float(a) * jitter, g)
    return g


def training_inputs(s: Spec, device="cpu", lengths=None) -> dict:
    """q, k, v, g, dO (and g_scalar, sink_bias, cu_seqlens when the spec has
    them) for one fwd+bwd step, cast to the spec's dtype except the fp32
    optional arguments."""
    gen = torch.Generator(device=device).manual_seed(s.seed)
    B, T = s.B, s.T
    cu = None
    if s.n_seq:
        lengths = lengths if lengths is not None else varlen_lengths(s)
        cu = cu_seqlens_of(lengths)
        B, T = 1, int(cu[-1])
    f32 = dict(generator=gen, device=device, dtype=torch.float32)
    q = torch.randn((B, T, s.HQ, s.K), **f32)
    k = torch.randn((B, T, s.H, s.K), **f32)
    v = torch.randn((B, T, s.H, s.V), **f32)
    g = _gate(gen, (B, T, s.HQ, s.K), s, device)
    dO = torch.randn((B, T, s.HQ, s.V), **f32)
    out = dict(q=q.to(s.dtype), k=k.to(s.dtype), v=v.to(s.dtype), g=g.to(s.dtype),
               dO=dO.to(s.dtype), g_scalar=None, sink_bias=None, cu_seqlens=None,
               window_size=s.window, scale=s.scale, B=B, T=T)
    if s.g_scalar:
        out["g_scalar"] = torch.nn.functional.logsigmoid(
            4.0 + torch.randn((B, T, s.HQ), **f32))
    if s.sink:
        out["sink_bias"] = torch.randn((s.HQ,), **f32)
    if cu is not None:
        out["cu_seqlens"] = cu.to(device)
    return out


def decode_batch_inputs(s: Spec, b: int, device="cpu", n_query_rows: int = 64) -> dict:
    """One batch row of the decode workload, generated on its own so a
    sampled row can be regenerated alone: k [T,H,K], v [T,H,V], g [T,HQ,K]
    and queries q for the last ``n_query_rows`` positions [n,HQ,K]."""
    gen = torch.Generator(device=device).manual_seed(s.seed * 1000 + b)
    f32 = dict(generator=gen, device=device, dtype=torch.float32)
    k = torch.randn((s.T, s.H, s.K), **f32).to(s.dtype)
    v = torch.randn((s.T, s.H, s.V), **f32).to(s.dtype)
    g = _gate(gen, (s.T, s.HQ, s.K), s, device).to(s.dtype)
    q = torch.randn((n_query_rows, s.HQ, s.K), **f32).to(s.dtype)
    return dict(k=k, v=v, g=g, q=q)


def decode_inputs(s: Spec, device="cpu", n_query_rows: int = 64) -> dict:
    """The whole decode workload, batch rows stacked: k [B,T,H,K],
    v [B,T,H,V], g [B,T,HQ,K], q_tail [B,n,HQ,K] (queries of the last n
    positions)."""
    k = torch.empty((s.B, s.T, s.H, s.K), dtype=s.dtype, device=device)
    v = torch.empty((s.B, s.T, s.H, s.V), dtype=s.dtype, device=device)
    g = torch.empty((s.B, s.T, s.HQ, s.K), dtype=s.dtype, device=device)
    q = torch.empty((s.B, n_query_rows, s.HQ, s.K), dtype=s.dtype, device=device)
    for b in range(s.B):
        x = decode_batch_inputs(s, b, device, n_query_rows)
        k[b], v[b], g[b], q[b] = x["k"], x["v"], x["g"], x["q"]
    return dict(k=k, v=v, g=g, q_tail=q, scale=s.scale, chunk=s.chunk)


def causal_pairs(T: int, window: int = 0) -> int:
    """Number of visible (i, j) pairs of one sequence of length T."""
    if window and window > 0 and window < T:
        W = window
        return W * (W + 1) // 2 + (T - W) * W
    return T * (T + 1) // 2


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = ["Spec", "CONFIGS", "spec", "varlen_lengths", "cu_seqlens_of", "training_inputs",
           "decode_batch_inputs", "decode_inputs", "causal_pairs", "ceil_div"]
