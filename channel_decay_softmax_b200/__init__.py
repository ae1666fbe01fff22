"""B200-native Wall Attention: hand-written sm_100a CUDA kernels behind a
C ABI (include/wall.h, libwall.so), with a thin torch binding.

Public API (wall-attention-release README "Usage" / "Decode"):
    wall_attn(q, k, v, g, scale=None, g_scalar=None, sink_bias=None,
              window_size=None, cu_seqlens=None)
    prefix_cumsum(g)                    # P = cumsum(g) / ln 2
    build_wall_kv_cache(k, P, chunk_size=64)
    wall_attn_decode(q, v, p_curr, k_tilde, r_cache, sink_bias, scale,
                     cache_chunk_size)
    WallDecodeCache                     # append-as-you-go serving loop
Beyond them: wall_attn_fwd / wall_attn_bwd (the two halves, from P),
wall_attn_fwd_gate (prefix scan fused into the forward), wall_attn_decode_chunk
(several queries against the cache: multi-token decode, chunked prefill) and
WallAttnStepGraph (a training step captured in a CUDA graph).
The C-ABI calls are also exposed one to one in ``channel_decay_softmax_b200._lib``.
"""
from .api import (WallAttnFunction, WallAttnStepGraph, WallDecodeCache, build_wall_kv_cache,
                  prefix_cumsum, wall_attn, wall_attn_bwd, wall_attn_decode,
                  wall_attn_decode_chunk, wall_attn_fwd, wall_attn_fwd_gate)

__all__ = ["wall_attn", "wall_attn_fwd", "wall_attn_fwd_gate", "wall_attn_bwd", "prefix_cumsum",
           "build_wall_kv_cache", "wall_attn_decode", "wall_attn_decode_chunk",
           "WallAttnFunction", "WallAttnStepGraph", "WallDecodeCache"]
