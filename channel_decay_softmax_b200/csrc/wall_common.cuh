// wall_common.cuh -- shared device helpers of the Wall Attention CUDA path.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "wall.h"

namespace wall {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kInvLn2 = 1.4426950408889634f;

// Records `code` in the device status word (the first error wins).  Kernels
// receive the word's address from the C ABI layer.
__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------------------
// element conversion

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Load 8 consecutive elements (16 B for bf16, 32 B for fp32) as floats.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* out) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float* out) {
  float4 a = reinterpret_cast<const float4*>(p)[0];
  float4 b = reinterpret_cast<const float4*>(p)[1];
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* in) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8(float* p, const float* in) {
  reinterpret_cast<float4*>(p)[0] = make_float4(in[0], in[1], in[2], in[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(in[4], in[5], in[6], in[7]);
}

// ---------------------------------------------------------------------------
// sequences: rows are flattened over B*T; sequence s covers rows
// [start(s), start(s) + len(s)).  Without cu_seqlens sequence s is batch row s.

// Offsets from cu_seqlens are clamped into [0, rows] so a malformed array
// cannot send a kernel out of bounds (a separate check reports it).
struct Seqs {
  const int32_t* cu;  // device, [n+1] or nullptr
  int n;              // number of sequences
  int T;              // rows per batch row (dense case)
  long rows;          // B*T
  __device__ __forceinline__ long clamp_row(long r) const {
    return r < 0 ? 0 : (r > rows ? rows : r);
  }
  __device__ __forceinline__ long start(int s) const {
    return cu ? clamp_row(cu[s]) : (long)s * T;
  }
  __device__ __forceinline__ int len(int s) const {
    if (!cu) return T;
    const long a = clamp_row(cu[s]), b = clamp_row(cu[s + 1]);
    return b > a ? (int)(b - a) : 0;
  }
};

// Maps a flat block index to (sequence, block within sequence) for blocks of
// `bs` rows; returns false past the last block.
__device__ __forceinline__ bool seq_block(const Seqs& S, int bs, int flat, int& seq, int& blk) {
  if (!S.cu) {
    int nb = (S.T + bs - 1) / bs;
    if (nb == 0) return false;
    seq = flat / nb;
    blk = flat % nb;
    return seq < S.n;
  }
  int acc = 0;
  for (int s = 0; s < S.n; ++s) {
    int nb = (S.len(s) + bs - 1) / bs;
    if (flat < acc + nb) {
      seq = s;
      blk = flat - acc;
      return true;
    }
    acc += nb;
  }
  return false;
}

inline int ceil_div(long a, long b) { return (int)((a + b - 1) / b); }

}  // namespace wall
