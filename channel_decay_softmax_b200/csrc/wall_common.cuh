// wall_common.cuh -- shared device helpers of the Wall Attention CUDA path.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "wall.h"

namespace wall {

constexpr float kLog2e = 1.4426950408889634f;

// 2^x on the FMA and integer pipes, for softmax exponents (x <= ~0), so that
// part of a tile's exponentials can bypass the 16-per-clock MUFU unit.
// Cody-Waite style range reduction x = n + f with n = round(x) (added to and
// subtracted from 1.5 * 2^23, which leaves n in the low mantissa bits) and
// |f| <= 1/2, then a degree-3 polynomial for 2^f whose coefficients are our
// own relative-error minimax fit on [-1/2, 1/2] (max relative error 7.6e-5,
// well under the 2^-9 step of the bf16 P it feeds), and n added to the
// exponent field.  x is clamped at -126, where 2^x no longer matters next to
// the row's leading terms; the result there is 0 or a tiny subnormal.
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -126.f);
  const float y = x + 12582912.f;
  const float f = x - (y - 12582912.f);
  const float p = fmaf(fmaf(fmaf(0.05517049878835678f, f, 0.24260851740837097f), f,
                            0.6932609677314758f),
                       f, 0.9999282360076904f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(y) << 23));
}
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kInvLn2 = 1.4426950408889634f;

// Records `code` in the device status word (the first error wins).  Kernels
// receive the word's address from the C ABI layer.
__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// The anchored operands of a unit beyond the anchored range are recomputed
// elsewhere, but the tensor-core kernels still read them (a key tile that
// runs past its sequence reads the next one's rows, with zero weight):
// clamped into the finite bf16 range, 0 times such a value stays 0.  Inside
// the range the clamp never acts.
__device__ __forceinline__ float saturate_bf16(float x) {
  return fminf(fmaxf(x, -3.3895313892515355e38f), 3.3895313892515355e38f);
}

// Sets a flag word that many threads may find set: the word is read first,
// so once it is set the threads that see it cost a load, not an atomic.
__device__ __forceinline__ void set_flag(int* f) {
  if (*reinterpret_cast<volatile int*>(f) == 0) atomicOr(f, 1);
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

// Where the tensor-core backward keeps its dS tiles (128 x 128, bf16).  A
// query block I of a sequence sees key blocks J in [jlo(I), I]: every block
// before it without a window, else the wb blocks a window of W keys reaches
// back, wb = ceil((W - 1) / 128).  A (sequence, head) stores its tiles row by
// row, tile (I, J) at rowstart(I) + J - jlo(I); the (sequence, head) pairs
// follow each other sequence-major: pair (s, h) starts at
// HQ * (tiles of the sequences before s) + h * tiles(nb(s)).
struct DsLayout {
  int wb;  // key blocks reached back beyond the query block; 1 << 28: no window
  __host__ __device__ static DsLayout of_window(int window) {
    DsLayout d;
    d.wb = window > 0 ? (window - 1 + 127) / 128 : (1 << 28);
    return d;
  }
  __host__ __device__ int jlo(int I) const { return I > wb ? I - wb : 0; }
  // tiles of the query blocks before I: sum over I' < I of min(I', wb) + 1
  __host__ __device__ long rowstart(int I) const {
    const long i = I, w = wb;
    return i <= w + 1 ? i * (i + 1) / 2 : (w + 1) * (w + 2) / 2 + (i - w - 1) * (w + 1);
  }
  __host__ __device__ long tiles(int nb) const { return rowstart(nb); }
  // first tile of (sequence s, head h)
  __device__ long pair_base(const Seqs& seqs, int HQ, int s, int h) const {
    long before = 0;
    int nb;
    if (!seqs.cu) {
      nb = (seqs.T + 127) / 128;
      before = (long)s * tiles(nb);
    } else {
      for (int x = 0; x < s; ++x) before += tiles((seqs.len(x) + 127) / 128);
      nb = (seqs.len(s) + 127) / 128;
    }
    return before * HQ + (long)h * tiles(nb);
  }
  // tiles of a whole problem: dense (B sequences of T rows), or a bound for
  // n_seq packed sequences of `rows` rows in all (a sequence's tiles grow
  // faster than its blocks, so one sequence holding every block is the most)
  __host__ static long total(const DsLayout& d, long rows, int T, int B, int HQ,
                             int n_seq_varlen) {
    if (n_seq_varlen > 0) return (long)HQ * d.tiles((int)((rows + 127) / 128) + n_seq_varlen);
    return (long)B * HQ * d.tiles((T + 127) / 128);
  }
};

}  // namespace wall
