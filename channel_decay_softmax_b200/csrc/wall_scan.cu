// wall_scan.cu -- segmented prefix scans along time.
//
// Forward scan: the base-2 gate prefix P = cumsum(g) / ln 2 (README "Decode":
// the prefix is the cumulative sum of g with scale 1/ln 2).  Reverse scan:
// the gate gradient dg_u = sum_{t >= u} dL_t within a sequence, the adjoint
// of that prefix, and the same for the scalar gate.
//
// Design (HBM-bound; every column is an independent scan of up to T rows):
// three passes that each stream with many independent loads in flight.
//   1. chunk sums: per 32-row chunk and column, a compensated sum
//   2. carries: per column, the exclusive running total of its chunk sums,
//      accumulated in double (32 columns x 8 chunk ranges per CTA, the
//      ranges combined through shared memory)
//   3. chunk scans: each chunk re-reads its rows and scans them from its
//      carry (compensated), writing the result
// Passes 1 and 3 read the input twice (2 B + 2 B + 4 B per element for bf16
// in, fp32 out) but keep a chunk's 32 rows of 16-byte loads in flight per
// thread, where a single pass would serialise on the carry.  The chunk sums
// and carries live in the chunk's first row of a caller-provided fp32
// [rows, C] scratch, which may be the output itself: pass 3 reads the carry
// of a chunk before its own thread overwrites that row.
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {

namespace {

constexpr int kChunk = 32;       // rows per chunk
constexpr int kInFlight = 16;    // rows of loads issued together
constexpr int kThreadsScan = 128;

// row of the sequence that holds chunk k's sum / carry: its first row in
// scan order
__device__ __forceinline__ long chunk_row(long start, long len, int k, bool reverse) {
  return reverse ? start + len - 1 - (long)k * kChunk : start + (long)k * kChunk;
}

template <typename T>
__device__ __forceinline__ void loadv(const T* p, float* out, int vec) {
  if (vec == 8) {
    load8(p, out);
  } else {
    out[0] = to_f32(p[0]);
  }
}

// pass 1: per (sequence, chunk, column group) compensated column sums
template <typename Tin, int VEC, bool kReverse>
__global__ void __launch_bounds__(kThreadsScan)
    chunk_sum_kernel(const Tin* __restrict__ x, float* __restrict__ scratch, long C, Seqs seqs) {
  int s, k;
  if (!seq_block(seqs, kChunk, (int)blockIdx.x, s, k)) return;
  const long start = seqs.start(s);
  const long len = seqs.len(s);
  const long lr0 = (long)k * kChunk;
  if (lr0 >= len) return;
  const long col = ((long)blockIdx.y * kThreadsScan + threadIdx.x) * VEC;
  if (col >= C) return;
  const int n = (int)min((long)kChunk, len - lr0);
  float sum[VEC], cmp[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) sum[v] = cmp[v] = 0.f;
  // fixed trip count, predicated: 16 rows of loads in flight at a time
#pragma unroll
  for (int r0 = 0; r0 < kChunk; r0 += kInFlight) {
    float a[kInFlight][VEC];
#pragma unroll
    for (int r = 0; r < kInFlight; ++r) {
      const long lr = lr0 + (r0 + r < n ? r0 + r : 0);
      const long pr = kReverse ? start + len - 1 - lr : start + lr;
      float t[8];
      loadv(x + pr * C + col, t, VEC);
#pragma unroll
      for (int v = 0; v < VEC; ++v) a[r][v] = r0 + r < n ? t[v] : 0.f;
    }
#pragma unroll
    for (int r = 0; r < kInFlight; ++r) {
#pragma unroll
      for (int v = 0; v < VEC; ++v) {
        const float yk = a[r][v] - cmp[v];
        const float tk = sum[v] + yk;
        cmp[v] = (tk - sum[v]) - yk;
        sum[v] = tk;
      }
    }
  }
  float* dst = scratch + chunk_row(start, len, k, kReverse) * C + col;
#pragma unroll
  for (int v = 0; v < VEC; ++v) dst[v] = sum[v];
}

// pass 2: per (sequence, column) exclusive carries of the chunk sums, in
// place.  A CTA takes 32 columns; its 8 warps take 8 consecutive ranges of
// chunks, load a range's sums 32 at a time (all in flight), and meet in
// shared memory for the range offsets.
constexpr int kCarryParts = 8;
constexpr int kCarryBatch = 32;
template <bool kReverse>
__global__ void __launch_bounds__(32 * kCarryParts)
    carry_kernel(float* __restrict__ scratch, long C, Seqs seqs, float mul,
                 const float* __restrict__ carry_in, float* __restrict__ carry_out) {
  __shared__ double part_sum[kCarryParts][32];
  const int s = blockIdx.y;
  const int lane = threadIdx.x % 32, part = threadIdx.x / 32;
  const long col = (long)blockIdx.x * 32 + lane;
  const bool valid = col < C;
  const long start = seqs.start(s);
  const long len = seqs.len(s);
  const int nchunk = (int)((len + kChunk - 1) / kChunk);
  const int per = (nchunk + kCarryParts - 1) / kCarryParts;
  const int k0 = min(nchunk, part * per), k1 = min(nchunk, k0 + per);
  // range total
  double tot = 0.0;
  for (int kb = k0; kb < k1; kb += kCarryBatch) {
    float v[kCarryBatch];
#pragma unroll
    for (int x = 0; x < kCarryBatch; ++x)
      v[x] = (valid && kb + x < k1) ? scratch[chunk_row(start, len, kb + x, kReverse) * C + col]
                                     : 0.f;
#pragma unroll
    for (int x = 0; x < kCarryBatch; ++x) tot += (double)v[x];
  }
  part_sum[part][lane] = tot;
  __syncthreads();
  double run = 0.0, all = 0.0;
#pragma unroll
  for (int q = 0; q < kCarryParts; ++q) {
    const double t = part_sum[q][lane];
    if (q < part) run += t;
    all += t;
  }
  // exclusive carries of the range, in place
  for (int kb = k0; kb < k1; kb += kCarryBatch) {
    float v[kCarryBatch];
#pragma unroll
    for (int x = 0; x < kCarryBatch; ++x)
      v[x] = (valid && kb + x < k1) ? scratch[chunk_row(start, len, kb + x, kReverse) * C + col]
                                     : 0.f;
#pragma unroll
    for (int x = 0; x < kCarryBatch; ++x) {
      if (valid && kb + x < k1) scratch[chunk_row(start, len, kb + x, kReverse) * C + col] = (float)run;
      run += (double)v[x];
    }
  }
  if (carry_out != nullptr && valid && part == 0) {
    const float cin = carry_in != nullptr ? carry_in[(long)s * C + col] : 0.f;
    carry_out[(long)s * C + col] = fmaf(mul, (float)all, cin);
  }
}

// pass 3: per (sequence, chunk, column group) scan from the chunk's carry
template <typename Tin, typename Tout, int VEC, bool kReverse>
__global__ void __launch_bounds__(kThreadsScan)
    chunk_scan_kernel(const Tin* __restrict__ x, Tout* __restrict__ y,
                      const float* __restrict__ scratch, long C, Seqs seqs, float mul,
                      const float* __restrict__ carry_in) {
  int s, k;
  if (!seq_block(seqs, kChunk, (int)blockIdx.x, s, k)) return;
  const long start = seqs.start(s);
  const long len = seqs.len(s);
  const long lr0 = (long)k * kChunk;
  if (lr0 >= len) return;
  const long col = ((long)blockIdx.y * kThreadsScan + threadIdx.x) * VEC;
  if (col >= C) return;
  const int n = (int)min((long)kChunk, len - lr0);
  float acc[VEC], cmp[VEC], cin[VEC];
  {
    // read before this thread overwrites the row (the scratch may be y)
    const float* c = scratch + chunk_row(start, len, k, kReverse) * C + col;
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
      acc[v] = c[v];
      cmp[v] = 0.f;
      cin[v] = carry_in != nullptr ? carry_in[(long)s * C + col + v] : 0.f;
    }
  }
  // fixed trip count, predicated: 16 rows of loads in flight at a time
#pragma unroll
  for (int r0 = 0; r0 < kChunk; r0 += kInFlight) {
  float a[kInFlight][VEC];
#pragma unroll
  for (int r = 0; r < kInFlight; ++r) {
    const long lr = lr0 + (r0 + r < n ? r0 + r : 0);
    const long pr = kReverse ? start + len - 1 - lr : start + lr;
    float t[8];
    loadv(x + pr * C + col, t, VEC);
#pragma unroll
    for (int v = 0; v < VEC; ++v) a[r][v] = t[v];
  }
#pragma unroll
  for (int rr = 0; rr < kInFlight; ++rr) {
    const int r = r0 + rr;
    const long lr = lr0 + r;
    const long pr = kReverse ? start + len - 1 - lr : start + lr;
    float o[8];
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
      const float yk = a[rr][v] - cmp[v];
      const float tk = acc[v] + yk;
      cmp[v] = (tk - acc[v]) - yk;
      acc[v] = tk;
      // one fused rounding; the one-token decode step forms P the same way
      o[v] = fmaf(mul, acc[v], cin[v]);
    }
    if (r < n) {
      if (VEC == 8) {
        store8(y + pr * C + col, o);
      } else {
        y[pr * C + col] = from_f32<Tout>(o[0]);
      }
    }
  }
  }
}

template <typename Tin, typename Tout, bool kReverse, int VEC>
int launch_scan_vec(const Tin* x, Tout* y, float* scratch, long C, const Seqs& seqs, float mul,
                    const float* carry_in, float* carry_out, cudaStream_t stream) {
  const long groups = (C / VEC + kThreadsScan - 1) / kThreadsScan;
  // chunks of all sequences, flattened (a bound for cu_seqlens: each
  // sequence adds at most one partial chunk)
  const long chunks = seqs.cu ? (seqs.rows + kChunk - 1) / kChunk + seqs.n
                              : (long)seqs.n * ((seqs.T + kChunk - 1) / kChunk);
  if (groups > 65535 || chunks > 0x7fffffffL || seqs.n > 65535) return WALL_ERR_UNSUPPORTED;
  if (chunks == 0 || groups == 0) return WALL_OK;
  const dim3 grid((unsigned)chunks, (unsigned)groups);
  chunk_sum_kernel<Tin, VEC, kReverse><<<grid, kThreadsScan, 0, stream>>>(x, scratch, C, seqs);
  const dim3 cgrid((unsigned)((C + 31) / 32), (unsigned)seqs.n);
  carry_kernel<kReverse>
      <<<cgrid, 32 * kCarryParts, 0, stream>>>(scratch, C, seqs, mul, carry_in, carry_out);
  chunk_scan_kernel<Tin, Tout, VEC, kReverse>
      <<<grid, kThreadsScan, 0, stream>>>(x, y, scratch, C, seqs, mul, carry_in);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

template <typename Tin, typename Tout, bool kReverse>
int launch_scan(const Tin* x, Tout* y, float* scratch, long C, const Seqs& seqs, float mul,
                const float* carry_in, float* carry_out, cudaStream_t stream) {
  if (seqs.n == 0 || C == 0) return WALL_OK;
  // 16-byte vectors need 8 columns per thread and 16-byte aligned rows
  const bool vec8 = (C % 8 == 0) && ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y) |
                                      reinterpret_cast<uintptr_t>(scratch)) % 16 == 0);
  return vec8 ? launch_scan_vec<Tin, Tout, kReverse, 8>(x, y, scratch, C, seqs, mul, carry_in,
                                                        carry_out, stream)
              : launch_scan_vec<Tin, Tout, kReverse, 1>(x, y, scratch, C, seqs, mul, carry_in,
                                                        carry_out, stream);
}

}  // namespace

int scan_prefix_log2(const void* g, int dtype, float* P, long C, const Seqs& seqs,
                     const float* carry_in, float* carry_out, cudaStream_t stream) {
  // the output doubles as the chunk scratch
  if (dtype == WALL_BF16)
    return launch_scan<__nv_bfloat16, float, false>(static_cast<const __nv_bfloat16*>(g), P, P, C,
                                                    seqs, kInvLn2, carry_in, carry_out, stream);
  return launch_scan<float, float, false>(static_cast<const float*>(g), P, P, C, seqs, kInvLn2,
                                          carry_in, carry_out, stream);
}

int scan_prefix_plain(const float* x, float* y, long C, const Seqs& seqs, cudaStream_t stream) {
  return launch_scan<float, float, false>(x, y, y, C, seqs, 1.f, nullptr, nullptr, stream);
}

int scan_reverse(const float* x, void* y, int out_dtype, float* scratch, long C, const Seqs& seqs,
                 cudaStream_t stream) {
  if (out_dtype == WALL_BF16)
    return launch_scan<float, __nv_bfloat16, true>(x, static_cast<__nv_bfloat16*>(y), scratch, C,
                                                   seqs, 1.f, nullptr, nullptr, stream);
  return launch_scan<float, float, true>(x, static_cast<float*>(y), scratch, C, seqs, 1.f,
                                         nullptr, nullptr, stream);
}

}  // namespace wall
