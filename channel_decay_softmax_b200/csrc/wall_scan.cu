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

// Chunks of the sequences before s: the first slot of sequence s in a
// compact [chunks, C] scratch (one row per chunk, in seq_block's order).
__device__ __forceinline__ long chunks_before(const Seqs& seqs, int s) {
  if (!seqs.cu) return (long)s * ((seqs.T + kChunk - 1) / kChunk);
  long n = 0;
  for (int x = 0; x < s; ++x) n += (seqs.len(x) + kChunk - 1) / kChunk;
  return n;
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
    chunk_sum_kernel(const Tin* __restrict__ x, float* __restrict__ scratch, long C, Seqs seqs,
                     int* __restrict__ zero = nullptr, int n_zero = 0, bool compact = false) {
  // words a later pass of the same call sets (the fused operand pass's unit
  // flags), cleared here so that no separate launch is needed
  if (zero && blockIdx.x == 0 && blockIdx.y == 0)
    for (int z = threadIdx.x; z < n_zero; z += blockDim.x) zero[z] = 0;
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
  // the flat chunk index is blockIdx.x: the compact slot
  float* dst = scratch + (compact ? (long)blockIdx.x : chunk_row(start, len, k, kReverse)) * C + col;
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
                 const float* __restrict__ carry_in, float* __restrict__ carry_out,
                 bool compact = false) {
  __shared__ double part_sum[kCarryParts][32];
  const int s = blockIdx.y;
  const int lane = threadIdx.x % 32, part = threadIdx.x / 32;
  const long col = (long)blockIdx.x * 32 + lane;
  const bool valid = col < C;
  const long start = seqs.start(s);
  const long len = seqs.len(s);
  const int nchunk = (int)((len + kChunk - 1) / kChunk);
  const int per = (nchunk + kCarryParts - 1) / kCarryParts;
  const long base = compact ? chunks_before(seqs, s) : 0;
  auto slot = [&](int k) {
    return compact ? base + k : chunk_row(start, len, k, kReverse);
  };
  const int k0 = min(nchunk, part * per), k1 = min(nchunk, k0 + per);
  // range total
  double tot = 0.0;
  for (int kb = k0; kb < k1; kb += kCarryBatch) {
    float v[kCarryBatch];
#pragma unroll
    for (int x = 0; x < kCarryBatch; ++x)
      v[x] = (valid && kb + x < k1) ? scratch[slot(kb + x) * C + col]
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
      v[x] = (valid && kb + x < k1) ? scratch[slot(kb + x) * C + col]
                                     : 0.f;
#pragma unroll
    for (int x = 0; x < kCarryBatch; ++x) {
      if (valid && kb + x < k1) scratch[slot(kb + x) * C + col] = (float)run;
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

// VW consecutive elements as floats (VW = 4: 8 B of bf16 / 16 B of fp32).
template <int VW>
__device__ __forceinline__ void loadw(const __nv_bfloat16* p, float* out) {
  if constexpr (VW == 8) {
    load8(p, out);
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
  }
}
template <int VW>
__device__ __forceinline__ void loadw(const float* p, float* out) {
  if constexpr (VW == 8) {
    load8(p, out);
  } else {
    const float4 a = *reinterpret_cast<const float4*>(p);
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  }
}
template <int VW>
__device__ __forceinline__ void storew(__nv_bfloat16* p, const float* in) {
  if constexpr (VW == 8) {
    store8(p, in);
  } else {
    __nv_bfloat162 h[2] = {__floats2bfloat162_rn(in[0], in[1]), __floats2bfloat162_rn(in[2], in[3])};
    *reinterpret_cast<uint2*>(p) = *reinterpret_cast<const uint2*>(h);
  }
}
template <int VW>
__device__ __forceinline__ void storew(float* p, const float* in) {
  if constexpr (VW == 8) {
    store8(p, in);
  } else {
    *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
  }
}

// pass 3 of the forward scan fused with the tensor-core forward's operand
// preparation (the prefix enters the forward without an HBM round trip of
// its own): per (sequence, chunk, VW columns of one query head) the same
// compensated scan from the chunk's carry as chunk_scan_kernel, bit for bit,
// writing P, and for each row
//   Qh = q * 2^(P - R),  Kh = k * 2^(R - P),  R = floor(P at the row's
//   128-row block start)   (the anchors, written at the block start row)
// as the forward's preparation kernel forms them, flagging the (sequence,
// head) units with an exponent |P - R| beyond kAnchorRange as it does.  R of a block whose start
// lies in an earlier chunk is that row's prefix, rebuilt from its chunk's
// carry: the scan's first step is carry + g, then one fused rounding.
// The carries come from a scratch that is not P, so no thread reads a carry
// another one has overwritten; it is compact, one row per 32-row chunk.  A thread walks its chunk's rows in order, so
// the walkers are latency-bound: 4 columns per thread instead of 8 doubles
// the threads in flight here (0.048 -> 0.039 ms at T = 8192); the dL walker
// below is faster with 8 (0.046 against 0.053 ms).
constexpr int kInFlightOps = 8;
constexpr int kWalkOps = 4;
constexpr int kWalkDl = 8;
template <int VW>
__global__ void __launch_bounds__(kThreadsScan, 4)
    chunk_scan_operands_kernel(const __nv_bfloat16* __restrict__ g,
                               const __nv_bfloat16* __restrict__ q,
                               const __nv_bfloat16* __restrict__ k,
                               const float* __restrict__ scratch, float* __restrict__ P, long C,
                               Seqs seqs, int HQ, int H, int K, __nv_bfloat16* __restrict__ qh,
                               __nv_bfloat16* __restrict__ kh, float* __restrict__ anchors,
                               int* __restrict__ units) {
  constexpr int BA = 128;  // anchor block rows of the tensor-core kernels
  __shared__ int s_blk_off;
  int s, kc;
  if (!seq_block(seqs, kChunk, (int)blockIdx.x, s, kc)) return;  // uniform in the CTA
  const long start = seqs.start(s);
  const long len = seqs.len(s);
  const long lr0 = (long)kc * kChunk;
  if (lr0 >= len) return;  // uniform in the CTA
  if (threadIdx.x == 0) {
    int off = 0;
    if (seqs.cu) {
      for (int x = 0; x < s; ++x) off += (seqs.len(x) + BA - 1) / BA;
    } else {
      off = s * ((seqs.T + BA - 1) / BA);
    }
    s_blk_off = off;
  }
  __syncthreads();
  const long col = ((long)blockIdx.y * kThreadsScan + threadIdx.x) * VW;
  if (col >= C) return;
  const int n = (int)min((long)kChunk, len - lr0);
  const int hh = (int)(col / K), n0 = (int)(col % K);
  const int G = HQ / H;
  // R: the anchor of the 128-row block this chunk lies in (the scratch is
  // compact: one row per chunk, chunk kc of this sequence at blockIdx.x)
  const long lb = (lr0 / BA) * BA;
  float R[VW];
  {
    const float* cb = scratch + ((long)blockIdx.x - kc + lb / kChunk) * C + col;
    float gb[VW];
    loadw<VW>(g + (start + lb) * C + col, gb);
#pragma unroll
    for (int v = 0; v < VW; ++v) R[v] = floorf(fmaf(kInvLn2, cb[v] + gb[v], 0.f));
  }
  float acc[VW], cmp[VW];
  {
    const float* c = scratch + (long)blockIdx.x * C + col;
#pragma unroll
    for (int v = 0; v < VW; ++v) {
      acc[v] = c[v];
      cmp[v] = 0.f;
    }
  }
  bool wide = false;  // some exponent of this thread's rows beyond kAnchorRange
#pragma unroll
  for (int r0 = 0; r0 < kChunk; r0 += kInFlightOps) {
    float a[kInFlightOps][VW], qa[kInFlightOps][VW], ka[kInFlightOps][VW];
#pragma unroll
    for (int r = 0; r < kInFlightOps; ++r) {
      const long pr = start + lr0 + (r0 + r < n ? r0 + r : 0);
      loadw<VW>(g + pr * C + col, a[r]);
      loadw<VW>(q + pr * C + col, qa[r]);
      loadw<VW>(k + (pr * H + hh / G) * K + n0, ka[r]);
    }
#pragma unroll
    for (int rr = 0; rr < kInFlightOps; ++rr) {
      const int r = r0 + rr;
      const long lr = lr0 + r;
      const long pr = start + lr;
      float o[VW];
#pragma unroll
      for (int v = 0; v < VW; ++v) {
        const float yk = a[rr][v] - cmp[v];
        const float tk = acc[v] + yk;
        cmp[v] = (tk - acc[v]) - yk;
        acc[v] = tk;
        o[v] = fmaf(kInvLn2, acc[v], 0.f);
      }
      if (r < n) {
        storew<VW>(P + pr * C + col, o);
        float e[VW], y[VW];
#pragma unroll
        for (int v = 0; v < VW; ++v) {
          e[v] = o[v] - R[v];
          wide |= fabsf(e[v]) > kAnchorRange;
          y[v] = saturate_bf16(qa[rr][v] * exp2f(e[v]));
        }
        storew<VW>(qh + pr * C + col, y);
#pragma unroll
        for (int v = 0; v < VW; ++v) y[v] = saturate_bf16(ka[rr][v] * exp2f(-e[v]));
        storew<VW>(kh + pr * C + col, y);
        if (lr == lb)
          storew<VW>(anchors + ((long)(s_blk_off + lr / BA) * HQ + hh) * K + n0, R);
      }
    }
  }
  if (wide) {
    set_flag(units + (long)s * HQ + hh);
    set_flag(units + (long)seqs.n * HQ);  // some unit is flagged
  }
}

// The backward's dq finalize fused with pass 1 of the reverse scan of dL
// (tensor-core path): per (sequence, chunk in reverse order, VW columns of
// one query head), for each row
//   dq = scale * 2^(P - R_I) (.) dq32          R_I = floor(P at the row's
//                                              128-row block start)
//   dL = q (.) dq - k (.) dk^(h)               (fp32, written over dq32)
// and the chunk's compensated sum of dL in the order chunk_sum_kernel adds
// it, into the chunk row of `scratch` (dk^(h) itself: this thread has read
// that row's dk^(h) by then, and no other thread reads this chunk's rows).
// For a (sequence, head) unit flagged in `units` the SIMT kernels have
// written the final dq into dq32, so its factor is not applied.
template <int VW>
__global__ void __launch_bounds__(kThreadsScan, 4)
    finalize_dl_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                       const float* __restrict__ P, float* __restrict__ dq32,
                       const float* __restrict__ dkh32, float* __restrict__ scratch,
                       __nv_bfloat16* __restrict__ dq, long C, Seqs seqs, int HQ, int H, int K,
                       float scale, const int* __restrict__ units) {
  constexpr int BA = 128;
  int s, kc;
  if (!seq_block(seqs, kChunk, (int)blockIdx.x, s, kc)) return;
  const long start = seqs.start(s);
  const long len = seqs.len(s);
  const long lr0 = (long)kc * kChunk;
  if (lr0 >= len) return;
  const long col = ((long)blockIdx.y * kThreadsScan + threadIdx.x) * VW;
  if (col >= C) return;
  const int n = (int)min((long)kChunk, len - lr0);
  const int hh = (int)(col / K), n0 = (int)(col % K);
  const int G = HQ / H;
  const bool final_dq = units[(long)s * HQ + hh] != 0;
  float sum[VW], cmp[VW];
#pragma unroll
  for (int v = 0; v < VW; ++v) sum[v] = cmp[v] = 0.f;
#pragma unroll 1
  for (int r0 = 0; r0 < kChunk; r0 += kInFlightOps) {
    float dl[kInFlightOps][VW];
#pragma unroll
    for (int r = 0; r < kInFlightOps; ++r) {
      const bool in = r0 + r < n;
      const long lr = lr0 + (in ? r0 + r : 0);
      const long pr = start + len - 1 - lr;  // reverse scan order
      const long off = pr * C + col;
      const long arow = start + ((pr - start) / BA) * BA;
      float pv[VW], rv[VW], a[VW], qq[VW], kk[VW], dkv[VW];
      loadw<VW>(P + off, pv);
      loadw<VW>(P + arow * C + col, rv);
      loadw<VW>(dq32 + off, a);
      loadw<VW>(q + off, qq);
      loadw<VW>(k + (pr * H + hh / G) * K + n0, kk);
      loadw<VW>(dkh32 + off, dkv);
      float o[VW];
#pragma unroll
      for (int v = 0; v < VW; ++v) {
        if (!final_dq) a[v] *= scale * exp2f(pv[v] - floorf(rv[v]));
        o[v] = qq[v] * a[v] - kk[v] * dkv[v];
        dl[r][v] = in ? o[v] : 0.f;
      }
      if (in) {
        storew<VW>(dq + off, a);
        storew<VW>(dq32 + off, o);
      }
    }
#pragma unroll
    for (int r = 0; r < kInFlightOps; ++r) {
#pragma unroll
      for (int v = 0; v < VW; ++v) {
        const float yk = dl[r][v] - cmp[v];
        const float tk = sum[v] + yk;
        cmp[v] = (tk - sum[v]) - yk;
        sum[v] = tk;
      }
    }
  }
  float* dst = scratch + chunk_row(start, len, kc, true) * C + col;
#pragma unroll
  for (int v = 0; v < VW; ++v) dst[v] = sum[v];
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

// Few columns (the scalar gate's scans, C = HQ): the three passes in one CTA
// per sequence, one launch instead of three.  Thread (part p, group of four
// columns) sums rows [p R, (p + 1) R) of its sequence in fp64; the parts'
// sums get their exclusive carries by a fixed-order Hillis-Steele scan over
// the parts in shared memory (fp64); each thread then scans its rows again
// from its carry.  Used while every sequence fits one CTA (all rows <=
// kSmallRows: at most kSmallRows / parts rows per thread).
constexpr int kSmallThreads = 1024;
constexpr long kSmallRows = 65536;
constexpr int kSmallMaxC = 64;

template <bool kReverse>
__global__ void __launch_bounds__(kSmallThreads)
    scan_small_kernel(const float* __restrict__ x, float* __restrict__ y, int C, Seqs seqs) {
  extern __shared__ double sm_small[];  // two buffers of [parts][C]
  const int s = blockIdx.x;
  const long start = seqs.start(s), len = seqs.len(s);
  const int ng = C / 4;                        // float4 groups per row
  const int parts = kSmallThreads / ng;
  const int tid = threadIdx.x, g = tid % ng, p = tid / ng;
  const bool active = p < parts;
  const long R = (len + parts - 1) / parts;
  const long r0 = active ? min(len, (long)p * R) : len;
  const long r1 = min(len, r0 + R);
  auto row_of = [&](long r) { return kReverse ? start + len - 1 - r : start + r; };
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (long r = r0; r < r1; ++r) {
    const float4 v = *reinterpret_cast<const float4*>(x + row_of(r) * C + g * 4);
    acc[0] += v.x;
    acc[1] += v.y;
    acc[2] += v.z;
    acc[3] += v.w;
  }
  // inclusive scan of the parts' sums, per column, then shifted to exclusive
  double* buf[2] = {sm_small, sm_small + (long)parts * C};
  const long slot = (long)p * C + g * 4;
  if (active)
    for (int e = 0; e < 4; ++e) buf[0][slot + e] = acc[e];
  __syncthreads();
  int cur = 0;
  for (int off = 1; off < parts; off <<= 1) {
    if (active)
      for (int e = 0; e < 4; ++e)
        buf[cur ^ 1][slot + e] =
            buf[cur][slot + e] + (p >= off ? buf[cur][slot - (long)off * C + e] : 0.0);
    __syncthreads();
    cur ^= 1;
  }
  if (!active || r0 >= r1) return;
  double run[4];
  for (int e = 0; e < 4; ++e) run[e] = p > 0 ? buf[cur][slot - C + e] : 0.0;
  for (long r = r0; r < r1; ++r) {
    const long pr = row_of(r);
    const float4 v = *reinterpret_cast<const float4*>(x + pr * C + g * 4);
    run[0] += v.x;
    run[1] += v.y;
    run[2] += v.z;
    run[3] += v.w;
    *reinterpret_cast<float4*>(y + pr * C + g * 4) =
        make_float4((float)run[0], (float)run[1], (float)run[2], (float)run[3]);
  }
}

// fp32 in and out, no carries, small C: the one-launch scan applies
bool small_scan_ok(const float* x, const float* y, long C, const Seqs& seqs) {
  return C >= 4 && C <= kSmallMaxC && C % 4 == 0 && seqs.rows <= kSmallRows &&
         ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) % 16) == 0;
}

template <bool kReverse>
int launch_small_scan(const float* x, float* y, long C, const Seqs& seqs, cudaStream_t stream) {
  const int parts = kSmallThreads / (int)(C / 4);
  const size_t smem = 2 * sizeof(double) * (size_t)parts * C;
  static bool attr[2][kMaxDevices] = {};
  if (!set_max_smem_once(scan_small_kernel<kReverse>, (int)smem, attr[kReverse ? 1 : 0]))
    return WALL_ERR_CUDA;
  scan_small_kernel<kReverse><<<seqs.n, kSmallThreads, smem, stream>>>(x, y, (int)C, seqs);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
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

int scan_prefix_operands(const __nv_bfloat16* g, const __nv_bfloat16* q, const __nv_bfloat16* k,
                         float* P, float* scratch, int HQ, int H, int K, const Seqs& seqs,
                         __nv_bfloat16* qh, __nv_bfloat16* kh, float* anchors, int* units,
                         cudaStream_t stream) {
  const long C = (long)HQ * K;
  if (seqs.n == 0 || C == 0) return WALL_OK;
  if (C % 8 != 0) return WALL_ERR_UNSUPPORTED;
  const long groups = (C / 8 + kThreadsScan - 1) / kThreadsScan;
  const long wgroups = (C / kWalkOps + kThreadsScan - 1) / kThreadsScan;
  const long chunks = seqs.cu ? (seqs.rows + kChunk - 1) / kChunk + seqs.n
                              : (long)seqs.n * ((seqs.T + kChunk - 1) / kChunk);
  if (wgroups > 65535 || chunks > 0x7fffffffL || seqs.n > 65535) return WALL_ERR_UNSUPPORTED;
  if (chunks == 0) return WALL_OK;
  const dim3 grid((unsigned)chunks, (unsigned)groups);
  timing_mark(T_PREFIX, stream);
  chunk_sum_kernel<__nv_bfloat16, 8, false><<<grid, kThreadsScan, 0, stream>>>(
      g, scratch, C, seqs, units, seqs.n * HQ + 1, /*compact=*/true);
  const dim3 cgrid((unsigned)((C + 31) / 32), (unsigned)seqs.n);
  carry_kernel<false><<<cgrid, 32 * kCarryParts, 0, stream>>>(scratch, C, seqs, kInvLn2, nullptr,
                                                              nullptr, /*compact=*/true);
  timing_mark(T_PREFIX, stream);
  timing_mark(T_OPERANDS, stream);
  chunk_scan_operands_kernel<kWalkOps>
      <<<dim3((unsigned)chunks, (unsigned)wgroups), kThreadsScan, 0, stream>>>(
          g, q, k, scratch, P, C, seqs, HQ, H, K, qh, kh, anchors, units);
  timing_mark(T_OPERANDS, stream);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

int finalize_dq_dl_sums(const __nv_bfloat16* q, const __nv_bfloat16* k, const float* P,
                        float* dq32, float* dkh32, __nv_bfloat16* dq, int HQ, int H, int K,
                        float scale, const Seqs& seqs, const int* units, cudaStream_t stream) {
  const long C = (long)HQ * K;
  if (seqs.n == 0 || C == 0) return WALL_OK;
  if (C % 8 != 0) return WALL_ERR_UNSUPPORTED;
  const long wgroups = (C / kWalkDl + kThreadsScan - 1) / kThreadsScan;
  const long chunks = seqs.cu ? (seqs.rows + kChunk - 1) / kChunk + seqs.n
                              : (long)seqs.n * ((seqs.T + kChunk - 1) / kChunk);
  if (wgroups > 65535 || chunks > 0x7fffffffL || seqs.n > 65535) return WALL_ERR_UNSUPPORTED;
  if (chunks == 0) return WALL_OK;
  finalize_dl_kernel<kWalkDl>
      <<<dim3((unsigned)chunks, (unsigned)wgroups), kThreadsScan, 0, stream>>>(
          q, k, P, dq32, dkh32, dkh32, dq, C, seqs, HQ, H, K, scale, units);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

int scan_reverse_from_sums(const float* x, void* y, int out_dtype, float* scratch, long C,
                           const Seqs& seqs, cudaStream_t stream) {
  if (seqs.n == 0 || C == 0) return WALL_OK;
  if (C % 8 != 0 || ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y) |
                      reinterpret_cast<uintptr_t>(scratch)) % 16) != 0)
    return WALL_ERR_UNSUPPORTED;
  const long groups = (C / 8 + kThreadsScan - 1) / kThreadsScan;
  const long chunks = seqs.cu ? (seqs.rows + kChunk - 1) / kChunk + seqs.n
                              : (long)seqs.n * ((seqs.T + kChunk - 1) / kChunk);
  if (groups > 65535 || chunks > 0x7fffffffL || seqs.n > 65535) return WALL_ERR_UNSUPPORTED;
  if (chunks == 0) return WALL_OK;
  const dim3 grid((unsigned)chunks, (unsigned)groups);
  const dim3 cgrid((unsigned)((C + 31) / 32), (unsigned)seqs.n);
  carry_kernel<true><<<cgrid, 32 * kCarryParts, 0, stream>>>(scratch, C, seqs, 1.f, nullptr,
                                                             nullptr);
  if (out_dtype == WALL_BF16)
    chunk_scan_kernel<float, __nv_bfloat16, 8, true><<<grid, kThreadsScan, 0, stream>>>(
        x, static_cast<__nv_bfloat16*>(y), scratch, C, seqs, 1.f, nullptr);
  else
    chunk_scan_kernel<float, float, 8, true><<<grid, kThreadsScan, 0, stream>>>(
        x, static_cast<float*>(y), scratch, C, seqs, 1.f, nullptr);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

int scan_prefix_plain(const float* x, float* y, long C, const Seqs& seqs, cudaStream_t stream) {
  if (seqs.n == 0 || C == 0) return WALL_OK;
  if (small_scan_ok(x, y, C, seqs)) return launch_small_scan<false>(x, y, C, seqs, stream);
  return launch_scan<float, float, false>(x, y, y, C, seqs, 1.f, nullptr, nullptr, stream);
}

int scan_reverse(const float* x, void* y, int out_dtype, float* scratch, long C, const Seqs& seqs,
                 cudaStream_t stream) {
  if (seqs.n == 0 || C == 0) return WALL_OK;
  if (out_dtype == WALL_FP32 && small_scan_ok(x, static_cast<float*>(y), C, seqs))
    return launch_small_scan<true>(x, static_cast<float*>(y), C, seqs, stream);
  if (out_dtype == WALL_BF16)
    return launch_scan<float, __nv_bfloat16, true>(x, static_cast<__nv_bfloat16*>(y), scratch, C,
                                                   seqs, 1.f, nullptr, nullptr, stream);
  return launch_scan<float, float, true>(x, static_cast<float*>(y), scratch, C, seqs, 1.f,
                                         nullptr, nullptr, stream);
}

}  // namespace wall
