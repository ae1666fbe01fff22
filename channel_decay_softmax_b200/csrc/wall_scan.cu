// wall_scan.cu -- segmented prefix scans along time.
//
// Forward scan: the base-2 gate prefix P = cumsum(g) / ln 2 (README "Decode":
// the prefix is the cumulative sum of g with scale 1/ln 2).  Reverse scan:
// the gate gradient dg_u = sum_{t >= u} dL_t within a sequence, the adjoint
// of that prefix, and the same for the scalar gate.
//
// Design (HBM-bound, 2 B in + 4 B out per element for bf16 -> fp32): a
// thread-block cluster of kCS CTAs owns one (sequence, 64-column group).
// Each CTA takes 256 rows of a 256*kCS-row super-tile; each of its threads
// holds 64 consecutive rows of one column in registers, so every element is
// read once.  Per-part and per-CTA column totals are combined through shared
// memory and the cluster's distributed shared memory, then each thread scans
// its registers and writes the result.  A running carry crosses super-tiles.
#include <cooperative_groups.h>

#include "wall_common.cuh"
#include "wall_internal.h"

namespace cg = cooperative_groups;

namespace wall {

constexpr int kCS = 8;          // CTAs per cluster
constexpr int kCols = 64;       // columns per cluster
constexpr int kParts = 4;       // row parts per CTA
constexpr int kRowsPerThread = 64;
constexpr int kRowsPerCta = kParts * kRowsPerThread;  // 256

template <typename Tin, typename Tout, bool kReverse>
__global__ void __launch_bounds__(kCols * kParts)
    scan_kernel(const Tin* __restrict__ x, Tout* __restrict__ y, long C, Seqs seqs, float mul,
                const float* __restrict__ carry_in, float* __restrict__ carry_out) {
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ float part_tot[kParts][kCols];
  __shared__ float cta_tot[2][kCols];

  const int rank = (int)cluster.block_rank();
  const int c = threadIdx.x % kCols;
  const int part = threadIdx.x / kCols;
  const long col = (long)blockIdx.y * kCols + c;
  const bool valid = col < C;
  const int s = blockIdx.z;
  const long start = seqs.start(s);
  const long len = seqs.len(s);

  const float cin = (carry_in != nullptr && valid) ? carry_in[(long)s * C + col] : 0.f;
  float run_hi = 0.f, run_lo = 0.f;  // compensated raw sum of the finished super-tiles
  int buf = 0;
  for (long base = 0; base < len; base += (long)kCS * kRowsPerCta, buf ^= 1) {
    const long row0 = base + (long)rank * kRowsPerCta + (long)part * kRowsPerThread;
    float vals[kRowsPerThread];
    float sum = 0.f, sum_c = 0.f;  // compensated (Kahan) sum of this thread's rows
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r) {
      const long lr = row0 + r;
      float v = 0.f;
      if (valid && lr < len) {
        const long pr = kReverse ? start + len - 1 - lr : start + lr;
        v = to_f32(x[pr * C + col]);
      }
      vals[r] = v;
      const float yk = v - sum_c;
      const float tk = sum + yk;
      sum_c = (tk - sum) - yk;
      sum = tk;
    }
    part_tot[part][c] = sum;
    __syncthreads();
    float pre_part = 0.f, cta_total = 0.f;
#pragma unroll
    for (int p = 0; p < kParts; ++p) {
      const float t = part_tot[p][c];
      if (p < part) pre_part += t;
      cta_total += t;
    }
    if (part == 0) cta_tot[buf][c] = cta_total;
    cluster.sync();
    float pre_cta = 0.f, super_total = 0.f;
    for (int r = 0; r < kCS; ++r) {
      const float* remote = cluster.map_shared_rank(&cta_tot[buf][c], r);
      const float t = *remote;
      if (r < rank) pre_cta += t;
      super_total += t;
    }
    // running compensated sum: acc + acc_c carries the prefix of this row
    float acc = run_hi + pre_cta + pre_part, acc_c = run_lo;
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r) {
      const long lr = row0 + r;
      const float yk = vals[r] - acc_c;
      const float tk = acc + yk;
      acc_c = (tk - acc) - yk;
      acc = tk;
      if (valid && lr < len) {
        const long pr = kReverse ? start + len - 1 - lr : start + lr;
        y[pr * C + col] = from_f32<Tout>(cin + mul * acc);
      }
    }
    {  // run (two-float) += super_total
      const float yk = super_total - run_lo;
      const float tk = run_hi + yk;
      run_lo = (tk - run_hi) - yk;
      run_hi = tk;
    }
  }
  if (carry_out != nullptr && valid && rank == 0 && part == 0)
    carry_out[(long)s * C + col] = cin + mul * (run_hi - run_lo);
  // keep this CTA's shared memory alive until every peer finished reading it
  cluster.sync();
}

template <typename Tin, typename Tout, bool kReverse>
static int launch_scan(const Tin* x, Tout* y, long C, const Seqs& seqs, float mul,
                       const float* carry_in, float* carry_out, cudaStream_t stream) {
  if (seqs.n == 0 || C == 0) return WALL_OK;
  long ny = (C + kCols - 1) / kCols;
  if (ny > 65535 || seqs.n > 65535) return WALL_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kCS, (unsigned)ny, (unsigned)seqs.n);
  cfg.blockDim = dim3(kCols * kParts);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, scan_kernel<Tin, Tout, kReverse>, x, y, C, seqs, mul,
                                     carry_in, carry_out);
  return e == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

int scan_prefix_log2(const void* g, int dtype, float* P, long C, const Seqs& seqs,
                     const float* carry_in, float* carry_out, cudaStream_t stream) {
  if (dtype == WALL_BF16)
    return launch_scan<__nv_bfloat16, float, false>(static_cast<const __nv_bfloat16*>(g), P, C,
                                                    seqs, kInvLn2, carry_in, carry_out, stream);
  return launch_scan<float, float, false>(static_cast<const float*>(g), P, C, seqs, kInvLn2,
                                          carry_in, carry_out, stream);
}

int scan_prefix_plain(const float* x, float* y, long C, const Seqs& seqs, cudaStream_t stream) {
  return launch_scan<float, float, false>(x, y, C, seqs, 1.f, nullptr, nullptr, stream);
}

int scan_reverse(const float* x, void* y, int out_dtype, long C, const Seqs& seqs,
                 cudaStream_t stream) {
  if (out_dtype == WALL_BF16)
    return launch_scan<float, __nv_bfloat16, true>(x, static_cast<__nv_bfloat16*>(y), C, seqs,
                                                   1.f, nullptr, nullptr, stream);
  return launch_scan<float, float, true>(x, static_cast<float*>(y), C, seqs, 1.f, nullptr,
                                         nullptr, stream);
}

}  // namespace wall
