// wall_attn_simt.cu -- fp32 CUDA-core Wall Attention forward and backward.
//
// This path computes with fp32 products throughout (no tensor cores), which
// is what fp32 inputs need to meet a 1e-5 error bound; it also carries every
// option (GQA, g_scalar, sink, window, varlen) for any head size up to 128.
// The same kernels, given a mask of (sequence, head) units, recompute the
// units the tensor-core path cannot represent (see wall_attn_fwd_sm100.cu).
//
// Per tile the decay exp2(P_i - P_j) (blog "Wall Attention", factorised
// form with base-2 prefix) is split with one anchor R per CTA (blog, fast
// training: per-block anchor, exp2(P_i - P_j) = exp2(P_i - R) exp2(R - P_j)),
// placed on the CTA block's boundary that faces the streamed operand:
//   forward / dq:  R = P at the CTA's first query row; the query tile is
//                  rescaled once by exp2(P_i - R), each key tile by
//                  exp2(R - P_j) as it is loaded.
//   dk / dv:       R = P at the CTA's last key row; the roles swap.
// Off the diagonal tile the anchor then lies between every key and every
// query, so for a decaying gate both factors are at most 1 (about 2 with
// rounding): they can only underflow, and only where the exact product is
// below 2^-126 as well, however strong the decay.  The diagonal tile pairs
// rows of the CTA's own block, where one factor grows by the block's whole
// accumulated gate; when that exceeds 2^kSpanExact on some channel the CTA
// evaluates its diagonal tile pair by pair, exp2(P_in - P_jn) per channel.
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

constexpr int BM = 64;
constexpr int BN = 64;
constexpr int kThreads = 256;
// anchored factors beyond 2^+-kSpanExact switch the diagonal tile to pairs
constexpr float kSpanExact = 60.f;

struct TileGeom {
  int seq, blk;
  long s0;  // first row of the sequence (flattened)
  int L;    // sequence length
};

__device__ __forceinline__ float warp4_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
  return x;
}
__device__ __forceinline__ float warp4_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

// Visible iff j <= i and (no window or i - j < window); i, j relative to the
// sequence start.
__device__ __forceinline__ bool visible(int i, int j, int window) {
  return j <= i && (window <= 0 || i - j < window);
}

// Work item -> (sequence, 64-row block, query head).  The kernels run a
// persistent grid over items; with a unit mask only the items of flagged
// (sequence, head) units are taken.  `reverse` hands out the last blocks of
// the flat order first (the longest query blocks of a causal problem).
__device__ __forceinline__ bool simt_item(const AttnProblem& pb, int item, bool reverse,
                                          int& seq, int& blk, int& h) {
  h = item % pb.HQ;
  const int b = item / pb.HQ;
  if (!seq_block(pb.seqs, BM, reverse ? pb.max_blocks64 - 1 - b : b, seq, blk)) return false;
  return pb.units == nullptr || pb.units[(long)seq * pb.HQ + h] != 0;
}

// dst[r][n] = src[row0+r, src_head, n] * exp2(sign * (P[row0+r, h, n] - R[n]))
// for sign = +1 or -1, or the raw element for sign = 0.  Returns true (in this
// thread) when some loaded |P - R| exceeds kSpanExact.
template <typename T, int KD>
__device__ __forceinline__ bool load_rows_anchored(float* dst, const T* src, const float* P,
                                                   const float* R, long row0, int nrows,
                                                   int nmax, int src_heads, int src_head,
                                                   int HQ, int h, int K, int sign) {
  bool wide = false;
  for (int e = threadIdx.x; e < nmax * KD; e += kThreads) {
    const int r = e / KD, n = e % KD;
    float val = 0.f;
    if (r < nrows && n < K) {
      const long row = row0 + r;
      val = to_f32(src[(row * src_heads + src_head) * (long)K + n]);
      if (sign != 0) {
        const float d = P[(row * HQ + h) * (long)K + n] - R[n];
        wide |= fabsf(d) > kSpanExact;
        val *= exp2f(sign > 0 ? d : -d);
      }
    }
    dst[r * (KD + 1) + n] = val;
  }
  return wide;
}

// sum_n x_n y_n 2^(pa_n - pb_n) over the K channels of two rows, x from
// shared memory (stride 1) and y, pa, pb from global memory: one pair of the
// diagonal tile evaluated without an anchor.
template <typename T>
__device__ __forceinline__ float exact_dot(const float* xs, const T* y, const float* pa,
                                           const float* pb, int K) {
  float acc = 0.f;
  for (int n = 0; n < K; ++n) acc += xs[n] * to_f32(y[n]) * exp2f(pa[n] - pb[n]);
  return acc;
}

template <typename T, int VD, int PAD>
__device__ __forceinline__ void load_rows_plain(float* dst, const T* src, long row0, int nrows,
                                                int nmax, int heads, int head, int V) {
  for (int e = threadIdx.x; e < nmax * VD; e += kThreads) {
    const int r = e / VD, c = e % VD;
    float val = 0.f;
    if (r < nrows && c < V) val = to_f32(src[((row0 + r) * heads + head) * (long)V + c]);
    dst[r * (VD + PAD) + c] = val;
  }
}

// ---------------------------------------------------------------------------
// forward

template <typename T, int KD, int VD>
__device__ __forceinline__ void fwd_simt_block(const AttnProblem& pb, const FwdArgs& a, float* sm,
                                               int seq, int blk, int h) {
  float* qt = sm;                      // [BM][KD+1]
  float* kt = qt + BM * (KD + 1);      // [BN][KD+1]
  float* vs = kt + BN * (KD + 1);      // [BN][VD]
  float* Ss = vs + BN * VD;            // [BM][BN+1]
  float* R = Ss + BM * (BN + 1);       // [KD]
  float* gsq = R + KD;                 // [BM]
  float* gsk = gsq + BM;               // [BN]

  const int kh = h / (pb.HQ / pb.H);
  const long s0 = pb.seqs.start(seq);
  const int L = pb.seqs.len(seq);
  const int i0 = blk * BM;
  const int ni = min(BM, L - i0);
  const int K = pb.K, V = pb.V, HQ = pb.HQ;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);

  for (int n = threadIdx.x; n < KD; n += kThreads)
    R[n] = n < K ? a.P[((s0 + i0) * HQ + h) * (long)K + n] : 0.f;
  __syncthreads();
  const bool wide = load_rows_anchored<T, KD>(qt, q, a.P, R, s0 + i0, ni, BM, HQ, h, HQ, h, K, 1);
  for (int r = threadIdx.x; r < BM; r += kThreads)
    gsq[r] = (a.GS && r < ni) ? a.GS[(s0 + i0 + r) * HQ + h] : 0.f;
  // every thread's flag reaches the whole CTA (this also orders the loads)
  const bool exact = __syncthreads_or(wide) != 0;

  const int row = threadIdx.x / 4, sub = threadIdx.x % 4;
  float m = -INFINITY, l = 0.f;
  float acc[VD / 4];
#pragma unroll
  for (int c = 0; c < VD / 4; ++c) acc[c] = 0.f;

  const int jlast = i0 + ni - 1;
  const int jfirst = pb.window > 0 ? max(0, i0 - pb.window + 1) : 0;
  const float sl2 = pb.scale * kLog2e;
  const long qrow = (s0 + i0 + min(row, ni - 1)) * HQ + h;
  for (int jb = jfirst / BN; jb <= jlast / BN; ++jb) {
    const int j0 = jb * BN;
    const int nj = min(BN, L - j0);
    // the diagonal tile of a wide block: raw keys, pair-by-pair decay
    const bool pairwise = exact && j0 == i0;
    __syncthreads();
    load_rows_anchored<T, KD>(kt, k, a.P, R, s0 + j0, nj, BN, pb.H, kh, HQ, h, K,
                              pairwise ? 0 : -1);
    load_rows_plain<T, VD, 0>(vs, v, s0 + j0, nj, BN, pb.H, kh, V);
    for (int r = threadIdx.x; r < BN; r += kThreads)
      gsk[r] = (a.GS && r < nj) ? a.GS[(s0 + j0 + r) * HQ + h] : 0.f;
    __syncthreads();

    float sc[BN / 4];
#pragma unroll
    for (int jj = 0; jj < BN / 4; ++jj) sc[jj] = 0.f;
    if (!pairwise) {
      for (int n = 0; n < KD; ++n) {
        const float qv = qt[row * (KD + 1) + n];
#pragma unroll
        for (int jj = 0; jj < BN / 4; ++jj) sc[jj] += qv * kt[(sub + 4 * jj) * (KD + 1) + n];
      }
    } else {
#pragma unroll 1
      for (int jj = 0; jj < BN / 4; ++jj) {
        const int jl = min(sub + 4 * jj, nj - 1);
        sc[jj] = exact_dot(kt + jl * (KD + 1), q + qrow * K, a.P + qrow * K,
                           a.P + ((s0 + j0 + jl) * HQ + h) * (long)K, K);
      }
    }
    const int i = i0 + row;
    float mt = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < BN / 4; ++jj) {
      const int jl = sub + 4 * jj;
      const bool vis = row < ni && jl < nj && visible(i, j0 + jl, pb.window);
      sc[jj] = vis ? sc[jj] * sl2 + (gsq[row] - gsk[jl]) * kLog2e : -INFINITY;
      mt = fmaxf(mt, sc[jj]);
    }
    mt = warp4_max(mt);
    const float m_new = fmaxf(m, mt);
    const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = exp2f(m - m_use);
    float ls = 0.f;
#pragma unroll
    for (int jj = 0; jj < BN / 4; ++jj) {
      const float p = exp2f(sc[jj] - m_use);
      ls += p;
      Ss[row * (BN + 1) + sub + 4 * jj] = p;
    }
    ls = warp4_sum(ls);
    l = l * alpha + ls;
    m = m_new;
#pragma unroll
    for (int c = 0; c < VD / 4; ++c) acc[c] *= alpha;
    __syncwarp();
    for (int j = 0; j < BN; ++j) {
      const float p = Ss[row * (BN + 1) + j];
#pragma unroll
      for (int c = 0; c < VD / 4; ++c) acc[c] += p * vs[j * VD + sub + 4 * c];
    }
  }
  if (a.sink) {
    const float s2 = a.sink[h] * kLog2e;
    const float m_new = fmaxf(m, s2);
    const float alpha = exp2f(m - m_new);
    l = l * alpha + exp2f(s2 - m_new);
#pragma unroll
    for (int c = 0; c < VD / 4; ++c) acc[c] *= alpha;
    m = m_new;
  }
  if (row < ni) {
    const long orow = (s0 + i0 + row) * HQ + h;
    T* o = static_cast<T*>(a.o);
    const float inv = 1.f / l;
#pragma unroll
    for (int c = 0; c < VD / 4; ++c) {
      const int cc = sub + 4 * c;
      if (cc < V) o[orow * V + cc] = from_f32<T>(acc[c] * inv);
    }
    if (sub == 0 && a.lse) a.lse[orow] = (m + log2f(l)) * kLn2;
  }
}

// With a unit mask, nothing to do unless some unit is flagged: the mask's
// last word (after the n_seq * HQ unit words) is set with any of them.
__device__ __forceinline__ bool no_flagged_units(const AttnProblem& pb) {
  return pb.units != nullptr &&
         !__syncthreads_or(threadIdx.x == 0 && pb.units[(long)pb.seqs.n * pb.HQ] != 0);
}

template <typename T, int KD, int VD>
__global__ void __launch_bounds__(kThreads) fwd_simt_kernel(AttnProblem pb, FwdArgs a) {
  extern __shared__ float sm[];
  if (no_flagged_units(pb)) return;
  const int n_items = pb.max_blocks64 * pb.HQ;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    int seq, blk, h;
    if (!simt_item(pb, item, true, seq, blk, h)) continue;  // uniform in the CTA
    __syncthreads();  // the previous item's shared-memory reads are done
    fwd_simt_block<T, KD, VD>(pb, a, sm, seq, blk, h);
  }
}

// ---------------------------------------------------------------------------
// backward, query side: D_i, dq, row part of the scalar-gate gradient (dsink
// follows from D in sink_grad; with a unit mask: dq only, D and the row part
// come from the tensor-core path's own pass)

template <typename T, int KD, int VD>
__device__ __forceinline__ void bwd_dq_simt_block(const AttnProblem& pb, const BwdArgs& a,
                                                  float* sm, int seq, int blk, int h) {
  float* qt = sm;                      // [BM][KD+1]
  float* kt = qt + BM * (KD + 1);      // [BN][KD+1]
  float* vs = kt + BN * (KD + 1);      // [BN][VD+1]
  float* dOs = vs + BN * (VD + 1);     // [BM][VD+1]
  float* Ss = dOs + BM * (VD + 1);     // [BM][BN+1]
  float* R = Ss + BM * (BN + 1);       // [KD]
  float* gsq = R + KD;                 // [BM]
  float* gsk = gsq + BM;               // [BN]
  float* lse2 = gsk + BN;              // [BM]
  float* Dv = lse2 + BM;               // [BM]

  const bool own_rows = pb.units == nullptr;
  const int kh = h / (pb.HQ / pb.H);
  const long s0 = pb.seqs.start(seq);
  const int L = pb.seqs.len(seq);
  const int i0 = blk * BM;
  const int ni = min(BM, L - i0);
  const int K = pb.K, V = pb.V, HQ = pb.HQ;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  const T* dO = static_cast<const T*>(a.dO);
  const T* o = static_cast<const T*>(a.o);

  for (int n = threadIdx.x; n < KD; n += kThreads)
    R[n] = n < K ? a.P[((s0 + i0) * HQ + h) * (long)K + n] : 0.f;
  __syncthreads();
  const bool wide = load_rows_anchored<T, KD>(qt, q, a.P, R, s0 + i0, ni, BM, HQ, h, HQ, h, K, 1);
  load_rows_plain<T, VD, 1>(dOs, dO, s0 + i0, ni, BM, HQ, h, V);
  for (int r = threadIdx.x; r < BM; r += kThreads) {
    gsq[r] = (a.GS && r < ni) ? a.GS[(s0 + i0 + r) * HQ + h] : 0.f;
    lse2[r] = r < ni ? a.lse[(s0 + i0 + r) * HQ + h] * kLog2e : 0.f;
  }
  const bool exact = __syncthreads_or(wide) != 0;
  const int row = threadIdx.x / 4, sub = threadIdx.x % 4;
  {  // D_i = dO_i . o_i
    float d = 0.f;
    if (row < ni)
      for (int c = sub; c < V; c += 4)
        d += dOs[row * (VD + 1) + c] * to_f32(o[((s0 + i0 + row) * HQ + h) * (long)V + c]);
    d = warp4_sum(d);
    if (sub == 0) {
      Dv[row] = d;
      if (own_rows && row < ni) a.D[(s0 + i0 + row) * HQ + h] = d;
    }
  }
  __syncthreads();

  float dqa[KD / 4];
#pragma unroll
  for (int c = 0; c < KD / 4; ++c) dqa[c] = 0.f;
  float dqe[KD / 4];  // the diagonal tile's pairwise terms of a wide block
#pragma unroll
  for (int c = 0; c < KD / 4; ++c) dqe[c] = 0.f;
  double rowsum = 0.0;  // fp64: the scalar-gate gradient sums many cancelling terms
  const float Di = Dv[row];
  const int jlast = i0 + ni - 1;
  const int jfirst = pb.window > 0 ? max(0, i0 - pb.window + 1) : 0;
  const float sl2 = pb.scale * kLog2e;
  const long qrow = (s0 + i0 + min(row, ni - 1)) * HQ + h;
  for (int jb = jfirst / BN; jb <= jlast / BN; ++jb) {
    const int j0 = jb * BN;
    const int nj = min(BN, L - j0);
    const bool pairwise = exact && j0 == i0;
    __syncthreads();
    load_rows_anchored<T, KD>(kt, k, a.P, R, s0 + j0, nj, BN, pb.H, kh, HQ, h, K,
                              pairwise ? 0 : -1);
    load_rows_plain<T, VD, 1>(vs, v, s0 + j0, nj, BN, pb.H, kh, V);
    for (int r = threadIdx.x; r < BN; r += kThreads)
      gsk[r] = (a.GS && r < nj) ? a.GS[(s0 + j0 + r) * HQ + h] : 0.f;
    __syncthreads();
    float sc[BN / 4], dp[BN / 4];
#pragma unroll
    for (int jj = 0; jj < BN / 4; ++jj) sc[jj] = dp[jj] = 0.f;
    if (!pairwise) {
      for (int n = 0; n < KD; ++n) {
        const float qv = qt[row * (KD + 1) + n];
#pragma unroll
        for (int jj = 0; jj < BN / 4; ++jj) sc[jj] += qv * kt[(sub + 4 * jj) * (KD + 1) + n];
      }
    } else {
#pragma unroll 1
      for (int jj = 0; jj < BN / 4; ++jj) {
        const int jl = min(sub + 4 * jj, nj - 1);
        sc[jj] = exact_dot(kt + jl * (KD + 1), q + qrow * K, a.P + qrow * K,
                           a.P + ((s0 + j0 + jl) * HQ + h) * (long)K, K);
      }
    }
    for (int c = 0; c < VD; ++c) {
      const float dv_ = dOs[row * (VD + 1) + c];
#pragma unroll
      for (int jj = 0; jj < BN / 4; ++jj) dp[jj] += dv_ * vs[(sub + 4 * jj) * (VD + 1) + c];
    }
    const int i = i0 + row;
#pragma unroll
    for (int jj = 0; jj < BN / 4; ++jj) {
      const int jl = sub + 4 * jj;
      const bool vis = row < ni && jl < nj && visible(i, j0 + jl, pb.window);
      float ds = 0.f;
      if (vis) {
        const float s2 = sc[jj] * sl2 + (gsq[row] - gsk[jl]) * kLog2e;
        const float p = exp2f(s2 - lse2[row]);
        ds = p * (dp[jj] - Di);
      }
      rowsum += ds;
      Ss[row * (BN + 1) + jl] = ds;
    }
    __syncwarp();
    if (!pairwise) {
      for (int j = 0; j < BN; ++j) {
        const float ds = Ss[row * (BN + 1) + j];
#pragma unroll
        for (int c = 0; c < KD / 4; ++c) dqa[c] += ds * kt[j * (KD + 1) + sub + 4 * c];
      }
    } else {
      // dq_in += dS_ij k_jn 2^(P_in - P_jn), pair by pair
      for (int j = 0; j < nj; ++j) {
        const float ds = Ss[row * (BN + 1) + j];
        if (ds == 0.f) continue;
        const float* pj = a.P + ((s0 + j0 + j) * HQ + h) * (long)K;
#pragma unroll
        for (int c = 0; c < KD / 4; ++c) {
          const int n = sub + 4 * c;
          if (n < K)
            dqe[c] += ds * kt[j * (KD + 1) + n] * exp2f(a.P[qrow * K + n] - pj[n]);
        }
      }
    }
  }
  rowsum += __shfl_xor_sync(0xffffffffu, rowsum, 1);
  rowsum += __shfl_xor_sync(0xffffffffu, rowsum, 2);
  if (row < ni) {
#pragma unroll
    for (int c = 0; c < KD / 4; ++c) {
      const int n = sub + 4 * c;
      if (n < K) {
        const float f = exp2f(a.P[qrow * K + n] - R[n]);
        a.dq32[qrow * K + n] = pb.scale * (f * dqa[c] + dqe[c]);
      }
    }
    if (own_rows && sub == 0) a.dgs_row[qrow] = (float)rowsum;
  }
}

template <typename T, int KD, int VD>
__global__ void __launch_bounds__(kThreads) bwd_dq_simt_kernel(AttnProblem pb, BwdArgs a) {
  extern __shared__ float sm[];
  const int n_items = pb.max_blocks64 * pb.HQ;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    int seq, blk, h;
    if (!simt_item(pb, item, true, seq, blk, h)) continue;  // uniform in the CTA
    __syncthreads();
    bwd_dq_simt_block<T, KD, VD>(pb, a, sm, seq, blk, h);
  }
}

// ---------------------------------------------------------------------------
// backward, key side: dk^(h), dv^(h) per query head, column part of the
// scalar-gate gradient

template <typename T, int KD, int VD>
__device__ __forceinline__ void bwd_dkdv_simt_block(const AttnProblem& pb, const BwdArgs& a,
                                                    float* sm, int seq, int blk, int h) {
  float* kt = sm;                      // [BN][KD+1]
  float* vs = kt + BN * (KD + 1);      // [BN][VD+1]
  float* qt = vs + BN * (VD + 1);      // [BM][KD+1]
  float* dOs = qt + BM * (KD + 1);     // [BM][VD+1]
  float* Ps = dOs + BM * (VD + 1);     // [BN][BM+1]
  float* dSs = Ps + BN * (BM + 1);     // [BN][BM+1]
  float* R = dSs + BN * (BM + 1);      // [KD]
  float* gsq = R + KD;                 // [BM]
  float* gsk = gsq + BM;               // [BN]
  float* lse2 = gsk + BN;              // [BM]
  float* Dv = lse2 + BM;               // [BM]

  const int kh = h / (pb.HQ / pb.H);
  const long s0 = pb.seqs.start(seq);
  const int L = pb.seqs.len(seq);
  const int j0 = blk * BN;
  const int nj = min(BN, L - j0);
  const int K = pb.K, V = pb.V, HQ = pb.HQ;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  const T* dO = static_cast<const T*>(a.dO);

  // the anchor at the block's last key row: every later query lies past it
  for (int n = threadIdx.x; n < KD; n += kThreads)
    R[n] = n < K ? a.P[((s0 + j0 + nj - 1) * HQ + h) * (long)K + n] : 0.f;
  __syncthreads();
  const bool wide =
      load_rows_anchored<T, KD>(kt, k, a.P, R, s0 + j0, nj, BN, pb.H, kh, HQ, h, K, -1);
  load_rows_plain<T, VD, 1>(vs, v, s0 + j0, nj, BN, pb.H, kh, V);
  for (int r = threadIdx.x; r < BN; r += kThreads)
    gsk[r] = (a.GS && r < nj) ? a.GS[(s0 + j0 + r) * HQ + h] : 0.f;
  const bool exact = __syncthreads_or(wide) != 0;

  const int jr = threadIdx.x / 4, sub = threadIdx.x % 4;
  const long krow = (s0 + j0 + min(jr, nj - 1)) * HQ + h;
  const T* kraw = k + ((s0 + j0 + min(jr, nj - 1)) * pb.H + kh) * (long)K;
  float dka[KD / 4], dva[VD / 4], dke[KD / 4];
#pragma unroll
  for (int c = 0; c < KD / 4; ++c) dka[c] = dke[c] = 0.f;
#pragma unroll
  for (int c = 0; c < VD / 4; ++c) dva[c] = 0.f;
  double colsum = 0.0;  // fp64, as the row sums

  const int ilast = pb.window > 0 ? min(L - 1, j0 + nj - 1 + pb.window - 1) : L - 1;
  const float sl2 = pb.scale * kLog2e;
  for (int ib = j0 / BM; ib <= ilast / BM; ++ib) {
    const int i0 = ib * BM;
    const int ni = min(BM, L - i0);
    const bool pairwise = exact && i0 == j0;
    __syncthreads();
    load_rows_anchored<T, KD>(qt, q, a.P, R, s0 + i0, ni, BM, HQ, h, HQ, h, K,
                              pairwise ? 0 : 1);
    load_rows_plain<T, VD, 1>(dOs, dO, s0 + i0, ni, BM, HQ, h, V);
    for (int r = threadIdx.x; r < BM; r += kThreads) {
      const bool in = r < ni;
      gsq[r] = (a.GS && in) ? a.GS[(s0 + i0 + r) * HQ + h] : 0.f;
      lse2[r] = in ? a.lse[(s0 + i0 + r) * HQ + h] * kLog2e : 0.f;
      Dv[r] = in ? a.D[(s0 + i0 + r) * HQ + h] : 0.f;
    }
    __syncthreads();
    float sc[BM / 4], dp[BM / 4];
#pragma unroll
    for (int ii = 0; ii < BM / 4; ++ii) sc[ii] = dp[ii] = 0.f;
    if (!pairwise) {
      for (int n = 0; n < KD; ++n) {
        const float kv_ = kt[jr * (KD + 1) + n];
#pragma unroll
        for (int ii = 0; ii < BM / 4; ++ii) sc[ii] += kv_ * qt[(sub + 4 * ii) * (KD + 1) + n];
      }
    } else {
#pragma unroll 1
      for (int ii = 0; ii < BM / 4; ++ii) {
        const int il = min(sub + 4 * ii, ni - 1);
        sc[ii] = exact_dot(qt + il * (KD + 1), kraw,
                           a.P + ((s0 + i0 + il) * HQ + h) * (long)K, a.P + krow * K, K);
      }
    }
    for (int c = 0; c < VD; ++c) {
      const float vv = vs[jr * (VD + 1) + c];
#pragma unroll
      for (int ii = 0; ii < BM / 4; ++ii) dp[ii] += vv * dOs[(sub + 4 * ii) * (VD + 1) + c];
    }
    const int j = j0 + jr;
#pragma unroll
    for (int ii = 0; ii < BM / 4; ++ii) {
      const int il = sub + 4 * ii;
      const bool vis = jr < nj && il < ni && visible(i0 + il, j, pb.window);
      float p = 0.f, ds = 0.f;
      if (vis) {
        const float s2 = sc[ii] * sl2 + (gsq[il] - gsk[jr]) * kLog2e;
        p = exp2f(s2 - lse2[il]);
        ds = p * (dp[ii] - Dv[il]);
      }
      colsum += ds;
      Ps[jr * (BM + 1) + il] = p;
      dSs[jr * (BM + 1) + il] = ds;
    }
    __syncwarp();
    if (!pairwise) {
      for (int i = 0; i < BM; ++i) {
        const float p = Ps[jr * (BM + 1) + i];
        const float ds = dSs[jr * (BM + 1) + i];
#pragma unroll
        for (int c = 0; c < VD / 4; ++c) dva[c] += p * dOs[i * (VD + 1) + sub + 4 * c];
#pragma unroll
        for (int c = 0; c < KD / 4; ++c) dka[c] += ds * qt[i * (KD + 1) + sub + 4 * c];
      }
    } else {
      // dk_jn += dS_ij q_in 2^(P_in - P_jn), pair by pair
      for (int i = 0; i < ni; ++i) {
        const float p = Ps[jr * (BM + 1) + i];
        const float ds = dSs[jr * (BM + 1) + i];
#pragma unroll
        for (int c = 0; c < VD / 4; ++c) dva[c] += p * dOs[i * (VD + 1) + sub + 4 * c];
        if (ds == 0.f) continue;
        const float* pi = a.P + ((s0 + i0 + i) * HQ + h) * (long)K;
#pragma unroll
        for (int c = 0; c < KD / 4; ++c) {
          const int n = sub + 4 * c;
          if (n < K) dke[c] += ds * qt[i * (KD + 1) + n] * exp2f(pi[n] - a.P[krow * K + n]);
        }
      }
    }
  }
  colsum += __shfl_xor_sync(0xffffffffu, colsum, 1);
  colsum += __shfl_xor_sync(0xffffffffu, colsum, 2);
  if (jr < nj) {
#pragma unroll
    for (int c = 0; c < KD / 4; ++c) {
      const int n = sub + 4 * c;
      if (n < K) {
        const float f = exp2f(R[n] - a.P[krow * K + n]);
        a.dkh32[krow * K + n] = pb.scale * (f * dka[c] + dke[c]);
      }
    }
#pragma unroll
    for (int c = 0; c < VD / 4; ++c) {
      const int cc = sub + 4 * c;
      if (cc < V) a.dvh32[krow * V + cc] = dva[c];
    }
    // the logit carries -GS_j for key j
    if (sub == 0) a.dgs_col[krow] = (float)-colsum;
  }
}

template <typename T, int KD, int VD>
__global__ void __launch_bounds__(kThreads) bwd_dkdv_simt_kernel(AttnProblem pb, BwdArgs a) {
  extern __shared__ float sm[];
  const int n_items = pb.max_blocks64 * pb.HQ;
  // the first key blocks of a causal problem see the most query tiles
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    int seq, blk, h;
    if (!simt_item(pb, item, false, seq, blk, h)) continue;  // uniform in the CTA
    __syncthreads();
    bwd_dkdv_simt_block<T, KD, VD>(pb, a, sm, seq, blk, h);
  }
}

// The masked units' whole backward in one launch: the key-side items (dk^(h),
// dv^(h), column sums) and the query-side items (dq), which read nothing the
// other writes.
template <typename T, int KD, int VD>
__global__ void __launch_bounds__(kThreads) bwd_units_simt_kernel(AttnProblem pb, BwdArgs a) {
  extern __shared__ float sm[];
  if (no_flagged_units(pb)) return;
  const int n1 = pb.max_blocks64 * pb.HQ;
  for (int item = blockIdx.x; item < 2 * n1; item += gridDim.x) {
    int seq, blk, h;
    const bool key_side = item < n1;
    if (!simt_item(pb, key_side ? item : item - n1, !key_side, seq, blk, h)) continue;
    __syncthreads();
    if (key_side)
      bwd_dkdv_simt_block<T, KD, VD>(pb, a, sm, seq, blk, h);
    else
      bwd_dq_simt_block<T, KD, VD>(pb, a, sm, seq, blk, h);
  }
}

// ---------------------------------------------------------------------------
// group reduction and gate-gradient summand:
//   dk[t,kh] = sum_{h in group} dk^(h)[t],  dv likewise,  dq = dq32,
//   dL[t,h] = q (.) dq32 - k[t,h/G] (.) dk^(h)   (written over dq32),
//   dGS = row part + column part (written over dgs_row)

template <typename T>
__global__ void bwd_reduce_kernel(AttnProblem pb, BwdArgs a, T* dq, T* dk, T* dv) {
  const int K = pb.K, V = pb.V, HQ = pb.HQ, H = pb.H, G = HQ / H;
  const long nq = pb.rows * HQ * (long)K;
  const long nk = pb.rows * H * (long)K;
  const long nv = pb.rows * H * (long)V;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const long stride = (long)gridDim.x * blockDim.x;
  const long tid0 = (long)blockIdx.x * blockDim.x + threadIdx.x;
  for (long e = tid0; e < nk; e += stride) {
    const long t = e / ((long)H * K);
    const int kh = (int)((e / K) % H);
    const int n = (int)(e % K);
    float s = 0.f;
    for (int g = 0; g < G; ++g) s += a.dkh32[(t * HQ + kh * G + g) * K + n];
    dk[e] = from_f32<T>(s);
  }
  for (long e = tid0; e < nv; e += stride) {
    const long t = e / ((long)H * V);
    const int kh = (int)((e / V) % H);
    const int c = (int)(e % V);
    float s = 0.f;
    for (int g = 0; g < G; ++g) s += a.dvh32[(t * HQ + kh * G + g) * V + c];
    dv[e] = from_f32<T>(s);
  }
  for (long e = tid0; e < nq; e += stride) {
    const long t = e / ((long)HQ * K);
    const int h = (int)((e / K) % HQ);
    const int n = (int)(e % K);
    const float dqv = a.dq32[e];
    dq[e] = from_f32<T>(dqv);
    const float kv = to_f32(k[(t * H + h / G) * K + n]);
    a.dq32[e] = to_f32(q[e]) * dqv - kv * a.dkh32[e];
  }
  if (a.GS) {
    const long ng = pb.rows * HQ;
    for (long e = tid0; e < ng; e += stride) a.dgs_row[e] += a.dgs_col[e];
  }
}

// A persistent grid: every SM holds as many CTAs as its shared memory allows
// (cached per device and kernel), never more CTAs than work items.
template <typename F>
int persistent_grid(F kernel, size_t smem, int n_items, int (&bps)[kMaxDevices]) {
  const int dev = current_device();
  if (dev < 0) return -1;
  if (bps[dev] == 0) {
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, kThreads, smem) != cudaSuccess)
      return -1;
    bps[dev] = b < 1 ? 1 : b;
  }
  const long g = 148L * bps[dev];
  return (int)(n_items < g ? n_items : g);
}

template <typename T, int KD, int VD>
int launch_fwd(const AttnProblem& pb, const FwdArgs& a, cudaStream_t stream) {
  const size_t smem = sizeof(float) * (size_t)(BM * (KD + 1) + BN * (KD + 1) + BN * VD +
                                               BM * (BN + 1) + KD + BM + BN);
  static bool attr[kMaxDevices] = {};
  static int bps[kMaxDevices] = {};
  if (!set_max_smem_once(fwd_simt_kernel<T, KD, VD>, (int)smem, attr)) return WALL_ERR_CUDA;
  const int grid = persistent_grid(fwd_simt_kernel<T, KD, VD>, smem, pb.max_blocks64 * pb.HQ, bps);
  if (grid < 0) return WALL_ERR_CUDA;
  fwd_simt_kernel<T, KD, VD><<<grid, kThreads, smem, stream>>>(pb, a);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

template <typename T, int KD, int VD>
int launch_bwd_dq(const AttnProblem& pb, const BwdArgs& a, cudaStream_t stream) {
  const size_t smem = sizeof(float) * (size_t)(2 * BM * (KD + 1) + BN * (VD + 1) +
                                               BM * (VD + 1) + BM * (BN + 1) + KD + 4 * BM);
  static bool attr[kMaxDevices] = {};
  static int bps[kMaxDevices] = {};
  if (!set_max_smem_once(bwd_dq_simt_kernel<T, KD, VD>, (int)smem, attr)) return WALL_ERR_CUDA;
  const int grid =
      persistent_grid(bwd_dq_simt_kernel<T, KD, VD>, smem, pb.max_blocks64 * pb.HQ, bps);
  if (grid < 0) return WALL_ERR_CUDA;
  bwd_dq_simt_kernel<T, KD, VD><<<grid, kThreads, smem, stream>>>(pb, a);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

template <typename T, int KD, int VD>
int launch_bwd_dkdv(const AttnProblem& pb, const BwdArgs& a, cudaStream_t stream) {
  const size_t smem = sizeof(float) * (size_t)(BN * (KD + 1) + BN * (VD + 1) + BM * (KD + 1) +
                                               BM * (VD + 1) + 2 * BN * (BM + 1) + KD + 4 * BM);
  static bool attr[kMaxDevices] = {};
  static int bps[kMaxDevices] = {};
  if (!set_max_smem_once(bwd_dkdv_simt_kernel<T, KD, VD>, (int)smem, attr)) return WALL_ERR_CUDA;
  const int grid =
      persistent_grid(bwd_dkdv_simt_kernel<T, KD, VD>, smem, pb.max_blocks64 * pb.HQ, bps);
  if (grid < 0) return WALL_ERR_CUDA;
  bwd_dkdv_simt_kernel<T, KD, VD><<<grid, kThreads, smem, stream>>>(pb, a);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

template <typename T, int KD, int VD>
int launch_bwd_units(const AttnProblem& pb, const BwdArgs& a, cudaStream_t stream) {
  const size_t smem_dq = sizeof(float) * (size_t)(2 * BM * (KD + 1) + BN * (VD + 1) +
                                                  BM * (VD + 1) + BM * (BN + 1) + KD + 4 * BM);
  const size_t smem_dk = sizeof(float) * (size_t)(BN * (KD + 1) + BN * (VD + 1) +
                                                  BM * (KD + 1) + BM * (VD + 1) +
                                                  2 * BN * (BM + 1) + KD + 4 * BM);
  const size_t smem = smem_dq > smem_dk ? smem_dq : smem_dk;
  static bool attr[kMaxDevices] = {};
  static int bps[kMaxDevices] = {};
  if (!set_max_smem_once(bwd_units_simt_kernel<T, KD, VD>, (int)smem, attr)) return WALL_ERR_CUDA;
  const int grid =
      persistent_grid(bwd_units_simt_kernel<T, KD, VD>, smem, 2 * pb.max_blocks64 * pb.HQ, bps);
  if (grid < 0) return WALL_ERR_CUDA;
  bwd_units_simt_kernel<T, KD, VD><<<grid, kThreads, smem, stream>>>(pb, a);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

// the kernel template for the problem's head sizes (64 or 128 columns)
#define WALL_SIMT_DISPATCH(LAUNCH, T, pb, ...)                            \
  ((pb).K <= 64 ? ((pb).V <= 64 ? LAUNCH<T, 64, 64>(pb, __VA_ARGS__)     \
                                : LAUNCH<T, 64, 128>(pb, __VA_ARGS__))   \
                : ((pb).V <= 64 ? LAUNCH<T, 128, 64>(pb, __VA_ARGS__)    \
                                : LAUNCH<T, 128, 128>(pb, __VA_ARGS__)))

int fwd_any(const AttnProblem& pb, const FwdArgs& a, cudaStream_t s) {
  return pb.dtype == WALL_BF16 ? WALL_SIMT_DISPATCH(launch_fwd, __nv_bfloat16, pb, a, s)
                               : WALL_SIMT_DISPATCH(launch_fwd, float, pb, a, s);
}
int bwd_dq_any(const AttnProblem& pb, const BwdArgs& a, cudaStream_t s) {
  return pb.dtype == WALL_BF16 ? WALL_SIMT_DISPATCH(launch_bwd_dq, __nv_bfloat16, pb, a, s)
                               : WALL_SIMT_DISPATCH(launch_bwd_dq, float, pb, a, s);
}
int bwd_dkdv_any(const AttnProblem& pb, const BwdArgs& a, cudaStream_t s) {
  return pb.dtype == WALL_BF16 ? WALL_SIMT_DISPATCH(launch_bwd_dkdv, __nv_bfloat16, pb, a, s)
                               : WALL_SIMT_DISPATCH(launch_bwd_dkdv, float, pb, a, s);
}
int bwd_units_any(const AttnProblem& pb, const BwdArgs& a, cudaStream_t s) {
  return pb.dtype == WALL_BF16 ? WALL_SIMT_DISPATCH(launch_bwd_units, __nv_bfloat16, pb, a, s)
                               : WALL_SIMT_DISPATCH(launch_bwd_units, float, pb, a, s);
}
#undef WALL_SIMT_DISPATCH

}  // namespace

int attn_fwd_simt(const AttnProblem& pb, const FwdArgs& a, cudaStream_t stream) {
  if (pb.max_blocks64 == 0) return WALL_OK;
  return fwd_any(pb, a, stream);
}

int attn_bwd_simt(const AttnProblem& pb, const BwdArgs& a, cudaStream_t stream) {
  if (pb.max_blocks64 == 0) return WALL_OK;
  // dkdv and dsink read the D the dq kernel writes; dsink's partials go
  // through dkh32 before the dkdv kernel writes it
  int rc = bwd_dq_any(pb, a, stream);
  if (!rc && a.sink && a.dsink) rc = sink_grad(a.D, a.lse, a.sink, pb.rows, pb.HQ, a.dkh32,
                                               a.dsink, stream);
  return rc ? rc : bwd_dkdv_any(pb, a, stream);
}

int attn_fwd_simt_units(const AttnProblem& pb, const FwdArgs& a, const int* units,
                        cudaStream_t stream) {
  if (pb.max_blocks64 == 0) return WALL_OK;
  AttnProblem p = pb;
  p.units = units;
  return fwd_any(p, a, stream);
}

int attn_bwd_simt_units(const AttnProblem& pb, const BwdArgs& a, const int* units,
                        cudaStream_t stream) {
  if (pb.max_blocks64 == 0) return WALL_OK;
  AttnProblem p = pb;
  p.units = units;
  return bwd_units_any(p, a, stream);
}

int attn_bwd_reduce(const AttnProblem& pb, const BwdArgs& a, void* dq, void* dk, void* dv,
                    cudaStream_t stream) {
  if (pb.rows == 0) return WALL_OK;
  const int threads = 256;
  const int blocks = 148 * 8;
  if (pb.dtype == WALL_BF16)
    bwd_reduce_kernel<__nv_bfloat16><<<blocks, threads, 0, stream>>>(
        pb, a, static_cast<__nv_bfloat16*>(dq), static_cast<__nv_bfloat16*>(dk),
        static_cast<__nv_bfloat16*>(dv));
  else
    bwd_reduce_kernel<float><<<blocks, threads, 0, stream>>>(
        pb, a, static_cast<float*>(dq), static_cast<float*>(dk), static_cast<float*>(dv));
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

}  // namespace wall
