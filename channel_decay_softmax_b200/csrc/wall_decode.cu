// wall_decode.cu -- pre-rescaled decode cache and the single-step decode.
//
// README "Decode": build_wall_kv_cache folds the decay into the keys,
// k_tilde[j] = k[j] * exp2(R_c - P[j]) with a per-chunk anchor R_c, so the
// decode kernel never re-accumulates the prefix; the blog (fast training,
// decode) adds that the inner loop carries no gate arithmetic.  Here the
// gate enters once per chunk through the query: for keys of chunk c,
//   s_j = scale * sum_n q_n exp2(p_curr_n - R_c,n) k_tilde_j,n,
// which equals scale * sum_n q_n k_j,n exp2(p_curr_n - P_j,n).
//
// Decode is HBM-bound (k_tilde is per query head).  Split-KV: a CTA owns one
// (batch row, kv head, key range); its G warps are the G query heads of that
// kv head, so each cached value row is fetched from HBM once per group.  Each
// lane scores one key per 32-key step with 16-byte loads, keeps an online
// softmax in the log2 domain, and accumulates o with warp shuffles of p.
// Splits are merged by their (max, sum) pairs in a second small kernel.
#include <cuda.h>

#include <type_traits>

#include "sm100_ptx.cuh"
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

using namespace sm100;
using T_bf16 = __nv_bfloat16;

// k_tilde = k * 2^(R_c - P) and r_cache = P at chunk starts (README
// "Decode").  A chunk whose gate sums past 2^kAnchorRange from its first row
// leaves k_tilde outside the range the decode reads it in: that records
// WALL_ERR_RANGE in `status` (the layout has no other place for the row).
template <typename T>
__global__ void __launch_bounds__(256)
    cache_kernel(const T* __restrict__ k, const float* __restrict__ P, int B, int Tn, int H,
                 int HQ, int K, int C, int t0, T* __restrict__ kt, float* __restrict__ rc,
                 int Tcap, int* status) {
  // a CTA takes whole rows (b, t): the row's split into (head, 8 channels)
  // groups needs only 32-bit arithmetic, and every group of the row shares
  // the chunk start's anchors (L1 hits after the first)
  const int G = HQ / H;
  const int NC = (Tcap + C - 1) / C;
  const int kgroups = K / 8;
  const int per_row = HQ * kgroups;
  const long rows = (long)B * Tn;
  bool wide = false;
  for (long row = blockIdx.x; row < rows; row += gridDim.x) {
    const long b = row / Tn;
    const long tt = row - b * Tn;
    const long t = t0 + tt;
    const long c = t / C;
    const long cstart = c * C;
    const float* prow = P + row * HQ * K;
    const float* rrow = cstart < t0 ? rc + (b * NC + c) * HQ * K
                                    : P + (b * Tn + (cstart - t0)) * HQ * K;
    const T* krow = k + row * H * K;
    T* ktrow = kt + (b * Tcap + t) * HQ * K;
    float* rcrow = t == cstart ? rc + (b * NC + c) * HQ * K : nullptr;
    for (int i = threadIdx.x; i < per_row; i += blockDim.x) {
      const int h = i / kgroups;
      const int n0 = (i - h * kgroups) * 8;
      const int off = h * K + n0;
      float pv[8], Rv[8], kv[8], out[8];
      load8(prow + off, pv);
      load8(rrow + off, Rv);
      load8(krow + (h / G) * K + n0, kv);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        out[e] = kv[e] * exp2f(Rv[e] - pv[e]);
        wide |= fabsf(Rv[e] - pv[e]) > kAnchorRange;
      }
      store8(ktrow + off, out);
      if (rcrow) store8(rcrow + off, pv);
    }
  }
  if (wide) record_status(status, WALL_ERR_RANGE);
}

template <typename T>
__device__ __forceinline__ void load_vec(const T* p, float* out, int n);

template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16>(const __nv_bfloat16* p, float* out,
                                                        int n) {
  // n in {2, 4}
  if (n == 4) {
    uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.x));
    float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.y));
    out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
  } else {
    unsigned u = __ldg(reinterpret_cast<const unsigned*>(p));
    float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u));
    out[0] = a.x; out[1] = a.y;
  }
}
template <>
__device__ __forceinline__ void load_vec<float>(const float* p, float* out, int n) {
  for (int i = 0; i < n; ++i) out[i] = __ldg(p + i);
}

__device__ __forceinline__ void load8_nc(const __nv_bfloat16* p, float* out) {
  uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8_nc(const float* p, float* out) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}

struct DecodeArgs {
  const void *q, *v, *kt;
  const float *pc, *rc, *sink;
  float scale;
  int C, B, T_kv, Tcap, H, HQ, K, V, splits, keys_per_split;
  float* ws_o;   // [B,Tq,HQ,splits,V]
  float* ws_ml;  // [B,Tq,HQ,splits,2]
  // query rows per batch row (1 for a decode step): q, p_curr, the partials
  // and the outputs hold B*Tq rows, row i of batch row b at cache position
  // T_kv - Tq + i, which sees the keys up to and including that position
  int Tq;
};

// The one-token streaming step (append + decode in one launch): the new
// token's inputs, the cache buffers it appends to and the per-head arrival
// counters of the split partials.  Unused (all null) for a plain decode.
struct StepArgs {
  const void *k, *v, *g;  // [B,H,K], [B,H,V], [B,HQ,K] bf16: the new token
  float* carry;           // [B,HQ,K] fp32: P at t-1 in, P at t out
  void* kt;               // [B,Tcap,HQ,K] k_tilde, row t written
  void* vc;               // [B,Tcap,H,V] value cache, row t written
  float* rc;              // [B,ceil(Tcap/C),HQ,K] anchors, chunk t/C written if t%C == 0
  unsigned* count;        // [B,HQ] split arrivals, zero between calls
  void* o;                // [B,HQ,V] bf16
  float* lse;             // [B,HQ] or nullptr
  int t;                  // position of the new token (= cached tokens before it)
};

template <typename T, int KD, int VD>
__global__ void decode_split_kernel(DecodeArgs a) {
  __shared__ float qh[32][KD];  // per warp (query head): scaled, anchored query
  const int s = blockIdx.x, kh = blockIdx.y;
  const int z = blockIdx.z;     // query row: batch row b, row z - b * Tq of its chunk
  const int b = z / a.Tq;
  const int G = a.HQ / a.H;
  const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = kh * G + w;
  const int K = a.K, V = a.V;
  const T* q = static_cast<const T*>(a.q);
  const T* v = static_cast<const T*>(a.v);
  const T* kt = static_cast<const T*>(a.kt);
  const int NC = (a.Tcap + a.C - 1) / a.C;
  const long k0 = (long)s * a.keys_per_split;
  const long k1 = min((long)a.T_kv - a.Tq + 1 + (z - (long)b * a.Tq), k0 + a.keys_per_split);
  constexpr int VPL = VD / 32;  // value channels per lane
  float m = -INFINITY, l = 0.f;
  float acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
  const float sl2 = a.scale * kLog2e;
  const long qoff = ((long)z * a.HQ + h) * K;
  for (long cs = k0; cs < k1; cs += a.C) {
    const long c = cs / a.C;
    // query scaled for this chunk: scale*log2e * q * exp2(p_curr - R_c)
    for (int n = lane; n < KD; n += 32) {
      float val = 0.f;
      if (n < K) {
        const float r = a.rc[(((long)b * NC + c) * a.HQ + h) * K + n];
        val = sl2 * to_f32(q[qoff + n]) * exp2f(a.pc[qoff + n] - r);
      }
      qh[w][n] = val;
    }
    __syncwarp();
    const long ce = min(k1, cs + a.C);
    for (long base = cs; base < ce; base += 32) {
      const long j = base + lane;
      const bool valid = j < ce;
      float sc = -INFINITY;
      if (valid) {
        const T* row = kt + (((long)b * a.Tcap + j) * a.HQ + h) * K;
        float d = 0.f;
#pragma unroll 4
        for (int n0 = 0; n0 < KD; n0 += 8) {
          if (n0 < K) {
            float x[8];
            load8_nc(row + n0, x);
#pragma unroll
            for (int i = 0; i < 8; ++i) d += qh[w][n0 + i] * x[i];
          }
        }
        sc = d;
      }
      float mt = sc;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float m_new = fmaxf(m, mt);
      const float alpha = exp2f(m - m_new);
      const float p = valid ? exp2f(sc - m_new) : 0.f;
      float ps = p;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l = l * alpha + ps;
      m = m_new;
#pragma unroll
      for (int i = 0; i < VPL; ++i) acc[i] *= alpha;
      const int nk = (int)min(32L, ce - base);
      for (int jj = 0; jj < nk; ++jj) {
        const float pj = __shfl_sync(0xffffffffu, p, jj);
        const T* vrow = v + (((long)b * a.Tcap + base + jj) * a.H + kh) * V + lane * VPL;
        if (lane * VPL < V) {
          float x[VPL];
          load_vec<T>(vrow, x, VPL);
#pragma unroll
          for (int i = 0; i < VPL; ++i) acc[i] += pj * x[i];
        }
      }
    }
    __syncwarp();
  }
  const long part = ((long)z * a.HQ + h) * a.splits + s;
  if (lane * VPL < V) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) a.ws_o[part * V + lane * VPL + i] = acc[i];
  }
  if (lane == 0) {
    a.ws_ml[part * 2] = m;
    a.ws_ml[part * 2 + 1] = l;
  }
}

// ---------------------------------------------------------------------------
// Streaming decode (bf16, K, V in {64, 128}, G <= 8, C a multiple of 32): a
// persistent grid, one CTA per SM, walks (batch row, kv head, key range)
// work items.  The last warp's lane 0 keeps a ring of TMA stages full: per
// 32-key tile the G heads' k_tilde boxes, the value box and the chunk's
// anchors, about 40 KB in flight per stage, so HBM sees long bulk reads
// instead of per-lane gathers.  Each query head has WPH warps that take
// alternate tiles with their own online-softmax state, merged at the end of
// the item through shared memory: lane = key for the scores (the 128-byte
// swizzle makes the 32 rows conflict-free, four independent accumulators),
// then lane = VD/32 value channels for P V.  Partials go to the same
// workspace as the split kernel above and are merged the same way.
constexpr int kDecTile = 32;

// The merge and append of a streaming step for one (batch row, query head),
// run by the finisher warp of the CTA whose split of that head arrived last
// (all the head's split partials are in the workspace):
//   P_t       = carry + g / ln 2 (per lane QPL channels), rounded as the scan
//   own score = scale * q . k_new: the decay factor of a key at the query's
//               own position is exp2(P_t - P_t) = 1, so no anchor enters
//   appends   = r_cache[t/C] = P_t when t starts a chunk, k_tilde row t =
//               k_new * exp2(R - P_t) rounded as the cache build rounds it
//               (and, as the cache build does, WALL_ERR_RANGE in the status
//               word when |R - P_t| exceeds kAnchorRange), value row t,
//               carry = P_t
// Every split of this head read the carry and the chunk anchors before it
// arrived, so the carry may be overwritten in place; row t and chunk t/C
// (when t starts it) are outside the keys any split reads.
template <int KD, int VD>
__device__ __forceinline__ void step_merge_append(const DecodeArgs& a, const StepArgs& st, int b,
                                                  int h, int kh, int g, int lane, float sl2,
                                                  int* status) {
  constexpr int VPL = VD / 32, QPL = KD / 32;
  const long bh = (long)b * a.HQ + h;
  if (lane == 0) st.count[bh] = 0u;  // every split of this call has arrived
  float qv[QPL], pv[QPL];
#pragma unroll
  for (int i = 0; i < QPL; ++i) {
    const long e = bh * KD + lane * QPL + i;
    qv[i] = to_f32(static_cast<const T_bf16*>(a.q)[e]);
    pv[i] = fmaf(kInvLn2, to_f32(static_cast<const T_bf16*>(st.g)[e]), st.carry[e]);
  }
  // the new token's chunk anchor, loaded early (written by an earlier call
  // unless this token starts the chunk)
  const int NC = (a.Tcap + a.C - 1) / a.C;
  const long t = st.t, c = t / a.C;
  const bool starts = t == c * a.C;
  float* rrow = st.rc + (((long)b * NC + c) * a.HQ + h) * KD + lane * QPL;
  float R[QPL];
#pragma unroll
  for (int i = 0; i < QPL; ++i) R[i] = starts ? pv[i] : rrow[i];

  const T_bf16* kn = static_cast<const T_bf16*>(st.k) + ((long)b * a.H + kh) * KD + lane * QPL;
  const T_bf16* vn = static_cast<const T_bf16*>(st.v) + ((long)b * a.H + kh) * VD + lane * VPL;
  float kx[QPL], vx[VPL];
  float d = 0.f;
#pragma unroll
  for (int i = 0; i < QPL; ++i) {
    kx[i] = to_f32(kn[i]);
    d = fmaf(qv[i], kx[i], d);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
  const float sd = d * sl2;  // log2 domain
#pragma unroll
  for (int i = 0; i < VPL; ++i) vx[i] = to_f32(vn[i]);

  // the partials: lanes stride the splits for (m, l); every lane then loads
  // its value channels of eight splits at a time, all in flight together,
  // so the merge costs a few L2 round trips whatever the split count
  const long base = bh * a.splits;
  const float2* ml = reinterpret_cast<const float2*>(a.ws_ml) + base;
  const float sk = a.sink ? a.sink[h] * kLog2e : -INFINITY;
  float m = fmaxf(sd, sk);
  for (int s = lane; s < a.splits; s += 32) m = fmaxf(m, __ldcg(ml + s).x);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  const float fd = exp2f(sd - m);
  float lp = 0.f;  // this lane's share of the splits' sums
  float acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = fd * vx[i];
  for (int s0 = 0; s0 < a.splits; s0 += 32) {
    float f = 0.f;  // weight of split s0 + lane (0 for a split without keys)
    if (s0 + lane < a.splits) {
      const float2 x = __ldcg(ml + s0 + lane);
      if (x.x != -INFINITY) {
        f = exp2f(x.x - m);
        lp = fmaf(x.y, f, lp);
      }
    }
    const int n = min(32, a.splits - s0);
    for (int j0 = 0; j0 < n; j0 += 8) {
      float x[8][VPL];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float* po = a.ws_o + (base + s0 + min(j0 + j, n - 1)) * VD + lane * VPL;
        if constexpr (VPL == 4) {
          const float4 u = __ldcg(reinterpret_cast<const float4*>(po));
          x[j][0] = u.x; x[j][1] = u.y; x[j][2] = u.z; x[j][3] = u.w;
        } else {
          const float2 u = __ldcg(reinterpret_cast<const float2*>(po));
          x[j][0] = u.x; x[j][1] = u.y;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float fj = __shfl_sync(0xffffffffu, f, (j0 + j) & 31);
        if (j0 + j < n) {
#pragma unroll
          for (int i = 0; i < VPL; ++i) acc[i] = fmaf(x[j][i], fj, acc[i]);
        }
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) lp += __shfl_xor_sync(0xffffffffu, lp, off);
  const float l = fd + (a.sink ? exp2f(sk - m) : 0.f) + lp;
  const float inv = 1.f / l;
  T_bf16* o = static_cast<T_bf16*>(st.o) + bh * VD + lane * VPL;
#pragma unroll
  for (int i = 0; i < VPL; ++i) o[i] = from_f32<T_bf16>(acc[i] * inv);
  if (lane == 0 && st.lse) st.lse[bh] = (m + log2f(l)) * kLn2;

  // append the token
  T_bf16* krow = static_cast<T_bf16*>(st.kt) + (((long)b * a.Tcap + t) * a.HQ + h) * KD + lane * QPL;
  float* crow = st.carry + bh * KD + lane * QPL;
  bool wide = false;
#pragma unroll
  for (int i = 0; i < QPL; ++i) {
    krow[i] = from_f32<T_bf16>(kx[i] * exp2f(R[i] - pv[i]));
    wide |= fabsf(R[i] - pv[i]) > kAnchorRange;
    if (starts) rrow[i] = pv[i];
    crow[i] = pv[i];
  }
  if (wide) record_status(status, WALL_ERR_RANGE);
  if (g == 0) {
    T_bf16* vrow = static_cast<T_bf16*>(st.vc) + (((long)b * a.Tcap + t) * a.H + kh) * VD + lane * VPL;
#pragma unroll
    for (int i = 0; i < VPL; ++i) vrow[i] = from_f32<T_bf16>(vx[i]);
  }
}

template <int KD, int VD, int WPH, bool kStep>
__global__ void __launch_bounds__(32 * (kStep ? 10 : 9), 1)
    decode_stream_kernel(const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, DecodeArgs a, StepArgs st,
                         int G, int n_items, int stages, int stage_bytes, int* status) {
  constexpr int VPL = VD / 32;  // value channels per lane
  constexpr int QPL = KD / 32;  // query channels per lane (for the scaled query)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  constexpr int kKBox = kDecTile * 128;             // one 64-channel box of 32 rows
  const int oV = G * (KD / 64) * kKBox;             // within a stage
  const int oR = oV + (VD / 64) * kKBox;            // anchors [G][KD] fp32
  const int nw = G * WPH;                           // consumer warps
  float* qts = reinterpret_cast<float*>(smem + stages * stage_bytes);  // [nw][KD]
  float* xch = qts + nw * KD;                       // [G][32][VPL + 2]: second warp's state
  uint64_t* bars = reinterpret_cast<uint64_t*>(xch + G * 32 * (VPL + 2));
  // a streaming step hands each head's split partial to the finisher warp
  // through a shared-memory slot [G][VD + 2] (o, m, l) behind the barriers
  float* pslot = reinterpret_cast<float*>(bars + 2 * stages + (kStep ? 4 : 2) * G);
  auto full = [&](int st) { return smem_u32(&bars[st]); };
  auto empty = [&](int st) { return smem_u32(&bars[stages + st]); };
  auto xfull = [&](int g) { return smem_u32(&bars[2 * stages + g]); };
  auto xempty = [&](int g) { return smem_u32(&bars[2 * stages + G + g]); };
  auto pfull = [&](int g) { return smem_u32(&bars[2 * stages + 2 * G + g]); };
  auto pempty = [&](int g) { return smem_u32(&bars[2 * stages + 3 * G + g]); };
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int NC = (a.Tcap + a.C - 1) / a.C;
  const int kps = a.keys_per_split;
  if (threadIdx.x == 0) {
    for (int st = 0; st < stages; ++st) {
      mbar_init(full(st), 1);
      mbar_init(empty(st), G);  // the G warps (one per head) that take the tile
    }
    for (int g = 0; g < G; ++g) {
      mbar_init(xfull(g), 1);
      mbar_init(xempty(g), 1);
      if (kStep) {
        mbar_init(pfull(g), 1);
        mbar_init(pempty(g), 1);
      }
    }
    fence_barrier_init();
  }
  __syncthreads();
  auto item_of = [&](int it, int& b, int& kh, int& s) {
    s = it % a.splits;
    kh = (it / a.splits) % a.H;
    b = it / (a.splits * a.H);
  };
  if (warp == nw) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const uint32_t bytes = (uint32_t)(oR + G * KD * 4);
      int seq = 0;  // tiles of this CTA so far (32-bit: the ring's stage and phase)
      bool ok = true;
      for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
        int b, kh, s;
        item_of(it, b, kh, s);
        const long k0 = (long)s * kps, k1 = min((long)a.T_kv, k0 + kps);
        for (long j0 = k0; j0 < k1; j0 += kDecTile, ++seq) {
          const int st = (int)(seq % stages);
          if (seq >= stages && !mbar_wait(empty(st), (uint32_t)((seq / stages - 1) & 1), status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(full(st), bytes);
          const uint32_t sb = sbase + st * stage_bytes;
          const int row = (int)((long)b * a.Tcap + j0);
          for (int g = 0; g < G; ++g)
            for (int bx = 0; bx < KD / 64; ++bx)
              tma_load_3d(sb + (g * (KD / 64) + bx) * kKBox, &tm_k, full(st), bx * 64,
                          kh * G + g, row);
          for (int bx = 0; bx < VD / 64; ++bx)
            tma_load_3d(sb + oV + bx * kKBox, &tm_v, full(st), bx * 64, kh, row);
          const int c = (int)j0 / a.C;
          bulk_load(sb + oR, a.rc + (((long)b * NC + c) * a.HQ + (long)kh * G) * KD, G * KD * 4,
                    full(st));
        }
      }
      // no copy may still be landing when the CTA exits
      for (int q = seq > stages ? seq - stages : 0; q < seq; ++q)
        mbar_wait(full((int)(q % stages)), (uint32_t)((q / stages) & 1), status);
    }
  } else if (warp < nw) {
    // ------------------------------------------------------------ query heads
    const int g = warp % G, par = warp / G;  // head of the group; which tiles
    const T_bf16* q = static_cast<const T_bf16*>(a.q);
    const float sl2 = a.scale * kLog2e;
    float* qt = qts + warp * KD;
    float* xs = xch + (g * 32 + lane) * (VPL + 2);
    int seq = 0;  // tiles of this CTA so far
    int n_it = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++n_it) {
      int b, kh, s;
      item_of(it, b, kh, s);
      const int h = kh * G + g;
      if (!ok) {
        // an earlier wait of this warp gave up (the status word says so):
        // no more waits; the plain decode marks this item's partial empty,
        // so its merge never reads what an earlier call left in the
        // workspace
        if constexpr (!kStep) {
          if (par == 0 && lane == 0) {
            const long part = ((long)b * a.HQ + h) * a.splits + s;
            a.ws_ml[part * 2] = -INFINITY;
            a.ws_ml[part * 2 + 1] = 0.f;
          }
        }
        continue;
      }
      const long k0 = (long)s * kps, k1 = min((long)a.T_kv, k0 + kps);
      const long qoff = ((long)b * a.HQ + h) * KD;
      float qv[QPL], pv[QPL];
#pragma unroll
      for (int i = 0; i < QPL; ++i) {
        qv[i] = to_f32(q[qoff + lane * QPL + i]);
        if constexpr (kStep)  // P_t = P_{t-1} + g_t / ln 2, rounded as the prefix scan does
          pv[i] = fmaf(kInvLn2, to_f32(static_cast<const T_bf16*>(st.g)[qoff + lane * QPL + i]),
                       st.carry[qoff + lane * QPL + i]);
        else
          pv[i] = a.pc[qoff + lane * QPL + i];
      }
      float m = -INFINITY, l = 0.f, acc[VPL];
#pragma unroll
      for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
      long c_last = -1;
      for (long j0 = k0; ok && j0 < k1; j0 += kDecTile, ++seq) {
        if ((((int)(j0 - k0) / kDecTile) % WPH) != par) continue;  // the other warp's tile
        const int st = (int)(seq % stages);
        {
          const bool got = mbar_wait(full(st), (uint32_t)((seq / stages) & 1), status);
          if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        }
        const uint8_t* sb = smem + st * stage_bytes;
        const int c = (int)j0 / a.C;
        if (c != c_last) {
          // the query scaled for this chunk: scale*log2e * q * 2^(p_curr - R_c)
          const float* R = reinterpret_cast<const float*>(sb + oR) + g * KD;
          __syncwarp();
#pragma unroll
          for (int i = 0; i < QPL; ++i)
            qt[lane * QPL + i] = sl2 * qv[i] * exp2f(pv[i] - R[lane * QPL + i]);
          __syncwarp();
          c_last = c;
        }
        // scores: lane = key of the tile, four independent partial sums
        const int r = lane;
        float d4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int bx = 0; bx < KD / 64; ++bx) {
          const uint8_t* krow = sb + (g * (KD / 64) + bx) * kKBox + r * 128;
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {
            const uint4 u = *reinterpret_cast<const uint4*>(krow + ((c8 ^ (r & 7)) << 4));
            const float4 qa = *reinterpret_cast<const float4*>(qt + bx * 64 + c8 * 8);
            const float4 qb = *reinterpret_cast<const float4*>(qt + bx * 64 + c8 * 8 + 4);
            const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&u);
            const float2 f0 = __bfloat1622float2(hv[0]), f1 = __bfloat1622float2(hv[1]);
            const float2 f2 = __bfloat1622float2(hv[2]), f3 = __bfloat1622float2(hv[3]);
            d4[0] = fmaf(f0.x, qa.x, d4[0]); d4[1] = fmaf(f0.y, qa.y, d4[1]);
            d4[2] = fmaf(f1.x, qa.z, d4[2]); d4[3] = fmaf(f1.y, qa.w, d4[3]);
            d4[0] = fmaf(f2.x, qb.x, d4[0]); d4[1] = fmaf(f2.y, qb.y, d4[1]);
            d4[2] = fmaf(f3.x, qb.z, d4[2]); d4[3] = fmaf(f3.y, qb.w, d4[3]);
          }
        }
        const bool valid = j0 + r < k1;
        const float sc = valid ? (d4[0] + d4[1]) + (d4[2] + d4[3]) : -INFINITY;
        float mt = sc;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
        const float m_new = fmaxf(m, mt);
        const float alpha = exp2f(m - m_new);
        const float p = valid ? exp2f(sc - m_new) : 0.f;
        float ps = p;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        l = l * alpha + ps;
        m = m_new;
#pragma unroll
        for (int i = 0; i < VPL; ++i) acc[i] *= alpha;
        // P V: lane = VPL value channels; keys past the range are skipped (their
        // rows may hold anything)
        const int nk = (int)min((long)kDecTile, k1 - j0);
        const int vbx = (lane * VPL) / 64, vch = (lane * VPL) % 64;
        const uint8_t* vbase = sb + oV + vbx * kKBox + (vch % 8) * 2;
        if (nk == kDecTile) {
#pragma unroll
          for (int jj = 0; jj < kDecTile; ++jj) {
            const float pj = __shfl_sync(0xffffffffu, p, jj);
            const uint8_t* vp = vbase + jj * 128 + (((vch / 8) ^ (jj & 7)) << 4);
            float x[VPL];
            if constexpr (VPL == 4) {
              const uint2 u = *reinterpret_cast<const uint2*>(vp);
              const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
              const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
              x[0] = f0.x; x[1] = f0.y; x[2] = f1.x; x[3] = f1.y;
            } else {
              const uint32_t u = *reinterpret_cast<const uint32_t*>(vp);
              const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
              x[0] = f0.x; x[1] = f0.y;
            }
#pragma unroll
            for (int i = 0; i < VPL; ++i) acc[i] = fmaf(pj, x[i], acc[i]);
          }
        } else {
          for (int jj = 0; jj < nk; ++jj) {
            const float pj = __shfl_sync(0xffffffffu, p, jj);
            const uint8_t* vp = vbase + jj * 128 + (((vch / 8) ^ (jj & 7)) << 4);
            const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(vp);
#pragma unroll
            for (int i = 0; i < VPL; i += 2) {
              const float2 f = __bfloat1622float2(hv[i / 2]);
              acc[i] = fmaf(pj, f.x, acc[i]);
              acc[i + 1] = fmaf(pj, f.y, acc[i + 1]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(st));
      }
      if (!__all_sync(0xffffffffu, ok)) ok = false;
      // the head's warps meet: the second hands its state to the first
      if (WPH == 2 && par == 1) {
        const bool got = n_it == 0 || mbar_wait(xempty(g), (uint32_t)((n_it - 1) & 1), status);
#pragma unroll
        for (int i = 0; i < VPL; ++i) xs[i] = acc[i];
        xs[VPL] = ok ? m : -INFINITY;  // a partial missing tiles counts as empty
        xs[VPL + 1] = ok ? l : 0.f;
        __syncwarp();
        if (lane == 0 && got) mbar_arrive(xfull(g));
        continue;
      }
      if (WPH == 2) {
        const bool got = mbar_wait(xfull(g), (uint32_t)(n_it & 1), status);
        if (got) {
          const float m1 = xs[VPL], l1 = xs[VPL + 1];
          const float mt = fmaxf(m, m1);
          const float a0 = (m == -INFINITY) ? 0.f : exp2f(m - mt);
          const float a1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - mt);
#pragma unroll
          for (int i = 0; i < VPL; ++i) acc[i] = acc[i] * a0 + xs[i] * a1;
          l = l * a0 + l1 * a1;
          m = mt;
        }
        if (!__all_sync(0xffffffffu, got)) ok = false;  // the partial lacks the other warp's keys
        __syncwarp();
        if (lane == 0) mbar_arrive(xempty(g));
      }
      if constexpr (kStep) {
        // to the finisher through shared memory: no global ordering on this
        // warp's path.  A split that gave up never hands over, so its head
        // is left unmerged and the status word reports the timeout.
        const bool free_slot =
            n_it == 0 || mbar_wait(pempty(g), (uint32_t)((n_it - 1) & 1), status);
        if (!__all_sync(0xffffffffu, free_slot)) ok = false;
        if (!ok) continue;
        float* slot = pslot + g * (VD + 2);
#pragma unroll
        for (int i = 0; i < VPL; ++i) slot[lane * VPL + i] = acc[i];
        if (lane == 0) {
          slot[VD] = m;
          slot[VD + 1] = l;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(pfull(g));
      } else {
        // a split that gave up on a wait is written as empty (max -inf, sum
        // 0): the merge then skips it instead of mixing in missing tiles
        const long part = ((long)b * a.HQ + h) * a.splits + s;
#pragma unroll
        for (int i = 0; i < VPL; ++i) a.ws_o[part * VD + lane * VPL + i] = acc[i];
        if (lane == 0) {
          a.ws_ml[part * 2] = ok ? m : -INFINITY;
          a.ws_ml[part * 2 + 1] = ok ? l : 0.f;
        }
      }
    }
  } else if constexpr (kStep) {
    // ------------------------------------------------------------ finisher
    // Per item: the G heads' partials from the slots to the workspace, one
    // fence, one arrival per head; the CTA whose split arrives last for a
    // head merges that head and appends the token (step_merge_append).
    const float sl2 = a.scale * kLog2e;
    int n_it = 0;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++n_it) {
      int b, kh, s;
      item_of(it, b, kh, s);
      bool ok = true;
      for (int g = 0; g < G; ++g) {
        const bool got = mbar_wait(pfull(g), (uint32_t)(n_it & 1), status);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        const float* slot = pslot + g * (VD + 2);
        const long part = ((long)b * a.HQ + kh * G + g) * a.splits + s;
#pragma unroll
        for (int i = 0; i < VPL; ++i) a.ws_o[part * VD + lane * VPL + i] = slot[lane * VPL + i];
        if (lane == 0) {
          a.ws_ml[part * 2] = slot[VD];
          a.ws_ml[part * 2 + 1] = slot[VD + 1];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(pempty(g));
      }
      if (!ok) break;
      __threadfence();  // this item's partials before its arrivals
      __syncwarp();
      unsigned prev = 0;
      if (lane < G) prev = atomicAdd(st.count + (long)b * a.HQ + kh * G + lane, 1u);
      const unsigned last =
          __ballot_sync(0xffffffffu, lane < G && prev + 1 == (unsigned)a.splits);
      if (last != 0u) {
        __threadfence();  // the other splits' partials after their arrivals
        for (int g = 0; g < G; ++g)
          if ((last >> g) & 1u)
            step_merge_append<KD, VD>(a, st, b, kh * G + g, kh, g, lane, sl2, status);
      }
    }
  }
}

template <typename T>
__global__ void decode_merge_kernel(DecodeArgs a, T* __restrict__ o, float* __restrict__ lse) {
  const int h = blockIdx.x, b = blockIdx.y;
  const long base = ((long)b * a.HQ + h) * a.splits;
  float m = a.sink ? a.sink[h] * kLog2e : -INFINITY;
  for (int s = 0; s < a.splits; ++s) m = fmaxf(m, a.ws_ml[(base + s) * 2]);
  float l = a.sink ? exp2f(a.sink[h] * kLog2e - m) : 0.f;
  for (int s = 0; s < a.splits; ++s) {
    const float ms = a.ws_ml[(base + s) * 2];
    if (ms != -INFINITY) l += a.ws_ml[(base + s) * 2 + 1] * exp2f(ms - m);
  }
  const float inv = 1.f / l;
  for (int c = threadIdx.x; c < a.V; c += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < a.splits; ++s) {
      const float ms = a.ws_ml[(base + s) * 2];
      if (ms != -INFINITY) acc += a.ws_o[(base + s) * a.V + c] * exp2f(ms - m);
    }
    o[((long)b * a.HQ + h) * a.V + c] = from_f32<T>(acc * inv);
  }
  if (threadIdx.x == 0 && lse) lse[(long)b * a.HQ + h] = (m + log2f(l)) * kLn2;
}

template <typename T, int KD, int VD>
int launch_decode(const DecodeArgs& a, T* o, float* lse, cudaStream_t stream) {
  const int G = a.HQ / a.H;
  dim3 grid(a.splits, a.H, a.B * a.Tq);
  decode_split_kernel<T, KD, VD><<<grid, 32 * G, 0, stream>>>(a);
  if (cudaGetLastError() != cudaSuccess) return WALL_ERR_CUDA;
  // the merge indexes query rows as batch rows: B*Tq of them
  decode_merge_kernel<T><<<dim3(a.HQ, a.B * a.Tq), 128, 0, stream>>>(a, o, lse);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

// the streaming kernel's shared memory: stages of (G heads' key boxes, the
// value box, anchors), the scaled queries and the barriers.  A plain decode
// merges the split partials in a second kernel; a streaming step merges them
// inside the first (the last split of each head to finish) and launches once.
template <int KD, int VD, int WPH, bool kStep>
int launch_decode_stream(const DecodeArgs& a, const StepArgs& st, __nv_bfloat16* o, float* lse,
                         cudaStream_t stream) {
  const int G = a.HQ / a.H;
  CUtensorMap tk, tv;
  if (!make_tile_map(&tk, a.kt, (long)a.B * a.Tcap, a.HQ, KD, kDecTile) ||
      !make_tile_map(&tv, a.v, (long)a.B * a.Tcap, a.H, VD, kDecTile))
    return WALL_ERR_CUDA;
  const int oR = G * (KD / 64) * kDecTile * 128 + (VD / 64) * kDecTile * 128;
  const int stage_bytes = (oR + G * KD * 4 + 1023) & ~1023;
  const int tail = G * WPH * KD * 4 + G * 32 * (VD / 32 + 2) * 4 + (2 * 4 + 2 * G) * 8 +
                   (kStep ? 2 * G * 8 + G * (VD + 2) * 4 : 0);
  const int budget = 227 * 1024 - 1024 - tail;
  int stages = budget / stage_bytes;
  if (stages > 4) stages = 4;
  if (stages < 2) return WALL_ERR_UNSUPPORTED;
  const int smem = stages * stage_bytes + tail + 1024;
  static bool attr[kMaxDevices] = {};
  if (!set_max_smem_once(decode_stream_kernel<KD, VD, WPH, kStep>, 227 * 1024, attr))
    return WALL_ERR_CUDA;
  const int n_items = a.B * a.H * a.splits;
  const int grid = n_items < 148 ? n_items : 148;
  const int warps = G * WPH + 1 + (kStep ? 1 : 0);  // consumers, TMA, finisher
  decode_stream_kernel<KD, VD, WPH, kStep><<<grid, 32 * warps, smem, stream>>>(
      tk, tv, a, st, G, n_items, stages, stage_bytes, device_status());
  if (cudaGetLastError() != cudaSuccess) return WALL_ERR_CUDA;
  if (kStep) return WALL_OK;
  decode_merge_kernel<__nv_bfloat16><<<dim3(a.HQ, a.B), 128, 0, stream>>>(a, o, lse);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

template <int WPH, bool kStep>
int launch_stream_dims(const DecodeArgs& a, const StepArgs& st, __nv_bfloat16* o, float* lse,
                       cudaStream_t s) {
  if (a.K == 128 && a.V == 128) return launch_decode_stream<128, 128, WPH, kStep>(a, st, o, lse, s);
  if (a.K == 128) return launch_decode_stream<128, 64, WPH, kStep>(a, st, o, lse, s);
  if (a.V == 128) return launch_decode_stream<64, 128, WPH, kStep>(a, st, o, lse, s);
  return launch_decode_stream<64, 64, WPH, kStep>(a, st, o, lse, s);
}

// two warps per query head while they fit in the 9-warp CTA
template <bool kStep>
int launch_stream(const DecodeArgs& a, const StepArgs& st, __nv_bfloat16* o, float* lse,
                  cudaStream_t s) {
  return a.HQ / a.H <= 4 ? launch_stream_dims<2, kStep>(a, st, o, lse, s)
                         : launch_stream_dims<1, kStep>(a, st, o, lse, s);
}

// the streaming kernel's domain: bf16, K and V in {64, 128}, up to 8 query
// heads per kv head, tiles of 32 keys that never straddle a cache chunk, and
// 16-byte aligned operands for the bulk copies
bool stream_supported(const DecodeArgs& a) {
  const int G = a.H > 0 ? a.HQ / a.H : 0;
  const bool aligned = ((reinterpret_cast<uintptr_t>(a.kt) | reinterpret_cast<uintptr_t>(a.v) |
                         reinterpret_cast<uintptr_t>(a.rc)) & 15) == 0;
  return (a.K == 64 || a.K == 128) && (a.V == 64 || a.V == 128) && G >= 1 && G <= 8 &&
         a.C % kDecTile == 0 && aligned;
}

template <typename T>
int decode_dispatch(const DecodeArgs& a, void* o, float* lse, cudaStream_t s) {
  T* out = static_cast<T*>(o);
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    if (stream_supported(a)) {
      const int rc = launch_stream<false>(a, StepArgs{}, out, lse, s);
      if (rc != WALL_ERR_UNSUPPORTED) return rc;
    }
  }
  const bool k64 = a.K <= 64, v64 = a.V <= 64;
  if (k64 && v64) return launch_decode<T, 64, 64>(a, out, lse, s);
  if (k64) return launch_decode<T, 64, 128>(a, out, lse, s);
  if (v64) return launch_decode<T, 128, 64>(a, out, lse, s);
  return launch_decode<T, 128, 128>(a, out, lse, s);
}

DecodeArgs decode_args(const void* q, const void* v, const float* p_curr, const void* k_tilde,
                       const float* r_cache, const float* sink, float scale, int C, int B,
                       int T_kv, int Tcap, int H, int HQ, int K, int V, float* ws, int splits) {
  DecodeArgs a;
  a.q = q; a.v = v; a.kt = k_tilde; a.pc = p_curr; a.rc = r_cache; a.sink = sink;
  a.scale = scale; a.C = C; a.B = B; a.T_kv = T_kv; a.Tcap = Tcap; a.H = H; a.HQ = HQ;
  a.K = K; a.V = V; a.splits = splits; a.Tq = 1;
  const long chunks = (T_kv + (long)C - 1) / C;
  const long chunks_per_split = (chunks + splits - 1) / splits;
  a.keys_per_split = (int)(chunks_per_split * C);
  a.ws_o = ws;
  a.ws_ml = ws + (long)B * HQ * splits * V;
  return a;
}

}  // namespace

int build_kv_cache(const void* k, const float* P, int dtype, int B, int Tn, int H, int HQ, int K,
                   int C, int t0, void* k_tilde, float* r_cache, int Tcap, cudaStream_t stream) {
  const long rows = (long)B * Tn;
  if (rows == 0 || HQ * (K / 8) == 0) return WALL_OK;
  const int threads = 256;
  // whole rows per CTA, eight CTAs per SM, the grid striding over the rest
  const int blocks = (int)(rows < 148L * 8 * 4 ? rows : 148L * 8 * 4);
  if (dtype == WALL_BF16)
    cache_kernel<__nv_bfloat16><<<blocks, threads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), P, B, Tn, H, HQ, K, C, t0,
        static_cast<__nv_bfloat16*>(k_tilde), r_cache, Tcap, device_status());
  else
    cache_kernel<float><<<blocks, threads, 0, stream>>>(static_cast<const float*>(k), P, B, Tn,
                                                        H, HQ, K, C, t0,
                                                        static_cast<float*>(k_tilde), r_cache,
                                                        Tcap, device_status());
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

// Splits per (batch row, kv head): about four waves of CTAs over the 148
// SMs, never more splits than chunks.  Non-decreasing in T_kv, so a
// workspace sized for the largest T_kv serves every shorter one.
int decode_splits(int B, int T_kv, int H, int C) {
  const long units = (long)B * H;
  const long chunks = (T_kv + (long)C - 1) / C;
  long s = (148L * 8 * 4 + units - 1) / units;
  if (s > chunks) s = chunks;
  if (s < 1) s = 1;
  return (int)s;
}

// Splits for a chunk of Tq query rows per batch row: the same waves, with
// every query row a unit of its own.
int decode_chunk_splits(int B, int Tq, int T_kv, int H, int C) {
  return decode_splits(B * Tq, T_kv, H, C);
}

int attn_decode_chunk_split(const void* q, const void* v, const float* p, const void* k_tilde,
                            const float* r_cache, const float* sink, float scale, int C,
                            int dtype, int B, int Tq, int T_kv, int Tcap, int H, int HQ, int K,
                            int V, void* o, float* lse, float* ws, int splits,
                            cudaStream_t stream) {
  if ((long)B * Tq == 0) return WALL_OK;
  DecodeArgs a = decode_args(q, v, p, k_tilde, r_cache, sink, scale, C, B, T_kv, Tcap, H, HQ, K,
                             V, ws, splits);
  a.Tq = Tq;
  a.ws_ml = ws + (long)B * Tq * HQ * splits * V;
  if (dtype == WALL_BF16) {
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(o);
    if (K <= 64 && V <= 64) return launch_decode<__nv_bfloat16, 64, 64>(a, out, lse, stream);
    if (K <= 64) return launch_decode<__nv_bfloat16, 64, 128>(a, out, lse, stream);
    if (V <= 64) return launch_decode<__nv_bfloat16, 128, 64>(a, out, lse, stream);
    return launch_decode<__nv_bfloat16, 128, 128>(a, out, lse, stream);
  }
  float* out = static_cast<float*>(o);
  if (K <= 64 && V <= 64) return launch_decode<float, 64, 64>(a, out, lse, stream);
  if (K <= 64) return launch_decode<float, 64, 128>(a, out, lse, stream);
  if (V <= 64) return launch_decode<float, 128, 64>(a, out, lse, stream);
  return launch_decode<float, 128, 128>(a, out, lse, stream);
}

int attn_decode(const void* q, const void* v, const float* p_curr, const void* k_tilde,
                const float* r_cache, const float* sink, float scale, int C, int dtype, int B,
                int T_kv, int Tcap, int H, int HQ, int K, int V, void* o, float* lse, float* ws,
                int splits, cudaStream_t stream) {
  if (B == 0) return WALL_OK;
  const DecodeArgs a = decode_args(q, v, p_curr, k_tilde, r_cache, sink, scale, C, B, T_kv, Tcap,
                                   H, HQ, K, V, ws, splits);
  return dtype == WALL_BF16 ? decode_dispatch<__nv_bfloat16>(a, o, lse, stream)
                            : decode_dispatch<float>(a, o, lse, stream);
}

int decode_step(const void* q, const void* k, const void* v, const void* g, float* carry,
                void* k_tilde, void* v_cache, float* r_cache, const float* sink, float scale,
                int C, int t, int B, int Tcap, int H, int HQ, int K, int V, void* o, float* lse,
                float* ws, unsigned* counters, int splits, cudaStream_t stream) {
  if (B == 0) return WALL_OK;
  // the cache holds positions [0, t); the new token is merged in by the kernel
  const DecodeArgs a = decode_args(q, v_cache, nullptr, k_tilde, r_cache, sink, scale, C, B, t,
                                   Tcap, H, HQ, K, V, ws, splits);
  if (!stream_supported(a)) return WALL_ERR_UNSUPPORTED;
  StepArgs st;
  st.k = k; st.v = v; st.g = g; st.carry = carry; st.kt = k_tilde; st.vc = v_cache;
  st.rc = r_cache; st.count = counters; st.o = o; st.lse = lse; st.t = t;
  return launch_stream<true>(a, st, static_cast<__nv_bfloat16*>(o), lse, stream);
}

}  // namespace wall
