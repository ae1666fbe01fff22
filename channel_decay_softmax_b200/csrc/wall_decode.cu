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
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

template <typename T>
__global__ void cache_kernel(const T* __restrict__ k, const float* __restrict__ P, int B, int Tn,
                             int H, int HQ, int K, int C, int t0, T* __restrict__ kt,
                             float* __restrict__ rc, int Tcap) {
  const int G = HQ / H;
  const int NC = (Tcap + C - 1) / C;
  const int kgroups = K / 8;
  const long total = (long)B * Tn * HQ * kgroups;
  for (long e = (long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long)gridDim.x * blockDim.x) {
    const int kg = (int)(e % kgroups);
    const int h = (int)((e / kgroups) % HQ);
    const long tt = (e / ((long)kgroups * HQ)) % Tn;
    const long b = e / ((long)kgroups * HQ * Tn);
    const long t = t0 + tt;
    const long c = t / C;
    const long cstart = c * C;
    const int n0 = kg * 8;
    float pv[8], Rv[8], kv[8], out[8];
    load8(P + ((b * Tn + tt) * HQ + h) * K + n0, pv);
    if (cstart < t0)
      load8(rc + ((b * NC + c) * HQ + h) * K + n0, Rv);
    else
      load8(P + ((b * Tn + (cstart - t0)) * HQ + h) * K + n0, Rv);
    load8(k + ((b * Tn + tt) * H + h / G) * K + n0, kv);
#pragma unroll
    for (int i = 0; i < 8; ++i) out[i] = kv[i] * exp2f(Rv[i] - pv[i]);
    store8(kt + ((b * Tcap + t) * HQ + h) * K + n0, out);
    if (t == cstart) store8(rc + ((b * NC + c) * HQ + h) * K + n0, pv);
  }
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
  float* ws_o;   // [B,HQ,splits,V]
  float* ws_ml;  // [B,HQ,splits,2]
};

template <typename T, int KD, int VD>
__global__ void decode_split_kernel(DecodeArgs a) {
  __shared__ float qh[32][KD];  // per warp (query head): scaled, anchored query
  const int s = blockIdx.x, kh = blockIdx.y, b = blockIdx.z;
  const int G = a.HQ / a.H;
  const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = kh * G + w;
  const int K = a.K, V = a.V;
  const T* q = static_cast<const T*>(a.q);
  const T* v = static_cast<const T*>(a.v);
  const T* kt = static_cast<const T*>(a.kt);
  const int NC = (a.Tcap + a.C - 1) / a.C;
  const long k0 = (long)s * a.keys_per_split;
  const long k1 = min((long)a.T_kv, k0 + a.keys_per_split);
  constexpr int VPL = VD / 32;  // value channels per lane
  float m = -INFINITY, l = 0.f;
  float acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
  const float sl2 = a.scale * kLog2e;
  const long qoff = ((long)b * a.HQ + h) * K;
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
  const long part = ((long)b * a.HQ + h) * a.splits + s;
  if (lane * VPL < V) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) a.ws_o[part * V + lane * VPL + i] = acc[i];
  }
  if (lane == 0) {
    a.ws_ml[part * 2] = m;
    a.ws_ml[part * 2 + 1] = l;
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
  dim3 grid(a.splits, a.H, a.B);
  decode_split_kernel<T, KD, VD><<<grid, 32 * G, 0, stream>>>(a);
  if (cudaGetLastError() != cudaSuccess) return WALL_ERR_CUDA;
  decode_merge_kernel<T><<<dim3(a.HQ, a.B), 128, 0, stream>>>(a, o, lse);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

template <typename T>
int decode_dispatch(const DecodeArgs& a, void* o, float* lse, cudaStream_t s) {
  T* out = static_cast<T*>(o);
  const bool k64 = a.K <= 64, v64 = a.V <= 64;
  if (k64 && v64) return launch_decode<T, 64, 64>(a, out, lse, s);
  if (k64) return launch_decode<T, 64, 128>(a, out, lse, s);
  if (v64) return launch_decode<T, 128, 64>(a, out, lse, s);
  return launch_decode<T, 128, 128>(a, out, lse, s);
}

}  // namespace

int build_kv_cache(const void* k, const float* P, int dtype, int B, int Tn, int H, int HQ, int K,
                   int C, int t0, void* k_tilde, float* r_cache, int Tcap, cudaStream_t stream) {
  const long total = (long)B * Tn * HQ * (K / 8);
  if (total == 0) return WALL_OK;
  const int threads = 256;
  const long want = (total + threads - 1) / threads;
  const int blocks = (int)(want < 148L * 64 ? want : 148L * 64);
  if (dtype == WALL_BF16)
    cache_kernel<__nv_bfloat16><<<blocks, threads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), P, B, Tn, H, HQ, K, C, t0,
        static_cast<__nv_bfloat16*>(k_tilde), r_cache, Tcap);
  else
    cache_kernel<float><<<blocks, threads, 0, stream>>>(static_cast<const float*>(k), P, B, Tn,
                                                        H, HQ, K, C, t0,
                                                        static_cast<float*>(k_tilde), r_cache,
                                                        Tcap);
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

int attn_decode(const void* q, const void* v, const float* p_curr, const void* k_tilde,
                const float* r_cache, const float* sink, float scale, int C, int dtype, int B,
                int T_kv, int Tcap, int H, int HQ, int K, int V, void* o, float* lse, float* ws,
                int splits, cudaStream_t stream) {
  if (B == 0) return WALL_OK;
  DecodeArgs a;
  a.q = q; a.v = v; a.kt = k_tilde; a.pc = p_curr; a.rc = r_cache; a.sink = sink;
  a.scale = scale; a.C = C; a.B = B; a.T_kv = T_kv; a.Tcap = Tcap; a.H = H; a.HQ = HQ;
  a.K = K; a.V = V; a.splits = splits;
  const long chunks = (T_kv + (long)C - 1) / C;
  const long chunks_per_split = (chunks + splits - 1) / splits;
  a.keys_per_split = (int)(chunks_per_split * C);
  a.ws_o = ws;
  a.ws_ml = ws + (long)B * HQ * splits * V;
  return dtype == WALL_BF16 ? decode_dispatch<__nv_bfloat16>(a, o, lse, stream)
                            : decode_dispatch<float>(a, o, lse, stream);
}

}  // namespace wall
