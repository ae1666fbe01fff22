// wall_attn_bwd_dq_sm100.cu -- tensor-core dq of the Wall Attention backward
// (bf16, K == V in {64, 128}), one CTA per 128-row query block, no atomics.
//
// Same anchored form as the forward (Tilde blog "Wall Attention", fast
// training section 1): for the CTA's query block I and key tile J,
// Kt_J = Kh_J (.) 2^(R_I - R_J) per channel, and
//   S  = Qh_I Kt_J^T           P_ij = 2^(S*scale*log2e + bias - lse2_i)
//   dP = dO_I V_J^T            dS_ij = P_ij (dP_ij - D_i)
//   dQa += dS Kt_J             (dS from TMEM, Kt MN-major from shared memory)
// so that dq_i = scale * 2^(P_i - R_I) (.) dQa_i; the factor is applied per row
// by the finalize kernel, which also forms the gate-gradient summand.  dq is
// written once per row: deterministic, and no fp32 atomics through L2.
//
// The block anchors are integers, so d = 2^(R_I - R_J) is an exact power of
// two and Kt_J = Kh_J (.) d is an exact packed bf16 multiply, done in place.
//
// CTA = 12 warps (3 per SM sub-partition, 168 registers each):
//   warp 0      TMA, lane 0: Qh_I, dO_I once and the key ring (Kh_J with its
//               block anchors, 4 stages); lane 1: the value ring (1 stage)
//   warp 1      TMEM owner and MMA issuer.  Per tile: dP(t+1) as soon as the
//               softmax has read dP(t), then dQa(t), then S(t+2)
//   warps 2-3   key rescale Kt_J = Kh_J (.) d in place; each thread keeps one
//               16-byte channel chunk, so its 8 factors stay in registers
//   warps 4-11  one thread per (query row, 64-key half of the tile): P, dS ->
//               bf16 pairs over the first 32 of the half's S columns; the two
//               warps of a TMEM lane quarter take the two halves; epilogue
//               dQa -> fp32 workspace
// TMEM columns: S0 [0,128), S1 [128,256), dP [256,384), dQa [384,512).
#include <cuda.h>

#include "sm100_ptx.cuh"
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kKS = 4;  // key stages: the refill (TMA + in-place scaling) spans a tile
constexpr int kVS = 1;  // value stages
constexpr int kThreads = 384;

struct DqParams {
  const float* anchors;  // [nblk, HQ, K]
  const float* lse;      // [rows, HQ]
  const float* D;        // [rows, HQ]
  const float* GS;       // [rows, HQ] or nullptr
  float* dq32;           // [rows, HQ, K]  raw dQa (without scale * 2^(P - R_I))
  Seqs seqs;
  int HQ, H;
  float scale_log2;
  int window;
  int n_blocks;
  int* status;
};

template <int KD>
struct DSmem {
  static constexpr int kT = BM * KD * 2;  // one 128-row bf16 tile
  static constexpr int oQ = 0;
  static constexpr int oO = oQ + kT;
  static constexpr int oK = oO + kT;           // kKS stages
  static constexpr int oV = oK + kKS * kT;     // kVS stages
  static constexpr int oRJ = oV + kVS * kT;     // float[kKS][KD]
  static constexpr int oBar = oRJ + kKS * KD * 4;
  static constexpr int kBars = 20;  // >= kNumBars
  static constexpr int oMisc = oBar + kBars * 8;
  static constexpr int kBytes = oMisc + 16;
  // no alignment slack: the shared window is used from its start, which the
  // kernel checks is 1 KB aligned (the 128-byte swizzle atoms need it)
  static constexpr int kAlloc = kBytes;
};

enum DBar {
  QO_FULL = 0,
  K_FULL = 1,                    // + stage (kKS)
  K_READY = K_FULL + kKS,        // + stage
  K_EMPTY = K_READY + kKS,       // + stage
  V_FULL = K_EMPTY + kKS,        // + stage (kVS)
  V_EMPTY = V_FULL + kVS,        // + stage
  SD_FULL = V_EMPTY + kVS,
  P_FULL = SD_FULL + 1,
  DQ_DONE = P_FULL + 1,
  MMA_DONE = DQ_DONE + 1,
  kNumBars = MMA_DONE + 1,
};
static_assert(kNumBars <= DSmem<128>::kBars, "barrier slots");
static_assert(DSmem<128>::kAlloc <= 227 * 1024, "shared memory");

// 2^k as bf16 bits for an integer k (the anchors are integers): exact in
// the normal range, 0 below it (a factor under 2^-126 scales a key that
// decays to nothing) and +inf above it, as the fp32 product would overflow.
__device__ __forceinline__ uint32_t pow2_bf16(float k) {
  const int e = (int)k;
  return e < -126 ? 0u : e > 127 ? 0x7F80u : uint32_t(e + 127) << 7;
}

constexpr uint32_t kColS = 0, kColDP = 256, kColDQ = 384;

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, int* status,
                                         volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > 1000000000ull) {
      record_status(status, WALL_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int KD>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  DqParams p) {
  using Lay = DSmem<KD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {  // uniform: every thread returns before any barrier
    if (threadIdx.x == 0) record_status(p.status, WALL_ERR_UNSUPPORTED);
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::oBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::oMisc + 4);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.x;
  const int HQ = p.HQ, K = KD;
  const int kh = h / (HQ / p.H);
  // longest query blocks first
  const int flat = p.n_blocks - 1 - (int)blockIdx.y;
  int seq, blk;
  if (!seq_block(p.seqs, BM, flat, seq, blk)) return;
  const int blk_off = flat - blk;
  const long s0 = p.seqs.start(seq);
  const int L = p.seqs.len(seq);
  const int i0 = blk * BM;
  const int ni = min(BM, L - i0);
  const int jb_hi = (i0 + ni - 1) / BN;
  const int jb_lo = p.window > 0 ? max(0, i0 - p.window + 1) / BN : 0;
  const int nT = jb_hi - jb_lo + 1;

  if (threadIdx.x == 0) {
    mbar_init(bar(QO_FULL), 1);
    for (int s = 0; s < kKS; ++s) {
      mbar_init(bar(K_FULL + s), 1);
      mbar_init(bar(K_READY + s), 2);
      mbar_init(bar(K_EMPTY + s), 1);
    }
    for (int s = 0; s < kVS; ++s) {
      mbar_init(bar(V_FULL + s), 1);
      mbar_init(bar(V_EMPTY + s), 1);
    }
    mbar_init(bar(SD_FULL), 1);
    mbar_init(bar(P_FULL), 8);
    mbar_init(bar(DQ_DONE), 1);
    mbar_init(bar(MMA_DONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    // lane 0: Qh, dO and the key ring; lane 1: the value ring.  The two lanes
    // wait on different barriers and progress independently.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_o);
      mbar_expect_tx(bar(QO_FULL), 2 * Lay::kT);
      for (int b = 0; b < K / 64; ++b) {
        tma_load_3d(sbase + Lay::oQ + b * (BM * 128), &tm_q, bar(QO_FULL), b * 64, h,
                    (int)(s0 + i0));
        tma_load_3d(sbase + Lay::oO + b * (BM * 128), &tm_o, bar(QO_FULL), b * 64, h,
                    (int)(s0 + i0));
      }
      int issued = 0;
      for (int t = 0; t < nT; ++t) {
        const int st = t % kKS;
        const int row = (int)(s0 + (long)(jb_lo + t) * BN);
        if (t >= kKS &&
            !wait_bar(bar(K_EMPTY + st), ((t / kKS) - 1) & 1, p.status, abort_flag))
          break;
        mbar_expect_tx(bar(K_FULL + st), Lay::kT + K * 4);
        for (int b = 0; b < K / 64; ++b)
          tma_load_3d(sbase + Lay::oK + st * Lay::kT + b * (BN * 128), &tm_k, bar(K_FULL + st),
                      b * 64, h, row);
        bulk_load(sbase + Lay::oRJ + st * K * 4,
                  p.anchors + ((long)(blk_off + jb_lo + t) * HQ + h) * K, K * 4,
                  bar(K_FULL + st));
        issued = t + 1;
      }
      for (int t = max(0, issued - kKS); t < issued; ++t)
        mbar_wait(bar(K_FULL + t % kKS), (t / kKS) & 1, p.status);
      mbar_wait(bar(QO_FULL), 0, p.status);
    } else if (lane == 1) {
      tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (int t = 0; t < nT; ++t) {
        const int st = t % kVS;
        if (t >= kVS && !wait_bar(bar(V_EMPTY + st), (t / kVS - 1) & 1, p.status, abort_flag))
          break;
        mbar_expect_tx(bar(V_FULL + st), Lay::kT);
        const int row = (int)(s0 + (long)(jb_lo + t) * BN);
        for (int b = 0; b < K / 64; ++b)
          tma_load_3d(sbase + Lay::oV + st * Lay::kT + b * (BN * 128), &tm_v, bar(V_FULL + st),
                      b * 64, kh, row);
        issued = t + 1;
      }
      for (int t = max(0, issued - kVS); t < issued; ++t)
        mbar_wait(bar(V_FULL + t % kVS), (t / kVS) & 1, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(BM, BN, false, false);   // S, dP
      const uint32_t id_dq = idesc_bf16(BM, KD, false, true);   // dQa (A from TMEM)
      bool ok = wait_bar(bar(QO_FULL), 0, p.status, abort_flag);
      auto issue_s = [&](int t) -> bool {
        const int st = t % kKS;
        if (!wait_bar(bar(K_READY + st), (t / kKS) & 1, p.status, abort_flag)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem + kColS + (t & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < KD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          umma_bf16_ss(d_tmem, sdesc_sw128(sbase + Lay::oQ + off, 16, 1024),
                       sdesc_sw128(sbase + Lay::oK + st * Lay::kT + off, 16, 1024), id_s,
                       kk > 0 ? 1u : 0u);
        }
        return true;
      };
      auto issue_dp = [&](int t) -> bool {
        const int vs = t % kVS;
        if (!wait_bar(bar(V_FULL + vs), (t / kVS) & 1, p.status, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < KD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          umma_bf16_ss(tmem + kColDP, sdesc_sw128(sbase + Lay::oO + off, 16, 1024),
                       sdesc_sw128(sbase + Lay::oV + vs * Lay::kT + off, 16, 1024), id_s,
                       kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(V_EMPTY + vs));
        umma_commit(bar(SD_FULL));  // S(t) was issued earlier: both are ready
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok) ok = issue_dp(0);
      if (ok && nT > 1) ok = issue_s(1);
      for (int t = 0; ok && t < nT; ++t) {
        const int st = t % kKS;
        if (!wait_bar(bar(P_FULL), t & 1, p.status, abort_flag)) break;
        tc_fence_after();
        // the softmax has read dP(t): dP(t+1) first, so that the softmax of
        // tile t+1 can start while the tensor core accumulates dQa(t)
        if (t + 1 < nT) ok = issue_dp(t + 1);
        // dQa += dS Kt: A = dS (bf16 pairs over the S buffer, 8 columns per 16
        // keys, the two 64-key halves 64 columns apart), B = Kt [keys x
        // channels] MN-major: 8-key groups 1 KB apart, 64-channel boxes BN*128
        // bytes apart
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_bf16_ts(tmem + kColDQ, tmem + kColS + (t & 1) * 128 + (kk >> 2) * 64 + (kk & 3) * 8,
                       sdesc_sw128(sbase + Lay::oK + st * Lay::kT + kk * 16 * 128, BN * 128,
                                   1024),
                       id_dq, (t > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(K_EMPTY + st));
        if (ok && t + 2 < nT) ok = issue_s(t + 2);  // in order after dQa(t) read dS(t)
      }
      umma_commit(bar(DQ_DONE));
      umma_commit(bar(MMA_DONE));
      mbar_wait(bar(MMA_DONE), 0, p.status);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ key rescale
    constexpr int kChunks = KD / 8;          // 16-byte chunks per row
    constexpr int kRowStep = 64 / kChunks;   // rows covered by one pass of 64 threads
    constexpr int kRows = BN / kRowStep;     // rows per thread
    const int tid = threadIdx.x - 64;
    const int ch = tid % kChunks;
    const int rs = tid / kChunks;
    // the query block's anchors: only these warps need them, so they load
    // them here rather than everyone before the setup barrier
    float ri[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) ri[e] = __ldg(p.anchors + ((long)(blk_off + blk) * HQ + h) * K + ch * 8 + e);
    for (int t = 0; t < nT; ++t) {
      const int st = t % kKS;
      {
        const bool got = wait_bar(bar(K_FULL + st), (t / kKS) & 1, p.status, abort_flag);
        if (!__all_sync(0xffffffffu, got)) break;
      }
      const float* rj = reinterpret_cast<const float*>(smem + Lay::oRJ + st * K * 4) + ch * 8;
      __nv_bfloat162 d[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t b = pow2_bf16(ri[2 * e] - rj[2 * e]) |
                           (pow2_bf16(ri[2 * e + 1] - rj[2 * e + 1]) << 16);
        d[e] = *reinterpret_cast<const __nv_bfloat162*>(&b);
      }
      uint8_t* kt = smem + Lay::oK + st * Lay::kT + (ch / 8) * (BN * 128);
      constexpr int kBatch = 8;
#pragma unroll
      for (int m0 = 0; m0 < kRows; m0 += kBatch) {
        uint4 v[kBatch];
#pragma unroll
        for (int x = 0; x < kBatch; ++x) {
          const int r = rs + (m0 + x) * kRowStep;
          v[x] = *reinterpret_cast<const uint4*>(kt + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
        }
#pragma unroll
        for (int x = 0; x < kBatch; ++x) {
          const int r = rs + (m0 + x) * kRowStep;
          __nv_bfloat162* w = reinterpret_cast<__nv_bfloat162*>(&v[x]);
#pragma unroll
          for (int e = 0; e < 4; ++e) w[e] = __hmul2(w[e], d[e]);
          *reinterpret_cast<uint4*>(kt + r * 128 + (((ch & 7) ^ (r & 7)) << 4)) = v[x];
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(K_READY + st));
    }
  } else {
    // ------------------------------------------------------------ dS per (query row, key half)
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;  // keys 64*half .. 64*half+63 of each tile
    const int r = quarter * 32 + lane;
    const int i = i0 + r;
    const bool row_ok = r < ni;
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    const bool has_gs = p.GS != nullptr;
    const int win = p.window > 0 ? p.window : 0x7fffffff;
    const long grow = (s0 + i) * HQ + h;
    const float lse2 = row_ok ? p.lse[grow] * kLog2e : 0.f;
    const float Di = row_ok ? p.D[grow] : 0.f;
    const float gs_i = (has_gs && row_ok) ? p.GS[grow] * kLog2e : 0.f;
    const float sl2 = p.scale_log2;
    const float off_i = (has_gs ? gs_i : 0.f) - lse2;
    bool ok = true;
    for (int t = 0; t < nT; ++t) {
      const int j0 = (jb_lo + t) * BN + half * 64;  // first key of this half
      {
        const bool got = wait_bar(bar(SD_FULL), t & 1, p.status, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      }
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_base + kColS + (t & 1) * 128 + half * 64;
      const uint32_t dp_addr = tmem + lane_base + kColDP + half * 64;
      const bool fast = __all_sync(0xffffffffu, row_ok && (j0 + 63 <= i) && (j0 + 64 <= L) &&
                                                    (i - j0 < win) && !has_gs);
#pragma unroll 1
      for (int c = 0; c < 64; c += 32) {
        uint32_t sv[32], dv[32];
        tmem_ld32(s_addr + c, sv);
        tmem_ld32(dp_addr + c, dv);
        tmem_wait_ld();
        uint32_t pk[16];
        if (fast) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float ds[2];
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              const float a = fmaf(__uint_as_float(sv[e + x]), sl2, off_i);
              // 3 of every 8 exponentials on the FMA pipe, the rest on MUFU
              const float pv = ((e + x) & 7) >= 5 ? exp2_fma(a) : exp2f(a);
              ds[x] = pv * (__uint_as_float(dv[e + x]) - Di);
            }
            pk[e / 2] = pack_bf16x2(ds[0], ds[1]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float ds[2];
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              const int j = j0 + c + e + x;
              const bool vis = row_ok & (j < L) & (j <= i) & (i - j < win);
              // the key prefix of the scalar gate, straight from global
              // memory (L1-resident across the warp; this path is rare)
              const float gk = (has_gs && j < L) ? p.GS[(s0 + j) * HQ + h] * kLog2e : 0.f;
              const float a = fmaf(__uint_as_float(sv[e + x]), sl2, off_i - gk);
              const float pv = vis ? exp2f(a) : 0.f;
              ds[x] = pv * (__uint_as_float(dv[e + x]) - Di);
            }
            pk[e / 2] = pack_bf16x2(ds[0], ds[1]);
          }
        }
        // keys [c, c+32) of the half -> its columns [c/2, c/2+16) (already read)
        tmem_st16(s_addr + c / 2, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(P_FULL));
    }
    // ---- epilogue: the raw dQa row, each half writes half of the channels
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(bar(DQ_DONE), 0, p.status, abort_flag));
    if (ok) {
      tc_fence_after();
      float* out = p.dq32 + grow * K;
#pragma unroll 1
      for (int c = half * (KD / 2); c < (half + 1) * (KD / 2); c += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + kColDQ + c, v);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(out + c + e) =
                make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                            __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// dq from the dS tiles the key-block kernel stored: for the CTA's query
// block I and every key tile J it sees (J <= I, within the window),
//   dQa += dS_IJ Kt_J,   Kt_J = Kh_J (.) 2^(R_I - R_J)  (exact, in place)
// one contraction per tile instead of four (S, dP and this one recomputed,
// and the exponentials); HBM carries the dS tiles, L2 keeps Kh.
//
// CTA = 8 warps (256 threads):
//   warp 0      TMA, lane 0: the dS ring (two 64-query boxes of 128 key rows
//               per tile, 4 stages, from HBM); lane 1: the key ring (Kh_J and
//               its block anchors, 3 stages, mostly from L2).  The rings have
//               barriers of their own, so the keys are scaled while the slower
//               dS tiles are still in flight.
//   warp 1      TMEM owner (128 columns) and MMA issuer: A = dS (queries x
//               keys, MN-major: queries contiguous in the stored rows),
//               B = Kt (keys x channels, MN-major)
//   warps 2-5   Kt_J = Kh_J (.) d in place, as in the kernel above (four
//               warps: with two, the in-place scaling set the tile rate)
//   warps 4-7   epilogue: dQa rows -> fp32 workspace
constexpr int kDSS = 4;  // dS stages
constexpr int kKS3 = 3;  // key stages
constexpr int kDsThreads = 256;

template <int KD>
struct QSmem {
  static constexpr int kDsT = 128 * 128 * 2;    // one stored dS tile
  static constexpr int kKT = BN * KD * 2;       // one Kh tile
  static constexpr int oDS = 0;                 // kDSS stages
  static constexpr int oK = oDS + kDSS * kDsT;  // kKS3 stages
  static constexpr int oRJ = oK + kKS3 * kKT;   // float[kKS3][KD]
  static constexpr int oBar = oRJ + kKS3 * KD * 4;
  static constexpr int kBars = 2 * kDSS + 3 * kKS3 + 2;
  static constexpr int oMisc = oBar + kBars * 8;
  static constexpr int kBytes = oMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1 KB alignment
};
static_assert(QSmem<128>::kAlloc <= 227 * 1024, "shared memory");

enum QBar {
  D_FULL = 0,                     // + dS stage
  D_EMPTY = kDSS,                 // + dS stage
  K_FULL3 = 2 * kDSS,             // + key stage
  K_READY3 = 2 * kDSS + kKS3,     // + key stage, 4 scaling warps
  K_EMPTY3 = 2 * kDSS + 2 * kKS3,  // + key stage
  QS_DONE = 2 * kDSS + 3 * kKS3,
  QS_MMA = QS_DONE + 1,
};

template <int KD>
__global__ void __launch_bounds__(kDsThreads, 1)
    bwd_dq_ds_kernel(const __grid_constant__ CUtensorMap tm_ds,
                     const __grid_constant__ CUtensorMap tm_k, DqParams p, DsLayout ds_lay) {
  using Lay = QSmem<KD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::oBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::oMisc + 4);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.x;
  const int HQ = p.HQ, K = KD;
  // longest query blocks first
  const int flat = p.n_blocks - 1 - (int)blockIdx.y;
  int seq, blk;
  if (!seq_block(p.seqs, BM, flat, seq, blk)) return;
  const int blk_off = flat - blk;
  const long s0 = p.seqs.start(seq);
  const int L = p.seqs.len(seq);
  const int i0 = blk * BM;
  const int ni = min(BM, L - i0);
  const int jlo = ds_lay.jlo(blk);  // key tiles jlo .. I
  const int nT = blk - jlo + 1;
  const long tile0 = ds_lay.pair_base(p.seqs, HQ, seq, h) + ds_lay.rowstart(blk);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDSS; ++s) {
      mbar_init(bar(D_FULL + s), 1);
      mbar_init(bar(D_EMPTY + s), 1);
    }
    for (int s = 0; s < kKS3; ++s) {
      mbar_init(bar(K_FULL3 + s), 1);
      mbar_init(bar(K_READY3 + s), 4);
      mbar_init(bar(K_EMPTY3 + s), 1);
    }
    mbar_init(bar(QS_DONE), 1);
    mbar_init(bar(QS_MMA), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      // the dS ring.  Each stored tile is read once: evict_first, so that
      // the 1 GB stream does not push out of L2 the key tiles that every
      // query block of the head reads again (those load with evict_last;
      // 0.218 against 0.237 ms at T = 8192, 1.09 GB of tiles)
      tma_prefetch_desc(&tm_ds);
      const uint64_t pol_ds = l2_evict_first();
      int issued = 0;
      for (int t = 0; t < nT; ++t) {
        const int st = t % kDSS;
        if (t >= kDSS && !wait_bar(bar(D_EMPTY + st), (t / kDSS - 1) & 1, p.status, abort_flag))
          break;
        mbar_expect_tx(bar(D_FULL + st), Lay::kDsT);
        const int drow = (int)((tile0 + t) * 128);
        for (int b = 0; b < 2; ++b)
          tma_load_2d_hint(sbase + Lay::oDS + st * Lay::kDsT + b * (128 * 128), &tm_ds,
                           bar(D_FULL + st), b * 64, drow, pol_ds);
        issued = t + 1;
      }
      // no copy may still be in flight when the CTA exits
      for (int t = max(0, issued - kDSS); t < issued; ++t)
        mbar_wait(bar(D_FULL + t % kDSS), (t / kDSS) & 1, p.status);
    } else if (lane == 1) {
      // the key ring
      tma_prefetch_desc(&tm_k);
      const uint64_t pol_k = l2_evict_last();
      int issued = 0;
      for (int t = 0; t < nT; ++t) {
        const int st = t % kKS3;
        if (t >= kKS3 && !wait_bar(bar(K_EMPTY3 + st), (t / kKS3 - 1) & 1, p.status, abort_flag))
          break;
        mbar_expect_tx(bar(K_FULL3 + st), Lay::kKT + K * 4);
        for (int b = 0; b < K / 64; ++b)
          tma_load_3d_hint(sbase + Lay::oK + st * Lay::kKT + b * (BN * 128), &tm_k,
                           bar(K_FULL3 + st), b * 64, h, (int)(s0 + (long)(jlo + t) * BN), pol_k);
        bulk_load(sbase + Lay::oRJ + st * K * 4,
                  p.anchors + ((long)(blk_off + jlo + t) * HQ + h) * K, K * 4,
                  bar(K_FULL3 + st));
        issued = t + 1;
      }
      for (int t = max(0, issued - kKS3); t < issued; ++t)
        mbar_wait(bar(K_FULL3 + t % kKS3), (t / kKS3) & 1, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t id = idesc_bf16(BM, KD, true, true);
      for (int t = 0; t < nT; ++t) {
        const int st = t % kDSS, kt = t % kKS3;
        if (!wait_bar(bar(D_FULL + st), (t / kDSS) & 1, p.status, abort_flag)) break;
        if (!wait_bar(bar(K_READY3 + kt), (t / kKS3) & 1, p.status, abort_flag)) break;
        tc_fence_after();
        // K = 16 keys per MMA: rows 16kk .. 16kk+15 of both operands; the two
        // 64-wide M (N) boxes of dS (Kt) are 128 rows x 128 B apart
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_bf16_ss(tmem,
                       sdesc_sw128(sbase + Lay::oDS + st * Lay::kDsT + kk * 16 * 128, 128 * 128,
                                   1024),
                       sdesc_sw128(sbase + Lay::oK + kt * Lay::kKT + kk * 16 * 128, BN * 128,
                                   1024),
                       id, (t > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(D_EMPTY + st));
        umma_commit(bar(K_EMPTY3 + kt));
      }
      umma_commit(bar(QS_DONE));
      umma_commit(bar(QS_MMA));
      mbar_wait(bar(QS_MMA), 0, p.status);
    }
  } else {
    if (warp < 6) {
      // ------------------------------------------------------------ key rescale
      constexpr int kChunks = KD / 8;
      constexpr int kRowStep = 128 / kChunks;
      constexpr int kRows = BN / kRowStep;
      const int tid = threadIdx.x - 64;
      const int ch = tid % kChunks;
      const int rs = tid / kChunks;
      float ri[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        ri[e] = __ldg(p.anchors + ((long)(blk_off + blk) * HQ + h) * K + ch * 8 + e);
      for (int t = 0; t < nT; ++t) {
        const int st = t % kKS3;
        {
          const bool got = wait_bar(bar(K_FULL3 + st), (t / kKS3) & 1, p.status, abort_flag);
          if (!__all_sync(0xffffffffu, got)) break;
        }
        const float* rj = reinterpret_cast<const float*>(smem + Lay::oRJ + st * K * 4) + ch * 8;
        __nv_bfloat162 d[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t b = pow2_bf16(ri[2 * e] - rj[2 * e]) |
                             (pow2_bf16(ri[2 * e + 1] - rj[2 * e + 1]) << 16);
          d[e] = *reinterpret_cast<const __nv_bfloat162*>(&b);
        }
        uint8_t* kt = smem + Lay::oK + st * Lay::kKT + (ch / 8) * (BN * 128);
        constexpr int kBatch = 8;
#pragma unroll
        for (int m0 = 0; m0 < kRows; m0 += kBatch) {
          uint4 v[kBatch];
#pragma unroll
          for (int x = 0; x < kBatch; ++x) {
            const int r = rs + (m0 + x) * kRowStep;
            v[x] = *reinterpret_cast<const uint4*>(kt + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
          }
#pragma unroll
          for (int x = 0; x < kBatch; ++x) {
            const int r = rs + (m0 + x) * kRowStep;
            __nv_bfloat162* w = reinterpret_cast<__nv_bfloat162*>(&v[x]);
#pragma unroll
            for (int e = 0; e < 4; ++e) w[e] = __hmul2(w[e], d[e]);
            *reinterpret_cast<uint4*>(kt + r * 128 + (((ch & 7) ^ (r & 7)) << 4)) = v[x];
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(K_READY3 + st));
      }
    }
    if (warp >= 4) {
      // ------------------------------------------------------------ epilogue
      const int quarter = warp & 3;
      const int r = quarter * 32 + lane;
      const uint32_t lane_base = uint32_t(quarter * 32) << 16;
      const bool ok = __all_sync(0xffffffffu, wait_bar(bar(QS_DONE), 0, p.status, abort_flag));
      if (ok) {
        tc_fence_after();
        float* out = p.dq32 + ((s0 + i0 + r) * HQ + h) * (long)K;
#pragma unroll 1
        for (int c = 0; c < KD; c += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + c, v);
          tmem_wait_ld();
          if (r < ni) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(out + c + e) =
                  make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                              __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

template <int KD>
int launch_dq_ds(const AttnProblem& pb, const BwdArgs& a, const TcFwdWs& ws, int* status,
                 cudaStream_t stream) {
  const DsLayout lay = DsLayout::of_window(pb.window);
  const long tiles = DsLayout::total(lay, pb.rows, pb.T, pb.B, pb.HQ, pb.extra_blocks);
  CUtensorMap tds, tk;
  if (!make_rows128_map(&tds, a.dS, tiles * 128, 128, 64) ||
      !make_tile_map(&tk, ws.kh, pb.rows, pb.HQ, KD, BN))
    return WALL_ERR_CUDA;
  static bool attr[kMaxDevices] = {};
  if (!set_max_smem_once(bwd_dq_ds_kernel<KD>, QSmem<KD>::kAlloc, attr)) return WALL_ERR_CUDA;
  DqParams p;
  p.anchors = ws.anchors;
  p.lse = a.lse;
  p.D = a.D;
  p.GS = a.GS;
  p.dq32 = a.dq32;
  p.seqs = pb.seqs;
  p.HQ = pb.HQ;
  p.H = pb.H;
  p.scale_log2 = pb.scale * kLog2e;
  p.window = pb.window;
  p.n_blocks = ws.n_blocks128;
  p.status = status;
  dim3 grid(pb.HQ, ws.n_blocks128);
  bwd_dq_ds_kernel<KD><<<grid, kDsThreads, QSmem<KD>::kAlloc, stream>>>(tds, tk, p, lay);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

template <int KD>
int launch_dq(const AttnProblem& pb, const BwdArgs& a, const TcFwdWs& ws, int* status,
              cudaStream_t stream) {
  CUtensorMap tq, tk, tv, to;
  if (!make_tile_map(&tq, ws.qh, pb.rows, pb.HQ, KD, BM) ||
      !make_tile_map(&tk, ws.kh, pb.rows, pb.HQ, KD, BN) ||
      !make_tile_map(&tv, a.v, pb.rows, pb.H, KD, BN) ||
      !make_tile_map(&to, a.dO, pb.rows, pb.HQ, KD, BM))
    return WALL_ERR_CUDA;
  static bool attr[kMaxDevices] = {};
  if (!set_max_smem_once(bwd_dq_kernel<KD>, DSmem<KD>::kAlloc, attr)) return WALL_ERR_CUDA;
  DqParams p;
  p.anchors = ws.anchors;
  p.lse = a.lse;
  p.D = a.D;
  p.GS = a.GS;
  p.dq32 = a.dq32;
  p.seqs = pb.seqs;
  p.HQ = pb.HQ;
  p.H = pb.H;
  p.scale_log2 = pb.scale * kLog2e;
  p.window = pb.window;
  p.n_blocks = ws.n_blocks128;
  p.status = status;
  dim3 grid(pb.HQ, ws.n_blocks128);
  bwd_dq_kernel<KD><<<grid, kThreads, DSmem<KD>::kAlloc, stream>>>(tq, tk, tv, to, p);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

}  // namespace

int attn_bwd_dq_tc(const AttnProblem& pb, const BwdArgs& a, const TcFwdWs& ws, int* status,
                   cudaStream_t stream) {
  if (pb.rows == 0 || ws.n_blocks128 == 0) return WALL_OK;
  if (a.dS) {  // the key-block kernel stored its dS tiles
    return pb.K == 128 ? launch_dq_ds<128>(pb, a, ws, status, stream)
                       : launch_dq_ds<64>(pb, a, ws, status, stream);
  }
  return pb.K == 128 ? launch_dq<128>(pb, a, ws, status, stream)
                     : launch_dq<64>(pb, a, ws, status, stream);
}

}  // namespace wall
