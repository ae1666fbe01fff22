// wall_attn_bwd_sm100.cu -- tensor-core (tcgen05 + TMEM + TMA) Wall
// Attention backward for bf16 with K == V in {64, 128}.
//
// Gradients of the anchored form used by the forward (Tilde blog "Wall
// Attention", fast training sections 1 and 2).  For a 128-row query tile I
// (anchor R_I) and the CTA's 128-row key block J (anchor R_J), with
// d = 2^(R_I - R_J) per channel and Qt_I = Qh_I (.) d:
//   S^T  = Kh_J Qt_I^T              P_ij = 2^(S*scale*log2e + bias - lse2_i)
//   dP^T = V_J dO_I^T               dS_ij = P_ij (dP_ij - D_i)
//   dV_J  += P^T dO_I               (P^T from TMEM)
//   dKa_J += dS^T Qt_I              (dS^T from TMEM); dk_j = scale 2^(R_J - P_j) dKa_j
// dq comes from a separate query-block kernel (wall_attn_bwd_dq_sm100.cu), so
// no fp32 atomics are needed.
// The gate gradient needs dk per query head before the GQA sum; it is fused
// into the finalize kernel as dL = q (.) dq - k (.) dk^(h) (blog, fast
// training section 2: the key-side term is -K_j (.) dK_j), followed by the
// reverse scan.  The row part of the scalar-gate gradient is analytic,
// sum_j dS_ij = D_i * p_sink,i, and the column part is summed per key thread.
//
// Operands that the tensor core would otherwise read twice from shared memory
// (P^T, dS^T) are written back into TMEM as bf16 pairs over the S^T / dP^T
// columns they came from and fed as TMEM A operands.  All MMAs are M = 128,
// N = 128.
//
// CTA = one 128-row key block of one (sequence, head), 10 warps:
//   warp 0      TMA: Kh_J, V_J once; Qh_I (2 stages) and dO_I (1 stage, freed
//               by the first MMA that reads it last) per tile
//   warp 1      TMEM owner and MMA issuer
//   warps 2-5   Qt_I = Qh_I (.) d in shared memory
//   warps 6-9   one thread per key: P, dS; P^T, dS^T -> TMEM; column sums;
//               dK, dV epilogue at the end
#include <cuda.h>

#include <type_traits>

#include "sm100_ptx.cuh"
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

using namespace sm100;

constexpr int BQ = 128;  // query rows per tile
constexpr int BK = 128;  // key rows per CTA
constexpr int kThreads = 320;

struct BwdTcParams {
  const float* anchors;  // [nblk128, HQ, K]
  const float* P;        // [rows, HQ, K]
  const float* lse;      // [rows, HQ]
  const float* D;        // [rows, HQ]
  const float* GS;       // [rows, HQ] or nullptr
  float* dkh32;          // [rows, HQ, K]
  float* dvh32;          // [rows, HQ, V]
  float* dgs_col;        // [rows, HQ] or nullptr
  Seqs seqs;
  int HQ, H;
  float scale, scale_log2;
  int window;
  int n_blocks;
  int* status;
};

template <int KD>
struct BSmem {
  static constexpr int kKV = BK * KD * 2;   // key or value block
  static constexpr int kQ = BQ * KD * 2;    // query or dO tile
  static constexpr int oK = 0;
  static constexpr int oV = oK + kKV;
  static constexpr int oQ = oV + kKV;       // 2 stages
  static constexpr int oO = oQ + 2 * kQ;    // 2 stages
  static constexpr int oDw = oO + 2 * kQ;          // float[4 warps][KD]
  static constexpr int oRow = oDw + 4 * KD * 4;    // float[4 warps][2][BQ]
  static constexpr int oRI = oRow + 4 * 2 * BQ * 4;  // float[2 stages][KD]
  static constexpr int oRJ = oRI + 2 * KD * 4;       // float[KD]
  static constexpr int oBar = oRJ + KD * 4;
  static constexpr int kBars = 16;
  static constexpr int oMisc = oBar + kBars * 8;
  static constexpr int kBytes = oMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

enum BBar {
  KV_FULL = 0,
  Q_FULL = 1,     // +stage
  O_FULL = 3,     // +stage
  Q_READY = 5,    // +stage
  QO_EMPTY = 7,   // +stage
  SD_FULL = 9,    // +half
  P_FULL = 11,    // +half
  MM_DONE = 13,
  MMA_DONE = 14,
};

// TMEM columns (lanes = keys): S^T of the two 64-query halves [0,64),
// [64,128); dP^T halves [128,192), [192,256); the softmax writes P^T (dS^T)
// bf16 pairs over the first 32 columns of each S^T (dP^T) half; dV
// [256,384), dK [384,512).  While one half is in the softmax, the tensor core
// works on the other.
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, int* status,
                                         volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    // sleeps inside the instruction until the phase completes (or ~0.1 ms)
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
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  BwdTcParams p) {
  using Lay = BSmem<KD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* sDw = reinterpret_cast<float*>(smem + Lay::oDw);
  float* sRow = reinterpret_cast<float*>(smem + Lay::oRow);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::oBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::oMisc + 4);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.x;
  const int HQ = p.HQ, K = KD, V = KD;
  const int kh = h / (HQ / p.H);
  int seq, blk;
  // key blocks in ascending order: the early ones have the most query tiles
  if (!seq_block(p.seqs, BK, (int)blockIdx.y, seq, blk)) return;
  const int blk_off = (int)blockIdx.y - blk;
  const long s0 = p.seqs.start(seq);
  const int L = p.seqs.len(seq);
  const int j0 = blk * BK;
  const int nj = min(BK, L - j0);
  const int i_last = p.window > 0 ? min(L - 1, j0 + nj - 1 + p.window - 1) : L - 1;
  const int I0 = j0 / BQ;                 // first query tile (the diagonal one)
  const int nT = i_last / BQ - I0 + 1;
  const float* anc = p.anchors + ((long)blk_off * HQ + h) * K;  // + block * HQ * K

  if (threadIdx.x == 0) {
    mbar_init(bar(KV_FULL), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(Q_FULL + s), 1);
      mbar_init(bar(O_FULL + s), 1);
      mbar_init(bar(Q_READY + s), 4);
      mbar_init(bar(QO_EMPTY + s), 1);
      mbar_init(bar(SD_FULL + s), 1);
      mbar_init(bar(P_FULL + s), 4);
    }
    mbar_init(bar(MM_DONE), 1);
    mbar_init(bar(MMA_DONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  {
    float* rjs = reinterpret_cast<float*>(smem + Lay::oRJ);
    for (int n = threadIdx.x; n < K; n += kThreads) rjs[n] = anc[(long)blk * HQ * K + n];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_o);
      mbar_expect_tx(bar(KV_FULL), 2 * Lay::kKV);
      for (int b = 0; b < K / 64; ++b) {
        tma_load_3d(sbase + Lay::oK + b * (BK * 128), &tm_k, bar(KV_FULL), b * 64, h,
                    (int)(s0 + j0));
        tma_load_3d(sbase + Lay::oV + b * (BK * 128), &tm_v, bar(KV_FULL), b * 64, kh,
                    (int)(s0 + j0));
      }
      int issued = 0;
      for (int t = 0; t < nT; ++t) {
        const int st = t & 1;
        const int row = (int)(s0 + (long)(I0 + t) * BQ);
        if (t >= 2 && !wait_bar(bar(QO_EMPTY + st), ((t >> 1) - 1) & 1, p.status, abort_flag))
          break;
        mbar_expect_tx(bar(Q_FULL + st), Lay::kQ + K * 4);
        mbar_expect_tx(bar(O_FULL + st), Lay::kQ);
        for (int b = 0; b < K / 64; ++b) {
          tma_load_3d(sbase + Lay::oQ + st * Lay::kQ + b * (BQ * 128), &tm_q, bar(Q_FULL + st),
                      b * 64, h, row);
          tma_load_3d(sbase + Lay::oO + st * Lay::kQ + b * (BQ * 128), &tm_o, bar(O_FULL + st),
                      b * 64, h, row);
        }
        bulk_load(sbase + Lay::oRI + st * K * 4, anc + (long)(I0 + t) * HQ * K, K * 4,
                  bar(Q_FULL + st));
        issued = t + 1;
      }
      for (int t = max(0, issued - 2); t < issued; ++t) {
        mbar_wait(bar(Q_FULL + (t & 1)), (t >> 1) & 1, p.status);
        mbar_wait(bar(O_FULL + (t & 1)), (t >> 1) & 1, p.status);
      }
      mbar_wait(bar(KV_FULL), 0, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t id_sd = idesc_bf16(128, 64, false, false);  // S^T, dP^T halves
      const uint32_t id_acc = idesc_bf16(128, KD, false, true);  // dV, dK (A from TMEM)
      bool ok = wait_bar(bar(KV_FULL), 0, p.status, abort_flag);
      // S^T and dP^T of one 64-query half: M = 128 keys, N = 64, K = channels
      auto issue_sd = [&](int t, int hf) {
        const int st = t & 1;
        const uint32_t qa = sbase + Lay::oQ + st * Lay::kQ + hf * 64 * 128;
        const uint32_t oa = sbase + Lay::oO + st * Lay::kQ + hf * 64 * 128;
#pragma unroll
        for (int kk = 0; kk < KD / 16; ++kk) {
          const uint32_t offA = (kk >> 2) * (BK * 128) + (kk & 3) * 32;
          const uint32_t offB = (kk >> 2) * (BQ * 128) + (kk & 3) * 32;
          umma_bf16_ss(tmem + kColS + hf * 64, sdesc_sw128(sbase + Lay::oK + offA, 16, 1024),
                       sdesc_sw128(qa + offB, 16, 1024), id_sd, kk > 0);
          umma_bf16_ss(tmem + kColDP + hf * 64, sdesc_sw128(sbase + Lay::oV + offA, 16, 1024),
                       sdesc_sw128(oa + offB, 16, 1024), id_sd, kk > 0);
        }
        umma_commit(bar(SD_FULL + hf));
      };
      // dV += P^T dO and dK += dS^T Qt over one half: A from TMEM (8 columns
      // per 16 queries), B = dO / Qt rows of the half, MN-major
      auto issue_acc = [&](int t, int hf) {
        const int st = t & 1;
        const uint32_t qa = sbase + Lay::oQ + st * Lay::kQ + hf * 64 * 128;
        const uint32_t oa = sbase + Lay::oO + st * Lay::kQ + hf * 64 * 128;
#pragma unroll
        for (int kk = 0; kk < 64 / 16; ++kk) {
          const uint32_t acc = (t > 0 || hf > 0 || kk > 0) ? 1u : 0u;
          umma_bf16_ts(tmem + kColDV, tmem + kColS + hf * 64 + kk * 8,
                       sdesc_sw128(oa + kk * 16 * 128, BQ * 128, 1024), id_acc, acc);
          umma_bf16_ts(tmem + kColDK, tmem + kColDP + hf * 64 + kk * 8,
                       sdesc_sw128(qa + kk * 16 * 128, BQ * 128, 1024), id_acc, acc);
        }
      };
      auto tile_ready = [&](int t) -> bool {
        const int st = t & 1;
        if (!wait_bar(bar(Q_READY + st), (t >> 1) & 1, p.status, abort_flag)) return false;
        if (!wait_bar(bar(O_FULL + st), (t >> 1) & 1, p.status, abort_flag)) return false;
        tc_fence_after();
        return true;
      };
      if (ok) ok = tile_ready(0);
      if (ok) {
        issue_sd(0, 0);
        issue_sd(0, 1);
      }
      for (int t = 0; ok && t < nT; ++t) {
        const int st = t & 1;
        if (!wait_bar(bar(P_FULL + 0), t & 1, p.status, abort_flag)) break;
        tc_fence_after();
        issue_acc(t, 0);
        const bool next = t + 1 < nT;
        if (next) {
          if (!tile_ready(t + 1)) break;
          issue_sd(t + 1, 0);  // overwrites half a: in order after its dV/dK
        }
        if (!wait_bar(bar(P_FULL + 1), t & 1, p.status, abort_flag)) break;
        tc_fence_after();
        issue_acc(t, 1);
        umma_commit(bar(QO_EMPTY + st));
        if (next) issue_sd(t + 1, 1);
      }
      umma_commit(bar(MM_DONE));
      umma_commit(bar(MMA_DONE));
      mbar_wait(bar(MMA_DONE), 0, p.status);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ Qt rescale
    const int wt = threadIdx.x - 64;
    const int wq = warp - 2;
    const float* rjs = reinterpret_cast<const float*>(smem + Lay::oRJ);
    float* d = sDw + wq * KD;
    for (int t = 0; t < nT; ++t) {
      const int st = t & 1;
      const bool got = wait_bar(bar(Q_FULL + st), (t >> 1) & 1, p.status, abort_flag);
      if (!__all_sync(0xffffffffu, got)) break;
      const float* ri = reinterpret_cast<const float*>(smem + Lay::oRI + st * K * 4);
      __syncwarp();
      for (int c = lane; c < K; c += 32) d[c] = exp2f(ri[c] - rjs[c]);
      __syncwarp();
      uint8_t* qt = smem + Lay::oQ + st * Lay::kQ;
      constexpr int kPer = (KD / 64) * BQ * 8 / 128;  // chunks per thread
      constexpr int kBatch = 4;
#pragma unroll 1
      for (int b0 = 0; b0 < kPer; b0 += kBatch) {
        uint4 u[kBatch];
        float dd[kBatch][8];
        uint4* ptr[kBatch];
#pragma unroll
        for (int x = 0; x < kBatch; ++x) {
          const int c = wt + (b0 + x) * 128;
          const int box = c / (BQ * 8);
          const int row = (c / 8) % BQ;
          const int pch = c % 8;
          const int ch0 = box * 64 + ((pch ^ (row & 7)) * 8);
          ptr[x] = reinterpret_cast<uint4*>(qt + box * (BQ * 128) + row * 128 + pch * 16);
          u[x] = *ptr[x];
          const float4 da = *reinterpret_cast<const float4*>(d + ch0);
          const float4 db = *reinterpret_cast<const float4*>(d + ch0 + 4);
          dd[x][0] = da.x; dd[x][1] = da.y; dd[x][2] = da.z; dd[x][3] = da.w;
          dd[x][4] = db.x; dd[x][5] = db.y; dd[x][6] = db.z; dd[x][7] = db.w;
        }
#pragma unroll
        for (int x = 0; x < kBatch; ++x) {
          uint32_t* w = reinterpret_cast<uint32_t*>(&u[x]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w[e]));
            w[e] = pack_bf16x2(f.x * dd[x][2 * e], f.y * dd[x][2 * e + 1]);
          }
          *ptr[x] = u[x];
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(Q_READY + st));
    }
  } else {
    // ------------------------------------------------------------ P, dS per key (warps 6-9)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;   // key row within the block
    const int jj = j0 + r;               // key index within the sequence
    const bool key_ok = r < nj;
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    const float gs_j = (p.GS && key_ok) ? p.GS[(s0 + jj) * HQ + h] * kLog2e : 0.f;
    float* rowv = sRow + (warp - 6) * 2 * BQ;  // this warp's copy of the tile's query terms
    const int win = p.window > 0 ? p.window : 0x7fffffff;
    float colsum = 0.f;
    bool ok = true;
    for (int t = 0; t < nT && ok; ++t) {
      for (int hf = 0; hf < 2; ++hf) {
        const int i0 = (I0 + t) * BQ + hf * 64;  // first query of this half
        __syncwarp();
        // per query: c_i = GS_i*log2e - lse_i*log2e (logit offset), D_i
        for (int c = lane; c < 64; c += 32) {
          const int i = i0 + c;
          const bool in = i < L;
          const float gsi = (in && p.GS) ? p.GS[(s0 + i) * HQ + h] * kLog2e : 0.f;
          rowv[c] = in ? gsi - p.lse[(s0 + i) * HQ + h] * kLog2e : 0.f;
          rowv[BQ + c] = in ? p.D[(s0 + i) * HQ + h] : 0.f;
        }
        __syncwarp();
        {
          const bool got = wait_bar(bar(SD_FULL + hf), t & 1, p.status, abort_flag);
          if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        }
        tc_fence_after();
        // every query of the half sees this key: no mask work in the loop
        const bool full = key_ok && (i0 >= jj) && (i0 + 64 <= L) && (i0 + 63 - jj < win);
        const uint32_t scol = kColS + hf * 64, dcol = kColDP + hf * 64;
#pragma unroll 1
        for (int c = 0; c < 64; c += 32) {
          uint32_t sv[32], dv[32];
          tmem_ld32(tmem + lane_base + scol + c, sv);
          tmem_ld32(tmem + lane_base + dcol + c, dv);
          tmem_wait_ld();
          uint32_t pp[16], dd[16];
          auto group = [&](int g8, auto masked) {
            float pe[8], de[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int q = c + g8 * 8 + e;
              const float x =
                  fmaf(__uint_as_float(sv[g8 * 8 + e]), p.scale_log2, rowv[q] - gs_j);
              float pv;
              if constexpr (decltype(masked)::value) {
                const int i = i0 + q;
                const bool vis = key_ok & (i < L) & (jj <= i) & (i - jj < win);
                pv = vis ? exp2f(x) : 0.f;
              } else {
                pv = exp2f(x);
              }
              pe[e] = pv;
              de[e] = pv * (__uint_as_float(dv[g8 * 8 + e]) - rowv[BQ + q]);
            }
            colsum += ((de[0] + de[1]) + (de[2] + de[3])) + ((de[4] + de[5]) + (de[6] + de[7]));
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              pp[g8 * 4 + e] = pack_bf16x2(pe[2 * e], pe[2 * e + 1]);
              dd[g8 * 4 + e] = pack_bf16x2(de[2 * e], de[2 * e + 1]);
            }
          };
          if (full) {
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) group(g8, std::false_type{});
          } else {
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) group(g8, std::true_type{});
          }
          // P^T, dS^T as bf16 pairs over the consumed S^T / dP^T columns
          tmem_st16(tmem + lane_base + scol + c / 2, pp);
          tmem_st16(tmem + lane_base + dcol + c / 2, dd);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(P_FULL + hf));
      }
    }
    // ---- dK, dV epilogue for this key block
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(bar(MM_DONE), 0, p.status, abort_flag));
    if (ok) {
      tc_fence_after();
      const long krow = (s0 + jj) * HQ + h;
#pragma unroll 1
      for (int c = 0; c < KD; c += 32) {
        uint32_t kv[32], vv[32];
        tmem_ld32(tmem + lane_base + kColDK + c, kv);
        tmem_ld32(tmem + lane_base + kColDV + c, vv);
        tmem_wait_ld();
        if (key_ok) {
          const float* Pj = p.P + krow * K + c;
          const float* Rj = anc + (long)blk * HQ * K + c;
          float* dk = p.dkh32 + krow * K + c;
          float* dvp = p.dvh32 + krow * V + c;
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 pj = *reinterpret_cast<const float4*>(Pj + e);
            const float4 rj = *reinterpret_cast<const float4*>(Rj + e);
            float4 o;
            o.x = p.scale * exp2f(rj.x - pj.x) * __uint_as_float(kv[e]);
            o.y = p.scale * exp2f(rj.y - pj.y) * __uint_as_float(kv[e + 1]);
            o.z = p.scale * exp2f(rj.z - pj.z) * __uint_as_float(kv[e + 2]);
            o.w = p.scale * exp2f(rj.w - pj.w) * __uint_as_float(kv[e + 3]);
            *reinterpret_cast<float4*>(dk + e) = o;
            *reinterpret_cast<float4*>(dvp + e) =
                make_float4(__uint_as_float(vv[e]), __uint_as_float(vv[e + 1]),
                            __uint_as_float(vv[e + 2]), __uint_as_float(vv[e + 3]));
          }
        }
      }
      // the logit carries -GS_j for key j
      if (key_ok && p.dgs_col) p.dgs_col[krow] = -colsum;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// D_i = dO_i . o_i; row part of the scalar-gate gradient, sum_j dS_ij =
// D_i exp(sink - lse_i) (0 without a sink); dsink_h = -sum_i of the same.
__global__ void bwd_pre_kernel(const __nv_bfloat16* __restrict__ dO,
                               const __nv_bfloat16* __restrict__ o, const float* __restrict__ lse,
                               const float* __restrict__ sink, long rows, int HQ, int V,
                               float* __restrict__ D, float* __restrict__ dgs_row,
                               float* __restrict__ dsink) {
  const int lanes = 8;  // 8 threads per (row, head), 8 channels each per step
  const long nrh = rows * HQ;
  const long gid = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const long e = gid / lanes;
  const int sub = (int)(gid % lanes);
  float acc = 0.f;
  if (e < nrh) {
    for (int c = sub * 8; c < V; c += lanes * 8) {
      float a[8], b[8];
      load8(dO + e * V + c, a);
      load8(o + e * V + c, b);
#pragma unroll
      for (int x = 0; x < 8; ++x) acc += a[x] * b[x];
    }
  }
#pragma unroll
  for (int off = lanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (e < nrh && sub == 0) {
    D[e] = acc;
    const int h = (int)(e % HQ);
    const float ps = sink ? exp2f((sink[h] - lse[e]) * kLog2e) : 0.f;
    if (dgs_row) dgs_row[e] = acc * ps;
    if (dsink && sink) atomicAdd(&dsink[h], -acc * ps);
  }
}

// dq = scale * 2^(P - R_I) (.) dq32 for the tensor-core path (R_I = P at the
// row's 128-row block start), then dL = q (.) dq - k (.) dk^(h) over dq32;
// dk, dv = group sums; dGS = row + column parts.
template <typename T>
__global__ void bwd_finalize_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                    const float* __restrict__ P, Seqs seqs, int HQ, int H, int K,
                                    int V, float scale, float* __restrict__ dq32,
                                    const float* __restrict__ dkh32,
                                    const float* __restrict__ dvh32, float* __restrict__ dgs_row,
                                    const float* __restrict__ dgs_col, T* __restrict__ dq,
                                    T* __restrict__ dk, T* __restrict__ dv) {
  const int s = blockIdx.y;
  const long s0 = seqs.start(s);
  const int L = seqs.len(s);
  const int G = HQ / H;
  const long stride = (long)gridDim.x * blockDim.x;
  const long tid0 = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const int kg = K / 8;
  const long nq = (long)L * HQ * kg;
  for (long e = tid0; e < nq; e += stride) {
    const int g8 = (int)(e % kg);
    const int hh = (int)((e / kg) % HQ);
    const int t = (int)(e / ((long)kg * HQ));
    const long row = s0 + t;
    const long arow = s0 + (long)(t / 128) * 128;
    const long off = (row * HQ + hh) * K + g8 * 8;
    float pv[8], rv[8], a[8], qq[8], kk[8], dkv[8], out[8];
    load8(P + off, pv);
    load8(P + (arow * HQ + hh) * K + g8 * 8, rv);
    load8(dq32 + off, a);
    load8(q + off, qq);
    load8(k + (row * H + hh / G) * K + g8 * 8, kk);
    load8(dkh32 + off, dkv);
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      a[x] *= scale * exp2f(pv[x] - rv[x]);
      out[x] = qq[x] * a[x] - kk[x] * dkv[x];
    }
    store8(dq + off, a);
    store8(dq32 + off, out);
  }
  const long nk = (long)L * H * kg;
  for (long e = tid0; e < nk; e += stride) {
    const int g8 = (int)(e % kg);
    const int kv = (int)((e / kg) % H);
    const int t = (int)(e / ((long)kg * H));
    const long row = s0 + t;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0}, x[8];
    for (int g = 0; g < G; ++g) {
      load8(dkh32 + (row * HQ + kv * G + g) * K + g8 * 8, x);
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] += x[c];
    }
    store8(dk + (row * H + kv) * K + g8 * 8, acc);
  }
  const int vg = V / 8;
  const long nv = (long)L * H * vg;
  for (long e = tid0; e < nv; e += stride) {
    const int g8 = (int)(e % vg);
    const int kv = (int)((e / vg) % H);
    const int t = (int)(e / ((long)vg * H));
    const long row = s0 + t;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0}, x[8];
    for (int g = 0; g < G; ++g) {
      load8(dvh32 + (row * HQ + kv * G + g) * V + g8 * 8, x);
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] += x[c];
    }
    store8(dv + (row * H + kv) * V + g8 * 8, acc);
  }
  if (dgs_row && dgs_col) {
    for (long e = tid0; e < (long)L * HQ; e += stride) dgs_row[s0 * HQ + e] += dgs_col[s0 * HQ + e];
  }
}

template <int KD>
int launch_bwd_tc(const AttnProblem& pb, const BwdArgs& a, const TcFwdWs& ws, int* status,
                  cudaStream_t stream) {
  CUtensorMap tq, tk, tv, to;
  if (!make_tile_map(&tq, ws.qh, pb.rows, pb.HQ, KD, BQ) ||
      !make_tile_map(&tk, ws.kh, pb.rows, pb.HQ, KD, BK) ||
      !make_tile_map(&tv, a.v, pb.rows, pb.H, KD, BK) ||
      !make_tile_map(&to, a.dO, pb.rows, pb.HQ, KD, BQ))
    return WALL_ERR_CUDA;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(bwd_tc_kernel<KD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             BSmem<KD>::kAlloc) != cudaSuccess)
      return WALL_ERR_CUDA;
    attr = true;
  }
  BwdTcParams p;
  p.anchors = ws.anchors;
  p.P = a.P;
  p.lse = a.lse;
  p.D = a.D;
  p.GS = a.GS;
  p.dkh32 = a.dkh32;
  p.dvh32 = a.dvh32;
  p.dgs_col = a.GS ? a.dgs_col : nullptr;
  p.seqs = pb.seqs;
  p.HQ = pb.HQ;
  p.H = pb.H;
  p.scale = pb.scale;
  p.scale_log2 = pb.scale * kLog2e;
  p.window = pb.window;
  p.n_blocks = ws.n_blocks128;
  p.status = status;
  dim3 grid(pb.HQ, ws.n_blocks128);
  bwd_tc_kernel<KD><<<grid, kThreads, BSmem<KD>::kAlloc, stream>>>(tq, tk, tv, to, p);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

}  // namespace

int attn_bwd_tc(const AttnProblem& pb, const BwdArgs& a, const TcFwdWs& ws, void* dq, void* dk,
                void* dv, int* status, cudaStream_t stream) {
  if (pb.rows == 0 || ws.n_blocks128 == 0) return WALL_OK;
  int rc = attn_prepare_operands(pb, a.q, a.k, a.P, ws, stream);
  if (rc) return rc;
  {
    const long threads = pb.rows * pb.HQ * 8;
    const int blocks = (int)((threads + 255) / 256);
    bwd_pre_kernel<<<blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(a.dO), static_cast<const __nv_bfloat16*>(a.o), a.lse,
        a.sink, pb.rows, pb.HQ, pb.V, a.D, a.GS ? a.dgs_row : nullptr, a.dsink);
    if (cudaGetLastError() != cudaSuccess) return WALL_ERR_CUDA;
  }
  rc = pb.K == 128 ? launch_bwd_tc<128>(pb, a, ws, status, stream)
                   : launch_bwd_tc<64>(pb, a, ws, status, stream);
  if (rc) return rc;
  rc = attn_bwd_dq_tc(pb, a, ws, status, stream);
  if (rc) return rc;
  dim3 grid((148 * 8 + pb.seqs.n - 1) / (pb.seqs.n < 1 ? 1 : pb.seqs.n), pb.seqs.n);
  bwd_finalize_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k), a.P,
      pb.seqs, pb.HQ, pb.H, pb.K, pb.V, pb.scale, a.dq32, a.dkh32, a.dvh32,
      a.GS ? a.dgs_row : nullptr, a.GS ? a.dgs_col : nullptr, static_cast<__nv_bfloat16*>(dq),
      static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv));
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

}  // namespace wall
