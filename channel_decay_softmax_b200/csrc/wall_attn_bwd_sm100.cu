// wall_attn_bwd_sm100.cu -- tensor-core (tcgen05 + TMEM + TMA) Wall
// Attention backward for bf16 with K == V in {64, 128}: the key-block kernel
// (dK, dV) plus the D / sink pre-pass and the finalize kernel.
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
// no fp32 atomics are needed.  Unless the tiles would exceed their workspace
// cap this kernel also stores every dS tile it forms (bf16, as the dK MMA
// reads it; packed per (sequence, head) in the banded layout DsLayout
// describes, which covers varlen packing and windows), and the dq kernel is
// then one contraction dQa = dS Kt per tile instead of recomputing S, P, dP
// and dS.
// The gate gradient needs dk per query head before the GQA sum; it is fused
// into the finalize kernel as dL = q (.) dq - k (.) dk^(h) (blog, fast
// training section 2: the key-side term is -K_j (.) dK_j), followed by the
// reverse scan.  The row part of the scalar-gate gradient is analytic,
// sum_j dS_ij = D_i * p_sink,i, and the column part is summed per key thread.
//
// Shared memory is the scarce resource on sm_100: an M = N = 128 SS MMA
// already reads 128 B/clk.  So P^T and dS^T go back into TMEM as bf16 pairs
// and are read from there by the dV / dK MMAs, S^T and dP^T are single
// M = N = 128 MMAs, and the per-tile factor d is applied in place, one
// 16-byte chunk per load and store, to the query tile TMA brought in.
//
// CTA = one 128-row key block of one (sequence, head), 12 warps (3 per SM
// sub-partition, 168 registers each):
//   warp 0      TMA: Kh_J, V_J once; Qh_I with its anchors R_I (3 stages) and
//               dO_I (1 stage: dP(t+1) is the last MMA of a tile, so its load
//               overlaps the softmax of P(t+1)) per tile
//   warp 1      TMEM owner and MMA issuer.  Order per tile t:
//               dV(t), S(t+1), dK(t), dP(t+1), so that the tensor core works
//               on the next tile while the softmax computes dS(t)
//   warps 2-3   Qt_I = Qh_I (.) d in place; per-query terms (lse, D, gate)
//               of the tile, loaded two tiles ahead
//   warps 4-11  P, dS: one thread per (key, 64-query half of the tile); the
//               two warps of a TMEM lane quarter take the two halves.  dK, dV
//               epilogue at the end
#include <cuda.h>

#include <string.h>

#include <algorithm>

#include <type_traits>

#include "sm100_ptx.cuh"
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

using namespace sm100;

constexpr int BQ = 128;  // query rows per tile
constexpr int BK = 128;  // key rows per CTA
constexpr int kThreads = 384;

struct BwdTcParams {
  const __nv_bfloat16* qh;  // [rows, HQ, K] anchored queries
  const float* anchors;     // [nblk128, HQ, K]
  const float* P;           // [rows, HQ, K]
  const float* lse;         // [rows, HQ]
  const float* D;           // [rows, HQ]
  const float* GS;          // [rows, HQ] or nullptr
  float* dkh32;             // [rows, HQ, K]
  float* dvh32;             // [rows, HQ, V]
  float* dgs_col;           // [rows, HQ] or nullptr
  // dS^T tiles for the dq kernel, or nullptr: tile (s, h, I, J) at row
  // (ds_lay.pair_base(s, h) + ds_lay.rowstart(I) + J - ds_lay.jlo(I)) * 128,
  // rows = keys, 128 queries per row
  __nv_bfloat16* dS;
  DsLayout ds_lay;
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
  static constexpr int kStages = 3;         // query tiles in flight
  static constexpr int oQ = oV + kKV;       // kStages stages of Qt
  static constexpr int oO = oQ + kStages * kQ;  // dO, one stage
  static constexpr int oRow = oO + kQ;      // float[kStages][2][BQ]: c_i, D_i
  static constexpr int oCol = oRow + kStages * 2 * BQ * 4;  // float[BK]: column sums of the second half
  static constexpr int oRI = oCol + BK * 4;                 // float[kStages][KD]: R_I
  static constexpr int oBar = oRI + kStages * KD * 4;
  static constexpr int kBars = 20;
  static constexpr int oMisc = oBar + kBars * 8;
  // per softmax warp: its 32 keys x 32 queries of dS^T (bf16) on their way
  // to the stored tile by TMA
  static constexpr int oStg = (oMisc + 16 + 1023) & ~1023;
  static constexpr int kStg = 32 * 32 * 2;
  static constexpr int kBytes = oStg + 8 * kStg;
  static constexpr int kAlloc = kBytes + 1024;
};
static_assert(BSmem<128>::kAlloc <= 227 * 1024, "shared memory");

// barrier slots, laid out from the query-stage count
constexpr int kQStages = BSmem<128>::kStages;
static_assert(BSmem<64>::kStages == kQStages, "one query-stage count");
enum BBar {
  KV_FULL = 0,
  Q_FULL = 1,                       // + stage, TMA
  Q_READY = Q_FULL + kQStages,      // + stage, 2 producer warps
  Q_EMPTY = Q_READY + kQStages,     // + stage, tcgen05.commit after dK(t)
  O_FULL = Q_EMPTY + kQStages,      // TMA
  O_EMPTY = O_FULL + 1,             // tcgen05.commit after dV(t)
  S_FULL = O_EMPTY + 1,
  DP_FULL = S_FULL + 1,
  P_READY = DP_FULL + 1,            // 8 softmax warps
  DS_READY = P_READY + 1,           // 8 softmax warps
  MM_DONE = DS_READY + 1,
  MMA_DONE = MM_DONE + 1,
  COL_READY = MMA_DONE + 1,         // 4 warps of the second half: column sums in shared memory
  EPI_STAGED = COL_READY + 1,       // 8 softmax warps: dK, dV staged in shared memory
  kNumBBars = EPI_STAGED + 1,
};
static_assert(kNumBBars <= BSmem<128>::kBars, "barrier slots");

// TMEM columns (lanes = keys): S^T [0,128), dP^T [128,256), dV [256,384),
// dK [384,512).  The softmax half h (queries 64h..64h+63) writes its P^T
// (dS^T) bf16 pairs over the first 32 of its own 64 S^T (dP^T) columns.
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

// 2^k as bf16 bits for an integer k (the anchors are integers): exact in
// the normal range, 0 below it (a factor under 2^-126 scales an operand that
// decays to nothing) and +inf above it, as the fp32 product would overflow.
__device__ __forceinline__ uint32_t pow2_bf16(float k) {
  const int e = (int)k;
  return e < -126 ? 0u : e > 127 ? 0x7F80u : uint32_t(e + 127) << 7;
}

// 8 bf16 times 8 per-channel powers of two (bf16x2 pairs): exact
__device__ __forceinline__ uint4 scale8(uint4 u, const __nv_bfloat162 (&d)[4]) {
  __nv_bfloat162* w = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) w[e] = __hmul2(w[e], d[e]);
  return u;
}

template <int KD, bool kGS>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const __grid_constant__ CUtensorMap tm_ds, BwdTcParams p) {
  using Lay = BSmem<KD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* sRow = reinterpret_cast<float*>(smem + Lay::oRow);
  float* sCol = reinterpret_cast<float*>(smem + Lay::oCol);
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
    for (int s = 0; s < Lay::kStages; ++s) {
      mbar_init(bar(Q_READY + s), 2);
      mbar_init(bar(Q_FULL + s), 1);
      mbar_init(bar(Q_EMPTY + s), 1);
    }
    mbar_init(bar(O_FULL), 1);
    mbar_init(bar(O_EMPTY), 1);
    mbar_init(bar(S_FULL), 1);
    mbar_init(bar(DP_FULL), 1);
    mbar_init(bar(P_READY), 8);
    mbar_init(bar(DS_READY), 8);
    mbar_init(bar(MM_DONE), 1);
    mbar_init(bar(MMA_DONE), 1);
    mbar_init(bar(COL_READY), 4);
    mbar_init(bar(EPI_STAGED), 8);
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
    // lane 0: Kh_J, V_J and the query ring; lane 1: dO (one stage).  The two
    // lanes wait on different barriers and progress independently.
    constexpr int NS = Lay::kStages;
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_expect_tx(bar(KV_FULL), 2 * Lay::kKV);
      for (int b = 0; b < K / 64; ++b) {
        tma_load_3d(sbase + Lay::oK + b * (BK * 128), &tm_k, bar(KV_FULL), b * 64, h,
                    (int)(s0 + j0));
        tma_load_3d(sbase + Lay::oV + b * (BK * 128), &tm_v, bar(KV_FULL), b * 64, kh,
                    (int)(s0 + j0));
      }
      int issued = 0;
      for (int t = 0; t < nT; ++t) {
        const int st = t % NS;
        if (t >= NS && !wait_bar(bar(Q_EMPTY + st), (t / NS - 1) & 1, p.status, abort_flag))
          break;
        mbar_expect_tx(bar(Q_FULL + st), Lay::kQ + K * 4);
        const int row = (int)(s0 + (long)(I0 + t) * BQ);
        for (int b = 0; b < K / 64; ++b)
          tma_load_3d(sbase + Lay::oQ + st * Lay::kQ + b * (BQ * 128), &tm_q, bar(Q_FULL + st),
                      b * 64, h, row);
        bulk_load(sbase + Lay::oRI + st * K * 4, anc + (long)(I0 + t) * HQ * K, K * 4,
                  bar(Q_FULL + st));
        issued = t + 1;
      }
      // no copy may still be in flight when the CTA exits
      for (int t = max(0, issued - NS); t < issued; ++t)
        mbar_wait(bar(Q_FULL + t % NS), (t / NS) & 1, p.status);
      mbar_wait(bar(KV_FULL), 0, p.status);
    } else if (lane == 1) {
      tma_prefetch_desc(&tm_o);
      int issued = 0;
      for (int t = 0; t < nT; ++t) {
        // dO(t) goes into the stage once dV(t - 1) has read dO(t - 1)
        if (t >= 1 && !wait_bar(bar(O_EMPTY), (t - 1) & 1, p.status, abort_flag)) break;
        mbar_expect_tx(bar(O_FULL), Lay::kQ);
        const int row = (int)(s0 + (long)(I0 + t) * BQ);
        for (int b = 0; b < K / 64; ++b)
          tma_load_3d(sbase + Lay::oO + b * (BQ * 128), &tm_o, bar(O_FULL), b * 64, h, row);
        issued = t + 1;
      }
      if (issued > 0) mbar_wait(bar(O_FULL), (issued - 1) & 1, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t id_sd = idesc_bf16(128, 128, false, false);  // S^T, dP^T
      const uint32_t id_acc = idesc_bf16(128, KD, false, true);   // dV, dK (A from TMEM)
      // S^T (dP^T) of the whole tile: M = 128 keys, N = 128 queries, K = channels
      auto issue_sd = [&](uint32_t a_off, uint32_t b_off, uint32_t col) {
#pragma unroll
        for (int kk = 0; kk < KD / 16; ++kk) {
          const uint32_t offA = (kk >> 2) * (BK * 128) + (kk & 3) * 32;
          const uint32_t offB = (kk >> 2) * (BQ * 128) + (kk & 3) * 32;
          umma_bf16_ss(tmem + col, sdesc_sw128(sbase + a_off + offA, 16, 1024),
                       sdesc_sw128(sbase + b_off + offB, 16, 1024), id_sd, kk > 0);
        }
      };
      // dV += P^T dO (dK += dS^T Qt): A from TMEM, 8 columns per 16 queries,
      // the two 64-query halves 64 columns apart; B = rows of the tile, MN-major
      auto issue_acc = [&](uint32_t a_col, uint32_t b_off, uint32_t d_col, bool first) {
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk) {
          umma_bf16_ts(tmem + d_col, tmem + a_col + (kk >> 2) * 64 + (kk & 3) * 8,
                       sdesc_sw128(sbase + b_off + kk * 16 * 128, BQ * 128, 1024), id_acc,
                       (first && kk == 0) ? 0u : 1u);
        }
      };
      constexpr int NS = Lay::kStages;
      auto q_off = [&](int t) { return (uint32_t)(Lay::oQ + (t % NS) * Lay::kQ); };
      const uint32_t o_off = Lay::oO;
      bool ok = wait_bar(bar(KV_FULL), 0, p.status, abort_flag);
      if (ok) ok = wait_bar(bar(Q_READY), 0, p.status, abort_flag);
      if (ok) ok = wait_bar(bar(O_FULL), 0, p.status, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_sd(Lay::oK, q_off(0), kColS);
        umma_commit(bar(S_FULL));
        issue_sd(Lay::oV, o_off, kColDP);
        umma_commit(bar(DP_FULL));
      }
      for (int t = 0; ok && t < nT; ++t) {
        const int st = t % NS;
        const bool next = t + 1 < nT;
        if (!wait_bar(bar(P_READY), t & 1, p.status, abort_flag)) break;
        tc_fence_after();
        issue_acc(kColS, o_off, kColDV, t == 0);
        umma_commit(bar(O_EMPTY));
        // S(t+1) may go before dK(t) (the tensor core then works while the
        // softmax finishes dS(t)), but only if its query tile is ready:
        // dK(t) frees the stage the tile after next is written to
        const uint32_t q_next = bar(Q_READY + (t + 1) % NS);
        const uint32_t q_par = ((t + 1) / NS) & 1;
        bool s_done = false;
        if (next && mbar_try_wait(q_next, q_par)) {
          tc_fence_after();
          issue_sd(Lay::oK, q_off(t + 1), kColS);  // in order after dV(t) read P^T
          umma_commit(bar(S_FULL));
          s_done = true;
        }
        if (!wait_bar(bar(DS_READY), t & 1, p.status, abort_flag)) break;
        tc_fence_after();
        issue_acc(kColDP, q_off(t), kColDK, t == 0);
        umma_commit(bar(Q_EMPTY + st));
        if (next && !s_done) {
          if (!wait_bar(q_next, q_par, p.status, abort_flag)) break;
          tc_fence_after();
          issue_sd(Lay::oK, q_off(t + 1), kColS);
          umma_commit(bar(S_FULL));
        }
        if (next) {
          if (!wait_bar(bar(O_FULL), (t + 1) & 1, p.status, abort_flag)) break;
          tc_fence_after();
          issue_sd(Lay::oV, o_off, kColDP);  // in order after dK(t) read dS^T
          umma_commit(bar(DP_FULL));
        }
      }
      umma_commit(bar(MM_DONE));
      umma_commit(bar(MMA_DONE));
      mbar_wait(bar(MMA_DONE), 0, p.status);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ Qt producer
    constexpr int kChunks = KD / 8;          // 16-byte chunks per row
    constexpr int kRowStep = 64 / kChunks;   // rows covered by one pass of 64 threads
    constexpr int kRows = BQ / kRowStep;     // rows per thread
    const int tid = threadIdx.x - 64;
    const int ch = tid % kChunks;
    const int rs = tid / kChunks;
    float rj[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) rj[e] = __ldg(anc + (long)blk * HQ * K + ch * 8 + e);
    // per-query terms two tiles ahead: plain loads take a few microseconds
    // while the tensor core streams
    float cc[2], dc[2], cn[2], dn[2];  // tiles t and t + 1
    auto rows_of = [&](int t, float (&c)[2], float (&dd)[2]) {
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int i = (I0 + t) * BQ + tid + 64 * x;
        const long e = (s0 + i) * HQ + h;
        const bool in = t < nT && i < L;
        c[x] = in ? ((kGS ? __ldg(p.GS + e) : 0.f) - __ldg(p.lse + e)) * kLog2e : 0.f;
        dd[x] = in ? __ldg(p.D + e) : 0.f;
      }
    };
    rows_of(0, cc, dc);
    rows_of(1, cn, dn);
    for (int t = 0; t < nT; ++t) {
      const int st = t % Lay::kStages;
      {
        const bool got = wait_bar(bar(Q_FULL + st), (t / Lay::kStages) & 1, p.status, abort_flag);
        if (!__all_sync(0xffffffffu, got)) break;
      }
      const float* ri = reinterpret_cast<const float*>(smem + Lay::oRI + st * K * 4) + ch * 8;
      __nv_bfloat162 d[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t b = pow2_bf16(ri[2 * e] - rj[2 * e]) |
                           (pow2_bf16(ri[2 * e + 1] - rj[2 * e + 1]) << 16);
        d[e] = *reinterpret_cast<const __nv_bfloat162*>(&b);
      }
      uint8_t* qt = smem + Lay::oQ + st * Lay::kQ + (ch / 8) * (BQ * 128);
      constexpr int kBatch = 8;
#pragma unroll
      for (int m0 = 0; m0 < kRows; m0 += kBatch) {
        uint4 v[kBatch];
#pragma unroll
        for (int x = 0; x < kBatch; ++x) {
          const int r = rs + (m0 + x) * kRowStep;
          v[x] = *reinterpret_cast<const uint4*>(qt + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
        }
#pragma unroll
        for (int x = 0; x < kBatch; ++x) {
          const int r = rs + (m0 + x) * kRowStep;
          *reinterpret_cast<uint4*>(qt + r * 128 + (((ch & 7) ^ (r & 7)) << 4)) = scale8(v[x], d);
        }
      }
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        sRow[st * 2 * BQ + tid + 64 * x] = cc[x];
        sRow[st * 2 * BQ + BQ + tid + 64 * x] = dc[x];
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(Q_READY + st));
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        cc[x] = cn[x];
        dc[x] = dn[x];
      }
      rows_of(t + 2, cn, dn);
    }
  } else {
    // ------------------------------------------------------------ P, dS (warps 4-11)
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;    // queries 64*half .. 64*half+63 of each tile
    const int r = quarter * 32 + lane;   // key row within the block
    const int jj = j0 + r;               // key index within the sequence
    const bool key_ok = r < nj;
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    const float gs_j = (kGS && key_ok) ? p.GS[(s0 + jj) * HQ + h] * kLog2e : 0.f;
    const int win = p.window > 0 ? p.window : 0x7fffffff;
    const uint32_t scol = kColS + half * 64, dcol = kColDP + half * 64;
    // the stored dS tile (I, J = blk) of every query tile I this key block
    // meets, rows = keys, 128 queries each; this warp's 32 keys x 32 queries
    // go through its staging block
    const bool store_ds = p.dS != nullptr;
    const long ds_base = store_ds ? p.ds_lay.pair_base(p.seqs, HQ, seq, h) : 0;
    auto ds_tile_of = [&](int I) {
      return ds_base + p.ds_lay.rowstart(I) + blk - p.ds_lay.jlo(I);
    };
    long ds_tile = store_ds ? ds_tile_of(I0) : 0;
    uint8_t* stg = smem + Lay::oStg + (warp - 4) * Lay::kStg;
    float colsum = 0.f;
    bool ok = true;
    for (int t = 0; t < nT && ok; ++t) {
      const int st = t % Lay::kStages;
      const int i0 = (I0 + t) * BQ + half * 64;  // first query of this half
      const float* cv = sRow + st * 2 * BQ + half * 64;
      const float* dvv = cv + BQ;
      // The logit offsets of the half's queries are read before the wait for
      // S: while the tensor core streams operands, a shared-memory load takes
      // hundreds of cycles, and here that latency overlaps the wait.
      float cr[64];
      {
        // acquire the producers' per-query terms (that phase has completed)
        const bool got =
            wait_bar(bar(Q_READY + st), (t / Lay::kStages) & 1, p.status, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      }
#pragma unroll
      for (int e = 0; e < 64; e += 4) {
        const float4 c4 = *reinterpret_cast<const float4*>(cv + e);
        cr[e] = c4.x;
        cr[e + 1] = c4.y;
        cr[e + 2] = c4.z;
        cr[e + 3] = c4.w;
      }
      {
        const bool got = wait_bar(bar(S_FULL), t & 1, p.status, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      }
      tc_fence_after();
      // every query of the half sees every key of the warp: no mask work in the
      // loop.  Warp-uniform, since the branch holds the warp-wide TMEM loads
      const bool full = __all_sync(
          0xffffffffu, key_ok && (i0 >= jj) && (i0 + 64 <= L) && (i0 + 63 - jj < win));
      float pv[64];
      auto p_part = [&](auto masked) {
        uint32_t sv[64];  // both loads in flight before the one wait
        tmem_ld32(tmem + lane_base + scol, sv);
        tmem_ld32(tmem + lane_base + scol + 32, sv + 32);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const float cx = cr[c + e + x];
              const float arg = fmaf(__uint_as_float(sv[c + e + x]), p.scale_log2,
                                     kGS ? cx - gs_j : cx);
              // all on MUFU: moving part of them to an FMA-pipe polynomial
              // costs more issue slots than it frees on MUFU (measured)
              const float ev = exp2f(arg);
              if constexpr (decltype(masked)::value) {
                const int i = i0 + c + e + x;
                const bool vis = key_ok & (i < L) & (jj <= i) & (i - jj < win);
                pv[c + e + x] = vis ? ev : 0.f;
              } else {
                pv[c + e + x] = ev;
              }
            }
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(pv[c + 2 * e], pv[c + 2 * e + 1]);
          tmem_st16(tmem + lane_base + scol + c / 2, pk);
        }
      };
      if (full)
        p_part(std::false_type{});
      else
        p_part(std::true_type{});
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(P_READY));
      {
        const bool got = wait_bar(bar(DP_FULL), t & 1, p.status, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      }
      tc_fence_after();
      uint32_t dv[64];
      tmem_ld32(tmem + lane_base + dcol, dv);
      tmem_ld32(tmem + lane_base + dcol + 32, dv + 32);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 d4 = *reinterpret_cast<const float4*>(dvv + c + e);
          const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const float ds = pv[c + e + x] * (__uint_as_float(dv[c + e + x]) - dd[x]);
            if (kGS) colsum += ds;
            pv[c + e + x] = ds;
          }
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(pv[c + 2 * e], pv[c + 2 * e + 1]);
        tmem_st16(tmem + lane_base + dcol + c / 2, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(DS_READY));
      if (store_ds) {
        // off the MMA's path: the same bf16 values, 32 queries at a time,
        // this key's 64 bytes into the staging block (64-byte swizzle: the
        // 16-byte chunk index XOR bits 1-2 of the row, conflict-free) once
        // the previous store has read it, then one TMA store of the warp's
        // 32 keys x 32 queries
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint4 v = make_uint4(pack_bf16x2(pv[c + 8 * e], pv[c + 8 * e + 1]),
                                       pack_bf16x2(pv[c + 8 * e + 2], pv[c + 8 * e + 3]),
                                       pack_bf16x2(pv[c + 8 * e + 4], pv[c + 8 * e + 5]),
                                       pack_bf16x2(pv[c + 8 * e + 6], pv[c + 8 * e + 7]));
            *reinterpret_cast<uint4*>(stg + lane * 64 + ((e ^ ((lane >> 1) & 3)) << 4)) = v;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tm_ds, smem_u32(stg), half * 64 + c, (int)(ds_tile * BK + quarter * 32));
            bulk_commit();
          }
        }
        ds_tile = ds_tile_of(I0 + t + 1);
      }
    }
    // The epilogue's rows of P and the block's anchors, loaded now so that
    // their latency overlaps the last MMAs and the staging below.  Warp w
    // takes rows w, w + 8, ...; lane = KD/32 consecutive channels;
    // dk_j = scale 2^(R_J - P_j) dKa_j
    constexpr int CPL = KD / 32;
    const int c0 = lane * CPL;
    float rjv[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) rjv[i] = anc[(long)blk * HQ * K + c0 + i];
    constexpr int kRowsPerWarp = BK / 8;
    float pj[kRowsPerWarp][CPL];
#pragma unroll
    for (int x = 0; x < kRowsPerWarp; ++x) {
      const int rr = (warp - 4) + 8 * x;
      const long krow = (s0 + j0 + (rr < nj ? rr : 0)) * HQ + h;
      if constexpr (CPL == 4) {
        const float4 a = *reinterpret_cast<const float4*>(p.P + krow * K + c0);
        pj[x][0] = a.x; pj[x][1] = a.y; pj[x][2 % CPL] = a.z; pj[x][3 % CPL] = a.w;
      } else {
        const float2 a = *reinterpret_cast<const float2*>(p.P + krow * K + c0);
        pj[x][0] = a.x; pj[x][1 % CPL] = a.y;
      }
    }
    // the stored tiles are complete before the CTA can exit
    if (store_ds && lane == 0) bulk_wait_all();
    // ---- dK, dV epilogue.  Thread = key row in TMEM, but a row per thread
    // makes every global access of a warp touch 32 rows: the accumulators go
    // through shared memory (free once every MMA has completed), then each
    // warp writes whole rows.  Staging layout: fp32 [2][BK][KD], 16-byte group
    // g of row r at group g ^ (r & 7), so both the row-wise writes and the
    // column-wise reads spread over all banks.
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(bar(MM_DONE), 0, p.status, abort_flag));
    float* stage = reinterpret_cast<float*>(smem);  // the K, V, query and dO buffers
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int c = half * (KD / 2); c < (half + 1) * (KD / 2); c += 32) {
        uint32_t kv[32], vv[32];
        tmem_ld32(tmem + lane_base + kColDK + c, kv);
        tmem_ld32(tmem + lane_base + kColDV + c, vv);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const int pos = r * KD + ((((c + e) >> 2) ^ (r & 7)) << 2);
          *reinterpret_cast<float4*>(stage + pos) =
              make_float4(__uint_as_float(kv[e]), __uint_as_float(kv[e + 1]),
                          __uint_as_float(kv[e + 2]), __uint_as_float(kv[e + 3]));
          *reinterpret_cast<float4*>(stage + BK * KD + pos) =
              make_float4(__uint_as_float(vv[e]), __uint_as_float(vv[e + 1]),
                          __uint_as_float(vv[e + 2]), __uint_as_float(vv[e + 3]));
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(EPI_STAGED));  // every warp arrives, even after an abort
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(bar(EPI_STAGED), 0, p.status, abort_flag));
    if (ok) {
#pragma unroll
      for (int x = 0; x < kRowsPerWarp; ++x) {
        const int rr = (warp - 4) + 8 * x;
        if (rr >= nj) break;
        const long krow = (s0 + j0 + rr) * HQ + h;
        const int pos = rr * KD + (((c0 >> 2) ^ (rr & 7)) << 2) + (c0 & 3);
        float ka[CPL], va[CPL], ko[CPL];
        if constexpr (CPL == 4) {
          const float4 b = *reinterpret_cast<const float4*>(stage + pos);
          const float4 d = *reinterpret_cast<const float4*>(stage + BK * KD + pos);
          ka[0] = b.x; ka[1] = b.y; ka[2 % CPL] = b.z; ka[3 % CPL] = b.w;
          va[0] = d.x; va[1] = d.y; va[2 % CPL] = d.z; va[3 % CPL] = d.w;
        } else {
          const float2 b = *reinterpret_cast<const float2*>(stage + pos);
          const float2 d = *reinterpret_cast<const float2*>(stage + BK * KD + pos);
          ka[0] = b.x; ka[1 % CPL] = b.y;
          va[0] = d.x; va[1 % CPL] = d.y;
        }
#pragma unroll
        for (int i = 0; i < CPL; ++i) ko[i] = p.scale * exp2f(rjv[i] - pj[x][i]) * ka[i];
        float* dk = p.dkh32 + krow * K + c0;
        float* dvp = p.dvh32 + krow * V + c0;
        if constexpr (CPL == 4) {
          *reinterpret_cast<float4*>(dk) = make_float4(ko[0], ko[1], ko[2 % CPL], ko[3 % CPL]);
          *reinterpret_cast<float4*>(dvp) = make_float4(va[0], va[1], va[2 % CPL], va[3 % CPL]);
        } else {
          *reinterpret_cast<float2*>(dk) = make_float2(ko[0], ko[1 % CPL]);
          *reinterpret_cast<float2*>(dvp) = make_float2(va[0], va[1 % CPL]);
        }
      }
    }
    if (kGS) {
      // column sums of the two halves meet in shared memory; the logit
      // carries -GS_j for key j
      if (half == 1) {
        sCol[r] = colsum;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(COL_READY));
      } else {
        const bool got = wait_bar(bar(COL_READY), 0, p.status, abort_flag);
        if (ok && got && key_ok && p.dgs_col) p.dgs_col[(s0 + jj) * HQ + h] = -(colsum + sCol[r]);
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

// D_i = dO_i . o_i; row part of the scalar-gate gradient, sum_j dS_ij =
// D_i exp(sink - lse_i) (0 without a sink).
__global__ void bwd_pre_kernel(const __nv_bfloat16* __restrict__ dO,
                               const __nv_bfloat16* __restrict__ o, const float* __restrict__ lse,
                               const float* __restrict__ sink, long rows, int HQ, int V,
                               float* __restrict__ D, float* __restrict__ dgs_row) {
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
  }
}

// dsink_h = -sum_i exp(sink_h - lse_i) D_i (the sink's logit has a zero value
// row), summed in a fixed order so that repeated calls agree bit for bit.
// Two passes: CTA b sums rows [b R, (b + 1) R) per head (thread t takes head
// t % HQ and every (256 / HQ)-th row, so a warp reads consecutive words),
// then one warp per head adds the CTAs' partials in a fixed order.
__global__ void __launch_bounds__(256)
    sink_partial_kernel(const float* __restrict__ D, const float* __restrict__ lse,
                        const float* __restrict__ sink, long rows, int HQ, long rows_per_cta,
                        float* __restrict__ part) {
  __shared__ float acc_s[256];
  const int per = 256 / HQ;  // threads per head
  const int t = threadIdx.x, h = t % HQ, k = t / HQ;
  float acc = 0.f;
  if (k < per) {
    const float s2 = sink[h] * kLog2e;
    const long r0 = (long)blockIdx.x * rows_per_cta;
    const long r1 = r0 + rows_per_cta < rows ? r0 + rows_per_cta : rows;
    for (long r = r0 + k; r < r1; r += per) {
      const long e = r * HQ + h;
      acc -= exp2f(s2 - lse[e] * kLog2e) * D[e];
    }
  }
  acc_s[t] = acc;
  __syncthreads();
  if (t < HQ) {
    float sum = 0.f;
    for (int x = 0; x < per; ++x) sum += acc_s[t + x * HQ];
    part[(long)blockIdx.x * HQ + t] = sum;
  }
}

// one warp per head: lane l adds partials l, l + 32, ... in order, then a
// fixed shuffle tree
__global__ void sink_final_kernel(const float* __restrict__ part, int nb, int HQ,
                                  float* __restrict__ dsink) {
  const int h = (int)((blockIdx.x * blockDim.x + threadIdx.x) / 32), lane = threadIdx.x % 32;
  if (h >= HQ) return;
  float sum = 0.f;
  for (int b = lane; b < nb; b += 32) sum += part[(long)b * HQ + h];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane == 0) dsink[h] = sum;
}

// The one-CTA-per-head form of the same sum, for more than 256 heads.
__global__ void __launch_bounds__(256)
    sink_grad_kernel(const float* __restrict__ D, const float* __restrict__ lse,
                     const float* __restrict__ sink, long rows, int HQ,
                     float* __restrict__ dsink) {
  __shared__ float part[256];
  const int h = blockIdx.x;
  const float s2 = sink[h] * kLog2e;
  float acc = 0.f;
  for (long t = threadIdx.x; t < rows; t += 256) {
    const long e = t * HQ + h;
    acc -= exp2f(s2 - lse[e] * kLog2e) * D[e];
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) dsink[h] = part[0];
}

// dk, dv = sums of the per-query-head dk^(h), dv^(h) over each GQA group;
// dGS = row + column parts.  (dq and the gate-gradient summand dL come from
// finalize_dq_dl_sums, fused with the reverse scan's first pass.)
template <typename T>
__global__ void bwd_finalize_kernel(Seqs seqs, int HQ, int H, int K, int V,
                                    const float* __restrict__ dkh32,
                                    const float* __restrict__ dvh32, float* __restrict__ dgs_row,
                                    const float* __restrict__ dgs_col, T* __restrict__ dk,
                                    T* __restrict__ dv) {
  // CTAs take rows of the sequence, threads the row's (kv head, 8 channels)
  // groups of dk then dv: 32-bit arithmetic only, and each group's G loads
  // issued together
  const int s = blockIdx.y;
  const long s0 = seqs.start(s);
  const int L = seqs.len(s);
  const int G = HQ / H;
  const int kg = K / 8, vg = V / 8;
  const int per_k = H * kg, per_row = H * (kg + vg);
  for (int t = blockIdx.x; t < L; t += gridDim.x) {
    const long row = s0 + t;
    for (int i = threadIdx.x; i < per_row; i += blockDim.x) {
      const bool is_k = i < per_k;
      const int j = is_k ? i : i - per_k;
      const int D = is_k ? K : V;
      const int ng = is_k ? kg : vg;
      const int kv = j / ng;
      const int n0 = (j - kv * ng) * 8;
      const float* src = (is_k ? dkh32 : dvh32) + (row * HQ + kv * G) * D + n0;
      float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0}, x[8];
#pragma unroll 4
      for (int g = 0; g < G; ++g) {
        load8(src + (long)g * D, x);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] += x[c];
      }
      store8((is_k ? dk : dv) + (row * H + kv) * D + n0, acc);
    }
  }
  if (dgs_row && dgs_col) {
    const long stride = (long)gridDim.x * blockDim.x;
    for (long e = (long)blockIdx.x * blockDim.x + threadIdx.x; e < (long)L * HQ; e += stride)
      dgs_row[s0 * HQ + e] += dgs_col[s0 * HQ + e];
  }
}

template <int KD, bool kGS>
int launch_bwd_tc(const AttnProblem& pb, const BwdArgs& a, const TcFwdWs& ws, int* status,
                  cudaStream_t stream) {
  CUtensorMap tq, tk, tv, to, tds;
  if (!make_tile_map(&tq, ws.qh, pb.rows, pb.HQ, KD, BQ) ||
      !make_tile_map(&tk, ws.kh, pb.rows, pb.HQ, KD, BK) ||
      !make_tile_map(&tv, a.v, pb.rows, pb.H, KD, BK) ||
      !make_tile_map(&to, a.dO, pb.rows, pb.HQ, KD, BQ))
    return WALL_ERR_CUDA;
  memset(&tds, 0, sizeof(tds));  // unused without stored dS tiles
  const DsLayout lay = DsLayout::of_window(pb.window);
  if (a.dS && !make_rows128_map(&tds, a.dS,
                                DsLayout::total(lay, pb.rows, pb.T, pb.B, pb.HQ,
                                                pb.extra_blocks) * BK,
                                32, 32))
    return WALL_ERR_CUDA;
  static bool attr[kMaxDevices] = {};
  if (!set_max_smem_once(bwd_tc_kernel<KD, kGS>, BSmem<KD>::kAlloc, attr)) return WALL_ERR_CUDA;
  BwdTcParams p;
  p.qh = static_cast<const __nv_bfloat16*>(ws.qh);
  p.anchors = ws.anchors;
  p.P = a.P;
  p.lse = a.lse;
  p.D = a.D;
  p.GS = a.GS;
  p.dkh32 = a.dkh32;
  p.dvh32 = a.dvh32;
  p.dgs_col = a.GS ? a.dgs_col : nullptr;
  p.dS = a.dS;
  p.ds_lay = lay;
  p.seqs = pb.seqs;
  p.HQ = pb.HQ;
  p.H = pb.H;
  p.scale = pb.scale;
  p.scale_log2 = pb.scale * kLog2e;
  p.window = pb.window;
  p.n_blocks = ws.n_blocks128;
  p.status = status;
  dim3 grid(pb.HQ, ws.n_blocks128);
  bwd_tc_kernel<KD, kGS><<<grid, kThreads, BSmem<KD>::kAlloc, stream>>>(tq, tk, tv, to, tds, p);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

template <int KD>
int launch_bwd_tc_gs(const AttnProblem& pb, const BwdArgs& a, const TcFwdWs& ws, int* status,
                     cudaStream_t stream) {
  return a.GS ? launch_bwd_tc<KD, true>(pb, a, ws, status, stream)
              : launch_bwd_tc<KD, false>(pb, a, ws, status, stream);
}

}  // namespace

int sink_grad(const float* D, const float* lse, const float* sink, long rows, int HQ,
              float* scratch, float* dsink, cudaStream_t stream) {
  if (rows <= 0 || HQ <= 0) return WALL_OK;
  if (HQ <= 256) {
    const long nb = std::min<long>((rows + 63) / 64, 4 * 148);
    const long per_cta = (rows + nb - 1) / nb;
    sink_partial_kernel<<<(unsigned)nb, 256, 0, stream>>>(D, lse, sink, rows, HQ, per_cta,
                                                           scratch);
    sink_final_kernel<<<(HQ * 32 + 255) / 256, 256, 0, stream>>>(scratch, (int)nb, HQ, dsink);
  } else {
    sink_grad_kernel<<<HQ, 256, 0, stream>>>(D, lse, sink, rows, HQ, dsink);
  }
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

int attn_bwd_tc(const AttnProblem& pb, const BwdArgs& a, const TcFwdWs& ws, bool prepare, void* dq,
                void* dk, void* dv, void* dg, int* status, cudaStream_t stream) {
  if (pb.rows == 0 || ws.n_blocks128 == 0) return WALL_OK;
  int rc = WALL_OK;
  if (prepare) {  // else the forward's operands are reused
    timing_mark(T_OPERANDS, stream);
    rc = attn_prepare_operands(pb, a.q, a.k, a.P, ws, stream);
    timing_mark(T_OPERANDS, stream);
    if (rc) return rc;
  }
  timing_mark(T_BWD_PRE, stream);
  {
    const long threads = pb.rows * pb.HQ * 8;
    const int blocks = (int)((threads + 255) / 256);
    bwd_pre_kernel<<<blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(a.dO), static_cast<const __nv_bfloat16*>(a.o), a.lse,
        a.sink, pb.rows, pb.HQ, pb.V, a.D, a.GS ? a.dgs_row : nullptr);
    if (cudaGetLastError() != cudaSuccess) return WALL_ERR_CUDA;
    // the partials go through dq32, which the dq kernels overwrite later
    if (a.dsink && a.sink) {
      rc = sink_grad(a.D, a.lse, a.sink, pb.rows, pb.HQ, a.dq32, a.dsink, stream);
      if (rc) return rc;
    }
  }
  timing_mark(T_BWD_PRE, stream);
  timing_mark(T_BWD_KEY, stream);
  rc = pb.K == 128 ? launch_bwd_tc_gs<128>(pb, a, ws, status, stream)
                   : launch_bwd_tc_gs<64>(pb, a, ws, status, stream);
  timing_mark(T_BWD_KEY, stream);
  if (rc) return rc;
  timing_mark(T_BWD_DQ, stream);
  rc = attn_bwd_dq_tc(pb, a, ws, status, stream);
  timing_mark(T_BWD_DQ, stream);
  if (rc) return rc;
  // the units beyond the anchored range, again on CUDA cores: dk^(h),
  // dv^(h), their column sums and the final dq, over what the tensor-core
  // kernels wrote for them (one launch that only reads the flags when none
  // is set)
  timing_mark(T_EXACT, stream);
  rc = attn_bwd_simt_units(pb, a, ws.units, stream);
  timing_mark(T_EXACT, stream);
  if (rc) return rc;
  // dk, dv group sums and the scalar-gate parts; they run before dL
  // overwrites dk^(h)'s chunk rows with its sums
  timing_mark(T_BWD_FIN, stream);
  {
    // a row's groups per CTA (a multiple of 32 threads, at most 256)
    const int per_row = pb.H * (pb.K / 8 + pb.V / 8);
    const int threads = std::min(256, (per_row + 31) / 32 * 32);
    dim3 grid((148 * 16 + pb.seqs.n - 1) / (pb.seqs.n < 1 ? 1 : pb.seqs.n), pb.seqs.n);
    bwd_finalize_kernel<__nv_bfloat16><<<grid, threads, 0, stream>>>(
        pb.seqs, pb.HQ, pb.H, pb.K, pb.V, a.dkh32, a.dvh32, a.GS ? a.dgs_row : nullptr,
        a.GS ? a.dgs_col : nullptr, static_cast<__nv_bfloat16*>(dk),
        static_cast<__nv_bfloat16*>(dv));
    if (cudaGetLastError() != cudaSuccess) return WALL_ERR_CUDA;
  }
  timing_mark(T_BWD_FIN, stream);
  // dq, dL and dL's chunk sums in one pass, then the reverse scan's
  // carries and chunk scans give dg
  timing_mark(T_BWD_FIN, stream);
  rc = finalize_dq_dl_sums(static_cast<const __nv_bfloat16*>(a.q),
                           static_cast<const __nv_bfloat16*>(a.k), a.P, a.dq32, a.dkh32,
                           static_cast<__nv_bfloat16*>(dq), pb.HQ, pb.H, pb.K, pb.scale,
                           pb.seqs, ws.units, stream);
  timing_mark(T_BWD_FIN, stream);
  if (rc) return rc;
  timing_mark(T_REV_SCAN, stream);
  rc = scan_reverse_from_sums(a.dq32, dg, WALL_BF16, a.dkh32, (long)pb.HQ * pb.K, pb.seqs,
                              stream);
  timing_mark(T_REV_SCAN, stream);
  return rc;
}

}  // namespace wall
