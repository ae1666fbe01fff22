// wall_attn_fwd_sm100.cu -- tensor-core (tcgen05 + TMEM + TMA) Wall
// Attention forward for bf16 with K == V in {64, 128}.
//
// Math (Tilde blog "Wall Attention": definition and factorised form; fast
// training section 1, per-block anchor):
//   s_ij = scale * sum_n q_in k_jn 2^(P_in - P_jn)
// Rows are cut into 128-row blocks per sequence; block I has anchor
// R_I = floor(P at its first row), per channel.  Integer anchors make every
// per-tile factor 2^(R_I - R_J) an exact power of two, so scaling a bf16
// operand by it is exact.  A preparation kernel writes
//   Qh_i = q_i * 2^(P_i - R_I)   (i in block I)      bounded by one block
//   Kh_j = k_j * 2^(R_J - P_j)   (j in block J)      bounded by one block
// so that s_ij = scale * sum_n Qh_in * (Kh_jn * 2^(R_I,n - R_J,n)).  Inside
// the kernel the per-tile, per-channel factor d = 2^(R_I - R_J) is applied to
// the key tile in shared memory (packed bf16 multiplies, exact), then
//   S = Qh * Kt^T   and   O += P * V   run on tcgen05 with fp32 accumulators
// in TMEM, and the online softmax (log2 domain) keeps one query row per
// thread.  For decaying gates d only shrinks towards zero for distant tiles,
// where the exact contribution is equally negligible; no exponent of a
// global prefix ever reaches bf16 (the blog's reason for the anchors).
//
// The key tiles of a query block are split between two softmax groups, even
// and odd tiles, each with its own running max, sum and O accumulator, so
// two tiles are in the softmax at once; the two partial results are merged
// once at the end, as a split-KV decode merges its splits.
//
// CTA = one 128-row query block of one (sequence, head), 12 warps (3 per SM
// sub-partition, 168 registers each):
//   warp 0      TMA producer, lane 0: Qh once and the key ring (3 stages,
//               released after S); lane 1: the value ring (2 stages,
//               released after PV)
//   warp 1      TMEM owner and MMA issuer (one thread)
//   warps 2-3   key rescale: Kt_J = Kh_J (.) d in place; each thread keeps one
//               16-byte channel chunk, so its 8 factors stay in registers
//   warps 4-7   softmax of the even tiles, warps 8-11 of the odd tiles: S from
//               TMEM, mask, exp2, P (bf16 pairs) written back over the consumed
//               S columns as the TMEM A operand of PV, lazy O rescale in TMEM
//               when the row max grows by more than 2^8; epilogue merges the
//               two groups, o = O / l, lse.
// TMEM columns: S0 [0,128), S1 [128,256), O_even [256, 256+V),
// O_odd [256+V, 256+2V).
#include <cuda.h>

#include "sm100_ptx.cuh"
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kThreads = 384;
constexpr int kKS = 3;                    // key stages
constexpr int kVS = 2;                    // value stages
constexpr float kRescaleThreshold = 8.f;  // log2 units: lazy O rescale
constexpr float kRescaleBound = 256.f;    // 2^kRescaleThreshold

struct FwdTcParams {
  const float* anchors;  // [nblk, HQ, K]
  const float* GS;       // [rows, HQ] or nullptr
  const float* sink;     // [HQ] or nullptr
  __nv_bfloat16* o;      // [rows, HQ, V]
  float* lse;            // [rows, HQ] or nullptr
  Seqs seqs;
  int HQ, H, K, V;
  float scale_log2;      // scale * log2(e)
  int window;
  int n_blocks;          // grid bound on 128-row blocks
  int* status;
  // a chunk of queries against the decode cache (kCache kernels only): keys
  // are k_tilde rows, whose factor against the query block is
  // 2^(R_I - R_c) with R_c the anchor of the key's cache chunk
  const float* rc;       // r_cache [B, NC, HQ, K]
  int C, NC;             // cache chunk size, r_cache chunks per batch row
  int t_off;             // cache position of query row 0 (T_kv - Tq)
  int T_kv;              // cached positions per batch row
};

template <int KD, bool kCache>
struct Smem {
  // anchor rows per key stage: a cache tile spans up to 128 / 32 chunks
  static constexpr int kRJRows = kCache ? 4 : 1;
  static constexpr int kT = BN * KD * 2;          // one 128-row bf16 tile
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + kT;              // kKS stages
  static constexpr int oV = oK + kKS * kT;        // kVS stages
  static constexpr int oRJ = oV + kVS * kT;        // float[kKS][kRJRows][KD] key anchors
  static constexpr int oGS = oRJ + kKS * kRJRows * KD * 4;  // float[8 warps][BN] key prefix
  static constexpr int oX = oGS + 8 * BN * 4;     // float[2 groups][2][BM]: m, l
  static constexpr int oBar = oX + 2 * 2 * BM * 4;
  static constexpr int kBars = 22;
  static constexpr int oMisc = oBar + kBars * 8;  // tmem base, abort flag
  static constexpr int kBytes = oMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;    // slack for 1 KB alignment
};

// barrier slots, laid out from the stage counts (so a change of kKS or kVS
// cannot make two barriers share a slot)
enum Bar {
  B_QFULL = 0,
  B_KFULL = 1,                  // + key stage
  B_KREADY = B_KFULL + kKS,     // + key stage, 2 rescale warps
  B_KEMPTY = B_KREADY + kKS,    // + key stage
  B_VFULL = B_KEMPTY + kKS,     // + value stage
  B_VEMPTY = B_VFULL + kVS,     // + value stage
  B_SFULL = B_VEMPTY + kVS,     // + S buffer (2)
  B_PFULL = B_SFULL + 2,        // + group (2), 4 warps each
  B_PVDONE = B_PFULL + 2,       // + group (2): O_group holds every PV issued so far
  B_XCHG = B_PVDONE + 2,        // epilogue exchange of m, l between the groups (8 warps)
  B_MMADONE = B_XCHG + 1,
  kNumBars = B_MMADONE + 1,
};
static_assert(kNumBars <= Smem<128, false>::kBars, "barrier slots");

// bounded wait that also gives up once another role has given up
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
// the normal range, 0 below it (a factor under 2^-126 scales a key that
// decays to nothing) and +inf above it, as the fp32 product would overflow.
__device__ __forceinline__ uint32_t pow2_bf16(float k) {
  const int e = (int)k;
  return e < -126 ? 0u : e > 127 ? 0x7F80u : uint32_t(e + 127) << 7;
}

// Cache position of the first key tile's chunk and the number of the tile's
// chunks that hold cached positions (kCache kernels).
__device__ __forceinline__ int cache_tile_chunks(const FwdTcParams& p, int j0, int& c0) {
  c0 = j0 / p.C;
  const int nc = p.C >= BN ? 1 : BN / p.C;
  return min(nc, (p.T_kv + p.C - 1) / p.C - c0);
}

// kGS: the problem has a scalar gate (never in the cache form)
template <int KD, bool kCache, bool kGS>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, FwdTcParams p) {
  using Lay = Smem<KD, kCache>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* sGS = reinterpret_cast<float*>(smem + Lay::oGS);
  float* sX = reinterpret_cast<float*>(smem + Lay::oX);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::oBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::oMisc + 4);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.x;
  const int HQ = p.HQ, K = KD, V = KD;
  const int kh = h / (HQ / p.H);
  // longest query blocks first (they have the most key tiles)
  const int flat = p.n_blocks - 1 - (int)blockIdx.y;
  int seq, blk;
  if (!seq_block(p.seqs, BM, flat, seq, blk)) return;
  const int blk_off = flat - blk;
  const long s0 = p.seqs.start(seq);
  const int Lq = p.seqs.len(seq);            // query rows of this sequence
  // keys: the same rows, or the cache's positions; query row i sits at
  // position i, or t_off + i in the cache
  const int L = kCache ? p.T_kv : Lq;
  const int pos0 = kCache ? p.t_off : 0;
  const int i0 = blk * BM;
  const int ni = min(BM, Lq - i0);
  const int jb_hi = (pos0 + i0 + ni - 1) / BN;
  const int jb_lo = p.window > 0 ? max(0, i0 - p.window + 1) / BN : 0;
  const int nT = jb_hi - jb_lo + 1;
  // Key tile t is block jb_lo + t, or with a scalar gate jb_hi - t: the
  // diagonal first, then back in time.  The gate's bias GS_i - GS_j falls
  // by the gate's whole sum over the distance (tens of units of log2 across
  // a 1024-key window), so in ascending order every tile would raise the
  // rows' running max past the one-pass softmax's bound; from the diagonal
  // back, the first tiles set the max and the later ones stay under it.
  constexpr bool rev = kGS;
  auto jb_of = [&](int t) { return rev ? jb_hi - t : jb_lo + t; };

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int s = 0; s < kKS; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KREADY + s), 2);
      mbar_init(bar(B_KEMPTY + s), 1);
    }
    for (int s = 0; s < kVS; ++s) {
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar(B_SFULL + g), 1);
      mbar_init(bar(B_PFULL + g), 4);
      mbar_init(bar(B_PVDONE + g), 1);
    }
    mbar_init(bar(B_XCHG), 8);
    mbar_init(bar(B_MMADONE), 1);
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
    // lane 0: Qh and the key ring; lane 1: the value ring.  The two lanes
    // wait on different barriers and progress independently.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      mbar_expect_tx(bar(B_QFULL), Lay::kT);
      for (int b = 0; b < K / 64; ++b)
        tma_load_3d(sbase + Lay::oQ + b * (BM * 128), &tm_q, bar(B_QFULL), b * 64, h,
                    (int)(s0 + i0));
      int issued = 0;
      for (int t = 0; t < nT; ++t) {
        const int st = t % kKS;
        if (t >= kKS && !wait_bar(bar(B_KEMPTY + st), (t / kKS - 1) & 1, p.status, abort_flag))
          break;
        const uint32_t rj_dst = sbase + Lay::oRJ + st * Lay::kRJRows * K * 4;
        if constexpr (kCache) {
          // k_tilde rows of batch row `seq` (zeros past T_kv) and the
          // anchors of the tile's cached chunks
          const int j0 = jb_of(t) * BN;
          int c0;
          const int nc = cache_tile_chunks(p, j0, c0);
          mbar_expect_tx(bar(B_KFULL + st), Lay::kT + nc * K * 4);
          for (int b = 0; b < K / 64; ++b)
            tma_load_4d(sbase + Lay::oK + st * Lay::kT + b * (BN * 128), &tm_k,
                        bar(B_KFULL + st), b * 64, h, j0, seq);
          for (int x = 0; x < nc; ++x)
            bulk_load(rj_dst + x * K * 4, p.rc + (((long)seq * p.NC + c0 + x) * HQ + h) * K,
                      K * 4, bar(B_KFULL + st));
        } else {
          mbar_expect_tx(bar(B_KFULL + st), Lay::kT + K * 4);
          const int row = (int)(s0 + (long)jb_of(t) * BN);
          for (int b = 0; b < K / 64; ++b)
            tma_load_3d(sbase + Lay::oK + st * Lay::kT + b * (BN * 128), &tm_k,
                        bar(B_KFULL + st), b * 64, h, row);
          bulk_load(rj_dst, p.anchors + ((long)(blk_off + jb_of(t)) * HQ + h) * K, K * 4,
                    bar(B_KFULL + st));
        }
        issued = t + 1;
      }
      // no bulk copy may still be landing in this CTA's shared memory at exit
      for (int t = max(0, issued - kKS); t < issued; ++t)
        mbar_wait(bar(B_KFULL + t % kKS), (t / kKS) & 1, p.status);
      mbar_wait(bar(B_QFULL), 0, p.status);
    } else if (lane == 1) {
      tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (int t = 0; t < nT; ++t) {
        const int st = t % kVS;
        if (t >= kVS && !wait_bar(bar(B_VEMPTY + st), (t / kVS - 1) & 1, p.status, abort_flag))
          break;
        mbar_expect_tx(bar(B_VFULL + st), Lay::kT);
        if constexpr (kCache) {
          for (int b = 0; b < V / 64; ++b)
            tma_load_4d(sbase + Lay::oV + st * Lay::kT + b * (BN * 128), &tm_v,
                        bar(B_VFULL + st), b * 64, kh, jb_of(t) * BN, seq);
        } else {
          const int row = (int)(s0 + (long)jb_of(t) * BN);
          for (int b = 0; b < V / 64; ++b)
            tma_load_3d(sbase + Lay::oV + st * Lay::kT + b * (BN * 128), &tm_v,
                        bar(B_VFULL + st), b * 64, kh, row);
        }
        issued = t + 1;
      }
      for (int t = max(0, issued - kVS); t < issued; ++t)
        mbar_wait(bar(B_VFULL + t % kVS), (t / kVS) & 1, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16(BM, BN, false, false);
      const uint32_t idesc_pv = idesc_bf16(BM, V, false, true);
      bool ok = wait_bar(bar(B_QFULL), 0, p.status, abort_flag);
      // S(t) into buffer t & 1; it is free once PV(t - 2) has read P(t - 2)
      auto issue_qk = [&](int t) -> bool {
        const int st = t % kKS;
        if (!wait_bar(bar(B_KREADY + st), (t / kKS) & 1, p.status, abort_flag)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (t & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < KD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          const uint64_t a = sdesc_sw128(sbase + Lay::oQ + off, 16, 1024);
          const uint64_t b = sdesc_sw128(sbase + Lay::oK + st * Lay::kT + off, 16, 1024);
          umma_bf16_ss(d_tmem, a, b, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(B_SFULL + (t & 1)));
        umma_commit(bar(B_KEMPTY + st));
        return true;
      };
      if (ok) ok = issue_qk(0);
      if (ok && nT > 1) ok = issue_qk(1);
      for (int t = 0; ok && t < nT; ++t) {
        const int g = t & 1;  // softmax group and S / O buffers of this tile
        const int vs = t % kVS;
        if (!wait_bar(bar(B_VFULL + vs), (t / kVS) & 1, p.status, abort_flag)) break;
        if (!wait_bar(bar(B_PFULL + g), (t >> 1) & 1, p.status, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // A = P [128 rows x 16 keys] from TMEM: the softmax wrote bf16 pairs
          // over the S buffer it had consumed, 8 columns per 16 keys
          const uint32_t a = tmem + g * 128 + kk * 8;
          // B = V [16 keys x V channels], MN-major: 8-key groups 1 KB apart,
          // 64-channel boxes BN*128 bytes apart
          const uint64_t b =
              sdesc_sw128(sbase + Lay::oV + vs * Lay::kT + kk * 16 * 128, BN * 128, 1024);
          umma_bf16_ts(tmem + 256 + g * V, a, b, idesc_pv, (t >= 2 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(B_PVDONE + g));
        umma_commit(bar(B_VEMPTY + vs));
        if (t + 2 < nT) ok = issue_qk(t + 2);
      }
      // every MMA of this CTA has completed before TMEM is released
      umma_commit(bar(B_MMADONE));
      mbar_wait(bar(B_MMADONE), 0, p.status);
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
        const bool got = wait_bar(bar(B_KFULL + st), (t / kKS) & 1, p.status, abort_flag);
        if (!__all_sync(0xffffffffu, got)) break;
      }
      const float* rj =
          reinterpret_cast<const float*>(smem + Lay::oRJ + st * Lay::kRJRows * K * 4) + ch * 8;
      uint8_t* kt = smem + Lay::oK + st * Lay::kT + (ch / 8) * (BN * 128);
      if constexpr (kCache) {
        // factor 2^(R_I - R_c) per cache chunk of the tile: not a power of
        // two, so it is rounded to bf16 and applied with packed bf16
        // multiplies (two roundings of 2^-9 on the key, as fine as the
        // k_tilde rounding itself); rows of a chunk that holds no cached
        // position are zeros and get factor 0
        int c0;
        const int nvalid = cache_tile_chunks(p, jb_of(t) * BN, c0);
        const int crows = p.C >= BN ? BN : p.C;  // tile rows per chunk
        for (int x = 0; x * crows < BN; ++x) {
          __nv_bfloat162 f[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            f[e] = x < nvalid ? __floats2bfloat162_rn(exp2f(ri[2 * e] - rj[x * K + 2 * e]),
                                                      exp2f(ri[2 * e + 1] - rj[x * K + 2 * e + 1]))
                              : __floats2bfloat162_rn(0.f, 0.f);
          constexpr int kBatch = 4;
          for (int m0 = x * crows / kRowStep; m0 < (x + 1) * crows / kRowStep; m0 += kBatch) {
            uint4 v[kBatch];
#pragma unroll
            for (int y = 0; y < kBatch; ++y) {
              const int r = rs + (m0 + y) * kRowStep;
              v[y] = *reinterpret_cast<const uint4*>(kt + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
            }
#pragma unroll
            for (int y = 0; y < kBatch; ++y) {
              const int r = rs + (m0 + y) * kRowStep;
              __nv_bfloat162* w = reinterpret_cast<__nv_bfloat162*>(&v[y]);
#pragma unroll
              for (int e = 0; e < 4; ++e) w[e] = __hmul2(w[e], f[e]);
              *reinterpret_cast<uint4*>(kt + r * 128 + (((ch & 7) ^ (r & 7)) << 4)) = v[y];
            }
          }
        }
      } else {
        __nv_bfloat162 d[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t b = pow2_bf16(ri[2 * e] - rj[2 * e]) |
                             (pow2_bf16(ri[2 * e + 1] - rj[2 * e + 1]) << 16);
          d[e] = *reinterpret_cast<const __nv_bfloat162*>(&b);
        }
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
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_KREADY + st));
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int grp = (warp - 4) >> 2;          // 0: even key tiles, 1: odd ones
    const int quarter = warp & 3;             // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;        // query row within the block
    const int qi = i0 + r;                    // query row within the sequence
    const int i = pos0 + qi;                  // its position among the keys
    const bool row_ok = r < ni;
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    constexpr bool has_gs = kGS;
    const int win = p.window > 0 ? p.window : 0x7fffffff;
    const float gs_i = (has_gs && row_ok) ? p.GS[(s0 + qi) * HQ + h] * kLog2e : 0.f;
    const uint32_t s_addr = tmem + lane_base + grp * 128;
    const uint32_t o_addr = tmem + lane_base + 256 + grp * V;
    float* gsk = sGS + (warp - 4) * BN;  // this warp's copy of the key prefix (or zeros)
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    // a chunk of fewer than 128 queries leaves whole warps without a row:
    // they only keep step with their group (S ready, P "written")
    const bool idle = kCache && !__any_sync(0xffffffffu, row_ok);
    // the scalar gate's key prefix of the group's next tile, one load per
    // lane and key quarter, issued a tile ahead so that its L2 latency
    // overlaps the current tile instead of preceding the wait for S
    float gnext[kGS ? BN / 32 : 1];
    auto load_gs = [&](int t) {
#pragma unroll
      for (int x = 0; x < BN / 32; ++x) {
        const int j = jb_of(t) * BN + lane + 32 * x;
        gnext[x] = (t < nT && j < L) ? p.GS[(s0 + j) * HQ + h] * kLog2e : 0.f;
      }
    };
    if constexpr (has_gs) load_gs(grp);
    for (int t = grp; t < nT; t += 2) {
      const int j0 = jb_of(t) * BN;
      if (idle) {
        const bool got = wait_bar(bar(B_SFULL + grp), (t >> 1) & 1, p.status, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PFULL + grp));
        continue;
      }
      if constexpr (has_gs) {
        __syncwarp();
#pragma unroll
        for (int x = 0; x < BN / 32; ++x) gsk[lane + 32 * x] = gnext[x];
        __syncwarp();
        load_gs(t + 2);
      } else if (t == grp) {
        __syncwarp();
        for (int c = lane; c < BN; c += 32) gsk[c] = 0.f;
        __syncwarp();
      }
      {
        const bool got = wait_bar(bar(B_SFULL + grp), (t >> 1) & 1, p.status, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      }
      tc_fence_after();
      // logits (log2 domain) with the causal / window / sequence mask.  The
      // common case -- a fully visible tile -- is a multiply (plus, with a
      // scalar gate, the bias GS_i - GS_j, from this warp's copy of the key
      // prefix); the decision is warp-uniform and hoisted out of the element
      // loops.
      // (rows past a cache chunk's queries compute on finite stand-in
      // queries and are never stored, so they do not hold the warp back)
      const bool fast =
          __all_sync(0xffffffffu, (kCache && !row_ok) ||
                                      (row_ok && (j0 + BN - 1 <= i) && (j0 + BN <= L) &&
                                       (i - j0 < win)));
      const float sl2 = p.scale_log2;
      const float bias_i = has_gs ? gs_i : 0.f;
      bool done = false;
      // One pass when every row's running max is set: exponentials against
      // it, P held packed in registers and stored only if no row's sum
      // exceeds 2^threshold (then no term does, so no row's max grew past
      // the lazy threshold; an overflow or NaN fails the test too);
      // otherwise S, still intact in TMEM, goes through the two passes below
      // (max, O rescale, exponentials).  The row max itself is not formed
      // here: issue slots, not the exponential unit, bound this loop.
      if (fast && __all_sync(0xffffffffu, m_use != -INFINITY)) {
        uint32_t pk1[64];
        float r0 = 0.f, r1 = 0.f;
        const float off = kGS ? bias_i - m_use : -m_use;
#pragma unroll
        for (int c = 0; c < BN; c += 64) {
          uint32_t sv[64];
          tmem_ld32(s_addr + c, sv);
          tmem_ld32(s_addr + c + 32, sv + 32);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 64; e += 4) {
            // with a scalar gate the key prefix, four keys per shared-memory
            // load (a broadcast); without one, a single FMA per logit
            float4 gk = make_float4(0.f, 0.f, 0.f, 0.f);
            if constexpr (kGS) gk = *reinterpret_cast<const float4*>(gsk + c + e);
            const float p0 = exp2f(fmaf(__uint_as_float(sv[e]), sl2, off - gk.x));
            const float p1 = exp2f(fmaf(__uint_as_float(sv[e + 1]), sl2, off - gk.y));
            const float p2 = exp2f(fmaf(__uint_as_float(sv[e + 2]), sl2, off - gk.z));
            const float p3 = exp2f(fmaf(__uint_as_float(sv[e + 3]), sl2, off - gk.w));
            r0 += p0 + p2;
            r1 += p1 + p3;
            pk1[(c + e) / 2] = pack_bf16x2(p0, p1);
            pk1[(c + e) / 2 + 1] = pack_bf16x2(p2, p3);
          }
        }
        if (!__any_sync(0xffffffffu, !(r0 + r1 <= kRescaleBound))) {
          // keys [32c, 32c+32) -> columns [16c, 16c+16): all of S was read
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_st16(s_addr + c * 16, pk1 + c * 16);
          tmem_wait_st();
          l += r0 + r1;
          done = true;
        }
      }
      if (!done) {
        // pass 1: row max
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < BN; c += 64) {
          uint32_t sv[64];
          tmem_ld32(s_addr + c, sv);
          tmem_ld32(s_addr + c + 32, sv + 32);
          tmem_wait_ld();
          if (fast && !has_gs) {
#pragma unroll
            for (int e = 0; e < 64; e += 4) {
              mx0 = fmaxf(mx0, __uint_as_float(sv[e]) * sl2);
              mx1 = fmaxf(mx1, __uint_as_float(sv[e + 1]) * sl2);
              mx2 = fmaxf(mx2, __uint_as_float(sv[e + 2]) * sl2);
              mx3 = fmaxf(mx3, __uint_as_float(sv[e + 3]) * sl2);
            }
          } else {  // masked, or with the scalar gate's bias
#pragma unroll
            for (int e = 0; e < 64; ++e) {
              const int j = j0 + c + e;
              const bool vis = row_ok & (j < L) & (j <= i) & (i - j < win);
              const float x = fmaf(__uint_as_float(sv[e]), sl2, bias_i - gsk[c + e]);
              mx0 = fmaxf(mx0, vis ? x : -INFINITY);
            }
          }
        }
        const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        const bool resc = mx > m_use + kRescaleThreshold;
        const float m_new = resc ? mx : m_use;
        const float alpha = (m_use == -INFINITY) ? 0.f : exp2f(m_use - m_new);
        if (t >= 2) {
          // this group's previous PV has landed in its O before O is rescaled
          const bool got = wait_bar(bar(B_PVDONE + grp), ((t >> 1) - 1) & 1, p.status, abort_flag);
          if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(0xffffffffu, resc)) {
            const float f = resc ? alpha : 1.f;
#pragma unroll 1
            for (int c = 0; c < V / 32; ++c) {
              uint32_t ov[32];
              tmem_ld32(o_addr + c * 32, ov);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
              tmem_st32(o_addr + c * 32, ov);
            }
            tmem_wait_st();
          }
        }
        if (resc) l *= alpha;
        m_use = m_new;
        const float m_eff = (m_use == -INFINITY) ? 0.f : m_use;
        // pass 2: p = exp2(s - m), row sum, bf16 P over the consumed S columns
        float rs0 = 0.f, rs1 = 0.f;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t sv[32];
          tmem_ld32(s_addr + c, sv);
          tmem_wait_ld();
          float e32[32];
          if (fast && !has_gs) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              e32[e] = exp2f(fmaf(__uint_as_float(sv[e]), sl2, -m_eff));
            }
          } else {  // masked, or with the scalar gate's bias
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int j = j0 + c + e;
              const bool vis = row_ok & (j < L) & (j <= i) & (i - j < win);
              const float x = fmaf(__uint_as_float(sv[e]), sl2, bias_i - gsk[c + e] - m_eff);
              e32[e] = vis ? exp2f(x) : 0.f;
            }
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            rs0 += e32[e];
            rs1 += e32[e + 1];
            pk[e / 2] = pack_bf16x2(e32[e], e32[e + 1]);
          }
          // keys [c, c+32) -> columns [c/2, c/2+16) of this S buffer; every S
          // column at or below them has been read already
          tmem_st16(s_addr + c / 2, pk);
        }
        tmem_wait_st();
        l += rs0 + rs1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_PFULL + grp));
    }
    // ---- epilogue: merge the two groups' (m, l, O), as split-KV partials
    const int n0 = (nT + 1) / 2, n1 = nT / 2;  // tiles per group
    const int nmine = grp == 0 ? n0 : n1;
    if (ok && nmine > 0)
      ok = __all_sync(0xffffffffu,
                      wait_bar(bar(B_PVDONE + grp), (nmine - 1) & 1, p.status, abort_flag));
    sX[(grp * 2) * BM + r] = m_use;
    sX[(grp * 2 + 1) * BM + r] = l;
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(B_XCHG));  // every warp arrives, even after an abort
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(bar(B_XCHG), 0, p.status, abort_flag));
    if (ok) {
      tc_fence_after();
      const float m0 = sX[0 * BM + r], l0 = sX[1 * BM + r];
      const float m1 = sX[2 * BM + r], l1 = sX[3 * BM + r];
      float m_f = fmaxf(m0, m1);
      if (p.sink) m_f = fmaxf(m_f, p.sink[h] * kLog2e);
      const float a0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - m_f);
      const float a1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - m_f);
      float lt = l0 * a0 + l1 * a1;
      if (p.sink) lt += exp2f(p.sink[h] * kLog2e - m_f);
      const float inv = 1.f / lt;
      const float f0 = a0 * inv, f1 = a1 * inv;
      __nv_bfloat16* orow = p.o + ((s0 + qi) * HQ + h) * (long)V;
      // each group writes half of the channels; O_odd exists only if the odd
      // group had tiles (warp-uniform)
#pragma unroll 1
      for (int c = grp * (V / 2); c < (grp + 1) * (V / 2); c += 32) {
        uint32_t ov0[32], ov1[32];
        tmem_ld32(tmem + lane_base + 256 + c, ov0);
        if (n1 > 0) tmem_ld32(tmem + lane_base + 256 + V + c, ov1);
        tmem_wait_ld();
        if (row_ok) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0 = __uint_as_float(ov0[2 * e]) * f0;
            float x1 = __uint_as_float(ov0[2 * e + 1]) * f0;
            if (n1 > 0) {
              x0 = fmaf(__uint_as_float(ov1[2 * e]), f1, x0);
              x1 = fmaf(__uint_as_float(ov1[2 * e + 1]), f1, x1);
            }
            pk[e] = pack_bf16x2(x0, x1);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      if (grp == 0 && row_ok && p.lse) p.lse[(s0 + qi) * HQ + h] = (m_f + log2f(lt)) * kLn2;
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
// preparation: anchored operands Qh, Kh (per query head) and block anchors.
// An anchored exponent |P - R| beyond kAnchorRange (a channel whose gate
// sums past 2^kAnchorRange inside one block) flags its (sequence, head) unit
// in `units`, which the SIMT kernels then recompute, or records
// WALL_ERR_RANGE in `status` (the chunk call, which has no such fallback).

__global__ void anchor_operands_kernel(const __nv_bfloat16* __restrict__ q,
                                       const __nv_bfloat16* __restrict__ k,
                                       const float* __restrict__ P, Seqs seqs, int HQ, int H,
                                       int K, __nv_bfloat16* __restrict__ qh,
                                       __nv_bfloat16* __restrict__ khat,
                                       float* __restrict__ anchors, int* __restrict__ units,
                                       int* status) {
  const int s = blockIdx.y;
  __shared__ int s_blk_off;
  if (threadIdx.x == 0) {
    int off = 0;
    if (seqs.cu) {
      for (int x = 0; x < s; ++x) off += (seqs.len(x) + BM - 1) / BM;
    } else {
      off = s * ((seqs.T + BM - 1) / BM);
    }
    s_blk_off = off;
  }
  __syncthreads();
  const long s0 = seqs.start(s);
  const int L = seqs.len(s);
  const int G = HQ / H;
  const int kg = K / 8;
  const int per_row = HQ * kg;
  // CTAs take rows of the sequence, threads the row's (head, 8 channels)
  // groups: 32-bit arithmetic only
  for (int t = blockIdx.x; t < L; t += gridDim.x) {
    for (int i = threadIdx.x; i < per_row; i += blockDim.x) {
      const int hh = i / kg;
      const int g8 = i - hh * kg;
      const int b = t / BM;
      const long row = s0 + t;
      const long arow = s0 + (long)b * BM;
      float pv[8], rv[8], x[8], y[8];
      load8(P + (row * HQ + hh) * K + g8 * 8, pv);
      load8(P + (arow * HQ + hh) * K + g8 * 8, rv);
      bool wide = false;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        rv[c] = floorf(rv[c]);
        wide |= fabsf(pv[c] - rv[c]) > kAnchorRange;
      }
      if (wide) {
        if (units) {
          set_flag(units + (long)s * HQ + hh);
          set_flag(units + (long)seqs.n * HQ);  // some unit is flagged
        }
        record_status(status, WALL_ERR_RANGE);
      }
      load8(q + (row * HQ + hh) * K + g8 * 8, x);
#pragma unroll
      for (int c = 0; c < 8; ++c) y[c] = saturate_bf16(x[c] * exp2f(pv[c] - rv[c]));
      store8(qh + (row * HQ + hh) * K + g8 * 8, y);
      if (k != nullptr) {  // without keys: the query operand and anchors only
        load8(k + (row * H + hh / G) * K + g8 * 8, x);
#pragma unroll
        for (int c = 0; c < 8; ++c) y[c] = saturate_bf16(x[c] * exp2f(rv[c] - pv[c]));
        store8(khat + (row * HQ + hh) * K + g8 * 8, y);
      }
      if (t == b * BM) store8(anchors + ((long)(s_blk_off + b) * HQ + hh) * K + g8 * 8, rv);
    }
  }
}

// ---------------------------------------------------------------------------
// host: tensor maps and launch

template <int KD>
int launch_fwd_tc(const AttnProblem& pb, const FwdArgs& a, const TcFwdWs& ws, int* status,
                  cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tq, ws.qh, pb.rows, pb.HQ, KD, BM) ||
      !make_tile_map(&tk, ws.kh, pb.rows, pb.HQ, KD, BN) ||
      !make_tile_map(&tv, a.v, pb.rows, pb.H, KD, BN))
    return WALL_ERR_CUDA;
  static bool attr[2][kMaxDevices] = {};
  if (!set_max_smem_once(fwd_tc_kernel<KD, false, false>, Smem<KD, false>::kAlloc, attr[0]) ||
      !set_max_smem_once(fwd_tc_kernel<KD, false, true>, Smem<KD, false>::kAlloc, attr[1]))
    return WALL_ERR_CUDA;
  FwdTcParams p;
  p.anchors = ws.anchors;
  p.GS = a.GS;
  p.sink = a.sink;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.seqs = pb.seqs;
  p.HQ = pb.HQ; p.H = pb.H; p.K = pb.K; p.V = pb.V;
  p.scale_log2 = pb.scale * kLog2e;
  p.window = pb.window;
  p.n_blocks = ws.n_blocks128;
  p.status = status;
  p.rc = nullptr;
  p.C = p.NC = p.t_off = p.T_kv = 0;
  dim3 grid(pb.HQ, ws.n_blocks128);
  if (a.GS)
    fwd_tc_kernel<KD, false, true><<<grid, kThreads, Smem<KD, false>::kAlloc, stream>>>(tq, tk, tv,
                                                                                        p);
  else
    fwd_tc_kernel<KD, false, false><<<grid, kThreads, Smem<KD, false>::kAlloc, stream>>>(tq, tk, tv,
                                                                                         p);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

// A chunk of queries against the decode cache: Qh, the query-block anchors,
// then the forward kernel in its cache form (keys = k_tilde rows, values =
// the value cache, both read through maps that end at T_kv).
template <int KD>
int launch_decode_chunk_tc(const FwdTcParams& p0, const void* k_tilde, const void* v, int B,
                           int Tq, int T_kv, int Tcap, int H, int HQ, const __nv_bfloat16* qh,
                           cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tq, qh, (long)B * Tq, HQ, KD, BM) ||
      !make_cache_map(&tk, k_tilde, B, T_kv, Tcap, HQ, KD, BN) ||
      !make_cache_map(&tv, v, B, T_kv, Tcap, H, KD, BN))
    return WALL_ERR_CUDA;
  static bool attr[kMaxDevices] = {};
  if (!set_max_smem_once(fwd_tc_kernel<KD, true, false>, Smem<KD, true>::kAlloc, attr))
    return WALL_ERR_CUDA;
  dim3 grid(HQ, p0.n_blocks);
  fwd_tc_kernel<KD, true, false><<<grid, kThreads, Smem<KD, true>::kAlloc, stream>>>(tq, tk, tv,
                                                                                      p0);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

}  // namespace

bool fwd_tc_supported(const AttnProblem& pb) {
  return pb.dtype == WALL_BF16 && pb.K == pb.V && (pb.K == 64 || pb.K == 128);
}

int attn_prepare_operands(const AttnProblem& pb, const void* q, const void* k, const float* P,
                          const TcFwdWs& ws, cudaStream_t stream) {
  if (pb.rows == 0 || pb.seqs.n == 0) return WALL_OK;
  if (cudaMemsetAsync(ws.units, 0, sizeof(int) * ((size_t)pb.seqs.n * pb.HQ + 1), stream) !=
      cudaSuccess)
    return WALL_ERR_CUDA;
  // enough CTAs to keep every SM streaming, split over the sequences
  const int per_seq = (148 * 8 + pb.seqs.n - 1) / pb.seqs.n;
  dim3 grid(per_seq < 1 ? 1 : per_seq, pb.seqs.n);
  anchor_operands_kernel<<<grid, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), P, pb.seqs,
      pb.HQ, pb.H, pb.K, ws.qh, ws.kh, ws.anchors, ws.units, nullptr);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

bool decode_chunk_tc_supported(int dtype, int K, int V, int C) {
  return dtype == WALL_BF16 && K == V && (K == 64 || K == 128) && C >= 32 && C % 32 == 0 &&
         (BN % C == 0 || C % BN == 0);
}

int attn_decode_chunk_tc(const void* q, const void* v, const float* p, const void* k_tilde,
                         const float* r_cache, const float* sink, float scale, int C, int B,
                         int Tq, int T_kv, int Tcap, int H, int HQ, int K, __nv_bfloat16* qh,
                         float* anchors, void* o, float* lse, int* status, cudaStream_t stream) {
  if ((long)B * Tq == 0) return WALL_OK;
  Seqs seqs;
  seqs.cu = nullptr;
  seqs.n = B;
  seqs.T = Tq;
  seqs.rows = (long)B * Tq;
  // Qh = q * 2^(p - R_I) and the query-block anchors R_I = floor(p at the
  // block's first row), as the training forward prepares its queries
  const int per_seq = (148 * 8 + B - 1) / B;
  anchor_operands_kernel<<<dim3(per_seq < 1 ? 1 : per_seq, B), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(q), nullptr, p, seqs, HQ, H, K, qh, nullptr, anchors,
      nullptr, status);
  if (cudaGetLastError() != cudaSuccess) return WALL_ERR_CUDA;
  FwdTcParams pr;
  pr.anchors = anchors;
  pr.GS = nullptr;
  pr.sink = sink;
  pr.o = static_cast<__nv_bfloat16*>(o);
  pr.lse = lse;
  pr.seqs = seqs;
  pr.HQ = HQ; pr.H = H; pr.K = K; pr.V = K;
  pr.scale_log2 = scale * kLog2e;
  pr.window = 0;
  pr.n_blocks = B * ((Tq + BM - 1) / BM);
  pr.status = status;
  pr.rc = r_cache;
  pr.C = C;
  pr.NC = (Tcap + C - 1) / C;
  pr.t_off = T_kv - Tq;
  pr.T_kv = T_kv;
  return K == 128 ? launch_decode_chunk_tc<128>(pr, k_tilde, v, B, Tq, T_kv, Tcap, H, HQ, qh, stream)
                  : launch_decode_chunk_tc<64>(pr, k_tilde, v, B, Tq, T_kv, Tcap, H, HQ, qh, stream);
}

int attn_fwd_tc(const AttnProblem& pb, const FwdArgs& a, const TcFwdWs& ws, int* status,
                cudaStream_t stream, bool prepared) {
  if (pb.rows == 0 || ws.n_blocks128 == 0) return WALL_OK;
  int rc = WALL_OK;
  if (!prepared) {
    timing_mark(T_OPERANDS, stream);
    rc = attn_prepare_operands(pb, a.q, a.k, a.P, ws, stream);
    timing_mark(T_OPERANDS, stream);
    if (rc) return rc;
  }
  timing_mark(T_FWD, stream);
  rc = pb.K == 128 ? launch_fwd_tc<128>(pb, a, ws, status, stream)
                   : launch_fwd_tc<64>(pb, a, ws, status, stream);
  timing_mark(T_FWD, stream);
  if (rc) return rc;
  // the units the anchored operands cannot represent, again on CUDA cores
  // (a persistent grid that only reads the flags when none is set)
  timing_mark(T_EXACT, stream);
  rc = attn_fwd_simt_units(pb, a, ws.units, stream);
  timing_mark(T_EXACT, stream);
  return rc;
}

}  // namespace wall
