// wall_internal.h -- launchers behind the C ABI (host side, namespace wall).
#pragma once

#include <cuda.h>
#include <nvtx3/nvToolsExt.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "wall.h"
#include "wall_common.cuh"

namespace wall {

// ---- per-stage timing (wall_timing.cu): records an event on `stream` for
// `slot` while timing is enabled; calls come in begin / end pairs ----
void timing_mark(int slot, cudaStream_t stream);
enum TimingSlot {
  T_PREFIX = 0, T_OPERANDS = 1, T_FWD = 2, T_BWD_PRE = 3, T_BWD_KEY = 4, T_BWD_DQ = 5,
  T_BWD_FIN = 6, T_REV_SCAN = 7, T_DECODE = 8, T_CACHE = 9, T_STEP = 10, T_CHUNK = 11,
  T_EXACT = 12,
};

// ---- scans (wall_scan.cu) ----
int scan_prefix_log2(const void* g, int dtype, float* P, long C, const Seqs& seqs,
                     const float* carry_in, float* carry_out, cudaStream_t stream);
int scan_prefix_plain(const float* x, float* y, long C, const Seqs& seqs, cudaStream_t stream);
// the forward prefix fused with the tensor-core operand preparation: P (as
// scan_prefix_log2 forms it, bit for bit), Qh, Kh and the 128-row block
// anchors (as attn_prepare_operands forms them); scratch: fp32 [chunks, HQ*K]
// for the chunk carries (one row per 32-row chunk of every sequence), not P
int scan_prefix_operands(const __nv_bfloat16* g, const __nv_bfloat16* q, const __nv_bfloat16* k,
                         float* P, float* scratch, int HQ, int H, int K, const Seqs& seqs,
                         __nv_bfloat16* qh, __nv_bfloat16* kh, float* anchors, int* units,
                         cudaStream_t stream);
// the tensor-core backward's dq finalize fused with pass 1 of dL's reverse
// scan: dq (bf16), dL over dq32, chunk sums of dL into dkh32's chunk rows;
// dq32 of the units flagged in `units` already holds the final dq
int finalize_dq_dl_sums(const __nv_bfloat16* q, const __nv_bfloat16* k, const float* P,
                        float* dq32, float* dkh32, __nv_bfloat16* dq, int HQ, int H, int K,
                        float scale, const Seqs& seqs, const int* units, cudaStream_t stream);
// passes 2 and 3 of the reverse scan, the chunk sums already in scratch
int scan_reverse_from_sums(const float* x, void* y, int out_dtype, float* scratch, long C,
                           const Seqs& seqs, cudaStream_t stream);
int scan_reverse(const float* x, void* y, int out_dtype, float* scratch, long C,
                 const Seqs& seqs, cudaStream_t stream);

// ---- attention problem description shared by the fwd/bwd launchers ----
struct AttnProblem {
  int dtype;
  int B, T, H, HQ, K, V;
  float scale;
  int window;        // <= 0: none
  Seqs seqs;         // sequences over the B*T flattened rows
  long rows;         // B*T
  int max_blocks64;  // upper bound on 64-row blocks over all sequences
  int extra_blocks;  // varlen: sequences (each may add one partial block), else 0
  // SIMT kernels only: nullptr, or [n_seq, HQ] flags; then only the flagged
  // (sequence, head) units are computed
  const int* units;
};

struct FwdArgs {
  const void *q, *k, *v;
  const float* P;
  const float* GS;    // inclusive prefix of g_scalar [rows,HQ] or nullptr
  const float* sink;  // [HQ] or nullptr
  void* o;
  float* lse;
};

struct BwdArgs {
  const void *dO, *q, *k, *v, *o;
  const float* P;
  const float* lse;
  const float* GS;
  const float* sink;
  // fp32 workspace
  float* D;       // [rows,HQ]
  float* dq32;    // [rows,HQ,K]  (becomes dL after the reduce)
  float* dkh32;   // [rows,HQ,K]
  float* dvh32;   // [rows,HQ,V]
  float* dgs_row; // [rows,HQ]
  float* dgs_col; // [rows,HQ]
  float* dsink;   // [HQ] or nullptr (accumulated atomically, zeroed by the caller)
  // tensor-core path, dense causal without a window: the key-block kernel
  // stores its dS tiles here and dq is one contraction per tile; nullptr:
  // the dq kernel recomputes S, P, dP and dS
  __nv_bfloat16* dS;  // [B * HQ * nb(nb+1)/2, 128, 128], nb = ceil(T / 128)
};

// ---- tensor-core forward (wall_attn_fwd_sm100.cu) ----
struct TcFwdWs {
  __nv_bfloat16* qh;   // [rows, HQ, K]  q * 2^(P - R_block)
  __nv_bfloat16* kh;   // [rows, HQ, K]  k * 2^(R_block - P)
  float* anchors;      // [n_blocks128, HQ, K]  P at each 128-row block start
  int n_blocks128;     // upper bound on 128-row blocks over all sequences
  // [n_seq * HQ + 1]: nonzero for a (sequence, head) unit some of whose
  // anchored exponents |P - R_block| exceed kAnchorRange, and in the last
  // word if any unit is; the operand pass sets them, the SIMT kernels
  // recompute those units
  int* units;
};
// Anchored exponents of the tensor-core operands stay within +-kAnchorRange:
// Qh, Kh and every per-tile rescaled key then stay normal bf16 numbers for
// inputs up to 2^20 in magnitude, and the products the MMAs form are exact
// to bf16 rounding.
constexpr float kAnchorRange = 100.f;
bool fwd_tc_supported(const AttnProblem& pb);
int attn_prepare_operands(const AttnProblem& pb, const void* q, const void* k, const float* P,
                          const TcFwdWs& ws, cudaStream_t stream);
// prepared: ws already holds Qh, Kh and the anchors (the fused prefix pass)
int attn_fwd_tc(const AttnProblem& pb, const FwdArgs& a, const TcFwdWs& ws, int* status,
                cudaStream_t stream, bool prepared = false);

// ---- tensor-core backward (wall_attn_bwd_sm100.cu) ----
// prepare: false when ws already holds the forward's anchored operands
// also writes dg (the reverse scan of dL) on this path
int attn_bwd_tc(const AttnProblem& pb, const BwdArgs& a, const TcFwdWs& ws, bool prepare,
                void* dq, void* dk, void* dv, void* dg, int* status, cudaStream_t stream);
// raw dq (without the per-row anchor factor) into a.dq32 (wall_attn_bwd_dq_sm100.cu)
int attn_bwd_dq_tc(const AttnProblem& pb, const BwdArgs& a, const TcFwdWs& ws, int* status,
                   cudaStream_t stream);

// ---- TMA tensor maps (wall_tma.cu) ----
bool make_tile_map(CUtensorMap* m, const void* base, long rows, int heads, int dim,
                   int box_rows);

bool make_rows128_map(CUtensorMap* m, const void* base, long rows, int box_rows, int box_cols);
bool make_cache_map(CUtensorMap* m, const void* base, int B, int T, int Tcap, int heads, int dim,
                    int box_rows);

// ---- a chunk of Tq queries against the decode cache (multi-token decode,
// chunked prefill); query row i of batch row b sits at cache position
// T_kv - Tq + i ----
// tensor-core path (wall_attn_fwd_sm100.cu): bf16, K == V in {64, 128},
// C a multiple of 32 that divides 128 or is a multiple of 128
bool decode_chunk_tc_supported(int dtype, int K, int V, int C);
int attn_decode_chunk_tc(const void* q, const void* v, const float* p, const void* k_tilde,
                         const float* r_cache, const float* sink, float scale, int C, int B,
                         int Tq, int T_kv, int Tcap, int H, int HQ, int K, __nv_bfloat16* qh,
                         float* anchors, void* o, float* lse, int* status, cudaStream_t stream);
// general path (wall_decode.cu): the split decode with one grid row per query
int decode_chunk_splits(int B, int Tq, int T_kv, int H, int C);
int attn_decode_chunk_split(const void* q, const void* v, const float* p, const void* k_tilde,
                            const float* r_cache, const float* sink, float scale, int C,
                            int dtype, int B, int Tq, int T_kv, int Tcap, int H, int HQ, int K,
                            int V, void* o, float* lse, float* ws, int splits,
                            cudaStream_t stream);

// dsink_h = -sum_i exp(sink_h - lse_i) D_i in a fixed order (bit-reproducible),
// from D and lse [rows, HQ]; scratch holds min(ceil(rows / 64), 592) * HQ
// floats until the launches complete (wall_attn_bwd_sm100.cu)
int sink_grad(const float* D, const float* lse, const float* sink, long rows, int HQ,
              float* scratch, float* dsink, cudaStream_t stream);

// ---- SIMT fp32 attention (wall_attn_simt.cu) ----
int attn_fwd_simt(const AttnProblem& pb, const FwdArgs& a, cudaStream_t stream);
int attn_bwd_simt(const AttnProblem& pb, const BwdArgs& a, cudaStream_t stream);
// the same kernels over the (sequence, head) units flagged in `units`
// [n_seq * HQ + 1] only (the last word: some unit is flagged): o and lse;
// dk^(h), dv^(h) and the column part of the scalar-gate gradient, and dq
// (final, fp32) into dq32, in one launch.  D, the row part and dsink are
// left to the tensor-core path's own pass.
int attn_fwd_simt_units(const AttnProblem& pb, const FwdArgs& a, const int* units,
                        cudaStream_t stream);
int attn_bwd_simt_units(const AttnProblem& pb, const BwdArgs& a, const int* units,
                        cudaStream_t stream);
// dq, dk, dv outputs and dL (in place of dq32) from the per-head fp32 grads
int attn_bwd_reduce(const AttnProblem& pb, const BwdArgs& a, void* dq, void* dk, void* dv,
                    cudaStream_t stream);

// ---- decode cache + decode (wall_decode.cu) ----
int build_kv_cache(const void* k, const float* P, int dtype, int B, int Tn, int H, int HQ, int K,
                   int C, int t0, void* k_tilde, float* r_cache, int Tcap, cudaStream_t stream);
int decode_splits(int B, int T_kv, int H, int C);
// the device status word kernels record bounded-wait timeouts in (wall_abi.cu)
int* device_status();

// An NVTX range named after the entry point it is opened in, so that a
// profiler's timeline or kernel filter (ncu --nvtx) can pick out the
// library's calls; with no tool attached the NVTX calls do nothing.
struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};

// Function attributes and symbol addresses belong to one device's context,
// so one-time setup is kept per device: a process may drive the library on
// several devices.
constexpr int kMaxDevices = 64;
// the calling thread's current device, or -1 (no device, or beyond kMaxDevices)
int current_device();

// Raises `kernel`'s dynamic shared-memory limit to `bytes` on the current
// device, once per device; `done` is the call site's own per-device flags.
template <typename F>
inline bool set_max_smem_once(F kernel, int bytes, bool (&done)[kMaxDevices]) {
  const int dev = current_device();
  if (dev < 0) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
      return false;
    done[dev] = true;
  }
  return true;
}

int attn_decode(const void* q, const void* v, const float* p_curr, const void* k_tilde,
                const float* r_cache, const float* sink, float scale, int C, int dtype, int B,
                int T_kv, int Tcap, int H, int HQ, int K, int V, void* o, float* lse,
                float* ws, int splits, cudaStream_t stream);
// one streaming token: prefix update, cache append and decode in one launch;
// WALL_ERR_UNSUPPORTED outside the streaming kernel's domain (bf16, K and V
// in {64, 128}, HQ/H <= 8, C % 32 == 0, 16-byte aligned caches)
int decode_step(const void* q, const void* k, const void* v, const void* g, float* carry,
                void* k_tilde, void* v_cache, float* r_cache, const float* sink, float scale,
                int C, int t, int B, int Tcap, int H, int HQ, int K, int V, void* o, float* lse,
                float* ws, unsigned* counters, int splits, cudaStream_t stream);

}  // namespace wall
