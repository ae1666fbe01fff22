// wall_abi.cu -- the extern "C" entry points of libwall.so: argument checks,
// workspace layout and dispatch to the kernels.  See include/wall.h.
#include <math.h>

#include "sm100_ptx.cuh"
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {

__device__ int g_status = 0;

namespace {

constexpr int kVersion = (0 << 16) | 1;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }
bool ok_head_dim(int d) { return d >= 8 && d <= 128 && d % 8 == 0; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// The status word's address on the current device (each device holds its
// own copy of g_status).
int* status_ptr() {
  static int* p[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return nullptr;
  if (!p[dev]) {
    int* q = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&q), g_status) != cudaSuccess)
      return nullptr;
    p[dev] = q;
  }
  return p[dev];
}

// cu_seqlens must start at 0, never decrease and end at `rows`; a violation
// is recorded in the status word (kernels clamp offsets, so none faults).
__global__ void check_cu_kernel(const int32_t* cu, int n, long rows, int* status) {
  for (int s = threadIdx.x; s <= n; s += blockDim.x) {
    bool bad = false;
    if (s == 0) bad = cu[0] != 0;
    else bad = cu[s] < cu[s - 1];
    if (s == n) bad = bad || cu[n] != rows;
    if (bad) record_status(status, WALL_ERR_INVALID_ARG);
  }
}

// A wait on an mbarrier that nothing ever arrives on: the bounded wait must
// give up after limit_ns and record WALL_ERR_TIMEOUT.
__global__ void selftest_timeout_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  const uint32_t b = sm100::smem_u32(&bar);
  if (threadIdx.x == 0) {
    sm100::mbar_init(b, 1);
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) sm100::mbar_wait(b, 0, status, limit_ns);
}

int check_cu(const int32_t* cu, int n, long rows, cudaStream_t stream) {
  check_cu_kernel<<<1, 256, 0, stream>>>(cu, n, rows, status_ptr());
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

// Common shape checks of the training calls; fills `pb`.
int make_problem(int dtype, int B, int T, int H, int HQ, int K, int V, float scale,
                 int window_size, const int32_t* cu_seqlens, int n_seq, AttnProblem& pb) {
  if (dtype != WALL_BF16 && dtype != WALL_FP32) return WALL_ERR_INVALID_ARG;
  if (B < 0 || T < 0 || H < 1 || HQ < 1 || HQ % H != 0) return WALL_ERR_INVALID_ARG;
  if (!ok_head_dim(K) || !ok_head_dim(V)) return WALL_ERR_UNSUPPORTED;
  if (cu_seqlens != nullptr) {
    if (B != 1 || n_seq < 0 || n_seq > 65535 || !aligned16(cu_seqlens)) return WALL_ERR_INVALID_ARG;
  }
  if ((long)B * T * HQ * (long)(K > V ? K : V) >= (1L << 40)) return WALL_ERR_UNSUPPORTED;
  pb.dtype = dtype;
  pb.B = B; pb.T = T; pb.H = H; pb.HQ = HQ; pb.K = K; pb.V = V;
  pb.scale = scale > 0.f ? scale : 1.f / sqrtf((float)K);
  pb.window = window_size > 0 ? window_size : 0;
  pb.rows = (long)B * T;
  pb.seqs.cu = cu_seqlens;
  pb.seqs.n = cu_seqlens ? n_seq : B;
  pb.seqs.T = T;
  pb.seqs.rows = pb.rows;
  pb.extra_blocks = cu_seqlens ? n_seq : 0;
  long nb = cu_seqlens ? (T + 63L) / 64 + n_seq : (long)B * ((T + 63L) / 64);
  if (nb > 0x7fffffffL || nb * HQ > 0x7fffffffL) return WALL_ERR_UNSUPPORTED;
  pb.max_blocks64 = (int)nb;
  pb.units = nullptr;
  if (HQ > 65535) return WALL_ERR_UNSUPPORTED;
  return WALL_OK;
}

struct FwdWs {
  size_t gs;       // inclusive prefix of g_scalar [rows, HQ]
  size_t qh, kh;   // anchored operands [rows, HQ, K] bf16 (tensor-core path)
  size_t anchors;  // [n_blocks128, HQ, K] fp32
  size_t units;    // [n_seq * HQ + 1] int: units beyond the anchored range
  int n_blocks128;
  size_t total;
};
// sequences the workspace serves: B, or the cu_seqlens count (extra_blocks)
size_t unit_flags_bytes(const AttnProblem& pb) {
  return align256(sizeof(int) *
                  ((size_t)(pb.extra_blocks > 0 ? pb.extra_blocks : pb.B) * pb.HQ + 1));
}
int blocks128(const AttnProblem& pb) {
  long nb = pb.extra_blocks > 0 ? (pb.T + 127L) / 128 + pb.extra_blocks
                                : (long)pb.B * ((pb.T + 127L) / 128);
  return (int)nb;
}
FwdWs fwd_ws_layout(const AttnProblem& pb, int has_gs) {
  FwdWs w;
  size_t off = 0;
  w.gs = off;
  off += has_gs ? align256(sizeof(float) * pb.rows * pb.HQ) : 0;
  w.qh = w.kh = w.anchors = w.units = off;
  w.n_blocks128 = 0;
  if (fwd_tc_supported(pb)) {
    w.n_blocks128 = blocks128(pb);
    w.qh = off;      off += align256((size_t)2 * pb.rows * pb.HQ * pb.K);
    w.kh = off;      off += align256((size_t)2 * pb.rows * pb.HQ * pb.K);
    w.anchors = off; off += align256(sizeof(float) * (size_t)w.n_blocks128 * pb.HQ * pb.K);
    w.units = off;   off += unit_flags_bytes(pb);
  }
  w.total = off;
  return w;
}

// The stored dS tiles of the tensor-core backward (dense sequences): at most
// this much workspace, beyond it the dq kernel recomputes S, P and dP.
constexpr size_t kMaxDsBytes = size_t(8) << 30;

struct BwdWs {
  size_t D, dq32, dkh32, dvh32, dgs_row, dgs_col, gs, qh, kh, anchors, units, dS, total;
  bool has_ds;
  int n_blocks128;
};
BwdWs bwd_ws_layout(const AttnProblem& pb, int has_gs, bool want_ds = true) {
  const long rows = pb.rows;
  const int HQ = pb.HQ, K = pb.K, V = pb.V;
  BwdWs w;
  size_t off = 0;
  w.D = off;       off += align256(sizeof(float) * rows * HQ);
  w.dq32 = off;    off += align256(sizeof(float) * rows * HQ * K);
  w.dkh32 = off;   off += align256(sizeof(float) * rows * HQ * K);
  w.dvh32 = off;   off += align256(sizeof(float) * rows * HQ * V);
  w.dgs_row = off; off += align256(sizeof(float) * rows * HQ);
  w.dgs_col = off; off += align256(sizeof(float) * rows * HQ);
  w.gs = off;      off += has_gs ? align256(sizeof(float) * rows * HQ) : 0;
  w.qh = w.kh = w.anchors = w.units = off;
  w.n_blocks128 = 0;
  if (fwd_tc_supported(pb)) {
    w.n_blocks128 = blocks128(pb);
    w.qh = off;      off += align256((size_t)2 * rows * HQ * K);
    w.kh = off;      off += align256((size_t)2 * rows * HQ * K);
    w.anchors = off; off += align256(sizeof(float) * (size_t)w.n_blocks128 * HQ * K);
    w.units = off;   off += unit_flags_bytes(pb);
  }
  w.dS = off;
  w.has_ds = false;
  if (fwd_tc_supported(pb) && want_ds) {
    // dS^T tiles (bf16, 128 x 128) of every (sequence, head, I, visible J),
    // packed in the banded layout of DsLayout
    const DsLayout lay = DsLayout::of_window(pb.window);
    const size_t bytes = (size_t)DsLayout::total(lay, pb.rows, pb.T, pb.B, HQ, pb.extra_blocks) *
                         128 * 128 * 2;
    if (bytes > 0 && bytes <= kMaxDsBytes) {
      w.has_ds = true;
      off += align256(bytes);
    }
  }
  w.total = off;
  return w;
}

inline char* at(void* base, size_t off) { return static_cast<char*>(base) + off; }

// The fused prefix pass's chunk carries: one fp32 row of HQ*K per 32-row
// chunk of every sequence (a bound for varlen packing: each sequence may add
// one partial chunk).
size_t gate_scratch_bytes(const AttnProblem& pb) {
  const long chunks = pb.extra_blocks > 0 ? (pb.rows + 31) / 32 + pb.extra_blocks
                                          : (long)pb.B * ((pb.T + 31) / 32);
  return align256(sizeof(float) * (size_t)chunks * pb.HQ * pb.K);
}

// wall_attn_decode_chunk's workspace: the anchored queries and their block
// anchors (tensor-core path) or the split partials (split path)
struct ChunkWs {
  bool tc;
  int splits;
  size_t qh, anchors, total;
};
ChunkWs chunk_ws_layout(int dtype, int B, int Tq, int T_kv, int H, int HQ, int K, int V, int C) {
  ChunkWs w;
  w.tc = decode_chunk_tc_supported(dtype, K, V, C);
  w.splits = 0;
  w.qh = w.anchors = 0;
  if (w.tc) {
    const size_t nqb = (size_t)B * ((Tq + 127) / 128);
    w.anchors = align256((size_t)2 * B * Tq * HQ * K);
    w.total = w.anchors + align256(sizeof(float) * nqb * HQ * K);
  } else {
    w.splits = decode_chunk_splits(B, Tq, T_kv, H, C);
    w.total = align256(sizeof(float) * (size_t)B * Tq * HQ * w.splits * (V + 2));
  }
  return w;
}

}  // namespace

int* device_status() { return status_ptr(); }

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

}  // namespace wall

using namespace wall;

extern "C" {

int wall_version(void) { return kVersion; }

const char* wall_error_string(int code) {
  switch (code) {
    case WALL_OK: return "ok";
    case WALL_ERR_INVALID_ARG: return "invalid argument";
    case WALL_ERR_UNSUPPORTED: return "unsupported dtype or size";
    case WALL_ERR_CUDA: return "CUDA error";
    case WALL_ERR_TIMEOUT: return "device wait timed out";
    case WALL_ERR_RANGE: return "gate prefix outside the decode cache's anchored range";
    default: return "unknown status";
  }
}

int wall_get_status(wall_stream_t stream) {
  const TraceRange trace(__func__);
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return WALL_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return WALL_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return WALL_ERR_CUDA;
  return v;
}

int wall_selftest_wait_timeout(int limit_us, wall_stream_t stream) {
  const TraceRange trace(__func__);
  if (limit_us < 1 || limit_us > 2000000) return WALL_ERR_INVALID_ARG;
  int* st = status_ptr();
  if (!st) return WALL_ERR_CUDA;
  selftest_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      st, 1000ull * (unsigned long long)limit_us);
  return cudaGetLastError() == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}

int wall_prefix_cumsum(const void* g, int dtype, float* P, int B, int T, int HQ, int K,
                       const int32_t* cu_seqlens, int n_seq, const float* carry_in,
                       float* carry_out, wall_stream_t stream) {
  const TraceRange trace(__func__);
  if (dtype != WALL_BF16 && dtype != WALL_FP32) return WALL_ERR_INVALID_ARG;
  if (B < 0 || T < 0 || HQ < 1 || K < 1) return WALL_ERR_INVALID_ARG;
  if (((long)HQ * K) % 8 != 0) return WALL_ERR_UNSUPPORTED;
  if (cu_seqlens && (B != 1 || n_seq < 0 || !aligned16(cu_seqlens))) return WALL_ERR_INVALID_ARG;
  const long rows = (long)B * T;
  if (rows > 0 && (!ok_ptr(g) || !ok_ptr(P))) return WALL_ERR_INVALID_ARG;
  if (!ok_opt(carry_in) || !ok_opt(carry_out)) return WALL_ERR_INVALID_ARG;
  Seqs seqs;
  seqs.cu = cu_seqlens;
  seqs.n = cu_seqlens ? n_seq : B;
  seqs.T = T;
  seqs.rows = rows;
  if (seqs.n > 65535) return WALL_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cu_seqlens) {
    int rc = check_cu(cu_seqlens, n_seq, rows, s);
    if (rc) return rc;
  }
  timing_mark(T_PREFIX, s);
  const int rc = scan_prefix_log2(g, dtype, P, (long)HQ * K, seqs, carry_in, carry_out, s);
  timing_mark(T_PREFIX, s);
  return rc;
}

size_t wall_attn_fwd_workspace(int dtype, int B, int T, int H, int HQ, int K, int V,
                               int has_g_scalar, int n_seq) {
  AttnProblem pb;
  if (make_problem(dtype, B, T, H, HQ, K, V, 0.f, 0, nullptr, 0, pb) != WALL_OK) return 0;
  // with cu_seqlens (B == 1, n_seq > 0) each sequence may add one partial block
  if (n_seq > 0 && B == 1) pb.extra_blocks = n_seq;
  return fwd_ws_layout(pb, has_g_scalar).total;
}

int wall_attn_fwd(const void* q, const void* k, const void* v, const float* P, int dtype, int B,
                  int T, int H, int HQ, int K, int V, float scale, const float* g_scalar,
                  const float* sink_bias, int window_size, const int32_t* cu_seqlens, int n_seq,
                  void* o, float* lse, void* workspace, size_t workspace_bytes,
                  wall_stream_t stream) {
  const TraceRange trace(__func__);
  AttnProblem pb;
  int rc = make_problem(dtype, B, T, H, HQ, K, V, scale, window_size, cu_seqlens, n_seq, pb);
  if (rc) return rc;
  if (pb.rows == 0) return WALL_OK;
  if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(P) || !ok_ptr(o)) return WALL_ERR_INVALID_ARG;
  if (!ok_opt(g_scalar) || !ok_opt(sink_bias) || !ok_opt(lse)) return WALL_ERR_INVALID_ARG;
  FwdWs w = fwd_ws_layout(pb, g_scalar != nullptr);
  if (w.total > 0 && (workspace == nullptr || workspace_bytes < w.total || !aligned16(workspace)))
    return WALL_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cu_seqlens) {
    rc = check_cu(cu_seqlens, n_seq, pb.rows, s);
    if (rc) return rc;
  }
  FwdArgs a;
  a.q = q; a.k = k; a.v = v; a.P = P; a.sink = sink_bias; a.o = o; a.lse = lse;
  a.GS = nullptr;
  if (g_scalar) {
    float* gs = reinterpret_cast<float*>(at(workspace, w.gs));
    rc = scan_prefix_plain(g_scalar, gs, HQ, pb.seqs, s);
    if (rc) return rc;
    a.GS = gs;
  }
  if (fwd_tc_supported(pb)) {
    TcFwdWs tw;
    tw.qh = reinterpret_cast<__nv_bfloat16*>(at(workspace, w.qh));
    tw.kh = reinterpret_cast<__nv_bfloat16*>(at(workspace, w.kh));
    tw.anchors = reinterpret_cast<float*>(at(workspace, w.anchors));
    tw.units = reinterpret_cast<int*>(at(workspace, w.units));
    tw.n_blocks128 = w.n_blocks128;
    return attn_fwd_tc(pb, a, tw, status_ptr(), s);
  }
  return attn_fwd_simt(pb, a, s);
}

size_t wall_attn_fwd_gate_workspace(int dtype, int B, int T, int H, int HQ, int K, int V,
                                    int has_g_scalar, int n_seq) {
  AttnProblem pb;
  if (make_problem(dtype, B, T, H, HQ, K, V, 0.f, 0, nullptr, 0, pb) != WALL_OK) return 0;
  if (n_seq > 0 && B == 1) pb.extra_blocks = n_seq;
  const FwdWs w = fwd_ws_layout(pb, has_g_scalar);
  // the forward's own layout first (wall_attn_bwd may reuse it), then the
  // chunk carries of the fused prefix pass
  return w.total + (fwd_tc_supported(pb) ? gate_scratch_bytes(pb) : 0);
}

int wall_attn_fwd_gate(const void* q, const void* k, const void* v, const void* g, int dtype,
                       int B, int T, int H, int HQ, int K, int V, float scale,
                       const float* g_scalar, const float* sink_bias, int window_size,
                       const int32_t* cu_seqlens, int n_seq, float* P, void* o, float* lse,
                       void* workspace, size_t workspace_bytes, wall_stream_t stream) {
  const TraceRange trace(__func__);
  AttnProblem pb;
  int rc = make_problem(dtype, B, T, H, HQ, K, V, scale, window_size, cu_seqlens, n_seq, pb);
  if (rc) return rc;
  if (pb.rows == 0) return WALL_OK;
  if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(g) || !ok_ptr(P) || !ok_ptr(o))
    return WALL_ERR_INVALID_ARG;
  if (!ok_opt(g_scalar) || !ok_opt(sink_bias) || !ok_opt(lse)) return WALL_ERR_INVALID_ARG;
  const FwdWs w = fwd_ws_layout(pb, g_scalar != nullptr);
  const bool tc = fwd_tc_supported(pb);
  const size_t need = w.total + (tc ? gate_scratch_bytes(pb) : 0);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
    return WALL_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cu_seqlens) {
    rc = check_cu(cu_seqlens, n_seq, pb.rows, s);
    if (rc) return rc;
  }
  FwdArgs a;
  a.q = q; a.k = k; a.v = v; a.P = P; a.sink = sink_bias; a.o = o; a.lse = lse;
  a.GS = nullptr;
  if (g_scalar) {
    float* gs = reinterpret_cast<float*>(at(workspace, w.gs));
    rc = scan_prefix_plain(g_scalar, gs, HQ, pb.seqs, s);
    if (rc) return rc;
    a.GS = gs;
  }
  if (!tc) {
    timing_mark(T_PREFIX, s);
    rc = scan_prefix_log2(g, dtype, P, (long)HQ * K, pb.seqs, nullptr, nullptr, s);
    timing_mark(T_PREFIX, s);
    if (rc) return rc;
    return attn_fwd_simt(pb, a, s);
  }
  TcFwdWs tw;
  tw.qh = reinterpret_cast<__nv_bfloat16*>(at(workspace, w.qh));
  tw.kh = reinterpret_cast<__nv_bfloat16*>(at(workspace, w.kh));
  tw.anchors = reinterpret_cast<float*>(at(workspace, w.anchors));
  tw.units = reinterpret_cast<int*>(at(workspace, w.units));
  tw.n_blocks128 = w.n_blocks128;
  rc = scan_prefix_operands(static_cast<const __nv_bfloat16*>(g),
                            static_cast<const __nv_bfloat16*>(q),
                            static_cast<const __nv_bfloat16*>(k), P,
                            reinterpret_cast<float*>(at(workspace, w.total)), HQ, H, K, pb.seqs,
                            tw.qh, tw.kh, tw.anchors, tw.units, s);
  if (rc) return rc;
  return attn_fwd_tc(pb, a, tw, status_ptr(), s, /*prepared=*/true);
}

size_t wall_attn_bwd_workspace(int dtype, int B, int T, int H, int HQ, int K, int V,
                               int has_g_scalar, int n_seq, int window_size) {
  AttnProblem pb;
  if (make_problem(dtype, B, T, H, HQ, K, V, 0.f, window_size, nullptr, 0, pb) != WALL_OK)
    return 0;
  if (n_seq > 0 && B == 1) pb.extra_blocks = n_seq;
  return bwd_ws_layout(pb, has_g_scalar).total;
}

size_t wall_attn_bwd_workspace_min(int dtype, int B, int T, int H, int HQ, int K, int V,
                                   int has_g_scalar, int n_seq) {
  AttnProblem pb;
  if (make_problem(dtype, B, T, H, HQ, K, V, 0.f, 0, nullptr, 0, pb) != WALL_OK) return 0;
  if (n_seq > 0 && B == 1) pb.extra_blocks = n_seq;
  return bwd_ws_layout(pb, has_g_scalar, /*want_ds=*/false).total;
}

int wall_attn_bwd(const void* dO, const void* q, const void* k, const void* v, const float* P,
                  const void* o, const float* lse, int dtype, int B, int T, int H, int HQ,
                  int K, int V, float scale, const float* g_scalar, const float* sink_bias,
                  int window_size, const int32_t* cu_seqlens, int n_seq, void* dq, void* dk,
                  void* dv, void* dg, float* dg_scalar, float* dsink, void* workspace,
                  size_t workspace_bytes, const void* fwd_workspace, wall_stream_t stream) {
  const TraceRange trace(__func__);
  AttnProblem pb;
  int rc = make_problem(dtype, B, T, H, HQ, K, V, scale, window_size, cu_seqlens, n_seq, pb);
  if (rc) return rc;
  if ((g_scalar == nullptr) != (dg_scalar == nullptr)) return WALL_ERR_INVALID_ARG;
  if (!ok_opt(fwd_workspace)) return WALL_ERR_INVALID_ARG;
  if (dsink != nullptr && sink_bias == nullptr) return WALL_ERR_INVALID_ARG;
  if (!ok_opt(g_scalar) || !ok_opt(sink_bias) || !ok_opt(dg_scalar) || !ok_opt(dsink))
    return WALL_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (pb.rows == 0) {
    // nothing to sum: dsink is 0 (otherwise the backward writes all of it)
    if (dsink && cudaMemsetAsync(dsink, 0, sizeof(float) * HQ, s) != cudaSuccess)
      return WALL_ERR_CUDA;
    return WALL_OK;
  }
  if (!ok_ptr(dO) || !ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(P) || !ok_ptr(o) ||
      !ok_ptr(lse) || !ok_ptr(dq) || !ok_ptr(dk) || !ok_ptr(dv) || !ok_ptr(dg))
    return WALL_ERR_INVALID_ARG;
  // the dS tiles if the workspace holds them, else the dq pass recomputes
  BwdWs w = bwd_ws_layout(pb, g_scalar != nullptr);
  if (workspace_bytes < w.total) w = bwd_ws_layout(pb, g_scalar != nullptr, false);
  if (workspace == nullptr || workspace_bytes < w.total || !aligned16(workspace))
    return WALL_ERR_INVALID_ARG;
  if (cu_seqlens) {
    rc = check_cu(cu_seqlens, n_seq, pb.rows, s);
    if (rc) return rc;
  }
  BwdArgs a;
  a.dO = dO; a.q = q; a.k = k; a.v = v; a.o = o; a.P = P; a.lse = lse;
  a.sink = sink_bias;
  a.dsink = dsink;
  a.D = reinterpret_cast<float*>(at(workspace, w.D));
  a.dq32 = reinterpret_cast<float*>(at(workspace, w.dq32));
  a.dkh32 = reinterpret_cast<float*>(at(workspace, w.dkh32));
  a.dvh32 = reinterpret_cast<float*>(at(workspace, w.dvh32));
  a.dgs_row = reinterpret_cast<float*>(at(workspace, w.dgs_row));
  a.dgs_col = reinterpret_cast<float*>(at(workspace, w.dgs_col));
  // dq from the stored dS tiles (tensor-core path, tiles within their cap)
  a.dS = w.has_ds ? reinterpret_cast<__nv_bfloat16*>(at(workspace, w.dS)) : nullptr;
  a.GS = nullptr;
  if (g_scalar && fwd_workspace != nullptr && fwd_tc_supported(pb)) {
    // the forward formed the prefix of the same g_scalar in its workspace
    a.GS = reinterpret_cast<float*>(
        at(const_cast<void*>(fwd_workspace), fwd_ws_layout(pb, 1).gs));
  } else if (g_scalar) {
    float* gs = reinterpret_cast<float*>(at(workspace, w.gs));
    rc = scan_prefix_plain(g_scalar, gs, HQ, pb.seqs, s);
    if (rc) return rc;
    a.GS = gs;
  }
  if (fwd_tc_supported(pb)) {
    TcFwdWs tw;
    tw.qh = reinterpret_cast<__nv_bfloat16*>(at(workspace, w.qh));
    tw.kh = reinterpret_cast<__nv_bfloat16*>(at(workspace, w.kh));
    tw.anchors = reinterpret_cast<float*>(at(workspace, w.anchors));
    tw.units = reinterpret_cast<int*>(at(workspace, w.units));
    tw.n_blocks128 = w.n_blocks128;
    const bool reuse = fwd_workspace != nullptr;
    if (reuse) {
      // the forward's anchored operands and unit flags, in its own layout
      const FwdWs fw = fwd_ws_layout(pb, g_scalar != nullptr);
      void* fws = const_cast<void*>(fwd_workspace);
      tw.qh = reinterpret_cast<__nv_bfloat16*>(at(fws, fw.qh));
      tw.kh = reinterpret_cast<__nv_bfloat16*>(at(fws, fw.kh));
      tw.anchors = reinterpret_cast<float*>(at(fws, fw.anchors));
      tw.units = reinterpret_cast<int*>(at(fws, fw.units));
    }
    // dg as well: dL's reverse scan starts inside the finalize pass
    rc = attn_bwd_tc(pb, a, tw, !reuse, dq, dk, dv, dg, status_ptr(), s);
    if (rc) return rc;
  } else {
    rc = attn_bwd_simt(pb, a, s);
    if (rc) return rc;
    rc = attn_bwd_reduce(pb, a, dq, dk, dv, s);
    if (rc) return rc;
    // dg = reverse cumulative sum of dL (held in dq32 after the reduce);
    // the per-head dk buffer is dead after the reduce: chunk scratch
    timing_mark(T_REV_SCAN, s);
    rc = scan_reverse(a.dq32, dg, dtype, a.dkh32, (long)HQ * K, pb.seqs, s);
    timing_mark(T_REV_SCAN, s);
    if (rc) return rc;
  }
  if (g_scalar) {
    timing_mark(T_REV_SCAN, s);
    rc = scan_reverse(a.dgs_row, dg_scalar, WALL_FP32, a.dgs_col, HQ, pb.seqs, s);
    timing_mark(T_REV_SCAN, s);
  }
  return rc;
}

int wall_build_kv_cache(const void* k, const float* P, int dtype, int B, int Tn, int H, int HQ,
                        int K, int C, int t0, void* k_tilde, float* r_cache, int Tcap,
                        wall_stream_t stream) {
  const TraceRange trace(__func__);
  if (dtype != WALL_BF16 && dtype != WALL_FP32) return WALL_ERR_INVALID_ARG;
  if (B < 0 || Tn < 0 || H < 1 || HQ < 1 || HQ % H != 0 || C < 1 || t0 < 0 || Tcap < 0)
    return WALL_ERR_INVALID_ARG;
  if ((long)t0 + Tn > Tcap) return WALL_ERR_INVALID_ARG;
  if (K < 8 || K % 8 != 0) return WALL_ERR_UNSUPPORTED;
  if ((long)B * Tn == 0) return WALL_OK;
  if (!ok_ptr(k) || !ok_ptr(P) || !ok_ptr(k_tilde) || !ok_ptr(r_cache)) return WALL_ERR_INVALID_ARG;
  timing_mark(T_CACHE, reinterpret_cast<cudaStream_t>(stream));
  const int rc = build_kv_cache(k, P, dtype, B, Tn, H, HQ, K, C, t0, k_tilde, r_cache, Tcap,
                                reinterpret_cast<cudaStream_t>(stream));
  timing_mark(T_CACHE, reinterpret_cast<cudaStream_t>(stream));
  return rc;
}

size_t wall_attn_decode_workspace(int B, int T_kv, int H, int HQ, int V, int C) {
  if (B < 0 || T_kv < 1 || H < 1 || HQ < 1 || HQ % H != 0 || V < 1 || C < 1) return 0;
  const int S = decode_splits(B, T_kv, H, C);
  return align256(sizeof(float) * (size_t)B * HQ * S * (V + 2));
}

int wall_attn_decode(const void* q, const void* v, const float* p_curr, const void* k_tilde,
                     const float* r_cache, const float* sink_bias, float scale, int C, int dtype,
                     int B, int T_kv, int Tcap, int H, int HQ, int K, int V, void* o, float* lse,
                     void* workspace, size_t workspace_bytes, wall_stream_t stream) {
  const TraceRange trace(__func__);
  if (dtype != WALL_BF16 && dtype != WALL_FP32) return WALL_ERR_INVALID_ARG;
  if (B < 0 || T_kv < 1 || Tcap < T_kv || H < 1 || HQ < 1 || HQ % H != 0 || C < 1)
    return WALL_ERR_INVALID_ARG;
  if (!ok_head_dim(K) || !ok_head_dim(V) || HQ / H > 32) return WALL_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535) return WALL_ERR_UNSUPPORTED;
  if (B == 0) return WALL_OK;
  if (!ok_ptr(q) || !ok_ptr(v) || !ok_ptr(p_curr) || !ok_ptr(k_tilde) || !ok_ptr(r_cache) ||
      !ok_ptr(o) || !ok_opt(sink_bias) || !ok_opt(lse))
    return WALL_ERR_INVALID_ARG;
  const int S = decode_splits(B, T_kv, H, C);
  const size_t need = align256(sizeof(float) * (size_t)B * HQ * S * (V + 2));
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace))
    return WALL_ERR_INVALID_ARG;
  const float sc = scale > 0.f ? scale : 1.f / sqrtf((float)K);
  timing_mark(T_DECODE, reinterpret_cast<cudaStream_t>(stream));
  const int rc = attn_decode(q, v, p_curr, k_tilde, r_cache, sink_bias, sc, C, dtype, B, T_kv,
                             Tcap, H, HQ, K, V, o, lse, static_cast<float*>(workspace), S,
                             reinterpret_cast<cudaStream_t>(stream));
  timing_mark(T_DECODE, reinterpret_cast<cudaStream_t>(stream));
  return rc;
}

size_t wall_attn_decode_chunk_workspace(int dtype, int B, int Tq, int T_kv, int H, int HQ, int K,
                                        int V, int C) {
  if (B < 0 || Tq < 0 || T_kv < 1 || Tq > T_kv || H < 1 || HQ < 1 || HQ % H != 0 || K < 1 ||
      V < 1 || C < 1)
    return 0;
  return chunk_ws_layout(dtype, B, Tq, T_kv, H, HQ, K, V, C).total;
}

int wall_attn_decode_chunk(const void* q, const void* v, const float* p, const void* k_tilde,
                           const float* r_cache, const float* sink_bias, float scale, int C,
                           int dtype, int B, int Tq, int T_kv, int Tcap, int H, int HQ, int K,
                           int V, void* o, float* lse, void* workspace, size_t workspace_bytes,
                           wall_stream_t stream) {
  const TraceRange trace(__func__);
  if (dtype != WALL_BF16 && dtype != WALL_FP32) return WALL_ERR_INVALID_ARG;
  if (B < 0 || Tq < 0 || T_kv < 1 || Tq > T_kv || Tcap < T_kv || H < 1 || HQ < 1 ||
      HQ % H != 0 || C < 1)
    return WALL_ERR_INVALID_ARG;
  if (!ok_head_dim(K) || !ok_head_dim(V) || HQ / H > 32) return WALL_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535 || HQ > 65535) return WALL_ERR_UNSUPPORTED;
  if ((long)B * Tq == 0) return WALL_OK;
  const ChunkWs w = chunk_ws_layout(dtype, B, Tq, T_kv, H, HQ, K, V, C);
  // grid rows: query rows (split path) or 128-row query blocks (tensor cores)
  if ((long)B * (w.tc ? (Tq + 127) / 128 : Tq) > 65535) return WALL_ERR_UNSUPPORTED;
  if (!ok_ptr(q) || !ok_ptr(v) || !ok_ptr(p) || !ok_ptr(k_tilde) || !ok_ptr(r_cache) ||
      !ok_ptr(o) || !ok_opt(sink_bias) || !ok_opt(lse))
    return WALL_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < w.total || !aligned16(workspace))
    return WALL_ERR_INVALID_ARG;
  const float sc = scale > 0.f ? scale : 1.f / sqrtf((float)K);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  timing_mark(T_CHUNK, st);
  int rc;
  if (w.tc)
    rc = attn_decode_chunk_tc(q, v, p, k_tilde, r_cache, sink_bias, sc, C, B, Tq, T_kv, Tcap, H,
                              HQ, K, reinterpret_cast<__nv_bfloat16*>(at(workspace, w.qh)),
                              reinterpret_cast<float*>(at(workspace, w.anchors)), o, lse,
                              status_ptr(), st);
  else
    rc = attn_decode_chunk_split(q, v, p, k_tilde, r_cache, sink_bias, sc, C, dtype, B, Tq, T_kv,
                                 Tcap, H, HQ, K, V, o, lse, static_cast<float*>(workspace),
                                 w.splits, st);
  timing_mark(T_CHUNK, st);
  return rc;
}

size_t wall_decode_step_workspace(int B, int Tcap, int H, int HQ, int V, int C) {
  if (B < 0 || Tcap < 1 || H < 1 || HQ < 1 || HQ % H != 0 || V < 1 || C < 1) return 0;
  const int S = decode_splits(B, Tcap, H, C);
  return align256(sizeof(float) * (size_t)B * HQ * S * (V + 2)) +
         align256(sizeof(unsigned) * (size_t)B * HQ);
}

int wall_decode_step(const void* q, const void* k, const void* v, const void* g, int dtype,
                     float* carry, void* k_tilde, void* v_cache, float* r_cache,
                     const float* sink_bias, float scale, int C, int t, int B, int Tcap, int H,
                     int HQ, int K, int V, void* o, float* lse, void* workspace,
                     size_t workspace_bytes, wall_stream_t stream) {
  const TraceRange trace(__func__);
  if (dtype != WALL_BF16 && dtype != WALL_FP32) return WALL_ERR_INVALID_ARG;
  if (B < 0 || t < 0 || Tcap < 1 || t >= Tcap || H < 1 || HQ < 1 || HQ % H != 0 || C < 1)
    return WALL_ERR_INVALID_ARG;
  if (dtype != WALL_BF16 || (K != 64 && K != 128) || (V != 64 && V != 128) || HQ / H > 8 ||
      C % 32 != 0 || B > 65535 || H > 65535)
    return WALL_ERR_UNSUPPORTED;
  if (B == 0) return WALL_OK;
  if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(g) || !ok_ptr(carry) ||
      !ok_ptr(k_tilde) || !ok_ptr(v_cache) || !ok_ptr(r_cache) || !ok_ptr(o) ||
      !ok_opt(sink_bias) || !ok_opt(lse))
    return WALL_ERR_INVALID_ARG;
  const size_t need = wall_decode_step_workspace(B, Tcap, H, HQ, V, C);
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace))
    return WALL_ERR_INVALID_ARG;
  // partials sized for the largest split count the capacity allows, then the
  // per-head arrival counters
  const int S_cap = decode_splits(B, Tcap, H, C);
  float* ws = static_cast<float*>(workspace);
  unsigned* counters = reinterpret_cast<unsigned*>(
      static_cast<char*>(workspace) + align256(sizeof(float) * (size_t)B * HQ * S_cap * (V + 2)));
  const float sc = scale > 0.f ? scale : 1.f / sqrtf((float)K);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  timing_mark(T_STEP, st);
  const int rc = decode_step(q, k, v, g, carry, k_tilde, v_cache, r_cache, sink_bias, sc, C, t,
                             B, Tcap, H, HQ, K, V, o, lse, ws, counters,
                             decode_splits(B, t, H, C), st);
  timing_mark(T_STEP, st);
  return rc;
}

}  // extern "C"
