/*
 * wall.h -- C ABI of the B200 Wall Attention hot path (libwall.so).
 *
 * Wall Attention (Tilde blog "Wall Attention", "Definition: Wall Attention";
 * wall-attention-release README, introduction) is causal softmax attention
 * whose logit carries a per-channel decay accumulated between the two
 * positions:
 *
 *     s_ij = scale * sum_n exp(sum_{r=j+1..i} g_{r,n}) q_{i,n} k_{j,n}
 *            [+ sum_{r=j+1..i} g_scalar_r]                 (optional)
 *     o_i  = sum_{j<=i} softmax_j(s_ij) v_j
 *
 * g is the natural-log gate per query head and channel, so g = 0 is vanilla
 * softmax attention.  The kernels work with the base-2 prefix
 * P_t = sum_{u<=t} g_u / ln 2 (README "Decode": cumulative sum of g with scale
 * 1/ln 2; blog: P_t = sum_{u<=t} log g_u), and use exp2(P_i - P_j) =
 * exp2(P_i - R) * exp2(R - P_j) with block anchors R (blog, fast training,
 * per-block anchor).
 *
 * Conventions shared by every call
 *   - Tensors are dense, row-major, in the README's BSHD layout:
 *       q [B,T,HQ,K], k [B,T,H,K], v [B,T,H,V], g and P [B,T,HQ,K],
 *       g_scalar [B,T,HQ], sink_bias [HQ], o [B,T,HQ,V], lse [B,T,HQ].
 *     With cu_seqlens (varlen packing, README "Usage": requires B == 1) the
 *     T rows hold n_seq sequences back to back; attention, P and the scalar
 *     gate prefix never cross a sequence boundary.
 *   - GQA: HQ % H == 0 and query head h reads kv head h / (HQ/H).
 *   - dtype is WALL_BF16 or WALL_FP32 and applies to q, k, v, g, o, dO, dq,
 *     dk, dv, dg, k_tilde.  P, lse, r_cache, g_scalar, sink_bias, dg_scalar,
 *     dsink and carries are always fp32; cu_seqlens is int32 [n_seq+1],
 *     starting at 0, non-decreasing and ending at T.
 *   - Pointers are device pointers, 16-byte aligned.  The caller allocates
 *     and owns every buffer, including workspaces whose sizes the *_workspace
 *     calls return; the library allocates no device memory and keeps no
 *     state between calls except one device status word (wall_get_status),
 *     the fixed scratch array of wall_attn_decode_noalloc and the events of
 *     the per-stage timing aid.  Calls run on the calling thread's current
 *     device (cudaSetDevice); the status word and the scratch array exist
 *     once per device, and per-device setup (kernel shared-memory limits,
 *     symbol addresses) is done on a device's first call, for up to 64
 *     devices in one process.  The timing aid times one device per process
 *     (its events are created on the device current at a stage's first
 *     timed launch).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Arguments are checked on the host before any launch;
 *     on a bad argument nothing is launched and the call returns an error.
 *     Kernels never trap: a device-side failure (a bounded wait that timed
 *     out) is recorded in the status word.
 *   - scale <= 0 selects K^-0.5 (README "Usage": scale = K ** -0.5).
 *     window_size <= 0 means no window; otherwise key j is visible from
 *     query i iff 0 <= i - j < window_size.
 *   - Empty problems (B == 0 or T == 0) are valid and launch nothing.
 *   - No call allocates or synchronizes except wall_get_status and
 *     wall_timing_read.  After an entry point's first call on a device
 *     (which sets its kernels' shared-memory limits), its calls may be
 *     captured in a CUDA graph and replayed; the timing aid must be off
 *     during a capture.
 *   - Every call that launches work (and wall_get_status) opens an NVTX
 *     range named after itself, for profiler timelines and ncu's --nvtx
 *     filters; without a profiler attached the range costs nothing.
 */
#ifndef WALL_H
#define WALL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* wall_stream_t; /* same type as cudaStream_t */

/* status codes */
#define WALL_OK 0
#define WALL_ERR_INVALID_ARG 1 /* null pointer, bad shape, HQ % H != 0, misalignment, ... */
#define WALL_ERR_UNSUPPORTED 2 /* dtype or head size not built */
#define WALL_ERR_CUDA 3        /* a CUDA launch or copy failed */
#define WALL_ERR_TIMEOUT 4     /* a kernel's bounded wait expired (from wall_get_status) */
#define WALL_ERR_RANGE 5       /* a gate prefix left the decode cache's anchored range
                                  (from wall_get_status; see wall_build_kv_cache) */

/* dtypes */
#define WALL_BF16 0
#define WALL_FP32 1

/* Library version, (major << 16) | minor. */
int wall_version(void);

/* Human-readable name of a status code (static string). */
const char* wall_error_string(int code);

/*
 * wall_prefix_cumsum -- base-2 inclusive prefix of the log-gate.
 * README "Decode": P = cumulative sum of g with scale 1/ln 2; blog
 * "Definition: Wall Attention": P_t = sum_{u<=t} log g_u.
 *
 *   P[b,t,h,n] = c[s,h,n] + (sum_{u = start(s) .. t} g[b,u,h,n]) / ln 2
 *
 * where s is the sequence holding row t (batch row b without cu_seqlens) and
 * c = carry_in (NULL: zero).  g [B,T,HQ,K] in `dtype`; P [B,T,HQ,K] fp32.
 * carry_in / carry_out: [n_s, HQ, K] fp32 with n_s = B (no cu_seqlens) or
 * n_seq; carry_out receives each sequence's last P (carry_in when empty), so
 * a stream of tokens can be scanned piece by piece.  Either may be NULL.
 * Returns WALL_ERR_UNSUPPORTED for HQ*K not a multiple of 8.
 */
int wall_prefix_cumsum(const void* g, int dtype, float* P, int B, int T, int HQ, int K,
                       const int32_t* cu_seqlens, int n_seq, const float* carry_in,
                       float* carry_out, wall_stream_t stream);

/*
 * wall_attn_fwd_workspace -- bytes of workspace wall_attn_fwd needs for
 * these sizes (0 is possible).  Returns 0 on bad sizes as well.
 */
size_t wall_attn_fwd_workspace(int dtype, int B, int T, int H, int HQ, int K, int V,
                               int has_g_scalar, int n_seq);

/*
 * wall_attn_fwd -- Wall Attention forward (README "Usage": wall_attn; blog
 * "Definition: Wall Attention").
 *
 * In:  q [B,T,HQ,K], k [B,T,H,K], v [B,T,H,V] in `dtype`; P [B,T,HQ,K] fp32
 *      from wall_prefix_cumsum of g; optional g_scalar [B,T,HQ] fp32 (FoX-
 *      style additive log-gate: the logit gains sum_{r=j+1..i} g_scalar_r,
 *      added after `scale`), sink_bias [HQ] fp32 (one extra logit per head
 *      with a zero value row, included in lse), window_size, cu_seqlens.
 * Out: o [B,T,HQ,V] in `dtype`; lse [B,T,HQ] fp32, natural log of the
 *      softmax denominator (sink included).  lse may be NULL.
 * Supported: K, V multiples of 8 up to 128; the
 * tensor-core path takes bf16 with K == V in {64, 128}, other cases use the
 * fp32 SIMT path.  fp32 inputs are computed with fp32 products throughout.
 */
int wall_attn_fwd(const void* q, const void* k, const void* v, const float* P, int dtype, int B,
                  int T, int H, int HQ, int K, int V, float scale, const float* g_scalar,
                  const float* sink_bias, int window_size, const int32_t* cu_seqlens, int n_seq,
                  void* o, float* lse, void* workspace, size_t workspace_bytes,
                  wall_stream_t stream);

/* wall_attn_fwd_gate_workspace -- bytes of workspace wall_attn_fwd_gate needs:
 * wall_attn_fwd_workspace's layout first, then the prefix scan's chunk
 * carries on the tensor-core path: fp32, one row of HQ*K per 32-row chunk
 * of every sequence (B * ceil(T / 32) rows dense; ceil(B*T / 32) + n_seq
 * rows with cu_seqlens). */
size_t wall_attn_fwd_gate_workspace(int dtype, int B, int T, int H, int HQ, int K, int V,
                                    int has_g_scalar, int n_seq);

/*
 * wall_attn_fwd_gate -- wall_prefix_cumsum and wall_attn_fwd in one call,
 * with the prefix fused into the forward (blog "Wall Attention", fast
 * training section 1: the anchored factors come from the prefix P of the
 * gates; README "Decode": P = cumsum(g) / ln 2).  From the gates g
 * [B,T,HQ,K] (`dtype`) it writes P [B,T,HQ,K] fp32 -- bit for bit what
 * wall_prefix_cumsum writes, for wall_attn_bwd -- and o, lse exactly as
 * wall_attn_fwd computes them from that P.  On the tensor-core path the
 * scan's last pass also forms the anchored operands, so P is not read back
 * (one pass over q, k, g instead of a scan and a preparation pass).  The
 * workspace (wall_attn_fwd_gate_workspace bytes, 16-byte aligned) begins with
 * wall_attn_fwd's layout, so it can be handed to wall_attn_bwd as its
 * fwd_workspace.  Arguments, options, errors and the supported cases are
 * those of wall_attn_fwd, plus g (non-null, 16-byte aligned).
 */
int wall_attn_fwd_gate(const void* q, const void* k, const void* v, const void* g, int dtype,
                       int B, int T, int H, int HQ, int K, int V, float scale,
                       const float* g_scalar, const float* sink_bias, int window_size,
                       const int32_t* cu_seqlens, int n_seq, float* P, void* o, float* lse,
                       void* workspace, size_t workspace_bytes, wall_stream_t stream);

/* wall_attn_bwd_workspace -- bytes of workspace wall_attn_bwd needs for a
 * problem with this window (window_size <= 0: none; a call with a window
 * fits a workspace sized for a wider one or none).  On the bf16 tensor-core
 * path it includes room for every dS tile the backward forms, bf16 128 x 128
 * per (sequence, head, query block I, visible key block J), when that is at
 * most 8 GiB; the dq pass then reads those tiles instead of recomputing them.
 * Dense: B*HQ*nb(nb+1)/2 tiles without a window, nb = ceil(T/128) (1.09 GB
 * at B=1, T=8192, HQ=16); a window of W keys keeps ceil((W-1)/128) + 1 key
 * blocks per query block; varlen packing (n_seq > 0) reserves the tiles of
 * one sequence holding every row plus n_seq partial blocks (a bound, since
 * the lengths are on the device). */
size_t wall_attn_bwd_workspace(int dtype, int B, int T, int H, int HQ, int K, int V,
                               int has_g_scalar, int n_seq, int window_size);

/* wall_attn_bwd_workspace_min -- the least workspace wall_attn_bwd accepts:
 * without room for the dS tiles (window-independent).  Given a workspace
 * smaller than wall_attn_bwd_workspace's size but at least this one, the
 * backward keeps no dS tiles and its dq pass recomputes S, P, dP and dS on
 * the tensor cores (for callers short of memory; the results agree to bf16
 * rounding). */
size_t wall_attn_bwd_workspace_min(int dtype, int B, int T, int H, int HQ, int K, int V,
                                   int has_g_scalar, int n_seq);

/*
 * wall_attn_bwd -- gradients of a scalar loss through wall_attn_fwd (README
 * "Usage": analytic gradients for q, k, v, g, and g_scalar).
 *
 * In:  dO [B,T,HQ,V], and the forward's q, k, v, P, options, o and lse.
 * Out: dq [B,T,HQ,K], dk [B,T,H,K], dv [B,T,H,V], dg [B,T,HQ,K] in `dtype`;
 *      dg_scalar [B,T,HQ] fp32 (must be NULL iff g_scalar is NULL);
 *      dsink [HQ] fp32 (optional, may be NULL; requires sink_bias).
 * The gate gradient follows the blog's fused gate gradient (fast training):
 * per query head, dL_t = q_t (.) dq_t - k_t (.) dk^(h)_t with the key-side
 * term -K_j (.) dK_j, then dg = the reverse cumulative sum of dL within each
 * sequence.  dk^(h), dv^(h) are summed over each GQA group.
 * fwd_workspace: NULL, or the workspace of the wall_attn_fwd (or
 * wall_attn_fwd_gate) call that produced o and lse, with the same q, k, P,
 * shapes and options and left unchanged since.  On the bf16 tensor-core
 * path the anchored operands (and, with g_scalar, the gate's prefix) that
 * call prepared in it are then read instead of recomputed; it is only read.
 * Elsewhere it is ignored.
 */
int wall_attn_bwd(const void* dO, const void* q, const void* k, const void* v, const float* P,
                  const void* o, const float* lse, int dtype, int B, int T, int H, int HQ,
                  int K, int V, float scale, const float* g_scalar, const float* sink_bias,
                  int window_size, const int32_t* cu_seqlens, int n_seq, void* dq, void* dk,
                  void* dv, void* dg, float* dg_scalar, float* dsink, void* workspace,
                  size_t workspace_bytes, const void* fwd_workspace, wall_stream_t stream);

/*
 * wall_build_kv_cache -- pre-rescaled decode cache (README "Decode":
 * build_wall_kv_cache; k_tilde[j] = k[j] * exp2(R_c - P[j]) with a per-chunk
 * anchor R_c).
 *
 * Writes cache positions t0 .. t0+Tn-1 of each batch row:
 *   c = t / C;  R_c = r_cache[b,c,h,:] if c*C < t0 (chunk already started:
 *   its anchor is kept), else R_c = P at position c*C (written to r_cache);
 *   k_tilde[b,t,h,:] = k[b,t-t0,h/G,:] * exp2(R_c - P[b,t-t0,h,:]).
 * In:  k [B,Tn,H,K] (`dtype`) and P [B,Tn,HQ,K] fp32 for positions t0..t0+Tn-1.
 * Out: k_tilde [B,Tcap,HQ,K] (`dtype`), r_cache [B,ceil(Tcap/C),HQ,K] fp32.
 * Requires t0 + Tn <= Tcap and C >= 1.  At chunk starts k_tilde equals k
 * bit for bit (the factor is exp2(0) = 1).
 */
int wall_build_kv_cache(const void* k, const float* P, int dtype, int B, int Tn, int H, int HQ,
                        int K, int C, int t0, void* k_tilde, float* r_cache, int Tcap,
                        wall_stream_t stream);

/* wall_attn_decode_workspace -- bytes of workspace wall_attn_decode needs. */
size_t wall_attn_decode_workspace(int B, int T_kv, int H, int HQ, int V, int C);

/*
 * wall_attn_decode -- one decode step against the pre-rescaled cache
 * (README "Decode": wall_attn_decode; blog: the decode kernel folds the gate
 * into the cached keys and needs no gate arithmetic in its inner loop).
 *
 * For each batch row b and query head h, with c(j) = j / C:
 *   s_j = scale * sum_n q[b,h,n] exp2(p_curr[b,h,n] - r_cache[b,c(j),h,n])
 *                  * k_tilde[b,j,h,n],      j = 0 .. T_kv-1
 *   o = sum_j softmax(s, sink)_j v[b,j,h/G,:],   lse = log-sum-exp (natural)
 * In:  q [B,1,HQ,K] (`dtype`), p_curr [B,1,HQ,K] fp32 (P at the current
 *      position), k_tilde [B,Tcap,HQ,K] and v [B,Tcap,H,V] (`dtype`, the
 *      first T_kv positions are read), r_cache [B,ceil(Tcap/C),HQ,K] fp32,
 *      sink_bias [HQ] or NULL.  The current token's own key must already be
 *      in the cache (position T_kv-1), so T_kv >= 1.
 * Out: o [B,1,HQ,V] (`dtype`), lse [B,1,HQ] fp32 (may be NULL).
 * Supported: bf16 or fp32, K and V multiples of 8 up to 128.
 */
int wall_attn_decode(const void* q, const void* v, const float* p_curr, const void* k_tilde,
                     const float* r_cache, const float* sink_bias, float scale, int C, int dtype,
                     int B, int T_kv, int Tcap, int H, int HQ, int K, int V, void* o, float* lse,
                     void* workspace, size_t workspace_bytes, wall_stream_t stream);

/*
 * wall_attn_decode_noalloc -- wall_attn_decode for callers that cannot
 * allocate device memory (code running during CUDA graph capture that must not
 * allocate, serving loops whose memory is planned once, bindings without a
 * device allocator).  The paper has no counterpart: it is a deployment variant.
 *
 * Same arguments, layout and results as wall_attn_decode, without the
 * workspace: the split partials live in a fixed 4 MiB scratch array inside the
 * library's device memory (every GPU that loads the library holds it until the
 * process exits).  Problems needing more, B * HQ * splits * (V + 2) > 2^20
 * floats with splits as wall_attn_decode chooses them, are rejected with
 * WALL_ERR_UNSUPPORTED before anything runs; use wall_attn_decode for those.
 * The entry point calls no allocator.  Its first call on a device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current, so
 * make that first call before any stream capture.  All calls share the one
 * array and each call overwrites every partial it reads, so nothing needs
 * clearing (after a device timeout, which wall_get_status reports, the splits
 * that gave up are written as empty partials, so no earlier call's values are
 * merged either); calls that overlap on the GPU (concurrent streams) race on
 * it.
 */
int wall_attn_decode_noalloc(const void* q, const void* v, const float* p_curr,
                             const void* k_tilde, const float* r_cache, const float* sink_bias,
                             float scale, int C, int dtype, int B, int T_kv, int Tcap, int H,
                             int HQ, int K, int V, void* o, float* lse, wall_stream_t stream);

/* wall_decode_step_workspace -- bytes of workspace wall_decode_step needs
 * for a cache of capacity Tcap (enough for every t < Tcap). */
size_t wall_decode_step_workspace(int B, int Tcap, int H, int HQ, int V, int C);

/*
 * wall_decode_step -- one token of the streaming decode loop in ONE launch:
 * prefix update, cache append and decode (README "Decode": the prefix is the
 * running sum of g / ln 2 and the cache holds k * exp2(R_c - P) with a
 * per-chunk anchor R_c; appending a token and decoding it are the serving
 * loop's two halves, fused here so a token costs one kernel launch).
 *
 * With t the number of tokens already cached (0 <= t < Tcap), for every batch
 * row b and query head h (kv head h/G):
 *   P_t = carry[b,h,:] + g[b,h,:] / ln 2            (fp32, one fused rounding,
 *                                                    as wall_prefix_cumsum)
 *   o, lse = decode of q[b,h,:] at P_t over positions 0 .. t: the cached
 *            positions as wall_attn_decode scores them, plus the new token,
 *            whose decay factor exp2(P_t - P_t) is 1, so its score is
 *            scale * q . k[b,h/G,:] taken from the input directly
 *   appends: r_cache[b,t/C,h,:] = P_t if t % C == 0 (a new chunk's anchor);
 *            k_tilde[b,t,h,:] = k[b,h/G,:] * exp2(r_cache[b,t/C,h,:] - P_t)
 *            rounded to bf16 as wall_build_kv_cache rounds it;
 *            v_cache[b,t,h/G,:] = v[b,h/G,:];  carry[b,h,:] = P_t
 * After the call the cache and carry are exactly what wall_prefix_cumsum
 * (with carry_in / carry_out) and wall_build_kv_cache (t0 = t) would leave.
 * In:  q [B,HQ,K], k [B,H,K], v [B,H,V], g [B,HQ,K] (bf16: `dtype` must be
 *      WALL_BF16), sink_bias [HQ] fp32 or NULL, scale (<= 0: K^-0.5).
 * In/out: carry [B,HQ,K] fp32 (P at t-1 in; zeros for t == 0 of a fresh
 *      sequence), k_tilde [B,Tcap,HQ,K] bf16, v_cache [B,Tcap,H,V] bf16,
 *      r_cache [B,ceil(Tcap/C),HQ,K] fp32: positions [0, t) are read, row t
 *      (and chunk t/C when t starts it) written.
 * Out: o [B,HQ,V] bf16, lse [B,HQ] fp32 natural log (may be NULL).
 * Workspace: wall_decode_step_workspace(B, Tcap, H, HQ, V, C) bytes, 16-byte
 * aligned, caller-owned.  Its tail holds per-head arrival counters of the
 * split-KV partials: they must be ZERO before the first call (clear the whole
 * workspace once) and every call that returns WALL_OK and whose status
 * (wall_get_status) is WALL_OK leaves them zero again; after a device timeout
 * clear the workspace before the next call.  Calls sharing a workspace must
 * not overlap on the GPU.
 * Supported: bf16, K and V in {64, 128}, HQ/H <= 8, C a multiple of 32;
 * anything else returns WALL_ERR_UNSUPPORTED before any launch (append with
 * wall_prefix_cumsum + wall_build_kv_cache and decode with wall_attn_decode
 * instead).  Errors: WALL_ERR_INVALID_ARG for null or misaligned pointers,
 * t outside [0, Tcap), a short workspace or bad shapes.
 */
int wall_decode_step(const void* q, const void* k, const void* v, const void* g, int dtype,
                     float* carry, void* k_tilde, void* v_cache, float* r_cache,
                     const float* sink_bias, float scale, int C, int t, int B, int Tcap, int H,
                     int HQ, int K, int V, void* o, float* lse, void* workspace,
                     size_t workspace_bytes, wall_stream_t stream);

/* wall_attn_decode_chunk_workspace -- bytes of workspace wall_attn_decode_chunk
 * needs for these arguments (its path depends on dtype, K, V and C). */
size_t wall_attn_decode_chunk_workspace(int dtype, int B, int Tq, int T_kv, int H, int HQ, int K,
                                        int V, int C);

/*
 * wall_attn_decode_chunk -- Tq queries per batch row against the pre-rescaled
 * cache at once: multi-token decode and chunked prefill.  The queries are the
 * LAST Tq cached positions (bottom-right aligned causal mask, as the course
 * slides on attention masks align a short query block with a longer key
 * sequence): query row i of batch row b sits at position t_i = T_kv - Tq + i
 * and sees the cached keys 0 .. t_i.  Append the chunk's keys and values
 * first (wall_prefix_cumsum with the carry, wall_build_kv_cache with
 * t0 = T_kv - Tq); then for each (b, i, h), with c(j) = j / C,
 *   s_j = scale * sum_n q[b,i,h,n] exp2(p[b,i,h,n] - r_cache[b,c(j),h,n])
 *                  * k_tilde[b,j,h,n],       j = 0 .. t_i
 *   o[b,i,h,:] = sum_j softmax(s, sink)_j v[b,j,h/G,:],  lse = log-sum-exp
 * which is wall_attn_decode of that row with T_kv = t_i + 1 (README "Decode":
 * the pre-rescaled cache with per-chunk anchors), and equals the training
 * forward's row t_i.
 * In:  q [B,Tq,HQ,K] (`dtype`), p [B,Tq,HQ,K] fp32 (P at the queries'
 *      positions), k_tilde [B,Tcap,HQ,K] and v [B,Tcap,H,V] (`dtype`, the
 *      first T_kv positions are read), r_cache [B,ceil(Tcap/C),HQ,K] fp32,
 *      sink_bias [HQ] fp32 or NULL.  1 <= T_kv <= Tcap, 0 <= Tq <= T_kv.
 * Out: o [B,Tq,HQ,V] (`dtype`), lse [B,Tq,HQ] fp32 natural log (may be NULL).
 * Workspace: wall_attn_decode_chunk_workspace(...) bytes, 16-byte aligned,
 * caller-owned; no state is kept in it between calls.
 * Paths: bf16 with K == V in {64, 128} and C a multiple of 32 that divides
 * 128 or is a multiple of 128 runs on the tensor cores (tcgen05, one CTA per
 * 128 query rows of a (batch row, head), key tiles of 128 cached positions
 * scaled per chunk by 2^(R_I - R_c) with R_I the query block's integer
 * anchor); every other supported shape (bf16 or fp32, K and V multiples of 8
 * up to 128, HQ/H <= 32, B*Tq <= 65535) runs the split-KV decode with one
 * grid row per query.  Errors: WALL_ERR_INVALID_ARG for null or misaligned
 * pointers, bad shapes or a short workspace; WALL_ERR_UNSUPPORTED outside
 * both paths.
 */
int wall_attn_decode_chunk(const void* q, const void* v, const float* p, const void* k_tilde,
                           const float* r_cache, const float* sink_bias, float scale, int C,
                           int dtype, int B, int Tq, int T_kv, int Tcap, int H, int HQ, int K,
                           int V, void* o, float* lse, void* workspace, size_t workspace_bytes,
                           wall_stream_t stream);

/*
 * wall_get_status -- synchronizes `stream`, returns the device status word
 * (WALL_OK or WALL_ERR_TIMEOUT) and clears it.  Returns WALL_ERR_CUDA if the
 * synchronization itself fails.
 */
int wall_get_status(wall_stream_t stream);

/*
 * wall_selftest_wait_timeout -- failure-detection self test.  Launches one
 * tiny kernel that waits on an mbarrier nothing ever arrives on, through the
 * same bounded wait every kernel of the library uses (limit_us
 * microseconds, 1 .. 2,000,000).  The wait gives up, records
 * WALL_ERR_TIMEOUT in the status word and the kernel returns normally: the
 * context stays usable.  The next wall_get_status returns WALL_ERR_TIMEOUT.
 * No counterpart on the pages: it exercises this library's own error path.
 */
int wall_selftest_wait_timeout(int limit_us, wall_stream_t stream);

/*
 * Per-stage device timing, for measurement (a profiling aid with no
 * counterpart on the pages).  While enabled, every launch of a timed stage
 * is bracketed by two CUDA events recorded on the stream the stage runs on;
 * the events are the library's own and are reused.  Stages (slot: name):
 *   0 prefix_scan     the three kernels of wall_prefix_cumsum
 *   1 operands        anchored-operand preparation (fwd and bwd each)
 *   2 fwd_tc          tensor-core forward
 *   3 bwd_pre         D / sink pre-pass
 *   4 bwd_keyblock    tensor-core key-block backward (dK, dV)
 *   5 bwd_dq          tensor-core query-block backward (dq)
 *   6 bwd_finalize    dq scaling, gate-gradient summand, GQA sums
 *   7 reverse_scan    the reverse scan(s) of wall_attn_bwd
 *   8 decode          wall_attn_decode (split and merge kernels)
 *   9 cache_build     wall_build_kv_cache
 *  10 decode_step     wall_decode_step (one launch per token)
 *  11 decode_chunk    wall_attn_decode_chunk (operands and attention)
 *  12 exact_units     the CUDA-core recomputation of (sequence, head) units
 *                     beyond the anchored operands' range (fwd and bwd)
 * wall_timing_enable(1) starts recording (and clears the totals);
 * wall_timing_enable(0) stops.  Not thread-safe: one host thread at a time.
 */
#define WALL_TIMING_SLOTS 13
int wall_timing_enable(int on);

/*
 * wall_timing_enable_slots -- as wall_timing_enable, for the slots whose bit
 * is set in `mask` only (bit i = slot i; 0 stops timing), so a measurement
 * can time one stage without recording events around all the others.
 * Returns WALL_ERR_INVALID_ARG for bits past WALL_TIMING_SLOTS.
 */
int wall_timing_enable_slots(unsigned mask);

/*
 * wall_timing_read -- for slots [0, n) (n <= WALL_TIMING_SLOTS) writes the
 * number of timed launches since the last read (or enable) and their total
 * device time in milliseconds, then clears them.  Synchronizes on the
 * recorded events.  `launches` and `ms` are host arrays of n entries; `names`
 * may be NULL, else it receives n static strings.  Returns WALL_ERR_CUDA if
 * an event query fails, WALL_ERR_INVALID_ARG for a bad n or null array.
 */
int wall_timing_read(int n, const char** names, int* launches, double* ms);

#ifdef __cplusplus
}
#endif

#endif /* WALL_H */
