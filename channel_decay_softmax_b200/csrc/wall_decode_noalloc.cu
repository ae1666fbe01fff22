// wall_decode_noalloc.cu -- a decode entry point that allocates nothing.
//
// wall_attn_decode needs a small workspace for its split-KV partials, which
// the caller allocates.  Some callers cannot: code that runs while a CUDA
// graph is being captured and must not allocate, serving loops whose memory
// is planned once up front, and bindings from runtimes that have no handle on
// a device allocator.  This entry point runs the same kernels with the
// partials in a fixed scratch array that lives in the library's own device
// memory, so it needs nothing but the inputs and outputs.
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

// 4 MiB of split partials: B * HQ * splits * (V + 2) floats at most.
constexpr size_t kScratchFloats = size_t(1) << 20;

// Every GPU that loads the library holds this array until the process exits.
__device__ __align__(256) float g_decode_scratch[kScratchFloats];

// The array's device address on the current device.  In host code the name
// g_decode_scratch is only a host-side stand-in, so the address is asked for
// once per device, with that device current, and kept.
float* scratch_on_current_device() {
  static float* addr[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return nullptr;
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<float*>(p);
  }
  return addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace wall

extern "C" int wall_attn_decode_noalloc(const void* q, const void* v, const float* p_curr,
                                        const void* k_tilde, const float* r_cache,
                                        const float* sink_bias, float scale, int C, int dtype,
                                        int B, int T_kv, int Tcap, int H, int HQ, int K, int V,
                                        void* o, float* lse, wall_stream_t stream) {
  using namespace wall;
  const TraceRange trace(__func__);
  if (dtype != WALL_BF16 && dtype != WALL_FP32) return WALL_ERR_INVALID_ARG;
  if (B < 0 || T_kv < 1 || Tcap < T_kv || H < 1 || HQ < 1 || HQ % H != 0 || C < 1)
    return WALL_ERR_INVALID_ARG;
  if (K < 8 || K > 128 || K % 8 != 0 || V < 8 || V > 128 || V % 8 != 0 || HQ / H > 32)
    return WALL_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535) return WALL_ERR_UNSUPPORTED;
  if (B == 0) return WALL_OK;
  const void* need_ptrs[] = {q, v, p_curr, k_tilde, r_cache, o};
  for (const void* ptr : need_ptrs)
    if (ptr == nullptr || !aligned16(ptr)) return WALL_ERR_INVALID_ARG;
  if (!aligned16(sink_bias) || !aligned16(lse)) return WALL_ERR_INVALID_ARG;
  const int S = decode_splits(B, T_kv, H, C);
  // beyond the fixed scratch: the caller must use wall_attn_decode
  if ((size_t)B * HQ * S * (V + 2) > kScratchFloats) return WALL_ERR_UNSUPPORTED;
  float* scratch = scratch_on_current_device();
  if (scratch == nullptr) return WALL_ERR_CUDA;
  // every split writes its whole partial (o, max, sum), or an empty one if a
  // bounded wait gave up, so nothing left in the scratch by an earlier call
  // is read and nothing needs clearing
  const float sc = scale > 0.f ? scale : 1.f / sqrtf((float)K);
  return attn_decode(q, v, p_curr, k_tilde, r_cache, sink_bias, sc, C, dtype, B, T_kv, Tcap, H, HQ,
                     K, V, o, lse, scratch, S, reinterpret_cast<cudaStream_t>(stream));
}
