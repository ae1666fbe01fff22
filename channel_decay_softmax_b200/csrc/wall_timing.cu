// wall_timing.cu -- per-stage device timing of this library's launches.
//
// Off unless wall_timing_enable(1): then each timed stage records a CUDA
// event before and after its launches, on the launch stream, and
// wall_timing_read sums the elapsed times per stage.  Events come from a
// per-slot pool that grows on demand and is reused after each read.
#include <cuda_runtime.h>

#include <vector>

#include "wall.h"
#include "wall_internal.h"

namespace wall {
namespace {

struct Slot {
  std::vector<cudaEvent_t> ev;  // pairs: begin, end
  int used = 0;                 // events recorded since the last read
};

unsigned g_mask = 0;  // timed slots
Slot g_slot[WALL_TIMING_SLOTS];
const char* const kNames[WALL_TIMING_SLOTS] = {
    "prefix_scan", "operands", "fwd_tc", "bwd_pre", "bwd_keyblock",
    "bwd_dq", "bwd_finalize", "reverse_scan", "decode", "cache_build",
    "decode_step", "decode_chunk", "exact_units"};

}  // namespace

void timing_mark(int slot, cudaStream_t stream) {
  if (slot < 0 || slot >= WALL_TIMING_SLOTS || !((g_mask >> slot) & 1u)) return;
  Slot& s = g_slot[slot];
  if (s.used == (int)s.ev.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return;
    s.ev.push_back(e);
  }
  cudaEventRecord(s.ev[s.used++], stream);
}

}  // namespace wall

extern "C" int wall_timing_enable(int on) {
  using namespace wall;
  g_mask = on != 0 ? (1u << WALL_TIMING_SLOTS) - 1u : 0u;
  for (auto& s : g_slot) s.used = 0;
  return WALL_OK;
}

extern "C" int wall_timing_enable_slots(unsigned mask) {
  using namespace wall;
  if (mask >> WALL_TIMING_SLOTS) return WALL_ERR_INVALID_ARG;
  g_mask = mask;
  for (auto& s : g_slot) s.used = 0;
  return WALL_OK;
}

extern "C" int wall_timing_read(int n, const char** names, int* launches, double* ms) {
  using namespace wall;
  if (n < 0 || n > WALL_TIMING_SLOTS || (n > 0 && (launches == nullptr || ms == nullptr)))
    return WALL_ERR_INVALID_ARG;
  int rc = WALL_OK;
  for (int i = 0; i < n; ++i) {
    Slot& s = g_slot[i];
    double tot = 0.0;
    const int pairs = s.used / 2;
    for (int k = 0; k < pairs; ++k) {
      float t = 0.f;
      if (cudaEventSynchronize(s.ev[2 * k + 1]) != cudaSuccess ||
          cudaEventElapsedTime(&t, s.ev[2 * k], s.ev[2 * k + 1]) != cudaSuccess) {
        rc = WALL_ERR_CUDA;
        break;
      }
      tot += t;
    }
    launches[i] = pairs;
    ms[i] = tot;
    if (names) names[i] = kNames[i];
    s.used = 0;
  }
  return rc;
}
