// Allocation-free variant of brs_decode_step.
//
// Who needs it: callers that must not allocate device memory themselves,
// for example a host framework whose own allocator owns every byte of the
// device and forbids side allocations, or a serving loop with a fixed memory
// budget and no allocation on its per-token path.  Those callers still
// provide the state, inputs and outputs, but not the scratch (workspace)
// buffer the regular entry point takes.
//
// The scratch lives in a file-scope device array of kScratchBytes bytes,
// reserved once per device when the library is loaded and held until the
// process exits.  Host code cannot use the array's name as a device address,
// so the first call on each device looks the address up with
// cudaGetSymbolAddress (that device current) and caches it; that first call
// should therefore be made before any stream capture.  All calls share the
// one array: calls that overlap on the GPU race on it, and each call clears
// the part it uses (the device flag word) before its kernel runs.  Flags the
// kernel raises stay in the array and are not reported by this entry.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "brs.h"
#include "brs_internal.h"

namespace {

constexpr size_t kScratchBytes = 4096;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// device address of g_scratch on the current device (looked up once)
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" brs_status brs_decode_step_noalloc(const brs_layout* L, const brs_writeback* wb,
                                              int64_t step, const void* packed_in,
                                              void* packed_out, void* aux, void* stats,
                                              const int16_t* perm, const uint16_t* q,
                                              const uint16_t* k, const uint16_t* v,
                                              const float* beta, const float* decay, float* o,
                                              void* stream) {
  size_t ws = 0;
  if (brs_state_bytes(L, nullptr, nullptr, &ws) == 0) return BRS_EINVAL;  // message already set
  char msg[256];
  if (ws > kScratchBytes) {
    snprintf(msg, sizeof(msg),
             "brs_decode_step_noalloc: the layout needs %zu bytes of scratch, the static array holds %zu",
             ws, kScratchBytes);
    brs::set_last_error(msg);
    return BRS_EINVAL;
  }
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "brs_decode_step_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    brs::set_last_error(msg);
    return BRS_ECUDA;
  }
  e = cudaMemsetAsync(scratch, 0, ws, (cudaStream_t)stream);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "brs_decode_step_noalloc: clearing the scratch: %s", cudaGetErrorString(e));
    brs::set_last_error(msg);
    return BRS_ECUDA;
  }
  return brs_decode_step(L, wb, step, packed_in, packed_out, aux, stats, scratch, perm, q, k, v,
                         beta, decay, o, stream);
}
