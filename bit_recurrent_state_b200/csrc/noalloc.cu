// Allocation-free variant of brs_decode_step, and the read-out of its flags.
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
// should therefore be made before any stream capture, and the device must
// not be reset (cudaDeviceReset) while the library stays loaded, since a
// reset invalidates the cached address.  All calls share the one array:
// calls that overlap on the GPU race on it.  Its first word collects the
// device flags of every call (it starts at zero when the library is loaded);
// brs_fetch_errors_noalloc reads and clears it.  The rest of the scratch (the
// per-row costs of variable-width decode) is written by each call before it
// is read, so nothing else needs clearing.
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

brs_status address_failed(const char* who, cudaError_t e) {
  char msg[256];
  snprintf(msg, sizeof(msg), "%s: cudaGetSymbolAddress: %s", who, cudaGetErrorString(e));
  brs::set_last_error(msg);
  return BRS_ECUDA;
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
  if (ws > kScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "brs_decode_step_noalloc: the layout needs %zu bytes of scratch, the static array holds %zu",
             ws, kScratchBytes);
    brs::set_last_error(msg);
    return BRS_EINVAL;
  }
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) return address_failed("brs_decode_step_noalloc", e);
  return brs_decode_step(L, wb, step, packed_in, packed_out, aux, stats, scratch, perm, q, k, v,
                         beta, decay, o, stream);
}

extern "C" brs_status brs_fetch_errors_noalloc(uint32_t* flags_out, void* stream) {
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) return address_failed("brs_fetch_errors_noalloc", e);
  return brs_fetch_errors(scratch, flags_out, stream);
}
