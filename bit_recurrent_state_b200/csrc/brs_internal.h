// Internal launch interfaces between the host ABI (brs_api.cu) and the
// kernels.  Not part of the public ABI.
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "brs.h"

namespace brs {

struct DecodeArgs {
  int B, H, Hk, k_hi, block, decay_per_key, mode;
  uint64_t seed;
  int64_t step;
  size_t head_bytes;
  float hscale;                  // float nearest 1/sqrt(d)
  const void* packed_in;
  void* packed_out;
  void* aux;
  const int16_t* perm;
  const uint16_t *q, *k, *v;
  const float *beta, *decay;
  float* o;
  uint32_t* flags;
};

cudaError_t launch_decode(const DecodeArgs& a, int d, int store, bool had, cudaStream_t st);
bool decode_supported(int d, int block, int k_hi);

struct PackArgs {
  int B, H, d, storage, k_hi, block, hadamard;
  size_t head_bytes;
  float hscale;
  const float* S;                // [B][H][d][d] key-channel order
  const int16_t* perm;
  void* packed;
  uint32_t* flags;
};

cudaError_t launch_pack(const PackArgs& a, cudaStream_t st);
cudaError_t launch_unpack(const PackArgs& a, float* S_out, const void* packed, cudaStream_t st);

void set_last_error(const char* msg);

}  // namespace brs
