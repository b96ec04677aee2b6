// Device helpers shared by the library's kernels: binary16/bfloat16
// conversion, Philox4x32-10, the per-row Hadamard butterflies across the
// threads of a row group, and the device flag word.
#pragma once
#include <cuda_fp16.h>
#include <cstdint>

#include "brs.h"

namespace brs {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
__device__ __forceinline__ float f16_to_f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }
__device__ __forceinline__ uint16_t f32_to_f16(float x) { return __half_as_ushort(__float2half_rn(x)); }
__device__ __forceinline__ bool f16_inf_or_nan(uint16_t h) { return ((h >> 10) & 31u) == 31u; }

__device__ __forceinline__ void raise_flag(uint32_t* flags, uint32_t bit) {
  if (flags) atomicOr(flags, bit);
}

// Philox4x32-10 (Salmon et al., SC'11): ten rounds, key bumped by the Weyl
// constants between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k.x += 0x9E3779B9u;
      k.y += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
  }
  return c;
}

// Stochastic choice between the two levels around t: floor(t) + 1 with
// probability frac(t), from 24 uniform bits.
__device__ __forceinline__ float sr_round(float t, uint32_t r24) {
  const float fl = floorf(t);
  const float fr = __fsub_rn(t, fl);
  return ((float)r24 < __fmul_rn(fr, 16777216.0f)) ? __fadd_rn(fl, 1.0f) : fl;
}

// Butterfly stages of the Sylvester Hadamard over one row of D values held
// as 4 consecutive values per thread by the D/4 threads of a row group
// (thread cb holds columns 4cb..4cb+3; the groups are aligned runs of D/4
// lanes).  Stages h = 1, 2 are thread-local, h >= 4 exchange with lane
// cb ^ (h/4).  Each output is the same single add or subtract as in the
// sequential transform, so the result does not depend on the layout.
// Must be called by every lane of the warp (full-mask shuffles).
template <int D>
__device__ __forceinline__ void row_fwht4(float (&x)[4], int cb, float scale) {
  float a0 = __fadd_rn(x[0], x[1]), a1 = __fsub_rn(x[0], x[1]);
  float a2 = __fadd_rn(x[2], x[3]), a3 = __fsub_rn(x[2], x[3]);
  x[0] = __fadd_rn(a0, a2);
  x[2] = __fsub_rn(a0, a2);
  x[1] = __fadd_rn(a1, a3);
  x[3] = __fsub_rn(a1, a3);
#pragma unroll
  for (int m = 1; m < D / 4; m <<= 1) {
    const bool hi = (cb & m) != 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float other = __shfl_xor_sync(0xffffffffu, x[c], m);
      x[c] = hi ? __fsub_rn(other, x[c]) : __fadd_rn(x[c], other);
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) x[c] = __fmul_rn(x[c], scale);
}

}  // namespace brs
