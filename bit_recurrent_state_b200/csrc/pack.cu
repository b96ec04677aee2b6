// State conversion between an FP32 state in key-channel order and the
// stored formats (FP32 permuted, DAMP FP16 + INT8 or INT4).  Not on the timed path:
// one CTA per head, one thread per stored row, the row kept in the thread's
// own (local) memory, deterministic rounding.
//
// Source: DAMP summary, Key Points > Implementation (a permutation per head
// places the protected channels contiguously; the low tier is INT8 after a
// Hadamard along the value axis) and Data & Methods > Quantization &
// calibration details (per-block asymmetric affine quantization with
// b = 8 or b = 4).
#include <cuda_runtime.h>
#include <cstdint>

#include "brs_device.cuh"
#include "brs_internal.h"

namespace brs {

template <int D>
__global__ void pack_kernel(const PackArgs a) {
  const int head = blockIdx.x, h = head % a.H, i = threadIdx.x;
  const int p = a.perm ? a.perm[h * D + i] : i;
  const float* src = a.S + ((size_t)head * D + p) * D;
  uint8_t* out = (uint8_t*)a.packed + (size_t)head * a.head_bytes;
  float row[D];
  for (int j = 0; j < D; ++j) row[j] = src[j];
  if (a.storage == BRS_STORE_FP32) {
    for (int j = 0; j < D; ++j) ((float*)out)[(size_t)i * D + j] = row[j];
    return;
  }
  const int nlo = D - a.k_hi, nb = D / a.block;
  const int lb = a.low_bits, rb = D * lb / 8;          // code bits, code bytes per row
  const float lv = (float)((1 << lb) - 1);             // top code
  if (i >= nlo) {
    uint16_t* f16 = (uint16_t*)(out + (size_t)nlo * rb) + (size_t)(i - nlo) * D;
    for (int j = 0; j < D; ++j) {
      const uint16_t hv = f32_to_f16(row[j]);
      if (f16_inf_or_nan(hv)) raise_flag(a.flags, isfinite(row[j]) ? BRS_FLAG_OVERFLOW : BRS_FLAG_NONFINITE);
      f16[j] = hv;
    }
    return;
  }
  if (a.hadamard) seq_fwht<D>(row, a.hscale);
  uint32_t* sz = (uint32_t*)(out + (size_t)nlo * rb + (size_t)a.k_hi * D * 2);
  uint8_t* crow = out + (size_t)i * rb;
  if (lb == 4)
    for (int j = 0; j < rb; ++j) crow[j] = 0;
  for (int bl = 0; bl < nb; ++bl) {
    const float* y = row + bl * a.block;
    float mn = y[0], mx = y[0];
    for (int j = 1; j < a.block; ++j) {
      if (y[j] < mn || (y[j] == mn && signbit(y[j]))) mn = y[j];
      if (y[j] > mx || (y[j] == mx && !signbit(y[j]))) mx = y[j];
    }
    if (!isfinite(mn) || !isfinite(mx)) raise_flag(a.flags, BRS_FLAG_NONFINITE);
    const uint16_t sh = f32_to_f16(__fdiv_rn(__fsub_rn(mx, mn), lv));
    const uint16_t zh = f32_to_f16(mn);
    if (f16_inf_or_nan(sh) || f16_inf_or_nan(zh)) raise_flag(a.flags, BRS_FLAG_OVERFLOW);
    const float s = f16_to_f32(sh), z = f16_to_f32(zh);
    const float rcp = (s == 0.0f) ? 0.0f : __frcp_rn(s);
    for (int j = 0; j < a.block; ++j) {
      float c = 0.0f;
      if (s != 0.0f) c = fminf(fmaxf(rintf(__fmul_rn(__fsub_rn(y[j], z), rcp)), 0.0f), lv);
      const int e = bl * a.block + j;
      if (lb == 8) crow[e] = (uint8_t)(int)c;
      else crow[e / 2] |= (uint8_t)((int)c << (4 * (e & 1)));
    }
    sz[i * nb + bl] = (uint32_t)sh | ((uint32_t)zh << 16);
  }
}

template <int D>
__global__ void unpack_kernel(const PackArgs a, float* S, const void* packed) {
  const int head = blockIdx.x, h = head % a.H, i = threadIdx.x;
  const int p = a.perm ? a.perm[h * D + i] : i;
  float* dst = S + ((size_t)head * D + p) * D;
  const uint8_t* in = (const uint8_t*)packed + (size_t)head * a.head_bytes;
  float row[D];
  if (a.storage == BRS_STORE_FP32) {
    for (int j = 0; j < D; ++j) dst[j] = ((const float*)in)[(size_t)i * D + j];
    return;
  }
  const int nlo = D - a.k_hi, nb = D / a.block;
  const int lb = a.low_bits, rb = D * lb / 8;
  if (i >= nlo) {
    const uint16_t* f16 = (const uint16_t*)(in + (size_t)nlo * rb) + (size_t)(i - nlo) * D;
    for (int j = 0; j < D; ++j) dst[j] = f16_to_f32(f16[j]);
    return;
  }
  const uint32_t* sz = (const uint32_t*)(in + (size_t)nlo * rb + (size_t)a.k_hi * D * 2);
  const uint8_t* crow = in + (size_t)i * rb;
  for (int j = 0; j < D; ++j) {
    const uint32_t v = sz[i * nb + j / a.block];
    const int code = (lb == 8) ? crow[j] : (crow[j / 2] >> (4 * (j & 1))) & 15;
    row[j] = __fmaf_rn((float)code, f16_to_f32((uint16_t)(v & 0xffffu)), f16_to_f32((uint16_t)(v >> 16)));
  }
  if (a.hadamard) seq_fwht<D>(row, a.hscale);
  for (int j = 0; j < D; ++j) dst[j] = row[j];
}

cudaError_t launch_pack(const PackArgs& a, cudaStream_t st) {
  const dim3 grid(a.B * a.H), block(a.d);
  switch (a.d) {
    case 32: pack_kernel<32><<<grid, block, 0, st>>>(a); break;
    case 64: pack_kernel<64><<<grid, block, 0, st>>>(a); break;
    case 128: pack_kernel<128><<<grid, block, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_unpack(const PackArgs& a, float* S, const void* packed, cudaStream_t st) {
  const dim3 grid(a.B * a.H), block(a.d);
  switch (a.d) {
    case 32: unpack_kernel<32><<<grid, block, 0, st>>>(a, S, packed); break;
    case 64: unpack_kernel<64><<<grid, block, 0, st>>>(a, S, packed); break;
    case 128: unpack_kernel<128><<<grid, block, 0, st>>>(a, S, packed); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace brs
