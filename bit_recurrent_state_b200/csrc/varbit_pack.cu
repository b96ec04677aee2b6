// Conversion between an FP32 state and the variable-width stored format
// ("Low-Bit Recurrent States in Hybrid Language Models", Levels and storage:
// per-row symmetric grid with a fitted clip factor, FP16 step, width map,
// prefix-sum row offsets).  Setup path, not timed: one thread per row,
// deterministic (nearest) rounding.
#include <cuda_runtime.h>
#include <cstdint>

#include "brs_device.cuh"
#include "brs_internal.h"

namespace brs {

static size_t r256(size_t x) { return (x + 255) / 256 * 256; }

VbSections varbit_sections(int B, int H, int d, double avg_bits) {
  VbSections s;
  const size_t rows = (size_t)H * d;
  s.payload_per_seq = (size_t)((double)(d / 8) * avg_bits * (double)rows);
  s.off_scale = r256(s.payload_per_seq * (size_t)B);
  s.off_width = s.off_scale + r256(rows * (size_t)B * 2);
  s.off_offsets = s.off_width + r256(rows * (size_t)B);
  s.total = s.off_offsets + r256((rows + 1) * (size_t)B * 4);
  return s;
}

// widths and row offsets of every sequence (one thread per sequence)
__global__ void varbit_layout_kernel(const VbPackArgs a) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= a.B) return;
  const int rows = a.H * a.d;
  uint8_t* packed = (uint8_t*)a.packed;
  uint8_t* wd = packed + a.sec.off_width + (size_t)b * rows;
  uint32_t* of = (uint32_t*)(packed + a.sec.off_offsets) + (size_t)b * (rows + 1);
  uint32_t off = 0;
  for (int r = 0; r < rows; ++r) {
    const int bw = a.widths ? a.widths[(size_t)b * rows + r] : (int)rint(a.avg_bits);
    wd[r] = (uint8_t)bw;
    of[r] = off;
    off += (uint32_t)(a.d / 8) * (uint32_t)bw;
  }
  of[rows] = off;
}

template <int D>
__global__ void varbit_pack_kernel(const VbPackArgs a) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;       // b*H*D + h*D + i
  const int rows = a.H * D;
  if (row >= a.B * rows) return;
  const int b = row / rows, r = row % rows;
  uint8_t* packed = (uint8_t*)a.packed;
  const int bw = packed[a.sec.off_width + (size_t)b * rows + r];
  const uint32_t off = ((const uint32_t*)(packed + a.sec.off_offsets))[(size_t)b * (rows + 1) + r];
  const int n = (1 << (bw - 1)) - 1;
  const float fn = (float)n;
  const float* x = a.S + (size_t)row * D;
  float R = 0.0f;
  for (int j = 0; j < D; ++j) R = fmaxf(R, fabsf(x[j]));
  uint16_t best_bits = 0;
  float best_step = 0.0f;
  if (bw == 1) {
    // one bit: the sign times the row's mean absolute value (FP16), the
    // magnitudes summed in element order
    float sum = 0.0f;
    for (int j = 0; j < D; ++j) sum = __fadd_rn(sum, fabsf(x[j]));
    best_bits = f32_to_f16(__fmul_rn(sum, 1.0f / (float)D));
    best_step = f16_to_f32(best_bits);
    if (!isfinite(best_step)) raise_flag(a.flags, BRS_FLAG_OVERFLOW);
  } else if (R > 0.0f) {
    float bestE = 0.0f;
    int best = -1;
    for (int m = 0; m < 16; ++m) {
      float step, inv;
      uint16_t bits;
      bool valid;
      varbit_candidate(m, R, n, step, inv, bits, valid);
      if (!valid) continue;
      float E = 0.0f;
      for (int j = 0; j < D; ++j) {
        const float res = __fsub_rn(x[j], __fmul_rn(step, varbit_nearest(x[j], inv, fn)));
        E = __fmaf_rn(res, res, E);
      }
      if (best < 0 || E < bestE) { best = m; bestE = E; best_bits = bits; best_step = step; }
    }
    if (best < 0) { raise_flag(a.flags, BRS_FLAG_OVERFLOW); best_bits = 0x7c00u; best_step = 0.0f; }
  }
  ((uint16_t*)(packed + a.sec.off_scale))[(size_t)b * rows + r] = best_bits;
  const float inv = (best_step != 0.0f && isfinite(best_step)) ? __frcp_rn(best_step) : 0.0f;
  uint32_t words[64];                                          // d * 16 bits at most
  for (int k = 0; k < 4 * bw; ++k) words[k] = 0u;
  for (int j = 0; j < D; ++j) {
    const uint32_t u = (bw == 1) ? (x[j] >= 0.0f ? 1u : 0u) : (uint32_t)((int)varbit_nearest(x[j], inv, fn) + n);
    const int bit = j * bw;
    words[bit >> 5] |= u << (bit & 31);
    if ((bit & 31) + bw > 32) words[(bit >> 5) + 1] |= u >> (32 - (bit & 31));
  }
  // a width map that does not sum to the budget would run past the payload
  if ((size_t)off + (size_t)D * bw / 8 > a.sec.payload_per_seq) {
    raise_flag(a.flags, BRS_FLAG_OVERFLOW);
    return;
  }
  uint32_t* dst = (uint32_t*)(packed + (size_t)b * a.sec.payload_per_seq + off);
  for (int k = 0; k < D * bw / 32; ++k) dst[k] = words[k];
}

template <int D>
__global__ void varbit_unpack_kernel(const VbPackArgs a, const void* packed_v, float* S) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  const int rows = a.H * D;
  if (row >= a.B * rows) return;
  const int b = row / rows, r = row % rows;
  const uint8_t* packed = (const uint8_t*)packed_v;
  const int bw = packed[a.sec.off_width + (size_t)b * rows + r];
  const uint32_t off = ((const uint32_t*)(packed + a.sec.off_offsets))[(size_t)b * (rows + 1) + r];
  const float step = f16_to_f32(((const uint16_t*)(packed + a.sec.off_scale))[(size_t)b * rows + r]);
  const int n = (1 << (bw - 1)) - 1;
  const uint32_t* src = (const uint32_t*)(packed + (size_t)b * a.sec.payload_per_seq + off);
  for (int j = 0; j < D; ++j) {
    const int bit = j * bw;
    uint32_t u = src[bit >> 5] >> (bit & 31);
    if ((bit & 31) + bw > 32) u |= src[(bit >> 5) + 1] << (32 - (bit & 31));
    u &= (1u << bw) - 1u;
    const int lv = (bw == 1) ? 2 * (int)u - 1 : (int)u - n;     // one bit: 2u - 1
    S[(size_t)row * D + j] = __fmul_rn((float)lv, step);
  }
}

cudaError_t launch_varbit_pack(const VbPackArgs& a, cudaStream_t st) {
  varbit_layout_kernel<<<(a.B + 63) / 64, 64, 0, st>>>(a);
  const int rows = a.B * a.H * a.d;
  switch (a.d) {
    case 32: varbit_pack_kernel<32><<<(rows + 127) / 128, 128, 0, st>>>(a); break;
    case 64: varbit_pack_kernel<64><<<(rows + 127) / 128, 128, 0, st>>>(a); break;
    case 128: varbit_pack_kernel<128><<<(rows + 127) / 128, 128, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_varbit_unpack(const VbPackArgs& a, const void* packed, float* S, cudaStream_t st) {
  const int rows = a.B * a.H * a.d;
  switch (a.d) {
    case 32: varbit_unpack_kernel<32><<<(rows + 127) / 128, 128, 0, st>>>(a, packed, S); break;
    case 64: varbit_unpack_kernel<64><<<(rows + 127) / 128, 128, 0, st>>>(a, packed, S); break;
    case 128: varbit_unpack_kernel<128><<<(rows + 127) / 128, 128, 0, st>>>(a, packed, S); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace brs
