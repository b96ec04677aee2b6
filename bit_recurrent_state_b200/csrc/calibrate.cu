// Protected-row selection on the GPU (DAMP summary, Key Points > Risk
// scoring and selection, and Data & Methods > Calibration): run the FP32
// recurrence on a calibration batch (the FP32-storage decode step, one
// launch per token), sample the state every `every` tokens, and score each
// key row u of each head by
//   E_u = mean over samples of the squared error energy of the row under
//         Hadamard-INT8 quantize -> dequantize (nearest, the stored grid),
//   a_eff,u = exp(mean log a_u),  P_u = 1 / max(1 - a_eff,u^2, tau),
//   C_u = E_u P_u;
// the k_hi largest scores of a head are protected (ties to the lower
// index).  The permutation lists the unprotected rows, then the protected
// ones, each group ascending: the protected rows sit contiguously at the
// end of the stored order.
//
// Setup work, not on the timed path.  The sums are taken in FP64 in a fixed
// order: per row over the row's values in order, per (h, u) over the
// calibration sequences in order and within each over the samples in time
// order (and likewise for the log-decay sum over sequences and tokens).
#include <cuda_runtime.h>
#include <cstdint>

#include "brs_device.cuh"
#include "brs_internal.h"

namespace brs {

// squared quantization error energy of every row of every calibration
// state: one CTA per (sequence, head), one thread per row
template <int D>
__global__ void calib_sample_kernel(const CalibArgs a) {
  const int head = blockIdx.x, i = threadIdx.x;
  const float* src = a.S + ((size_t)head * D + i) * D;
  float row[D];
  for (int j = 0; j < D; ++j) row[j] = src[j];
  if (a.hadamard) seq_fwht<D>(row, a.hscale);
  double err = 0.0;
  const int nb = D / a.block;
  for (int bl = 0; bl < nb; ++bl) {
    const float* y = row + bl * a.block;
    float mn = y[0], mx = y[0];
    for (int j = 1; j < a.block; ++j) {
      if (y[j] < mn || (y[j] == mn && signbit(y[j]))) mn = y[j];
      if (y[j] > mx || (y[j] == mx && !signbit(y[j]))) mx = y[j];
    }
    if (!isfinite(mn) || !isfinite(mx)) raise_flag(a.flags, BRS_FLAG_NONFINITE);
    const float s = f16_to_f32(f32_to_f16(__fdiv_rn(__fsub_rn(mx, mn), a.levels)));
    const float z = f16_to_f32(f32_to_f16(mn));
    const float rcp = (s == 0.0f) ? 0.0f : __frcp_rn(s);
    for (int j = 0; j < a.block; ++j) {
      float c = 0.0f;
      if (s != 0.0f) c = fminf(fmaxf(rintf(__fmul_rn(__fsub_rn(y[j], z), rcp)), 0.0f), a.levels);
      const double e = (double)y[j] - (double)__fmaf_rn(c, s, z);
      err = __dadd_rn(err, __dmul_rn(e, e));
    }
  }
  a.err[((size_t)a.sample * a.B * a.H + head) * D + i] = err;
}

// C_u per (head, row): one thread each
__global__ void calib_score_kernel(const CalibArgs a) {
  const int id = blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= a.H * a.d) return;
  const int h = id / a.d, u = id - h * a.d;
  double E = 0.0, sl = 0.0;
  for (int b = 0; b < a.B; ++b) {
    for (int s = 0; s < a.nsamp; ++s) E = __dadd_rn(E, a.err[(((size_t)s * a.B + b) * a.H + h) * a.d + u]);
    for (int t = 0; t < a.T; ++t) {
      const size_t bh = ((size_t)t * a.B + b) * a.H + h;
      const float av = a.decay_per_key ? a.decay[bh * a.d + u] : a.decay[bh];
      sl = __dadd_rn(sl, log((double)av));
    }
  }
  const double ns = (double)a.B * (double)a.nsamp, nt = (double)a.B * (double)a.T;
  const double aeff = exp(__ddiv_rn(sl, nt));
  double den = __dadd_rn(1.0, -__dmul_rn(aeff, aeff));
  if (den < a.tau) den = a.tau;
  a.score[id] = __dmul_rn(__ddiv_rn(E, ns), __ddiv_rn(1.0, den));
}

// the k_hi largest scores of head blockIdx.x (ties to the lower index),
// then the permutation: unprotected rows ascending, protected ascending
__global__ void calib_select_kernel(const CalibArgs a) {
  if (threadIdx.x != 0) return;
  const int h = blockIdx.x, d = a.d;
  const double* sc = a.score + (size_t)h * d;
  uint32_t prot[4] = {0u, 0u, 0u, 0u};             // d <= 128 bits
  for (int c = 0; c < a.k_hi; ++c) {
    int pick = -1;
    for (int i = 0; i < d; ++i)
      if (!((prot[i >> 5] >> (i & 31)) & 1u) && (pick < 0 || sc[i] > sc[pick])) pick = i;
    prot[pick >> 5] |= 1u << (pick & 31);
  }
  int n = 0;
  int16_t* out = a.perm + (size_t)h * d;
  for (int i = 0; i < d; ++i)
    if (!((prot[i >> 5] >> (i & 31)) & 1u)) out[n++] = (int16_t)i;
  for (int i = 0; i < d; ++i)
    if ((prot[i >> 5] >> (i & 31)) & 1u) out[n++] = (int16_t)i;
}

cudaError_t launch_calib_sample(const CalibArgs& a, cudaStream_t st) {
  const dim3 grid(a.B * a.H), block(a.d);
  switch (a.d) {
    case 32: calib_sample_kernel<32><<<grid, block, 0, st>>>(a); break;
    case 64: calib_sample_kernel<64><<<grid, block, 0, st>>>(a); break;
    case 128: calib_sample_kernel<128><<<grid, block, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_calib_finish(const CalibArgs& a, cudaStream_t st) {
  const int n = a.H * a.d;
  calib_score_kernel<<<(n + 127) / 128, 128, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  calib_select_kernel<<<a.H, 32, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace brs
