// Decode step for FP32 and DAMP storage: one token for every (sequence,
// head).  One CTA per head; 2*D threads; thread t owns the 4 consecutive
// columns 4*(t % (D/4)) .. +3 of the R = D/8 consecutive stored rows
// R*(t / (D/4)) .. +R-1, so the D x D FP32 state of the head lives in
// registers for the whole step and every state byte crosses HBM once in
// and once out.
//
// Sources: DAMP summary, Key Points > Implementation (fused executor:
// reconstruct the INT8 channels, update in FP32, re-quantize, write back;
// static permutation with the protected channels contiguous); "Low-Bit
// Recurrent States in Hybrid Language Models", Accumulated readout error
// (outputs precede quantization) and Protocol (quantized and dequantized
// before reuse).
//
// Sums over key rows are fmaf chains over stored rows 0..D-1 in order: the
// 8 row groups pass the running column sums to each other through shared
// memory, one group at a time.
//
// With the Hadamard enabled the update runs in the Hadamard basis: the INT8
// rows are used as stored (already rotated), the protected FP16 rows and v
// are rotated in, o and the FP16 rows are rotated out.
#include <cuda_runtime.h>
#include <cstdint>

#include "brs_device.cuh"
#include "brs_internal.h"

namespace brs {

template <int D, int STORE, bool ROT>
__global__ void __launch_bounds__(2 * D) decode_kernel(const DecodeArgs a) {
  constexpr int NT = 2 * D;
  constexpr int LPR = D / 4;   // threads per row
  constexpr int R = D / 8;     // rows per thread
  static_assert(NT % 32 == 0, "whole warps");

  __shared__ float kk[D], qq[D], aa[D], vv[D], ww[D];
  __shared__ float4 carry[LPR];

  const int t = threadIdx.x;
  const int cb = t % LPR, rb = t / LPR;
  const int row0 = rb * R, col0 = 4 * cb;
  const int head = blockIdx.x;
  const int b = head / a.H, h = head - b * a.H;
  const int kh = h * a.Hk / a.H;
  const int nlo = D - a.k_hi;  // INT8 rows are stored rows 0..nlo-1

  // ---- gather this token's inputs in stored row order
  if (t < D) {
    const int p = a.perm ? a.perm[h * D + t] : t;
    const size_t qk = ((size_t)b * a.Hk + kh) * D;
    kk[t] = bf16_to_f32(a.k[qk + p]);
    qq[t] = bf16_to_f32(a.q[qk + p]);
    aa[t] = a.decay_per_key ? a.decay[(size_t)head * D + p] : a.decay[head];
    vv[t] = bf16_to_f32(a.v[(size_t)head * D + t]);
  }
  const float beta = a.beta[head];

  // ---- load the head into registers
  float x[R][4];
  const uint8_t* hin = (const uint8_t*)a.packed_in + (size_t)head * a.head_bytes;
  if constexpr (STORE == BRS_STORE_FP32) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float4 f = *(const float4*)(hin + ((size_t)(row0 + r) * D + col0) * 4);
      x[r][0] = f.x; x[r][1] = f.y; x[r][2] = f.z; x[r][3] = f.w;
    }
  } else {
    const int nb = D / a.block;
    const uint8_t* f16base = hin + (size_t)nlo * D;
    const uint32_t* szbase = (const uint32_t*)(hin + (size_t)nlo * D + (size_t)a.k_hi * D * 2);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = row0 + r;
      if (i < nlo) {
        const uint32_t c4 = *(const uint32_t*)(hin + (size_t)i * D + col0);
        const uint32_t sz = szbase[i * nb + col0 / a.block];
        const float s = f16_to_f32((uint16_t)(sz & 0xffffu));
        const float z = f16_to_f32((uint16_t)(sz >> 16));
#pragma unroll
        for (int c = 0; c < 4; ++c) x[r][c] = __fmaf_rn(__uint2float_rn((c4 >> (8 * c)) & 0xffu), s, z);
      } else {
        const uint2 hv = *(const uint2*)(f16base + ((size_t)(i - nlo) * D + col0) * 2);
        x[r][0] = f16_to_f32((uint16_t)(hv.x & 0xffffu));
        x[r][1] = f16_to_f32((uint16_t)(hv.x >> 16));
        x[r][2] = f16_to_f32((uint16_t)(hv.y & 0xffffu));
        x[r][3] = f16_to_f32((uint16_t)(hv.y >> 16));
      }
    }
  }
  __syncthreads();  // kk/qq/aa/vv visible

  if constexpr (ROT) {
    // protected rows to the Hadamard basis (row groups are warp-aligned
    // runs of lanes; loop bounds are kept warp-uniform for the shuffles)
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const bool mine = (row0 + r) >= nlo;
      if (__any_sync(0xffffffffu, mine)) {
        float y[4] = {x[r][0], x[r][1], x[r][2], x[r][3]};
        row_fwht4<D>(y, cb, a.hscale);
        if (mine) {
#pragma unroll
          for (int c = 0; c < 4; ++c) x[r][c] = y[c];
        }
      }
    }
    // v to the Hadamard basis: warp 0, butterflies on shared memory
    if (t < 32) {
      for (int hs = 1; hs < D; hs <<= 1) {
        for (int p = t; p < D / 2; p += 32) {
          const int i = (p / hs) * 2 * hs + (p % hs);
          const float u0 = vv[i], u1 = vv[i + hs];
          vv[i] = __fadd_rn(u0, u1);
          vv[i + hs] = __fsub_rn(u0, u1);
        }
        __syncwarp();
      }
      for (int j = t; j < D; j += 32) vv[j] = __fmul_rn(vv[j], a.hscale);
    }
  }

  // ---- decay: S <- Diag(a) S
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const float ar = aa[row0 + r];
#pragma unroll
    for (int c = 0; c < 4; ++c) x[r][c] = __fmul_rn(ar, x[r][c]);
  }

  // ---- u = S^T k, fmaf chain over stored rows 0..D-1
  for (int s = 0; s < 8; ++s) {
    if (rb == s) {
      float4 acc = s ? carry[cb] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float kv = kk[row0 + r];
        acc.x = __fmaf_rn(kv, x[r][0], acc.x);
        acc.y = __fmaf_rn(kv, x[r][1], acc.y);
        acc.z = __fmaf_rn(kv, x[r][2], acc.z);
        acc.w = __fmaf_rn(kv, x[r][3], acc.w);
      }
      carry[cb] = acc;
    }
    __syncthreads();
  }
  // w = beta (v - u)
  if (t < D) {
    const float u = ((const float*)carry)[t];
    if (!isfinite(u)) raise_flag(a.flags, BRS_FLAG_NONFINITE);
    ww[t] = __fmul_rn(beta, __fsub_rn(vv[t], u));
  }
  __syncthreads();

  // ---- S <- S + k w^T
  {
    const float4 w4 = ((const float4*)ww)[cb];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float kv = kk[row0 + r];
      x[r][0] = __fmaf_rn(kv, w4.x, x[r][0]);
      x[r][1] = __fmaf_rn(kv, w4.y, x[r][1]);
      x[r][2] = __fmaf_rn(kv, w4.z, x[r][2]);
      x[r][3] = __fmaf_rn(kv, w4.w, x[r][3]);
    }
  }

  // ---- o = S^T q from the updated FP32 state (before quantization)
  for (int s = 0; s < 8; ++s) {
    if (rb == s) {
      float4 acc = s ? carry[cb] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float qv = qq[row0 + r];
        acc.x = __fmaf_rn(qv, x[r][0], acc.x);
        acc.y = __fmaf_rn(qv, x[r][1], acc.y);
        acc.z = __fmaf_rn(qv, x[r][2], acc.z);
        acc.w = __fmaf_rn(qv, x[r][3], acc.w);
      }
      carry[cb] = acc;
    }
    __syncthreads();
  }
  if constexpr (ROT) {
    if (t < 32) {
      float* oo = (float*)carry;
      for (int hs = 1; hs < D; hs <<= 1) {
        for (int p = t; p < D / 2; p += 32) {
          const int i = (p / hs) * 2 * hs + (p % hs);
          const float u0 = oo[i], u1 = oo[i + hs];
          oo[i] = __fadd_rn(u0, u1);
          oo[i + hs] = __fsub_rn(u0, u1);
        }
        __syncwarp();
      }
      for (int j = t; j < D; j += 32) oo[j] = __fmul_rn(oo[j], a.hscale);
    }
    __syncthreads();
  }
  if (t < D) {
    const float ov = ((const float*)carry)[t];
    if (!isfinite(ov)) raise_flag(a.flags, BRS_FLAG_NONFINITE);
    a.o[(size_t)head * D + t] = ov;
  }

  // ---- write-back
  uint8_t* hout = (uint8_t*)a.packed_out + (size_t)head * a.head_bytes;
  if constexpr (STORE == BRS_STORE_FP32) {
#pragma unroll
    for (int r = 0; r < R; ++r)
      *(float4*)(hout + ((size_t)(row0 + r) * D + col0) * 4) =
          make_float4(x[r][0], x[r][1], x[r][2], x[r][3]);
  } else {
    const int nb = D / a.block;
    uint8_t* f16base = hout + (size_t)nlo * D;
    uint32_t* szbase = (uint32_t*)(hout + (size_t)nlo * D + (size_t)a.k_hi * D * 2);
    const int gl = a.block / 4;                          // threads per block
    const uint32_t lane = t & 31;
    // lanes of this thread's block group and of its row group (aligned runs)
    const uint32_t gmask = (gl >= 32) ? 0xffffffffu : (((1u << gl) - 1u) << (lane & ~(uint32_t)(gl - 1)));
    const uint32_t rmask = (LPR >= 32) ? 0xffffffffu : (((1u << LPR) - 1u) << (lane & ~(uint32_t)(LPR - 1)));
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = row0 + r;
      if constexpr (ROT) {
        const bool mine = i >= nlo;
        if (__any_sync(0xffffffffu, mine)) {
          float y[4] = {x[r][0], x[r][1], x[r][2], x[r][3]};
          row_fwht4<D>(y, cb, a.hscale);
          if (mine) {
#pragma unroll
            for (int c = 0; c < 4; ++c) x[r][c] = y[c];
          }
        }
      }
      if (i >= nlo) {
        // protected row: FP16, nearest
        uint16_t hv[4];
        bool ovf = false;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          hv[c] = f32_to_f16(x[r][c]);
          ovf |= f16_inf_or_nan(hv[c]) && isfinite(x[r][c]);
        }
        if (ovf) raise_flag(a.flags, BRS_FLAG_OVERFLOW);
        *(uint2*)(f16base + ((size_t)(i - nlo) * D + col0) * 2) =
            make_uint2((uint32_t)hv[0] | ((uint32_t)hv[1] << 16), (uint32_t)hv[2] | ((uint32_t)hv[3] << 16));
        continue;
      }
      // INT8 row, asymmetric block quantizer
      float y[4] = {x[r][0], x[r][1], x[r][2], x[r][3]};
      uint16_t* auxrow = nullptr;
      if (a.mode == BRS_ROUND_ERRFEEDBACK) {
        auxrow = (uint16_t*)a.aux + ((size_t)head * nlo + i) * D + col0;
        const uint2 ev = *(const uint2*)auxrow;
        y[0] = __fadd_rn(y[0], f16_to_f32((uint16_t)(ev.x & 0xffffu)));
        y[1] = __fadd_rn(y[1], f16_to_f32((uint16_t)(ev.x >> 16)));
        y[2] = __fadd_rn(y[2], f16_to_f32((uint16_t)(ev.y & 0xffffu)));
        y[3] = __fadd_rn(y[3], f16_to_f32((uint16_t)(ev.y >> 16)));
      }
      float mn = fminf(fminf(y[0], y[1]), fminf(y[2], y[3]));
      float mx = fmaxf(fmaxf(y[0], y[1]), fmaxf(y[2], y[3]));
      for (int m = 1; m < gl; m <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(rmask, mn, m));
        mx = fmaxf(mx, __shfl_xor_sync(rmask, mx, m));
      }
      if (mn == 0.0f || mx == 0.0f) {
        // a zero extreme: -0 ranks below +0 (uniform within the block group)
        bool negz = false, posz = false;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          negz |= (y[c] == 0.0f) && signbit(y[c]);
          posz |= (y[c] == 0.0f) && !signbit(y[c]);
        }
        const unsigned nz = __reduce_or_sync(gmask, negz ? 1u : 0u);
        const unsigned pz = __reduce_or_sync(gmask, posz ? 1u : 0u);
        if (mn == 0.0f) mn = nz ? -0.0f : 0.0f;
        if (mx == 0.0f) mx = pz ? 0.0f : -0.0f;
      }
      const uint16_t sh = f32_to_f16(__fdiv_rn(__fsub_rn(mx, mn), 255.0f));
      const uint16_t zh = f32_to_f16(mn);
      if (f16_inf_or_nan(sh) || f16_inf_or_nan(zh)) raise_flag(a.flags, BRS_FLAG_OVERFLOW);
      const float s = f16_to_f32(sh), z = f16_to_f32(zh);
      const float rcp = (s == 0.0f) ? 0.0f : __frcp_rn(s);
      uint4 rnd = make_uint4(0, 0, 0, 0);
      if (a.mode == BRS_ROUND_STOCHASTIC)
        rnd = philox4x32_10(make_uint4((uint32_t)(i * (D / 4) + cb), (uint32_t)a.step, (uint32_t)h, (uint32_t)b),
                            make_uint2((uint32_t)a.seed, (uint32_t)(a.seed >> 32)));
      const uint32_t rw[4] = {rnd.x >> 8, rnd.y >> 8, rnd.z >> 8, rnd.w >> 8};
      uint32_t packed4 = 0;
      uint16_t e16[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float code = 0.0f;
        if (s != 0.0f) {
          const float tt = __fmul_rn(__fsub_rn(y[c], z), rcp);
          code = (a.mode == BRS_ROUND_STOCHASTIC) ? sr_round(tt, rw[c]) : rintf(tt);
          code = fminf(fmaxf(code, 0.0f), 255.0f);
        }
        packed4 |= ((uint32_t)(int)code) << (8 * c);
        if (a.mode == BRS_ROUND_ERRFEEDBACK) {
          const float xhat = __fmaf_rn(code, s, z);
          float e = __fsub_rn(y[c], xhat);
          if (e > s) e = s;
          else if (e < -s) e = -s;
          e16[c] = f32_to_f16(e);
        }
      }
      *(uint32_t*)(hout + (size_t)i * D + col0) = packed4;
      if ((col0 % a.block) == 0) szbase[i * nb + col0 / a.block] = (uint32_t)sh | ((uint32_t)zh << 16);
      if (a.mode == BRS_ROUND_ERRFEEDBACK)
        *(uint2*)auxrow = make_uint2((uint32_t)e16[0] | ((uint32_t)e16[1] << 16),
                                     (uint32_t)e16[2] | ((uint32_t)e16[3] << 16));
    }
  }
}

template <int D>
static cudaError_t launch_d(const DecodeArgs& a, int store, bool rot, cudaStream_t st) {
  const dim3 grid(a.B * a.H), block(2 * D);
  if (store == BRS_STORE_FP32)
    decode_kernel<D, BRS_STORE_FP32, false><<<grid, block, 0, st>>>(a);
  else if (rot)
    decode_kernel<D, BRS_STORE_DAMP, true><<<grid, block, 0, st>>>(a);
  else
    decode_kernel<D, BRS_STORE_DAMP, false><<<grid, block, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, int d, int store, bool rot, cudaStream_t st) {
  switch (d) {
    case 32: return launch_d<32>(a, store, rot, st);
    case 64: return launch_d<64>(a, store, rot, st);
    case 128: return launch_d<128>(a, store, rot, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace brs
