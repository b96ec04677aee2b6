// Chunked prefill with deferred write-back (DAMP storage): the state is
// dequantized once per chunk of C = 64 tokens, the chunk's 64 delta-rule
// steps are evaluated together in WY form, and the state is requantized
// once at the chunk's end ("Low-Bit Recurrent States in Hybrid Language
// Models", Accumulated readout error: write-back once per prefill chunk;
// Protocol: quantized and dequantized before reuse).
//
// WY form of one chunk (t, s = 0..63 tokens, i = key channel, j = value
// column), derived from S_t = D_t S_{t-1} + k_t w_t^T with
// w_t = beta_t (v_t - (D_t S_{t-1})^T k_t):
//   Gamma_t = prod_{r <= t} a_r (per key channel), K~ = K * Gamma,
//   K^ = K / Gamma, Q~ = Q * Gamma;
//   A  = strictly-lower(diag(beta) K~ K^T);
//   (I + A) W = diag(beta) (V - K~ S_0)        (forward substitution)
//   O  = Q~ S_0 + lower-incl(Q~ K^T) W;
//   S_C = diag(Gamma_63) (S_0 + K^T W).
// The chunk arithmetic runs in FP32 (not the token-by-token order of the
// oracle; results agree within the output tolerance and the stored codes
// are the oracle quantizer applied to this S_C, checked by replay).
//
// One CTA (256 threads) per (sequence, head) walks the chunks in order;
// the FP32 state and the chunk operands live in shared memory.
#include <cuda_runtime.h>
#include <cstdint>

#include "brs_device.cuh"
#include "brs_internal.h"

namespace brs {

constexpr int kPfD = 128, kPfC = 64, kPfThreads = 256;

struct PfSmem {
  float S[kPfD][kPfD];          // state (value basis, stored row order)
  float KT[kPfC][kPfD];         // K~
  float KH[kPfC][kPfD];         // K^
  float QT[kPfC][kPfD];         // Q~
  float VW[kPfC][kPfD];         // V, then diag(beta)(V - K~ S_0), then W
  float AM[kPfC][kPfC];         // A, then lower-incl(Q~ K^T)
  float gam[kPfD];              // Gamma_63
  float beta[kPfC];
};

// C(m, n) = sum_k Aop(m, k) * Bop(k, n) over a TM x TN tile per thread;
// the (M / TM) x (N / TN) tiles cover the CTA's 256 threads.
template <int M, int N, int K, int TM, int TN, class FA, class FB, class FE>
__device__ __forceinline__ void cta_gemm(FA Aop, FB Bop, FE epi) {
  static_assert((M / TM) * (N / TN) == kPfThreads, "one tile per thread");
  const int t = threadIdx.x;
  const int m0 = (t / (N / TN)) * TM, n0 = (t % (N / TN)) * TN;
  float acc[TM][TN];
#pragma unroll
  for (int m = 0; m < TM; ++m)
#pragma unroll
    for (int n = 0; n < TN; ++n) acc[m][n] = 0.f;
#pragma unroll 4
  for (int k = 0; k < K; ++k) {
    float av[TM], bv[TN];
#pragma unroll
    for (int m = 0; m < TM; ++m) av[m] = Aop(m0 + m, k);
#pragma unroll
    for (int n = 0; n < TN; ++n) bv[n] = Bop(k, n0 + n);
#pragma unroll
    for (int m = 0; m < TM; ++m)
#pragma unroll
      for (int n = 0; n < TN; n += 2) fma2(acc[m][n], acc[m][n + 1], av[m], av[m], bv[n], bv[n + 1], acc[m][n], acc[m][n + 1]);
  }
#pragma unroll
  for (int m = 0; m < TM; ++m)
#pragma unroll
    for (int n = 0; n < TN; ++n) epi(m0 + m, n0 + n, acc[m][n]);
}

// dequantize the stored head into S (value basis)
template <bool HAD, int BLOCK>
__device__ void pf_load_state(PfSmem& sm, const uint8_t* head, int nlo, int k_hi, float hscale) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, col0 = 4 * lane;
  constexpr int NB = kPfD / BLOCK;
  const uint8_t* f16in = head + (size_t)nlo * kPfD;
  const uint32_t* szin = (const uint32_t*)(head + (size_t)nlo * kPfD + (size_t)k_hi * kPfD * 2);
  for (int r = warp; r < kPfD; r += kPfThreads / 32) {
    float x[4];
    if (r < nlo) {
      const uint32_t c4 = *(const uint32_t*)(head + (size_t)r * kPfD + col0);
      const uint32_t sz = szin[r * NB + col0 / BLOCK];
      const float s = f16_to_f32((uint16_t)(sz & 0xffffu)), z = f16_to_f32((uint16_t)(sz >> 16));
#pragma unroll
      for (int c = 0; c < 4; ++c) x[c] = __fmaf_rn(__fsub_rn(byte_magic(c4, c), kTwo23), s, z);
      if (HAD) row_fwht4<kPfD>(x, lane, hscale);        // back to the value basis
    } else {
      const uint2 hv = *(const uint2*)(f16in + ((size_t)(r - nlo) * kPfD + col0) * 2);
      x[0] = f16_to_f32((uint16_t)(hv.x & 0xffffu)); x[1] = f16_to_f32((uint16_t)(hv.x >> 16));
      x[2] = f16_to_f32((uint16_t)(hv.y & 0xffffu)); x[3] = f16_to_f32((uint16_t)(hv.y >> 16));
    }
    *(float4*)&sm.S[r][col0] = make_float4(x[0], x[1], x[2], x[3]);
  }
}

// quantize S into the stored head (and continue from the stored values)
template <bool HAD, int BLOCK, int MODE>
__device__ void pf_store_state(PfSmem& sm, uint8_t* head, uint16_t* aux, int nlo, int k_hi, float hscale,
                               const PrefillArgs& a, int64_t step, int h, int b, float* sdump,
                               uint32_t* flags) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, col0 = 4 * lane;
  constexpr int NB = kPfD / BLOCK, GL = BLOCK / 4;
  uint16_t* f16out = (uint16_t*)(head + (size_t)nlo * kPfD);
  uint32_t* szout = (uint32_t*)(head + (size_t)nlo * kPfD + (size_t)k_hi * kPfD * 2);
  for (int r = warp; r < kPfD; r += kPfThreads / 32) {
    float4 v4 = *(const float4*)&sm.S[r][col0];
    if (sdump) *(float4*)&sdump[(size_t)r * kPfD + col0] = v4;
    float x[4] = {v4.x, v4.y, v4.z, v4.w};
    if (r >= nlo) {
      const uint32_t lo = f16x2_of(x[0], x[1]), hi = f16x2_of(x[2], x[3]);
      if ((((lo >> 10) & 31u) == 31u) || (((lo >> 26) & 31u) == 31u) || (((hi >> 10) & 31u) == 31u) ||
          (((hi >> 26) & 31u) == 31u))
        raise_flag(flags, BRS_FLAG_OVERFLOW);
      *(uint2*)&f16out[(size_t)(r - nlo) * kPfD + col0] = make_uint2(lo, hi);
      *(float4*)&sm.S[r][col0] = make_float4(f16_to_f32((uint16_t)(lo & 0xffffu)), f16_to_f32((uint16_t)(lo >> 16)),
                                              f16_to_f32((uint16_t)(hi & 0xffffu)), f16_to_f32((uint16_t)(hi >> 16)));
      continue;
    }
    if (HAD) row_fwht4<kPfD>(x, lane, hscale);
    if (MODE == BRS_ROUND_ERRFEEDBACK) {
      const uint2 ev = *(const uint2*)&aux[(size_t)r * kPfD + col0];
      x[0] = __fadd_rn(x[0], f16_to_f32((uint16_t)(ev.x & 0xffffu)));
      x[1] = __fadd_rn(x[1], f16_to_f32((uint16_t)(ev.x >> 16)));
      x[2] = __fadd_rn(x[2], f16_to_f32((uint16_t)(ev.y & 0xffffu)));
      x[3] = __fadd_rn(x[3], f16_to_f32((uint16_t)(ev.y >> 16)));
    }
    float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
    float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
#pragma unroll
    for (int m = 1; m < GL; m <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, m));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
    }
    if (mn == 0.0f || mx == 0.0f) {             // -0 ranks below +0 (uniform per block group)
      bool nz = false, pz = false;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        nz |= (x[c] == 0.0f) && signbit(x[c]);
        pz |= (x[c] == 0.0f) && !signbit(x[c]);
      }
      const uint32_t gmask = (GL >= 32) ? 0xffffffffu : (((1u << GL) - 1u) << (lane & ~(uint32_t)(GL - 1)));
      const unsigned anz = __reduce_or_sync(gmask, nz ? 1u : 0u), apz = __reduce_or_sync(gmask, pz ? 1u : 0u);
      if (mn == 0.0f) mn = anz ? -0.0f : 0.0f;
      if (mx == 0.0f) mx = apz ? 0.0f : -0.0f;
    }
    if (!isfinite(mn) || !isfinite(mx)) raise_flag(flags, BRS_FLAG_NONFINITE);
    const uint16_t sh = f32_to_f16(__fdiv_rn(__fsub_rn(mx, mn), 255.0f));
    const uint16_t zh = f32_to_f16(mn);
    if (f16_inf_or_nan(sh) || f16_inf_or_nan(zh)) raise_flag(flags, BRS_FLAG_OVERFLOW);
    const float s = f16_to_f32(sh), z = f16_to_f32(zh);
    const float rcp = (s == 0.0f) ? 0.0f : __frcp_rn(s);
    uint4 rnd = make_uint4(0, 0, 0, 0);
    if (MODE == BRS_ROUND_STOCHASTIC)
      rnd = philox4x32_10(make_uint4((uint32_t)(r * (kPfD / 4) + lane), (uint32_t)step, (uint32_t)h, (uint32_t)b),
                          make_uint2((uint32_t)a.seed, (uint32_t)(a.seed >> 32)));
    const uint32_t rw[4] = {rnd.x >> 8, rnd.y >> 8, rnd.z >> 8, rnd.w >> 8};
    uint32_t packed4 = 0;
    float xh[4];
    uint16_t e16[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float code = 0.0f;
      if (s != 0.0f) {
        const float tt = __fmul_rn(__fsub_rn(x[c], z), rcp);
        code = (MODE == BRS_ROUND_STOCHASTIC) ? sr_round(tt, rw[c]) : rintf(tt);
        code = fminf(fmaxf(code, 0.0f), 255.0f);
      }
      packed4 |= ((uint32_t)(int)code) << (8 * c);
      xh[c] = __fmaf_rn(code, s, z);
      if (MODE == BRS_ROUND_ERRFEEDBACK) {
        float e = __fsub_rn(x[c], xh[c]);
        if (e > s) e = s;
        else if (e < -s) e = -s;
        e16[c] = f32_to_f16(e);
      }
    }
    *(uint32_t*)(head + (size_t)r * kPfD + col0) = packed4;
    if ((col0 % BLOCK) == 0) szout[r * NB + col0 / BLOCK] = (uint32_t)sh | ((uint32_t)zh << 16);
    if (MODE == BRS_ROUND_ERRFEEDBACK)
      *(uint2*)&aux[(size_t)r * kPfD + col0] = make_uint2((uint32_t)e16[0] | ((uint32_t)e16[1] << 16),
                                                          (uint32_t)e16[2] | ((uint32_t)e16[3] << 16));
    if (HAD) row_fwht4<kPfD>(xh, lane, hscale);         // continue from the stored values
    *(float4*)&sm.S[r][col0] = make_float4(xh[0], xh[1], xh[2], xh[3]);
  }
}

template <bool HAD, int BLOCK, int MODE>
__global__ void __launch_bounds__(kPfThreads, 1) prefill_kernel(const PrefillArgs a) {
  extern __shared__ __align__(16) unsigned char pf_raw[];
  PfSmem& sm = *(PfSmem*)pf_raw;
  const int t = threadIdx.x;
  const int head = blockIdx.x;
  const int b = head / a.H, h = head - b * a.H;
  const int kh = h * a.Hk / a.H;
  const int nlo = kPfD - a.k_hi;
  uint8_t* hst = (uint8_t*)a.packed + (size_t)head * a.head_bytes;
  uint16_t* aux = (MODE == BRS_ROUND_ERRFEEDBACK) ? (uint16_t*)a.aux + (size_t)head * nlo * kPfD : nullptr;

  pf_load_state<HAD, BLOCK>(sm, hst, nlo, a.k_hi, a.hscale);
  const int nchunks = a.T / kPfC;
  for (int ch = 0; ch < nchunks; ++ch) {
    const int t0 = ch * kPfC;
    __syncthreads();
    // ---- chunk inputs: cumulative decay per key channel; K~, K^, Q~; V; beta
    if (t < kPfD) {
      const int p = a.perm ? a.perm[h * kPfD + t] : t;
      float g = 1.0f;
      for (int r = 0; r < kPfC; ++r) {
        const size_t tok = (size_t)b * a.T + t0 + r;
        const float av = a.decay_per_key ? a.decay[(tok * a.H + h) * kPfD + p] : a.decay[tok * a.H + h];
        g = __fmul_rn(g, av);
        const float kv = bf16_to_f32(a.k[(tok * a.Hk + kh) * kPfD + p]);
        const float qv = bf16_to_f32(a.q[(tok * a.Hk + kh) * kPfD + p]);
        sm.KT[r][t] = __fmul_rn(kv, g);
        sm.KH[r][t] = __fdiv_rn(kv, g);
        sm.QT[r][t] = __fmul_rn(qv, g);
      }
      sm.gam[t] = g;
    } else {
      const int j = t - kPfD;
      for (int r = 0; r < kPfC; ++r) {
        const size_t tok = (size_t)b * a.T + t0 + r;
        sm.VW[r][j] = bf16_to_f32(a.v[(tok * a.H + h) * kPfD + j]);
      }
      if (j < kPfC) sm.beta[j] = a.beta[((size_t)b * a.T + t0 + j) * a.H + h];
    }
    __syncthreads();
    // ---- A = strictly-lower(diag(beta) K~ K^T)
    cta_gemm<kPfC, kPfC, kPfD, 4, 4>(
        [&](int m, int k) { return sm.KT[m][k]; }, [&](int k, int n) { return sm.KH[n][k]; },
        [&](int m, int n, float v) { sm.AM[m][n] = (n < m) ? __fmul_rn(sm.beta[m], v) : 0.0f; });
    __syncthreads();
    // ---- right-hand side diag(beta) (V - K~ S_0), in place over V
    cta_gemm<kPfC, kPfD, kPfD, 4, 8>(
        [&](int m, int k) { return sm.KT[m][k]; }, [&](int k, int n) { return sm.S[k][n]; },
        [&](int m, int n, float v) { sm.VW[m][n] = __fmul_rn(sm.beta[m], __fsub_rn(sm.VW[m][n], v)); });
    __syncthreads();
    // ---- (I + A) W = rhs by forward substitution; column j by thread j
    if (t < kPfD) {
      float w[kPfC];
#pragma unroll
      for (int r = 0; r < kPfC; ++r) {
        float acc = sm.VW[r][t];
#pragma unroll
        for (int s = 0; s < r; ++s) acc = __fmaf_rn(-sm.AM[r][s], w[s], acc);
        w[r] = acc;
      }
#pragma unroll
      for (int r = 0; r < kPfC; ++r) sm.VW[r][t] = w[r];
    }
    __syncthreads();
    // ---- lower-incl(Q~ K^T), then O = Q~ S_0 + that * W
    cta_gemm<kPfC, kPfC, kPfD, 4, 4>(
        [&](int m, int k) { return sm.QT[m][k]; }, [&](int k, int n) { return sm.KH[n][k]; },
        [&](int m, int n, float v) { sm.AM[m][n] = (n <= m) ? v : 0.0f; });
    __syncthreads();
    {
      const int m0 = (t / 16) * 4, n0 = (t % 16) * 8;
      float acc[4][8];
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int n = 0; n < 8; ++n) acc[m][n] = 0.f;
#pragma unroll 4
      for (int k = 0; k < kPfD; ++k)
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float av = sm.QT[m0 + m][k];
#pragma unroll
          for (int n = 0; n < 8; ++n) acc[m][n] = __fmaf_rn(av, sm.S[k][n0 + n], acc[m][n]);
        }
#pragma unroll 4
      for (int k = 0; k < kPfC; ++k)
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float av = sm.AM[m0 + m][k];
#pragma unroll
          for (int n = 0; n < 8; ++n) acc[m][n] = __fmaf_rn(av, sm.VW[k][n0 + n], acc[m][n]);
        }
      bool bad = false;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const size_t tok = (size_t)b * a.T + t0 + m0 + m;
        float* od = a.o + (tok * a.H + h) * kPfD + n0;
#pragma unroll
        for (int n = 0; n < 8; ++n) bad |= !isfinite(acc[m][n]);
        *(float4*)od = make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
        *(float4*)(od + 4) = make_float4(acc[m][4], acc[m][5], acc[m][6], acc[m][7]);
      }
      if (bad) raise_flag(a.flags, BRS_FLAG_NONFINITE);
    }
    __syncthreads();
    // ---- S_C = diag(Gamma_63) (S_0 + K^T W), in place
    cta_gemm<kPfD, kPfD, kPfC, 8, 8>(
        [&](int m, int k) { return sm.KH[k][m]; }, [&](int k, int n) { return sm.VW[k][n]; },
        [&](int m, int n, float v) { sm.S[m][n] = __fmul_rn(sm.gam[m], __fadd_rn(sm.S[m][n], v)); });
    __syncthreads();
    // ---- write-back of the chunk
    const bool last = ch == nchunks - 1;
    pf_store_state<HAD, BLOCK, MODE>(sm, hst, aux, nlo, a.k_hi, a.hscale, a, a.step0 + t0 + kPfC - 1, h, b,
                                     (last && a.sdump) ? a.sdump + (size_t)head * kPfD * kPfD : nullptr,
                                     a.flags);
  }
}

template <bool HAD, int BLOCK>
static cudaError_t pf_launch_hb(const PrefillArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(PfSmem);
  cudaError_t e;
  switch (a.mode) {
#define PF_CASE(M)                                                                                     \
  case M:                                                                                              \
    e = cudaFuncSetAttribute(prefill_kernel<HAD, BLOCK, M>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             (int)smem);                                                               \
    if (e != cudaSuccess) return e;                                                                    \
    prefill_kernel<HAD, BLOCK, M><<<a.B * a.H, kPfThreads, smem, st>>>(a);                             \
    break;
    PF_CASE(BRS_ROUND_NEAREST)
    PF_CASE(BRS_ROUND_STOCHASTIC)
    PF_CASE(BRS_ROUND_ERRFEEDBACK)
#undef PF_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

bool prefill_supported(int d, int block, int k_hi, int C) {
  return d == kPfD && C == kPfC && (block == 128 || block == 32) && k_hi % 4 == 0 && k_hi <= kPfD;
}

cudaError_t launch_prefill(const PrefillArgs& a, bool had, cudaStream_t st) {
  if (a.block == 128) return had ? pf_launch_hb<true, 128>(a, st) : pf_launch_hb<false, 128>(a, st);
  if (a.block == 32) return had ? pf_launch_hb<true, 32>(a, st) : pf_launch_hb<false, 32>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace brs
