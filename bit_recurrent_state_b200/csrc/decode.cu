// Decode step for FP32 and DAMP storage: one token for every (sequence,
// head).  One CTA per head; 2*D threads (D/16 warps); thread t owns the 4
// consecutive columns 4*(t % (D/4)) .. +3 of the R = D/8 consecutive stored
// rows R*(t / (D/4)) .. +R-1 (its "row group"), so the D x D FP32 state of
// the head lives in registers for the whole step and every state byte
// crosses HBM once in and once out.
//
// Sources: DAMP summary, Key Points > Implementation (fused executor:
// reconstruct the INT8 channels, update in FP32, re-quantize, write back;
// static permutation with the protected channels contiguous) and Data &
// Methods > Quantization & calibration details (per-block asymmetric INT8
// after a Hadamard along the value axis); "Low-Bit Recurrent States in
// Hybrid Language Models", Accumulated readout error (outputs precede
// quantization) and Protocol (quantized and dequantized before reuse).
//
// Evaluation order (the library's documented one; the oracle's mixed-basis
// mode): each tier of a DAMP head is updated in the basis it is stored in,
// the INT8 rows in the Hadamard basis, the FP16 rows in the value basis.
//   u = U2 + T(U1), w = beta (v - u), S_i += k_i T(w) (INT8 rows),
//   S_i += k_i w (FP16 rows), o = O2 + T(O1),
// with U1/O1 and U2/O2 fmaf chains over the INT8 and the FP16 rows in
// stored order and T the Hadamard (or the identity).  Only three vectors of
// D values are transformed per head.  Paired f32x2 instructions are two
// independent IEEE operations, so pairing changes no result.
#include <cuda_runtime.h>
#include <cstdint>

#include "brs_device.cuh"
#include "brs_internal.h"

namespace brs {

template <int D>
struct Geo {
  static constexpr int NT = 2 * D;      // threads per CTA
  static constexpr int NW = NT / 32;    // warps
  static constexpr int LPR = D / 4;     // threads per row
  static constexpr int R = D / 8;       // rows per thread (8 row groups)
  static constexpr int RPW = 32 / LPR;  // row groups per warp
};

struct __align__(16) QPrm {
  f2_t zz, rr;                          // (zero, zero), (1/scale, 1/scale)
  f2_t ss;                              // (scale, scale)
  uint32_t ok, pad;                     // grid keeps every rounded code in [0, 255]
};

template <int D>
struct __align__(16) DecodeSmem {
  f2_t kk2[D], qq2[D], aa2[D];          // gathered k, q, a, each duplicated into a pair
  float vv[D], ww[D], wt[D];            // v, w (value basis), T(w)
  float c1[D], c2[D];                   // running / final sums of the two tiers
  QPrm prm[D][D / 32];                  // per (row, block) quantization grid
};

__device__ __forceinline__ void bar_sync_n(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ void bar_arrive_n(int id, int n) { asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// The row chains: row groups [0, ng1) accumulate into sm.c1, row groups
// [ng1, 8) into sm.c2, each an fmaf chain over its rows in stored order
// from +0.  With one row group per warp (D = 128) consecutive warps hand
// off through named barriers (the two tiers run concurrently); otherwise
// the row groups take turns between CTA-wide barriers.  Ends with a
// CTA-wide barrier.
template <int D>
__device__ __forceinline__ void row_chains(DecodeSmem<D>& sm, const f2_t* coef, const f2_t (&x)[D / 8][2],
                                           int rb, int cb, int ng1) {
  using G = Geo<D>;
  auto body = [&](bool first, float* acc) {
    f2_t a01 = 0ull, a23 = 0ull;
    if (!first) {
      a01 = *(const f2_t*)&acc[4 * cb];
      a23 = *(const f2_t*)&acc[4 * cb + 2];
    }
#pragma unroll
    for (int r = 0; r < G::R; ++r) {
      const f2_t k = coef[rb * G::R + r];
      a01 = f2fma(k, x[r][0], a01);
      a23 = f2fma(k, x[r][1], a23);
    }
    *(f2_t*)&acc[4 * cb] = a01;
    *(f2_t*)&acc[4 * cb + 2] = a23;
  };
  if constexpr (G::RPW == 1) {
    const bool tier1 = rb < ng1;
    const int first = tier1 ? 0 : ng1, last = tier1 ? ng1 - 1 : 7;
    if (rb > first) bar_sync_n(rb, 64);
    body(rb == first, tier1 ? sm.c1 : sm.c2);
    if (rb < last) bar_arrive_n(rb + 1, 64);
    __syncthreads();
  } else {
    for (int s = 0; s < 8; ++s) {
      if (rb == s) body(s == 0 || s == ng1, (s < ng1) ? sm.c1 : sm.c2);
      __syncthreads();
    }
  }
}

// T of one D-vector in shared memory, in place, by the calling warp.
template <int D>
__device__ __forceinline__ void vec_fwht(float* v, float hscale) {
  const int lane = threadIdx.x % 32;
  const int cb = lane % Geo<D>::LPR;
  float x[4];
  const float4 a = *(const float4*)&v[4 * cb];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  row_fwht4<D>(x, cb, hscale);
  __syncwarp();
  if (lane < Geo<D>::LPR) *(float4*)&v[4 * cb] = make_float4(x[0], x[1], x[2], x[3]);
  __syncwarp();
}

__device__ __forceinline__ uint32_t f16x2_overflow(uint32_t w) {
  return (((w >> 10) & 31u) == 31u) | (((w >> 26) & 31u) == 31u);
}

template <int D, int STORE, bool HAD, int BLOCK, int MODE>
__global__ void __launch_bounds__(2 * D, (D == 128) ? 2 : 4) decode_kernel(const DecodeArgs a) {
  using G = Geo<D>;
  constexpr int R = G::R, LPR = G::LPR;
  constexpr int GL = BLOCK / 4;          // threads per quantization block
  constexpr int NB = D / BLOCK;          // blocks per row
  constexpr int V = 2 * R;               // (min, max) values per thread
  constexpr int VPL = V / GL;            // values per lane after the reduce-scatter
  constexpr int RPL = (VPL >= 2) ? VPL / 2 : 1;
  static_assert(V >= GL, "reduce-scatter needs 2R >= BLOCK/4");
  __shared__ DecodeSmem<D> sm;

  const int t = threadIdx.x, lane = t % 32;
  const int cb = t % LPR, rb = t / LPR;
  const int row0 = rb * R, col0 = 4 * cb;
  const int head = blockIdx.x;
  const int b = head / a.H, h = head - b * a.H;
  const int kh = h * a.Hk / a.H;
  const int nlo = (STORE == BRS_STORE_FP32) ? D : D - a.k_hi;  // INT8 rows: 0..nlo-1
  const int ng1 = nlo / R;               // row groups of the INT8 tier
  const bool tier1 = rb < ng1;           // whole row group in one tier (k_hi % R == 0)
  const uint8_t* hin = (const uint8_t*)a.packed_in + (size_t)head * a.head_bytes;
  uint8_t* hout = (uint8_t*)a.packed_out + (size_t)head * a.head_bytes;

  // ---- issue the state loads first, then gather the inputs
  f2_t x[R][2];
  uint32_t c4[R], sz[R];
  if constexpr (STORE == BRS_STORE_FP32) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const ulonglong2 f = __ldg((const ulonglong2*)(hin + ((size_t)(row0 + r) * D + col0) * 4));
      x[r][0] = f.x;
      x[r][1] = f.y;
    }
  } else if (tier1) {
    const uint32_t* szin = (const uint32_t*)(hin + (size_t)nlo * D + (size_t)a.k_hi * D * 2);
#pragma unroll
    for (int r = 0; r < R; ++r) c4[r] = __ldg((const uint32_t*)(hin + (size_t)(row0 + r) * D + col0));
    if constexpr (NB == 1) {
#pragma unroll
      for (int r = 0; r < R; r += 4) {
        const uint4 q4 = __ldg((const uint4*)(szin + row0 + r));
        sz[r] = q4.x; sz[r + 1] = q4.y; sz[r + 2] = q4.z; sz[r + 3] = q4.w;
      }
    } else {
#pragma unroll
      for (int r = 0; r < R; ++r) sz[r] = __ldg(szin + (row0 + r) * NB + col0 / BLOCK);
    }
  } else {
    const uint8_t* f16in = hin + (size_t)nlo * D;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint2 hv = __ldg((const uint2*)(f16in + ((size_t)(row0 + r - nlo) * D + col0) * 2));
      c4[r] = hv.x;
      sz[r] = hv.y;
    }
  }
  if (t < D) {
    const int p = a.perm ? a.perm[h * D + t] : t;
    const size_t qk = ((size_t)b * a.Hk + kh) * D;
    sm.kk2[t] = f2dup(bf16_to_f32(a.k[qk + p]));
    sm.qq2[t] = f2dup(bf16_to_f32(a.q[qk + p]));
    sm.aa2[t] = f2dup(a.decay_per_key ? a.decay[(size_t)head * D + p] : a.decay[head]);
    sm.vv[t] = bf16_to_f32(a.v[(size_t)head * D + t]);
    sm.c2[t] = 0.0f;                     // an empty FP16 tier sums to +0
  }
  const float beta = a.beta[head];

  // ---- dequantize
  if constexpr (STORE != BRS_STORE_FP32) {
    if (tier1) {
      const f2_t two23 = f2dup(kTwo23);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const f2_t ss = f2dup(f16_to_f32((uint16_t)(sz[r] & 0xffffu)));
        const f2_t zz = f2dup(f16_to_f32((uint16_t)(sz[r] >> 16)));
        const f2_t c01 = f2sub(f2make(byte_magic(c4[r], 0), byte_magic(c4[r], 1)), two23);
        const f2_t c23 = f2sub(f2make(byte_magic(c4[r], 2), byte_magic(c4[r], 3)), two23);
        x[r][0] = f2fma(c01, ss, zz);
        x[r][1] = f2fma(c23, ss, zz);
      }
    } else {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        x[r][0] = f2make(f16_to_f32((uint16_t)(c4[r] & 0xffffu)), f16_to_f32((uint16_t)(c4[r] >> 16)));
        x[r][1] = f2make(f16_to_f32((uint16_t)(sz[r] & 0xffffu)), f16_to_f32((uint16_t)(sz[r] >> 16)));
      }
    }
  }
  __syncthreads();  // inputs visible

  // ---- decay: S <- Diag(a) S
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const f2_t ar = sm.aa2[row0 + r];
    x[r][0] = f2mul(ar, x[r][0]);
    x[r][1] = f2mul(ar, x[r][1]);
  }

  // ---- u = U2 + T(U1);  w = beta (v - u);  T(w)
  row_chains<D>(sm, sm.kk2, x, rb, cb, ng1);
  if (t < 32) {
    if constexpr (STORE != BRS_STORE_FP32 && HAD) vec_fwht<D>(sm.c1, a.hscale);
    for (int j = t; j < D; j += 32) {
      const float u = (STORE == BRS_STORE_FP32) ? sm.c1[j] : __fadd_rn(sm.c2[j], sm.c1[j]);
      if (!isfinite(u)) raise_flag(a.flags, BRS_FLAG_NONFINITE);
      const float w = __fmul_rn(beta, __fsub_rn(sm.vv[j], u));
      sm.ww[j] = w;
      sm.wt[j] = w;
    }
    __syncwarp();
    if constexpr (STORE != BRS_STORE_FP32 && HAD) vec_fwht<D>(sm.wt, a.hscale);
  }
  __syncthreads();

  // ---- S_i <- S_i + k_i T(w) (INT8 tier), S_i + k_i w (FP16 tier)
  {
    const float* wsrc = tier1 ? sm.wt : sm.ww;
    const f2_t w01 = *(const f2_t*)&wsrc[col0], w23 = *(const f2_t*)&wsrc[col0 + 2];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const f2_t kv = sm.kk2[row0 + r];
      x[r][0] = f2fma(kv, w01, x[r][0]);
      x[r][1] = f2fma(kv, w23, x[r][1]);
    }
  }

  // ---- o = O2 + T(O1) from the updated FP32 state (before quantization)
  if (t < D) sm.c2[t] = 0.0f;
  __syncthreads();
  row_chains<D>(sm, sm.qq2, x, rb, cb, ng1);
  if (t < 32) {
    if constexpr (STORE != BRS_STORE_FP32 && HAD) vec_fwht<D>(sm.c1, a.hscale);
    for (int j = t; j < D; j += 32) {
      const float ov = (STORE == BRS_STORE_FP32) ? sm.c1[j] : __fadd_rn(sm.c2[j], sm.c1[j]);
      if (!isfinite(ov)) raise_flag(a.flags, BRS_FLAG_NONFINITE);
      a.o[(size_t)head * D + j] = ov;
    }
  }

  // ---- write-back
  if constexpr (STORE == BRS_STORE_FP32) {
#pragma unroll
    for (int r = 0; r < R; ++r)
      *(ulonglong2*)(hout + ((size_t)(row0 + r) * D + col0) * 4) = make_ulonglong2(x[r][0], x[r][1]);
    return;
  } else {
    if (!tier1) {
      // protected rows: FP16, nearest
      uint16_t* f16out = (uint16_t*)(hout + (size_t)nlo * D);
      uint32_t ovf = 0;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint32_t lo = f16x2_of(f2lo(x[r][0]), f2hi(x[r][0]));
        const uint32_t hi = f16x2_of(f2lo(x[r][1]), f2hi(x[r][1]));
        ovf |= f16x2_overflow(lo) | f16x2_overflow(hi);
        *(uint2*)&f16out[(size_t)(row0 + r - nlo) * D + col0] = make_uint2(lo, hi);
      }
      if (ovf) raise_flag(a.flags, BRS_FLAG_OVERFLOW);
      return;
    }
    // INT8 rows: error-feedback target, block extremes
    uint16_t* auxb = (MODE == BRS_ROUND_ERRFEEDBACK) ? (uint16_t*)a.aux + (size_t)head * nlo * D : nullptr;
    if constexpr (MODE == BRS_ROUND_ERRFEEDBACK) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint2 ev = *(const uint2*)&auxb[(size_t)(row0 + r) * D + col0];
        x[r][0] = f2add(x[r][0], f2make(f16_to_f32((uint16_t)(ev.x & 0xffffu)), f16_to_f32((uint16_t)(ev.x >> 16))));
        x[r][1] = f2add(x[r][1], f2make(f16_to_f32((uint16_t)(ev.y & 0xffffu)), f16_to_f32((uint16_t)(ev.y >> 16))));
      }
    }
    // lanes of this row group (every lane of a row group takes this path)
    const uint32_t rmask = (LPR >= 32) ? 0xffffffffu : (((1u << LPR) - 1u) << (lane & ~(uint32_t)(LPR - 1)));
    float v[V];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float y0 = f2lo(x[r][0]), y1 = f2hi(x[r][0]), y2 = f2lo(x[r][1]), y3 = f2hi(x[r][1]);
      v[2 * r] = fminf(fminf(y0, y1), fminf(y2, y3));
      v[2 * r + 1] = fmaxf(fmaxf(y0, y1), fmaxf(y2, y3));
    }
    // reduce-scatter over the GL lanes of the block group: afterwards lane
    // g (of its group) holds entries [g*VPL, (g+1)*VPL) reduced over the
    // group (even entries minima, odd entries maxima)
#pragma unroll
    for (int m = GL / 2, len = V; m >= 1; m >>= 1, len >>= 1) {
      const bool up = (lane & m) != 0;
#pragma unroll
      for (int i = 0; i < len / 2; ++i) {
        const float lo = v[i], hi = v[i + len / 2];
        const float other = __shfl_xor_sync(rmask, up ? lo : hi, m);
        const float mine = up ? hi : lo;
        if (len / 2 >= 2)
          v[i] = (i & 1) ? fmaxf(mine, other) : fminf(mine, other);
        else
          v[i] = (lane & 1) ? fmaxf(mine, other) : fminf(mine, other);
      }
    }
    float mnv[RPL], mxv[RPL];
    if constexpr (VPL >= 2) {
#pragma unroll
      for (int q = 0; q < RPL; ++q) { mnv[q] = v[2 * q]; mxv[q] = v[2 * q + 1]; }
    } else {
      const float other = __shfl_xor_sync(rmask, v[0], 1);
      mnv[0] = (lane & 1) ? other : v[0];
      mxv[0] = (lane & 1) ? v[0] : other;
    }
    const int g = (lane % LPR) % GL;            // lane within its block group
    const int blk = (lane % LPR) / GL;          // block index within the row
    const int lr0 = (VPL >= 2) ? g * RPL : g / 2;
    // a zero extreme takes the sign rule (-0 below +0): rare, warp-wide
    bool zc = false;
#pragma unroll
    for (int q = 0; q < RPL; ++q) zc |= (mnv[q] == 0.0f) || (mxv[q] == 0.0f);
    if (__any_sync(rmask, zc)) {
      uint32_t nz = 0, pz = 0;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float y[4] = {f2lo(x[r][0]), f2hi(x[r][0]), f2lo(x[r][1]), f2hi(x[r][1])};
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (y[c] == 0.0f) {
            if (signbit(y[c])) nz |= 1u << r; else pz |= 1u << r;
          }
      }
#pragma unroll
      for (int m = 1; m < GL; m <<= 1) {
        nz |= __shfl_xor_sync(rmask, nz, m);
        pz |= __shfl_xor_sync(rmask, pz, m);
      }
#pragma unroll
      for (int q = 0; q < RPL; ++q) {
        const int lr = lr0 + q;
        if (mnv[q] == 0.0f) mnv[q] = ((nz >> lr) & 1u) ? -0.0f : 0.0f;
        if (mxv[q] == 0.0f) mxv[q] = ((pz >> lr) & 1u) ? 0.0f : -0.0f;
      }
    }
    // grid of each (row, block): one division per row, spread over lanes.
    // ok: the smallest and largest grid coordinates of the block (the same
    // FP32 operations as the elements', which are monotone in y) round into
    // [0, 255], so no code of the block needs the clip at the rails.
    bool ok_all = true;
    uint32_t* szout = (uint32_t*)(hout + (size_t)nlo * D + (size_t)a.k_hi * D * 2);
#pragma unroll
    for (int q = 0; q < RPL; ++q) {
      const int i = row0 + lr0 + q;               // stored row
      if ((VPL >= 2) || ((lane & 1) == 0)) {
        if (!isfinite(mnv[q]) || !isfinite(mxv[q])) raise_flag(a.flags, BRS_FLAG_NONFINITE);
        const uint16_t sh = f32_to_f16(__fdiv_rn(__fsub_rn(mxv[q], mnv[q]), 255.0f));
        const uint16_t zh = f32_to_f16(mnv[q]);
        if (f16_inf_or_nan(sh) || f16_inf_or_nan(zh)) raise_flag(a.flags, BRS_FLAG_OVERFLOW);
        const float s = f16_to_f32(sh), z = f16_to_f32(zh);
        const float rcp = (s == 0.0f) ? 0.0f : __frcp_rn(s);
        const float tlo = __fmul_rn(__fsub_rn(mnv[q], z), rcp), thi = __fmul_rn(__fsub_rn(mxv[q], z), rcp);
        const bool ok = (tlo >= -0.5f) && (thi < 255.5f);
        ok_all &= ok;
        QPrm pr;
        pr.zz = f2dup(z); pr.rr = f2dup(rcp); pr.ss = f2dup(s); pr.ok = ok; pr.pad = 0;
        sm.prm[i][blk] = pr;
        szout[i * NB + blk] = (uint32_t)sh | ((uint32_t)zh << 16);
      }
    }
    const bool fast = (MODE != BRS_ROUND_STOCHASTIC) && __all_sync(rmask, ok_all);
    __syncwarp();

    // quantize and store: code = clamp(round((y - zero) * (1/scale)), 0, 255);
    // when scale is 0 the factor 1/scale is 0 and every code is 0
    const f2_t magic = f2dup(kRoundMagic);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = row0 + r;
      const QPrm& pr = sm.prm[i][col0 / BLOCK];
      const f2_t t01 = f2mul(f2sub(x[r][0], pr.zz), pr.rr);
      const f2_t t23 = f2mul(f2sub(x[r][1], pr.zz), pr.rr);
      f2_t m01, m23;
      if (fast) {
        // nearest integer (ties to even): the low byte of (t + 1.5*2^23)
        m01 = f2add(t01, magic);
        m23 = f2add(t23, magic);
      } else {
        float c[4] = {f2lo(t01), f2hi(t01), f2lo(t23), f2hi(t23)};
        if constexpr (MODE == BRS_ROUND_STOCHASTIC) {
          const uint4 rnd = philox4x32_10(
              make_uint4((uint32_t)(i * (D / 4) + cb), (uint32_t)a.step, (uint32_t)h, (uint32_t)b),
              make_uint2((uint32_t)a.seed, (uint32_t)(a.seed >> 32)));
          c[0] = sr_round(c[0], rnd.x >> 8);
          c[1] = sr_round(c[1], rnd.y >> 8);
          c[2] = sr_round(c[2], rnd.z >> 8);
          c[3] = sr_round(c[3], rnd.w >> 8);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) c[k] = fminf(fmaxf(c[k], 0.0f), 255.0f);
        m01 = f2add(f2make(c[0], c[1]), magic);
        m23 = f2add(f2make(c[2], c[3]), magic);
      }
      const uint32_t packed4 = __byte_perm(__byte_perm((uint32_t)m01, (uint32_t)(m01 >> 32), 0x0040u),
                                           __byte_perm((uint32_t)m23, (uint32_t)(m23 >> 32), 0x0040u), 0x5410u);
      *(uint32_t*)(hout + (size_t)i * D + col0) = packed4;
      if constexpr (MODE == BRS_ROUND_ERRFEEDBACK) {
        const f2_t q01 = f2fma(f2sub(m01, magic), pr.ss, pr.zz);   // stored value
        const f2_t q23 = f2fma(f2sub(m23, magic), pr.ss, pr.zz);
        const f2_t e01 = f2sub(x[r][0], q01), e23 = f2sub(x[r][1], q23);
        const float s = f2lo(pr.ss);
        float e[4] = {f2lo(e01), f2hi(e01), f2lo(e23), f2hi(e23)};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (e[k] > s) e[k] = s;
          else if (e[k] < -s) e[k] = -s;
        }
        *(uint2*)&auxb[(size_t)i * D + col0] = make_uint2(f16x2_of(e[0], e[1]), f16x2_of(e[2], e[3]));
      }
    }
  }
}

template <int D, int BLOCK, int MODE>
static cudaError_t launch_dbm(const DecodeArgs& a, int store, bool had, cudaStream_t st) {
  const dim3 grid(a.B * a.H), block(2 * D);
  if (store == BRS_STORE_FP32)
    decode_kernel<D, BRS_STORE_FP32, false, D, BRS_ROUND_NEAREST><<<grid, block, 0, st>>>(a);
  else if (had)
    decode_kernel<D, BRS_STORE_DAMP, true, BLOCK, MODE><<<grid, block, 0, st>>>(a);
  else
    decode_kernel<D, BRS_STORE_DAMP, false, BLOCK, MODE><<<grid, block, 0, st>>>(a);
  return cudaGetLastError();
}

template <int D, int BLOCK>
static cudaError_t launch_db(const DecodeArgs& a, int store, bool had, cudaStream_t st) {
  switch (a.mode) {
    case BRS_ROUND_NEAREST: return launch_dbm<D, BLOCK, BRS_ROUND_NEAREST>(a, store, had, st);
    case BRS_ROUND_STOCHASTIC: return launch_dbm<D, BLOCK, BRS_ROUND_STOCHASTIC>(a, store, had, st);
    case BRS_ROUND_ERRFEEDBACK: return launch_dbm<D, BLOCK, BRS_ROUND_ERRFEEDBACK>(a, store, had, st);
  }
  return cudaErrorInvalidValue;
}

bool decode_supported(int d, int block, int k_hi) {
  const bool shape = (d == 128 && (block == 128 || block == 32)) || (d == 64 && block == 64) ||
                     (d == 32 && block == 32);
  return shape && k_hi % (d / 8) == 0 && k_hi <= d / 4;
}

cudaError_t launch_decode(const DecodeArgs& a, int d, int store, bool had, cudaStream_t st) {
  if (store == BRS_STORE_FP32) {
    DecodeArgs f = a;
    f.mode = BRS_ROUND_NEAREST;
    f.k_hi = 0;
    switch (d) {
      case 32: return launch_dbm<32, 32, BRS_ROUND_NEAREST>(f, store, false, st);
      case 64: return launch_dbm<64, 64, BRS_ROUND_NEAREST>(f, store, false, st);
      case 128: return launch_dbm<128, 128, BRS_ROUND_NEAREST>(f, store, false, st);
    }
    return cudaErrorInvalidValue;
  }
  if (d == 128 && a.block == 128) return launch_db<128, 128>(a, store, had, st);
  if (d == 128 && a.block == 32) return launch_db<128, 32>(a, store, had, st);
  if (d == 64 && a.block == 64) return launch_db<64, 64>(a, store, had, st);
  if (d == 32 && a.block == 32) return launch_db<32, 32>(a, store, had, st);
  return cudaErrorInvalidValue;
}

}  // namespace brs
