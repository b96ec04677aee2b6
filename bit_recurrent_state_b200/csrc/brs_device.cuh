// Device helpers shared by the library's kernels: binary16/bfloat16
// conversion, paired FP32 arithmetic (sm_100 f32x2), Philox4x32-10, the
// per-row Hadamard butterflies across the threads of a row group, and the
// device flag word.
#pragma once
#include <cuda_fp16.h>
#include <cstdint>

#include "brs.h"

namespace brs {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
__device__ __forceinline__ float f16_to_f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }
__device__ __forceinline__ uint16_t f32_to_f16(float x) { return __half_as_ushort(__float2half_rn(x)); }
__device__ __forceinline__ bool f16_inf_or_nan(uint16_t h) { return ((h >> 10) & 31u) == 31u; }

// two floats -> f16x2 word (lo = a, hi = b), round to nearest even
__device__ __forceinline__ uint32_t f16x2_of(float a, float b) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}

__device__ __forceinline__ void raise_flag(uint32_t* flags, uint32_t bit) {
  if (flags) atomicOr(flags, bit);
}

// ---- paired FP32 (one instruction, two independent IEEE operations)
__device__ __forceinline__ uint64_t pk(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
// (a0,a1) * (b0,b1) + (c0,c1), each a single-rounding fma
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1,
                                     float c0, float c1) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(pk(a0, a1)), "l"(pk(b0, b1)), "l"(pk(c0, c1)));
  upk(r, d0, d1);
}
__device__ __forceinline__ void mul2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk(a0, a1)), "l"(pk(b0, b1)));
  upk(r, d0, d1);
}
__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk(a0, a1)), "l"(pk(b0, b1)));
  upk(r, d0, d1);
}
__device__ __forceinline__ void sub2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk(a0, a1)), "l"(pk(b0, b1)));
  upk(r, d0, d1);
}

// packed pairs kept in 64-bit registers (no repacking between operations)
typedef unsigned long long f2_t;
__device__ __forceinline__ f2_t f2fma(f2_t a, f2_t b, f2_t c) {
  f2_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ f2_t f2mul(f2_t a, f2_t b) {
  f2_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f2_t f2add(f2_t a, f2_t b) {
  f2_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f2_t f2sub(f2_t a, f2_t b) {
  f2_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float f2lo(f2_t a) { return __uint_as_float((uint32_t)a); }
__device__ __forceinline__ float f2hi(f2_t a) { return __uint_as_float((uint32_t)(a >> 32)); }
__device__ __forceinline__ f2_t f2make(float lo, float hi) { return pk(lo, hi); }
__device__ __forceinline__ f2_t f2dup(float x) { return pk(x, x); }

// The library's order of every sum over key rows (per tier): groups of 8
// consecutive rows, each an fmaf chain in row order from +0, whose sums are
// added in a pairwise tree -- adjacent pairs first, an unpaired last element
// passing up unchanged, until one value remains.  GroupTree takes the group
// sums in row order (up to 16 groups): level k holds the pending left
// operand of a block of 2^k groups, and a block is added to its right
// neighbour as soon as that one is complete, which gives the tree's
// additions.  The result then adds the pending blocks from the smallest
// (rightmost) to the largest: with n groups, the blocks of n's set bits.
template <int C>
struct GroupTree {
  float lv[5][C];
  int n;

  __device__ __forceinline__ GroupTree() : n(0) {}

  __device__ __forceinline__ static void vadd(float (&d)[C], const float (&a)[C], const float (&b)[C]) {
#pragma unroll
    for (int c = 0; c < C; ++c) d[c] = __fadd_rn(a[c], b[c]);
  }
  __device__ __forceinline__ static void vcopy(float (&d)[C], const float (&a)[C]) {
#pragma unroll
    for (int c = 0; c < C; ++c) d[c] = a[c];
  }
  // the next group's sum (consumed)
  __device__ __forceinline__ void push(float (&e)[C]) {
    if ((n & 1) == 0) {
      vcopy(lv[0], e);
    } else {
      vadd(e, lv[0], e);
      if ((n & 2) == 0) {
        vcopy(lv[1], e);
      } else {
        vadd(e, lv[1], e);
        if ((n & 4) == 0) {
          vcopy(lv[2], e);
        } else {
          vadd(e, lv[2], e);
          if ((n & 8) == 0) {
            vcopy(lv[3], e);
          } else {
            vadd(e, lv[3], e);
            vcopy(lv[4], e);
          }
        }
      }
    }
    ++n;
  }
  // the tree's root (+0 when no group was pushed)
  __device__ __forceinline__ void result(float (&out)[C]) const {
    bool have = false;
#pragma unroll
    for (int c = 0; c < C; ++c) out[c] = 0.0f;
#pragma unroll
    for (int k = 0; k < 5; ++k)
      if ((n >> k) & 1) {
        if (have) vadd(out, lv[k], out);
        else vcopy(out, lv[k]);
        have = true;
      }
  }
};

// byte k of w as an exact float: the bits 0x4B0000bb are 2^23 + bb
__device__ __forceinline__ float byte_magic(uint32_t w, int k) {
  return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u | (uint32_t)k));
}
constexpr float kTwo23 = 8388608.0f;          // 2^23
constexpr float kRoundMagic = 12582912.0f;    // 1.5 * 2^23: x + magic rounds to an integer (RNE)

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
  float a0, a1, a2, a3;
  add2(a0, a2, x[0], x[2], x[1], x[3]);
  sub2(a1, a3, x[0], x[2], x[1], x[3]);
  add2(x[0], x[1], a0, a1, a2, a3);
  sub2(x[2], x[3], a0, a1, a2, a3);
#pragma unroll
  for (int m = 1; m < D / 4; m <<= 1) {
    const bool hi = (cb & m) != 0;
    float o[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) o[c] = __shfl_xor_sync(0xffffffffu, x[c], m);
    if (hi) {
      sub2(x[0], x[1], o[0], o[1], x[0], x[1]);
      sub2(x[2], x[3], o[2], o[3], x[2], x[3]);
    } else {
      add2(x[0], x[1], x[0], x[1], o[0], o[1]);
      add2(x[2], x[3], x[2], x[3], o[2], o[3]);
    }
  }
  mul2(x[0], x[1], x[0], x[1], scale, scale);
  mul2(x[2], x[3], x[2], x[3], scale, scale);
}

// Sylvester Hadamard, unnormalised butterflies h = 1, 2, 4, ... then one
// scaling, on a row held by one thread.
template <int D>
__device__ inline void seq_fwht(float* x, float scale) {
  for (int hs = 1; hs < D; hs <<= 1)
    for (int i = 0; i < D; i += 2 * hs)
      for (int j = i; j < i + hs; ++j) {
        const float u0 = x[j], u1 = x[j + hs];
        x[j] = __fadd_rn(u0, u1);
        x[j + hs] = __fsub_rn(u0, u1);
      }
  for (int j = 0; j < D; ++j) x[j] = __fmul_rn(x[j], scale);
}

}  // namespace brs

namespace brs {

// Variable-width row quantizer ("Low-Bit Recurrent States in Hybrid Language
// Models", Levels and storage): levels {-n..n} * step, n = 2^(w-1) - 1,
// step = fp16(f * R / n) with R the row's absolute maximum and f fitted over
// the 16 values f_m = (5+m)/20 by squared error (nearest rounding on the
// target, an fmaf chain over the row's values in order, ties to the smaller
// f).  Candidate m's step and reciprocal; reciprocal 0 when the step is 0.
__device__ __forceinline__ void varbit_candidate(int m, float R, int n, float& step, float& inv,
                                                 uint16_t& bits, bool& valid) {
  const float f = __fdiv_rn((float)(5 + m), 20.0f);
  bits = f32_to_f16(__fdiv_rn(__fmul_rn(f, R), (float)n));
  step = f16_to_f32(bits);
  valid = isfinite(step);
  inv = (step == 0.0f || !valid) ? 0.0f : __frcp_rn(step);
}

// nearest level index of y on a grid with reciprocal step inv, clipped
__device__ __forceinline__ float varbit_nearest(float y, float inv, float fn) {
  const float q = rintf(__fmul_rn(y, inv));
  return fminf(fmaxf(q, -fn), fn);
}

}  // namespace brs
