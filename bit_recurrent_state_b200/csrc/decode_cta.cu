// Decode step for DAMP storage at d = 128: one CTA of 8 warps per head, the
// head's FP32 state held in registers for the whole step.
//
// Warp w owns stored rows 16w .. 16w+15 (one tier each: the number of INT8
// rows, 128 - k_hi, is a multiple of 16), lane l owns columns 4l .. 4l+3 of
// those rows, so a thread holds 64 state values.  Per head:
//   A  every warp dequantizes and decays its 16 rows (each element once) and
//      forms its part of u: the chains of its two 8-row groups, added (the
//      first level of the pairwise tree of the library's row-sum order);
//   -- barrier --
//   W  the last warp finishes u's trees over the warps' parts (INT8 tier and
//      FP16 tier), u = U2 + T(U1), w = beta (v - u), T(w);
//   -- barrier --
//   B  every warp applies the write to its rows (k_i T(w) on INT8 rows, k_i w
//      on FP16 rows), forms its part of o the same way, and requantizes its
//      rows straight from registers: block extremes (redux.sync for a block
//      of 128 columns, shuffles for blocks of 32), the grid of each
//      (row, block), the codes (nearest / Philox stochastic / error
//      feedback), FP16 rows;
//   -- barrier --
//   O  the last warp finishes o's trees, o = O2 + T(O1).
// The arithmetic (and so every stored byte) is the library's documented
// order, the same as the warp-per-head kernel's: 8-row fmaf chains in
// stored order added in a pairwise tree (GroupTree), per tier.
//
// The CTAs are persistent: CTA c takes heads c, c + gridDim, ...  Each
// head's stored bytes, its input vectors (q, k, v, the permutation, the
// per-key decays; the permutation gather then reads shared memory) and, for
// error feedback, its residuals arrive in a shared-memory buffer by bulk
// copies (cp.async.bulk, the TMA engine) with one mbarrier; the copies of
// the CTA's next head are issued when a head starts, so they are in flight
// during the whole step; its scalars (beta, a GDN head's decay) come by
// cp.async on the same mbarrier.  Every wait on a copy is
// bounded (200 ms by %globaltimer): a CTA whose copy does not arrive raises
// BRS_FLAG_TIMEOUT, waits (again bounded) for its copies in flight and
// leaves; all its threads take that decision together at a barrier.
//
// The low tier is INT8 or INT4 (b = 4: a lane's four codes are 16 bits of
// the code row, spread to bytes before the dequantization and gathered back
// after the rounding; the grid divides the block's range by 15).
//
// Sources: DAMP summary, Key Points > Implementation (fused executor:
// reconstruct INT8 channels, update in FP32, re-quantize, write back) and
// Data & Methods > Quantization & calibration details (per-block asymmetric
// quantization with b = 8 or 4 after a Hadamard along the value axis); "Low-Bit Recurrent States in
// Hybrid Language Models", Accumulated readout error (outputs precede
// quantization) and Protocol (quantized and dequantized before reuse).
#include <cuda_runtime.h>
#include <cstdint>
#include <type_traits>

#include "brs_device.cuh"
#include "brs_internal.h"

namespace brs {
namespace {

constexpr int kD = 128, kW = 8, kRW = 16, kC = 4, kThreads = 32 * kW;
// kernel instantiation of k-bit residual memory (modes BRS_ROUND_RESIDUAL2..4; k at run time)
constexpr int kModeResidual = 16;
constexpr unsigned long long kWaitNs = 200000000ull;   // bound on one copy wait (200 ms)
// a head's input vectors at the start of its buffer: q, k, v (bf16), the
// permutation (int16), the per-key decays (f32)
constexpr uint32_t kOffQ = 0, kOffK = 256, kOffV = 512, kOffPerm = 768, kOffDecay = 1024, kOffBeta = 1536,
                   kInBytes = 1552;

struct __align__(16) CtaShared {
  unsigned long long bar[2];     // completion of the two head buffers' copies
  unsigned long long pad_[2];
  float4 ka[kD];                 // per stored row: (k, k, a, a)
  float4 kq[kD];                 // per stored row: (k, k, q, q)
  float4 sz[kD][4];              // per (row, block): (scale, scale, zero, zero)
  float4 upart[kW][32];          // per warp: its two u group sums, added
  float4 opart[kW][32];          // per warp: its two o group sums, added
  float4 wv[32], wtv[32];        // w and T(w)
  uint32_t tmem;                 // base address of the CTA's tensor-memory columns
  float4 prm[kW][8][4];          // per warp: grid (zero, zero, 1/scale, 1/scale) of a batch's (row, block)
  float prs[kW][8][4];           // per warp: the scale of a batch's (row, block)
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void bulk_load(uint32_t bar, uint32_t dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// wait for a phase of a buffer's barrier; false once kWaitNs have passed
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try(bar, parity))
    if (global_ns() - t0 > kWaitNs) return false;
  return true;
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  return mbar_try(bar, parity) || mbar_wait_slow(bar, parity);
}

__device__ __forceinline__ float warp_min(float v) {
  float r;
  asm volatile("redux.sync.min.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ uint32_t warp_or(uint32_t v) {
  uint32_t r;
  asm volatile("redux.sync.or.b32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
  return r;
}

// The paired FP32 instructions take their scalar factors as a register pair
// holding the value twice; shared memory keeps every per-row scalar
// duplicated ((k, k, a, a), (s, s, z, z), ...) so that one 128-bit load
// yields two ready pairs, and the helpers below take both halves.
// four INT8 codes (one u32, column order) -> fmaf(code, scale, zero)
__device__ __forceinline__ void dequant4(float (&x)[4], uint32_t w, const float4 sz) {
  float c0 = byte_magic(w, 0), c1 = byte_magic(w, 1), c2 = byte_magic(w, 2), c3 = byte_magic(w, 3);
  sub2(c0, c1, c0, c1, kTwo23, kTwo23);
  sub2(c2, c3, c2, c3, kTwo23, kTwo23);
  fma2(x[0], x[1], c0, c1, sz.x, sz.y, sz.z, sz.w);
  fma2(x[2], x[3], c2, c3, sz.x, sz.y, sz.z, sz.w);
}
// x *= (a0, a1)
__device__ __forceinline__ void scale4(float (&x)[4], float a0, float a1) {
  mul2(x[0], x[1], x[0], x[1], a0, a1);
  mul2(x[2], x[3], x[2], x[3], a0, a1);
}
// acc += (k0, k1) * x
__device__ __forceinline__ void chain4(float (&acc)[4], float k0, float k1, const float (&x)[4]) {
  fma2(acc[0], acc[1], k0, k1, x[0], x[1], acc[0], acc[1]);
  fma2(acc[2], acc[3], k0, k1, x[2], x[3], acc[2], acc[3]);
}
// x += (k0, k1) * w
__device__ __forceinline__ void axpy4(float (&x)[4], float k0, float k1, const float4 w) {
  fma2(x[0], x[1], k0, k1, w.x, w.y, x[0], x[1]);
  fma2(x[2], x[3], k0, k1, w.z, w.w, x[2], x[3]);
}
__device__ __forceinline__ float min3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ void f16x4_to_f32(float (&x)[4], uint2 h) {
  x[0] = f16_to_f32((uint16_t)(h.x & 0xffffu));
  x[1] = f16_to_f32((uint16_t)(h.x >> 16));
  x[2] = f16_to_f32((uint16_t)(h.y & 0xffffu));
  x[3] = f16_to_f32((uint16_t)(h.y >> 16));
}
__device__ __forceinline__ uint32_t f16x2_overflow(uint32_t w) {
  return (((w >> 10) & 31u) == 31u) | (((w >> 26) & 31u) == 31u);
}

// fl(x / 255) for any float x, as fl32(fl64(x * fl64(1/255))).  The
// quotient of a float by 255 is never a float rounding midpoint and stays
// at least 2^-33 (relative) away from every midpoint (x - 255 M is an odd
// multiple of M's half-ulp scale for any midpoint M), while the double
// product is within 2^-52 of it, so the final rounding is the correctly
// rounded quotient.
__device__ __forceinline__ float div255(float x) { return (float)((double)x * (1.0 / 255.0)); }

// the 4-bit low tier: four codes of 4 bits (16 bits, element e in bits 4e)
// spread to one byte each, and back
__device__ __forceinline__ uint32_t nib_spread(uint32_t w) {
  w = (w | (w << 8)) & 0x00FF00FFu;
  return (w | (w << 4)) & 0x0F0F0F0Fu;
}
__device__ __forceinline__ uint32_t nib_gather(uint32_t w) {
  w = (w | (w >> 4)) & 0x00FF00FFu;
  return (w | (w >> 8)) & 0xFFFFu;
}

// fl(1 / s) for s a positive binary16 value (held as a float): one
// Newton-Raphson correction of the hardware approximation r0,
// r = r0 + r0 (1 - s r0), with the residual 1 - s r0 exact in one fma
// (s has 11 significant bits).  r0 (1 + e) is within 2^-40 (relative) of
// 1/s, while 1/s for an 11-bit s stays at least 2^-36 away from every
// float rounding midpoint, so the fma's single rounding gives the
// correctly rounded reciprocal.
__device__ __forceinline__ float rcp_of_f16(float s) {
  float r0;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(s));
  const float e = __fmaf_rn(-s, r0, 1.0f);
  return __fmaf_rn(r0, e, r0);
}

// Sylvester Hadamard of a 128-vector held 4 values per lane (lane l holds
// elements 4l .. 4l+3): butterflies h = 1, 2, 4, ... then one scaling
__device__ __forceinline__ void fwht128(float (&x)[4], int lane, float scale) {
  float a0, a1, a2, a3;
  a0 = __fadd_rn(x[0], x[1]); a1 = __fsub_rn(x[0], x[1]);
  a2 = __fadd_rn(x[2], x[3]); a3 = __fsub_rn(x[2], x[3]);
  x[0] = __fadd_rn(a0, a2); x[2] = __fsub_rn(a0, a2);
  x[1] = __fadd_rn(a1, a3); x[3] = __fsub_rn(a1, a3);
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool hi = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, x[i], m);
      x[i] = hi ? __fsub_rn(o, x[i]) : __fadd_rn(x[i], o);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) x[i] = __fmul_rn(x[i], scale);
}

// ---- tensor memory: a warp reaches the 32 lanes of its quarter (warp % 4);
// address = (lane << 16) | column.  16 consecutive FP32 columns of this
// thread's lane per instruction.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]),
      "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]), "=f"(v[8]),
        "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void to4(float (&x)[4], const float4 v) { x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w; }

__device__ __forceinline__ float4 add4(const float4 a, const float4 b) {
  return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z), __fadd_rn(a.w, b.w));
}

// The pairwise tree over the parts lo .. lo+n-1 of one tier (n <= 8), read
// from shared memory.  Each part already holds the sum of a warp's two
// 8-row groups (the tree's first level), so the parts are the level-1
// elements of the tier's tree: in that tree the first 4 parts form a
// complete block added to the block of the rest, 2 parts a pair, and so on
// (adjacent pairs first, an unpaired last element passing up).  +0 when
// n = 0.
__device__ __forceinline__ float4 part_tree(const float4 (*part)[32], int lo, int n, int lane) {
  if (n <= 0) return make_float4(0.f, 0.f, 0.f, 0.f);
  auto upto4 = [&](int l, int m) -> float4 {       // 1 <= m <= 4
    if (m == 1) return part[l][lane];
    const float4 p01 = add4(part[l][lane], part[l + 1][lane]);
    if (m == 2) return p01;
    const float4 p23 = (m == 3) ? part[l + 2][lane] : add4(part[l + 2][lane], part[l + 3][lane]);
    return add4(p01, p23);
  };
  if (n <= 4) return upto4(lo, n);
  return add4(upto4(lo, 4), upto4(lo + 4, n - 4));
}

// the INT8 rows of a batch of 8 (rows i0 .. i0+7 of my warp, values xb(r))
// -> codes, grids (and residuals) in global memory
template <int NB, int MODE, int LB>
struct Requant {
  static constexpr bool EF = MODE == BRS_ROUND_ERRFEEDBACK;
  static constexpr bool DM = MODE == BRS_ROUND_DIRECTION;
  static constexpr bool RM = MODE == kModeResidual;
  static constexpr int CR = kD * LB / 8;           // bytes of one code row
  static constexpr float LV = (float)((1 << LB) - 1);   // top code: 255 or 15
  const DecodeArgs& a;
  CtaShared& sm;
  int warp, lane, blk, col0, b, h;
  uint8_t* hout;
  uint32_t* szout;
  const uint16_t* auxs;
  uint16_t* auxg;
  uint32_t& err;
  float one;
  // direction memory: the head's stored bytes in shared memory (the values
  // the step started from) and its 2-bit counters (global, four to a byte);
  // residual memory: its k-bit integers (global, two to a byte) and k
  const uint8_t* hin;
  uint8_t* mem;
  int rmk;

  __device__ __forceinline__ void operator()(float (&xb)[8][kC], int i0) const {
    const int prow = lane & 7;                     // the batch row whose grid this lane computes
    // direction memory: the batch's counter bytes, all loads issued before
    // the first use (they would otherwise wait behind the previous row's stores)
    uint32_t dmo[DM ? 8 : 1] = {};
    if constexpr (DM) {
#pragma unroll
      for (int r = 0; r < 8; ++r) dmo[r] = mem[(size_t)(i0 + r) * (kD / 4) + lane];
    }
    if constexpr (RM) {
      // the target y + m (sprev / 2^k): sprev the block's stored step the
      // token started from, m the k-bit integer kept for the element
      const float rinv = __fdiv_rn(1.0f, (float)(1 << rmk));    // 2^-k, exact
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const uint32_t rw = *(const uint16_t*)(mem + (size_t)(i0 + r) * (kD / 2) + col0 / 2);
        const float su = __fmul_rn(sm.sz[i0 + r][blk].x, rinv);  // exact
#pragma unroll
        for (int c = 0; c < kC; ++c) {
          const int f = (int)((rw >> (4 * c)) & 15u);
          const int m = (f & 8) ? f - 16 : f;
          xb[r][c] = __fadd_rn(xb[r][c], __fmul_rn((float)m, su));
        }
      }
    }
    if constexpr (EF) {
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const uint2 ev = *(const uint2*)(auxs + (size_t)(i0 + r) * kD + col0);
        xb[r][0] = __fadd_rn(xb[r][0], f16_to_f32((uint16_t)(ev.x & 0xffffu)));
        xb[r][1] = __fadd_rn(xb[r][1], f16_to_f32((uint16_t)(ev.x >> 16)));
        xb[r][2] = __fadd_rn(xb[r][2], f16_to_f32((uint16_t)(ev.y & 0xffffu)));
        xb[r][3] = __fadd_rn(xb[r][3], f16_to_f32((uint16_t)(ev.y >> 16)));
      }
    }
    // ---- block extremes; lane l keeps those of row (l & 7) of its block
    float mnv = 0.f, mxv = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float mn = min3(min3(xb[r][0], xb[r][1], xb[r][2]), xb[r][3], xb[r][3]);
      float mx = max3(max3(xb[r][0], xb[r][1], xb[r][2]), xb[r][3], xb[r][3]);
      if constexpr (NB == 1) {
        mn = warp_min(mn);
        mx = warp_max(mx);
      } else {
#pragma unroll
        for (int m = 1; m < 8; m <<= 1) {
          mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, m));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
        }
      }
      if (prow == r) {
        mnv = mn;
        mxv = mx;
      }
    }
    // a zero extreme takes the sign rule (-0 below +0): rare, warp-wide
    if (__any_sync(0xffffffffu, (mnv == 0.0f) || (mxv == 0.0f))) {
      uint32_t nz = 0, pz = 0;
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < kC; ++c)
          if (xb[r][c] == 0.0f) {
            if (signbit(xb[r][c])) nz |= 1u << r; else pz |= 1u << r;
          }
      if constexpr (NB == 1) {
        nz = warp_or(nz);
        pz = warp_or(pz);
      } else {
#pragma unroll
        for (int m = 1; m < 8; m <<= 1) {
          nz |= __shfl_xor_sync(0xffffffffu, nz, m);
          pz |= __shfl_xor_sync(0xffffffffu, pz, m);
        }
      }
      if (mnv == 0.0f) mnv = ((nz >> prow) & 1u) ? -0.0f : 0.0f;
      if (mxv == 0.0f) mxv = ((pz >> prow) & 1u) ? 0.0f : -0.0f;
    }
    // the grid: scale = fp16(fl((max - min) / 255)), zero = fp16(min); ok =
    // the block's extreme grid coordinates (the same monotone FP32
    // operations as its elements') round into [0, 255]
    bool ok;
    {
      const float rng = __fsub_rn(mxv, mnv);
      const uint32_t g = f16x2_of(LB == 8 ? div255(rng) : __fdiv_rn(rng, LV), mnv);   // lo scale, hi zero
      const float sc = f16_to_f32((uint16_t)(g & 0xffffu)), z = f16_to_f32((uint16_t)(g >> 16));
      err |= (!isfinite(mnv) || !isfinite(mxv)) ? BRS_FLAG_NONFINITE : 0u;
      err |= f16x2_overflow(g) ? BRS_FLAG_OVERFLOW : 0u;
      const float rcp = (sc == 0.0f) ? 0.0f : rcp_of_f16(sc);
      float tlo, thi;
      sub2(tlo, thi, mnv, mxv, z, z);
      mul2(tlo, thi, tlo, thi, rcp, rcp);
      ok = (tlo >= -0.5f) && (thi < LV + 0.5f);
      if (NB == 4 || lane < 8) {
        sm.prm[warp][prow][blk] = make_float4(z, z, rcp, rcp);
        if constexpr (EF || DM || RM) sm.prs[warp][prow][blk] = sc;
        szout[(i0 + prow) * NB + blk] = g;
      }
    }
    const bool fast = (MODE != BRS_ROUND_STOCHASTIC) && __all_sync(0xffffffffu, ok);
    __syncwarp();
    // ---- codes: clamp(round((y - zero) * (1/scale)), 0, 255); a zero
    // scale has 1/scale = 0, so every code of the block is 0
    if (fast) codes<false>(xb, i0, dmo);
    else codes<true>(xb, i0, dmo);
    __syncwarp();                                  // prm reused by the next batch
  }

  template <bool CLIP>
  __device__ __forceinline__ void codes(float (&xb)[8][kC], int i0, const uint32_t* dmo) const {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int i = i0 + r;
      const float4 p = sm.prm[warp][r][blk];     // (zero, zero, 1/scale, 1/scale)
      float tq[kC];
      sub2(tq[0], tq[1], xb[r][0], xb[r][1], p.x, p.y);
      sub2(tq[2], tq[3], xb[r][2], xb[r][3], p.x, p.y);
      mul2(tq[0], tq[1], tq[0], tq[1], p.z, p.w);
      mul2(tq[2], tq[3], tq[2], tq[3], p.z, p.w);
      if constexpr (CLIP) {
        if constexpr (MODE == BRS_ROUND_STOCHASTIC) {
          const int e0 = i * kD + col0;
          const uint4 rnd = philox4x32_10(make_uint4((uint32_t)(e0 / 4), (uint32_t)a.step, (uint32_t)h, (uint32_t)b),
                                          make_uint2((uint32_t)a.seed, (uint32_t)(a.seed >> 32)));
          tq[0] = sr_round(tq[0], rnd.x >> 8);
          tq[1] = sr_round(tq[1], rnd.y >> 8);
          tq[2] = sr_round(tq[2], rnd.z >> 8);
          tq[3] = sr_round(tq[3], rnd.w >> 8);
        }
#pragma unroll
        for (int c = 0; c < kC; ++c) tq[c] = fminf(fmaxf(tq[c], 0.0f), LV);
      }
      // nearest integer (ties to even): the low byte of t + 1.5*2^23, the
      // add written as t * 1 + magic with the 1 read at run time, so that it
      // stays a separately rounded operation after the multiply (the sum is
      // the same single rounding as an add)
      float mq[kC];
      fma2(mq[0], mq[1], tq[0], tq[1], one, one, kRoundMagic, kRoundMagic);
      fma2(mq[2], mq[3], tq[2], tq[3], one, one, kRoundMagic, kRoundMagic);
      if constexpr (DM) {
        // votes of the proposed changes y - xp inside (scale/8, scale/2), xp
        // the stored value the step started from (dequantized again from the
        // head's bytes in shared memory); a counter at +-2 moves the nearest
        // code one level (clipped to [0, LV]) and is reset.  A lane's four
        // counters are one byte.
        float xp[kC];
        if constexpr (LB == 8) dequant4(xp, *(const uint32_t*)(hin + (size_t)i * CR + col0), sm.sz[i][blk]);
        else dequant4(xp, nib_spread(*(const uint16_t*)(hin + (size_t)i * CR + col0 / 2)), sm.sz[i][blk]);
        uint8_t* dmp = mem + (size_t)i * (kD / 4) + lane;
        const uint32_t old = dmo[r];
        const float sc = sm.prs[warp][r][blk];
        const float lo = __fmul_rn(sc, 0.125f), hi = __fmul_rn(sc, 0.5f);
        uint32_t nb = 0;
#pragma unroll
        for (int c = 0; c < kC; ++c) {
          const int f = (int)((old >> (2 * c)) & 3u);
          int m = (f & 2) ? f - 4 : f;
          const float dl = __fsub_rn(xb[r][c], xp[c]);
          const float ad = fabsf(dl);
          if (ad > lo && ad < hi) m += (dl > 0.0f) ? 1 : -1;
          if (m >= 2 || m <= -2) {
            const uint32_t mb = __float_as_uint(mq[c]);
            const int code = min(max((int)(mb & 0xffu) + (m > 0 ? 1 : -1), 0), (int)LV);
            mq[c] = __uint_as_float((mb & ~0xffu) | (uint32_t)code);
            m = 0;
          }
          nb |= ((uint32_t)m & 3u) << (2 * c);
        }
        *dmp = (uint8_t)nb;
      }
      if constexpr (RM) {
        // the new integers: rne((y - value) * (1/scale) * 2^k), clipped to
        // +-(2^(k-1) - 1); a lane's four are 16 bits
        const float unit = (float)(1 << rmk);
        const int rmax = (1 << (rmk - 1)) - 1;
        const float sc = sm.prs[warp][r][blk];
        uint32_t nb = 0;
#pragma unroll
        for (int c = 0; c < kC; ++c) {
          const float code = __fsub_rn(mq[c], kRoundMagic);          // exact
          const float res = __fsub_rn(xb[r][c], __fmaf_rn(code, sc, p.x));
          const float q = rintf(__fmul_rn(__fmul_rn(res, p.z), unit));
          const int m = (q != q) ? 0 : (int)fminf(fmaxf(q, (float)-rmax), (float)rmax);
          nb |= ((uint32_t)m & 15u) << (4 * c);
        }
        *(uint16_t*)(mem + (size_t)i * (kD / 2) + col0 / 2) = (uint16_t)nb;
      }
      const uint32_t cw = __byte_perm(__byte_perm(__float_as_uint(mq[0]), __float_as_uint(mq[1]), 0x0040u),
                                      __byte_perm(__float_as_uint(mq[2]), __float_as_uint(mq[3]), 0x0040u), 0x5410u);
      if constexpr (LB == 8) *(uint32_t*)(hout + (size_t)i * CR + col0) = cw;
      else *(uint16_t*)(hout + (size_t)i * CR + col0 / 2) = (uint16_t)nib_gather(cw);
      if constexpr (EF) {
        const float sc = sm.prs[warp][r][blk];
        uint16_t ev[kC];
#pragma unroll
        for (int c = 0; c < kC; ++c) {
          const float code = __fsub_rn(mq[c], kRoundMagic);          // exact
          float e = __fsub_rn(xb[r][c], __fmaf_rn(code, sc, p.x));
          if (e > sc) e = sc;
          else if (e < -sc) e = -sc;
          ev[c] = f32_to_f16(e);
        }
        *(uint2*)(auxg + (size_t)i * kD + col0) =
            make_uint2((uint32_t)ev[0] | ((uint32_t)ev[1] << 16), (uint32_t)ev[2] | ((uint32_t)ev[3] << 16));
      }
    }
  }
};

// o = O2 + T(O1) of head `head` from the warps' o parts (one warp)
template <bool HAD>
__device__ __forceinline__ void out_o(const CtaShared& sm, const DecodeArgs& a, int nw8, int lane, int col0, int head,
                                      uint32_t& err) {
  float o1[kC], o2[kC];
  to4(o1, part_tree(sm.opart, 0, nw8, lane));
  to4(o2, part_tree(sm.opart, nw8, kW - nw8, lane));
  if constexpr (HAD) fwht128(o1, lane, a.hscale);
  bool bad = false;
  float ov[kC];
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    ov[c] = __fadd_rn(o2[c], o1[c]);
    bad |= !isfinite(ov[c]);
  }
  err |= bad ? BRS_FLAG_NONFINITE : 0u;
  *(float4*)(a.o + (size_t)head * kD + col0) = make_float4(ov[0], ov[1], ov[2], ov[3]);
}

template <bool HAD, int BLOCK, int MODE, int LB, bool DEF>
__global__ void __launch_bounds__(kThreads, 3) decode_cta_kernel(const DecodeArgs a) {
  constexpr int NB = kD / BLOCK;                   // blocks per row: 1 (whole row) or 4
  // deferred write-back (write-back every C > 1 tokens): rows come from the
  // FP32 interval state when src32 is set, and go to it instead of the
  // write-back when dst32 is set (DEF instantiations only)
  const bool src32 = DEF && a.src32, dst32 = DEF && a.dst32;
  constexpr int CR = kD * LB / 8;                  // bytes of one code row (INT8 or INT4)
  static_assert(NB == 1 || NB == 4, "blocks of 128 or 32 columns");
  constexpr bool EF = MODE == BRS_ROUND_ERRFEEDBACK;
  extern __shared__ __align__(128) uint8_t dsm[];
  CtaShared& sm = *reinterpret_cast<CtaShared*>(dsm);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nlo = kD - a.k_hi;                     // INT8 rows 0 .. nlo-1, FP16 rows after
  const int nw8 = nlo / kRW;                       // INT8 warps
  const int r0 = warp * kRW;                       // my first stored row
  const bool int8w = r0 < nlo;
  const bool wwarp = warp == kW - 1;               // the warp that forms w
  const bool owarp = warp == kW - 2;               // the warp that forms o (of the previous head)
  const int col0 = kC * lane;
  const int blk = (NB == 1) ? 0 : lane / 8;        // my block of a row
  const int heads = a.B * a.H;
  const uint32_t hbp = (uint32_t)((a.head_bytes + 127) & ~(size_t)127);
  const uint32_t aux_bytes = (uint32_t)nlo * kD * 2;            // residuals of one head
  const uint32_t auxp = (aux_bytes + 127u) & ~127u;
  // buffer j: the head's input vectors (kInBytes), then its stored bytes;
  // after both buffers, the two residual buffers (error feedback)
  uint8_t* bufs = dsm + sizeof(CtaShared);
  const uint32_t bstride = kInBytes + hbp;
  const uint32_t bar0 = smem_u32(&sm.bar[0]);
  // heads advance by gridDim.x: (sequence, head) advance by (gq, gr)
  const int gq = (int)gridDim.x / a.H, gr = (int)gridDim.x - gq * a.H;

  // the copies of head (hb_, hh) = hd into buffer j (thread 0): q, k, v, the
  // permutation and the per-key decays (16-byte aligned rows of 256 or 512
  // bytes), the stored bytes, the residuals by the bulk-copy engine; beta
  // and a GDN head's decay (4 bytes each) by cp.async, whose completion
  // arrives on the same barrier (two arrivals per phase)
  auto issue = [&](int hd, int hb_, int hh, int j) {
    const uint32_t bar = bar0 + 8u * j;
    const size_t qk = ((size_t)hb_ * a.Hk + hh * a.Hk / a.H) * kD;
    const uint32_t in = smem_u32(bufs + j * bstride);
    // the stored bytes are read only when the rows come from them; the
    // residuals only at a write-back
    const bool codes_in = !src32, ef_in = EF && !dst32;
    const uint32_t tx = (codes_in ? (uint32_t)a.head_bytes : 0u) + 3u * kD * 2 + (a.perm ? kD * 2u : 0u) +
                        (a.decay_per_key ? kD * 4u : 0u) + (ef_in ? aux_bytes : 0u) + a.tx_extra;
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(in + kOffBeta), "l"(a.beta + hd) : "memory");
    if (!a.decay_per_key)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(in + kOffDecay), "l"(a.decay + hd) : "memory");
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
    expect_tx(bar, tx);
    bulk_load(bar, in + kOffQ, a.q + qk, kD * 2);
    bulk_load(bar, in + kOffK, a.k + qk, kD * 2);
    bulk_load(bar, in + kOffV, a.v + (size_t)hd * kD, kD * 2);
    if (a.perm) bulk_load(bar, in + kOffPerm, a.perm + (size_t)hh * kD, kD * 2);
    if (a.decay_per_key) bulk_load(bar, in + kOffDecay, a.decay + (size_t)hd * kD, kD * 4);
    if (codes_in)
      bulk_load(bar, in + kInBytes, (const uint8_t*)a.packed_in + (size_t)hd * a.head_bytes, (uint32_t)a.head_bytes);
    if (ef_in && aux_bytes > 0)
      bulk_load(bar, smem_u32(bufs + 2 * bstride + j * auxp), (const uint8_t*)a.aux + (size_t)hd * aux_bytes,
                aux_bytes);
  };
  int b = (int)blockIdx.x / a.H, h = (int)blockIdx.x - b * a.H;    // the current head's (sequence, head)
  if (warp == 0) {
    // 128 tensor-memory columns: warp w keeps its 16 rows x 4 columns in
    // columns 64 (w / 4) .. +63 of its lane quarter, row r at columns 4r..4r+3
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)),
                 "r"(128));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 2;" ::"r"(bar0));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 2;" ::"r"(bar0 + 8u));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t trow = sm.tmem + ((uint32_t)(32 * (warp % 4)) << 16) + 64u * (uint32_t)(warp / 4);
  if (threadIdx.x == 0 && (int)blockIdx.x < heads) issue(blockIdx.x, b, h, 0);

  uint32_t err = 0;                                // flag bits, raised once at the end
  const float one = a.one;                         // 1, read at run time
  bool alive = true;
  int prev_head = -1;                              // the head whose o is still to be formed
  for (int it = 0;; ++it) {
    const int head = blockIdx.x + it * gridDim.x;
    if (head >= heads) break;
    const int j = it & 1;
    const uint32_t parity = (uint32_t)((it >> 1) & 1);
    const int next = head + gridDim.x;
    int bn = b + gq, hn = h + gr;                  // the next head's (sequence, head)
    if (hn >= a.H) {
      hn -= a.H;
      ++bn;
    }
    // ---- A: wait for the head's copies
    const bool ok_wait = __all_sync(0xffffffffu, mbar_wait(bar0 + 8u * j, parity));   // warp-uniform
    const uint8_t* inb = bufs + j * bstride;
    const uint8_t* hb = inb + kInBytes;
    __syncwarp();                                  // my warp's reads of the previous head's rows are done
    if (ok_wait) {
      // my rows' inputs, gathered through the permutation from the copied
      // vectors; the grids of my INT8 rows, as ready pairs
      if (lane < kRW) {
        const int i = r0 + lane;
        const int p = a.perm ? ((const int16_t*)(inb + kOffPerm))[i] : i;
        const float kv = bf16_to_f32(((const uint16_t*)(inb + kOffK))[p]);
        const float qv = bf16_to_f32(((const uint16_t*)(inb + kOffQ))[p]);
        const float av = ((const float*)(inb + kOffDecay))[a.decay_per_key ? p : 0];
        sm.ka[i] = make_float4(kv, kv, av, av);
        sm.kq[i] = make_float4(kv, kv, qv, qv);
      }
      if (int8w && !src32) {
        const uint32_t* szin = (const uint32_t*)(hb + (size_t)nlo * CR + (size_t)a.k_hi * kD * 2);
#pragma unroll
        for (int e = lane; e < kRW * NB; e += 32) {
          const int i = r0 + e / NB, bb = e % NB;
          const uint32_t g = szin[i * NB + bb];
          const float sv = f16_to_f32((uint16_t)(g & 0xffffu)), zv = f16_to_f32((uint16_t)(g >> 16));
          sm.sz[i][bb] = make_float4(sv, sv, zv, zv);
        }
      }
      __syncwarp();
      // two rounds of 8 rows (rows q..q+3 and q+8..q+11, q = 0, 4): the two
      // groups' chains side by side; each round's rows go to tensor memory
      float g0[kC] = {0.f, 0.f, 0.f, 0.f}, g1[kC] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 8; q += 4) {
        float xa[4][kC], xc[4][kC];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int ra = q + r, rc = q + r + 8;
          const float4 ka = sm.ka[r0 + ra], kc = sm.ka[r0 + rc];
          if (src32) {
            // the interval state's rows (stored order, each tier in its basis)
            const float* srow = a.s32 + ((size_t)head * kD + r0) * kD + col0;
            to4(xa[r], __ldg((const float4*)(srow + (size_t)ra * kD)));
            to4(xc[r], __ldg((const float4*)(srow + (size_t)rc * kD)));
          } else if (int8w) {
            const uint8_t* crow = hb + (size_t)r0 * CR + col0 * LB / 8;
            if constexpr (LB == 8) {
              dequant4(xa[r], *(const uint32_t*)(crow + ra * CR), sm.sz[r0 + ra][blk]);
              dequant4(xc[r], *(const uint32_t*)(crow + rc * CR), sm.sz[r0 + rc][blk]);
            } else {
              dequant4(xa[r], nib_spread(*(const uint16_t*)(crow + ra * CR)), sm.sz[r0 + ra][blk]);
              dequant4(xc[r], nib_spread(*(const uint16_t*)(crow + rc * CR)), sm.sz[r0 + rc][blk]);
            }
          } else {
            const uint8_t* frow = hb + (size_t)nlo * CR + (size_t)(r0 - nlo) * kD * 2 + 2 * col0;
            f16x4_to_f32(xa[r], *(const uint2*)(frow + ra * kD * 2));
            f16x4_to_f32(xc[r], *(const uint2*)(frow + rc * kD * 2));
          }
          scale4(xa[r], ka.z, ka.w);
          scale4(xc[r], kc.z, kc.w);
          chain4(g0, ka.x, ka.y, xa[r]);
          chain4(g1, kc.x, kc.y, xc[r]);
        }
        tmem_st16(trow + 4u * q, &xa[0][0]);
        tmem_st16(trow + 4u * (q + 8), &xc[0][0]);
      }
      sm.upart[warp][lane] = make_float4(__fadd_rn(g0[0], g1[0]), __fadd_rn(g0[1], g1[1]),
                                         __fadd_rn(g0[2], g1[2]), __fadd_rn(g0[3], g1[3]));
      tmem_wait_st();
    }
    if (!__syncthreads_and(ok_wait)) {
      // a copy did not arrive: wait (bounded) for the copies still in
      // flight, raise the flag, leave together (tensor memory is freed below)
      if (threadIdx.x == 0) {
        mbar_wait(bar0 + 8u * j, parity);
        if (next < heads) mbar_wait(bar0 + 8u * (j ^ 1), (uint32_t)(((it + 1) >> 1) & 1));
      }
      alive = false;
      break;
    }
    // every warp is past the previous head's phase B, the last reader of
    // buffer j^1: the next head's copies go there
    if (threadIdx.x == 0 && next < heads) issue(next, bn, hn, j ^ 1);
    // my first batch of rows starts back from tensor memory during the W step
    float xb0[8][kC];
    tmem_ld16(trow, &xb0[0][0]);
    tmem_ld16(trow + 16u, &xb0[4][0]);

    // ---- W: u = U2 + T(U1), w = beta (v - u), T(w); and, by another warp,
    // O of the previous head
    if (owarp && prev_head >= 0) out_o<HAD>(sm, a, nw8, lane, col0, prev_head, err);
    if (wwarp) {
      float u1[kC], u2[kC], w[kC], wt[kC], vv[kC];
      to4(u1, part_tree(sm.upart, 0, nw8, lane));
      to4(u2, part_tree(sm.upart, nw8, kW - nw8, lane));
      const float beta = *(const float*)(inb + kOffBeta);
      {
        const uint2 vw = *(const uint2*)(inb + kOffV + 2 * col0);
        vv[0] = bf16_to_f32((uint16_t)(vw.x & 0xffffu)); vv[1] = bf16_to_f32((uint16_t)(vw.x >> 16));
        vv[2] = bf16_to_f32((uint16_t)(vw.y & 0xffffu)); vv[3] = bf16_to_f32((uint16_t)(vw.y >> 16));
      }
      if constexpr (HAD) fwht128(u1, lane, a.hscale);
      bool bad = false;
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        const float u = __fadd_rn(u2[c], u1[c]);
        bad |= !isfinite(u);
        w[c] = __fmul_rn(beta, __fsub_rn(vv[c], u));
        wt[c] = w[c];
      }
      err |= bad ? BRS_FLAG_NONFINITE : 0u;
      if constexpr (HAD) fwht128(wt, lane, a.hscale);
      sm.wv[lane] = make_float4(w[0], w[1], w[2], w[3]);
      sm.wtv[lane] = make_float4(wt[0], wt[1], wt[2], wt[3]);
    }
    __syncthreads();

    // ---- B: per batch of 8 rows: back from tensor memory, the write, o's
    // part, then the write-back of the rows
    uint8_t* hout = (uint8_t*)a.packed_out + (size_t)head * a.head_bytes;
    {
      const float4 wl = int8w ? sm.wtv[lane] : sm.wv[lane];
      float ga[kC] = {0.f, 0.f, 0.f, 0.f}, gb[kC] = {0.f, 0.f, 0.f, 0.f};
      uint8_t* mem = nullptr;                      // direction counters / residual integers of the head
      if constexpr (MODE == BRS_ROUND_DIRECTION) mem = (uint8_t*)a.aux + (size_t)head * nlo * (kD / 4);
      if constexpr (MODE == kModeResidual) mem = (uint8_t*)a.aux + (size_t)head * nlo * (kD / 2);
      const Requant<NB, MODE, LB> rq{a, sm, warp, lane, blk, col0, b, h, hout,
                                     (uint32_t*)(hout + (size_t)nlo * CR + (size_t)a.k_hi * kD * 2),
                                     EF ? (const uint16_t*)(bufs + 2 * bstride + j * auxp) : nullptr,
                                     EF ? (uint16_t*)a.aux + (size_t)head * nlo * kD : nullptr, err, one,
                                     hb, mem, a.mode - BRS_ROUND_RESIDUAL2 + 2};
      uint32_t ovf = 0;
#pragma unroll
      for (int bt = 0; bt < 2; ++bt) {
        float xb[8][kC];
        if (bt == 0) {
          tmem_wait_ld();
#pragma unroll
          for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int c = 0; c < kC; ++c) xb[r][c] = xb0[r][c];
        } else {
          tmem_ld16(trow + 32u, &xb[0][0]);
          tmem_ld16(trow + 48u, &xb[4][0]);
          tmem_wait_ld();
        }
        float (&g)[kC] = bt ? gb : ga;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float4 kq = sm.kq[r0 + 8 * bt + r];
          axpy4(xb[r], kq.x, kq.y, wl);
          chain4(g, kq.z, kq.w, xb[r]);
        }
        if (dst32) {
          // the updated rows to the interval state instead of a write-back
          float* drow = a.s32 + ((size_t)head * kD + r0 + 8 * bt) * kD + col0;
#pragma unroll
          for (int r = 0; r < 8; ++r)
            *(float4*)(drow + (size_t)r * kD) = make_float4(xb[r][0], xb[r][1], xb[r][2], xb[r][3]);
        } else if (int8w) {
          rq(xb, r0 + 8 * bt);
        } else {
          // protected rows: FP16, nearest
          uint16_t* f16out = (uint16_t*)(hout + (size_t)nlo * CR) + (size_t)(r0 + 8 * bt - nlo) * kD + col0;
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const uint32_t lo = f16x2_of(xb[r][0], xb[r][1]), hi = f16x2_of(xb[r][2], xb[r][3]);
            ovf |= f16x2_overflow(lo) | f16x2_overflow(hi);
            *(uint2*)(f16out + (size_t)r * kD) = make_uint2(lo, hi);
          }
        }
      }
      err |= ovf ? BRS_FLAG_OVERFLOW : 0u;
      sm.opart[warp][lane] = make_float4(__fadd_rn(ga[0], gb[0]), __fadd_rn(ga[1], gb[1]),
                                         __fadd_rn(ga[2], gb[2]), __fadd_rn(ga[3], gb[3]));
    }
    prev_head = head;
    b = bn;
    h = hn;
  }
  // every warp is past its last phase B (o's parts written) and its last
  // tensor-memory access
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (owarp && alive && prev_head >= 0) out_o<HAD>(sm, a, nw8, lane, col0, prev_head, err);
  if (!alive && threadIdx.x == 0) raise_flag(a.flags, BRS_FLAG_TIMEOUT);
  if (err) raise_flag(a.flags, err);
  // free the tensor-memory columns
  if (warp == 0) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(sm.tmem), "r"(128));
  }
}

template <bool HAD, int BLOCK, int MODE, int LB, bool DEF>
cudaError_t launch_hbm(const DecodeArgs& a, cudaStream_t st) {
  const int heads = a.B * a.H;
  const size_t hbp = (a.head_bytes + 127) & ~(size_t)127;
  const size_t auxp = ((size_t)(kD - a.k_hi) * kD * 2 + 127) & ~(size_t)127;
  const size_t smem = sizeof(CtaShared) + 2 * (kInBytes + hbp) + (MODE == BRS_ROUND_ERRFEEDBACK ? 2 * auxp : 0);
  auto kern = decode_cta_kernel<HAD, BLOCK, MODE, LB, DEF>;
  // per instantiation: the opt-in shared-memory size (largest seen) and the
  // device's SM count
  static size_t set_smem = 0;
  static int sms = 0;
  if (smem > set_smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)   // all of the SM's unified memory as shared memory: several CTAs per SM
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    set_smem = smem;
  }
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      sms = 148;
  }
  // CTAs per SM from the kernel's own resources: registers, shared memory
  // (plus the 1 KB the driver reserves per CTA) and the SM's 512
  // tensor-memory columns (128 per CTA)
  static int per_sm = 0;
  static size_t per_sm_smem = 0;
  if (per_sm == 0 || per_sm_smem != smem) {
    int dev = 0, smem_sm = 0;
    cudaFuncAttributes fa{};
    per_sm = 1;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) == cudaSuccess &&
        cudaFuncGetAttributes(&fa, kern) == cudaSuccess && fa.numRegs > 0) {
      const int by_regs = 65536 / (fa.numRegs * kThreads);
      const int by_smem = smem_sm / (int)(smem + 1024);
      const int by_tmem = 512 / 128;
      per_sm = by_regs < by_smem ? by_regs : by_smem;
      if (per_sm > by_tmem) per_sm = by_tmem;
      if (per_sm < 1) per_sm = 1;
    }
    per_sm_smem = smem;
  }
  const int grid = heads < per_sm * sms ? heads : per_sm * sms;
  kern<<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <bool HAD, int BLOCK, int LB>
cudaError_t launch_hbl(const DecodeArgs& a, cudaStream_t st) {
  if (a.src32 || a.dst32) {
    // a token inside a write-back interval (the deferred instantiations)
    switch (a.mode) {
      case BRS_ROUND_NEAREST: return launch_hbm<HAD, BLOCK, BRS_ROUND_NEAREST, LB, true>(a, st);
      case BRS_ROUND_STOCHASTIC: return launch_hbm<HAD, BLOCK, BRS_ROUND_STOCHASTIC, LB, true>(a, st);
      case BRS_ROUND_ERRFEEDBACK: return launch_hbm<HAD, BLOCK, BRS_ROUND_ERRFEEDBACK, LB, true>(a, st);
    }
    return cudaErrorInvalidValue;
  }
  switch (a.mode) {
    case BRS_ROUND_NEAREST: return launch_hbm<HAD, BLOCK, BRS_ROUND_NEAREST, LB, false>(a, st);
    case BRS_ROUND_STOCHASTIC: return launch_hbm<HAD, BLOCK, BRS_ROUND_STOCHASTIC, LB, false>(a, st);
    case BRS_ROUND_ERRFEEDBACK: return launch_hbm<HAD, BLOCK, BRS_ROUND_ERRFEEDBACK, LB, false>(a, st);
    case BRS_ROUND_DIRECTION: return launch_hbm<HAD, BLOCK, BRS_ROUND_DIRECTION, LB, false>(a, st);
    case BRS_ROUND_RESIDUAL2:
    case BRS_ROUND_RESIDUAL3:
    case BRS_ROUND_RESIDUAL4: return launch_hbm<HAD, BLOCK, kModeResidual, LB, false>(a, st);
  }
  return cudaErrorInvalidValue;
}

// the low tier's width: 8 (INT8) or 4 (two codes per byte)
template <bool HAD, int BLOCK>
cudaError_t launch_hb(const DecodeArgs& a, cudaStream_t st) {
  return a.low_bits == 4 ? launch_hbl<HAD, BLOCK, 4>(a, st) : launch_hbl<HAD, BLOCK, 8>(a, st);
}

}  // namespace

bool decode_cta_supported(int d, int store, int block, int k_hi, int mode) {
  return d == kD && store == BRS_STORE_DAMP && (block == 128 || block == 32) && k_hi % kRW == 0 &&
         mode >= BRS_ROUND_NEAREST && mode <= BRS_ROUND_RESIDUAL4;
}

cudaError_t launch_decode_cta(const DecodeArgs& a, bool had, cudaStream_t st) {
  if (a.block == 128) return had ? launch_hb<true, 128>(a, st) : launch_hb<false, 128>(a, st);
  if (a.block == 32) return had ? launch_hb<true, 32>(a, st) : launch_hb<false, 32>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace brs
