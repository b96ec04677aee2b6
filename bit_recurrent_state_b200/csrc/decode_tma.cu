// Decode step for DAMP storage at d = 128 with the stored rows staged
// through shared memory by the bulk-copy (TMA) engine.
//
// One warp per head, lane l owning columns 4l .. 4l+3 of every row, as in
// the general decode kernel; the arithmetic (and so every stored byte and
// every output) is the same:
//   u = U2 + T(U1), w = beta (v - u), S_i += k_i T(w) (INT8 rows, Hadamard
//   basis), S_i += k_i w (FP16 rows), o = O2 + T(O1),
// U1/O1 and U2/O2 fmaf chains over the INT8 and FP16 rows in stored order.
// What differs is how the rows arrive and how a block's extremes are found:
//   * the head's stored rows are cut into 2 KB slots (16 INT8 rows or 8 FP16
//     rows) and streamed twice (pass 1: u; pass 2: write, o, requantize)
//     through a per-warp ring of shared-memory stages filled by
//     cp.async.bulk with mbarrier completion, so each warp keeps several KB
//     of loads in flight without holding them in registers;
//   * a row's min and max over its 128-column block come from one
//     redux.sync.{min,max}.f32 each (sm_100a) instead of a shuffle tree;
//   * the clip test of a batch is taken once, outside the row loop.
//
// Sources: DAMP summary, Key Points > Implementation (fused executor:
// reconstruct INT8 channels, update in FP32, re-quantize, write back) and
// Data & Methods > Quantization & calibration details (per-block asymmetric
// INT8 after a Hadamard along the value axis); "Low-Bit Recurrent States in
// Hybrid Language Models", Accumulated readout error and Protocol.
#include <cuda_runtime.h>
#include <cstdint>
#include <type_traits>

#include "brs_device.cuh"
#include "brs_internal.h"

namespace brs {
namespace {

constexpr int kD = 128, kC = 4, kNrb = 8;
constexpr int kTmaWarps = 1;                       // heads per CTA (one: finest spread over the SMs)
constexpr int kSlot = 2048;                        // bytes per ring stage
constexpr int kStages = 3;                         // ring stages while every head is resident at once
constexpr int kRows8 = kSlot / kD;                 // INT8 rows per slot
constexpr int kRows16 = kSlot / (2 * kD);          // FP16 rows per slot
constexpr unsigned long long kWaitNs = 200000000ull;   // bound on one slot wait (200 ms)

struct __align__(16) Scal {
  float4 ka, sz;                                   // (k, k, a, a), (s, s, z, z)
};

template <int NST>
struct __align__(128) TmaSmem {
  uint8_t ring[NST][kSlot];
  Scal rs[kD];
  float2 qq[kD];
  float4 prm[kNrb][4];                             // (zero, 1/scale, scale, -) per (batch row, block)
  unsigned long long bar[NST];
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void bulk_load(uint32_t bar, uint32_t dst, const void* src, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
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

// wait for a phase of a stage's barrier; false once kWaitNs have passed
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

// value of entry (lane & 7) of an 8-entry register array
__device__ __forceinline__ float pick8(const float (&v)[8], int lane) {
  const bool b0 = lane & 1, b1 = lane & 2, b2 = lane & 4;
  const float a0 = b0 ? v[1] : v[0], a1 = b0 ? v[3] : v[2], a2 = b0 ? v[5] : v[4], a3 = b0 ? v[7] : v[6];
  const float c0 = b1 ? a1 : a0, c1 = b1 ? a3 : a2;
  return b2 ? c1 : c0;
}

// four INT8 codes (one u32, column order) -> fmaf(code, scale, zero)
__device__ __forceinline__ void dequant4(float (&x)[4], uint32_t w, float s, float z) {
  float c0 = byte_magic(w, 0), c1 = byte_magic(w, 1), c2 = byte_magic(w, 2), c3 = byte_magic(w, 3);
  sub2(c0, c1, c0, c1, kTwo23, kTwo23);
  sub2(c2, c3, c2, c3, kTwo23, kTwo23);
  fma2(x[0], x[1], c0, c1, s, s, z, z);
  fma2(x[2], x[3], c2, c3, s, s, z, z);
}

__device__ __forceinline__ void scale4(float (&x)[4], float a) {
  mul2(x[0], x[1], x[0], x[1], a, a);
  mul2(x[2], x[3], x[2], x[3], a, a);
}
// acc += k * x
__device__ __forceinline__ void chain4(float (&acc)[4], float k, const float (&x)[4]) {
  fma2(acc[0], acc[1], k, k, x[0], x[1], acc[0], acc[1]);
  fma2(acc[2], acc[3], k, k, x[2], x[3], acc[2], acc[3]);
}
// x += k * w
__device__ __forceinline__ void axpy4(float (&x)[4], float k, const float (&w)[4]) {
  fma2(x[0], x[1], k, k, w[0], w[1], x[0], x[1]);
  fma2(x[2], x[3], k, k, w[2], w[3], x[2], x[3]);
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

// Sylvester Hadamard of the head's 128-vector (4 values per lane),
// butterflies h = 1, 2, 4, ... then one scaling
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

template <bool HAD, int BLOCK, int MODE, int NST>
__global__ void __launch_bounds__(32 * kTmaWarps, 16) decode_tma_kernel(const DecodeArgs a) {
  constexpr int NB = kD / BLOCK;                   // blocks per row: 1 (whole row) or 4
  static_assert(NB == 1 || NB == 4, "blocks of 128 or 32 columns");
  __shared__ TmaSmem<NST> smem_all[kTmaWarps];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int head = blockIdx.x * kTmaWarps + warp;
  if (head >= a.B * a.H) return;                   // whole warp leaves together
  TmaSmem<NST>& sm = smem_all[warp];
  const int b = head / a.H, h = head - b * a.H;
  const int kh = h * a.Hk / a.H;
  const int nlo = kD - a.k_hi;                     // INT8 rows 0 .. nlo-1, FP16 rows after
  const int col0 = kC * lane;
  const int blk = (NB == 1) ? 0 : lane / 8;        // my block of the row
  const uint8_t* hin = (const uint8_t*)a.packed_in + (size_t)head * a.head_bytes;
  uint8_t* hout = (uint8_t*)a.packed_out + (size_t)head * a.head_bytes;
  const uint8_t* f16in = hin + (size_t)nlo * kD;
  uint16_t* f16out = (uint16_t*)(hout + (size_t)nlo * kD);
  const uint32_t* szin = (const uint32_t*)(f16in + (size_t)a.k_hi * kD * 2);
  uint32_t* szout = (uint32_t*)((uint8_t*)f16out + (size_t)a.k_hi * kD * 2);
  uint16_t* auxb = (MODE == BRS_ROUND_ERRFEEDBACK) ? (uint16_t*)a.aux + (size_t)head * nlo * kD : nullptr;

  // ---- slot plan: per pass n8 INT8 slots then nf FP16 slots; both passes
  // stream the same sequence.  Producer (lane 0 issues, every lane keeps
  // the counters): pj slots issued, pst next stage, ps next slot of a pass.
  const int n8 = (nlo + kRows8 - 1) / kRows8, nf = a.k_hi / kRows16;
  const int nslot = n8 + nf, total = 2 * nslot;
  const uint32_t bar0 = smem_u32(&sm.bar[0]), ring0 = smem_u32(&sm.ring[0][0]);
  int pj = 0, pst = 0, ps = 0;
  auto issue_next = [&]() {
    if (pj < total) {
      const uint8_t* src;
      uint32_t bytes;
      if (ps < n8) {
        src = hin + (size_t)ps * kSlot;
        bytes = (uint32_t)min(kSlot, (nlo - ps * kRows8) * kD);
      } else {
        src = f16in + (size_t)(ps - n8) * kSlot;
        bytes = (uint32_t)kSlot;
      }
      if (lane == 0) bulk_load(bar0 + 8u * pst, ring0 + (uint32_t)(pst * kSlot), src, bytes);
      ++pj;
      pst = (pst + 1 == NST) ? 0 : pst + 1;
      ps = (ps + 1 == nslot) ? 0 : ps + 1;
    }
  };
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < NST; ++st)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8u * st));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
#pragma unroll
  for (int st = 0; st < NST; ++st) issue_next();

  // ---- inputs (while the first slots are in flight): k, a, q through the
  // permutation and the grid of every INT8 row, as ready pairs; v, beta
  for (int i = lane; i < kD; i += 32) {
    const int p = a.perm ? a.perm[h * kD + i] : i;
    const size_t qk = ((size_t)b * a.Hk + kh) * kD;
    const float kv = bf16_to_f32(a.k[qk + p]);
    const float av = a.decay_per_key ? a.decay[(size_t)head * kD + p] : a.decay[head];
    const float qv = bf16_to_f32(a.q[qk + p]);
    float sv = 0.f, zv = 0.f;
    if (NB == 1 && i < nlo) {
      const uint32_t g = __ldg(szin + i);
      sv = f16_to_f32((uint16_t)(g & 0xffffu));
      zv = f16_to_f32((uint16_t)(g >> 16));
    }
    Scal r;
    r.ka = make_float4(kv, kv, av, av);
    r.sz = make_float4(sv, sv, zv, zv);
    sm.rs[i] = r;
    sm.qq[i] = make_float2(qv, qv);
  }
  float vv[kC];
  {
    const uint2 vw = __ldg((const uint2*)(a.v + (size_t)head * kD + col0));
    vv[0] = bf16_to_f32((uint16_t)(vw.x & 0xffffu)); vv[1] = bf16_to_f32((uint16_t)(vw.x >> 16));
    vv[2] = bf16_to_f32((uint16_t)(vw.y & 0xffffu)); vv[3] = bf16_to_f32((uint16_t)(vw.y >> 16));
  }
  const float beta = a.beta[head];
  __syncwarp();

  // grid of (row i, my block) for blocks narrower than the row
  auto grid_of = [&](int i, float& s, float& z) {
    const uint32_t g = __ldg(szin + i * NB + blk);
    s = f16_to_f32((uint16_t)(g & 0xffffu));
    z = f16_to_f32((uint16_t)(g >> 16));
  };

  // ---- consumer: cst the stage of the next slot, cph its phase parity,
  // cj slots consumed
  int cst = 0, cj = 0;
  uint32_t cph = 0;
  auto acquire = [&]() -> bool {
    return __all_sync(0xffffffffu, mbar_wait(bar0 + 8u * cst, cph));
  };
  auto release = [&]() {                           // every lane is done with the stage
    __syncwarp();
    ++cj;
    cst = (cst + 1 == NST) ? 0 : cst + 1;
    cph ^= (cst == 0) ? 1u : 0u;
    issue_next();
  };
  // after a timeout: the loads still in flight are waited for (bounded)
  // before the warp leaves, then the flag is raised
  auto abandon = [&]() {
    for (int jj = cj; jj < pj; ++jj) mbar_wait(bar0 + 8u * (jj % NST), (uint32_t)((jj / NST) & 1));
    raise_flag(a.flags, BRS_FLAG_TIMEOUT);
  };
  uint32_t err = 0;                                // flag bits, raised once at the end

  // ---- pass 1: u = U2 + T(U1) over the decayed rows
  float u1[kC] = {0.f, 0.f, 0.f, 0.f}, u2[kC] = {0.f, 0.f, 0.f, 0.f};
  auto p1_int8 = [&](const uint8_t* buf, int r0) {   // 8 INT8 rows from r0
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const uint32_t w = *(const uint32_t*)(buf + r * kD + col0);
      const Scal sc = sm.rs[r0 + r];
      float x[kC];
      if constexpr (NB == 1) {
        dequant4(x, w, sc.sz.x, sc.sz.z);
      } else {
        float gs, gz;
        grid_of(r0 + r, gs, gz);
        dequant4(x, w, gs, gz);
      }
      scale4(x, sc.ka.z);
      chain4(u1, sc.ka.x, x);
    }
  };
  for (int s = 0; s < nslot; ++s) {
    if (!acquire()) { abandon(); return; }
    const uint8_t* buf = sm.ring[cst];
    if (s < n8) {
      const int r0 = s * kRows8;
      p1_int8(buf, r0);
      if (r0 + 8 < nlo) p1_int8(buf + 8 * kD, r0 + 8);
    } else {
      const int r0 = nlo + (s - n8) * kRows16;
#pragma unroll
      for (int r = 0; r < kRows16; ++r) {
        const uint2 hv = *(const uint2*)(buf + r * 2 * kD + 2 * col0);
        const float4 ka = sm.rs[r0 + r].ka;
        float x[kC];
        f16x4_to_f32(x, hv);
        scale4(x, ka.z);
        chain4(u2, ka.x, x);
      }
    }
    release();
  }

  float w[kC], wt[kC];
  {
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
  }

  // ---- pass 2: write, o, requantize
  float o1[kC] = {0.f, 0.f, 0.f, 0.f}, o2[kC] = {0.f, 0.f, 0.f, 0.f};
  const int prow = lane & 7;                       // row of the batch whose grid this lane computes
  auto p2_int8 = [&](const uint8_t* buf, int i0) {   // a batch of 8 INT8 rows from i0
    float x[kNrb][kC];
#pragma unroll
    for (int r = 0; r < kNrb; ++r) {
      const uint32_t cw = *(const uint32_t*)(buf + r * kD + col0);
      const Scal sc = sm.rs[i0 + r];
      const float2 qv = sm.qq[i0 + r];
      if constexpr (NB == 1) {
        dequant4(x[r], cw, sc.sz.x, sc.sz.z);
      } else {
        float gs, gz;
        grid_of(i0 + r, gs, gz);
        dequant4(x[r], cw, gs, gz);
      }
      scale4(x[r], sc.ka.z);
      axpy4(x[r], sc.ka.x, wt);
      chain4(o1, qv.x, x[r]);
    }
    if constexpr (MODE == BRS_ROUND_ERRFEEDBACK) {
#pragma unroll
      for (int r = 0; r < kNrb; ++r) {
        const uint2 e = *(const uint2*)(auxb + (size_t)(i0 + r) * kD + col0);
        x[r][0] = __fadd_rn(x[r][0], f16_to_f32((uint16_t)(e.x & 0xffffu)));
        x[r][1] = __fadd_rn(x[r][1], f16_to_f32((uint16_t)(e.x >> 16)));
        x[r][2] = __fadd_rn(x[r][2], f16_to_f32((uint16_t)(e.y & 0xffffu)));
        x[r][3] = __fadd_rn(x[r][3], f16_to_f32((uint16_t)(e.y >> 16)));
      }
    }
    // ---- block extremes of the batch's rows, in every lane of the block
    float mn[kNrb], mx[kNrb];
#pragma unroll
    for (int r = 0; r < kNrb; ++r) {
      mn[r] = fminf(fminf(x[r][0], x[r][1]), fminf(x[r][2], x[r][3]));
      mx[r] = fmaxf(fmaxf(x[r][0], x[r][1]), fmaxf(x[r][2], x[r][3]));
    }
    if constexpr (NB == 1) {
#pragma unroll
      for (int r = 0; r < kNrb; ++r) {
        mn[r] = warp_min(mn[r]);
        mx[r] = warp_max(mx[r]);
      }
    } else {
#pragma unroll
      for (int m = 1; m < 8; m <<= 1)
#pragma unroll
        for (int r = 0; r < kNrb; ++r) {
          mn[r] = fminf(mn[r], __shfl_xor_sync(0xffffffffu, mn[r], m));
          mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], m));
        }
    }
    // lane l takes the grid of row (l & 7) of its block
    float mnv = pick8(mn, lane), mxv = pick8(mx, lane);
    // a zero extreme takes the sign rule (-0 below +0): rare, warp-wide
    if (__any_sync(0xffffffffu, (mnv == 0.0f) || (mxv == 0.0f))) {
      uint32_t nz = 0, pz = 0;
#pragma unroll
      for (int r = 0; r < kNrb; ++r)
#pragma unroll
        for (int c = 0; c < kC; ++c)
          if (x[r][c] == 0.0f) {
            if (signbit(x[r][c])) nz |= 1u << r; else pz |= 1u << r;
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
    // the grid: scale = fp16(fl((max - min) / 255)), zero = fp16(min);
    // ok = the block's extreme grid coordinates (the same monotone FP32
    // operations as its elements') round into [0, 255]
    bool ok;
    {
      const uint32_t g = f16x2_of(div255(__fsub_rn(mxv, mnv)), mnv);   // lo scale, hi zero
      const float sc = f16_to_f32((uint16_t)(g & 0xffffu)), z = f16_to_f32((uint16_t)(g >> 16));
      err |= (!isfinite(mnv) || !isfinite(mxv)) ? BRS_FLAG_NONFINITE : 0u;
      err |= f16x2_overflow(g) ? BRS_FLAG_OVERFLOW : 0u;
      const float rcp = (sc == 0.0f) ? 0.0f : rcp_of_f16(sc);
      float tlo, thi;
      sub2(tlo, thi, mnv, mxv, z, z);
      mul2(tlo, thi, tlo, thi, rcp, rcp);
      ok = (tlo >= -0.5f) && (thi < 255.5f);
      if (NB == 4 || lane < 8) {
        sm.prm[prow][blk] = make_float4(z, rcp, sc, 1.0f);
        szout[(i0 + prow) * NB + blk] = g;
      }
    }
    const bool fast = (MODE != BRS_ROUND_STOCHASTIC) && __all_sync(0xffffffffu, ok);
    __syncwarp();
    // ---- codes: clamp(round((y - zero) * (1/scale)), 0, 255); a zero
    // scale has 1/scale = 0, so every code of the block is 0
    auto quant = [&](auto clip_tag) {
      constexpr bool CLIP = decltype(clip_tag)::value;
#pragma unroll
      for (int r = 0; r < kNrb; ++r) {
        const int i = i0 + r;
        const float4 p = sm.prm[r][blk];           // (zero, 1/scale, scale, 1)
        float tq[kC];
        sub2(tq[0], tq[1], x[r][0], x[r][1], p.x, p.x);
        sub2(tq[2], tq[3], x[r][2], x[r][3], p.x, p.x);
        mul2(tq[0], tq[1], tq[0], tq[1], p.y, p.y);
        mul2(tq[2], tq[3], tq[2], tq[3], p.y, p.y);
        if constexpr (CLIP) {
          if constexpr (MODE == BRS_ROUND_STOCHASTIC) {
            const int e0 = i * kD + col0;
            const uint4 rnd = philox4x32_10(
                make_uint4((uint32_t)(e0 / 4), (uint32_t)a.step, (uint32_t)h, (uint32_t)b),
                make_uint2((uint32_t)a.seed, (uint32_t)(a.seed >> 32)));
            tq[0] = sr_round(tq[0], rnd.x >> 8);
            tq[1] = sr_round(tq[1], rnd.y >> 8);
            tq[2] = sr_round(tq[2], rnd.z >> 8);
            tq[3] = sr_round(tq[3], rnd.w >> 8);
          }
#pragma unroll
          for (int c = 0; c < kC; ++c) tq[c] = fminf(fmaxf(tq[c], 0.0f), 255.0f);
        }
        // nearest integer (ties to even): the low byte of t + 1.5*2^23,
        // the add written as t * 1 + magic with the 1 read from the grid
        // record, so that it stays a separately rounded operation after
        // the multiply (the sum is the same single rounding as an add)
        float mq[kC];
        fma2(mq[0], mq[1], tq[0], tq[1], p.w, p.w, kRoundMagic, kRoundMagic);
        fma2(mq[2], mq[3], tq[2], tq[3], p.w, p.w, kRoundMagic, kRoundMagic);
        *(uint32_t*)(hout + (size_t)i * kD + col0) =
            __byte_perm(__byte_perm(__float_as_uint(mq[0]), __float_as_uint(mq[1]), 0x0040u),
                        __byte_perm(__float_as_uint(mq[2]), __float_as_uint(mq[3]), 0x0040u), 0x5410u);
        if constexpr (MODE == BRS_ROUND_ERRFEEDBACK) {
          uint16_t ev[kC];
#pragma unroll
          for (int c = 0; c < kC; ++c) {
            const float code = __fsub_rn(mq[c], kRoundMagic);          // exact
            float e = __fsub_rn(x[r][c], __fmaf_rn(code, p.z, p.x));
            if (e > p.z) e = p.z;
            else if (e < -p.z) e = -p.z;
            ev[c] = f32_to_f16(e);
          }
          *(uint2*)(auxb + (size_t)i * kD + col0) =
              make_uint2((uint32_t)ev[0] | ((uint32_t)ev[1] << 16), (uint32_t)ev[2] | ((uint32_t)ev[3] << 16));
        }
      }
    };
    if (fast) quant(std::false_type{});
    else quant(std::true_type{});
    __syncwarp();                                  // prm reused by the next batch
  };
  for (int s = 0; s < nslot; ++s) {
    if (!acquire()) { abandon(); return; }
    const uint8_t* buf = sm.ring[cst];
    if (s < n8) {
      const int r0 = s * kRows8;
      p2_int8(buf, r0);
      if (r0 + 8 < nlo) p2_int8(buf + 8 * kD, r0 + 8);
    } else {
      // protected rows: FP16, nearest
      const int r0 = nlo + (s - n8) * kRows16;
      uint32_t ovf = 0;
#pragma unroll
      for (int r = 0; r < kRows16; ++r) {
        const int i = r0 + r;
        const uint2 hv = *(const uint2*)(buf + r * 2 * kD + 2 * col0);
        const float4 ka = sm.rs[i].ka;
        const float2 qv = sm.qq[i];
        float x[kC];
        f16x4_to_f32(x, hv);
        scale4(x, ka.z);
        axpy4(x, ka.x, w);
        chain4(o2, qv.x, x);
        const uint32_t lo = f16x2_of(x[0], x[1]), hi = f16x2_of(x[2], x[3]);
        ovf |= f16x2_overflow(lo) | f16x2_overflow(hi);
        *(uint2*)(f16out + (size_t)(i - nlo) * kD + col0) = make_uint2(lo, hi);
      }
      err |= ovf ? BRS_FLAG_OVERFLOW : 0u;
    }
    release();
  }

  // ---- o = O2 + T(O1)
  if constexpr (HAD) fwht128(o1, lane, a.hscale);
  float ov[kC];
  bool bad = false;
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    ov[c] = __fadd_rn(o2[c], o1[c]);
    bad |= !isfinite(ov[c]);
  }
  err |= bad ? BRS_FLAG_NONFINITE : 0u;
  *(float4*)(a.o + (size_t)head * kD + col0) = make_float4(ov[0], ov[1], ov[2], ov[3]);
  if (err) raise_flag(a.flags, err);
}

template <int BLOCK, int MODE>
cudaError_t launch_bm(const DecodeArgs& a, bool had, cudaStream_t st) {
  const int heads = a.B * a.H;
  const dim3 grid((heads + kTmaWarps - 1) / kTmaWarps), block(32 * kTmaWarps);
  // more heads than one wave of 16 per SM: two ring stages, whose smaller
  // shared-memory footprint lets more warps share an SM
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      sms = 148;
  }
  const bool many = heads > 16 * sms;
  if (had) {
    if (many) decode_tma_kernel<true, BLOCK, MODE, 2><<<grid, block, 0, st>>>(a);
    else decode_tma_kernel<true, BLOCK, MODE, kStages><<<grid, block, 0, st>>>(a);
  } else {
    if (many) decode_tma_kernel<false, BLOCK, MODE, 2><<<grid, block, 0, st>>>(a);
    else decode_tma_kernel<false, BLOCK, MODE, kStages><<<grid, block, 0, st>>>(a);
  }
  return cudaGetLastError();
}

template <int BLOCK>
cudaError_t launch_b(const DecodeArgs& a, bool had, cudaStream_t st) {
  switch (a.mode) {
    case BRS_ROUND_NEAREST: return launch_bm<BLOCK, BRS_ROUND_NEAREST>(a, had, st);
    case BRS_ROUND_STOCHASTIC: return launch_bm<BLOCK, BRS_ROUND_STOCHASTIC>(a, had, st);
    case BRS_ROUND_ERRFEEDBACK: return launch_bm<BLOCK, BRS_ROUND_ERRFEEDBACK>(a, had, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool decode_tma_supported(int d, int store, int block, int k_hi) {
  return d == kD && store == BRS_STORE_DAMP && (block == 128 || block == 32) && k_hi % kRows16 == 0;
}

cudaError_t launch_decode_tma(const DecodeArgs& a, bool had, cudaStream_t st) {
  if (a.block == 128) return launch_b<128>(a, had, st);
  if (a.block == 32) return launch_b<32>(a, had, st);
  return cudaErrorInvalidValue;
}

}  // namespace brs
