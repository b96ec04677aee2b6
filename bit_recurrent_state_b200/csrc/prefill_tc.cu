// Chunked prefill on the tcgen05 tensor cores (DAMP storage, d = 128,
// C = 64): the chunk's WY-form contractions run as TF32 UMMA with FP32
// accumulation in tensor memory, each product split 3 ways
// (hi*hi + hi*lo + lo*hi, hi = the operand truncated to TF32, lo = the
// remainder) so the contractions keep FP32-level accuracy; the forward
// substitution, the masks, the requantization and the write-back run on
// the CUDA cores.  The state is written back once per chunk ("Low-Bit
// Recurrent States in Hybrid Language Models", Accumulated readout error:
// write-back once per prefill chunk; Protocol: quantized and dequantized
// before reuse).  The chunk in WY form:
//   Gamma_t = prod_{r <= t} a_r, K~ = K * Gamma, K^ = K * (1 / Gamma), Q~ = Q * Gamma;
//   A = strictly-lower(diag(beta) K~ K^T);  (I + A) W = diag(beta)(V - K~ S_0);
//   O = Q~ S_0 + lower-incl(Q~ K^T) W;  S_C = diag(Gamma_63)(S_0 + K^T W).
//
// One CTA of 512 threads per (sequence, head) walks the chunks in order.
// A tcgen05.mma instruction takes about the same time for any N up to 256
// (and M = 64 or 128), so the products are packed into few wide
// instructions: operands that share A are stacked along N, and the hi and lo
// halves of a B operand sit next to each other so one instruction forms
// hi*hi and hi*lo.  Tensor-memory accumulators (lanes x columns, FP32):
//   phase 1, columns 0..191 (lanes t: K~ rows 0..63, Q~ rows 64..127):
//     [K~;Q~] . [S_0 | K^^T]  ->  K~ S_0, Q~ S_0 (cols 0..127), K~ K^^T, Q~ K^^T (128..191)
//   phase 2, columns 0..255 (lanes 64..127 = t):  P W, hi*hi + lo*hi (0..127), hi*lo (128..255)
//   phase 2, columns 256..511 (lanes i):          K^^T W, the same split
// All operands are K-major, no swizzle: 8-row x 16-byte core matrices,
// consecutive along K at 128 B, row groups of 8 at Kt/4 * 128 B.
// Products in tensor-memory orientation (A rows = lanes, B rows = columns):
//   phase 1:  A = X[t][i] ([K~;Q~]),  B = X[n][i] = [S_0^T (n = j) ; K^ (n = s)]    (K = i, 4 slices of 32)
//   phase 2:  A = X[t][s] (rows 64.. = P = lower-incl(Q~ K^^T); rows below unused),  B = X[j][s] = [W_hi ; W_lo]
//             A = X[i][s] (K^^T),                                                     B = [W_hi ; W_lo]
// The right side of the substitution, diag(beta)(V - K~ S_0), is read out by
// rows t and handed to the column threads j through shared memory.
// The FP32 state S_0 between chunks lives in a global scratch (dequantized
// stored state, stored row order, value basis).
#include <cuda_runtime.h>
#include <cstdint>

#include "brs_device.cuh"
#include "brs_internal.h"

namespace brs {
namespace {

constexpr int kD = 128, kC = 64, kThreads = 512;
constexpr int kParts = kThreads / 128;                   // warps per tensor-memory sub-partition
constexpr int kSl = 32;                                   // K slice of the i-contractions
constexpr unsigned long long kTcWaitNs = 200000000ull;    // bound on one MMA wait (200 ms)

// ---- shared-memory map (bytes from the 1 KB-aligned dynamic base)
// chunk inputs, FP32 rows of stride kRS floats (stored-row order columns):
//   Kt = K~ [64 t][128 i], Kh = K^, Qt = Q~
constexpr int kRS = 132;
constexpr int kRowB = kRS * 4;
// phase 1: one slice buffer: KQ hi, KQ lo [128][32], then the B operands
// [S0T [128 j][32] ; KH [64 s][32]] hi and lo (192 rows each)
constexpr int kKQ = 128 * kSl * 4, kKH = 64 * kSl * 4, kS0T = 128 * kSl * 4;
constexpr int kBN = kS0T + kKH;                           // one [S0T ; KH] operand
constexpr int kOffSlice = 0;
constexpr int kSliceB = 2 * (kKQ + kBN);                  // 80 KB
constexpr int kOffKt = kOffSlice + kSliceB, kOffKh = kOffKt + kC * kRowB, kOffQt = kOffKh + kC * kRowB;
// phase 2: KT hi/lo [128 i][64 s] over the slice buffer, P hi/lo [64 t][64 s] and A fp32 [64][68]
// over Kt, W hi/lo [128 j][64 s] over Qt (W hi first holds the substitution's right side,
// [64 t][128 j] FP32 with 16-byte groups swizzled by t); Kh stays readable while KT is built
constexpr int kWt = 128 * 64 * 4, kKT = 128 * 64 * 4, kPt = 64 * 64 * 4;
constexpr int kAStride = 68;
constexpr int kOffKT = 0, kOffP = kOffKT + 2 * kKT, kOffA = kOffP + 2 * kPt, kOffW = kOffQt;
constexpr int kRegion = kOffW + 2 * kWt;                   // 210 KB
// requantization: S [128][132] fp32 at the start of the region
constexpr int kSStride = 132;
constexpr int kOffG63 = kRegion;                           // Gamma_63 [128]
constexpr int kOffBeta = kOffG63 + kD * 4;                 // beta [64]
constexpr int kOffMisc = kOffBeta + kC * 4;                // mbarriers, tensor-memory base
constexpr int kOffPerm = kOffMisc + 64;                    // stored row -> key channel [128] int16
constexpr int kSmem = kOffPerm + kD * 2;
static_assert(kOffA + 64 * kAStride * 4 <= kOffKh, "P and A leave Kh intact");
static_assert(kOffKT + 2 * kKT <= kOffKt, "KT over the slice buffer only");
static_assert(kOffQt + kC * kRowB <= kRegion, "Qt inside the region");
static_assert(kD * kSStride * 4 <= kOffW, "requantization rows fit below W");
static_assert(kSmem <= 227 * 1024, "shared memory of one CTA");
static_assert(kOffP >= 8 * 2048 && kOffP + kPt >= 8 * 2048, "the unused rows of the P operand stay in shared memory");
static_assert(kC * kD * 4 <= kWt, "the right side fits the W hi tile");

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// ---- K-major no-swizzle operand tile X[R][Kt]: byte offset of (r, k)
__device__ __forceinline__ uint32_t kmaj(int r, int k, int Kt) {
  return (uint32_t)(((r >> 3) * (Kt >> 2) + (k >> 2)) * 128 + (r & 7) * 16 + (k & 3) * 4);
}
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t sbo) {
  // start >> 4, leading offset 128 B (next 4 elements along K), stride offset
  // sbo (next 8 rows), descriptor version 1, no swizzle
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) | ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) |
         (1ull << 46);
}
// kind::tf32 instruction descriptor: D f32, A/B tf32, both K-major
constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma_tf32(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
// 3-way split product D (+)= Ah Bh + Ah Bl + Al Bh from prebuilt hi/lo operand
// descriptors; off16 = byte offset / 16 added to the start-address field (no
// carry: shared addresses are below 256 KB)
__device__ __forceinline__ void umma3d(uint32_t d, uint64_t ah, uint64_t al, uint64_t bh, uint64_t bl, uint32_t off16,
                                       uint32_t idesc, uint32_t acc) {
  umma_tf32(d, ah + off16, bh + off16, idesc, acc);
  umma_tf32(d, ah + off16, bl + off16, idesc, 1u);
  umma_tf32(d, al + off16, bh + off16, idesc, 1u);
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// one phase of an mbarrier; a thread parked in try_wait is suspended for at
// most ~128 ns per attempt (parked without a bound it can stay suspended for
// microseconds after the phase completes)
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 128; selp.u32 %0, 1, 0, p; }"
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
// hand-over of a head between CTAs: the chunk count a CTA has finished,
// published with release semantics and read with acquire semantics (GPU scope)
__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// bounded wait for one phase of an MMA-completion barrier
__device__ __forceinline__ bool mbar_wait_tc(uint32_t bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_try(bar, parity))
    if (global_ns() - t0 > kTcWaitNs) return false;
  return true;
}

// 16 consecutive FP32 columns of this thread's tensor-memory lane
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int c = 0; c < 16; ++c) v[c] = __uint_as_float(r[c]);
}

// fl(x / 255) for any float x, as fl32(fl64(x * fl64(1/255))): the quotient
// of a float by 255 stays at least 2^-33 (relative) from every float
// rounding midpoint while the double product is within 2^-52 of it
__device__ __forceinline__ float div255(float x) { return (float)((double)x * (1.0 / 255.0)); }
// fl(1 / s) for s a positive binary16 value: one Newton-Raphson correction
// of the hardware approximation (exact residual; 1/s for an 11-bit s stays
// at least 2^-36 from every midpoint, the corrected value within 2^-40)
__device__ __forceinline__ float rcp_of_f16(float s) {
  float r0;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(s));
  const float e = __fmaf_rn(-s, r0, 1.0f);
  return __fmaf_rn(r0, e, r0);
}

// the operand split: hi = x truncated to TF32, lo = x - hi (exact)
__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }
// store 4 consecutive-K values of row r at (hi tile, lo tile)
__device__ __forceinline__ void st_split4(uint8_t* hi, uint8_t* lo, uint32_t off, float x0, float x1, float x2,
                                          float x3) {
  const float h0 = tf32_hi(x0), h1 = tf32_hi(x1), h2 = tf32_hi(x2), h3 = tf32_hi(x3);
  *(float4*)(hi + off) = make_float4(h0, h1, h2, h3);
  *(float4*)(lo + off) = make_float4(__fsub_rn(x0, h0), __fsub_rn(x1, h1), __fsub_rn(x2, h2), __fsub_rn(x3, h3));
}

// stored head -> FP32 rows (stored order, value basis) in the global scratch
// the 4-bit low tier: a lane's four codes (16 bits, element e in bits 4e)
// spread to one byte each, and four codes held one per byte gathered back
__device__ __forceinline__ uint32_t pf_nib_spread(uint32_t w) {
  w = (w | (w << 8)) & 0x00FF00FFu;
  return (w | (w << 4)) & 0x0F0F0F0Fu;
}
__device__ __forceinline__ uint32_t pf_nib_gather(uint32_t w) {
  w = (w | (w >> 4)) & 0x00FF00FFu;
  return (w | (w >> 8)) & 0xFFFFu;
}

// LB: the low tier's width, 8 (INT8) or 4 (two codes per byte)
template <bool HAD, int BLOCK, int LB>
__device__ void tc_load_state(const uint8_t* head, float* S, int nlo, int k_hi, float hscale) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, col0 = 4 * lane;
  constexpr int NB = kD / BLOCK, CR = kD * LB / 8;
  const uint8_t* f16in = head + (size_t)nlo * CR;
  const uint32_t* szin = (const uint32_t*)(head + (size_t)nlo * CR + (size_t)k_hi * kD * 2);
  for (int r = warp; r < kD; r += kThreads / 32) {
    float x[4];
    if (r < nlo) {
      const uint32_t c4 = (LB == 8) ? *(const uint32_t*)(head + (size_t)r * CR + col0)
                                    : pf_nib_spread(*(const uint16_t*)(head + (size_t)r * CR + col0 / 2));
      const uint32_t sz = szin[r * NB + col0 / BLOCK];
      const float s = f16_to_f32((uint16_t)(sz & 0xffffu)), z = f16_to_f32((uint16_t)(sz >> 16));
#pragma unroll
      for (int c = 0; c < 4; ++c) x[c] = __fmaf_rn(__fsub_rn(byte_magic(c4, c), kTwo23), s, z);
      if (HAD) row_fwht4<kD>(x, lane, hscale);
    } else {
      const uint2 hv = *(const uint2*)(f16in + ((size_t)(r - nlo) * kD + col0) * 2);
      x[0] = f16_to_f32((uint16_t)(hv.x & 0xffffu)); x[1] = f16_to_f32((uint16_t)(hv.x >> 16));
      x[2] = f16_to_f32((uint16_t)(hv.y & 0xffffu)); x[3] = f16_to_f32((uint16_t)(hv.y >> 16));
    }
    *(float4*)&S[(size_t)r * kD + col0] = make_float4(x[0], x[1], x[2], x[3]);
  }
}

// Write-back of the chunk, a warp per stored row (rows warp, warp + 16, ...),
// lane l owning columns 4l .. 4l+3: S_C = Gamma_63 (S_0 + K^^T W) from the
// product rows Ds (shared, stride kSStride) and S_0 (the global scratch,
// whole rows per load), then the stored row; the dequantized row (the state
// the next chunk starts from) replaces S_0 in the scratch.
template <bool HAD, int BLOCK, int MODE, int LB>
__device__ void tc_store_state(const float* Ds, const float* g63, float* S, uint8_t* head, uint16_t* aux, int nlo,
                               int k_hi, float hscale, const PrefillArgs& a, int64_t step, int h, int b, float* sdump,
                               uint32_t& err) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, col0 = 4 * lane;
  constexpr int NB = kD / BLOCK, GL = BLOCK / 4, kRowsW = kD / (kThreads / 32), CR = kD * LB / 8;
  constexpr float LV = (float)((1 << LB) - 1);    // top code: 255 or 15
  uint16_t* f16out = (uint16_t*)(head + (size_t)nlo * CR);
  uint32_t* szout = (uint32_t*)(head + (size_t)nlo * CR + (size_t)k_hi * kD * 2);
  float4 s0r[kRowsW];                              // this warp's S_0 rows, all loads in flight at once
#pragma unroll
  for (int k = 0; k < kRowsW; ++k) s0r[k] = *(const float4*)&S[(size_t)(warp + 16 * k) * kD + col0];
#pragma unroll
  for (int k = 0; k < kRowsW; ++k) {
    const int r = warp + 16 * k;
    const float4 d4 = *(const float4*)&Ds[r * kSStride + col0];
    const float gi = g63[r];
    // Gamma_63 * (S_0 + K^^T W); the product as an fma with -0 (the same
    // rounded product) so that it is never merged with the transform's adds
    float x[4] = {__fmaf_rn(gi, __fadd_rn(s0r[k].x, d4.x), -0.0f), __fmaf_rn(gi, __fadd_rn(s0r[k].y, d4.y), -0.0f),
                  __fmaf_rn(gi, __fadd_rn(s0r[k].z, d4.z), -0.0f), __fmaf_rn(gi, __fadd_rn(s0r[k].w, d4.w), -0.0f)};
    if (sdump) *(float4*)&sdump[(size_t)r * kD + col0] = make_float4(x[0], x[1], x[2], x[3]);
    if (r >= nlo) {
      const uint32_t lo = f16x2_of(x[0], x[1]), hi = f16x2_of(x[2], x[3]);
      if ((((lo >> 10) & 31u) == 31u) || (((lo >> 26) & 31u) == 31u) || (((hi >> 10) & 31u) == 31u) ||
          (((hi >> 26) & 31u) == 31u))
        err |= BRS_FLAG_OVERFLOW;
      *(uint2*)&f16out[(size_t)(r - nlo) * kD + col0] = make_uint2(lo, hi);
      *(float4*)&S[(size_t)r * kD + col0] =
          make_float4(f16_to_f32((uint16_t)(lo & 0xffffu)), f16_to_f32((uint16_t)(lo >> 16)),
                      f16_to_f32((uint16_t)(hi & 0xffffu)), f16_to_f32((uint16_t)(hi >> 16)));
      continue;
    }
    if (HAD) row_fwht4<kD>(x, lane, hscale);
    if (MODE == BRS_ROUND_ERRFEEDBACK) {
      const uint2 ev = *(const uint2*)&aux[(size_t)r * kD + col0];
      x[0] = __fadd_rn(x[0], f16_to_f32((uint16_t)(ev.x & 0xffffu)));
      x[1] = __fadd_rn(x[1], f16_to_f32((uint16_t)(ev.x >> 16)));
      x[2] = __fadd_rn(x[2], f16_to_f32((uint16_t)(ev.y & 0xffffu)));
      x[3] = __fadd_rn(x[3], f16_to_f32((uint16_t)(ev.y >> 16)));
    }
    float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
    float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    if constexpr (GL == 32) {
      asm volatile("redux.sync.min.f32 %0, %0, 0xffffffff;" : "+f"(mn));
      asm volatile("redux.sync.max.f32 %0, %0, 0xffffffff;" : "+f"(mx));
    } else {
#pragma unroll
      for (int m = 1; m < GL; m <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, m));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
      }
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
    if (!isfinite(mn) || !isfinite(mx)) err |= BRS_FLAG_NONFINITE;
    const float rng = __fsub_rn(mx, mn);
    const uint32_t gz = f16x2_of(LB == 8 ? div255(rng) : __fdiv_rn(rng, LV), mn);    // lo scale, hi zero
    const uint16_t sh = (uint16_t)(gz & 0xffffu), zh = (uint16_t)(gz >> 16);
    if (f16_inf_or_nan(sh) || f16_inf_or_nan(zh)) err |= BRS_FLAG_OVERFLOW;
    const float s = f16_to_f32(sh), z = f16_to_f32(zh);
    const float rcp = (s == 0.0f) ? 0.0f : rcp_of_f16(s);
    uint4 rnd = make_uint4(0, 0, 0, 0);
    if (MODE == BRS_ROUND_STOCHASTIC)
      rnd = philox4x32_10(make_uint4((uint32_t)(r * (kD / 4) + lane), (uint32_t)step, (uint32_t)h, (uint32_t)b),
                          make_uint2((uint32_t)a.seed, (uint32_t)(a.seed >> 32)));
    const uint32_t rw[4] = {rnd.x >> 8, rnd.y >> 8, rnd.z >> 8, rnd.w >> 8};
    uint32_t packed4 = 0;
    float xh[4];
    uint16_t e16[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      // a zero scale has 1/scale = 0: every code is 0
      float tt = __fmul_rn(__fsub_rn(x[c], z), rcp);
      if (MODE == BRS_ROUND_STOCHASTIC) tt = sr_round(tt, rw[c]);
      // clip, then the nearest integer (ties to even) as the low byte of
      // t + 1.5*2^23 (exact for the integers SR produces)
      const float m = __fadd_rn(fminf(fmaxf(tt, 0.0f), LV), kRoundMagic);
      const float code = __fsub_rn(m, kRoundMagic);
      packed4 |= (__float_as_uint(m) & 0xffu) << (8 * c);
      xh[c] = __fmaf_rn(code, s, z);
      if (MODE == BRS_ROUND_ERRFEEDBACK) {
        float e = __fsub_rn(x[c], xh[c]);
        if (e > s) e = s;
        else if (e < -s) e = -s;
        e16[c] = f32_to_f16(e);
      }
    }
    if (LB == 8) *(uint32_t*)(head + (size_t)r * CR + col0) = packed4;
    else *(uint16_t*)(head + (size_t)r * CR + col0 / 2) = (uint16_t)pf_nib_gather(packed4);
    if ((col0 % BLOCK) == 0) szout[r * NB + col0 / BLOCK] = (uint32_t)sh | ((uint32_t)zh << 16);
    if (MODE == BRS_ROUND_ERRFEEDBACK)
      *(uint2*)&aux[(size_t)r * kD + col0] =
          make_uint2((uint32_t)e16[0] | ((uint32_t)e16[1] << 16), (uint32_t)e16[2] | ((uint32_t)e16[3] << 16));
    if (HAD) row_fwht4<kD>(xh, lane, hscale);          // continue from the stored values
    *(float4*)&S[(size_t)r * kD + col0] = make_float4(xh[0], xh[1], xh[2], xh[3]);
  }
}

template <bool HAD, int BLOCK, int MODE, int LB>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const PrefillArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int sub = warp & 3;                        // tensor-memory lanes 32 sub .. 32 sub + 31
  const int part = warp >> 2;                      // which part of a readout's columns
  const int nlo = kD - a.k_hi;
  float* Kt = (float*)(smem + kOffKt);
  float* Kh = (float*)(smem + kOffKh);
  float* Qt = (float*)(smem + kOffQt);
  float* g63 = (float*)(smem + kOffG63);
  float* betas = (float*)(smem + kOffBeta);
  unsigned long long* bars = (unsigned long long*)(smem + kOffMisc);   // phase 1, phase 2
  uint32_t* tslot = (uint32_t*)(smem + kOffMisc + 32);
  int16_t* permS = (int16_t*)(smem + kOffPerm);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = smem_u32(&bars[0]);
  uint32_t err = 0;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8u));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tslot;
  const uint32_t tO = tm, tD4 = tm + 256;         // phase 1 uses columns 0..191, phase 2 all 512
  const uint32_t lrow = (uint32_t)(32 * sub) << 16;          // this warp's lane base in tensor memory
  const int myrow = 32 * sub + lane;                          // the tensor-memory lane this thread reads
  uint32_t ph0 = 0, ph1 = 0;
  bool alive = true;
  // thread 0 waits on the mbarrier, the others at the CTA barrier; the CTA
  // agrees on the outcome
  auto wait_all = [&](int which, uint32_t& ph) -> bool {
    const bool ok = (tid == 0) ? mbar_wait_tc(bar0 + 8u * which, ph) : true;
    ph ^= 1u;
    return !__syncthreads_or(ok ? 0 : 1);
  };

  // This CTA's share of the (head, chunk) units, in head-major order: units
  // [u0, u1) with equal shares per CTA (one CTA per SM, all resident).  The
  // share is cut at head boundaries into segments, taken in this order: the
  // leading chunks of the last head when it is cut (another CTA continues
  // it, so they come first), whole heads, and last the continuation of the
  // first head when it is cut (its leading chunks are the previous CTA's
  // first segment; a bounded wait on that head's hand-over counter).
  const int nchunks = a.T / kC, heads = a.B * a.H;
  const long long U = (long long)heads * nchunks;
  const long long u0 = U * blockIdx.x / gridDim.x, u1 = U * (blockIdx.x + 1) / gridDim.x;
  const int hf = (int)(u0 / nchunks), kf = (int)(u0 % nchunks);
  const int hl = (int)((u1 - 1) / nchunks), ke = (int)((u1 - 1) % nchunks) + 1;
  const int nmid = hl > hf ? hl - hf - 1 : 0;
  const bool lead = hl > hf && ke < nchunks;       // the last head's leading chunks
  const bool cont = kf > 0;                        // the first head's continuation
  const int nseg = (u1 <= u0) ? 0
                   : (hl == hf) ? 1
                                : (lead ? 1 : 0) + (kf == 0 ? 1 : 0) + nmid + (ke == nchunks ? 1 : 0) + (cont ? 1 : 0);
  for (int sg = 0; sg < nseg && alive; ++sg) {
    int head, c0, c1;
    {
      int idx = sg;
      if (hl == hf) {
        head = hf; c0 = kf; c1 = ke;
      } else if (lead && idx == 0) {
        head = hl; c0 = 0; c1 = ke;
      } else {
        idx -= lead ? 1 : 0;
        if (kf == 0 && idx == 0) {
          head = hf; c0 = 0; c1 = nchunks;
        } else {
          idx -= (kf == 0) ? 1 : 0;
          if (idx < nmid) {
            head = hf + 1 + idx; c0 = 0; c1 = nchunks;
          } else if (ke == nchunks && idx == nmid) {
            head = hl; c0 = 0; c1 = nchunks;
          } else {
            head = hf; c0 = kf; c1 = nchunks;      // the continuation
          }
        }
      }
    }
    const int b = head / a.H, h = head - b * a.H, kh = h * a.Hk / a.H;
    uint8_t* hst = (uint8_t*)a.packed + (size_t)head * a.head_bytes;
    uint16_t* aux = (MODE == BRS_ROUND_ERRFEEDBACK) ? (uint16_t*)a.aux + (size_t)head * nlo * kD : nullptr;
    float* S0g = a.s0 + (size_t)head * kD * kD;    // FP32 state between chunks
    if (tid < kD) permS[tid] = a.perm ? a.perm[h * kD + tid] : (int16_t)tid;
    if (c0 == 0) {
      tc_load_state<HAD, BLOCK, LB>(hst, S0g, nlo, a.k_hi, a.hscale);
    } else {
      // the head's state after chunk c0 - 1 is in the scratch, the stored
      // state and the residuals once the hand-over counter reaches c0
      bool ok = true;
      if (tid == 0) {
        const unsigned long long tw = global_ns();
        while (ld_acquire_u32(a.handover + head) < (uint32_t)c0)
          if (global_ns() - tw > kTcWaitNs) {
            ok = false;
            break;
          }
      }
      if (!__syncthreads_and(ok)) {
        alive = false;
        break;
      }
      __threadfence();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  for (int ch = c0; ch < c1 && alive; ++ch) {
    const int t0 = ch * kC;
    const size_t tokb = (size_t)b * a.T + t0;                 // first token of the chunk
    // ---- chunk inputs: thread (row i, quarter qq) takes tokens 16 qq .. 16 qq + 15
    // of stored row i: cumulative decay (local products, then the earlier
    // quarters' totals), K~ = K Gamma, K^ = K (1 / Gamma), Q~ = Q Gamma
    {
      const int i = tid & 127, qq = tid >> 7, p = permS[i];
      float av[16], kv[16], qv[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {                 // all loads in flight at once
        const size_t tok = tokb + 16 * qq + r;
        av[r] = a.decay_per_key ? a.decay[(tok * a.H + h) * kD + p] : a.decay[tok * a.H + h];
        kv[r] = bf16_to_f32(a.k[(tok * a.Hk + kh) * kD + p]);
        qv[r] = bf16_to_f32(a.q[(tok * a.Hk + kh) * kD + p]);
      }
      if (tid < kC) betas[tid] = a.beta[(tokb + tid) * a.H + h];
#pragma unroll
      for (int r = 1; r < 16; ++r) av[r] = __fmul_rn(av[r - 1], av[r]);
      float* tot = (float*)(smem + kOffSlice);       // [4][128] quarter totals
      tot[qq * kD + i] = av[15];
      __syncthreads();
      float carry = 1.0f;
      for (int u = 0; u < qq; ++u) carry = __fmul_rn(carry, tot[u * kD + i]);
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const float g = qq ? __fmul_rn(carry, av[r]) : av[r];
        const int t = 16 * qq + r;
        Kt[t * kRS + i] = __fmul_rn(kv[r], g);
        Kh[t * kRS + i] = __fmul_rn(kv[r], __frcp_rn(g));
        Qt[t * kRS + i] = __fmul_rn(qv[r], g);
        if (t == kC - 1) g63[i] = g;
      }
      __syncthreads();
    }

    // ---- phase 1: D1 = [K~;Q~] K^^T, D2 = S_0^T [K~;Q~]^T over 4 slices of
    // 32 stored rows i (one slice buffer)
    for (int sl = 0; sl < kD / kSl; ++sl) {
      const int i0 = sl * kSl;
      // this thread's two S_0^T tasks (rows j, 4 stored rows i each), loaded
      // from the global scratch while the previous slice's MMAs run
      float pre[2][4];
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        const int u = tid + q2 * kThreads, j = u & 127, i = i0 + 4 * (u >> 7);
#pragma unroll
        for (int c = 0; c < 4; ++c) pre[q2][c] = S0g[(size_t)(i + c) * kD + j];
      }
      if (sl > 0) {
        alive = wait_all(0, ph0);                    // the previous slice's MMAs read the buffer
        if (!alive) break;
      }
      uint8_t* B0 = smem + kOffSlice;
      uint8_t *KQh = B0, *KQl = B0 + kKQ, *STh = B0 + 2 * kKQ, *KHh = STh + kS0T, *STl = STh + kBN, *KHl = STl + kS0T;
#pragma unroll
      for (int q = 0; q < 2560 / kThreads; ++q) {
        const int task = tid + q * kThreads;
        if (q < 1024 / kThreads) {                   // [K~;Q~] rows t, columns 4g .. 4g+3 of the slice
          const int t = task & 127, g = task >> 7;
          const float4 x = *(const float4*)((t < 64) ? &Kt[t * kRS + i0 + 4 * g] : &Qt[(t - 64) * kRS + i0 + 4 * g]);
          st_split4(KQh, KQl, kmaj(t, 4 * g, kSl), x.x, x.y, x.z, x.w);
        } else if (q < 1536 / kThreads) {            // K^ rows s
          const int u = task - 1024, s = u & 63, g = u >> 6;
          const float4 x = *(const float4*)&Kh[s * kRS + i0 + 4 * g];
          st_split4(KHh, KHl, kmaj(s, 4 * g, kSl), x.x, x.y, x.z, x.w);
        } else {                                     // S_0^T rows j
          const int u = task - 1536, j = u & 127, g = u >> 7;
          const int q2 = (q * kThreads - 1536) / kThreads;
          st_split4(STh, STl, kmaj(j, 4 * g, kSl), pre[q2][0], pre[q2][1], pre[q2][2], pre[q2][3]);
        }
      }
      proxy_fence();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        const uint32_t base = sbase + kOffSlice;
        constexpr uint32_t sbo = (kSl / 4) * 128;
        // [K~;Q~] . [S_0^T ; K^]: N = 192, three instructions per k-step
        const uint64_t dKQh = sdesc(base, sbo), dKQl = sdesc(base + kKQ, sbo);
        const uint64_t dBh = sdesc(base + 2 * kKQ, sbo), dBl = sdesc(base + 2 * kKQ + kBN, sbo);
#pragma unroll
        for (int k = 0; k < kSl / 8; ++k) {
          const uint32_t o16 = 16u * k, acc = (sl > 0 || k > 0) ? 1u : 0u;
          umma3d(tO, dKQh, dKQl, dBh, dBl, o16, idesc_tf32(128, 3 * kC), acc);
        }
        umma_commit(bar0);
      }
    }
    if (!alive) break;
    if (sub < 2) {                                   // this thread's part of a V row into L1 while the MMAs run
      const uint16_t* vrow = a.v + ((tokb + myrow) * a.H + h) * kD + 32 * part;
      asm volatile("prefetch.global.L1 [%0];" ::"l"(vrow));
    }
    alive = wait_all(0, ph0);
    if (!alive) break;
    tc_fence_after();

    // ---- phase-1 readout, every warp: tensor-memory lanes t of its
    // sub-partition, value columns 32 part .. 32 part + 31, key columns
    // 16 part .. 16 part + 15 (Q~ S_0 stays in tensor memory for O)
    float* Am = (float*)(smem + kOffA);
    float* Rs = (float*)(smem + kOffW);              // right side [64 t][128 j], 16-byte groups ^ (t & 7)
    {
      float v[16];
      const int c0 = 16 * part;
      if (sub < 2) {
        // right side diag(beta)(V - K~ S_0), by rows
        const int t = myrow;
        const float bt = betas[t];
        const uint4* vp = (const uint4*)(a.v + ((tokb + t) * a.H + h) * kD + 32 * part);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          tmem_ld16(tO + lrow + 32 * part + 16 * q, v);
          const uint4 r0 = vp[2 * q], r1 = vp[2 * q + 1];
          const uint32_t vw[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
          float x[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float vv = bf16_to_f32((uint16_t)((c & 1) ? (vw[c >> 1] >> 16) : (vw[c >> 1] & 0xffffu)));
            x[c] = __fmul_rn(bt, __fsub_rn(vv, v[c]));
          }
#pragma unroll
          for (int c = 0; c < 16; c += 4) {
            const int g = (32 * part + 16 * q + c) >> 2;
            *(float4*)&Rs[t * kD + ((g ^ (t & 7)) << 2)] = make_float4(x[c], x[c + 1], x[c + 2], x[c + 3]);
          }
        }
        // A = strictly-lower(diag(beta) K~ K^T), FP32
        tmem_ld16(tO + lrow + kD + c0, v);
#pragma unroll
        for (int c = 0; c < 16; c += 4)
          *(float4*)&Am[t * kAStride + c0 + c] =
              make_float4((c0 + c + 0 < t) ? __fmul_rn(bt, v[c + 0]) : 0.0f, (c0 + c + 1 < t) ? __fmul_rn(bt, v[c + 1]) : 0.0f,
                          (c0 + c + 2 < t) ? __fmul_rn(bt, v[c + 2]) : 0.0f, (c0 + c + 3 < t) ? __fmul_rn(bt, v[c + 3]) : 0.0f);
      } else {
        // P = lower-incl(Q~ K^T) as the split operand X[t][s]
        const int t = myrow - 64;
        tmem_ld16(tO + lrow + kD + c0, v);
#pragma unroll
        for (int c = 0; c < 16; c += 4)
          st_split4(smem + kOffP, smem + kOffP + kPt, kmaj(t, c0 + c, 64), (c0 + c + 0 <= t) ? v[c + 0] : 0.0f,
                    (c0 + c + 1 <= t) ? v[c + 1] : 0.0f, (c0 + c + 2 <= t) ? v[c + 2] : 0.0f,
                    (c0 + c + 3 <= t) ? v[c + 3] : 0.0f);
      }
    }
    tc_fence_before();
    __syncthreads();                                 // right side, A and P complete; key columns read

    const bool solver = (sub < 2) && (part < 2);     // warps 0, 1, 4, 5: one value column each
    if (solver) {
      // ---- W by forward substitution, one value column j per thread:
      // (I + A) W = diag(beta)(V - K~ S_0)
      const int j = 32 * (2 * part + sub) + lane;
      float w[kC];
#pragma unroll
      for (int t = 0; t < kC; ++t) w[t] = Rs[t * kD + ((((j >> 2) ^ (t & 7))) << 2) + (j & 3)];
      asm volatile("bar.sync 1, 128;" ::: "memory");   // every column read before W replaces the right side
      // blocks of 16 rows: the terms from earlier blocks are 16 independent
      // sums, then the block's own triangle is solved row by row
#pragma unroll
      for (int B = 0; B < kC / 16; ++B) {
        float acc[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) acc[r] = 0.0f;
#pragma unroll
        for (int s = 0; s < 16 * B; s += 4)
#pragma unroll
          for (int r = 0; r < 16; ++r) {
            const float4 a4 = *(const float4*)&Am[(16 * B + r) * kAStride + s];
            acc[r] = __fmaf_rn(a4.x, w[s], acc[r]);
            acc[r] = __fmaf_rn(a4.y, w[s + 1], acc[r]);
            acc[r] = __fmaf_rn(a4.z, w[s + 2], acc[r]);
            acc[r] = __fmaf_rn(a4.w, w[s + 3], acc[r]);
          }
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const int t = 16 * B + r;
          float x = acc[r];
#pragma unroll
          for (int s = 16 * B; s < t; ++s) x = __fmaf_rn(Am[t * kAStride + s], w[s], x);
          w[t] = __fsub_rn(w[t], x);
        }
      }
#pragma unroll
      for (int s = 0; s < kC; s += 4)
        st_split4(smem + kOffW, smem + kOffW + kWt, kmaj(j, s, 64), w[s], w[s + 1], w[s + 2], w[s + 3]);
    } else {
      if (sub >= 2) {
        // zero the hi*lo columns of O (lanes 64..127, columns 128..255): phase 2
        // accumulates onto Q~ S_0 in columns 0..127 and onto zero here
        uint32_t zr = 0;
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
            "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(tO + lrow + kD + 32 * part), "r"(zr)
            : "memory");
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      }
      // ---- K^ transposed: X[i][s] = K^[s][i], by the other 12 warps
      const int wr = (warp < 8) ? 2 * (warp >> 2) + (warp & 3) - 2 : warp - 4;
      for (int task = 32 * wr + lane; task < kD * (kC / 4); task += kThreads - 128) {
        const int i = task & 127, sg = task >> 7;
        st_split4(smem + kOffKT, smem + kOffKT + kKT, kmaj(i, 4 * sg, 64), Kh[(4 * sg) * kRS + i],
                  Kh[(4 * sg + 1) * kRS + i], Kh[(4 * sg + 2) * kRS + i], Kh[(4 * sg + 3) * kRS + i]);
      }
    }
    proxy_fence();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      // ---- phase 2: B = [W_hi ; W_lo] (N = 256) gives hi*hi and hi*lo in one
      // instruction, B = W_hi adds lo*hi to the first half.
      //   O: A = X[t'][s] whose rows 64..127 are P (rows 0..63: the 16 KB
      //      below P, unused lanes), accumulated onto Q~ S_0;
      //   K^^T W: A = X[i][s], fresh.
      tc_fence_after();
      constexpr uint32_t sbo = (64 / 4) * 128;
      const uint32_t aKTh = sbase + kOffKT, aKTl = aKTh + kKT;
      const uint32_t aPh = sbase + kOffP - 8 * sbo, aPl = sbase + kOffP + kPt - 8 * sbo;
      const uint64_t dW = sdesc(sbase + kOffW, sbo), dKTh = sdesc(aKTh, sbo), dKTl = sdesc(aKTl, sbo),
                     dPh = sdesc(aPh, sbo), dPl = sdesc(aPl, sbo);
#pragma unroll
      for (int k = 0; k < kC / 8; ++k) {
        const uint32_t o16 = 16u * k;
        umma_tf32(tO, dPh + o16, dW + o16, idesc_tf32(128, 2 * kD), 1u);
        umma_tf32(tO, dPl + o16, dW + o16, idesc_tf32(128, kD), 1u);
        umma_tf32(tD4, dKTh + o16, dW + o16, idesc_tf32(128, 2 * kD), k > 0 ? 1u : 0u);
        umma_tf32(tD4, dKTl + o16, dW + o16, idesc_tf32(128, kD), 1u);
      }
      umma_commit(bar0 + 8u);
    }
    constexpr int kCols = kD / kParts;               // this thread's columns of a product row
    alive = wait_all(1, ph1);
    if (!alive) break;
    tc_fence_after();

    // ---- O = (Q~ S_0 + P W) rows to global (lanes 64..127); K^^T W rows to
    // shared memory for the write-back
    {
      float v[16], u[16];
      if (sub >= 2) {
        const int t = myrow - 64;
        float* orow = a.o + ((tokb + t) * a.H + h) * kD + 32 * part;
        bool bad = false;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          tmem_ld16(tO + lrow + 32 * part + 16 * q, v);
          tmem_ld16(tO + lrow + kD + 32 * part + 16 * q, u);
#pragma unroll
          for (int c = 0; c < 16; c += 4) {
            const float4 x = make_float4(__fadd_rn(v[c], u[c]), __fadd_rn(v[c + 1], u[c + 1]),
                                         __fadd_rn(v[c + 2], u[c + 2]), __fadd_rn(v[c + 3], u[c + 3]));
            bad |= !isfinite(x.x) || !isfinite(x.y) || !isfinite(x.z) || !isfinite(x.w);
            *(float4*)&orow[16 * q + c] = x;
          }
        }
        if (bad) err |= BRS_FLAG_NONFINITE;
      }
      float* Ds = (float*)smem;                     // K^^T W rows for the write-back
      const int i = myrow;
#pragma unroll
      for (int q = 0; q < kCols / 16; ++q) {
        const int c0 = kCols * part + 16 * q;
        tmem_ld16(tD4 + lrow + c0, v);
        tmem_ld16(tD4 + lrow + kD + c0, u);
#pragma unroll
        for (int c = 0; c < 16; c += 4)
          *(float4*)&Ds[i * kSStride + c0 + c] = make_float4(__fadd_rn(v[c], u[c]), __fadd_rn(v[c + 1], u[c + 1]),
                                                             __fadd_rn(v[c + 2], u[c + 2]), __fadd_rn(v[c + 3], u[c + 3]));
      }
    }
    tc_fence_before();
    __syncthreads();
    // ---- write-back of the chunk
    const bool last = ch == nchunks - 1;
    tc_store_state<HAD, BLOCK, MODE, LB>((const float*)smem, g63, S0g, hst, aux, nlo, a.k_hi, a.hscale, a,
                                     a.step0 + t0 + kC - 1, h, b,
                                     (last && a.sdump) ? a.sdump + (size_t)head * kD * kD : nullptr, err);
    __syncthreads();
  }
    if (alive && c1 < nchunks) {
      // hand the head over: every thread's writes of the scratch, the stored
      // state and the residuals are made visible, then the counter moves
      __threadfence();
      __syncthreads();
      if (tid == 0 && !a.skip_handover) st_release_u32(a.handover + head, (uint32_t)c1);
    }
  }
  if (!alive) err |= BRS_FLAG_TIMEOUT;
  if (err) raise_flag(a.flags, err);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(512));
}

template <bool HAD, int BLOCK, int MODE, int LB>
cudaError_t tc_launch(const PrefillArgs& a, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<HAD, BLOCK, MODE, LB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  // one CTA per SM (the kernel's shared memory and tensor-memory columns
  // allow one), at most one per head; a cooperative launch, so that every
  // CTA is resident while another waits for its hand-over
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return cudaErrorInvalidValue;
  }
  int grid = a.B * a.H < sms ? a.B * a.H : sms;
  const int cap = prefill_cta_cap();
  if (cap > 0 && cap < grid) grid = cap;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prefill_tc_kernel<HAD, BLOCK, MODE, LB>, a);
}

template <bool HAD, int BLOCK, int LB>
cudaError_t tc_launch_hbl(const PrefillArgs& a, cudaStream_t st) {
  switch (a.mode) {
    case BRS_ROUND_NEAREST: return tc_launch<HAD, BLOCK, BRS_ROUND_NEAREST, LB>(a, st);
    case BRS_ROUND_STOCHASTIC: return tc_launch<HAD, BLOCK, BRS_ROUND_STOCHASTIC, LB>(a, st);
    case BRS_ROUND_ERRFEEDBACK: return tc_launch<HAD, BLOCK, BRS_ROUND_ERRFEEDBACK, LB>(a, st);
  }
  return cudaErrorInvalidValue;
}

template <bool HAD, int BLOCK>
cudaError_t tc_launch_hb(const PrefillArgs& a, cudaStream_t st) {
  return a.low_bits == 4 ? tc_launch_hbl<HAD, BLOCK, 4>(a, st) : tc_launch_hbl<HAD, BLOCK, 8>(a, st);
}

}  // namespace

bool prefill_supported(int d, int block, int k_hi, int C) {
  return d == kD && C == kC && (block == 128 || block == 32) && k_hi % 4 == 0 && k_hi <= kD;
}

size_t prefill_tc_scratch_bytes(int B, int H) { return (size_t)B * H * kD * kD * sizeof(float); }

cudaError_t launch_prefill_tc(const PrefillArgs& a, bool had, cudaStream_t st) {
  if (a.block == 128) return had ? tc_launch_hb<true, 128>(a, st) : tc_launch_hb<false, 128>(a, st);
  if (a.block == 32) return had ? tc_launch_hb<true, 32>(a, st) : tc_launch_hb<false, 32>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace brs
