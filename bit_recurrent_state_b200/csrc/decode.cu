// Decode step for FP32 and DAMP storage: one token for every (sequence,
// head).  One warp per head: lane l owns the CPL = D/32 consecutive columns
// CPL*l .. CPL*l+CPL-1 of every row and streams the head's rows in stored
// order twice: pass 1 dequantizes, decays and accumulates u = S^T k; pass 2
// reads the rows again (from L2), repeats the identical dequantize and
// decay, applies the delta-rule write, accumulates o = S^T q and requantizes
// in batches of NRB rows.  Every sum over rows is therefore lane-local (8-row
// chains and their pairwise tree), no thread block barrier is involved, and
// many heads run concurrently on every SM.
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
// with U1/O1 and U2/O2 the sums over the INT8 and the FP16 rows and T the
// Hadamard (or the identity).  Every sum over rows is taken in the library's
// order: 8-row fmaf chains in stored order, added in a pairwise tree
// (GroupTree).  Paired f32x2 instructions are two independent IEEE
// operations: pairing changes no result.
//
// Write-back modes: nearest, stochastic (Philox4x32-10), error feedback
// (FP16 residual), and direction memory ("When Quantization Breaks Memory",
// Post-training write-back interventions and diagnostics; Trajectory
// analysis): nearest codes plus a 2-bit sign counter per INT8 element that
// takes a vote from every proposed change inside (scale/8, scale/2) and
// moves the code one level at +-2; and k-bit residual memory (error feedback
// whose residual is kept as a k-bit integer of step/2^k, nibbles in the
// auxiliary buffer).  The kernel also carries the FP32 state
// between write-backs when the write-back interval is C > 1 (interval-state
// flags).
#include <cuda_runtime.h>
#include <cstdint>

#include "brs_device.cuh"
#include "brs_internal.h"

namespace brs {

constexpr int kWarpsPerCta = 2;   // small CTAs: an even spread of heads over the SMs
// kernel instantiation of k-bit residual memory (ABI modes BRS_ROUND_RESIDUAL2..4; k at run time)
constexpr int kModeResidual = 16;

template <int D>
struct WGeo {
  static constexpr int CPL = D / 32;             // columns per lane
  static constexpr int NRB = (D >= 64) ? 8 : 4;  // rows per requantization batch
};

// per stored row, duplicated into pairs for the paired FP32 instructions:
// ka = (k, k, a, a), sz = (scale, scale, zero, zero) of an INT8 row with one
// block per row, qq = (q, q)
struct __align__(16) RowScal {
  float4 ka, sz;
};

struct __align__(16) QPrm {
  float z, rcp, s;
  uint32_t pad;
};

template <int D>
struct __align__(16) WarpSmem {
  RowScal rs[D];                                 // per stored row: k, a, grid
  float2 qq[D];                                  // per stored row: q
  float vec[D];                                  // vector scratch (sums, w)
  QPrm prm[8][D / 32];                           // grids of one batch (row, block)
};

// ---- per-lane vector helpers over CPL values (pairs use f32x2); scalar
// factors arrive as the two halves of a duplicated pair
template <int C>
__device__ __forceinline__ void v_fma_s(float (&acc)[C], float k0, float k1, const float (&x)[C]) {
  if constexpr (C == 1) {
    acc[0] = __fmaf_rn(k0, x[0], acc[0]);
  } else {
#pragma unroll
    for (int c = 0; c < C; c += 2) fma2(acc[c], acc[c + 1], k0, k1, x[c], x[c + 1], acc[c], acc[c + 1]);
  }
}
template <int C>
__device__ __forceinline__ void v_fma_vec(float (&x)[C], float k0, float k1, const float (&w)[C]) {
  if constexpr (C == 1) {
    x[0] = __fmaf_rn(k0, w[0], x[0]);
  } else {
#pragma unroll
    for (int c = 0; c < C; c += 2) fma2(x[c], x[c + 1], k0, k1, w[c], w[c + 1], x[c], x[c + 1]);
  }
}
template <int C>
__device__ __forceinline__ void v_scale(float (&x)[C], float a0, float a1) {
  if constexpr (C == 1) {
    x[0] = __fmul_rn(a0, x[0]);
  } else {
#pragma unroll
    for (int c = 0; c < C; c += 2) mul2(x[c], x[c + 1], a0, a1, x[c], x[c + 1]);
  }
}

// dequantize CPL INT8 codes (the low CPL bytes of w, in column order):
// value = fmaf(code, scale, zero)
template <int C>
__device__ __forceinline__ void dequant_int8(float (&x)[C], uint32_t w, float s0, float s1, float z0,
                                             float z1) {
  if constexpr (C == 1) {
    const float c0 = __fsub_rn(byte_magic(w, 0), kTwo23);
    x[0] = __fmaf_rn(c0, s0, z0);
  } else {
#pragma unroll
    for (int c = 0; c < C; c += 2) {
      float c0 = byte_magic(w, c), c1 = byte_magic(w, c + 1);
      sub2(c0, c1, c0, c1, kTwo23, kTwo23);
      fma2(x[c], x[c + 1], c0, c1, s0, s1, z0, z1);
    }
  }
}

// CPL codes of the low tier starting at byte p (the lane's first column):
// LB = 8, one byte each; LB = 4, two to a byte (element e in bits 4 (e % 2)),
// for CPL = 1 the lane's nibble (column parity nsh / 4) alone
template <int C, int LB>
__device__ __forceinline__ uint32_t ld_codes(const uint8_t* p, int nsh) {
  if constexpr (LB == 8) {
    if constexpr (C == 4) return __ldg((const uint32_t*)p);
    else if constexpr (C == 2) return __ldg((const uint16_t*)p);
    else return __ldg(p);
  } else {
    if constexpr (C == 4) return __ldg((const uint16_t*)p);
    else if constexpr (C == 2) return __ldg(p);
    else return ((uint32_t)__ldg(p) >> nsh) & 15u;
  }
}

// dequantize CPL codes of either width: value = fmaf(code, scale, zero)
template <int C, int LB>
__device__ __forceinline__ void dequant_codes(float (&x)[C], uint32_t w, float s0, float s1, float z0,
                                              float z1) {
  if constexpr (LB == 8) {
    dequant_int8<C>(x, w, s0, s1, z0, z1);
  } else if constexpr (C == 1) {
    const float c0 = __fsub_rn(__uint_as_float(0x4B000000u | (w & 15u)), kTwo23);
    x[0] = __fmaf_rn(c0, s0, z0);
  } else {
#pragma unroll
    for (int c = 0; c < C; c += 2) {
      float c0 = __uint_as_float(0x4B000000u | ((w >> (4 * c)) & 15u));
      float c1 = __uint_as_float(0x4B000000u | ((w >> (4 * c + 4)) & 15u));
      sub2(c0, c1, c0, c1, kTwo23, kTwo23);
      fma2(x[c], x[c + 1], c0, c1, s0, s1, z0, z1);
    }
  }
}

// Sylvester Hadamard of a D-vector held CPL values per lane (lane l holds
// elements CPL*l ..), butterflies h = 1, 2, 4, ... then one scaling; every
// output is the same single add or subtract as in the sequential
// transform.
template <int D>
__device__ __forceinline__ void warp_fwht(float (&x)[D / 32], int lane, float scale) {
  constexpr int C = D / 32;
#pragma unroll
  for (int hs = 1; hs < C; hs <<= 1)
#pragma unroll
    for (int i = 0; i < C; ++i)
      if ((i & hs) == 0) {
        const float u0 = x[i], u1 = x[i + hs];
        x[i] = __fadd_rn(u0, u1);
        x[i + hs] = __fsub_rn(u0, u1);
      }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool hi = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < C; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, x[i], m);
      x[i] = hi ? __fsub_rn(o, x[i]) : __fadd_rn(x[i], o);
    }
  }
#pragma unroll
  for (int i = 0; i < C; ++i) x[i] = __fmul_rn(x[i], scale);
}

__device__ __forceinline__ uint32_t f16x2_overflow(uint32_t w) {
  return (((w >> 10) & 31u) == 31u) | (((w >> 26) & 31u) == 31u);
}

// packed code byte of a float holding (code + 1.5*2^23)
__device__ __forceinline__ uint32_t magic_byte(float m) { return __float_as_uint(m) & 0xffu; }

template <int D, int STORE, bool HAD, int BLOCK, int MODE, int LB>
__global__ void __launch_bounds__(32 * kWarpsPerCta, 8) decode_warp_kernel(const DecodeArgs a) {
  using G = WGeo<D>;
  constexpr int C = G::CPL, NRB = G::NRB;
  constexpr int RB = D * LB / 8;                 // bytes of one low-tier code row
  constexpr float LV = (float)((1 << LB) - 1);   // top code: 255 (INT8) or 15 (INT4)
  constexpr int NB = D / BLOCK;                  // blocks per row
  constexpr int GL = BLOCK / C;                  // lanes per block
  constexpr int V = 2 * NRB;                     // (min, max) entries per lane and batch
  constexpr int HALV = (V < GL) ? V : GL;        // halving stages keep min(V, GL) entries apart
  static_assert(GL <= 32 && (GL & (GL - 1)) == 0, "block spans a power-of-two run of lanes");
  __shared__ WarpSmem<D> smem_all[kWarpsPerCta];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int head = blockIdx.x * kWarpsPerCta + warp;
  if (head >= a.B * a.H) return;                 // whole warp leaves together
  WarpSmem<D>& sm = smem_all[warp];
  const int b = head / a.H, h = head - b * a.H;
  const int kh = h * a.Hk / a.H;
  const int nlo = (STORE == BRS_STORE_FP32) ? D : D - a.k_hi;   // INT8 rows 0..nlo-1
  const int col0 = C * lane;
  const int cb0 = col0 * LB / 8, nsh = 4 * (col0 & 1);   // my first code byte; my nibble (LB = 4, CPL = 1)
  const uint8_t* hin = (const uint8_t*)a.packed_in + (size_t)head * a.head_bytes;
  uint8_t* hout = (uint8_t*)a.packed_out + (size_t)head * a.head_bytes;
  const uint32_t* szin = (const uint32_t*)(hin + (size_t)nlo * RB + (size_t)a.k_hi * D * 2);
  uint32_t* szout = (uint32_t*)(hout + (size_t)nlo * RB + (size_t)a.k_hi * D * 2);
  const uint8_t* f16in = hin + (size_t)nlo * RB;
  uint16_t* f16out = (uint16_t*)(hout + (size_t)nlo * RB);
  uint16_t* auxb = (MODE == BRS_ROUND_ERRFEEDBACK) ? (uint16_t*)a.aux + (size_t)head * nlo * D : nullptr;
  // direction memory: 2-bit counters, four to a byte in column order
  uint8_t* dmb = (MODE == BRS_ROUND_DIRECTION) ? (uint8_t*)a.aux + (size_t)head * nlo * (D / 4) : nullptr;
  // residual memory: k-bit integers, two to a byte in column order
  uint8_t* rmb = (MODE == kModeResidual) ? (uint8_t*)a.aux + (size_t)head * nlo * (D / 2) : nullptr;
  const int rm_k = (MODE == kModeResidual) ? a.mode - BRS_ROUND_RESIDUAL2 + 2 : 2;   // residual bits
  const float rm_unit = (float)(1 << rm_k), rm_inv = __fdiv_rn(1.0f, rm_unit);   // 2^k, 2^-k (exact)
  const int rm_max = (1 << (rm_k - 1)) - 1;

  // ---- inputs: k, a, q gathered through the permutation and the stored
  // grid of every INT8 row, as ready pairs; v of my columns
  for (int i = lane; i < D; i += 32) {
    const int p = a.perm ? a.perm[h * D + i] : i;
    const size_t qk = ((size_t)b * a.Hk + kh) * D;
    const float kv = bf16_to_f32(a.k[qk + p]);
    const float av = a.decay_per_key ? a.decay[(size_t)head * D + p] : a.decay[head];
    const float qv = bf16_to_f32(a.q[qk + p]);
    float sv = 0.f, zv = 0.f;
    if (STORE != BRS_STORE_FP32 && NB == 1 && i < nlo) {
      const uint32_t w = __ldg(szin + i);
      sv = f16_to_f32((uint16_t)(w & 0xffffu));
      zv = f16_to_f32((uint16_t)(w >> 16));
    }
    RowScal r;
    r.ka = make_float4(kv, kv, av, av);
    r.sz = make_float4(sv, sv, zv, zv);
    sm.rs[i] = r;
    sm.qq[i] = make_float2(qv, qv);
  }
  float vv[C];
#pragma unroll
  for (int c = 0; c < C; ++c) vv[c] = bf16_to_f32(a.v[(size_t)head * D + col0 + c]);
  const float beta = a.beta[head];
  __syncwarp();

  float* s32h = (STORE != BRS_STORE_FP32 && a.s32) ? a.s32 + (size_t)head * D * D : nullptr;
  const bool src32 = (STORE != BRS_STORE_FP32) && a.src32;   // rows from the interval state
  const bool dst32 = (STORE != BRS_STORE_FP32) && a.dst32;   // updated rows to the interval state
  // one stored row -> FP32 values of my columns (before decay)
  auto load_row = [&](int i, float (&x)[C]) {
    if (STORE == BRS_STORE_FP32 || src32) {
      const float* src = (STORE == BRS_STORE_FP32) ? (const float*)hin + (size_t)i * D + col0
                                                  : s32h + (size_t)i * D + col0;
      if constexpr (C == 4) {
        const float4 f = __ldg((const float4*)src);
        x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
      } else if constexpr (C == 2) {
        const float2 f = __ldg((const float2*)src);
        x[0] = f.x; x[1] = f.y;
      } else {
        x[0] = __ldg(src);
      }
    } else {
      if (i < nlo) {
        const uint32_t w = ld_codes<C, LB>(hin + (size_t)i * RB + cb0, nsh);
        if constexpr (NB == 1) {
          const float4 g = sm.rs[i].sz;
          dequant_codes<C, LB>(x, w, g.x, g.y, g.z, g.w);
        } else {
          const uint32_t szw = __ldg(szin + i * NB + col0 / BLOCK);
          const float sv = f16_to_f32((uint16_t)(szw & 0xffffu)), zv = f16_to_f32((uint16_t)(szw >> 16));
          dequant_codes<C, LB>(x, w, sv, sv, zv, zv);
        }
      } else {
        const uint16_t* src = (const uint16_t*)f16in + (size_t)(i - nlo) * D + col0;
        if constexpr (C == 4) {
          const uint2 hv = __ldg((const uint2*)src);
          x[0] = f16_to_f32((uint16_t)(hv.x & 0xffffu)); x[1] = f16_to_f32((uint16_t)(hv.x >> 16));
          x[2] = f16_to_f32((uint16_t)(hv.y & 0xffffu)); x[3] = f16_to_f32((uint16_t)(hv.y >> 16));
        } else if constexpr (C == 2) {
          const uint32_t hv = __ldg((const uint32_t*)src);
          x[0] = f16_to_f32((uint16_t)(hv & 0xffffu)); x[1] = f16_to_f32((uint16_t)(hv >> 16));
        } else {
          x[0] = f16_to_f32(__ldg(src));
        }
      }
    }
  };

  // ---- pass 1: u = U2 + T(U1) over the decayed rows.  INT8 rows stream in
  // chunks of CH rows with the next chunk's codes and grids already in
  // flight (double buffering keeps 2*CH row loads per warp outstanding).
  // sums over rows in the library's order: rows arrive in stored order; a
  // group closes after 8 rows of its tier (or at the tier's end) and goes to
  // the tier's tree; the INT8 tier's tree gives U1, the FP16 tier's U2
  float u1[C], u2[C], acc[C];
  GroupTree<C> tree;
#pragma unroll
  for (int c = 0; c < C; ++c) { u1[c] = 0.f; u2[c] = 0.f; acc[c] = 0.f; }
  auto feed = [&](int i, float k0, float k1, const float (&x)[C], float (&t1)[C]) {
    v_fma_s<C>(acc, k0, k1, x);
    const bool lo_tier = i < nlo;
    const int rel = lo_tier ? i : i - nlo;
    if ((rel & 7) == 7 || i + 1 == (lo_tier ? nlo : D)) {
      tree.push(acc);
#pragma unroll
      for (int c = 0; c < C; ++c) acc[c] = 0.f;
    }
    if (i + 1 == nlo) {
      tree.result(t1);
      tree.n = 0;
    }
  };
  if constexpr (STORE == BRS_STORE_FP32) {
#pragma unroll 8
    for (int i = 0; i < D; ++i) {
      float x[C];
      load_row(i, x);
      const float4 ka = sm.rs[i].ka;
      v_scale<C>(x, ka.z, ka.w);
      feed(i, ka.x, ka.y, x, u1);
    }
  } else if (src32) {
    // FP32 rows from the interval state: the same chains, INT8 tier then
    // FP16 tier, in batches of NRB rows with the next batch's loads in flight
    float xb[2][NRB][C];
    const float* rb = s32h + col0;
    auto fetch32 = [&](int buf, int i0) {
#pragma unroll
      for (int r = 0; r < NRB; ++r) {
        const float* src = rb + (size_t)(i0 + r) * D;
        if constexpr (C == 4) {
          const float4 f = __ldg((const float4*)src);
          xb[buf][r][0] = f.x; xb[buf][r][1] = f.y; xb[buf][r][2] = f.z; xb[buf][r][3] = f.w;
        } else if constexpr (C == 2) {
          const float2 f = __ldg((const float2*)src);
          xb[buf][r][0] = f.x; xb[buf][r][1] = f.y;
        } else {
          xb[buf][r][0] = __ldg(src);
        }
      }
    };
    auto consume32 = [&](int buf, int i0) {
#pragma unroll
      for (int r = 0; r < NRB; ++r) {
        const float4 ka = sm.rs[i0 + r].ka;
        v_scale<C>(xb[buf][r], ka.z, ka.w);
        feed(i0 + r, ka.x, ka.y, xb[buf][r], u1);
      }
    };
    static_assert(D % (2 * NRB) == 0, "pairs of batches");
    fetch32(0, 0);
    for (int i0 = 0; i0 < D; i0 += 2 * NRB) {
      fetch32(1, i0 + NRB);
      consume32(0, i0);
      if (i0 + 2 * NRB < D) fetch32(0, i0 + 2 * NRB);
      consume32(1, i0 + NRB);
    }
  } else {
    // chunks of CH = NRB rows (nlo is a multiple of NRB), two in flight
    constexpr int CH = NRB;
    uint32_t cw[2][CH], sw[2][(NB > 1) ? CH : 1];
    const uint8_t* crow = hin + cb0;
    const uint32_t* srow = szin + col0 / BLOCK;
    auto fetch = [&](int buf) {
#pragma unroll
      for (int r = 0; r < CH; ++r) {
        cw[buf][r] = ld_codes<C, LB>(crow + r * RB, nsh);
        if constexpr (NB > 1) sw[buf][r] = __ldg(srow + r * NB);
      }
      crow += CH * RB;
      srow += CH * NB;
    };
    auto consume = [&](int buf, int i0) {
#pragma unroll
      for (int r = 0; r < CH; ++r) {
        float x[C];
        const RowScal rsc = sm.rs[i0 + r];
        if constexpr (NB == 1) {
          dequant_codes<C, LB>(x, cw[buf][r], rsc.sz.x, rsc.sz.y, rsc.sz.z, rsc.sz.w);
        } else {
          const float sv = f16_to_f32((uint16_t)(sw[buf][r] & 0xffffu));
          const float zv = f16_to_f32((uint16_t)(sw[buf][r] >> 16));
          dequant_codes<C, LB>(x, cw[buf][r], sv, sv, zv, zv);
        }
        v_scale<C>(x, rsc.ka.z, rsc.ka.w);
        feed(i0 + r, rsc.ka.x, rsc.ka.y, x, u1);
      }
    };
    const int nch = nlo / CH;
    if (nch > 0) fetch(0);
    for (int ch = 0; ch < nch; ch += 2) {
      if (ch + 1 < nch) fetch(1);
      consume(0, ch * CH);
      if (ch + 2 < nch) fetch(0);
      if (ch + 1 < nch) consume(1, (ch + 1) * CH);
    }
#pragma unroll 8
    for (int i = nlo; i < D; ++i) {
      float x[C];
      load_row(i, x);
      const float4 ka = sm.rs[i].ka;
      v_scale<C>(x, ka.z, ka.w);
      feed(i, ka.x, ka.y, x, u1);
    }
  }
  if (STORE != BRS_STORE_FP32) tree.result(u2);     // the FP16 tier (+0 when it is empty)
  float w[C], wt[C];
  {
    if constexpr (STORE != BRS_STORE_FP32 && HAD) warp_fwht<D>(u1, lane, a.hscale);
    bool bad = false;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const float u = (STORE == BRS_STORE_FP32) ? u1[c] : __fadd_rn(u2[c], u1[c]);
      bad |= !isfinite(u);
      w[c] = __fmul_rn(beta, __fsub_rn(vv[c], u));
      wt[c] = w[c];
    }
    if (bad) raise_flag(a.flags, BRS_FLAG_NONFINITE);
    if constexpr (STORE != BRS_STORE_FP32 && HAD) warp_fwht<D>(wt, lane, a.hscale);
  }

  // ---- pass 2: write, o, requantize (batches of NRB rows)
  float o1[C], o2[C];
#pragma unroll
  for (int c = 0; c < C; ++c) { o1[c] = 0.f; o2[c] = 0.f; acc[c] = 0.f; }
  tree.n = 0;
  // the next batch's rows are fetched while this batch is requantized
  uint32_t pw[NRB], ps[(NB > 1) ? NRB : 1];
  const uint8_t* prow = hin + cb0;
  const uint32_t* psrow = szin + col0 / BLOCK;
  auto prefetch = [&]() {
#pragma unroll
    for (int r = 0; r < NRB; ++r) {
      pw[r] = ld_codes<C, LB>(prow + r * RB, nsh);
      if constexpr (NB > 1) ps[r] = __ldg(psrow + r * NB);
    }
    prow += NRB * RB;
    psrow += NRB * NB;
  };
  if (STORE != BRS_STORE_FP32 && !src32 && nlo > 0) prefetch();
  for (int i0 = 0; i0 < D; i0 += NRB) {
    const bool int8_batch = (STORE != BRS_STORE_FP32) && (i0 < nlo);   // batches are tier-uniform
    float x[NRB][C];
    float xp[(MODE == BRS_ROUND_DIRECTION) ? NRB : 1][C];   // stored values the step started from
    float sp[(MODE == kModeResidual) ? NRB : 1];                // stored steps the step started from
    // the batch's rows: dequantized from the prefetched codes, or loaded
    // (all NRB loads issued before the first use)
    if (int8_batch && !src32) {
#pragma unroll
      for (int r = 0; r < NRB; ++r) {
        if constexpr (NB == 1) {
          const float4 g = sm.rs[i0 + r].sz;
          dequant_codes<C, LB>(x[r], pw[r], g.x, g.y, g.z, g.w);
          if constexpr (MODE == kModeResidual) sp[r] = g.x;
        } else {
          const float sv = f16_to_f32((uint16_t)(ps[r] & 0xffffu)), zv = f16_to_f32((uint16_t)(ps[r] >> 16));
          dequant_codes<C, LB>(x[r], pw[r], sv, sv, zv, zv);
          if constexpr (MODE == kModeResidual) sp[r] = sv;
        }
        if constexpr (MODE == BRS_ROUND_DIRECTION) {
#pragma unroll
          for (int c = 0; c < C; ++c) xp[r][c] = x[r][c];
        }
      }
    } else {
#pragma unroll
      for (int r = 0; r < NRB; ++r) load_row(i0 + r, x[r]);
    }
#pragma unroll
    for (int r = 0; r < NRB; ++r) {
      const int i = i0 + r;
      const RowScal rsc = sm.rs[i];
      const float2 qv = sm.qq[i];
      v_scale<C>(x[r], rsc.ka.z, rsc.ka.w);
      if (STORE == BRS_STORE_FP32 || i0 < nlo) v_fma_vec<C>(x[r], rsc.ka.x, rsc.ka.y, wt);
      else v_fma_vec<C>(x[r], rsc.ka.x, rsc.ka.y, w);
      feed(i, qv.x, qv.y, x[r], o1);
    }
    if (STORE != BRS_STORE_FP32 && !src32 && i0 + NRB < nlo) prefetch();
    if (STORE == BRS_STORE_FP32 || dst32) {
      // FP32 rows: the stored state (FP32 storage) or the interval state
#pragma unroll
      for (int r = 0; r < NRB; ++r) {
        float* dst = (STORE == BRS_STORE_FP32) ? (float*)hout + (size_t)(i0 + r) * D + col0
                                              : s32h + (size_t)(i0 + r) * D + col0;
        if constexpr (C == 4) *(float4*)dst = make_float4(x[r][0], x[r][1], x[r][2], x[r][3]);
        else if constexpr (C == 2) *(float2*)dst = make_float2(x[r][0], x[r][1]);
        else *dst = x[r][0];
      }
      continue;
    }
    if constexpr (STORE != BRS_STORE_FP32) {
      if (!int8_batch) {
        // protected rows: FP16, nearest
        uint32_t ovf = 0;
#pragma unroll
        for (int r = 0; r < NRB; ++r) {
          uint16_t* dst = f16out + (size_t)(i0 + r - nlo) * D + col0;
          if constexpr (C == 4) {
            const uint32_t lo = f16x2_of(x[r][0], x[r][1]), hi = f16x2_of(x[r][2], x[r][3]);
            ovf |= f16x2_overflow(lo) | f16x2_overflow(hi);
            *(uint2*)dst = make_uint2(lo, hi);
          } else if constexpr (C == 2) {
            const uint32_t lo = f16x2_of(x[r][0], x[r][1]);
            ovf |= f16x2_overflow(lo);
            *(uint32_t*)dst = lo;
          } else {
            const uint16_t hv = f32_to_f16(x[r][0]);
            ovf |= f16_inf_or_nan(hv);
            *dst = hv;
          }
        }
        if (ovf) raise_flag(a.flags, BRS_FLAG_OVERFLOW);
        continue;
      }
      // ---- INT8 batch: error-feedback target
      if constexpr (MODE == BRS_ROUND_ERRFEEDBACK) {
#pragma unroll
        for (int r = 0; r < NRB; ++r) {
          const uint16_t* e = auxb + (size_t)(i0 + r) * D + col0;
          uint16_t ev[C];
          if constexpr (C == 4) {
            const uint2 q = *(const uint2*)e;
            ev[0] = (uint16_t)(q.x & 0xffffu); ev[1] = (uint16_t)(q.x >> 16);
            ev[2] = (uint16_t)(q.y & 0xffffu); ev[3] = (uint16_t)(q.y >> 16);
          } else if constexpr (C == 2) {
            const uint32_t q = *(const uint32_t*)e;
            ev[0] = (uint16_t)(q & 0xffffu); ev[1] = (uint16_t)(q >> 16);
          } else {
            ev[0] = *e;
          }
#pragma unroll
          for (int c = 0; c < C; ++c) x[r][c] = __fadd_rn(x[r][c], f16_to_f32(ev[c]));
        }
      }
      // ---- INT8 batch: residual-memory target y + m (sprev / 2^k)
      uint32_t rmw[(MODE == kModeResidual) ? NRB : 1];     // my elements' integers, 4 bits each
      if constexpr (MODE == kModeResidual) {
#pragma unroll
        for (int r = 0; r < NRB; ++r) {
          const uint8_t* src = rmb + ((size_t)(i0 + r) * D + col0) / 2;
          if constexpr (C == 4) rmw[r] = *(const uint16_t*)src;
          else if constexpr (C == 2) rmw[r] = *src;
          else rmw[r] = (*src >> (4 * (col0 & 1))) & 15u;
          const float su = __fmul_rn(sp[r], rm_inv);       // exact
#pragma unroll
          for (int c = 0; c < C; ++c) {
            const int f = (int)((rmw[r] >> (4 * c)) & 15u);
            const int m = (f & 8) ? f - 16 : f;
            x[r][c] = __fadd_rn(x[r][c], __fmul_rn((float)m, su));
          }
        }
      }
      // ---- block extremes: local, then a reduce-scatter over the GL lanes
      // of the block; entry 2r / 2r+1 is the min / max of batch row r
      float v[V];
#pragma unroll
      for (int r = 0; r < NRB; ++r) {
        float mn = x[r][0], mx = x[r][0];
#pragma unroll
        for (int c = 1; c < C; ++c) { mn = fminf(mn, x[r][c]); mx = fmaxf(mx, x[r][c]); }
        v[2 * r] = mn;
        v[2 * r + 1] = mx;
      }
      // halving stages (offsets GL/2 .. GL/HALV), then all-reduce stages
      // (offsets below GL/HALV); afterwards lane g of the block group holds
      // entries [j0, j0 + VPL) with j0 = (g / (GL/HALV)) * VPL
      constexpr int VPL = V / HALV;
      static_assert(VPL <= 2, "one row per lane after the reduce-scatter");
#pragma unroll
      for (int m = GL / 2, len = V; m >= 1; m >>= 1) {
        if (len > VPL) {
          const bool up = (lane & m) != 0;
#pragma unroll
          for (int e = 0; e < len / 2; ++e) {
            const float lo = v[e], hi = v[e + len / 2];
            const float other = __shfl_xor_sync(0xffffffffu, up ? lo : hi, m);
            const float mine = up ? hi : lo;
            // entry parity: e's own while the kept length stays even,
            // else the lane bit that chose the half
            const bool is_max = (len / 2 >= 2) ? (e & 1) : up;
            v[e] = is_max ? fmaxf(mine, other) : fminf(mine, other);
          }
          len >>= 1;
        } else {
#pragma unroll
          for (int e = 0; e < VPL; ++e) {
            const float other = __shfl_xor_sync(0xffffffffu, v[e], m);
            const bool is_max = (VPL >= 2) ? (e & 1) : ((lane & (GL / HALV)) != 0);
            v[e] = is_max ? fmaxf(v[e], other) : fminf(v[e], other);
          }
        }
      }
      const int g = lane % GL, blk = col0 / BLOCK;
      const int j0 = (g / (GL / HALV)) * VPL;          // first entry held by this lane
      float mnv, mxv;
      int prow;
      bool param_lane;
      if constexpr (VPL >= 2) {
        mnv = v[0]; mxv = v[1];
        prow = j0 / 2;
        param_lane = (g % (GL / HALV)) == 0;
      } else {
        const int pbit = GL / HALV;                    // lane bit of the entry parity
        const float other = __shfl_xor_sync(0xffffffffu, v[0], pbit);
        const bool odd = (lane & pbit) != 0;
        mnv = odd ? other : v[0];
        mxv = odd ? v[0] : other;
        prow = j0 / 2;
        param_lane = (g % (2 * pbit)) == 0;
      }
      // a zero extreme takes the sign rule (-0 below +0): rare, warp-wide
      const bool zc = param_lane && ((mnv == 0.0f) || (mxv == 0.0f));
      if (__any_sync(0xffffffffu, zc)) {
        uint32_t nz = 0, pz = 0;
#pragma unroll
        for (int r = 0; r < NRB; ++r)
#pragma unroll
          for (int c = 0; c < C; ++c)
            if (x[r][c] == 0.0f) {
              if (signbit(x[r][c])) nz |= 1u << r; else pz |= 1u << r;
            }
#pragma unroll
        for (int m = 1; m < GL; m <<= 1) {
          nz |= __shfl_xor_sync(0xffffffffu, nz, m);
          pz |= __shfl_xor_sync(0xffffffffu, pz, m);
        }
        if (mnv == 0.0f) mnv = ((nz >> prow) & 1u) ? -0.0f : 0.0f;
        if (mxv == 0.0f) mxv = ((pz >> prow) & 1u) ? 0.0f : -0.0f;
      }
      // the grid of each (row, block), one division per lane; ok = the
      // block's extreme grid coordinates (the same monotone FP32 operations
      // as its elements') round into [0, LV]: no clip needed
      bool ok = true;
      if (param_lane) {
        const int i = i0 + prow;
        if (!isfinite(mnv) || !isfinite(mxv)) raise_flag(a.flags, BRS_FLAG_NONFINITE);
        const uint16_t sh = f32_to_f16(__fdiv_rn(__fsub_rn(mxv, mnv), LV));
        const uint16_t zh = f32_to_f16(mnv);
        if (f16_inf_or_nan(sh) || f16_inf_or_nan(zh)) raise_flag(a.flags, BRS_FLAG_OVERFLOW);
        const float s = f16_to_f32(sh), z = f16_to_f32(zh);
        const float rcp = (s == 0.0f) ? 0.0f : __frcp_rn(s);
        const float tlo = __fmul_rn(__fsub_rn(mnv, z), rcp), thi = __fmul_rn(__fsub_rn(mxv, z), rcp);
        ok = (tlo >= -0.5f) && (thi < LV + 0.5f);
        QPrm p;
        p.z = z; p.rcp = rcp; p.s = s; p.pad = 0;
        sm.prm[prow][blk] = p;
        szout[i * NB + blk] = (uint32_t)sh | ((uint32_t)zh << 16);
      }
      const bool fast = (MODE != BRS_ROUND_STOCHASTIC) && __all_sync(0xffffffffu, ok);
      __syncwarp();
      // ---- codes: clamp(round((y - zero) * (1/scale)), 0, LV); a zero
      // scale has 1/scale = 0, so every code of the block is 0
#pragma unroll
      for (int r = 0; r < NRB; ++r) {
        const int i = i0 + r;
        const QPrm p = sm.prm[r][blk];
        float tq[C];
#pragma unroll
        for (int c = 0; c < C; c += (C >= 2 ? 2 : 1)) {
          if constexpr (C >= 2) {
            float d0, d1;
            sub2(d0, d1, x[r][c], x[r][c + 1], p.z, p.z);
            mul2(tq[c], tq[c + 1], d0, d1, p.rcp, p.rcp);
          } else {
            tq[c] = __fmul_rn(__fsub_rn(x[r][c], p.z), p.rcp);
          }
        }
        if (!fast) {
          if constexpr (MODE == BRS_ROUND_STOCHASTIC) {
            const int e0 = i * D + col0;
            const uint4 rnd = philox4x32_10(make_uint4((uint32_t)(e0 / 4), (uint32_t)a.step, (uint32_t)h, (uint32_t)b),
                                            make_uint2((uint32_t)a.seed, (uint32_t)(a.seed >> 32)));
            const uint32_t words[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
#pragma unroll
            for (int c = 0; c < C; ++c) tq[c] = sr_round(tq[c], words[(e0 + c) & 3] >> 8);
          }
#pragma unroll
          for (int c = 0; c < C; ++c) tq[c] = fminf(fmaxf(tq[c], 0.0f), LV);
        }
        // nearest integer (ties to even): the low byte of t + 1.5*2^23; the
        // paired add is written t * one + magic with one = 1 read at run
        // time (the same single rounding), so it cannot be merged with the
        // multiply before it
        float mq[C];
#pragma unroll
        for (int c = 0; c < C; c += (C >= 2 ? 2 : 1)) {
          if constexpr (C >= 2) fma2(mq[c], mq[c + 1], tq[c], tq[c + 1], a.one, a.one, kRoundMagic, kRoundMagic);
          else mq[c] = __fadd_rn(tq[c], kRoundMagic);
        }
        if constexpr (MODE == BRS_ROUND_DIRECTION) {
          // votes of the proposed changes y - xp inside (scale/8, scale/2);
          // a counter at +-2 moves the nearest code one level (clipped to
          // [0, LV]) and is reset.  The lanes of one counter byte merge
          // their fields before one of them stores it.
          uint8_t* dmp = dmb + (size_t)i * (D / 4) + col0 / 4;
          const uint32_t old = *dmp;
          const int sh0 = 2 * (col0 & 3);
          const float lo = __fmul_rn(p.s, 0.125f), hi = __fmul_rn(p.s, 0.5f);
          uint32_t nb = 0;
#pragma unroll
          for (int c = 0; c < C; ++c) {
            const int f = (int)((old >> (sh0 + 2 * c)) & 3u);
            int m = (f & 2) ? f - 4 : f;
            const float dl = __fsub_rn(x[r][c], xp[r][c]);
            const float ad = fabsf(dl);
            if (ad > lo && ad < hi) m += (dl > 0.0f) ? 1 : -1;
            if (m >= 2 || m <= -2) {
              const uint32_t mb = __float_as_uint(mq[c]);
              const int code = min(max((int)(mb & 0xffu) + (m > 0 ? 1 : -1), 0), (int)LV);
              mq[c] = __uint_as_float((mb & ~0xffu) | (uint32_t)code);
              m = 0;
            }
            nb |= ((uint32_t)m & 3u) << (sh0 + 2 * c);
          }
          if constexpr (C <= 2) nb |= __shfl_xor_sync(0xffffffffu, nb, 1);
          if constexpr (C == 1) nb |= __shfl_xor_sync(0xffffffffu, nb, 2);
          if ((col0 & 3) == 0) *dmp = (uint8_t)nb;
        }
        uint8_t* dst = hout + (size_t)i * RB + cb0;
        if constexpr (LB == 4) {
          // codes 0..15 in the low nibble of each magic float's byte
          uint32_t nbl = 0;
#pragma unroll
          for (int c = 0; c < C; ++c) nbl |= (magic_byte(mq[c]) & 15u) << (4 * c);
          if constexpr (C == 4) {
            *(uint16_t*)dst = (uint16_t)nbl;
          } else if constexpr (C == 2) {
            *dst = (uint8_t)nbl;
          } else {
            nbl <<= nsh;
            nbl |= __shfl_xor_sync(0xffffffffu, nbl, 1);
            if ((col0 & 1) == 0) *dst = (uint8_t)nbl;
          }
        } else if constexpr (C == 4) {
          *(uint32_t*)dst = __byte_perm(__byte_perm(__float_as_uint(mq[0]), __float_as_uint(mq[1]), 0x0040u),
                                        __byte_perm(__float_as_uint(mq[2]), __float_as_uint(mq[3]), 0x0040u), 0x5410u);
        } else if constexpr (C == 2) {
          *(uint16_t*)dst = (uint16_t)__byte_perm(__float_as_uint(mq[0]), __float_as_uint(mq[1]), 0x0040u);
        } else {
          *dst = (uint8_t)magic_byte(mq[0]);
        }
        if constexpr (MODE == kModeResidual) {
          // the new integers: rne((y - value) * (1/scale) * 2^k), clipped to
          // +-(2^(k-1) - 1); the lanes of one byte merge their nibbles
          uint32_t nb = 0;
#pragma unroll
          for (int c = 0; c < C; ++c) {
            const float code = __fsub_rn(mq[c], kRoundMagic);          // exact
            const float res = __fsub_rn(x[r][c], __fmaf_rn(code, p.s, p.z));
            const float q = rintf(__fmul_rn(__fmul_rn(res, p.rcp), rm_unit));
            int m = (q != q) ? 0 : (int)fminf(fmaxf(q, (float)-rm_max), (float)rm_max);
            nb |= ((uint32_t)m & 15u) << (4 * c);
          }
          uint8_t* dst = rmb + ((size_t)i * D + col0) / 2;
          if constexpr (C == 4) {
            *(uint16_t*)dst = (uint16_t)nb;
          } else if constexpr (C == 2) {
            *dst = (uint8_t)nb;
          } else {
            nb <<= 4 * (col0 & 1);
            nb |= __shfl_xor_sync(0xffffffffu, nb, 1);
            if ((col0 & 1) == 0) *dst = (uint8_t)nb;
          }
        }
        if constexpr (MODE == BRS_ROUND_ERRFEEDBACK) {
          uint16_t ev[C];
#pragma unroll
          for (int c = 0; c < C; ++c) {
            const float code = __fsub_rn(mq[c], kRoundMagic);          // exact
            float e = __fsub_rn(x[r][c], __fmaf_rn(code, p.s, p.z));
            if (e > p.s) e = p.s;
            else if (e < -p.s) e = -p.s;
            ev[c] = f32_to_f16(e);
          }
          uint16_t* ed = auxb + (size_t)i * D + col0;
          if constexpr (C == 4) *(uint2*)ed = make_uint2((uint32_t)ev[0] | ((uint32_t)ev[1] << 16), (uint32_t)ev[2] | ((uint32_t)ev[3] << 16));
          else if constexpr (C == 2) *(uint32_t*)ed = (uint32_t)ev[0] | ((uint32_t)ev[1] << 16);
          else *ed = ev[0];
        }
      }
      __syncwarp();                                    // sm.prm reused by the next batch
    }
  }

  // ---- o = O2 + T(O1)
  if (STORE != BRS_STORE_FP32) tree.result(o2);
  if constexpr (STORE != BRS_STORE_FP32 && HAD) warp_fwht<D>(o1, lane, a.hscale);
  float ov[C];
  bool bad = false;
#pragma unroll
  for (int c = 0; c < C; ++c) {
    ov[c] = (STORE == BRS_STORE_FP32) ? o1[c] : __fadd_rn(o2[c], o1[c]);
    bad |= !isfinite(ov[c]);
  }
  if (bad) raise_flag(a.flags, BRS_FLAG_NONFINITE);
  float* od = a.o + (size_t)head * D + col0;
  if constexpr (C == 4) *(float4*)od = make_float4(ov[0], ov[1], ov[2], ov[3]);
  else if constexpr (C == 2) *(float2*)od = make_float2(ov[0], ov[1]);
  else *od = ov[0];
}

template <int D, int BLOCK, int MODE, int LB = 8>
static cudaError_t launch_dbm(const DecodeArgs& a, int store, bool had, cudaStream_t st) {
  const int heads = a.B * a.H;
  const dim3 grid((heads + kWarpsPerCta - 1) / kWarpsPerCta), block(32 * kWarpsPerCta);
  if (store == BRS_STORE_FP32)
    decode_warp_kernel<D, BRS_STORE_FP32, false, D, BRS_ROUND_NEAREST, 8><<<grid, block, 0, st>>>(a);
  else if (had)
    decode_warp_kernel<D, BRS_STORE_DAMP, true, BLOCK, MODE, LB><<<grid, block, 0, st>>>(a);
  else
    decode_warp_kernel<D, BRS_STORE_DAMP, false, BLOCK, MODE, LB><<<grid, block, 0, st>>>(a);
  return cudaGetLastError();
}

template <int D, int BLOCK, int LB>
static cudaError_t launch_dbl(const DecodeArgs& a, int store, bool had, cudaStream_t st) {
  switch (a.mode) {
    case BRS_ROUND_NEAREST: return launch_dbm<D, BLOCK, BRS_ROUND_NEAREST, LB>(a, store, had, st);
    case BRS_ROUND_STOCHASTIC: return launch_dbm<D, BLOCK, BRS_ROUND_STOCHASTIC, LB>(a, store, had, st);
    case BRS_ROUND_ERRFEEDBACK: return launch_dbm<D, BLOCK, BRS_ROUND_ERRFEEDBACK, LB>(a, store, had, st);
    case BRS_ROUND_DIRECTION: return launch_dbm<D, BLOCK, BRS_ROUND_DIRECTION, LB>(a, store, had, st);
    case BRS_ROUND_RESIDUAL2:
    case BRS_ROUND_RESIDUAL3:
    case BRS_ROUND_RESIDUAL4: return launch_dbm<D, BLOCK, kModeResidual, LB>(a, store, had, st);
  }
  return cudaErrorInvalidValue;
}

// low tier width: 8 (INT8) or 4 (two codes per byte)
template <int D, int BLOCK>
static cudaError_t launch_db(const DecodeArgs& a, int store, bool had, cudaStream_t st) {
  if (a.low_bits == 4) return launch_dbl<D, BLOCK, 4>(a, store, had, st);
  return launch_dbl<D, BLOCK, 8>(a, store, had, st);
}

cudaError_t launch_decode_deferred(const DecodeArgs& a, int d, bool had, cudaStream_t st) {
  if (d == 128 && a.block == 128) return launch_db<128, 128>(a, BRS_STORE_DAMP, had, st);
  if (d == 128 && a.block == 32) return launch_db<128, 32>(a, BRS_STORE_DAMP, had, st);
  if (d == 64 && a.block == 64) return launch_db<64, 64>(a, BRS_STORE_DAMP, had, st);
  if (d == 32 && a.block == 32) return launch_db<32, 32>(a, BRS_STORE_DAMP, had, st);
  return cudaErrorInvalidValue;
}

bool decode_supported(int d, int block, int k_hi) {
  const bool shape = (d == 128 && (block == 128 || block == 32)) || (d == 64 && block == 64) ||
                     (d == 32 && block == 32);
  const int nrb = (d >= 64) ? 8 : 4;
  return shape && k_hi % nrb == 0;
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
  if (decode_cta_supported(d, store, a.block, a.k_hi, a.mode)) return launch_decode_cta(a, had, st);
  if (d == 128 && a.block == 128) return launch_db<128, 128>(a, store, had, st);
  if (d == 128 && a.block == 32) return launch_db<128, 32>(a, store, had, st);
  if (d == 64 && a.block == 64) return launch_db<64, 64>(a, store, had, st);
  if (d == 32 && a.block == 32) return launch_db<32, 32>(a, store, had, st);
  return cudaErrorInvalidValue;
}

}  // namespace brs
