// Decode step for variable-width storage ("Low-Bit Recurrent States in
// Hybrid Language Models": State bit allocation, Allocation units, Levels
// and storage; the widths are recomputed at every write-back from
// c_i = Gamma_hat_i * R~_i^2 under a layer-wise budget).
//
// Three launches per token, because a row's width depends on the updated
// state of every head of its sequence:
//   1. varbit_kernel<PHASE 0>, one warp per head: dequantize, decay, delta
//      write, o = S^T q (written out), the row ranges R_i of the updated
//      FP32 state, the chunk-aware EMA statistics (a^2 and
//      beta (2 - beta) k^2, span 64) and the costs c_i -> workspace;
//   2. the allocator (allocate.cu) over each budget group -> widths and
//      row offsets of the output state;
//   3. varbit_kernel<PHASE 1>, one warp per head: the identical update again
//      (same FP32 operations, same results), then per row the fitted step
//      (16 clip factors, one quarter of a warp per row, four candidates per
//      lane, so each fit-error sum is an fmaf chain over the row in order),
//      the codes (nearest / Philox stochastic / error feedback) and the
//      bit-packed row at its new offset.
// Layout of the update: lane l owns columns 4l..4l+3 (d = 128) of every
// row, so each sum over rows is lane-local: 8-row fmaf chains in row order
// added in a pairwise tree (the library's order, GroupTree).
#include <cuda_runtime.h>
#include <cstdint>
#include <type_traits>

#include "brs_device.cuh"
#include "brs_internal.h"

namespace brs {

constexpr int kVbWarps = 2;      // warps (heads) per CTA
constexpr int kVbBatch = 8;      // rows per requantization batch

struct __align__(16) VbRow {
  float4 ka;                     // (k, k, a, a)
  float2 qq;                     // (q, q)
  float step;                    // stored step of the input row
  int bw;                        // input width
  uint32_t off;                  // input byte offset within the sequence payload
  int n;                         // 2^(bw-1) - 1 (1 for one-bit rows)
  int one;                       // one-bit row: level = 2 u - 1
  float pad;
};

template <int D, bool WIDE>
struct __align__(16) VbSmem {
  VbRow row[D];
  float R[D];                    // row ranges (phase 0)
  float y[kVbBatch][D + 4];      // one batch of target magnitudes (phase 1), rows 16-byte aligned
  uint32_t pk[kVbBatch][WIDE ? 64 : 32];   // bit-packed output rows of the batch (widths up to 16 / 8)
  float pstep[kVbBatch], pinv[kVbBatch];
};

// decode the CPL codes of lane `lane` in one input row (widths up to 8: C *
// width <= 32 bits over one or two words; WIDE, up to 16: <= 64 bits over up
// to three words)
template <int C, bool WIDE, bool ONE>
__device__ __forceinline__ void vb_dequant(float (&x)[C], const uint8_t* rowbase, const VbRow& r, int lane) {
  const uint32_t* rp = (const uint32_t*)rowbase;
  const int sb = C * lane * r.bw;
  const int sh = sb & 31;
  uint64_t chunk;
  if constexpr (WIDE) {
    const int w0 = sb >> 5, need = sh + C * r.bw;
    uint64_t lo = __ldg(rp + w0);
    if (need > 32) lo |= (uint64_t)__ldg(rp + w0 + 1) << 32;
    chunk = lo >> sh;
    if (need > 64) chunk |= (uint64_t)__ldg(rp + w0 + 2) << (64 - sh);
  } else {
    // both words loaded unconditionally (no divergent second load): the word
    // after a row's last one is the next row's, or past the payload the
    // first of the step section, inside the stored state either way
    chunk = __funnelshift_r(__ldg(rp + (sb >> 5)), __ldg(rp + (sb >> 5) + 1), sh);
  }
  const uint32_t mask = (1u << r.bw) - 1u;
#pragma unroll
  for (int c = 0; c < C; ++c) {
    const uint32_t u = (uint32_t)(chunk >> (c * r.bw)) & mask;
    const int qv = ONE ? (int)(u << r.one) - r.n : (int)u - r.n;   // one bit: 2u - 1
    x[c] = __fmul_rn(__fsub_rn(__int_as_float(0x4B400000 + qv), kRoundMagic), r.step);  // (u - n) * step
  }
}

template <int D, int PHASE, int MODE, bool WIDE, bool ONE>
__global__ void __launch_bounds__(32 * kVbWarps) varbit_kernel(const VbArgs a) {
  constexpr int C = D / 32;
  static_assert(D == 128, "variable-width decode is built for d = 128");
  __shared__ VbSmem<D, WIDE> smem_all[kVbWarps];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int head = blockIdx.x * kVbWarps + warp;
  if (head >= a.B * a.H) return;
  VbSmem<D, WIDE>& sm = smem_all[warp];
  const int b = head / a.H, h = head - b * a.H;
  const int rows = a.H * D;
  const int col0 = C * lane;
  const uint8_t* pin = (const uint8_t*)a.packed_in;
  uint8_t* pout = (uint8_t*)a.packed_out;
  const uint8_t* pay_in = pin + (size_t)b * a.sec.payload_per_seq;
  const uint16_t* sc_in = (const uint16_t*)(pin + a.sec.off_scale) + (size_t)b * rows + h * D;
  const uint8_t* wd_in = pin + a.sec.off_width + (size_t)b * rows + h * D;
  const uint32_t* of_in = (const uint32_t*)(pin + a.sec.off_offsets) + (size_t)b * (rows + 1) + h * D;

  // ---- per-row records
  for (int i = lane; i < D; i += 32) {
    const size_t qk = ((size_t)b * a.Hk + h * a.Hk / a.H) * D;
    const float kv = bf16_to_f32(a.k[qk + i]);
    const float av = a.decay_per_key ? a.decay[(size_t)head * D + i] : a.decay[head];
    const float qv = bf16_to_f32(a.q[qk + i]);
    VbRow r;
    r.ka = make_float4(kv, kv, av, av);
    r.qq = make_float2(qv, qv);
    r.step = f16_to_f32(sc_in[i]);
    r.bw = wd_in[i];
    r.off = of_in[i];
    r.one = r.bw == 1;
    r.n = r.one ? 1 : (1 << (r.bw - 1)) - 1;
    r.pad = 0.f;
    sm.row[i] = r;
  }
  float vv[C];
#pragma unroll
  for (int c = 0; c < C; ++c) vv[c] = bf16_to_f32(a.v[(size_t)head * D + col0 + c]);
  const float beta = a.beta[head];
  __syncwarp();

  // ---- pass 1: u = S^T k over the decayed rows (8-row chains, pairwise tree)
  float u[C];
  GroupTree<C> tree;
  for (int g = 0; g < D / 8; ++g) {
    float acc[C];
#pragma unroll
    for (int c = 0; c < C; ++c) acc[c] = 0.f;
#pragma unroll 4
    for (int i = 8 * g; i < 8 * g + 8; ++i) {
      const VbRow r = sm.row[i];
      float x[C];
      vb_dequant<C, WIDE, ONE>(x, pay_in + r.off, r, lane);
#pragma unroll
      for (int c = 0; c < C; c += 2) {
        mul2(x[c], x[c + 1], r.ka.z, r.ka.w, x[c], x[c + 1]);
        fma2(acc[c], acc[c + 1], r.ka.x, r.ka.y, x[c], x[c + 1], acc[c], acc[c + 1]);
      }
    }
    tree.push(acc);
  }
  tree.result(u);
  float w[C];
  {
    bool bad = false;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      bad |= !isfinite(u[c]);
      w[c] = __fmul_rn(beta, __fsub_rn(vv[c], u[c]));
    }
    if (bad) raise_flag(a.flags, BRS_FLAG_NONFINITE);
  }

  // ---- pass 2 in batches (a batch is one 8-row group of o's sum)
  static_assert(kVbBatch == 8, "a requantization batch is one group of the row sums");
  float o[C];
  tree.n = 0;
  const uint8_t* pay_out = pout + (size_t)b * a.sec.payload_per_seq;
  const uint8_t* wd_out = pout + a.sec.off_width + (size_t)b * rows + h * D;
  const uint32_t* of_out = (const uint32_t*)(pout + a.sec.off_offsets) + (size_t)b * (rows + 1) + h * D;
  uint16_t* sc_out = (uint16_t*)(pout + a.sec.off_scale) + (size_t)b * rows + h * D;
  uint16_t* auxh = (MODE == BRS_ROUND_ERRFEEDBACK) ? (uint16_t*)a.aux + (size_t)head * D * D : nullptr;

  for (int i0 = 0; i0 < D; i0 += kVbBatch) {
    float x[kVbBatch][C], og[C];
#pragma unroll
    for (int c = 0; c < C; ++c) og[c] = 0.f;
#pragma unroll
    for (int r = 0; r < kVbBatch; ++r) {
      const VbRow rr = sm.row[i0 + r];
      vb_dequant<C, WIDE, ONE>(x[r], pay_in + rr.off, rr, lane);
#pragma unroll
      for (int c = 0; c < C; c += 2) {
        mul2(x[r][c], x[r][c + 1], rr.ka.z, rr.ka.w, x[r][c], x[r][c + 1]);
        fma2(x[r][c], x[r][c + 1], rr.ka.x, rr.ka.y, w[c], w[c + 1], x[r][c], x[r][c + 1]);
      }
      if constexpr (PHASE == 0) {
#pragma unroll
        for (int c = 0; c < C; c += 2) fma2(og[c], og[c + 1], rr.qq.x, rr.qq.y, x[r][c], x[r][c + 1], og[c], og[c + 1]);
      }
    }
    if constexpr (PHASE == 0) tree.push(og);
    if constexpr (MODE == BRS_ROUND_ERRFEEDBACK && PHASE == 1) {
#pragma unroll
      for (int r = 0; r < kVbBatch; ++r) {
        const uint2 ev = *(const uint2*)&auxh[(size_t)(i0 + r) * D + col0];
        x[r][0] = __fadd_rn(x[r][0], f16_to_f32((uint16_t)(ev.x & 0xffffu)));
        x[r][1] = __fadd_rn(x[r][1], f16_to_f32((uint16_t)(ev.x >> 16)));
        x[r][2] = __fadd_rn(x[r][2], f16_to_f32((uint16_t)(ev.y & 0xffffu)));
        x[r][3] = __fadd_rn(x[r][3], f16_to_f32((uint16_t)(ev.y >> 16)));
      }
    }
    // row absolute maxima of this batch (updated state in phase 0, the
    // quantization target in phase 1): halving stages leave entry
    // j = lane / 4 on lanes 4j..4j+3, reduced over the warp
    float v[kVbBatch];
#pragma unroll
    for (int r = 0; r < kVbBatch; ++r) {
      float m = fabsf(x[r][0]);
#pragma unroll
      for (int c = 1; c < C; ++c) m = fmaxf(m, fabsf(x[r][c]));
      v[r] = m;
    }
#pragma unroll
    for (int m = 16, len = kVbBatch; m >= 1; m >>= 1) {
      if (len > 1) {
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int e = 0; e < len / 2; ++e) {
          const float lo = v[e], hi = v[e + len / 2];
          const float other = __shfl_xor_sync(0xffffffffu, up ? lo : hi, m);
          v[e] = fmaxf(up ? hi : lo, other);
        }
        len >>= 1;
      } else {
        v[0] = fmaxf(v[0], __shfl_xor_sync(0xffffffffu, v[0], m));
      }
    }
    const int jr = lane >> 2;                       // batch row of this lane's entry
    if constexpr (PHASE == 0) {
      if ((lane & 3) == 0) sm.R[i0 + jr] = v[0];
      continue;
    } else {
      const float R = v[0];
      // ---- magnitudes of the batch's targets to shared memory (rows padded
      // by one): the fit error of -y equals that of y (rounding to nearest
      // even and the clip at +-n are odd functions, each residual only
      // changes sign), so the fit runs on |y| with a one-sided clip
#pragma unroll
      for (int r = 0; r < kVbBatch; ++r)
        *(float4*)&sm.y[r][col0] = make_float4(fabsf(x[r][0]), fabsf(x[r][1]), fabsf(x[r][2]), fabsf(x[r][3]));
      __syncwarp();
      // ---- fitted step: row jr, candidates m = q, q+4, q+8, q+12
      const int q4 = lane & 3;
      const int bw = wd_out[i0 + jr];
      const bool one = ONE && bw == 1;             // one-bit row: no fitted step
      const int n = one ? 1 : (1 << (bw - 1)) - 1;
      const float fn = (float)n;
      float st[4], iv[4], E[4];
      uint16_t sb[4];
      bool ok[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        varbit_candidate(q4 + 4 * k, R, n, st[k], iv[k], sb[k], ok[k]);
        E[k] = 0.f;
      }
      const float* yrow = sm.y[jr];
#pragma unroll 2
      for (int j4 = 0; j4 < (one ? 0 : D); j4 += 4) {
        const float4 y4 = *(const float4*)&yrow[j4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
        const float y = jj == 0 ? y4.x : jj == 1 ? y4.y : jj == 2 ? y4.z : y4.w;
        float t0, t1, t2, t3;
        mul2(t0, t1, y, y, iv[0], iv[1]);
        mul2(t2, t3, y, y, iv[2], iv[3]);
        // nearest integer (ties to even); t * one + magic with one = 1 read at
        // run time, the add's single rounding, never merged with the multiply
        fma2(t0, t1, t0, t1, a.one, a.one, kRoundMagic, kRoundMagic);
        fma2(t2, t3, t2, t3, a.one, a.one, kRoundMagic, kRoundMagic);
        sub2(t0, t1, t0, t1, kRoundMagic, kRoundMagic);
        sub2(t2, t3, t2, t3, kRoundMagic, kRoundMagic);
        t0 = fminf(t0, fn);
        t1 = fminf(t1, fn);
        t2 = fminf(t2, fn);
        t3 = fminf(t3, fn);
        mul2(t0, t1, st[0], st[1], t0, t1);                 // step * level
        mul2(t2, t3, st[2], st[3], t2, t3);
        sub2(t0, t1, y, y, t0, t1);                         // residual
        sub2(t2, t3, y, y, t2, t3);
        fma2(E[0], E[1], t0, t1, t0, t1, E[0], E[1]);
        fma2(E[2], E[3], t2, t3, t2, t3, E[2], E[3]);
        }
      }
      // best of the lane (ascending m), then of the row's four lanes
      int bm = 99;
      float bE = 0.f;
      uint16_t bbits = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (ok[k] && (bm == 99 || E[k] < bE)) { bm = q4 + 4 * k; bE = E[k]; bbits = sb[k]; }
#pragma unroll
      for (int m = 1; m <= 2; m <<= 1) {
        const int om = __shfl_xor_sync(0xffffffffu, bm, m);
        const float oE = __shfl_xor_sync(0xffffffffu, bE, m);
        const uint16_t ob = (uint16_t)__shfl_xor_sync(0xffffffffu, (uint32_t)bbits, m);
        const bool take = (om != 99) && (bm == 99 || oE < bE || (oE == bE && om < bm));
        if (take) { bm = om; bE = oE; bbits = ob; }
      }
      if (R == 0.0f) { bm = 0; bbits = 0; }
      if (one) {
        // one-bit row ([LB] Levels and storage): the sign times the row's mean
        // absolute value, the magnitudes summed in element order by the row's
        // first lane, times 1/d, stored as the FP16 scale
        if (q4 == 0) {
          float sum = 0.0f;
          for (int j = 0; j < D; ++j) sum = __fadd_rn(sum, yrow[j]);
          bbits = f32_to_f16(__fmul_rn(sum, 1.0f / (float)D));
        }
        bm = 0;
      }
      if (bm == 99) { bbits = 0x7c00u; if (q4 == 0) raise_flag(a.flags, BRS_FLAG_OVERFLOW); }
      if (q4 == 0) {
        const float step = f16_to_f32(bbits);
        const bool good = step != 0.0f && isfinite(step);
        sm.pstep[jr] = good ? step : 0.0f;
        sm.pinv[jr] = good ? __frcp_rn(step) : 0.0f;
        sc_out[i0 + jr] = bbits;
      }
      for (int k = lane; k < kVbBatch * (WIDE ? 64 : 32); k += 32) (&sm.pk[0][0])[k] = 0u;
      __syncwarp();
      // ---- codes of my columns, bit-packed into the batch rows
#pragma unroll
      for (int r = 0; r < kVbBatch; ++r) {
        const int i = i0 + r;
        const int rbw = wd_out[i];
        const bool rone = ONE && rbw == 1;
        const int rn = rone ? 0 : (1 << (rbw - 1)) - 1;
        const float rfn = (float)rn;
        const float step = sm.pstep[r], inv = sm.pinv[r];
        float qv[C];
        uint4 rnd = make_uint4(0, 0, 0, 0);
        if constexpr (MODE == BRS_ROUND_STOCHASTIC)
          rnd = philox4x32_10(make_uint4((uint32_t)((i * D + col0) / 4), (uint32_t)a.step, (uint32_t)h, (uint32_t)b),
                              make_uint2((uint32_t)a.seed, (uint32_t)(a.seed >> 32)));
        const uint32_t words[4] = {rnd.x >> 8, rnd.y >> 8, rnd.z >> 8, rnd.w >> 8};
        using chunk_t = std::conditional_t<WIDE, uint64_t, uint32_t>;
        chunk_t chunk = 0;
#pragma unroll
        for (int c = 0; c < C; ++c) {
          const float t = __fmul_rn(x[r][c], inv);
          float qf;
          uint32_t u;
          if (rone) {
            // one bit: +mu for a target >= 0 (nearest), or with probability
            // (t + 1) / 2 (stochastic); the level is +-1
            if (MODE == BRS_ROUND_STOCHASTIC) {
              const float cc = fminf(fmaxf(sr_round(__fmul_rn(__fadd_rn(t, 1.0f), 0.5f), words[c]), 0.0f), 1.0f);
              u = cc > 0.0f ? 1u : 0u;
            } else {
              u = x[r][c] >= 0.0f ? 1u : 0u;
            }
            qf = u ? 1.0f : -1.0f;
          } else {
            qf = (MODE == BRS_ROUND_STOCHASTIC) ? sr_round(t, words[c]) : rintf(t);
            qf = fminf(fmaxf(qf, -rfn), rfn);
            u = (uint32_t)((int)qf + rn);
          }
          qv[c] = qf;
          chunk |= (chunk_t)u << (c * rbw);
        }
        const int sbit = C * lane * rbw, sh = sbit & 31, w0 = sbit >> 5;
        if constexpr (WIDE) {
          atomicOr(&sm.pk[r][w0], (uint32_t)(chunk << sh));
          if (sh + C * rbw > 32) atomicOr(&sm.pk[r][w0 + 1], (uint32_t)(chunk >> (32 - sh)));
          if (sh + C * rbw > 64) atomicOr(&sm.pk[r][w0 + 2], (uint32_t)(chunk >> (64 - sh)));
        } else {
          const uint32_t c32 = (uint32_t)chunk;
          atomicOr(&sm.pk[r][w0], c32 << sh);
          if (sh + C * rbw > 32) atomicOr(&sm.pk[r][w0 + 1], c32 >> (32 - sh));
        }
        if constexpr (MODE == BRS_ROUND_ERRFEEDBACK) {
          uint16_t e16[C];
          const float lim = rone ? __fmul_rn(2.0f, step) : step;   // one bit: the distance between the levels
#pragma unroll
          for (int c = 0; c < C; ++c) {
            float e = __fsub_rn(x[r][c], __fmul_rn(step, qv[c]));
            if (e > lim) e = lim;
            else if (e < -lim) e = -lim;
            e16[c] = f32_to_f16(e);
          }
          *(uint2*)&auxh[(size_t)i * D + col0] =
              make_uint2((uint32_t)e16[0] | ((uint32_t)e16[1] << 16), (uint32_t)e16[2] | ((uint32_t)e16[3] << 16));
        }
      }
      __syncwarp();
#pragma unroll
      for (int r = 0; r < kVbBatch; ++r) {
        const int i = i0 + r;
        const int nw = D * wd_out[i] / 32;               // 32-bit words of the row
        if constexpr (WIDE) {
          for (int k = lane; k < nw; k += 32) ((uint32_t*)(pay_out + of_out[i]))[k] = sm.pk[r][k];
        } else {
          if (lane < nw) ((uint32_t*)(pay_out + of_out[i]))[lane] = sm.pk[r][lane];
        }
      }
      __syncwarp();
    }
  }

  if constexpr (PHASE == 0) {
    // ---- o
    tree.result(o);
    bool bad = false;
#pragma unroll
    for (int c = 0; c < C; ++c) bad |= !isfinite(o[c]);
    if (bad) raise_flag(a.flags, BRS_FLAG_NONFINITE);
    *(float4*)&a.o[(size_t)head * D + col0] = make_float4(o[0], o[1], o[2], o[3]);
    __syncwarp();
    // ---- statistics and costs of the head's rows: mean square of the
    // ranges (FP64, rows in order), EMA of a^2 and of beta (2-beta) k^2,
    // Gamma_hat = 1 / (C expm1(2 (s + r))), c = Gamma_hat * R~^2
    double ms = 0.0;
    for (int i = 0; i < D; ++i) {
      const double Ri = (double)sm.R[i];
      ms += Ri * Ri;
    }
    const double rms = sqrt(ms / (double)D);
    for (int i = lane; i < D; i += 32) {
      const VbRow r = sm.row[i];
      const double av = (double)r.ka.z, be = (double)beta, kd = (double)r.ka.x;
      const double a2 = av * av, kk = (be * (2.0 - be)) * (kd * kd);
      double* st = a.stats + ((size_t)head * D + i) * 2;
      double A, K;
      if (a.first) {
        A = a2;
        K = kk;
      } else {
        A = a.lambda * st[0] + (1.0 - a.lambda) * a2;
        K = a.lambda * st[1] + (1.0 - a.lambda) * kk;
      }
      st[0] = A;
      st[1] = K;
      const double s_hat = -0.5 * log(A);
      double gam;
      if (a.persistence == 0) {                    // erasure rate Gamma_hat
        const double rr = 0.5 * K;
        double arg = 2.0 * (s_hat + rr);
        if (!(arg >= 1e-9)) arg = 1e-9;
        gam = 1.0 / ((double)a.C * expm1(arg));
      } else {                                     // w^(1) = 1/(1 - e^-2s), h^(C) = 1/(1 - e^-2Cs)
        double arg = 2.0 * s_hat * (double)(a.persistence == 2 ? a.C : 1);
        if (!(arg >= 1e-9)) arg = 1e-9;
        gam = 1.0 / -expm1(-arg);
      }
      const double rt = rms > 0.0 ? (double)sm.R[i] / rms : 0.0;
      a.cost[(size_t)b * rows + h * D + i] = gam * (rt * rt);
    }
  }
}

cudaError_t launch_varbit_offsets(const VbArgs& a, cudaStream_t st);

template <int PHASE, bool WIDE, bool ONE>
static cudaError_t launch_phase_w(const VbArgs& a, cudaStream_t st) {
  const dim3 grid((a.B * a.H + kVbWarps - 1) / kVbWarps), block(32 * kVbWarps);
  switch (a.mode) {
    case BRS_ROUND_NEAREST: varbit_kernel<128, PHASE, BRS_ROUND_NEAREST, WIDE, ONE><<<grid, block, 0, st>>>(a); break;
    case BRS_ROUND_STOCHASTIC: varbit_kernel<128, PHASE, BRS_ROUND_STOCHASTIC, WIDE, ONE><<<grid, block, 0, st>>>(a); break;
    case BRS_ROUND_ERRFEEDBACK: varbit_kernel<128, PHASE, BRS_ROUND_ERRFEEDBACK, WIDE, ONE><<<grid, block, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// widths above 8 (b_max up to 16) take the wide packing, b_min = 1 the
// one-bit rows
template <int PHASE>
static cudaError_t launch_phase(const VbArgs& a, cudaStream_t st) {
  if (a.b_min == 1)
    return a.b_max > 8 ? launch_phase_w<PHASE, true, true>(a, st) : launch_phase_w<PHASE, false, true>(a, st);
  return a.b_max > 8 ? launch_phase_w<PHASE, true, false>(a, st) : launch_phase_w<PHASE, false, false>(a, st);
}

cudaError_t launch_varbit_decode(const VbArgs& a, cudaStream_t st) {
  cudaError_t e = launch_phase<0>(a, st);
  if (e != cudaSuccess) return e;
  AllocArgs al{};
  const int rows = a.H * 128;
  al.rows_per_group = a.budget_scope ? rows : 128;
  al.groups = a.B * rows / al.rows_per_group;
  al.b_min = a.b_min;
  al.b_max = a.b_max;
  al.avg_bits = a.avg_bits;
  al.offset_unit = 128 / 8;
  al.cost = a.cost;
  uint8_t* pout = (uint8_t*)a.packed_out;
  al.bits = pout + a.sec.off_width;
  al.offsets = (uint32_t*)(pout + a.sec.off_offsets);
  if (a.budget_scope) {
    e = launch_allocate(al, st);
    if (e != cudaSuccess) return e;
  } else {
    // per-head budgets: offsets must still run over the whole sequence
    al.offsets = nullptr;
    e = launch_allocate(al, st);
    if (e != cudaSuccess) return e;
    e = launch_varbit_offsets(a, st);
    if (e != cudaSuccess) return e;
  }
  return launch_phase<1>(a, st);
}

// row offsets of every sequence from its widths (per-head budgets)
__global__ void varbit_offsets_kernel(const VbArgs a) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= a.B) return;
  const int rows = a.H * 128;
  uint8_t* pout = (uint8_t*)a.packed_out;
  const uint8_t* wd = pout + a.sec.off_width + (size_t)b * rows;
  uint32_t* of = (uint32_t*)(pout + a.sec.off_offsets) + (size_t)b * (rows + 1);
  uint32_t off = 0;
  for (int r = 0; r < rows; ++r) {
    of[r] = off;
    off += 16u * wd[r];
  }
  of[rows] = off;
}

cudaError_t launch_varbit_offsets(const VbArgs& a, cudaStream_t st) {
  varbit_offsets_kernel<<<(a.B + 63) / 64, 64, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace brs
