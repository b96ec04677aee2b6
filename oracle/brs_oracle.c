/*
 * Plain CPU oracle for the fused recurrent-state update with quantized
 * write-back of gated delta-rule layers (KDA: decay per key channel; GDN:
 * decay per head).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It is deliberately
 * slow: one scalar loop per definition, one Philox call per element, no
 * blocking or fusion beyond what the definitions below state.
 *
 * Precision.  The recurrence and the quantizers run in FP32, the precision
 * the DAMP summary names for the fused update ([DAMP] Key Points >
 * Implementation: reconstruct INT8 channels, compute the update in FP32,
 * re-quantize, write back).  The bit allocator runs in FP64.  Build with
 * -ffp-contract=off so that every a*b+c written below is two roundings and
 * every fmaf() is one.
 *
 * Operation order (the pages fix FP32 but not the order of a sum; these
 * orders are this implementation's reading and the CUDA library follows the
 * same written definition):
 *   - every sum over key rows (over one tier's rows in the mixed basis)
 *     is taken in groups of 8 consecutive rows, each an fmaf chain in row
 *     order from +0, whose sums are then added in a pairwise tree (adjacent
 *     pairs first, an unpaired last element passing up): row_sum below;
 *   - every sum over value columns (variable-width fit error) runs
 *     j = 0, 1, ..., d-1 as an fmaf chain starting from +0;
 *   - the Hadamard transform is the unnormalised butterfly, stages
 *     h = 1, 2, 4, ..., n/2, each pair (x, y) -> (x + y, x - y), followed by
 *     one multiplication by the float nearest to 1/sqrt(n).
 *
 * Parity status:
 *   pinned: binary16 conversion (against numpy float16), Philox4x32-10
 *     (published known-answer vectors), Hadamard (explicit Sylvester matrix),
 *     INT8 block quantizer and variable-width quantizer (exhaustive level
 *     search on random blocks), stochastic rounding (mean over seeds),
 *     allocator (worked example, budget, monotonicity, brute force),
 *     erasure rate (worked example, closed form and brute-force Gramian),
 *     recurrence (FP64 dense-matrix recurrence, beta=0/a=1 identity, unit-key
 *     invariant, dead zone and error feedback), storage accounting.
 *   parity unpinned: the order of FP32 operations inside a sum (a reading,
 *     see above) and the rotated-domain and mixed-basis modes, which are
 *     pinned only against the canonical mode (teacher-forced: outputs to
 *     FP32 rounding, codes apart only next to a rounding boundary).
 */
#include "brs_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* binary16 and bfloat16                                                     */
/* ------------------------------------------------------------------------ */

/* IEEE 754 binary16, round to nearest, ties to even, subnormals kept,
 * overflow to infinity.  Written from the format definition: the value is
 * rounded to the quantum of its binade (2^(E-10), with E clamped at -14 for
 * the subnormal range) in FP64, where the division by a power of two and
 * the rounding are exact. */
uint16_t orc_f16_from_f32(float f) {
  uint32_t bits;
  memcpy(&bits, &f, 4);
  uint16_t sign = (uint16_t)((bits >> 16) & 0x8000u);
  if (isnan(f)) return (uint16_t)(sign | 0x7e00u);
  if (isinf(f)) return (uint16_t)(sign | 0x7c00u);
  double a = fabs((double)f);
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e);
  int E = e - 1;                       /* floor(log2 a) */
  if (E < -14) E = -14;
  double quantum = ldexp(1.0, E - 10);
  double n = nearbyint(a / quantum);   /* ties to even */
  double r = n * quantum;
  if (r > 65504.0) return (uint16_t)(sign | 0x7c00u);
  if (r < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)n); /* subnormal */
  frexp(r, &e);
  int E2 = e - 1;
  int M = (int)(r / ldexp(1.0, E2 - 10)); /* in [1024, 2047] */
  return (uint16_t)(sign | (uint16_t)((E2 + 15) << 10) | (uint16_t)(M - 1024));
}

float orc_f32_from_f16(uint16_t h) {
  int E = (h >> 10) & 31, M = h & 1023;
  double v;
  if (E == 0) v = ldexp((double)M, -24);
  else if (E == 31) v = M ? NAN : INFINITY;
  else v = ldexp((double)(1024 + M), E - 25);
  return (float)((h & 0x8000u) ? -v : v);
}

float orc_f32_from_bf16(uint16_t b) {
  uint32_t bits = (uint32_t)b << 16;
  float f;
  memcpy(&f, &bits, 4);
  return f;
}

static int f16_is_inf_or_nan(uint16_t h) { return ((h >> 10) & 31) == 31; }

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as   */
/* easy as 1, 2, 3", SC'11): ten rounds of two 32x32->64 multiplications     */
/* with the round keys bumped by the Weyl constants between rounds.          */
/* ------------------------------------------------------------------------ */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    uint64_t p0 = (uint64_t)0xD2511F53u * c0;
    uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c1 ^ k0;
    uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

/* 24 uniform bits for element `elem` of head (b, h) at write-back step
 * `step`: counter (elem/4, step, h, b), key (seed low, seed high), word
 * elem % 4, top 24 bits. */
static uint32_t sr_bits24(uint64_t seed, int64_t step, int h, int b, int elem) {
  uint32_t ctr[4] = {(uint32_t)(elem / 4), (uint32_t)step, (uint32_t)h, (uint32_t)b};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t out[4];
  orc_philox4x32_10(ctr, key, out);
  return out[elem % 4] >> 8;
}

/* ------------------------------------------------------------------------ */
/* Hadamard along the value axis ([DAMP] Data & Methods > Quantization &     */
/* calibration details: a Hadamard transform along the value dimension      */
/* within each key channel before INT8 quantization).  Sylvester matrix in   */
/* natural order, normalised to be orthonormal; it is its own inverse.       */
/* ------------------------------------------------------------------------ */
float orc_hadamard_scale(int n) { return (float)(1.0 / sqrt((double)n)); }

void orc_fwht(float* x, int n) {
  for (int h = 1; h < n; h *= 2)
    for (int i = 0; i < n; i += 2 * h)
      for (int j = i; j < i + h; ++j) {
        float a = x[j], b = x[j + h];
        x[j] = a + b;
        x[j + h] = a - b;
      }
  float s = orc_hadamard_scale(n);
  for (int j = 0; j < n; ++j) x[j] = x[j] * s;
}

/* ------------------------------------------------------------------------ */
/* Write-back rounding rules ([WB] Quantized GRU formulation and the         */
/* Chinese summary's sections on error feedback and stochastic rounding):    */
/*   nearest      q = Q(h): nearest level, half-steps to the even index,     */
/*                clipped at the grid rails;                                  */
/*   stochastic   one of the two adjacent levels, chosen with probability    */
/*                set by the position between them (unbiased);               */
/*   error feedb. q = Q(h + e_prev), e = h + e_prev - q clipped to +-Delta.  */
/* ------------------------------------------------------------------------ */
static float sr_round(float t, uint32_t r24) {
  float fl = floorf(t);
  float fr = t - fl;
  return ((float)r24 < fr * 16777216.0f) ? fl + 1.0f : fl;
}

/* Asymmetric affine block ([DAMP] Quantization & calibration details:
 * per-block asymmetric affine quantization with b = 8 or 4; the stored
 * scale and zero are FP16), L = 2^b - 1 levels above zero:
 * scale = fp16((max - min) / L), zero = fp16(min),
 * code = clamp(round((y - zero) * (1 / scale)), 0, L),
 * value = fmaf(code, scale, zero). */
int orc_lowbit_block(const float* y, int n, int levels, int mode, uint64_t seed, int64_t step, int h,
                     int b, int elem0, uint16_t* e_inout, uint8_t* codes, uint16_t* scale_h,
                     uint16_t* zero_h, float* t_out) {
  int flags = 0;
  if (n <= 0) return ORC_EINVAL;
  float* tgt = (float*)malloc(sizeof(float) * (size_t)n);
  for (int j = 0; j < n; ++j) {
    tgt[j] = y[j];
    if (mode == ORC_ROUND_ERRFEEDBACK) tgt[j] = y[j] + orc_f32_from_f16(e_inout[j]);
    if (!isfinite(tgt[j])) flags |= ORC_ENONFINITE;
  }
  /* block minimum and maximum, -0 ordered below +0 */
  float mn = tgt[0], mx = tgt[0];
  for (int j = 1; j < n; ++j) {
    if (tgt[j] < mn || (tgt[j] == mn && signbit(tgt[j]))) mn = tgt[j];
    if (tgt[j] > mx || (tgt[j] == mx && !signbit(tgt[j]))) mx = tgt[j];
  }
  uint16_t sh = orc_f16_from_f32((mx - mn) / (float)levels);
  uint16_t zh = orc_f16_from_f32(mn);
  if (f16_is_inf_or_nan(sh) || f16_is_inf_or_nan(zh)) flags |= ORC_EOVERFLOW;
  float s = orc_f32_from_f16(sh), z = orc_f32_from_f16(zh);
  float rcp = (s == 0.0f) ? 0.0f : 1.0f / s;
  for (int j = 0; j < n; ++j) {
    float t = 0.0f, c = 0.0f;
    if (s != 0.0f) {
      t = (tgt[j] - z) * rcp;
      if (mode == ORC_ROUND_STOCHASTIC)
        c = sr_round(t, sr_bits24(seed, step, h, b, elem0 + j));
      else
        c = nearbyintf(t);
      if (c < 0.0f) c = 0.0f;
      if (c > (float)levels) c = (float)levels;
      if (!(c == c)) c = 0.0f;
    }
    codes[j] = (uint8_t)(int)c;
    if (t_out) t_out[j] = t;
    if (mode == ORC_ROUND_ERRFEEDBACK) {
      float xhat = fmaf(c, s, z);
      float e = tgt[j] - xhat;
      if (e > s) e = s;
      else if (e < -s) e = -s;
      e_inout[j] = orc_f16_from_f32(e);
    }
  }
  *scale_h = sh;
  *zero_h = zh;
  free(tgt);
  return flags;
}

/* The INT8 block (b = 8, L = 255). */
int orc_int8_block(const float* y, int n, int mode, uint64_t seed, int64_t step, int h, int b,
                   int elem0, uint16_t* e_inout, uint8_t* codes, uint16_t* scale_h,
                   uint16_t* zero_h, float* t_out) {
  return orc_lowbit_block(y, n, 255, mode, seed, step, h, b, elem0, e_inout, codes, scale_h, zero_h, t_out);
}

/* Direction memory on the INT8 block ([WB] Post-training write-back
 * interventions and diagnostics: signed sub-threshold votes, a trigger that
 * moves the stored state by one level and resets the counter, transitions
 * clipped at the grid rails; Trajectory analysis: the voting region
 * Delta/8 < |delta| < Delta/2; the Chinese summary's core method: a k-bit sign
 * counter with threshold T_k = 2^(k-1)).  Counter of k = 2 bits: m in
 * {-1, 0, 1}, T = 2.  The grid and the codes are those of nearest write-back
 * of y; then per element the proposed change delta = y - xprev (xprev: the
 * stored value the step started from, in the stored basis) votes sign(delta)
 * when Delta/8 < |delta| < Delta/2 (Delta: the block's new step); a counter
 * that reaches +-2 moves the code one level that way (clipped to [0, 255])
 * and returns to 0. */
static int lowbit_block_dm(const float* y, const float* xprev, int n, int levels, int8_t* m_inout,
                           uint8_t* codes, uint16_t* scale_h, uint16_t* zero_h, float* t_out) {
  int flags = orc_lowbit_block(y, n, levels, ORC_ROUND_NEAREST, 0, 0, 0, 0, 0, NULL, codes, scale_h, zero_h,
                               t_out);
  float s = orc_f32_from_f16(*scale_h);
  float lo = s * 0.125f, hi = s * 0.5f;
  for (int j = 0; j < n; ++j) {
    float dl = y[j] - xprev[j];
    float ad = fabsf(dl);
    int m = m_inout[j];
    if (ad > lo && ad < hi) m += (dl > 0.0f) ? 1 : -1;
    if (m >= 2 || m <= -2) {
      int c = (int)codes[j] + (m > 0 ? 1 : -1);
      if (c < 0) c = 0;
      if (c > levels) c = levels;
      codes[j] = (uint8_t)c;
      m = 0;
    }
    m_inout[j] = (int8_t)m;
  }
  return flags;
}

int orc_int8_block_dm(const float* y, const float* xprev, int n, int8_t* m_inout, uint8_t* codes,
                      uint16_t* scale_h, uint16_t* zero_h, float* t_out) {
  return lowbit_block_dm(y, xprev, n, 255, m_inout, codes, scale_h, zero_h, t_out);
}

/* k-bit residual memory ([WB] Post-training write-back interventions and
 * diagnostics: error feedback's auxiliary residual carries the quantization
 * error forward, with evaluated widths k = 2, 3, 4; Matched recurrent-memory
 * training campaign: a 4-bit visible state plus two auxiliary bits; the
 * Chinese summary's core method lists k-bit quantized residual memory beside
 * error feedback).  Reading: error feedback whose residual is kept in k bits,
 * as the signed integer m of step/2^k nearest to it, symmetric range
 * |m| <= 2^(k-1) - 1.  The target is y + m_prev * (sprev / 2^k), sprev being
 * the block's step when m_prev was stored; the grid and codes are those of
 * nearest rounding of the target; then m = clamp(rne(r * (1/scale) * 2^k))
 * with r = target - value. */
static int lowbit_block_rm(const float* y, int n, int levels, int kbits, float sprev, int8_t* m_inout,
                           uint8_t* codes, uint16_t* scale_h, uint16_t* zero_h, float* t_out) {
  if (kbits < 2 || kbits > 4 || n <= 0) return ORC_EINVAL;
  const float unit = ldexpf(1.0f, kbits);                 /* 2^k */
  const float sunit = sprev / unit;                       /* exact: a power-of-two scaling of an FP16 value */
  const int mmax = (1 << (kbits - 1)) - 1;
  float* tgt = (float*)calloc((size_t)n, sizeof(float));
  for (int j = 0; j < n; ++j) tgt[j] = y[j] + (float)m_inout[j] * sunit;
  int flags = orc_lowbit_block(tgt, n, levels, ORC_ROUND_NEAREST, 0, 0, 0, 0, 0, NULL, codes, scale_h, zero_h,
                               t_out);
  float s = orc_f32_from_f16(*scale_h), z = orc_f32_from_f16(*zero_h);
  float rcp = (s == 0.0f) ? 0.0f : 1.0f / s;
  for (int j = 0; j < n; ++j) {
    float r = tgt[j] - fmaf((float)codes[j], s, z);
    float q = nearbyintf((r * rcp) * unit);
    int m = (q != q) ? 0 : (q > (float)mmax ? mmax : (q < (float)-mmax ? -mmax : (int)q));
    m_inout[j] = (int8_t)m;
  }
  free(tgt);
  return flags;
}

int orc_int8_block_rm(const float* y, int n, int kbits, float sprev, int8_t* m_inout, uint8_t* codes,
                      uint16_t* scale_h, uint16_t* zero_h, float* t_out) {
  return lowbit_block_rm(y, n, 255, kbits, sprev, m_inout, codes, scale_h, zero_h, t_out);
}

/* Variable-width symmetric row ([LB] Levels and storage): levels
 * {-n..n}*Delta, n = 2^(b-1) - 1, Delta = f*R/n with R the row's absolute
 * maximum and f fitted over 16 values in [1/4, 1] (read as f_m = (5+m)/20)
 * by squared error, the chosen Delta stored as an FP16 scale.  The fit
 * error of every candidate is evaluated with nearest rounding on the target
 * (x, or x + e_prev under error feedback); ties keep the smaller f. */
int orc_varbit_row(const float* x, int n, int bw, int mode, uint64_t seed, int64_t step, int h,
                   int b, int elem0, uint16_t* e_inout, int32_t* q_out, uint16_t* delta_h,
                   int* m_star, float* t_out) {
  return orc_varbit_group(x, n, bw, mode, seed, step, h, b, elem0, 1, e_inout, q_out, delta_h,
                          m_star, t_out);
}

/* The same quantizer on any scale group: a row of a row unit, or one block
 * of 32 key channels of one column of a head unit ([LB] Allocation units:
 * scales per block of 32 key channels).  Only the stochastic-rounding
 * element index depends on where the group sits in the head. */
int orc_varbit_group(const float* x, int n, int bw, int mode, uint64_t seed, int64_t step, int h,
                     int b, int elem0, int estride, uint16_t* e_inout, int32_t* q_out,
                     uint16_t* delta_h, int* m_star, float* t_out) {
  int flags = 0;
  int nl = (1 << (bw - 1)) - 1;
  float fnl = (float)nl;
  float* tgt = (float*)malloc(sizeof(float) * (size_t)n);
  float R = 0.0f;
  for (int j = 0; j < n; ++j) {
    tgt[j] = x[j];
    if (mode == ORC_ROUND_ERRFEEDBACK) tgt[j] = x[j] + orc_f32_from_f16(e_inout[j]);
    if (!isfinite(tgt[j])) flags |= ORC_ENONFINITE;
    float a = fabsf(tgt[j]);
    if (a > R) R = a;
  }
  if (bw == 1) {
    /* One bit ([LB] Levels and storage): the sign times the row's mean
     * absolute value, that mean stored as the FP16 scale.  Mean: the
     * absolute values summed in element order in FP32, times 1/n (n a power
     * of two, so exact).  Code 1 holds +mu, code 0 holds -mu.  Nearest: 1
     * for a target >= 0 (a zero target is a tie between the two levels and
     * takes +mu).  Stochastic: +mu with probability (t/mu + 1)/2, clipped to
     * [0, 1].  Error feedback: residual clipped to +-2 mu, the distance
     * between the two levels. */
    float sum = 0.0f;
    for (int j = 0; j < n; ++j) sum = sum + fabsf(tgt[j]);
    uint16_t mh = orc_f16_from_f32(sum * (1.0f / (float)n));
    float mu = orc_f32_from_f16(mh);
    int okm = isfinite(mu);
    if (!okm) flags |= ORC_EOVERFLOW;
    float inv1 = (okm && mu != 0.0f) ? 1.0f / mu : 0.0f;
    for (int j = 0; j < n; ++j) {
      float t = tgt[j] * inv1;
      int u;
      if (mode == ORC_ROUND_STOCHASTIC) {
        float c = sr_round((t + 1.0f) * 0.5f, sr_bits24(seed, step, h, b, elem0 + j * estride));
        if (c < 0.0f) c = 0.0f;
        if (c > 1.0f) c = 1.0f;
        if (!(c == c)) c = 0.0f;
        u = (int)c;
      } else {
        u = tgt[j] >= 0.0f ? 1 : 0;
      }
      q_out[j] = u;
      if (t_out) t_out[j] = t;
      if (mode == ORC_ROUND_ERRFEEDBACK) {
        float xhat = okm ? (u ? mu : -mu) : 0.0f;
        float e = tgt[j] - xhat;
        float lim = okm ? 2.0f * mu : 0.0f;
        if (e > lim) e = lim;
        else if (e < -lim) e = -lim;
        e_inout[j] = orc_f16_from_f32(e);
      }
    }
    *delta_h = mh;
    if (m_star) *m_star = 0;
    free(tgt);
    return flags;
  }
  uint16_t dh = 0;
  int best = -1;
  if (R > 0.0f) {
    float bestE = 0.0f;
    for (int m = 0; m < 16; ++m) {
      float f = (float)(5 + m) / 20.0f;
      uint16_t ch = orc_f16_from_f32((f * R) / fnl);
      float dm = orc_f32_from_f16(ch);
      if (!isfinite(dm)) continue;
      float E = 0.0f;
      if (dm == 0.0f) {
        for (int j = 0; j < n; ++j) E = fmaf(tgt[j], tgt[j], E);
      } else {
        float inv = 1.0f / dm;
        for (int j = 0; j < n; ++j) {
          float qf = nearbyintf(tgt[j] * inv);
          if (qf < -fnl) qf = -fnl;
          if (qf > fnl) qf = fnl;
          float r = tgt[j] - dm * qf;
          E = fmaf(r, r, E);
        }
      }
      if (best < 0 || E < bestE) {
        best = m;
        bestE = E;
        dh = ch;
      }
    }
    if (best < 0) {
      flags |= ORC_EOVERFLOW;
      dh = 0x7c00u;
      best = 15;
    }
  } else {
    best = 0;
  }
  float D = orc_f32_from_f16(dh);
  int ok = (D != 0.0f) && isfinite(D);
  float inv = ok ? 1.0f / D : 0.0f;
  for (int j = 0; j < n; ++j) {
    float t = 0.0f, qf = 0.0f;
    if (ok) {
      t = tgt[j] * inv;
      if (mode == ORC_ROUND_STOCHASTIC)
        qf = sr_round(t, sr_bits24(seed, step, h, b, elem0 + j * estride));
      else
        qf = nearbyintf(t);
      if (qf < -fnl) qf = -fnl;
      if (qf > fnl) qf = fnl;
      if (!(qf == qf)) qf = 0.0f;
    }
    q_out[j] = (int32_t)qf;
    if (t_out) t_out[j] = t;
    if (mode == ORC_ROUND_ERRFEEDBACK) {
      float xhat = D * qf;
      if (!ok) xhat = 0.0f;
      float e = tgt[j] - xhat;
      float lim = ok ? D : 0.0f;
      if (e > lim) e = lim;
      else if (e < -lim) e = -lim;
      e_inout[j] = orc_f16_from_f32(e);
    }
  }
  *delta_h = dh;
  if (m_star) *m_star = best;
  free(tgt);
  return flags;
}

/* ------------------------------------------------------------------------ */
/* Decay-aware allocation ([LB] Approximate erasure rate, Range              */
/* normalization, State bit allocation; [LBX] worked example).               */
/* ------------------------------------------------------------------------ */

/* Gamma_hat = rho / [C * expm1(2 (s + r))], rho = 1, with s = -ln(A)/2 the
 * decay rate estimated from A = EMA(a^2) and r = K/2 from
 * K = EMA(beta (2 - beta) k^2).  The argument is floored at 1e-9. */
double orc_gamma_hat(double A, double K, int C) {
  double s = -0.5 * log(A);
  double r = 0.5 * K;
  double arg = 2.0 * (s + r);
  if (!(arg >= 1e-9)) arg = 1e-9;
  return 1.0 / ((double)C * expm1(arg));
}

/* The row weight of the allocation cost c = weight * R~^2 ([LB] Choice of
 * persistence factor): 0 the erasure rate Gamma_hat above; 1 DAMP's
 * uncapped persistence w^(1) = 1 / (1 - e^(-2 s)); 2 the write-back-time
 * factor h^(C) = 1 / (1 - e^(-2 C s)); s = -ln(A)/2, the exponent's
 * argument floored at 1e-9 as for Gamma_hat. */
double orc_persistence(int kind, double A, double K, int C) {
  if (kind == 0) return orc_gamma_hat(A, K, C);
  double s = -0.5 * log(A);
  double arg = 2.0 * s * (double)(kind == 2 ? C : 1);
  if (!(arg >= 1e-9)) arg = 1e-9;
  return 1.0 / -expm1(-arg);
}

/* b*_i = avg + log2(c_i / GM(c)) / 2 (the minimiser of sum c_i 2^(-2 b_i)
 * at a fixed mean), GM over the rows with c_i > 0; rounded to nearest
 * (ties to even), clipped to [b_min, b_max]; rows with c_i = 0 take b_min
 * (all rows take round(avg) when every c_i is 0).  The sum is then brought
 * to avg*N one bit at a time: while over budget, take a bit from the row
 * whose cost rises least (3 c_i 4^(-b_i)); while under, give one to the
 * row whose cost falls most (3/4 c_i 4^(-b_i)); ties to the lower row. */
int orc_allocate_bits(int N, const double* c, double avg_bits, int b_min, int b_max,
                      uint8_t* bits) {
  double tgt = avg_bits * (double)N;
  long target = (long)tgt;
  if ((double)target != tgt || target < (long)N * b_min || target > (long)N * b_max ||
      b_min < 1 || b_max > 16 || b_min > b_max)
    return ORC_EINVAL;
  int* b = (int*)malloc(sizeof(int) * (size_t)N);
  int cnt = 0;
  double sumlog = 0.0;
  for (int i = 0; i < N; ++i)
    if (c[i] > 0.0) {
      sumlog += log(c[i]);
      ++cnt;
    }
  if (cnt == 0) {
    for (int i = 0; i < N; ++i) b[i] = (int)nearbyint(avg_bits);
  } else {
    double gm = exp(sumlog / (double)cnt);
    for (int i = 0; i < N; ++i) {
      if (c[i] > 0.0) {
        double bs = avg_bits + 0.5 * log2(c[i] / gm);
        double br = nearbyint(bs);
        if (br < (double)b_min) br = (double)b_min;
        if (br > (double)b_max) br = (double)b_max;
        b[i] = (int)br;
      } else {
        b[i] = b_min;
      }
    }
  }
  for (int i = 0; i < N; ++i) {
    if (b[i] < b_min) b[i] = b_min;
    if (b[i] > b_max) b[i] = b_max;
  }
  long sum = 0;
  for (int i = 0; i < N; ++i) sum += b[i];
  while (sum > target) {
    int pick = -1;
    double pv = 0.0;
    for (int i = 0; i < N; ++i)
      if (b[i] > b_min) {
        double m = (3.0 * c[i]) * ldexp(1.0, -2 * b[i]);
        if (pick < 0 || m < pv) {
          pick = i;
          pv = m;
        }
      }
    b[pick] -= 1;
    sum -= 1;
  }
  while (sum < target) {
    int pick = -1;
    double pv = 0.0;
    for (int i = 0; i < N; ++i)
      if (b[i] < b_max) {
        double m = (0.75 * c[i]) * ldexp(1.0, -2 * b[i]);
        if (pick < 0 || m > pv) {
          pick = i;
          pv = m;
        }
      }
    b[pick] += 1;
    sum += 1;
  }
  for (int i = 0; i < N; ++i) bits[i] = (uint8_t)b[i];
  free(b);
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Storage layout (the byte format the CUDA library documents in its        */
/* header; restated here independently).                                    */
/*   FP32:   float [B][H][d][d], rows in stored (permuted) order.            */
/*   DAMP:   per head, contiguous, in stored row order: INT8 codes          */
/*           [d-k_hi][d] (rows 0..d-k_hi-1), FP16 rows [k_hi][d] (the        */
/*           protected rows d-k_hi..d-1), then per INT8 row and block an     */
/*           FP16 (scale, zero) pair.  Residuals: FP16 [B][H][d-k_hi][d].   */
/*   VARBIT: [payload B x P bytes][FP16 scale B*H*d][u8 width B*H*d]         */
/*           [u32 row offset B*(H*d+1)], each section starting on a 256-byte */
/*           boundary; P = (d/8) * avg_bits * H * d; row i of sequence b     */
/*           starts at byte offset[i] = (d/8) * sum of the widths before it. */
/*           Residuals FP16 [B][H][d][d]; statistics FP64 [B][H][d][2].      */
/* ------------------------------------------------------------------------ */
static size_t round256(size_t x) { return (x + 255) / 256 * 256; }

/* width of the DAMP low tier and its top code */
static int low_bits(const orc_layout* L) { return L->low_bits == 4 ? 4 : 8; }
static int low_levels(const orc_layout* L) { return (1 << low_bits(L)) - 1; }
/* code e of a low-tier code array (bytes, or two codes to a byte with code e
 * in bits 4 (e % 2) for the 4-bit tier) */
static int code_get(const uint8_t* c, size_t e, int bits) {
  return bits == 8 ? c[e] : (c[e >> 1] >> (4 * (e & 1))) & 15;
}
static void code_put(uint8_t* c, size_t e, int bits, int v) {
  if (bits == 8) {
    c[e] = (uint8_t)v;
  } else {
    int sh = 4 * (int)(e & 1);
    c[e >> 1] = (uint8_t)((c[e >> 1] & ~(15 << sh)) | ((v & 15) << sh));
  }
}

/* head layout: low-tier codes [d - k_hi][d * b / 8], FP16 rows [k_hi][d],
 * (scale, zero) FP16 pairs [d - k_hi][d / block] */
static size_t damp_code_bytes(const orc_layout* L) {
  return (size_t)(L->d - L->k_hi) * (size_t)L->d * (size_t)low_bits(L) / 8;
}
static size_t damp_head_bytes(const orc_layout* L) {
  size_t d = (size_t)L->d, kh = (size_t)L->k_hi;
  return kh * d * 2 + damp_code_bytes(L) + (d - kh) * (d / (size_t)L->block) * 4;
}

typedef struct {
  size_t payload_per_seq, off_scale, off_width, off_offsets, total;
} vb_sections;

/* Row units: one FP16 step, width and offset per row.  Head units ([LB]
 * Allocation units, per-head decay): one width and offset per head, one
 * FP16 step per (block of 32 key channels, column). */
static vb_sections varbit_sections(const orc_layout* L) {
  vb_sections s;
  size_t rows = (size_t)L->H * (size_t)L->d, B = (size_t)L->B;
  s.payload_per_seq = (size_t)((double)(L->d / 8) * L->avg_bits * (double)rows);
  s.off_scale = round256(s.payload_per_seq * B);
  if (L->storage == ORC_STORE_VARBIT_HEAD) {
    size_t H = (size_t)L->H, d = (size_t)L->d;
    s.off_width = s.off_scale + round256(B * H * (d / 32) * d * 2);
    s.off_offsets = s.off_width + round256(B * H);
    s.total = s.off_offsets + round256(B * (H + 1) * 4);
    return s;
  }
  s.off_width = s.off_scale + round256(rows * B * 2);
  s.off_offsets = s.off_width + round256(rows * B);
  s.total = s.off_offsets + round256((rows + 1) * B * 4);
  return s;
}

size_t orc_state_bytes(const orc_layout* L, size_t* aux_bytes, size_t* stats_bytes) {
  size_t heads = (size_t)L->B * (size_t)L->H, d = (size_t)L->d;
  size_t total = 0, aux = 0, stats = 0;
  if (L->storage == ORC_STORE_FP32) {
    total = heads * d * d * 4;
  } else if (L->storage == ORC_STORE_DAMP) {
    total = heads * damp_head_bytes(L);
    aux = heads * (d - (size_t)L->k_hi) * d * 2;
  } else {
    total = varbit_sections(L).total;
    aux = heads * d * d * 2;
    stats = heads * d * 2 * sizeof(double);
  }
  if (aux_bytes) *aux_bytes = aux;
  if (stats_bytes) *stats_bytes = stats;
  return total;
}

/* Bits per stored value counted the way the pages count them: DAMP = FP16
 * rows + INT8 rows + 32 bits of (scale, zero) per block ([LB] Related work;
 * [DAMP] main operating point); VARBIT = mean width + one FP16 scale and one
 * 3-bit width per row ([LB] Levels and storage). */
double orc_bits_per_value(const orc_layout* L) {
  double d = (double)L->d, kh = (double)L->k_hi;
  if (L->storage == ORC_STORE_FP32) return 32.0;
  if (L->storage == ORC_STORE_DAMP)
    return (kh * d * 16.0 + (d - kh) * d * (double)low_bits(L) + (d - kh) * (d / L->block) * 32.0) / (d * d);
  if (L->storage == ORC_STORE_VARBIT_HEAD)   /* 16-bit step per 32 values; one width per head */
    return L->avg_bits + 16.0 / 32.0 + (L->b_max > 8 ? 4.0 : 3.0) / (d * d);
  return L->avg_bits + (16.0 + 3.0) / d;
}

/* ------------------------------------------------------------------------ */
/* Per-head state in the working domain                                      */
/* ------------------------------------------------------------------------ */
static int rotated(const orc_layout* L) {
  return L->domain == ORC_DOMAIN_ROTATED && L->storage == ORC_STORE_DAMP && L->hadamard;
}

/* Mixed basis: each tier of a DAMP head is updated in the basis it is
 * stored in (INT8 rows in the Hadamard basis when the Hadamard is on, FP16
 * rows in the value basis); only the k- and q-weighted row sums and w move
 * between the bases. */
static int mixed(const orc_layout* L) {
  return L->domain == ORC_DOMAIN_MIXED && L->storage == ORC_STORE_DAMP;
}

/* Dequantize one DAMP head into S (d x d, stored row order: the d - k_hi
 * INT8 rows first, then the k_hi protected FP16 rows).  In the canonical
 * domain INT8 rows are returned to the value basis with the Hadamard (its
 * own inverse); in the rotated domain the FP16 rows are taken to the
 * Hadamard basis instead. */
static void damp_load(const orc_layout* L, const uint8_t* head, float* S) {
  int d = L->d, nlo = d - L->k_hi, nb = d / L->block, bits = low_bits(L);
  const uint8_t* codes = head;
  const uint16_t* f16rows = (const uint16_t*)(head + damp_code_bytes(L));
  const uint16_t* sz = (const uint16_t*)(head + damp_code_bytes(L) + (size_t)L->k_hi * d * 2);
  for (int i = 0; i < d; ++i) {
    float* row = S + (size_t)i * d;
    if (i >= nlo) {
      for (int j = 0; j < d; ++j) row[j] = orc_f32_from_f16(f16rows[(size_t)(i - nlo) * d + j]);
      if (rotated(L)) orc_fwht(row, d);
    } else {
      for (int j = 0; j < d; ++j) {
        int bl = j / L->block;
        float s = orc_f32_from_f16(sz[((size_t)i * nb + bl) * 2 + 0]);
        float z = orc_f32_from_f16(sz[((size_t)i * nb + bl) * 2 + 1]);
        row[j] = fmaf((float)code_get(codes, (size_t)i * d + j, bits), s, z);
      }
      if (L->hadamard && !rotated(L) && !mixed(L)) orc_fwht(row, d);
    }
  }
}

/* 2-bit two's-complement direction counters, four to a byte in column
 * order (element e of a head at bits 2(e mod 4) of byte e/4) */
static int dm_get(const uint8_t* dm, size_t e) {
  int f = (dm[e >> 2] >> (2 * (e & 3))) & 3;
  return (f & 2) ? f - 4 : f;
}
static void dm_put(uint8_t* dm, size_t e, int m) {
  int sh = 2 * (int)(e & 3);
  dm[e >> 2] = (uint8_t)((dm[e >> 2] & ~(3 << sh)) | ((m & 3) << sh));
}

/* k-bit residual-memory integers, two to a byte in column order (element e
 * of a head in bits 4(e mod 2) .. +3 of byte e/2, two's complement) */
static int rm_get(const uint8_t* rm, size_t e) {
  int f = (rm[e >> 1] >> (4 * (e & 1))) & 15;
  return (f & 8) ? f - 16 : f;
}
static void rm_put(uint8_t* rm, size_t e, int m) {
  int sh = 4 * (int)(e & 1);
  rm[e >> 1] = (uint8_t)((rm[e >> 1] & ~(15 << sh)) | ((m & 15) << sh));
}

/* prev: the stored head this write-back replaces (read block by block just
 * before it is overwritten, so it may be the same memory as head); used by
 * direction memory only, whose counters sit in aux_head as bytes. */
static int damp_store(const orc_layout* L, const orc_writeback* wb, int64_t step, int b, int h,
                      const float* S, const uint8_t* prev, uint8_t* head, uint16_t* aux_head,
                      float* t_head) {
  int d = L->d, nlo = d - L->k_hi, nb = d / L->block, flags = 0;
  int bits = low_bits(L), levels = low_levels(L);
  uint8_t* codes = head;
  uint16_t* f16rows = (uint16_t*)(head + damp_code_bytes(L));
  uint16_t* sz = (uint16_t*)(head + damp_code_bytes(L) + (size_t)L->k_hi * d * 2);
  const uint16_t* psz = (const uint16_t*)(prev + damp_code_bytes(L) + (size_t)L->k_hi * d * 2);
  float* xp = (float*)malloc(sizeof(float) * (size_t)L->block);
  int8_t* mm = (int8_t*)malloc((size_t)L->block);
  uint8_t* cb = (uint8_t*)malloc((size_t)L->block);           /* one block's codes, one per byte */
  float* tmp = (float*)malloc(sizeof(float) * (size_t)d);
  for (int i = 0; i < d; ++i) {
    memcpy(tmp, S + (size_t)i * d, sizeof(float) * (size_t)d);
    if (i >= nlo) {
      if (rotated(L)) orc_fwht(tmp, d);
      for (int j = 0; j < d; ++j) {
        if (!isfinite(tmp[j])) flags |= ORC_ENONFINITE;
        uint16_t hv = orc_f16_from_f32(tmp[j]);
        if (f16_is_inf_or_nan(hv) && isfinite(tmp[j])) flags |= ORC_EOVERFLOW;
        f16rows[(size_t)(i - nlo) * d + j] = hv;
        if (t_head) t_head[(size_t)i * d + j] = 0.0f;
      }
    } else {
      if (L->hadamard && !rotated(L) && !mixed(L)) orc_fwht(tmp, d);
      for (int bl = 0; bl < nb; ++bl) {
        int j0 = bl * L->block;
        uint16_t* sh = &sz[((size_t)i * nb + bl) * 2 + 0];
        uint16_t* zh = &sz[((size_t)i * nb + bl) * 2 + 1];
        float* tb = t_head ? t_head + (size_t)i * d + j0 : NULL;
        if (wb->mode >= ORC_ROUND_RESIDUAL2 && wb->mode <= ORC_ROUND_RESIDUAL4) {
          uint8_t* rmh = (uint8_t*)aux_head;
          float ps = orc_f32_from_f16(psz[((size_t)i * nb + bl) * 2 + 0]);
          for (int j = 0; j < L->block; ++j) mm[j] = (int8_t)rm_get(rmh, (size_t)i * d + j0 + j);
          flags |= lowbit_block_rm(tmp + j0, L->block, levels, wb->mode - 2, ps, mm, cb, sh, zh, tb);
          for (int j = 0; j < L->block; ++j) rm_put(rmh, (size_t)i * d + j0 + j, mm[j]);
        } else if (wb->mode == ORC_ROUND_DIRECTION) {
          uint8_t* dmh = (uint8_t*)aux_head;
          float ps = orc_f32_from_f16(psz[((size_t)i * nb + bl) * 2 + 0]);
          float pz = orc_f32_from_f16(psz[((size_t)i * nb + bl) * 2 + 1]);
          for (int j = 0; j < L->block; ++j) {
            xp[j] = fmaf((float)code_get(prev, (size_t)i * d + j0 + j, bits), ps, pz);
            mm[j] = (int8_t)dm_get(dmh, (size_t)i * d + j0 + j);
          }
          flags |= lowbit_block_dm(tmp + j0, xp, L->block, levels, mm, cb, sh, zh, tb);
          for (int j = 0; j < L->block; ++j) dm_put(dmh, (size_t)i * d + j0 + j, mm[j]);
        } else {
          uint16_t* e = aux_head ? aux_head + (size_t)i * d + j0 : NULL;
          flags |= orc_lowbit_block(tmp + j0, L->block, levels, wb->mode, wb->seed, step, h, b, i * d + j0, e,
                                    cb, sh, zh, tb);
        }
        for (int j = 0; j < L->block; ++j) code_put(codes, (size_t)i * d + j0 + j, bits, cb[j]);
      }
    }
  }
  free(tmp);
  free(xp);
  free(mm);
  free(cb);
  return flags;
}

/* One write-back of given FP32 states (the quantizer of the recurrence on
 * its own, so that a state computed elsewhere can be replayed through it):
 * units [u0, u1) of S [B][H][d][d] (stored row order, in the working basis of
 * the layout's domain) are quantized with the rounding of wb at token
 * `step` into packed (DAMP storage), with residuals or direction counters in
 * aux as orc_run keeps them.  For direction memory packed holds, on entry,
 * the stored state the write-back replaces.  Returns ORC_* flags. */
int orc_damp_writeback(const orc_layout* L, const orc_writeback* wb, int64_t step, int u0, int u1,
                       const float* S, void* packed, void* aux) {
  if (L->storage != ORC_STORE_DAMP || u0 < 0 || u1 > L->B * L->H || u0 > u1) return ORC_EINVAL;
  int d = L->d, flags = 0;
  size_t hb = damp_head_bytes(L), nel = (size_t)(d - L->k_hi) * d;
  for (int u = u0; u < u1; ++u) {
    uint8_t* head = (uint8_t*)packed + (size_t)u * hb;
    uint16_t* aux_head = NULL;
    if (aux) {
      if (wb->mode == ORC_ROUND_DIRECTION) aux_head = (uint16_t*)((uint8_t*)aux + (size_t)u * (nel / 4));
      else if (wb->mode >= ORC_ROUND_RESIDUAL2) aux_head = (uint16_t*)((uint8_t*)aux + (size_t)u * (nel / 2));
      else aux_head = (uint16_t*)aux + (size_t)u * nel;
    }
    flags |= damp_store(L, wb, step, u / L->H, u % L->H, S + (size_t)u * d * d, head, head, aux_head, NULL);
  }
  return flags;
}

/* ------------------------------------------------------------------------ */
/* One token of the gated delta rule on one head, in FP32 ([DAMP] Error      */
/* propagation model: S = Q(A_t S + beta_t k_t v_t^T) with A_t the decayed   */
/* delta-rule map; [LB] Accumulated readout error: outputs are read before   */
/* the write-back quantizes the state):                                     */
/*   S <- Diag(a) S;  u = S^T k;  w = beta (v - u);  S <- S + k w^T;         */
/*   o = S^T q.                                                              */
/* kk, qq, aa are gathered in stored row order; vv and the returned oo are  */
/* in the basis of S's columns.                                             */
/* ------------------------------------------------------------------------ */
/* Sum over the key rows i0 .. i1-1 of c_i S_ij (column j), in the order of
 * the arithmetic contract: each group of 8 consecutive rows (the last one
 * may be shorter) is an fmaf chain in row order from +0; the group sums are
 * then added in a pairwise tree, adjacent pairs first (g0 + g1, g2 + g3,
 * ...), an unpaired last element passing up unchanged, level after level
 * until one value remains.  No rows: +0. */
static float row_sum(const float* c, const float* S, int d, int j, int i0, int i1) {
  float part[64];
  int n = 0;
  for (int g = i0; g < i1; g += 8) {
    float acc = 0.0f;
    int ge = g + 8 < i1 ? g + 8 : i1;
    for (int i = g; i < ge; ++i) acc = fmaf(c[i], S[(size_t)i * d + j], acc);
    part[n++] = acc;
  }
  if (n == 0) return 0.0f;
  while (n > 1) {
    int m = 0;
    for (int p = 0; p + 1 < n; p += 2) part[m++] = part[p] + part[p + 1];
    if (n & 1) part[m++] = part[n - 1];
    n = m;
  }
  return part[0];
}

static void delta_rule_token(int d, float* S, const float* kk, const float* qq, const float* aa,
                             const float* vv, float bt, float* w, float* oo) {
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) S[(size_t)i * d + j] = aa[i] * S[(size_t)i * d + j];
  for (int j = 0; j < d; ++j) {
    float u = row_sum(kk, S, d, j, 0, d);
    w[j] = bt * (vv[j] - u);
  }
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) S[(size_t)i * d + j] = fmaf(kk[i], w[j], S[(size_t)i * d + j]);
  for (int j = 0; j < d; ++j) oo[j] = row_sum(qq, S, d, j, 0, d);
}

/* The same token in the mixed basis: rows 0..nlo-1 (INT8 tier) are in the
 * basis T (the Hadamard, or the identity without it), rows nlo..d-1 (FP16
 * tier) in the value basis.
 *   u  = U2 + T(U1),  U1 = sum over rows < nlo of k_i S_i,  U2 = the rest;
 *   w  = beta (v - u);  S_i += k_i T(w) for rows < nlo, S_i += k_i w else;
 *   o  = O2 + T(O1) with O1, O2 the q-weighted sums of the updated rows.
 * Each partial sum is a row_sum over its tier's rows (8-row chains in stored
 * order, then the pairwise tree). */
static void delta_rule_token_mixed(int d, int nlo, int had, float* S, const float* kk,
                                   const float* qq, const float* aa, const float* vv, float bt,
                                   float* w, float* oo) {
  float* p1 = (float*)malloc(sizeof(float) * (size_t)d);
  float* wt = (float*)malloc(sizeof(float) * (size_t)d);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) S[(size_t)i * d + j] = aa[i] * S[(size_t)i * d + j];
  for (int j = 0; j < d; ++j) {
    p1[j] = row_sum(kk, S, d, j, 0, nlo);
    oo[j] = row_sum(kk, S, d, j, nlo, d);
  }
  if (had) orc_fwht(p1, d);
  for (int j = 0; j < d; ++j) {
    float u = oo[j] + p1[j];
    w[j] = bt * (vv[j] - u);
    wt[j] = w[j];
  }
  if (had) orc_fwht(wt, d);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j)
      S[(size_t)i * d + j] = fmaf(kk[i], (i < nlo) ? wt[j] : w[j], S[(size_t)i * d + j]);
  for (int j = 0; j < d; ++j) {
    p1[j] = row_sum(qq, S, d, j, 0, nlo);
    oo[j] = row_sum(qq, S, d, j, nlo, d);
  }
  if (had) orc_fwht(p1, d);
  for (int j = 0; j < d; ++j) oo[j] = oo[j] + p1[j];
  free(p1);
  free(wt);
}

typedef struct {
  const uint16_t *q, *k, *v;
  const float *beta, *decay;
  float* o;
} orc_inputs;

/* Gather token t's inputs for head (b, h) in stored row order. */
static void gather_token(const orc_layout* L, const orc_inputs* in, int t, int b, int h,
                         const int16_t* perm_h, float* kk, float* qq, float* aa, float* vv,
                         float* bt) {
  int d = L->d, B = L->B, H = L->H, Hk = L->Hk;
  int kh = h * Hk / H;
  size_t qk_base = (((size_t)t * B + b) * Hk + kh) * d;
  size_t v_base = (((size_t)t * B + b) * H + h) * d;
  for (int i = 0; i < d; ++i) {
    int p = perm_h ? perm_h[i] : i;
    kk[i] = orc_f32_from_bf16(in->k[qk_base + p]);
    qq[i] = orc_f32_from_bf16(in->q[qk_base + p]);
    aa[i] = L->decay_per_key ? in->decay[v_base + p] : in->decay[((size_t)t * B + b) * H + h];
  }
  for (int j = 0; j < d; ++j) vv[j] = orc_f32_from_bf16(in->v[v_base + j]);
  *bt = in->beta[((size_t)t * B + b) * H + h];
}

static int run_head_unit(const orc_layout* L, const orc_writeback* wb, int64_t step0, int T,
                         int b, int h, const uint8_t* pin, uint8_t* pout, uint16_t* aux,
                         const int16_t* perm, const orc_inputs* in, float* t_dump,
                         float* s_dump) {
  int d = L->d, flags = 0;
  size_t unit = (size_t)b * L->H + h;
  float* S = (float*)malloc(sizeof(float) * (size_t)d * d);
  float *kk = malloc(sizeof(float) * d), *qq = malloc(sizeof(float) * d),
        *aa = malloc(sizeof(float) * d), *vv = malloc(sizeof(float) * d),
        *w = malloc(sizeof(float) * d), *oo = malloc(sizeof(float) * d);
  const int16_t* perm_h = perm ? perm + (size_t)h * d : NULL;
  size_t hb = (L->storage == ORC_STORE_FP32) ? (size_t)d * d * 4 : damp_head_bytes(L);

  if (L->storage == ORC_STORE_FP32)
    memcpy(S, pin + unit * hb, hb);
  else
    damp_load(L, pin + unit * hb, S);

  for (int t = 0; t < T; ++t) {
    int64_t step = step0 + t;
    float bt;
    gather_token(L, in, t, b, h, perm_h, kk, qq, aa, vv, &bt);
    if (mixed(L)) {
      delta_rule_token_mixed(d, d - L->k_hi, L->hadamard, S, kk, qq, aa, vv, bt, w, oo);
    } else {
      if (rotated(L)) orc_fwht(vv, d);
      delta_rule_token(d, S, kk, qq, aa, vv, bt, w, oo);
      if (rotated(L)) orc_fwht(oo, d);
    }
    memcpy(in->o + (((size_t)t * L->B + b) * L->H + h) * d, oo, sizeof(float) * (size_t)d);
    if ((step + 1) % wb->C == 0) {
      if (s_dump) memcpy(s_dump + unit * (size_t)d * d, S, sizeof(float) * (size_t)d * d);
      /* write-back: quantize, then continue from the dequantized state
       * ([LB] Protocol: each write-back is quantized and dequantized before
       * reuse; no unquantized residual is retained) */
      if (L->storage == ORC_STORE_FP32) {
        for (size_t e = 0; e < (size_t)d * d; ++e)
          if (!isfinite(S[e])) flags |= ORC_ENONFINITE;
        memcpy(pout + unit * hb, S, hb);
      } else {
        size_t nel = (size_t)(d - L->k_hi) * d;
        uint16_t* aux_head = NULL;
        if (aux) {
          if (wb->mode == ORC_ROUND_DIRECTION) aux_head = (uint16_t*)((uint8_t*)aux + unit * (nel / 4));
          else if (wb->mode >= ORC_ROUND_RESIDUAL2) aux_head = (uint16_t*)((uint8_t*)aux + unit * (nel / 2));
          else aux_head = aux + unit * nel;
        }
        float* th = t_dump ? t_dump + unit * (size_t)d * d : NULL;
        const uint8_t* prev = (t == 0) ? pin + unit * hb : pout + unit * hb;
        flags |= damp_store(L, wb, step, b, h, S, prev, pout + unit * hb, aux_head, th);
        damp_load(L, pout + unit * hb, S);
      }
    }
  }
  free(S);
  free(kk);
  free(qq);
  free(aa);
  free(vv);
  free(w);
  free(oo);
  return flags;
}

/* ---- variable-width storage ([LB] State bit allocation, Allocation units,
 * Levels and storage) ---- */
static uint32_t get_bits(const uint8_t* p, size_t bitpos, int nb) {
  uint32_t v = 0;
  for (int k = 0; k < nb; ++k) {
    size_t bp = bitpos + (size_t)k;
    v |= (uint32_t)((p[bp >> 3] >> (bp & 7)) & 1u) << k;
  }
  return v;
}

static void put_bits(uint8_t* p, size_t bitpos, int nb, uint32_t v) {
  for (int k = 0; k < nb; ++k) {
    size_t bp = bitpos + (size_t)k;
    uint8_t m = (uint8_t)(1u << (bp & 7));
    if ((v >> k) & 1u)
      p[bp >> 3] |= m;
    else
      p[bp >> 3] &= (uint8_t)~m;
  }
}

static void varbit_load_seq(const orc_layout* L, const uint8_t* packed, int b, float* S) {
  vb_sections sec = varbit_sections(L);
  int d = L->d, rows = L->H * d;
  const uint8_t* pay = packed + (size_t)b * sec.payload_per_seq;
  const uint16_t* sc = (const uint16_t*)(packed + sec.off_scale) + (size_t)b * rows;
  const uint8_t* wd = packed + sec.off_width + (size_t)b * rows;
  const uint32_t* of = (const uint32_t*)(packed + sec.off_offsets) + (size_t)b * (rows + 1);
  for (int r = 0; r < rows; ++r) {
    int bw = wd[r];
    int nl = (1 << (bw - 1)) - 1;
    float D = orc_f32_from_f16(sc[r]);
    for (int j = 0; j < d; ++j) {
      uint32_t u = get_bits(pay + of[r], (size_t)j * bw, bw);
      /* one bit: code 1 = +scale, 0 = -scale */
      int lv = (bw == 1) ? 2 * (int)u - 1 : (int)u - nl;
      S[(size_t)r * d + j] = (float)lv * D;
    }
  }
}

/* Head units: element (i, j) of head h at bit (i d + j) w_h of the head's
 * payload; value = (u - n) * step of (block i / 32, column j). */
static void varbit_head_load_seq(const orc_layout* L, const uint8_t* packed, int b, float* S) {
  vb_sections sec = varbit_sections(L);
  int d = L->d, H = L->H, nbk = d / 32;
  const uint8_t* pay = packed + (size_t)b * sec.payload_per_seq;
  const uint16_t* sc = (const uint16_t*)(packed + sec.off_scale) + (size_t)b * H * nbk * d;
  const uint8_t* wd = packed + sec.off_width + (size_t)b * H;
  const uint32_t* of = (const uint32_t*)(packed + sec.off_offsets) + (size_t)b * (H + 1);
  for (int h = 0; h < H; ++h) {
    int bw = wd[h];
    int nl = (1 << (bw - 1)) - 1;
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < d; ++j) {
        uint32_t u = get_bits(pay + of[h], ((size_t)i * d + j) * bw, bw);
        float D = orc_f32_from_f16(sc[((size_t)h * nbk + i / 32) * d + j]);
        S[((size_t)h * d + i) * d + j] = (float)((int)u - nl) * D;
      }
  }
}

/* Quantize every head of sequence b with widths bits[H]: each (block of 32
 * key channels, column) group gets its own fitted step. */
static int varbit_head_store_seq(const orc_layout* L, const orc_writeback* wb, int64_t step, int b,
                                 const float* S, const uint8_t* bits, uint8_t* packed, uint16_t* aux,
                                 float* t_dump) {
  vb_sections sec = varbit_sections(L);
  int d = L->d, H = L->H, nbk = d / 32, flags = 0;
  uint8_t* pay = packed + (size_t)b * sec.payload_per_seq;
  uint16_t* sc = (uint16_t*)(packed + sec.off_scale) + (size_t)b * H * nbk * d;
  uint8_t* wd = packed + sec.off_width + (size_t)b * H;
  uint32_t* of = (uint32_t*)(packed + sec.off_offsets) + (size_t)b * (H + 1);
  float x[32], tt[32];
  uint16_t e[32];
  int32_t q[32];
  uint32_t off = 0;
  for (int h = 0; h < H; ++h) {
    of[h] = off;
    off += (uint32_t)(d * d / 8) * bits[h];
  }
  of[H] = off;
  for (int h = 0; h < H; ++h) {
    int bw = bits[h], nl = (1 << (bw - 1)) - 1;
    wd[h] = (uint8_t)bw;
    for (int g = 0; g < nbk; ++g)
      for (int j = 0; j < d; ++j) {
        for (int r = 0; r < 32; ++r) {
          size_t el = ((size_t)h * d + 32 * g + r) * d + j;
          x[r] = S[el];
          if (aux) e[r] = aux[(size_t)b * H * d * d + el];
        }
        flags |= orc_varbit_group(x, 32, bw, wb ? wb->mode : ORC_ROUND_NEAREST, wb ? wb->seed : 0,
                                  step, h, b, 32 * g * d + j, d, aux ? e : NULL, q,
                                  &sc[((size_t)h * nbk + g) * d + j], NULL, tt);
        for (int r = 0; r < 32; ++r) {
          size_t el = ((size_t)h * d + 32 * g + r) * d + j;
          if (aux) aux[(size_t)b * H * d * d + el] = e[r];
          if (t_dump) t_dump[(size_t)b * H * d * d + el] = tt[r];
          put_bits(pay + of[h], ((size_t)(32 * g + r) * d + j) * bw, bw, (uint32_t)(q[r] + nl));
        }
      }
  }
  return flags;
}

/* Quantize every row of sequence b with widths `bits` and write payload,
 * scales, widths and offsets. */
static int varbit_store_seq(const orc_layout* L, const orc_writeback* wb, int64_t step, int b,
                            const float* S, const uint8_t* bits, uint8_t* packed, uint16_t* aux,
                            float* t_dump) {
  vb_sections sec = varbit_sections(L);
  int d = L->d, rows = L->H * d, flags = 0;
  uint8_t* pay = packed + (size_t)b * sec.payload_per_seq;
  uint16_t* sc = (uint16_t*)(packed + sec.off_scale) + (size_t)b * rows;
  uint8_t* wd = packed + sec.off_width + (size_t)b * rows;
  uint32_t* of = (uint32_t*)(packed + sec.off_offsets) + (size_t)b * (rows + 1);
  int32_t* q = (int32_t*)malloc(sizeof(int32_t) * (size_t)d);
  uint32_t off = 0;
  for (int r = 0; r < rows; ++r) {
    of[r] = off;
    off += (uint32_t)(d / 8) * bits[r];
  }
  of[rows] = off;
  for (int r = 0; r < rows; ++r) {
    int h = r / d, i = r % d, bw = bits[r];
    int nl = (1 << (bw - 1)) - 1;
    uint16_t* e = aux ? aux + ((size_t)b * rows + r) * d : NULL;
    float* tt = t_dump ? t_dump + ((size_t)b * rows + r) * d : NULL;
    flags |= orc_varbit_row(S + (size_t)r * d, d, bw, wb ? wb->mode : ORC_ROUND_NEAREST,
                            wb ? wb->seed : 0, step, h, b, i * d, e, q, &sc[r], NULL, tt);
    wd[r] = (uint8_t)bw;
    for (int j = 0; j < d; ++j) put_bits(pay + of[r], (size_t)j * bw, bw, (uint32_t)(q[j] + nl));
  }
  free(q);
  return flags;
}

static int run_seq_unit(const orc_layout* L, const orc_writeback* wb, int64_t step0, int T, int b,
                        const uint8_t* pin, uint8_t* pout, uint16_t* aux, double* stats,
                        const orc_inputs* in, float* t_dump) {
  int d = L->d, H = L->H, rows = H * d, flags = 0;
  float* S = (float*)malloc(sizeof(float) * (size_t)rows * d);
  float *kk = malloc(sizeof(float) * d), *qq = malloc(sizeof(float) * d),
        *aa = malloc(sizeof(float) * d), *vv = malloc(sizeof(float) * d),
        *w = malloc(sizeof(float) * d), *oo = malloc(sizeof(float) * d);
  double* ca2 = (double*)calloc((size_t)rows, sizeof(double));
  double* ck = (double*)calloc((size_t)rows, sizeof(double));
  double* cost = (double*)malloc(sizeof(double) * (size_t)rows);
  double* Rr = (double*)malloc(sizeof(double) * (size_t)rows);
  uint8_t* bits = (uint8_t*)malloc((size_t)rows);
  double* st = stats + (size_t)b * rows * 2;
  int C = wb->C;
  double lam = 1.0;
  for (int c = 0; c < C; ++c) lam *= (1.0 - 2.0 / 65.0);

  int head_units = L->storage == ORC_STORE_VARBIT_HEAD;
  if (head_units)
    varbit_head_load_seq(L, pin, b, S);
  else
    varbit_load_seq(L, pin, b, S);
  for (int t = 0; t < T; ++t) {
    int64_t step = step0 + t;
    for (int h = 0; h < H; ++h) {
      float bt;
      gather_token(L, in, t, b, h, NULL, kk, qq, aa, vv, &bt);
      delta_rule_token(d, S + (size_t)h * d * d, kk, qq, aa, vv, bt, w, oo);
      memcpy(in->o + (((size_t)t * L->B + b) * H + h) * d, oo, sizeof(float) * (size_t)d);
      /* per-token erasure statistics ([LB] State bit allocation: EMA of
       * e^(2g) = a^2 and of beta (2 - beta) k^2) */
      for (int i = 0; i < d; ++i) {
        double a = (double)aa[i], be = (double)bt, kd = (double)kk[i];
        ca2[h * d + i] += a * a;
        ck[h * d + i] += (be * (2.0 - be)) * (kd * kd);
      }
    }
    if ((step + 1) % C == 0) {
      /* chunk-aware EMA with a 64-token span, initialised at the first
       * write-back */
      for (int r = 0; r < rows; ++r) {
        double ma = ca2[r] / (double)C, mk = ck[r] / (double)C;
        if (step + 1 == C) {
          st[2 * r + 0] = ma;
          st[2 * r + 1] = mk;
        } else {
          st[2 * r + 0] = lam * st[2 * r + 0] + (1.0 - lam) * ma;
          st[2 * r + 1] = lam * st[2 * r + 1] + (1.0 - lam) * mk;
        }
        ca2[r] = 0.0;
        ck[r] = 0.0;
      }
      if (head_units) {
        /* head units ([LB] Allocation units): R~ = 1, so the cost of a head
         * is its decay weight alone, the mean of its rows' weights (rows
         * summed in order in FP64); one budget over the layer's heads */
        for (int h = 0; h < H; ++h) {
          double sum = 0.0;
          for (int i = 0; i < d; ++i) {
            int r = h * d + i;
            sum += orc_persistence(L->persistence, st[2 * r + 0], st[2 * r + 1], C);
          }
          cost[h] = sum / (double)d;
        }
        flags |= orc_allocate_bits(H, cost, L->avg_bits, L->b_min, L->b_max, bits);
        if (flags & ORC_EINVAL) break;
        flags |= varbit_head_store_seq(L, wb, step, b, S, bits, pout, aux, t_dump);
        varbit_head_load_seq(L, pout, b, S);
        continue;
      }
      /* cost c_i = Gamma_hat_i * R~_i^2 with R~ the row range normalised by
       * the RMS of the ranges of its output group (one head) */
      for (int r = 0; r < rows; ++r) {
        float R = 0.0f;
        for (int j = 0; j < d; ++j) {
          float a = fabsf(S[(size_t)r * d + j]);
          if (a > R) R = a;
        }
        Rr[r] = (double)R;
      }
      for (int h = 0; h < H; ++h) {
        double ms = 0.0;
        for (int i = 0; i < d; ++i) ms += Rr[h * d + i] * Rr[h * d + i];
        double rms = sqrt(ms / (double)d);
        for (int i = 0; i < d; ++i) {
          int r = h * d + i;
          double rt = rms > 0.0 ? Rr[r] / rms : 0.0;
          cost[r] = orc_persistence(L->persistence, st[2 * r + 0], st[2 * r + 1], C) * (rt * rt);
        }
      }
      if (L->budget_scope == 1) {
        flags |= orc_allocate_bits(rows, cost, L->avg_bits, L->b_min, L->b_max, bits);
      } else {
        for (int h = 0; h < H; ++h)
          flags |= orc_allocate_bits(d, cost + h * d, L->avg_bits, L->b_min, L->b_max,
                                     bits + h * d);
      }
      if (flags & ORC_EINVAL) break;
      flags |= varbit_store_seq(L, wb, step, b, S, bits, pout, aux, t_dump);
      varbit_load_seq(L, pout, b, S);
    }
  }
  free(S);
  free(kk);
  free(qq);
  free(aa);
  free(vv);
  free(w);
  free(oo);
  free(ca2);
  free(ck);
  free(cost);
  free(Rr);
  free(bits);
  return flags;
}

static int layout_ok(const orc_layout* L) {
  if (L->low_bits != 0 && L->low_bits != 8 && L->low_bits != 4) return 0;
  if (L->B <= 0 || L->H <= 0 || L->Hk <= 0 || L->H % L->Hk) return 0;
  if (L->d != 16 && L->d != 32 && L->d != 64 && L->d != 128) return 0;
  if (L->storage == ORC_STORE_DAMP) {
    if (L->k_hi < 0 || L->k_hi > L->d || L->block <= 0 || L->d % L->block) return 0;
  }
  if (L->storage == ORC_STORE_VARBIT) {
    /* b_min = 1 for row units, b_max = 8, or 16 at C = 1 ([LB] State bit
     * allocation, Allocation units) */
    if (L->hadamard || L->b_min < 1 || L->b_max > 16 || L->b_min > L->b_max) return 0;
    double tot = L->avg_bits * (double)(L->H * L->d);
    if (tot != floor(tot)) return 0;
  }
  if (L->storage == ORC_STORE_VARBIT_HEAD) {
    /* head units: b_min >= 2 (a one-bit head is ruled out), blocks of 32
     * key channels, one budget over the layer's heads */
    if (L->hadamard || L->b_min < 2 || L->b_max > 16 || L->b_min > L->b_max) return 0;
    if (L->d % 32 || L->budget_scope != 1) return 0;
    double tot = L->avg_bits * (double)L->H;
    if (tot != floor(tot) || L->avg_bits < L->b_min || L->avg_bits > L->b_max) return 0;
  }
  if (L->storage < ORC_STORE_FP32 || L->storage > ORC_STORE_VARBIT_HEAD) return 0;
  return 1;
}

int orc_run(const orc_layout* L, const orc_writeback* wb, int64_t step0, int T, int u0, int u1,
            const void* packed_in, void* packed_out, void* aux, double* stats,
            const int16_t* perm, const uint16_t* q, const uint16_t* k, const uint16_t* v,
            const float* beta, const float* decay, float* o, float* t_dump, float* s_dump) {
  if (!layout_ok(L) || wb->C <= 0 || step0 % wb->C || T % wb->C) return ORC_EINVAL;
  if (wb->mode < ORC_ROUND_NEAREST || wb->mode > ORC_ROUND_RESIDUAL4) return ORC_EINVAL;
  /* residual memory: DAMP storage, integers kept in the auxiliary buffer */
  if (wb->mode >= ORC_ROUND_RESIDUAL2 && (L->storage != ORC_STORE_DAMP || !aux)) return ORC_EINVAL;
  /* direction memory: DAMP at a write-back every token (the votes compare
   * each token's proposal with the value stored after the previous token) */
  if (wb->mode == ORC_ROUND_DIRECTION && (L->storage != ORC_STORE_DAMP || wb->C != 1 || !aux))
    return ORC_EINVAL;
  orc_inputs in = {q, k, v, beta, decay, o};
  int flags = 0;
  if (L->storage == ORC_STORE_VARBIT || L->storage == ORC_STORE_VARBIT_HEAD) {
    for (int b = u0; b < u1; ++b)
      flags |= run_seq_unit(L, wb, step0, T, b, (const uint8_t*)packed_in, (uint8_t*)packed_out,
                            (uint16_t*)aux, stats, &in, t_dump);
  } else {
    for (int u = u0; u < u1; ++u)
      flags |= run_head_unit(L, wb, step0, T, u / L->H, u % L->H, (const uint8_t*)packed_in,
                             (uint8_t*)packed_out, (uint16_t*)aux, perm, &in, t_dump, s_dump);
  }
  return flags;
}

/* ------------------------------------------------------------------------ */
/* State conversion (deterministic rounding)                                 */
/* ------------------------------------------------------------------------ */
int orc_state_pack(const orc_layout* L, const float* S, const int16_t* perm,
                   const uint8_t* widths, void* packed) {
  if (!layout_ok(L)) return ORC_EINVAL;
  int d = L->d, flags = 0;
  orc_writeback wb = {ORC_ROUND_NEAREST, 0, 1};
  orc_layout Lc = *L;
  Lc.domain = ORC_DOMAIN_CANONICAL;
  float* tmp = (float*)malloc(sizeof(float) * (size_t)d * d);
  if (L->storage == ORC_STORE_VARBIT_HEAD) {
    /* widths [B][H] (or avg_bits for every head) summing to avg_bits * H */
    int H = L->H;
    uint8_t* bits = (uint8_t*)malloc((size_t)H);
    for (int b = 0; b < L->B && !(flags & ORC_EINVAL); ++b) {
      long sum = 0;
      for (int h = 0; h < H; ++h) {
        bits[h] = widths ? widths[(size_t)b * H + h] : (uint8_t)nearbyint(L->avg_bits);
        sum += bits[h];
        if (bits[h] < 1 || bits[h] > 16) flags |= ORC_EINVAL;
      }
      if ((double)sum != L->avg_bits * (double)H) flags |= ORC_EINVAL;
      if (!(flags & ORC_EINVAL))
        flags |= varbit_head_store_seq(L, NULL, 0, b, S + (size_t)b * H * d * d, bits, (uint8_t*)packed,
                                       NULL, NULL);
    }
    free(bits);
  } else if (L->storage == ORC_STORE_VARBIT) {
    int rows = L->H * d;
    uint8_t* bits = (uint8_t*)malloc((size_t)rows);
    float* seq = (float*)malloc(sizeof(float) * (size_t)rows * d);
    for (int r = 0; r < rows; ++r) bits[r] = widths ? widths[r] : (uint8_t)nearbyint(L->avg_bits);
    /* every sequence must fill exactly its payload: widths summing to avg_bits * H * d */
    for (int b = 0; b < L->B; ++b) {
      long sum = 0;
      for (int r = 0; r < rows; ++r) sum += widths ? widths[(size_t)b * rows + r] : bits[r];
      if ((double)sum != L->avg_bits * (double)rows) {
        free(bits);
        free(tmp);
        return ORC_EINVAL;
      }
    }
    for (int b = 0; b < L->B; ++b) {
      memcpy(seq, S + (size_t)b * rows * d, sizeof(float) * (size_t)rows * d);
      flags |= varbit_store_seq(L, NULL, 0, b, seq, widths ? widths + (size_t)b * rows : bits,
                                (uint8_t*)packed, NULL, NULL);
    }
    free(bits);
    free(seq);
  } else {
    size_t hb = (L->storage == ORC_STORE_FP32) ? (size_t)d * d * 4 : damp_head_bytes(L);
    for (int b = 0; b < L->B; ++b)
      for (int h = 0; h < L->H; ++h) {
        const float* src = S + ((size_t)b * L->H + h) * d * d;
        for (int i = 0; i < d; ++i) {
          int p = perm ? perm[(size_t)h * d + i] : i;
          memcpy(tmp + (size_t)i * d, src + (size_t)p * d, sizeof(float) * (size_t)d);
        }
        uint8_t* dst = (uint8_t*)packed + ((size_t)b * L->H + h) * hb;
        if (L->storage == ORC_STORE_FP32)
          memcpy(dst, tmp, hb);
        else
          flags |= damp_store(&Lc, &wb, 0, b, h, tmp, dst, dst, NULL, NULL);
      }
  }
  free(tmp);
  return flags;
}

int orc_state_unpack(const orc_layout* L, const void* packed, const int16_t* perm, float* S) {
  if (!layout_ok(L)) return ORC_EINVAL;
  int d = L->d;
  orc_layout Lc = *L;
  Lc.domain = ORC_DOMAIN_CANONICAL;
  if (L->storage == ORC_STORE_VARBIT || L->storage == ORC_STORE_VARBIT_HEAD) {
    for (int b = 0; b < L->B; ++b) {
      if (L->storage == ORC_STORE_VARBIT_HEAD)
        varbit_head_load_seq(L, (const uint8_t*)packed, b, S + (size_t)b * L->H * d * d);
      else
        varbit_load_seq(L, (const uint8_t*)packed, b, S + (size_t)b * L->H * d * d);
    }
    return ORC_OK;
  }
  float* tmp = (float*)malloc(sizeof(float) * (size_t)d * d);
  size_t hb = (L->storage == ORC_STORE_FP32) ? (size_t)d * d * 4 : damp_head_bytes(L);
  for (int b = 0; b < L->B; ++b)
    for (int h = 0; h < L->H; ++h) {
      const uint8_t* src = (const uint8_t*)packed + ((size_t)b * L->H + h) * hb;
      if (L->storage == ORC_STORE_FP32)
        memcpy(tmp, src, hb);
      else
        damp_load(&Lc, src, tmp);
      float* dst = S + ((size_t)b * L->H + h) * d * d;
      for (int i = 0; i < d; ++i) {
        int p = perm ? perm[(size_t)h * d + i] : i;
        memcpy(dst + (size_t)p * d, tmp + (size_t)i * d, sizeof(float) * (size_t)d);
      }
    }
  free(tmp);
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Protected-row selection ([DAMP] Risk scoring and selection; Calibration): */
/*   E_u  = mean squared error energy of row u under Hadamard-INT8 (INT4)    */
/*          quantize -> dequantize, over the sampled calibration states;     */
/*   a_eff,u = exp(mean log a_u);  P_u = 1 / max(1 - a_eff,u^2, tau);        */
/*   C_u = E_u P_u; the top k_hi rows of each head are protected (ties to    */
/*   the lower index).  The permutation lists the unprotected rows, then the */
/*   protected ones, each group in ascending order: the protected rows sit   */
/*   contiguously at the end of the stored order.                            */
/* ------------------------------------------------------------------------ */
int orc_calibrate(const orc_layout* L, int Bc, int T, int every, double tau,
                  const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* beta,
                  const float* decay, double* score_out, int16_t* perm_out) {
  orc_layout Lc = *L;
  Lc.B = Bc;
  if (!layout_ok(&Lc) || L->storage != ORC_STORE_DAMP || every <= 0) return ORC_EINVAL;
  int d = L->d, H = L->H, nb = d / L->block;
  orc_inputs in = {q, k, v, beta, decay, NULL};
  double* E = (double*)calloc((size_t)H * d, sizeof(double));
  double* sl = (double*)calloc((size_t)H * d, sizeof(double));
  float* S = (float*)malloc(sizeof(float) * (size_t)d * d);
  float *kk = malloc(sizeof(float) * d), *qq = malloc(sizeof(float) * d),
        *aa = malloc(sizeof(float) * d), *vv = malloc(sizeof(float) * d),
        *w = malloc(sizeof(float) * d), *oo = malloc(sizeof(float) * d),
        *row = malloc(sizeof(float) * d);
  uint8_t* codes = (uint8_t*)malloc((size_t)L->block);
  long nsamp = 0;
  for (int b = 0; b < Bc; ++b)
    for (int h = 0; h < H; ++h) {
      memset(S, 0, sizeof(float) * (size_t)d * d);
      for (int t = 0; t < T; ++t) {
        float bt;
        gather_token(&Lc, &in, t, b, h, NULL, kk, qq, aa, vv, &bt);
        for (int i = 0; i < d; ++i) sl[h * d + i] += log((double)aa[i]);
        delta_rule_token(d, S, kk, qq, aa, vv, bt, w, oo);
        if ((t + 1) % every == 0) {
          if (b == 0 && h == 0) ++nsamp;
          for (int i = 0; i < d; ++i) {
            memcpy(row, S + (size_t)i * d, sizeof(float) * (size_t)d);
            if (L->hadamard) orc_fwht(row, d);
            double err = 0.0;
            for (int bl = 0; bl < nb; ++bl) {
              uint16_t sh, zh;
              int j0 = bl * L->block;
              orc_lowbit_block(row + j0, L->block, low_levels(L), ORC_ROUND_NEAREST, 0, 0, 0, 0, 0, NULL,
                               codes, &sh, &zh, NULL);
              float s = orc_f32_from_f16(sh), z = orc_f32_from_f16(zh);
              for (int j = 0; j < L->block; ++j) {
                double e = (double)row[j0 + j] - (double)fmaf((float)codes[j], s, z);
                err += e * e;
              }
            }
            E[h * d + i] += err;
          }
        }
      }
    }
  double ns = (double)Bc * (double)nsamp, nt = (double)Bc * (double)T;
  int* idx = (int*)malloc(sizeof(int) * (size_t)d);
  double* sc = (double*)malloc(sizeof(double) * (size_t)d);
  char* prot = (char*)malloc((size_t)d);
  for (int h = 0; h < H; ++h) {
    for (int i = 0; i < d; ++i) {
      double aeff = exp(sl[h * d + i] / nt);
      double den = 1.0 - aeff * aeff;
      if (den < tau) den = tau;
      sc[i] = (E[h * d + i] / ns) * (1.0 / den);
      if (score_out) score_out[(size_t)h * d + i] = sc[i];
      prot[i] = 0;
    }
    /* pick the k_hi largest scores, ties to the lower index */
    for (int c = 0; c < L->k_hi; ++c) {
      int pick = -1;
      for (int i = 0; i < d; ++i)
        if (!prot[i] && (pick < 0 || sc[i] > sc[pick])) pick = i;
      prot[pick] = 1;
    }
    int n = 0;
    for (int i = 0; i < d; ++i)
      if (!prot[i]) idx[n++] = i;
    for (int i = 0; i < d; ++i)
      if (prot[i]) idx[n++] = i;
    for (int i = 0; i < d; ++i) perm_out[(size_t)h * d + i] = (int16_t)idx[i];
  }
  free(idx);
  free(sc);
  free(prot);
  free(E);
  free(sl);
  free(S);
  free(kk);
  free(qq);
  free(aa);
  free(vv);
  free(w);
  free(oo);
  free(row);
  free(codes);
  return ORC_OK;
}
