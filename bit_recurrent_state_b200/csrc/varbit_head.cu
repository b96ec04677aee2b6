// Variable-width storage with one width per head ("Low-Bit Recurrent
// States in Hybrid Language Models", Allocation units: when decay and
// normalization are per head, as in Gated DeltaNet, each head has one width
// and one FP16 step per block of 32 key channels; R~ = 1, so the decay alone
// sets the widths; b_min = 2.  State bit allocation: one budget over the
// layer's heads.  Levels and storage: symmetric levels {-n..n} step, the
// step fitted over 16 clip factors by squared error per scale group).
//
// Layout of the work: one CTA of four warps per head; warp w owns columns
// 32w..32w+31 and lane l owns column 32w + l of every row.  A scale group
// (rows 32g..32g+31 of one column) therefore lives in one lane: its range,
// its fit and every sum over key rows (8-row fmaf chains in row order,
// added in a pairwise tree) are lane-local.
//
// Three launches per token, as for row units: phase 0 (update, o, the
// statistics and the head's cost), the allocator over each sequence's
// heads, phase 1 (the identical update, then per block of 32 rows the
// fitted steps, the codes and the bit-packed rows at the head's new
// offset).
#include <cuda_runtime.h>
#include <cstdint>

#include "brs_device.cuh"
#include "brs_internal.h"

namespace brs {

namespace {

constexpr int kVhD = 128;          // head dimension of the kernels
constexpr int kVhWarps = kVhD / 32;
constexpr int kVhBlocks = kVhD / 32;   // scale blocks of 32 key channels

size_t vh_r256(size_t x) { return (x + 255) / 256 * 256; }

struct __align__(16) VhRow {
  float k, a, q, pad;
};

// the stored code of element bit position p (width bw, mask (1 << bw) - 1).
// Both words are loaded unconditionally (no divergent second load): the
// word after a head's last one is the next head's, or past the payload the
// first of the step section, inside the stored state either way.
__device__ __forceinline__ uint32_t vh_code(const uint32_t* words, uint32_t p, int bw, uint32_t mask) {
  const uint32_t wi = p >> 5;
  return __funnelshift_r(__ldg(words + wi), __ldg(words + wi + 1), p & 31u) & mask;
}

// fitted step of one scale group of 32 targets y (levels -n..n): the
// candidate with the least squared error, ties to the smaller clip factor.
// The error of -y equals that of y (round-to-nearest-even and the clip are
// odd), so the scan runs on |y| with a one-sided clip.  Returns the FP16
// bits; *bad is set when no candidate is finite.
__device__ __forceinline__ uint16_t vh_fit(const float (&y)[32], int n, float one, bool* bad) {
  float R = 0.0f;
#pragma unroll
  for (int r = 0; r < 32; ++r) R = fmaxf(R, fabsf(y[r]));
  *bad = false;
  if (R == 0.0f) return 0;
  const float fn = (float)n;
  int bm = -1;
  float bE = 0.0f;
  uint16_t bbits = 0;
#pragma unroll 1
  for (int m0 = 0; m0 < 16; m0 += 4) {
    float st[4], iv[4], E[4];
    uint16_t sb[4];
    bool ok[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      varbit_candidate(m0 + k, R, n, st[k], iv[k], sb[k], ok[k]);
      E[k] = 0.0f;
    }
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const float v = fabsf(y[r]);
      float t0, t1, t2, t3;
      mul2(t0, t1, v, v, iv[0], iv[1]);
      mul2(t2, t3, v, v, iv[2], iv[3]);
      // nearest integer (ties to even): t * one + magic, one = 1 read at run
      // time so the add keeps its own rounding
      fma2(t0, t1, t0, t1, one, one, kRoundMagic, kRoundMagic);
      fma2(t2, t3, t2, t3, one, one, kRoundMagic, kRoundMagic);
      sub2(t0, t1, t0, t1, kRoundMagic, kRoundMagic);
      sub2(t2, t3, t2, t3, kRoundMagic, kRoundMagic);
      t0 = fminf(t0, fn);
      t1 = fminf(t1, fn);
      t2 = fminf(t2, fn);
      t3 = fminf(t3, fn);
      mul2(t0, t1, st[0], st[1], t0, t1);
      mul2(t2, t3, st[2], st[3], t2, t3);
      sub2(t0, t1, v, v, t0, t1);
      sub2(t2, t3, v, v, t2, t3);
      fma2(E[0], E[1], t0, t1, t0, t1, E[0], E[1]);
      fma2(E[2], E[3], t2, t3, t2, t3, E[2], E[3]);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (ok[k] && (bm < 0 || E[k] < bE)) {
        bm = m0 + k;
        bE = E[k];
        bbits = sb[k];
      }
  }
  if (bm < 0) {
    *bad = true;
    return 0x7c00u;
  }
  return bbits;
}

// the warp's 32 codes of one row segment (lane l's code at bit l * bw)
// OR-ed into bw words.  A width that divides 32 puts 32 / bw whole codes in
// each word: the lanes of a word combine theirs with a butterfly of
// shuffles and the word's first lane stores it.  Other widths straddle
// words: one OR-reduction over the warp per word, lane k storing word k.
__device__ __forceinline__ void vh_store_segment(uint32_t* dst, uint32_t u, int bw, int lane) {
  if ((bw & (bw - 1)) == 0) {
    const int g = 32 >> (__ffs(bw) - 1);              // lanes per word
    uint32_t v = u << ((lane & (g - 1)) * bw);
    for (int s = 1; s < g; s <<= 1) v |= __shfl_xor_sync(0xffffffffu, v, s);
    if ((lane & (g - 1)) == 0) dst[lane / g] = v;
    return;
  }
  const int lb = lane * bw, lw = lb >> 5, sh = lb & 31;
  const uint32_t lo = u << sh;
  const uint32_t hi = (sh + bw > 32) ? (u >> (32 - sh)) : 0u;
  for (int k = 0; k < bw; ++k) {
    const uint32_t part = (lw == k ? lo : 0u) | (lw + 1 == k ? hi : 0u);
    const uint32_t word = __reduce_or_sync(0xffffffffu, part);
    if (lane == k) dst[k] = word;
  }
}

template <int PHASE, int MODE>
__global__ void __launch_bounds__(32 * kVhWarps, PHASE == 0 ? 1 : 7) varbit_head_kernel(const VbArgs a) {
  constexpr int D = kVhD;
  __shared__ VhRow rows[D];
  __shared__ double gam[D];
  const int head = blockIdx.x;
  if (head >= a.B * a.H) return;
  const int b = head / a.H, h = head - b * a.H;
  const int t = threadIdx.x, lane = t % 32;
  const int j = t;                                   // my column (warp w: 32w + lane)
  const uint8_t* pin = (const uint8_t*)a.packed_in;
  uint8_t* pout = (uint8_t*)a.packed_out;
  const int bw_in = pin[a.sec.off_width + head];
  const uint32_t off_in = ((const uint32_t*)(pin + a.sec.off_offsets))[(size_t)b * (a.H + 1) + h];
  const uint32_t* win = (const uint32_t*)(pin + (size_t)b * a.sec.payload_per_seq + off_in);
  const uint16_t* sc_in = (const uint16_t*)(pin + a.sec.off_scale) + (size_t)head * kVhBlocks * D;

  {
    const size_t qk = ((size_t)b * a.Hk + h * a.Hk / a.H) * D;
    VhRow r;
    r.k = bf16_to_f32(a.k[qk + t]);
    r.q = bf16_to_f32(a.q[qk + t]);
    r.a = a.decay_per_key ? a.decay[(size_t)head * D + t] : a.decay[head];
    r.pad = 0.0f;
    rows[t] = r;
  }
  const float vj = bf16_to_f32(a.v[(size_t)head * D + j]);
  const float beta = a.beta[head];
  const int n_in = (1 << (bw_in - 1)) - 1;
  const uint32_t mask_in = (bw_in >= 32) ? 0xffffffffu : ((1u << bw_in) - 1u);
  __syncthreads();

  // stored value of (i, j) after the decay; step = the stored step of
  // (block i / 32, column j)
  auto decayed = [&](int i, const VhRow& r, float step) {
    const uint32_t u = vh_code(win, (uint32_t)(i * D + j) * (uint32_t)bw_in, bw_in, mask_in);
    const float s = __fmul_rn((float)((int)u - n_in), step);
    return __fmul_rn(r.a, s);
  };

  // ---- pass 1: u_j = sum_i k_i (a_i S_ij)
  float u;
  {
    GroupTree<1> tree;
    for (int g = 0; g < kVhBlocks; ++g) {
      const float step = f16_to_f32(sc_in[g * D + j]);
#pragma unroll
      for (int g8 = 0; g8 < 4; ++g8) {
        float acc[1] = {0.0f};
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int i = 32 * g + 8 * g8 + r;
          const VhRow rr = rows[i];
          acc[0] = __fmaf_rn(rr.k, decayed(i, rr, step), acc[0]);
        }
        tree.push(acc);
      }
    }
    float res[1];
    tree.result(res);
    u = res[0];
  }
  if (!isfinite(u)) raise_flag(a.flags, BRS_FLAG_NONFINITE);
  const float w = __fmul_rn(beta, __fsub_rn(vj, u));

  // ---- pass 2 in blocks of 32 rows
  GroupTree<1> otree;
  int bw_out = 0, n_out = 0;
  uint32_t* wout = nullptr;
  uint16_t* sc_out = nullptr;
  uint16_t* auxh = (MODE == BRS_ROUND_ERRFEEDBACK) ? (uint16_t*)a.aux + (size_t)head * D * D : nullptr;
  if constexpr (PHASE == 1) {
    bw_out = pout[a.sec.off_width + head];
    n_out = (1 << (bw_out - 1)) - 1;
    const uint32_t off_out = ((const uint32_t*)(pout + a.sec.off_offsets))[(size_t)b * (a.H + 1) + h];
    wout = (uint32_t*)(pout + (size_t)b * a.sec.payload_per_seq + off_out);
    sc_out = (uint16_t*)(pout + a.sec.off_scale) + (size_t)head * kVhBlocks * D;
  }
  for (int g = 0; g < kVhBlocks; ++g) {
    const float step_g = f16_to_f32(sc_in[g * D + j]);
    float y[32];
#pragma unroll
    for (int r8 = 0; r8 < 4; ++r8) {
      float acc[1] = {0.0f};
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int i = 32 * g + 8 * r8 + r;
        const VhRow rr = rows[i];
        const float x = __fmaf_rn(rr.k, w, decayed(i, rr, step_g));
        if constexpr (PHASE == 0) acc[0] = __fmaf_rn(rr.q, x, acc[0]);
        y[8 * r8 + r] = x;
      }
      if constexpr (PHASE == 0) otree.push(acc);
    }
    if constexpr (PHASE == 1) {
      if constexpr (MODE == BRS_ROUND_ERRFEEDBACK) {
#pragma unroll
        for (int r = 0; r < 32; ++r) y[r] = __fadd_rn(y[r], f16_to_f32(auxh[(size_t)(32 * g + r) * D + j]));
      }
      bool bad;
      const uint16_t sb = vh_fit(y, n_out, a.one, &bad);
      if (bad) raise_flag(a.flags, BRS_FLAG_OVERFLOW);
      sc_out[g * D + j] = sb;
      const float step = f16_to_f32(sb);
      const bool good = step != 0.0f && isfinite(step);
      const float inv = good ? __frcp_rn(step) : 0.0f;
      const float fn = (float)n_out;
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        const int i = 32 * g + r;
        float qf = 0.0f;
        if (good) {
          const float tq = __fmul_rn(y[r], inv);
          if constexpr (MODE == BRS_ROUND_STOCHASTIC) {
            const uint32_t e = (uint32_t)(i * D + j);
            const uint4 rnd = philox4x32_10(make_uint4(e / 4, (uint32_t)a.step, (uint32_t)h, (uint32_t)b),
                                            make_uint2((uint32_t)a.seed, (uint32_t)(a.seed >> 32)));
            const uint32_t wd = (e & 3u) == 0 ? rnd.x : (e & 3u) == 1 ? rnd.y : (e & 3u) == 2 ? rnd.z : rnd.w;
            qf = sr_round(tq, wd >> 8);
          } else {
            qf = rintf(tq);
          }
          qf = fminf(fmaxf(qf, -fn), fn);
          if (qf != qf) qf = 0.0f;
        }
        if constexpr (MODE == BRS_ROUND_ERRFEEDBACK) {
          float e = __fsub_rn(y[r], good ? __fmul_rn(step, qf) : 0.0f);
          const float lim = good ? step : 0.0f;
          if (e > lim) e = lim;
          else if (e < -lim) e = -lim;
          auxh[(size_t)i * D + j] = f32_to_f16(e);
        }
        const uint32_t code = (uint32_t)((int)qf + n_out);
        // the warp's segment of row i: bits (i D + 32 w) bw_out
        vh_store_segment(wout + (size_t)(i * (D / 32) + (j >> 5)) * bw_out, code, bw_out, lane);
      }
    }
  }

  if constexpr (PHASE == 0) {
    float o[1];
    otree.result(o);
    if (!isfinite(o[0])) raise_flag(a.flags, BRS_FLAG_NONFINITE);
    a.o[(size_t)head * D + j] = o[0];
    // ---- statistics (thread t: row t) and the head's cost, the mean of
    // its rows' decay weights (R~ = 1), rows summed in order in FP64
    const VhRow rr = rows[t];
    const double av = (double)rr.a, be = (double)beta, kd = (double)rr.k;
    const double a2 = av * av, kk = (be * (2.0 - be)) * (kd * kd);
    double* st = a.stats + ((size_t)head * D + t) * 2;
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
    double gm;
    if (a.persistence == 0) {                      // erasure rate Gamma_hat
      double arg = 2.0 * (s_hat + 0.5 * K);
      if (!(arg >= 1e-9)) arg = 1e-9;
      gm = 1.0 / ((double)a.C * expm1(arg));
    } else {                                       // w^(1), h^(C)
      double arg = 2.0 * s_hat * (double)(a.persistence == 2 ? a.C : 1);
      if (!(arg >= 1e-9)) arg = 1e-9;
      gm = 1.0 / -expm1(-arg);
    }
    gam[t] = gm;
    __syncthreads();
    if (t == 0) {
      double sum = 0.0;
      for (int i = 0; i < D; ++i) sum += gam[i];
      a.cost[head] = sum / (double)D;
    }
  }
}

template <int PHASE>
cudaError_t launch_vh_phase(const VbArgs& a, cudaStream_t st) {
  const dim3 grid(a.B * a.H), block(32 * kVhWarps);
  switch (a.mode) {
    case BRS_ROUND_NEAREST: varbit_head_kernel<PHASE, BRS_ROUND_NEAREST><<<grid, block, 0, st>>>(a); break;
    case BRS_ROUND_STOCHASTIC: varbit_head_kernel<PHASE, BRS_ROUND_STOCHASTIC><<<grid, block, 0, st>>>(a); break;
    case BRS_ROUND_ERRFEEDBACK: varbit_head_kernel<PHASE, BRS_ROUND_ERRFEEDBACK><<<grid, block, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// ---- state conversion: widths and head offsets of every sequence (one
// thread per sequence), checked against the payload's budget first
__global__ void vh_layout_kernel(const VbPackArgs a) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= a.B) return;
  uint8_t* packed = (uint8_t*)a.packed;
  uint8_t* wd = packed + a.sec.off_width + (size_t)b * a.H;
  uint32_t* of = (uint32_t*)(packed + a.sec.off_offsets) + (size_t)b * (a.H + 1);
  const int uni = (int)rint(a.avg_bits);
  uint32_t tot = 0;
  bool bad = false;
  for (int h = 0; h < a.H; ++h) {
    const int bw = a.widths ? a.widths[(size_t)b * a.H + h] : uni;
    bad |= bw < 1 || bw > 16;
    tot += (uint32_t)bw;
  }
  // a width map off the budget would place heads past the payload: the
  // sequence gets width 0 everywhere (the pack kernel then writes nothing)
  bad |= (double)tot != a.avg_bits * (double)a.H;
  if (bad) raise_flag(a.flags, BRS_FLAG_INVALID);
  uint32_t off = 0;
  for (int h = 0; h < a.H; ++h) {
    const int bw = bad ? 0 : (a.widths ? a.widths[(size_t)b * a.H + h] : uni);
    wd[h] = (uint8_t)bw;
    of[h] = off;
    off += (uint32_t)(kVhD * kVhD / 8) * (uint32_t)bw;
  }
  of[a.H] = off;
}

// one CTA per head, one thread per column: nearest rounding of each scale
// group with its fitted step
__global__ void __launch_bounds__(kVhD) vh_pack_kernel(const VbPackArgs a) {
  constexpr int D = kVhD;
  const int head = blockIdx.x, j = threadIdx.x, lane = j % 32;
  const int b = head / a.H, h = head - b * a.H;
  uint8_t* packed = (uint8_t*)a.packed;
  const int bw = packed[a.sec.off_width + head];
  if (bw == 0) return;                               // rejected width map
  const uint32_t off = ((const uint32_t*)(packed + a.sec.off_offsets))[(size_t)b * (a.H + 1) + h];
  uint32_t* wout = (uint32_t*)(packed + (size_t)b * a.sec.payload_per_seq + off);
  uint16_t* sc = (uint16_t*)(packed + a.sec.off_scale) + (size_t)head * kVhBlocks * D;
  const float* S = a.S + (size_t)head * D * D;
  const int n = (1 << (bw - 1)) - 1;
  const float fn = (float)n;
  for (int g = 0; g < kVhBlocks; ++g) {
    float y[32];
#pragma unroll
    for (int r = 0; r < 32; ++r) y[r] = S[(size_t)(32 * g + r) * D + j];
    bool bad;
    const uint16_t sb = vh_fit(y, n, a.one, &bad);
    if (bad) raise_flag(a.flags, BRS_FLAG_OVERFLOW);
    sc[g * D + j] = sb;
    const float step = f16_to_f32(sb);
    const bool good = step != 0.0f && isfinite(step);
    const float inv = good ? __frcp_rn(step) : 0.0f;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      float qf = good ? fminf(fmaxf(rintf(__fmul_rn(y[r], inv)), -fn), fn) : 0.0f;
      if (qf != qf) qf = 0.0f;
      const int i = 32 * g + r;
      vh_store_segment(wout + (size_t)(i * (D / 32) + (j >> 5)) * bw, (uint32_t)((int)qf + n), bw, lane);
    }
  }
}

__global__ void __launch_bounds__(kVhD) vh_unpack_kernel(const VbPackArgs a, const void* packed_v, float* S) {
  constexpr int D = kVhD;
  const int head = blockIdx.x, j = threadIdx.x;
  const int b = head / a.H, h = head - b * a.H;
  const uint8_t* packed = (const uint8_t*)packed_v;
  const int bw = packed[a.sec.off_width + head];
  const uint32_t off = ((const uint32_t*)(packed + a.sec.off_offsets))[(size_t)b * (a.H + 1) + h];
  const uint32_t* win = (const uint32_t*)(packed + (size_t)b * a.sec.payload_per_seq + off);
  const uint16_t* sc = (const uint16_t*)(packed + a.sec.off_scale) + (size_t)head * kVhBlocks * D;
  float* dst = S + (size_t)head * D * D;
  if (bw < 1 || bw > 16) {
    for (int i = 0; i < D; ++i) dst[(size_t)i * D + j] = 0.0f;
    return;
  }
  const int n = (1 << (bw - 1)) - 1;
  const uint32_t mask = (1u << bw) - 1u;
  for (int i = 0; i < D; ++i) {
    const uint32_t u = vh_code(win, (uint32_t)(i * D + j) * (uint32_t)bw, bw, mask);
    dst[(size_t)i * D + j] = __fmul_rn((float)((int)u - n), f16_to_f32(sc[(i >> 5) * D + j]));
  }
}

}  // namespace

VbSections varbit_head_sections(int B, int H, int d, double avg_bits) {
  VbSections s;
  const size_t Bz = (size_t)B, Hz = (size_t)H, dz = (size_t)d;
  s.payload_per_seq = (size_t)((double)(dz * dz / 8) * avg_bits * (double)Hz);
  s.off_scale = vh_r256(s.payload_per_seq * Bz);
  s.off_width = s.off_scale + vh_r256(Bz * Hz * (dz / 32) * dz * 2);
  s.off_offsets = s.off_width + vh_r256(Bz * Hz);
  s.total = s.off_offsets + vh_r256(Bz * (Hz + 1) * 4);
  return s;
}

cudaError_t launch_varbit_head_decode(const VbArgs& a, cudaStream_t st) {
  cudaError_t e = launch_vh_phase<0>(a, st);
  if (e != cudaSuccess) return e;
  AllocArgs al{};
  al.groups = a.B;
  al.rows_per_group = a.H;
  al.b_min = a.b_min;
  al.b_max = a.b_max;
  al.avg_bits = a.avg_bits;
  al.offset_unit = kVhD * kVhD / 8;
  al.cost = a.cost;
  uint8_t* pout = (uint8_t*)a.packed_out;
  al.bits = pout + a.sec.off_width;
  al.offsets = (uint32_t*)(pout + a.sec.off_offsets);
  e = launch_allocate(al, st);
  if (e != cudaSuccess) return e;
  return launch_vh_phase<1>(a, st);
}

cudaError_t launch_varbit_head_pack(const VbPackArgs& a, cudaStream_t st) {
  vh_layout_kernel<<<(a.B + 63) / 64, 64, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  vh_pack_kernel<<<a.B * a.H, kVhD, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_varbit_head_unpack(const VbPackArgs& a, const void* packed, float* S, cudaStream_t st) {
  vh_unpack_kernel<<<a.B * a.H, kVhD, 0, st>>>(a, packed, S);
  return cudaGetLastError();
}

}  // namespace brs
