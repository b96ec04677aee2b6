// Decay-aware width allocation on the GPU ("Low-Bit Recurrent States in
// Hybrid Language Models", State bit allocation; the explainer's worked
// example): minimise sum c_i 2^(-2 b_i) at a fixed mean width.
//
// One CTA per group of rows (a layer's H*d rows, or one head's d rows), in
// FP64:
//   b*_i = avg + log2(c_i / GM(c)) / 2, GM over the rows with c_i > 0;
//   b_i  = clamp(round-to-nearest-even(b*_i), b_min, b_max); b_min for
//          c_i = 0; round(avg) for every row when all c_i are 0;
//   then the total is brought to avg * N one bit at a time in the order
//   of the greedy rule: over budget, take bits where the cost rises least
//   (3 c_i 4^(-b_i)); under budget, give bits where it falls most
//   (3/4 c_i 4^(-b_i)); ties to the lower row.
// The greedy's sequence of moves equals taking the E cheapest (value, row)
// candidates, because a row's successive candidates only grow (or shrink)
// by 4x; the kernel finds them with a radix select over the candidates'
// FP64 bit patterns (non-negative, so bit order is numeric order).
#include <cuda_runtime.h>

#include <cstdint>

#include "brs_device.cuh"
#include "brs_internal.h"

namespace brs {

constexpr int kAllocThreads = 512;
constexpr int kMaxRowsPerThread = 16;      // groups up to 8192 rows

struct AllocShared {
  double dsum[kAllocThreads / 32];
  int isum[kAllocThreads / 32];
  unsigned hist[256];
  unsigned long long prefix;               // radix-select state
  int rank;                                // candidates still to take below the prefix
  int uniq;                                // the selected digit holds one candidate
  double gm;
  int all_zero;
  long long total;
};

// deterministic block sums: per-thread partials, then warps in order
__device__ double block_sum_d(double v, AllocShared& sh) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  __syncthreads();
  if (lane == 0) sh.dsum[warp] = v;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < kAllocThreads / 32; ++w) t += sh.dsum[w];
  return t;
}

__device__ long long block_sum_i(long long v, AllocShared& sh) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  __syncthreads();
  if (lane == 0) sh.isum[warp] = (int)v;
  __syncthreads();
  long long t = 0;
  for (int w = 0; w < kAllocThreads / 32; ++w) t += sh.isum[w];
  return t;
}

// exclusive prefix over threads of a per-thread count (thread order = row order)
__device__ long long block_exclusive_scan(long long v, AllocShared& sh, long long* total) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  long long x = v;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, m);
    if (lane >= m) x += y;
  }
  __syncthreads();
  if (lane == 31) sh.isum[warp] = (int)x;
  __syncthreads();
  long long before = 0, all = 0;
  for (int w = 0; w < kAllocThreads / 32; ++w) {
    if (w < warp) before += sh.isum[w];
    all += sh.isum[w];
  }
  *total = all;
  return before + x - v;
}

// candidate value of (row, level L) as ordered bits: decrements take levels
// b, b-1, ..., b_min+1 with cost (3c) 4^-L; increments take levels b, b+1,
// ..., b_max-1 with gain (3/4 c) 4^-L, ordered descending (complemented
// bits).  p is the row's product 3c or 0.75c; scaling it by 4^-L only lowers
// the exponent field by 2L while the result stays normal, so the key is p's
// bit pattern minus 2L << 52 (exact, the same double as p * 4^-L); a zero,
// subnormal or underflowing result takes the multiplication itself.
__device__ __forceinline__ unsigned long long cand_key(double p, int level, bool dec) {
  const unsigned long long pb = (unsigned long long)__double_as_longlong(p);
  const int ex = (int)((pb >> 52) & 0x7ffu);
  const unsigned long long k = (ex > 2 * level && ex < 0x7ff) ? pb - ((unsigned long long)(2 * level) << 52)
                                                              : (unsigned long long)__double_as_longlong(p * ldexp(1.0, -2 * level));
  return dec ? k : ~k;
}

// RPT rows per thread at most (8 for groups up to 4096 rows: fewer registers)
template <int RPT>
__global__ void __launch_bounds__(kAllocThreads) allocate_kernel(const AllocArgs a) {
  __shared__ AllocShared sh;
  const int t = threadIdx.x;
  const int N = a.rows_per_group;
  const int g = blockIdx.x;
  const double* c = a.cost + (size_t)g * N;
  const int rpt = (N + kAllocThreads - 1) / kAllocThreads;   // rows per thread, contiguous
  const int r0 = t * rpt;
  double cv[RPT];
  int bv[RPT];
#pragma unroll
  for (int q = 0; q < RPT; ++q) {
    cv[q] = 0.0;
    bv[q] = 0;
    if (q < rpt && r0 + q < N) cv[q] = c[r0 + q];
  }
  // ---- geometric mean over the rows with c > 0
  double ls = 0.0;
  int cnt = 0;
#pragma unroll
  for (int q = 0; q < RPT; ++q)
    if (q < rpt && r0 + q < N && cv[q] > 0.0) {
      ls += log(cv[q]);
      ++cnt;
    }
  const double sumlog = block_sum_d(ls, sh);
  const long long ncnt = block_sum_i(cnt, sh);
  const double gm = ncnt ? exp(sumlog / (double)ncnt) : 0.0;
  // ---- rounded, clipped widths
  long long mysum = 0;
#pragma unroll
  for (int q = 0; q < RPT; ++q) {
    if (q < rpt && r0 + q < N) {
      int b;
      if (ncnt == 0) {
        b = (int)rint(a.avg_bits);
      } else if (cv[q] > 0.0) {
        double br = rint(a.avg_bits + 0.5 * log2(cv[q] / gm));
        br = fmin(fmax(br, (double)a.b_min), (double)a.b_max);
        b = (int)br;
      } else {
        b = a.b_min;
      }
      b = min(max(b, a.b_min), a.b_max);
      bv[q] = b;
      mysum += b;
    }
  }
  const long long target = (long long)(a.avg_bits * (double)N);
  const long long sum = block_sum_i(mysum, sh);
  const long long E = sum - target;
  if (E != 0) {
    const bool dec = E > 0;
    const long long need = dec ? E : -E;
    // ---- radix select: the need-th smallest candidate key, 8 bits at a time
    if (t == 0) { sh.prefix = 0ull; sh.rank = (int)need; sh.uniq = 0; }
    __syncthreads();
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int i = t; i < 256; i += kAllocThreads) sh.hist[i] = 0u;
      __syncthreads();
      const unsigned long long pre = sh.prefix;
      const unsigned long long hmask = (shift == 56) ? 0ull : (~0ull << (shift + 8));
      // a thread's candidates come in runs with the same digit (a row's
      // levels differ by a factor of 4): count a run, add it once
      unsigned run_digit = 0xffffffffu, run_n = 0;
#pragma unroll
      for (int q = 0; q < RPT; ++q) {
        if (q < rpt && r0 + q < N) {
          const int lo = dec ? a.b_min + 1 : bv[q], hi = dec ? bv[q] : a.b_max - 1;
          const double pq = dec ? 3.0 * cv[q] : 0.75 * cv[q];
          for (int L = lo; L <= hi; ++L) {
            const unsigned long long k = cand_key(pq, L, dec);
            if ((k & hmask) == (pre & hmask)) {
              const unsigned dg = (unsigned)((k >> shift) & 0xffu);
              if (dg != run_digit) {
                if (run_n) atomicAdd(&sh.hist[run_digit], run_n);
                run_digit = dg;
                run_n = 0;
              }
              ++run_n;
            }
          }
        }
      }
      if (run_n) atomicAdd(&sh.hist[run_digit], run_n);
      __syncthreads();
      if (t < 32) {
        // the digit holding the rank-th candidate: lane l scans digits
        // 8l .. 8l+7 after an exclusive prefix of the lanes' totals
        const int lane = t;
        unsigned cnt[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) { cnt[e] = sh.hist[8 * lane + e]; tot += cnt[e]; }
        unsigned incl = tot;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
          const unsigned y = __shfl_up_sync(0xffffffffu, incl, m);
          if (lane >= m) incl += y;
        }
        const int r = sh.rank;
        const unsigned before = incl - tot;
        if ((int)before < r && r <= (int)incl) {
          int rr = r - (int)before;
          unsigned digit = 8 * lane, dcnt = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (rr <= (int)cnt[e]) { digit = 8 * lane + e; dcnt = cnt[e]; break; }
            rr -= (int)cnt[e];
          }
          sh.prefix = pre | ((unsigned long long)digit << shift);
          sh.rank = rr;
          sh.uniq = dcnt == 1u;
        }
      }
      __syncthreads();
      if (sh.uniq && shift > 0) {
        // one candidate carries the selected prefix: its key is the answer,
        // found in one pass instead of the remaining digit passes
        const unsigned long long pre2 = sh.prefix, m2 = ~0ull << shift;
#pragma unroll
        for (int q = 0; q < RPT; ++q) {
          if (q < rpt && r0 + q < N) {
            const int lo = dec ? a.b_min + 1 : bv[q], hi = dec ? bv[q] : a.b_max - 1;
            const double pq = dec ? 3.0 * cv[q] : 0.75 * cv[q];
            for (int L = lo; L <= hi; ++L) {
              const unsigned long long k = cand_key(pq, L, dec);
              if ((k & m2) == pre2) sh.prefix = k;
            }
          }
        }
        __syncthreads();
        break;
      }
    }
    const unsigned long long tau = sh.prefix;   // key of the need-th candidate
    // every candidate below tau is taken; among those equal to tau, the
    // first (need - #below) in row order
    long long below = 0, myeq = 0;
    int eq[RPT];
#pragma unroll
    for (int q = 0; q < RPT; ++q) {
      eq[q] = 0;
      if (q < rpt && r0 + q < N) {
        const int lo = dec ? a.b_min + 1 : bv[q], hi = dec ? bv[q] : a.b_max - 1;
        const double pq = dec ? 3.0 * cv[q] : 0.75 * cv[q];
        for (int L = lo; L <= hi; ++L) {
          const unsigned long long k = cand_key(pq, L, dec);
          if (k < tau) ++below;
          else if (k == tau) ++eq[q];
        }
        myeq += eq[q];
      }
    }
    const long long nbelow = block_sum_i(below, sh);
    long long eqtot = 0;
    long long eqbefore = block_exclusive_scan(myeq, sh, &eqtot);
    long long rem = need - nbelow;                // taken among the ties
#pragma unroll
    for (int q = 0; q < RPT; ++q) {
      if (q < rpt && r0 + q < N) {
        const int lo = dec ? a.b_min + 1 : bv[q], hi = dec ? bv[q] : a.b_max - 1;
        long long take = 0;
        const double pq = dec ? 3.0 * cv[q] : 0.75 * cv[q];
        for (int L = lo; L <= hi; ++L)
          if (cand_key(pq, L, dec) < tau) ++take;
        long long tie = rem - eqbefore;
        tie = tie < 0 ? 0 : (tie > (long long)eq[q] ? (long long)eq[q] : tie);
        eqbefore += eq[q];
        take += tie;
        bv[q] += dec ? -(int)take : (int)take;
      }
    }
  }
  // ---- widths and prefix offsets
  long long mybits = 0;
#pragma unroll
  for (int q = 0; q < RPT; ++q)
    if (q < rpt && r0 + q < N) {
      a.bits[(size_t)g * N + r0 + q] = (uint8_t)bv[q];
      mybits += bv[q];
    }
  long long tot = 0;
  long long off = block_exclusive_scan(mybits, sh, &tot);
  if (a.offsets) {
    uint32_t* of = a.offsets + (size_t)g * (N + 1);
#pragma unroll
    for (int q = 0; q < RPT; ++q)
      if (q < rpt && r0 + q < N) {
        of[r0 + q] = (uint32_t)(off * a.offset_unit);
        off += bv[q];
      }
    if (t == kAllocThreads - 1) of[N] = (uint32_t)(tot * a.offset_unit);
  }
}

cudaError_t launch_allocate(const AllocArgs& a, cudaStream_t st) {
  if (a.rows_per_group <= kAllocThreads * 8)
    allocate_kernel<8><<<a.groups, kAllocThreads, 0, st>>>(a);
  else
    allocate_kernel<kMaxRowsPerThread><<<a.groups, kAllocThreads, 0, st>>>(a);
  return cudaGetLastError();
}

int allocate_max_rows() { return kAllocThreads * kMaxRowsPerThread; }

}  // namespace brs
