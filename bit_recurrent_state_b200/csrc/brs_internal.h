// Internal launch interfaces between the host ABI (brs_api.cu) and the
// kernels.  Not part of the public ABI.
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "brs.h"

namespace brs {

struct DecodeArgs {
  int B, H, Hk, k_hi, block, decay_per_key, mode;
  uint64_t seed;
  int64_t step;
  size_t head_bytes;
  float hscale;                  // float nearest 1/sqrt(d)
  float one = 1.0f;              // 1 read at run time: a multiplier the compiler cannot fold
  const void* packed_in;
  void* packed_out;
  void* aux;
  const int16_t* perm;
  const uint16_t *q, *k, *v;
  const float *beta, *decay;
  float* o;
  uint32_t* flags;
  // deferred write-back (DAMP): the FP32 state between write-backs,
  // [B*H][d][d] in stored row order and the tiers' own bases; src32 reads the
  // rows from it instead of the stored state, dst32 writes the updated rows
  // to it instead of the write-back
  float* s32 = nullptr;
  int src32 = 0, dst32 = 0;
  // test hook (brs_test_starve_copies): bytes a head's copy barrier expects
  // beyond what its copies deliver (0 in normal use)
  uint32_t tx_extra = 0;
  int low_bits = 8;              // DAMP low tier: 8 (INT8) or 4 (two codes per byte)
};

// the host thread's test-hook setting (brs_test_starve_copies)
uint32_t starve_tx_bytes();

cudaError_t launch_decode(const DecodeArgs& a, int d, int store, bool had, cudaStream_t st);
// the general (warp-per-head) kernel for every shape it supports, with the
// interval-state flags honoured (DAMP storage)
cudaError_t launch_decode_deferred(const DecodeArgs& a, int d, bool had, cudaStream_t st);
bool decode_supported(int d, int block, int k_hi);

struct CalibArgs {
  int B, H, d, block, hadamard, k_hi, T, nsamp, sample, decay_per_key;
  float levels;                  // top code of the low tier: 255 (INT8) or 15 (INT4)
  float hscale;
  double tau;
  const float* S;                // [B][H][d][d] FP32 calibration states
  double* err;                   // [nsamp][B][H][d] per-sample error energies
  const float* decay;            // [T][B][H][d] or [T][B][H]
  double* score;                 // [H][d]
  int16_t* perm;                 // [H][d]
  uint32_t* flags;
};
cudaError_t launch_calib_sample(const CalibArgs& a, cudaStream_t st);
cudaError_t launch_calib_finish(const CalibArgs& a, cudaStream_t st);
// d = 128 DAMP decode, one CTA per head with the state in registers
// (persistent CTAs, bulk-copy staging of each head's stored bytes)
bool decode_cta_supported(int d, int store, int block, int k_hi, int mode);
cudaError_t launch_decode_cta(const DecodeArgs& a, bool had, cudaStream_t st);

struct PackArgs {
  int B, H, d, storage, k_hi, block, hadamard;
  int low_bits;                  // DAMP low tier: 8 or 4
  size_t head_bytes;
  float hscale;
  const float* S;                // [B][H][d][d] key-channel order
  const int16_t* perm;
  void* packed;
  uint32_t* flags;
};

cudaError_t launch_pack(const PackArgs& a, cudaStream_t st);
cudaError_t launch_unpack(const PackArgs& a, float* S_out, const void* packed, cudaStream_t st);

// Sections of a variable-width stored state (see the header's layout).
struct VbSections {
  size_t payload_per_seq, off_scale, off_width, off_offsets, total;
};
VbSections varbit_sections(int B, int H, int d, double avg_bits);

struct VbPackArgs {
  int B, H, d;
  double avg_bits;
  float one = 1.0f;              // 1 read at run time: a multiplier the compiler cannot fold
  VbSections sec;
  const float* S;                // [B][H][d][d]
  const uint8_t* widths;         // [B][H*d] or null (avg_bits everywhere)
  void* packed;
  uint32_t* flags;
};
cudaError_t launch_varbit_pack(const VbPackArgs& a, cudaStream_t st);
cudaError_t launch_varbit_unpack(const VbPackArgs& a, const void* packed, float* S, cudaStream_t st);

struct VbArgs {
  int B, H, Hk, decay_per_key, mode, first, C, b_min, b_max, budget_scope, persistence;
  uint64_t seed;
  int64_t step;
  double lambda, avg_bits;
  float one = 1.0f;              // 1 read at run time: a multiplier the compiler cannot fold
  VbSections sec;
  const void* packed_in;
  void* packed_out;
  void* aux;
  double* stats;
  double* cost;                  // workspace: one FP64 cost per row
  const uint16_t *q, *k, *v;
  const float *beta, *decay;
  float* o;
  uint32_t* flags;
};
cudaError_t launch_varbit_decode(const VbArgs& a, cudaStream_t st);
cudaError_t launch_varbit_offsets(const VbArgs& a, cudaStream_t st);

// per-head widths (one width per head, steps per block of 32 key channels)
VbSections varbit_head_sections(int B, int H, int d, double avg_bits);
cudaError_t launch_varbit_head_decode(const VbArgs& a, cudaStream_t st);
cudaError_t launch_varbit_head_pack(const VbPackArgs& a, cudaStream_t st);
cudaError_t launch_varbit_head_unpack(const VbPackArgs& a, const void* packed, float* S, cudaStream_t st);

struct PrefillArgs {
  int B, H, Hk, T, k_hi, block, decay_per_key, mode;
  int low_bits = 8;              // DAMP low tier: 8 or 4
  uint64_t seed;
  int64_t step0;
  size_t head_bytes;
  float hscale;
  void* packed;                  // updated in place
  void* aux;
  const int16_t* perm;
  const uint16_t *q, *k, *v;     // [B][T][Hk|H][d]
  const float *beta, *decay;     // [B][T][H], [B][T][H][d] or [B][T][H]
  float* o;                      // [B][T][H][d]
  float* sdump;                  // optional [B][H][d][d]
  uint32_t* flags;
  float* s0;                     // scratch [B][H][d][d]: the FP32 state between chunks
  uint32_t* handover;            // [B*H] chunks finished by the CTA that hands a head over (zeroed per call)
  int skip_handover = 0;         // test hook (brs_test_prefill_withhold): producers publish nothing
};
size_t prefill_tc_scratch_bytes(int B, int H);
// the host thread's test-hook setting (brs_test_prefill_ctas): a cap on the
// prefill's CTAs (0: one per SM), so that small batches exercise hand-overs
int prefill_cta_cap();
int prefill_withhold();
cudaError_t launch_prefill_tc(const PrefillArgs& a, bool had, cudaStream_t st);
bool prefill_supported(int d, int block, int k_hi, int C);

struct AllocArgs {
  int groups, rows_per_group, b_min, b_max;
  double avg_bits;
  uint32_t offset_unit;
  const double* cost;
  uint8_t* bits;
  uint32_t* offsets;
};

cudaError_t launch_allocate(const AllocArgs& a, cudaStream_t st);
int allocate_max_rows();

void set_last_error(const char* msg);

}  // namespace brs
