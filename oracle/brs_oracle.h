/*
 * Plain CPU oracle for the fused recurrent-state update with quantized
 * write-back.  TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and
 * the benchmark's CPU-baseline leg may load it; the product path never does.
 * It shares no source with the CUDA library (its own structs, its own byte
 * offsets, its own binary16 and Philox code).
 *
 * Sources, cited by page title and section:
 *   [WB]   "When Quantization Breaks Memory: Recurrent-State Write-Back in
 *          Low-Precision Temporal Inference" (English summary and the
 *          Chinese-language summary of the same paper)
 *   [LB]   "Low-Bit Recurrent States in Hybrid Language Models"
 *   [LBX]  "Allocate low-bit recurrent state precision by channel decay"
 *          (explainer of [LB])
 *   [DAMP] summary of "DAMP: Decay-Aware Mixed-Precision recurrent-state
 *          quantization" (arXiv 2608.27513)
 *
 * Parity status of each function is stated beside it in brs_oracle.c.
 */
#ifndef BRS_ORACLE_H
#define BRS_ORACLE_H
#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_STORE_FP32 = 0, ORC_STORE_DAMP = 1, ORC_STORE_VARBIT = 2, ORC_STORE_VARBIT_HEAD = 3 };
enum { ORC_ROUND_NEAREST = 0, ORC_ROUND_STOCHASTIC = 1, ORC_ROUND_ERRFEEDBACK = 2, ORC_ROUND_DIRECTION = 3,
       ORC_ROUND_RESIDUAL2 = 4, ORC_ROUND_RESIDUAL3 = 5, ORC_ROUND_RESIDUAL4 = 6 };
enum { ORC_DOMAIN_CANONICAL = 0, ORC_DOMAIN_ROTATED = 1, ORC_DOMAIN_MIXED = 2 };

/* status flags (OR-ed) */
enum { ORC_OK = 0, ORC_EINVAL = 1, ORC_ENONFINITE = 2, ORC_EOVERFLOW = 4 };

typedef struct {
  int B, H, Hk, d;      /* batch, value heads, key heads, d_k = d_v = d      */
  int storage;          /* ORC_STORE_*                                        */
  int k_hi;             /* protected FP16 rows per head (DAMP)                */
  int block;            /* INT8 block length along the value axis (DAMP)      */
  int hadamard;         /* 1: INT8 rows stored after a d-point Hadamard       */
  int decay_per_key;    /* 1: KDA, decay per key channel; 0: GDN, per head    */
  double avg_bits;      /* VARBIT mean width (layer budget)                   */
  int b_min, b_max;     /* VARBIT width limits                                */
  int budget_scope;     /* VARBIT: 1 layer (all H*d rows of a sequence), 0 head */
  int domain;           /* ORC_DOMAIN_*: where the FP32 update is computed    */
  int persistence;      /* VARBIT cost weight: 0 erasure rate Gamma_hat, 1 w^(1), 2 h^(C) */
  int low_bits;         /* DAMP low tier: 8 (also 0) or 4 bits per code       */
} orc_layout;

/* persistence weight of a row from A = EMA(a^2), K = EMA(beta (2-beta) k^2) */
double orc_persistence(int kind, double A, double K, int C);

typedef struct {
  int mode;             /* ORC_ROUND_*                                        */
  uint64_t seed;        /* Philox key for stochastic rounding                 */
  int C;                /* write-back interval in tokens                      */
} orc_writeback;

/* ---- scalar building blocks (exported so the tests can pin them) ---- */
uint16_t orc_f16_from_f32(float f);
float    orc_f32_from_f16(uint16_t h);
float    orc_f32_from_bf16(uint16_t b);
void     orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
void     orc_fwht(float* x, int n);
float    orc_hadamard_scale(int n);

/* One INT8 asymmetric block (DAMP low tier).  y: target values (already in
 * the quantized domain, error-feedback residual NOT yet added); e_inout: FP16
 * residuals (mode ERRFEEDBACK) or NULL.  step/h/b/elem0 feed the Philox
 * counter of stochastic rounding (elem0 = index of y[0] within the head's
 * row-major storage).  t_out (optional) receives the pre-rounding grid
 * coordinate of every value.  Returns ORC_* flags. */
int orc_int8_block(const float* y, int n, int mode, uint64_t seed, int64_t step, int h, int b,
                   int elem0, uint16_t* e_inout, uint8_t* codes, uint16_t* scale_h,
                   uint16_t* zero_h, float* t_out);

/* The same asymmetric block with `levels` + 1 codes (255: INT8, 15: INT4):
 * scale = fp16((max - min) / levels), codes clipped to [0, levels]. */
int orc_lowbit_block(const float* y, int n, int levels, int mode, uint64_t seed, int64_t step, int h,
                     int b, int elem0, uint16_t* e_inout, uint8_t* codes, uint16_t* scale_h,
                     uint16_t* zero_h, float* t_out);

/* The INT8 block under direction memory: nearest codes of y on the block's
 * grid, then 2-bit sign counters m_inout (values -1, 0, 1) take a vote from
 * each proposed change y - xprev inside (scale/8, scale/2); a counter that
 * reaches +-2 moves its code one level (clipped to [0, 255]) and is reset. */
int orc_int8_block_dm(const float* y, const float* xprev, int n, int8_t* m_inout, uint8_t* codes,
                      uint16_t* scale_h, uint16_t* zero_h, float* t_out);

/* The INT8 block under k-bit residual memory (k = 2, 3, 4): error feedback
 * whose residual is kept as a k-bit signed integer m (|m| <= 2^(k-1) - 1) in
 * units of step/2^k.  e_prev = m * (sprev / 2^k) with sprev the block's step
 * when m was stored (0 when sprev is 0); the target y + e_prev is quantized
 * with nearest rounding; the new m = clamp(rne((y + e_prev - value) *
 * (1/scale) * 2^k)) with the new block's scale (0 when the scale is 0). */
int orc_int8_block_rm(const float* y, int n, int kbits, float sprev, int8_t* m_inout, uint8_t* codes,
                      uint16_t* scale_h, uint16_t* zero_h, float* t_out);

/* One variable-width row (decay-aware allocation tier), width bw in [1, 16]. */
int orc_varbit_row(const float* x, int n, int bw, int mode, uint64_t seed, int64_t step, int h,
                   int b, int elem0, uint16_t* e_inout, int32_t* q_out, uint16_t* delta_h,
                   int* m_star, float* t_out);

/* One scale group of the same quantizer whose elements sit estride apart in
 * the head (element j of the group is element elem0 + j * estride of the
 * head for the stochastic-rounding counters); x, e_inout, q_out and t_out
 * hold the group contiguously.  orc_varbit_row is the case estride = 1. */
int orc_varbit_group(const float* x, int n, int bw, int mode, uint64_t seed, int64_t step, int h,
                     int b, int elem0, int estride, uint16_t* e_inout, int32_t* q_out,
                     uint16_t* delta_h, int* m_star, float* t_out);

/* Approximate erasure-rate persistence weight, rho = 1. */
double orc_gamma_hat(double A, double K, int C);

/* Width allocation (FP64).  Returns ORC_* flags; bits[i] in [b_min, b_max]
 * with sum(bits) == avg_bits * N. */
int orc_allocate_bits(int N, const double* c, double avg_bits, int b_min, int b_max,
                      uint8_t* bits);

/* ---- storage accounting ---- */
size_t orc_state_bytes(const orc_layout* L, size_t* aux_bytes, size_t* stats_bytes);
double orc_bits_per_value(const orc_layout* L);

/* ---- state conversion (deterministic rounding) ---- */
int orc_state_pack(const orc_layout* L, const float* S, const int16_t* perm,
                   const uint8_t* widths, void* packed);
int orc_state_unpack(const orc_layout* L, const void* packed, const int16_t* perm, float* S);

/* ---- the recurrence ----
 * Runs tokens [step0, step0 + T) for units [u0, u1): a unit is one
 * (sequence, head) pair b*H+h for FP32/DAMP storage and one sequence b for
 * VARBIT storage (its width budget spans the sequence's heads).
 * Inputs are token-major: q,k [T][B][Hk][d] bf16 bits; v [T][B][H][d] bf16
 * bits; beta [T][B][H]; decay [T][B][H][d] (KDA) or [T][B][H] (GDN), holding
 * a = exp(-s).  o [T][B][H][d].  packed_in may equal packed_out.  aux: FP16
 * error-feedback residuals, stats: FP64 EMA statistics (VARBIT).
 * t_dump (optional): pre-rounding grid coordinate of every stored code of
 * the LAST write-back, laid out like the codes.  s_dump (optional,
 * FP32/DAMP storage): the FP32 state just before the LAST write-back,
 * [B][H][d][d] in stored row order, in the working basis of the mode.
 * Write-back happens after
 * every token whose global index t satisfies (t + 1) % C == 0; step0 and T
 * must be multiples of C.  Returns ORC_* flags. */
int orc_run(const orc_layout* L, const orc_writeback* wb, int64_t step0, int T, int u0, int u1,
            const void* packed_in, void* packed_out, void* aux, double* stats,
            const int16_t* perm, const uint16_t* q, const uint16_t* k, const uint16_t* v,
            const float* beta, const float* decay, float* o, float* t_dump, float* s_dump);

/* One write-back (quantizer only) of the FP32 states of units [u0, u1)
 * (S [B][H][d][d], stored row order, the domain's working basis) at token
 * `step` into DAMP storage `packed`, residuals / counters in aux. */
int orc_damp_writeback(const orc_layout* L, const orc_writeback* wb, int64_t step, int u0, int u1,
                       const float* S, void* packed, void* aux);

/* Protected-row selection by the DAMP risk score on a calibration run.
 * Inputs as orc_run for Bc sequences and T tokens (FP32 recurrence from a
 * zero state, identity order); the state is sampled every `every` tokens.
 * score_out [H][d] (optional), perm_out [H][d]. */
int orc_calibrate(const orc_layout* L, int Bc, int T, int every, double tau,
                  const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* beta,
                  const float* decay, double* score_out, int16_t* perm_out);

#ifdef __cplusplus
}
#endif
#endif
