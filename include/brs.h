/*
 * brs.h -- C ABI of the B200 (sm_100a) library for the fused recurrent-state
 * update with quantized write-back of gated delta-rule linear-attention
 * layers (KDA: decay per key channel; GDN: decay per head).
 *
 * Sources, cited by page title and section:
 *   [WB]   "When Quantization Breaks Memory: Recurrent-State Write-Back in
 *          Low-Precision Temporal Inference" (English and Chinese summaries)
 *   [LB]   "Low-Bit Recurrent States in Hybrid Language Models"
 *   [LBX]  "Allocate low-bit recurrent state precision by channel decay"
 *   [DAMP] summary of "DAMP: Decay-Aware Mixed-Precision recurrent-state
 *          quantization" (arXiv 2608.27513)
 *
 * Conventions shared by every entry point
 *   - Plain C types only.  Device pointers are CUDA global-memory addresses
 *     on the current device; `stream` is a cudaStream_t (NULL = legacy
 *     default stream).  bfloat16 inputs are passed as their uint16_t bit
 *     patterns, FP16 fields are uint16_t bit patterns.
 *   - Ownership: the caller allocates and owns every buffer (state, residual,
 *     statistics, workspace, inputs, outputs) and the stream.  The library
 *     allocates no device memory and keeps no state between calls except the
 *     thread-local error string.
 *   - Execution: every call that launches work is asynchronous on `stream`.
 *     Argument errors are detected on the host and returned at once (no work
 *     is launched).  Errors detected by the kernels (non-finite values, FP16
 *     overflow) are OR-ed into a flag word at the start of `workspace` and
 *     reported by brs_fetch_errors(), which synchronises the stream.
 *   - Alignment: every device pointer must be 16-byte aligned (BRS_EALIGN).
 *   - Dimensions: d_k = d_v = d with d in {32, 64, 128}.
 *   - Inputs of one token (decode): q, k [B][H_k][d] bf16; v [B][H][d] bf16;
 *     beta [B][H] f32; decay [B][H][d] f32 (KDA) or [B][H] f32 (GDN), holding
 *     a = exp(-s) (not s); output o [B][H][d] f32.  q and k are expected
 *     L2-normalised.  Value head h reads key head h * H_k / H (grouped value
 *     heads).
 *
 * Stored state formats (byte layouts; all multi-byte fields little-endian)
 *   BRS_STORE_FP32   float [B][H][d][d], rows in stored order.
 *   BRS_STORE_DAMP   [DAMP] Key Points > Main operating point and
 *                    Implementation; Quantization & calibration details.
 *                    Per head (b, h), contiguous, head stride
 *                      (d-k_hi)*d + k_hi*d*2 + (d-k_hi)*(d/block)*4 bytes:
 *                      u8  codes[d-k_hi][d]      stored rows 0..d-k_hi-1,
 *                                                asymmetric INT8 of the row
 *                                                after the d-point Hadamard
 *                                                (when `hadamard` is set);
 *                      f16 rows [k_hi][d]        protected rows
 *                                                d-k_hi..d-1, in the value
 *                                                basis;
 *                      f16 sz[d-k_hi][d/block][2] (scale, zero) per block;
 *                                                value = fmaf(code, scale,
 *                                                zero).
 *                    Stored row i holds key channel perm[h][i] (the
 *                    protected channels are the last k_hi entries).
 *                    With low_bits = 4 (b = 4 of the same section) the code
 *                    rows hold two codes per byte ((d-k_hi)*d/2 bytes;
 *                    element e of a row in bits 4 (e % 2) of byte e/2),
 *                    codes run 0..15 and the scale divides the block's
 *                    range by 15; the rest is unchanged.  Every entry
 *                    point that takes DAMP storage accepts it.
 *                    Error-feedback residuals: f16 [B][H][d-k_hi][d].
 *   BRS_STORE_VARBIT [LB] State bit allocation, Allocation units, Levels and
 *                    storage.  Sections, each starting on a 256-byte
 *                    boundary: payload [B][P] bytes with
 *                    P = (d/8) * avg_bits * H * d; f16 step [B][H*d];
 *                    u8 width [B][H*d] (2..8); u32 row offset [B][H*d+1].
 *                    Row r of sequence b holds d codes u = q + n,
 *                    n = 2^(w-1) - 1, w bits each, little-endian bit order,
 *                    starting at byte offset[r] = (d/8) * (sum of the
 *                    widths of rows < r); value = (u - n) * step.
 *                    Residuals f16 [B][H][d][d]; statistics f64
 *                    [B][H][d][2] = (EMA of a^2, EMA of beta (2-beta) k^2).
 *   BRS_STORE_VARBIT_HEAD [LB] Allocation units (per-head decay, as in
 *                    Gated DeltaNet): one width per head, one FP16 step
 *                    per block of 32 key channels and column.  Sections,
 *                    each starting on a 256-byte boundary: payload [B][P]
 *                    with P = d*d/8 * avg_bits * H; f16 step
 *                    [B][H][d/32][d]; u8 width [B][H] (b_min >= 2);
 *                    u32 head offset [B][H+1].  Head h of sequence b holds
 *                    element (i, j) (key channel i, value column j) as a
 *                    w-bit code u = q + n at bit (i*d + j)*w of its bytes,
 *                    starting at offset[h] = d*d/8 * (sum of the widths of
 *                    heads < h); value = (u - n) * step[i/32][j].  The
 *                    steps are fitted per (block, column) group as for a
 *                    row; the allocator runs over each sequence's H heads
 *                    with a head's cost the mean of its rows' decay
 *                    weights (no range term).  d = 128; residuals and
 *                    statistics as for VARBIT; the workspace holds the
 *                    flag word and one f64 cost per head.
 *
 * Arithmetic (identical on every path that produces stored codes)
 *   The update runs in FP32 ([DAMP] Implementation): per token and head,
 *   S <- Diag(a) S; u = S^T k; w = beta (v - u); S <- S + k w^T; o = S^T q.
 *   FP32 storage: each sum over key rows is an fmaf chain over stored rows
 *   0..d-1 from +0.  DAMP storage: each tier is updated in the basis it is
 *   stored in (INT8 rows in the basis T = the Hadamard when `hadamard` is
 *   set, else the identity; FP16 rows in the value basis):
 *     u = U2 + T(U1), w = beta (v - u), INT8 rows S_i += k_i T(w),
 *     FP16 rows S_i += k_i w, o = O2 + T(O1),
 *   where U1/O1 (U2/O2) are fmaf chains over the INT8 (FP16) rows in stored
 *   order from +0.  T is the unnormalised Sylvester butterfly (stages 1, 2,
 *   4, ...) followed by one multiplication by the float nearest 1/sqrt(d).
 *   INT8 block: scale = fp16((max - min) / 255), zero = fp16(min),
 *   code = clamp(round((y - zero) * (1/scale)), 0, 255).  Rounding
 *   ([WB] Quantized GRU formulation; Chinese summary, error feedback and
 *   stochastic rounding): nearest = ties to the even code; stochastic =
 *   floor(t) + [r24 < frac(t) * 2^24] with r24 the top 24 bits of word
 *   (e % 4) of Philox4x32-10(counter (e/4, step, h, b), key (seed_lo,
 *   seed_hi)), e = row * d + column; error feedback = y = x + e_prev,
 *   e_new = fp16(clamp(y - value, -scale, +scale)).
 */
#ifndef BRS_H
#define BRS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BRS_OK = 0,
  BRS_EINVAL = 1,        /* bad argument (shape, null pointer, infeasible budget) */
  BRS_EUNSUPPORTED = 2,  /* valid but not implemented combination              */
  BRS_EALIGN = 3,        /* a device pointer is not 16-byte aligned             */
  BRS_ECUDA = 4,         /* a CUDA runtime call failed                          */
  BRS_ENONFINITE = 5,    /* a kernel met a non-finite state value               */
  BRS_EOVERFLOW = 6,     /* an FP16 row, scale or zero overflowed               */
  BRS_ETIMEOUT = 7       /* a bounded device-side wait gave up                  */
} brs_status;

typedef enum { BRS_STORE_FP32 = 0, BRS_STORE_DAMP = 1, BRS_STORE_VARBIT = 2, BRS_STORE_VARBIT_HEAD = 3 } brs_storage;

typedef enum {
  BRS_ROUND_NEAREST = 0,
  BRS_ROUND_STOCHASTIC = 1,
  BRS_ROUND_ERRFEEDBACK = 2,
  /* Direction memory ([WB] Post-training write-back interventions; the
     voting region of its Trajectory analysis): nearest write-back plus a
     2-bit sign counter per INT8 element.  A proposed change y - x_prev (x_prev:
     the stored value the token started from) with scale/8 < |y - x_prev| <
     scale/2 votes its sign; a counter reaching +-2 moves the code one level
     that way (clipped to [0, 255]) and is reset.  DAMP decode with C = 1
     only.  The counters live in the first B*H*(d-k_hi)*d/4 bytes of the
     residual buffer (four to a byte, column order, two's complement), which
     starts zeroed. */
  BRS_ROUND_DIRECTION = 3,
  /* k-bit residual memory, k = 2, 3, 4 ([WB] Post-training write-back
     interventions: error feedback's residual with evaluated widths
     k = 2, 3, 4; Matched recurrent-memory training campaign: a 4-bit visible
     state plus two auxiliary bits): error feedback whose residual is kept as
     a k-bit signed integer m of step/2^k, |m| <= 2^(k-1) - 1.  The target is
     y + m (sprev / 2^k), sprev the block's stored step the token started
     from; codes and grid are those of nearest write-back of the target; the
     new m = clamp(rne((target - value) * (1/scale) * 2^k)).  DAMP decode with
     C = 1 only.  The integers live in the first B*H*(d-k_hi)*d/2 bytes of
     the residual buffer (two to a byte, column order, element e in bits
     4 (e % 2), two's complement), which starts zeroed. */
  BRS_ROUND_RESIDUAL2 = 4,
  BRS_ROUND_RESIDUAL3 = 5,
  BRS_ROUND_RESIDUAL4 = 6
} brs_round;

/* Device flag bits OR-ed into the first 32-bit word of `workspace`. */
#define BRS_FLAG_NONFINITE 0x1u
#define BRS_FLAG_OVERFLOW 0x2u
#define BRS_FLAG_TIMEOUT 0x4u
#define BRS_FLAG_INVALID 0x8u   /* a device-side argument check failed (e.g. widths off the budget) */

typedef struct {
  int32_t B;             /* sequences                                          */
  int32_t H;             /* value heads                                        */
  int32_t H_k;           /* key heads (H % H_k == 0)                           */
  int32_t d;             /* d_k = d_v, in {32, 64, 128}                        */
  int32_t storage;       /* brs_storage                                        */
  int32_t k_hi;          /* DAMP: protected FP16 rows per head (multiple of 4) */
  int32_t block;         /* DAMP: INT8 block length along the value axis      */
  int32_t hadamard;      /* DAMP: 1 = INT8 rows stored after the Hadamard     */
  int32_t decay_per_key; /* 1 = KDA (decay [B][H][d]), 0 = GDN ([B][H])        */
  double avg_bits;       /* VARBIT: mean width; avg_bits*H*d integral          */
  int32_t b_min, b_max;  /* VARBIT: width limits, 1 <= b_min <= b_max <= 16    */
  int32_t budget_scope;  /* VARBIT: 1 = layer (all H*d rows of a sequence),
                            0 = head                                           */
  int32_t persistence;   /* VARBIT: row weight of the allocation cost ([LB]
                            Choice of persistence factor): 0 = the erasure
                            rate Gamma_hat, 1 = DAMP's uncapped w^(1) =
                            1/(1 - e^-2s), 2 = h^(C) = 1/(1 - e^-2Cs)           */
  int32_t low_bits;      /* DAMP: width b of the low tier, 8 (0 reads as 8) or
                            4 ([DAMP] Data & Methods > Quantization &
                            calibration details: b = 8 or b = 4)               */
} brs_layout;

typedef struct {
  int32_t mode;          /* brs_round                                          */
  uint64_t seed;         /* Philox key of stochastic rounding                  */
  int32_t C;             /* write-back interval in tokens ([LB] Accumulated
                            readout error: once per chunk, per token, or every
                            C tokens)                                          */
} brs_writeback;

/* Bytes of the stored state for layout L; optionally the bytes of the
 * auxiliary buffer (error-feedback residuals; direction-memory counters use
 * its first quarter), of the allocator statistics and of the workspace a
 * call needs.  Returns 0 for an invalid layout (see
 * brs_last_error). */
size_t brs_state_bytes(const brs_layout* L, size_t* aux_bytes, size_t* stats_bytes,
                       size_t* workspace_bytes);

/* FP32 state S [B][H][d][d] (rows in key-channel order) -> stored format,
 * deterministic rounding.  perm [H][d] int16 (stored row i of head h holds
 * channel perm[h][i]); NULL = identity.  widths (VARBIT only) u8 [B][H*d]
 * device array of row widths (VARBIT_HEAD: u8 [B][H], head widths), NULL =
 * avg_bits for every row or head (which must then be an integer).  A
 * VARBIT_HEAD width map whose sequence total is not avg_bits * H, or with a
 * width outside 1..16, stores nothing for that sequence and raises
 * BRS_FLAG_INVALID.  All pointers device, `packed` sized by
 * brs_state_bytes.  [DAMP] Implementation (static permuted layout). */
brs_status brs_state_pack(const brs_layout* L, const float* S, const int16_t* perm,
                          const uint8_t* widths, void* packed, void* workspace, void* stream);

/* Stored format -> FP32 state S [B][H][d][d] in key-channel order. */
brs_status brs_state_unpack(const brs_layout* L, const void* packed, const int16_t* perm,
                            float* S, void* workspace, void* stream);

/* One decode token for every head: dequantize the stored state, apply the
 * decay and the delta-rule write in FP32, read o from the updated FP32
 * state, then (when (step + 1) % C == 0) requantize and write back
 * ([DAMP] Implementation; [LB] Accumulated readout error: outputs precede
 * quantization; [LB] Protocol: each write-back is quantized and dequantized
 * before reuse).  Decode supports C == 1 (brs_decode_step_deferred takes
 * C > 1).
 *   packed_in / packed_out: stored state before / after; they may alias
 *     for FP32 and DAMP storage, must not alias for VARBIT and
 *     VARBIT_HEAD.
 *   aux: residuals (ERRFEEDBACK), direction counters (DIRECTION) or
 *     residual integers (RESIDUAL2..4; the last two DAMP only), updated in
 *     place; else may be NULL.
 *   stats: VARBIT / VARBIT_HEAD statistics, updated in place (else may be
 *     NULL).
 *   workspace: brs_state_bytes(...workspace) bytes; its first word
 *     collects device flags and must be zeroed once before first use
 *     (brs_fetch_errors clears it).
 *   perm: [H][d] int16 device, NULL = identity.
 * Inputs and o: see the conventions above. */
brs_status brs_decode_step(const brs_layout* L, const brs_writeback* wb, int64_t step,
                           const void* packed_in, void* packed_out, void* aux, void* stats,
                           void* workspace, const int16_t* perm, const uint16_t* q,
                           const uint16_t* k, const uint16_t* v, const float* beta,
                           const float* decay, float* o, void* stream);

/* Decode with deferred write-back ([LB] Accumulated readout error: the state
 * is written back every C tokens; between write-backs it is carried in FP32).
 * DAMP storage.  One token for every head, as brs_decode_step, with write-back
 * rounding `wb` applied when (step + 1) % C == 0; the other tokens leave the
 * stored state untouched and carry the updated FP32 state in `state32`:
 *   state32: device, brs_decode_state32_bytes(L) bytes, [B][H][d][d] FP32 in
 *     stored row order, each tier in the basis its arithmetic uses (INT8-tier
 *     rows after the Hadamard, FP16-tier rows in the value basis).  Read when
 *     step % C != 0 (else the stored state is read), written when
 *     (step + 1) % C != 0.  May be NULL when C == 1.
 *   packed: stored state, updated in place at write-backs.  aux: residuals
 *     (error feedback), used and updated at write-backs only; direction and
 *     residual memory need C == 1.
 *   workspace: flag word (as brs_decode_step).
 * Calls must cover consecutive steps, starting at a multiple of C, for the
 * result to equal the recurrence with write-back every C tokens (the state
 * between write-backs is exactly the FP32 state of the token-by-token
 * arithmetic).  C == 1 is brs_decode_step.  Returns BRS_EUNSUPPORTED for
 * other storage formats or shapes outside brs_decode_step's. */
size_t brs_decode_state32_bytes(const brs_layout* L);
brs_status brs_decode_step_deferred(const brs_layout* L, const brs_writeback* wb, int64_t step, void* packed,
                                    void* aux, void* workspace, void* state32, const int16_t* perm,
                                    const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* beta,
                                    const float* decay, float* o, void* stream);

/* Chunked prefill with deferred write-back ([LB] Accumulated readout error:
 * write-back once per prefill chunk; [LB] Protocol).  Tokens
 * [step0, step0 + T) of every (sequence, head) with write-back after every
 * chunk of C tokens: the chunk's C delta-rule steps are evaluated together
 * (WY form: A = strictly-lower(diag(beta) K~ K^T), (I + A) W =
 * diag(beta) (V - K~ S0), O = Q~ S0 + lower(Q~ K^T) W,
 * S_C = diag(Gamma_C) (S0 + K^T W), with Gamma the cumulative decay, K~ =
 * K Gamma, K^ = K / Gamma, Q~ = Q Gamma) in FP32, then the state is
 * requantized (value basis -> Hadamard -> INT8 blocks; FP16 rows) with the
 * write-back rounding of `wb` at the chunk's last token.  DAMP storage,
 * d = 128, C = 64, block 128 or 32.
 *   packed: stored state, updated in place.  aux: residuals (error
 *     feedback; direction memory is not built for the prefill).
 *   workspace: brs_prefill_workspace_bytes(L) bytes, 16-byte aligned: the
 *     flag word in its first 256 bytes (as brs_decode_step), then the FP32
 *     state carried between the chunks of the call, B*H*d*d floats, then
 *     B*H u32 hand-over counters (rounded to 256 bytes), all of which the
 *     call overwrites (their contents between calls do not matter).  The
 *     call runs one CTA per SM, each taking an equal share of the
 *     (head, chunk) units; a head cut between two CTAs passes from one to
 *     the next through the scratch state and its counter (a bounded wait:
 *     BRS_ETIMEOUT if the hand-over does not come).
 *   q, k [B][T][H_k][d] bf16; v [B][T][H][d] bf16; beta [B][T][H] f32;
 *     decay [B][T][H][d] (KDA) or [B][T][H] (GDN) f32; o [B][T][H][d] f32.
 *   state_dump (optional): [B][H][d][d] f32, the state just before the last
 *     write-back of the call (stored row order, value basis).
 * The contractions run on the tensor cores in TF32 with each operand split
 * into a TF32 part and its remainder (three products), which keeps FP32-level
 * accuracy.  Results agree with the token-by-token recurrence within the
 * rounding of the reordered sums; the stored codes are the documented
 * quantizer applied to state_dump.  A call over several chunks equals
 * consecutive one-chunk calls bit for bit.  The call allocates nothing.
 * Per-channel decays whose 64-token product underflows FP32 are outside the
 * form (the outputs become non-finite: BRS_ENONFINITE).
 * brs_prefill_workspace_bytes: the workspace size for layout L (0 for an
 * invalid layout or one the prefill does not support; see brs_last_error). */
size_t brs_prefill_workspace_bytes(const brs_layout* L);
brs_status brs_chunk_prefill(const brs_layout* L, const brs_writeback* wb, int64_t step0, int T,
                             void* packed, void* aux, void* workspace, const int16_t* perm,
                             const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             const float* beta, const float* decay, float* o, float* state_dump,
                             void* stream);

/* Decay-aware width allocation ([LB] State bit allocation; [LBX] Worked
 * example).  For each of n_rows / rows_per_group groups of rows (a layer's
 * H*d rows, or one head's d rows), in FP64: b*_i = avg + log2(c_i/GM)/2
 * with GM the geometric mean over the rows with c_i > 0; rounded to
 * nearest (ties to even) and clipped to [b_min, b_max] (b_min when
 * c_i = 0; round(avg) for every row when all c_i are 0); then bits are
 * moved one at a time, while over budget from the row whose cost
 * 3 c_i 4^(-b_i) is smallest, while under budget to the row whose gain
 * 3/4 c_i 4^(-b_i) is largest, ties to the lower row, until the group sums
 * to avg * rows_per_group.
 *   cost: device f64 [n_rows]; bits_out: device u8 [n_rows];
 *   offsets_out (optional): device u32 [groups][rows_per_group + 1], the
 *   exclusive prefix sums of the widths times offset_unit.
 * rows_per_group <= 8192; avg * rows_per_group must be an integer in
 * [b_min, b_max] * rows_per_group (BRS_EINVAL). */
brs_status brs_allocate_bits(int n_rows, int rows_per_group, const double* cost, double avg_bits,
                             int b_min, int b_max, uint32_t offset_unit, uint8_t* bits_out,
                             uint32_t* offsets_out, void* stream);

/* Protected-row selection on a calibration run ([DAMP] Risk scoring and
 * selection; Calibration): the FP32 recurrence (the FP32-storage decode
 * step) runs from a zero state over T tokens of a calibration batch of Bc
 * sequences; every `every` tokens each key row u of each head is scored by
 * the squared error energy of its Hadamard-INT8 quantize -> dequantize
 * (nearest rounding, L's block and Hadamard setting); then
 *   E_u = the mean energy over sequences and samples,
 *   a_eff,u = exp(mean over sequences and tokens of log a_u),
 *   C_u = E_u / max(1 - a_eff,u^2, tau),
 * and the k_hi largest C_u of a head (ties to the lower row) are protected.
 *   L: a DAMP layout (B is ignored; d in {32, 64, 128}, k_hi <= d).
 *   q, k: device bf16 [T][Bc][H_k][d]; v: bf16 [T][Bc][H][d];
 *   beta: f32 [T][Bc][H]; decay: f32 [T][Bc][H][d] (KDA) or [T][Bc][H]
 *   (GDN), key-channel order, no permutation.
 *   workspace: device, brs_calibrate_workspace_bytes(L, Bc, T, every) bytes,
 *   16-byte aligned; its first 256 bytes are the device flag word
 *   (brs_fetch_errors).
 *   score_out (optional): device f64 [H][d], C_u in key-channel order (kept
 *   in the workspace when NULL).
 *   perm_out: device int16 [H][d], the stored order to pass to the other
 *   calls: the unprotected rows ascending, then the protected rows
 *   ascending.
 * Sums are taken in FP64 in a fixed order (per row over its values; per
 * (head, row) over sequences, then samples or tokens in order).  Setup
 * work; the call issues T + T/every + 2 kernels on the stream. */
size_t brs_calibrate_workspace_bytes(const brs_layout* L, int Bc, int T, int every);
brs_status brs_calibrate(const brs_layout* L, int Bc, int T, int every, double tau,
                         const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* beta,
                         const float* decay, void* workspace, double* score_out, int16_t* perm_out,
                         void* stream);

/* Allocation-free variant of brs_decode_step (the pages have no
 * counterpart; it exists for callers that cannot allocate device memory,
 * such as a host framework whose allocator owns the whole device or a
 * serving loop with a fixed memory budget).  Same arguments and semantics
 * as brs_decode_step without `workspace`: the scratch is a static device
 * array of 4096 bytes inside the library, reserved on every device that
 * loads it until the process exits.  Layouts whose workspace
 * (brs_state_bytes) exceeds 4096 bytes are rejected with BRS_EINVAL.  The
 * first call on a device looks the array's address up (cudaGetSymbolAddress)
 * and should precede any stream capture; the device must not be reset
 * (cudaDeviceReset) while the library stays loaded, since that invalidates
 * the address.  All calls share the array, so calls that overlap on the GPU
 * race.  The array's first word collects the device flags of every call on
 * that device (zero when the library is loaded) until
 * brs_fetch_errors_noalloc reads and clears it; the rest of the layout's
 * scratch is written by each call before it is read. */
brs_status brs_decode_step_noalloc(const brs_layout* L, const brs_writeback* wb, int64_t step,
                                   const void* packed_in, void* packed_out, void* aux, void* stats,
                                   const int16_t* perm, const uint16_t* q, const uint16_t* k,
                                   const uint16_t* v, const float* beta, const float* decay,
                                   float* o, void* stream);

/* brs_fetch_errors for the static scratch of brs_decode_step_noalloc on the
 * current device: reads and clears the flags its calls raised (synchronises
 * `stream`). */
brs_status brs_fetch_errors_noalloc(uint32_t* flags_out, void* stream);

/* Reads and clears the device flag word of `workspace` (synchronises
 * `stream`).  Returns BRS_OK, or BRS_ENONFINITE / BRS_EOVERFLOW /
 * BRS_ETIMEOUT for the first flag set; *flags_out (optional) receives the
 * raw bits. */
brs_status brs_fetch_errors(void* workspace, uint32_t* flags_out, void* stream);

/* Test hook for the prefill's work split (the pages have no counterpart).
 * While `n` is positive, brs_chunk_prefill calls made from this host thread
 * launch at most n CTAs (by default one per SM, at most one per head), so
 * that small batches cut heads between CTAs and exercise the hand-over.
 * Results do not depend on n.  0 restores the default; not for use outside
 * tests. */
void brs_test_prefill_ctas(int n);

/* Test hook for the bounded wait of the prefill's hand-over (the pages have
 * no counterpart).  While `on` is nonzero, brs_chunk_prefill calls made from
 * this host thread hand no head over: a CTA that continues a head cut at
 * the start of its share waits out its bound (200 ms), raises
 * BRS_FLAG_TIMEOUT and leaves that head where it is; nothing faults and the
 * context stays usable (brs_fetch_errors reports BRS_ETIMEOUT).  Off by
 * default; not for use outside tests. */
void brs_test_prefill_withhold(int on);

/* Test hook for the bounded device waits (the pages have no counterpart).
 * While `on` is nonzero, brs_decode_step calls made from this host thread
 * make the copy barrier of every head of the CTA-per-head decode kernel
 * (DAMP storage, d = 128) expect 16 bytes more than the head's copies
 * deliver: the copies complete, the barrier never does, every bounded wait
 * runs out (200 ms), and the kernel raises BRS_FLAG_TIMEOUT and returns
 * without writing the stored state or the outputs.  Nothing faults and the
 * context stays usable; brs_fetch_errors then reports BRS_ETIMEOUT.  Off by
 * default; not for use outside tests. */
void brs_test_starve_copies(int on);

/* Message of the last error returned on this host thread ("" if none). */
const char* brs_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* BRS_H */
