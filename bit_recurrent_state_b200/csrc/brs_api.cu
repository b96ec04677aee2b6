// Host side of the C ABI declared in include/brs.h: argument validation,
// byte-layout arithmetic, kernel dispatch, error reporting.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "brs.h"
#include "brs_internal.h"

namespace {

thread_local char g_err[512] = "";
thread_local uint32_t g_starve_tx = 0;   // test hook: brs_test_starve_copies
thread_local int g_prefill_ctas = 0;     // test hook: brs_test_prefill_ctas
thread_local int g_prefill_withhold = 0; // test hook: brs_test_prefill_withhold

brs_status fail(brs_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

brs_status ok() {
  g_err[0] = 0;
  return BRS_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// float nearest to 1/sqrt(d)
float hadamard_scale(int d) { return (float)(1.0 / std::sqrt((double)d)); }

brs_status check_layout(const brs_layout* L) {
  if (!L) return fail(BRS_EINVAL, "layout is NULL");
  if (L->B <= 0 || L->H <= 0 || L->H_k <= 0) return fail(BRS_EINVAL, "B, H, H_k must be positive");
  if (L->H % L->H_k) return fail(BRS_EINVAL, "H (%d) must be a multiple of H_k (%d)", L->H, L->H_k);
  if (L->d != 32 && L->d != 64 && L->d != 128) return fail(BRS_EINVAL, "d must be 32, 64 or 128 (got %d)", L->d);
  if (L->storage == BRS_STORE_DAMP) {
    if (L->k_hi < 0 || L->k_hi > L->d || (L->k_hi % 4)) return fail(BRS_EINVAL, "k_hi must be a multiple of 4 in [0, d]");
    if (!pow2(L->block) || L->block < 4 || L->block > L->d)
      return fail(BRS_EINVAL, "block must be a power of two in [4, d] (got %d)", L->block);
    if (L->low_bits != 0 && L->low_bits != 8 && L->low_bits != 4)
      return fail(BRS_EINVAL, "low_bits must be 8 (or 0) or 4 (got %d)", L->low_bits);
  } else if (L->storage == BRS_STORE_VARBIT) {
    if (L->hadamard) return fail(BRS_EUNSUPPORTED, "variable-width storage is stored without the Hadamard");
    if (L->b_min < 1 || L->b_max > 16 || L->b_min > L->b_max) return fail(BRS_EINVAL, "need 1 <= b_min <= b_max <= 16");
    if (L->persistence < 0 || L->persistence > 2) return fail(BRS_EINVAL, "persistence must be 0, 1 or 2");
    const double tot = L->avg_bits * (double)L->H * (double)L->d;
    if (tot != std::floor(tot)) return fail(BRS_EINVAL, "avg_bits * H * d must be an integer");
    if (L->avg_bits < L->b_min || L->avg_bits > L->b_max) return fail(BRS_EINVAL, "avg_bits outside [b_min, b_max]");
  } else if (L->storage == BRS_STORE_VARBIT_HEAD) {
    if (L->hadamard) return fail(BRS_EUNSUPPORTED, "variable-width storage is stored without the Hadamard");
    if (L->d != 128) return fail(BRS_EUNSUPPORTED, "per-head widths are built for d = 128 (got %d)", L->d);
    if (L->b_min < 2 || L->b_max > 16 || L->b_min > L->b_max)
      return fail(BRS_EINVAL, "per-head widths need 2 <= b_min <= b_max <= 16");
    if (L->budget_scope != 1) return fail(BRS_EINVAL, "per-head widths share one budget over the layer (budget_scope 1)");
    if (L->persistence < 0 || L->persistence > 2) return fail(BRS_EINVAL, "persistence must be 0, 1 or 2");
    const double tot = L->avg_bits * (double)L->H;
    if (tot != std::floor(tot)) return fail(BRS_EINVAL, "avg_bits * H must be an integer");
    if (L->avg_bits < L->b_min || L->avg_bits > L->b_max) return fail(BRS_EINVAL, "avg_bits outside [b_min, b_max]");
  } else if (L->storage != BRS_STORE_FP32) {
    return fail(BRS_EINVAL, "unknown storage %d", L->storage);
  }
  return BRS_OK;
}

bool varbit_like(const brs_layout* L) {
  return L->storage == BRS_STORE_VARBIT || L->storage == BRS_STORE_VARBIT_HEAD;
}

brs::VbSections vb_sections_of(const brs_layout* L) {
  return L->storage == BRS_STORE_VARBIT_HEAD ? brs::varbit_head_sections(L->B, L->H, L->d, L->avg_bits)
                                             : brs::varbit_sections(L->B, L->H, L->d, L->avg_bits);
}

// width of the DAMP low tier: 8 unless the layout asks for 4
int low_bits(const brs_layout* L) { return L->low_bits == 4 ? 4 : 8; }

size_t damp_head_bytes(const brs_layout* L) {
  const size_t d = (size_t)L->d, kh = (size_t)L->k_hi;
  return (d - kh) * d * (size_t)low_bits(L) / 8 + kh * d * 2 + (d - kh) * (d / (size_t)L->block) * 4;
}

size_t head_bytes(const brs_layout* L) {
  return L->storage == BRS_STORE_FP32 ? (size_t)L->d * L->d * 4 : damp_head_bytes(L);
}

brs_status cuda_fail(cudaError_t e, const char* what) {
  return fail(BRS_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace

namespace brs {
// lets other translation units of the library report through brs_last_error
void set_last_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }
uint32_t starve_tx_bytes() { return g_starve_tx; }
int prefill_cta_cap() { return g_prefill_ctas; }
int prefill_withhold() { return g_prefill_withhold; }
}  // namespace brs

extern "C" {

const char* brs_last_error(void) { return g_err; }

void brs_test_starve_copies(int on) { g_starve_tx = on ? 16u : 0u; }

void brs_test_prefill_ctas(int n) { g_prefill_ctas = n > 0 ? n : 0; }

void brs_test_prefill_withhold(int on) { g_prefill_withhold = on ? 1 : 0; }

size_t brs_state_bytes(const brs_layout* L, size_t* aux_bytes, size_t* stats_bytes,
                       size_t* workspace_bytes) {
  if (check_layout(L) != BRS_OK) return 0;
  const size_t heads = (size_t)L->B * L->H, d = (size_t)L->d;
  size_t total = 0, aux = 0, stats = 0, ws = 256;
  if (L->storage == BRS_STORE_FP32) {
    total = heads * d * d * 4;
  } else if (L->storage == BRS_STORE_DAMP) {
    total = heads * damp_head_bytes(L);
    aux = heads * (d - (size_t)L->k_hi) * d * 2;
  } else {
    total = vb_sections_of(L).total;
    aux = heads * d * d * 2;
    stats = heads * d * 2 * sizeof(double);
    // flag word, then one FP64 cost per row (per head for head units)
    ws = 256 + heads * (L->storage == BRS_STORE_VARBIT_HEAD ? 1 : d) * sizeof(double);
  }
  if (aux_bytes) *aux_bytes = aux;
  if (stats_bytes) *stats_bytes = stats;
  if (workspace_bytes) *workspace_bytes = ws;
  ok();
  return total;
}

brs_status brs_state_pack(const brs_layout* L, const float* S, const int16_t* perm,
                          const uint8_t* widths, void* packed, void* workspace, void* stream) {
  brs_status st = check_layout(L);
  if (st != BRS_OK) return st;
  if (!S || !packed || !workspace) return fail(BRS_EINVAL, "S, packed and workspace are required");
  if (varbit_like(L)) {
    if (perm) return fail(BRS_EINVAL, "variable-width storage keeps rows in key-channel order (perm must be NULL)");
    if (!widths && L->avg_bits != std::floor(L->avg_bits))
      return fail(BRS_EINVAL, "uniform widths need an integer avg_bits");
    if (!aligned16(S) || !aligned16(packed) || !aligned16(workspace))
      return fail(BRS_EALIGN, "device pointers must be 16-byte aligned");
    brs::VbPackArgs v{};
    v.B = L->B; v.H = L->H; v.d = L->d; v.avg_bits = L->avg_bits;
    v.sec = vb_sections_of(L);
    v.S = S; v.widths = widths; v.packed = packed; v.flags = (uint32_t*)workspace;
    cudaError_t e = L->storage == BRS_STORE_VARBIT_HEAD ? brs::launch_varbit_head_pack(v, (cudaStream_t)stream)
                                                        : brs::launch_varbit_pack(v, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "variable-width pack launch");
    return ok();
  }
  (void)widths;
  if (!aligned16(S) || !aligned16(packed) || !aligned16(workspace) || (perm && !aligned16(perm)))
    return fail(BRS_EALIGN, "device pointers must be 16-byte aligned");
  brs::PackArgs a{};
  a.B = L->B; a.H = L->H; a.d = L->d; a.storage = L->storage; a.k_hi = L->k_hi;
  a.block = L->block; a.hadamard = L->hadamard; a.low_bits = low_bits(L); a.head_bytes = head_bytes(L);
  a.hscale = hadamard_scale(L->d); a.S = S; a.perm = perm; a.packed = packed;
  a.flags = (uint32_t*)workspace;
  cudaError_t e = brs::launch_pack(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  return ok();
}

brs_status brs_state_unpack(const brs_layout* L, const void* packed, const int16_t* perm,
                            float* S, void* workspace, void* stream) {
  brs_status st = check_layout(L);
  if (st != BRS_OK) return st;
  if (!S || !packed) return fail(BRS_EINVAL, "S and packed are required");
  if (varbit_like(L)) {
    if (perm) return fail(BRS_EINVAL, "variable-width storage keeps rows in key-channel order (perm must be NULL)");
    if (!aligned16(S) || !aligned16(packed)) return fail(BRS_EALIGN, "device pointers must be 16-byte aligned");
    brs::VbPackArgs v{};
    v.B = L->B; v.H = L->H; v.d = L->d; v.avg_bits = L->avg_bits;
    v.sec = vb_sections_of(L);
    v.flags = (uint32_t*)workspace;
    cudaError_t e = L->storage == BRS_STORE_VARBIT_HEAD
                        ? brs::launch_varbit_head_unpack(v, packed, S, (cudaStream_t)stream)
                        : brs::launch_varbit_unpack(v, packed, S, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "variable-width unpack launch");
    return ok();
  }
  if (!aligned16(S) || !aligned16(packed) || (perm && !aligned16(perm)))
    return fail(BRS_EALIGN, "device pointers must be 16-byte aligned");
  brs::PackArgs a{};
  a.B = L->B; a.H = L->H; a.d = L->d; a.storage = L->storage; a.k_hi = L->k_hi;
  a.block = L->block; a.hadamard = L->hadamard; a.low_bits = low_bits(L); a.head_bytes = head_bytes(L);
  a.hscale = hadamard_scale(L->d); a.perm = perm; a.flags = (uint32_t*)workspace;
  cudaError_t e = brs::launch_unpack(a, S, packed, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "unpack launch");
  return ok();
}

brs_status brs_decode_step(const brs_layout* L, const brs_writeback* wb, int64_t step,
                           const void* packed_in, void* packed_out, void* aux, void* stats,
                           void* workspace, const int16_t* perm, const uint16_t* q,
                           const uint16_t* k, const uint16_t* v, const float* beta,
                           const float* decay, float* o, void* stream) {
  brs_status st = check_layout(L);
  if (st != BRS_OK) return st;
  (void)stats;
  if (!wb) return fail(BRS_EINVAL, "writeback is NULL");
  if (wb->C != 1) return fail(BRS_EUNSUPPORTED, "decode writes back every token (C = 1); got C = %d", wb->C);
  if (wb->mode < 0 || wb->mode > 6) return fail(BRS_EINVAL, "unknown rounding mode %d", wb->mode);
  if (wb->mode >= BRS_ROUND_DIRECTION && L->storage != BRS_STORE_DAMP)
    return fail(BRS_EUNSUPPORTED, "direction and residual memory are built for DAMP storage");
  if (wb->mode >= BRS_ROUND_DIRECTION && !aux)
    return fail(BRS_EINVAL, "direction and residual memory need the auxiliary buffer");
  if (step < 0) return fail(BRS_EINVAL, "step must be >= 0");
  if (!packed_in || !packed_out || !workspace || !q || !k || !v || !beta || !decay || !o)
    return fail(BRS_EINVAL, "a required pointer is NULL");
  if (varbit_like(L)) {
    if (L->d != 128) return fail(BRS_EUNSUPPORTED, "variable-width decode is built for d = 128");
    if (packed_in == packed_out) return fail(BRS_EINVAL, "variable-width decode needs packed_out != packed_in");
    if (perm) return fail(BRS_EINVAL, "variable-width storage keeps rows in key-channel order (perm must be NULL)");
    if (!stats) return fail(BRS_EINVAL, "variable-width decode needs the statistics buffer");
    if (wb->mode == BRS_ROUND_ERRFEEDBACK && !aux) return fail(BRS_EINVAL, "error feedback needs the residual buffer");
    const void* ptrs[] = {packed_in, packed_out, aux, stats, workspace, q, k, v, beta, decay, o};
    for (const void* p : ptrs)
      if (p && !aligned16(p)) return fail(BRS_EALIGN, "device pointers must be 16-byte aligned");
    brs::VbArgs a{};
    a.B = L->B; a.H = L->H; a.Hk = L->H_k; a.decay_per_key = L->decay_per_key; a.mode = wb->mode;
    a.first = step == 0; a.C = wb->C; a.b_min = L->b_min; a.b_max = L->b_max;
    a.budget_scope = L->budget_scope; a.persistence = L->persistence; a.seed = wb->seed; a.step = step;
    double lam = 1.0;
    for (int c = 0; c < wb->C; ++c) lam *= (1.0 - 2.0 / 65.0);   // EMA weight of a C-token chunk, span 64
    a.lambda = lam; a.avg_bits = L->avg_bits;
    a.sec = vb_sections_of(L);
    a.packed_in = packed_in; a.packed_out = packed_out; a.aux = aux; a.stats = (double*)stats;
    a.cost = (double*)((uint8_t*)workspace + 256);
    a.q = q; a.k = k; a.v = v; a.beta = beta; a.decay = decay; a.o = o; a.flags = (uint32_t*)workspace;
    cudaError_t e = L->storage == BRS_STORE_VARBIT_HEAD ? brs::launch_varbit_head_decode(a, (cudaStream_t)stream)
                                                        : brs::launch_varbit_decode(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "variable-width decode launch");
    return ok();
  }
  if (L->storage == BRS_STORE_DAMP && !brs::decode_supported(L->d, L->block, L->k_hi))
    return fail(BRS_EUNSUPPORTED,
                "decode kernel built for (d, block) in {(128,128), (128,32), (64,64), (32,32)} and "
                "k_hi a multiple of d/8 up to d/4 (got d=%d block=%d k_hi=%d)", L->d, L->block, L->k_hi);
  if (L->storage == BRS_STORE_DAMP && wb->mode == BRS_ROUND_ERRFEEDBACK && !aux)
    return fail(BRS_EINVAL, "error feedback needs the residual buffer");
  const void* ptrs[] = {packed_in, packed_out, aux, workspace, perm, q, k, v, beta, decay, o};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(BRS_EALIGN, "device pointers must be 16-byte aligned");
  brs::DecodeArgs a{};
  a.B = L->B; a.H = L->H; a.Hk = L->H_k;
  a.k_hi = L->storage == BRS_STORE_DAMP ? L->k_hi : 0;
  a.block = L->storage == BRS_STORE_DAMP ? L->block : L->d;
  a.decay_per_key = L->decay_per_key; a.mode = wb->mode; a.seed = wb->seed; a.step = step;
  a.head_bytes = head_bytes(L); a.hscale = hadamard_scale(L->d);
  a.packed_in = packed_in; a.packed_out = packed_out; a.aux = aux; a.perm = perm;
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.decay = decay; a.o = o;
  a.flags = (uint32_t*)workspace;
  a.tx_extra = brs::starve_tx_bytes();
  a.low_bits = L->storage == BRS_STORE_DAMP ? low_bits(L) : 8;
  const bool had = L->storage == BRS_STORE_DAMP && L->hadamard;
  cudaError_t e = brs::launch_decode(a, L->d, L->storage, had, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return ok();
}

size_t brs_decode_state32_bytes(const brs_layout* L) {
  if (check_layout(L) != BRS_OK) return 0;
  if (L->storage != BRS_STORE_DAMP) {
    fail(BRS_EUNSUPPORTED, "the interval state is defined for DAMP storage");
    return 0;
  }
  ok();
  return (size_t)L->B * L->H * L->d * L->d * sizeof(float);
}

brs_status brs_decode_step_deferred(const brs_layout* L, const brs_writeback* wb, int64_t step, void* packed,
                                    void* aux, void* workspace, void* state32, const int16_t* perm,
                                    const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* beta,
                                    const float* decay, float* o, void* stream) {
  brs_status st = check_layout(L);
  if (st != BRS_OK) return st;
  if (!wb) return fail(BRS_EINVAL, "writeback is NULL");
  if (L->storage != BRS_STORE_DAMP) return fail(BRS_EUNSUPPORTED, "deferred decode write-back is built for DAMP storage");
  if (wb->C < 1) return fail(BRS_EINVAL, "write-back interval C must be >= 1 (got %d)", wb->C);
  if (wb->mode < 0 || wb->mode > 6) return fail(BRS_EINVAL, "unknown rounding mode %d", wb->mode);
  if (wb->mode >= BRS_ROUND_DIRECTION && wb->C != 1)
    return fail(BRS_EUNSUPPORTED, "direction and residual memory are built for write-back every token (C = 1)");
  if (wb->mode >= BRS_ROUND_DIRECTION && !aux)
    return fail(BRS_EINVAL, "direction and residual memory need the auxiliary buffer");
  if (step < 0) return fail(BRS_EINVAL, "step must be >= 0");
  if (!brs::decode_supported(L->d, L->block, L->k_hi))
    return fail(BRS_EUNSUPPORTED,
                "decode kernel built for (d, block) in {(128,128), (128,32), (64,64), (32,32)} and "
                "k_hi a multiple of d/8 up to d/4 (got d=%d block=%d k_hi=%d)", L->d, L->block, L->k_hi);
  const bool src32 = step % wb->C != 0, dst32 = (step + 1) % wb->C != 0;
  if (!packed || !workspace || !q || !k || !v || !beta || !decay || !o)
    return fail(BRS_EINVAL, "a required pointer is NULL");
  if ((src32 || dst32) && !state32) return fail(BRS_EINVAL, "C > 1 needs the interval state");
  if (wb->mode == BRS_ROUND_ERRFEEDBACK && !aux) return fail(BRS_EINVAL, "error feedback needs the residual buffer");
  const void* ptrs[] = {packed, aux, workspace, state32, perm, q, k, v, beta, decay, o};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(BRS_EALIGN, "device pointers must be 16-byte aligned");
  brs::DecodeArgs a{};
  a.B = L->B; a.H = L->H; a.Hk = L->H_k; a.k_hi = L->k_hi; a.block = L->block;
  a.decay_per_key = L->decay_per_key; a.mode = wb->mode; a.seed = wb->seed; a.step = step;
  a.head_bytes = head_bytes(L); a.hscale = hadamard_scale(L->d);
  a.packed_in = packed; a.packed_out = packed; a.aux = aux; a.perm = perm;
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.decay = decay; a.o = o;
  a.flags = (uint32_t*)workspace;
  a.s32 = (float*)state32; a.src32 = src32; a.dst32 = dst32;
  a.low_bits = low_bits(L);
  // the CTA-per-head kernel takes every token it supports (its deferred
  // instantiations inside an interval), the general kernel the rest
  const bool cta = brs::decode_cta_supported(L->d, L->storage, L->block, L->k_hi, wb->mode);
  cudaError_t e = (src32 || dst32) && !cta ? brs::launch_decode_deferred(a, L->d, L->hadamard != 0, (cudaStream_t)stream)
                                           : brs::launch_decode(a, L->d, L->storage, L->hadamard != 0, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return ok();
}

brs_status brs_chunk_prefill(const brs_layout* L, const brs_writeback* wb, int64_t step0, int T,
                             void* packed, void* aux, void* workspace, const int16_t* perm,
                             const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             const float* beta, const float* decay, float* o, float* state_dump,
                             void* stream) {
  brs_status st = check_layout(L);
  if (st != BRS_OK) return st;
  if (!wb) return fail(BRS_EINVAL, "writeback is NULL");
  if (L->storage != BRS_STORE_DAMP) return fail(BRS_EUNSUPPORTED, "chunked prefill is built for DAMP storage");
  if (!brs::prefill_supported(L->d, L->block, L->k_hi, wb->C))
    return fail(BRS_EUNSUPPORTED, "chunked prefill is built for d = 128, C = 64, block 128 or 32");
  if (wb->mode < 0 || wb->mode > 6) return fail(BRS_EINVAL, "unknown rounding mode %d", wb->mode);
  if (wb->mode >= BRS_ROUND_DIRECTION)
    return fail(BRS_EUNSUPPORTED, "direction and residual memory are not built for the prefill");
  if (T <= 0 || T % wb->C || step0 < 0 || step0 % wb->C)
    return fail(BRS_EINVAL, "T and step0 must be multiples of C (T = %d, C = %d)", T, wb->C);
  if (!packed || !workspace || !q || !k || !v || !beta || !decay || !o)
    return fail(BRS_EINVAL, "a required pointer is NULL");
  if (wb->mode == BRS_ROUND_ERRFEEDBACK && !aux) return fail(BRS_EINVAL, "error feedback needs the residual buffer");
  const void* ptrs[] = {packed, aux, workspace, perm, q, k, v, beta, decay, o, state_dump};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(BRS_EALIGN, "device pointers must be 16-byte aligned");
  brs::PrefillArgs a{};
  a.B = L->B; a.H = L->H; a.Hk = L->H_k; a.T = T; a.k_hi = L->k_hi; a.block = L->block;
  a.decay_per_key = L->decay_per_key; a.mode = wb->mode; a.seed = wb->seed; a.step0 = step0;
  a.head_bytes = head_bytes(L); a.hscale = hadamard_scale(L->d);
  a.packed = packed; a.aux = aux; a.perm = perm; a.q = q; a.k = k; a.v = v; a.beta = beta;
  a.decay = decay; a.o = o; a.sdump = state_dump; a.flags = (uint32_t*)workspace;
  // the FP32 state between chunks: the caller's workspace after the flag
  // word; then the heads' hand-over counters, zeroed for this call
  a.s0 = (float*)((uint8_t*)workspace + 256);
  a.handover = (uint32_t*)((uint8_t*)workspace + 256 + brs::prefill_tc_scratch_bytes(L->B, L->H));
  cudaError_t e = cudaMemsetAsync(a.handover, 0, (size_t)L->B * L->H * 4, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "prefill hand-over counters");
  a.skip_handover = brs::prefill_withhold();
  a.low_bits = low_bits(L);
  e = brs::launch_prefill_tc(a, L->hadamard != 0, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  return ok();
}

size_t brs_prefill_workspace_bytes(const brs_layout* L) {
  if (check_layout(L) != BRS_OK) return 0;
  if (L->storage != BRS_STORE_DAMP || L->d != 128) {
    fail(BRS_EUNSUPPORTED, "chunked prefill is built for DAMP storage at d = 128");
    return 0;
  }
  ok();
  return 256 + brs::prefill_tc_scratch_bytes(L->B, L->H) + round256((size_t)L->B * L->H * 4);
}

brs_status brs_allocate_bits(int n_rows, int rows_per_group, const double* cost, double avg_bits,
                             int b_min, int b_max, uint32_t offset_unit, uint8_t* bits_out,
                             uint32_t* offsets_out, void* stream) {
  if (n_rows <= 0 || rows_per_group <= 0 || n_rows % rows_per_group)
    return fail(BRS_EINVAL, "n_rows must be a positive multiple of rows_per_group");
  if (rows_per_group > brs::allocate_max_rows())
    return fail(BRS_EUNSUPPORTED, "groups of up to %d rows", brs::allocate_max_rows());
  if (b_min < 1 || b_max > 16 || b_min > b_max) return fail(BRS_EINVAL, "need 1 <= b_min <= b_max <= 16");
  const double tgt = avg_bits * (double)rows_per_group;
  if (tgt != std::floor(tgt) || tgt < (double)b_min * rows_per_group || tgt > (double)b_max * rows_per_group)
    return fail(BRS_EINVAL, "avg_bits * rows_per_group must be an integer inside [b_min, b_max] * rows");
  if (!cost || !bits_out) return fail(BRS_EINVAL, "cost and bits_out are required");
  if (!aligned16(cost) || (offsets_out && !aligned16(offsets_out)))
    return fail(BRS_EALIGN, "device pointers must be 16-byte aligned");
  brs::AllocArgs a{};
  a.groups = n_rows / rows_per_group; a.rows_per_group = rows_per_group; a.b_min = b_min; a.b_max = b_max;
  a.avg_bits = avg_bits; a.offset_unit = offset_unit; a.cost = cost; a.bits = bits_out; a.offsets = offsets_out;
  cudaError_t e = brs::launch_allocate(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "allocate launch");
  return ok();
}

namespace {
// calibration workspace: [flag word, 256 B][states Bc*H*d*d f32][o Bc*H*d f32]
// [err nsamp*Bc*H*d f64][score H*d f64]
struct CalibLayout {
  size_t states, o, err, score, total;
};
CalibLayout calib_layout(const brs_layout* L, int Bc, int T, int every) {
  CalibLayout c{};
  const size_t heads = (size_t)Bc * L->H, d = (size_t)L->d;
  const size_t nsamp = (size_t)(T / every);
  c.states = 256;
  c.o = c.states + round256(heads * d * d * 4);
  c.err = c.o + round256(heads * d * 4);
  c.score = c.err + round256(nsamp * heads * d * 8);
  c.total = c.score + round256((size_t)L->H * d * 8);
  return c;
}
}  // namespace

size_t brs_calibrate_workspace_bytes(const brs_layout* L, int Bc, int T, int every) {
  if (!L || Bc <= 0 || T <= 0 || every <= 0 || L->d <= 0 || L->H <= 0) return 0;
  return calib_layout(L, Bc, T, every).total;
}

brs_status brs_calibrate(const brs_layout* L, int Bc, int T, int every, double tau,
                         const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* beta,
                         const float* decay, void* workspace, double* score_out, int16_t* perm_out,
                         void* stream) {
  if (!L) return fail(BRS_EINVAL, "layout is NULL");
  brs_layout Lc = *L;
  Lc.B = Bc > 0 ? Bc : 1;
  brs_status st = check_layout(&Lc);
  if (st != BRS_OK) return st;
  if (L->storage != BRS_STORE_DAMP) return fail(BRS_EINVAL, "calibration scores the rows of a DAMP layout");
  if (Bc <= 0 || T <= 0 || every <= 0 || every > T) return fail(BRS_EINVAL, "need Bc > 0 and 0 < every <= T");
  if (!(tau > 0.0)) return fail(BRS_EINVAL, "tau must be positive");
  if (!q || !k || !v || !beta || !decay || !workspace || !perm_out)
    return fail(BRS_EINVAL, "q, k, v, beta, decay, workspace and perm_out are required");
  const void* ptrs[] = {q, k, v, beta, decay, workspace, score_out, perm_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(BRS_EALIGN, "device pointers must be 16-byte aligned");
  const CalibLayout cl = calib_layout(L, Bc, T, every);
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* ws = (uint8_t*)workspace;
  float* states = (float*)(ws + cl.states);
  double* score = score_out ? score_out : (double*)(ws + cl.score);
  cudaError_t e = cudaMemsetAsync(ws, 0, cl.o, s);                 // flag word and zero states
  if (e != cudaSuccess) return cuda_fail(e, "calibration state clear");
  brs::DecodeArgs a{};
  a.B = Bc; a.H = L->H; a.Hk = L->H_k; a.k_hi = 0; a.block = L->d;
  a.decay_per_key = L->decay_per_key; a.mode = BRS_ROUND_NEAREST; a.seed = 0;
  a.head_bytes = (size_t)L->d * L->d * 4; a.hscale = hadamard_scale(L->d);
  a.packed_in = states; a.packed_out = states; a.aux = nullptr; a.perm = nullptr;
  a.o = (float*)(ws + cl.o); a.flags = (uint32_t*)ws;
  brs::CalibArgs c{};
  c.B = Bc; c.H = L->H; c.d = L->d; c.block = L->block; c.hadamard = L->hadamard; c.k_hi = L->k_hi;
  c.T = T; c.nsamp = T / every; c.decay_per_key = L->decay_per_key; c.hscale = hadamard_scale(L->d);
  c.levels = (float)((1 << low_bits(L)) - 1);
  c.tau = tau; c.S = states; c.err = (double*)(ws + cl.err); c.decay = decay; c.score = score;
  c.perm = perm_out; c.flags = (uint32_t*)ws;
  const size_t qk = (size_t)Bc * L->H_k * L->d, vv = (size_t)Bc * L->H * L->d, bh = (size_t)Bc * L->H;
  const size_t dk = L->decay_per_key ? vv : bh;
  for (int t = 0; t < T && e == cudaSuccess; ++t) {
    a.step = t;
    a.q = q + t * qk; a.k = k + t * qk; a.v = v + t * vv; a.beta = beta + t * bh; a.decay = decay + t * dk;
    e = brs::launch_decode(a, L->d, BRS_STORE_FP32, false, s);
    if (e == cudaSuccess && (t + 1) % every == 0) {
      c.sample = (t + 1) / every - 1;
      e = brs::launch_calib_sample(c, s);
    }
  }
  if (e == cudaSuccess) e = brs::launch_calib_finish(c, s);
  if (e != cudaSuccess) return cuda_fail(e, "calibration launch");
  return ok();
}

brs_status brs_fetch_errors(void* workspace, uint32_t* flags_out, void* stream) {
  if (!workspace) return fail(BRS_EINVAL, "workspace is NULL");
  uint32_t fl = 0;
  cudaError_t e = cudaMemcpyAsync(&fl, workspace, 4, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, 4, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device flag word");
  if (flags_out) *flags_out = fl;
  if (fl & BRS_FLAG_NONFINITE) return fail(BRS_ENONFINITE, "a kernel met a non-finite state value");
  if (fl & BRS_FLAG_OVERFLOW) return fail(BRS_EOVERFLOW, "an FP16 row, scale or zero overflowed");
  if (fl & BRS_FLAG_TIMEOUT) return fail(BRS_ETIMEOUT, "a bounded device wait gave up");
  if (fl & BRS_FLAG_INVALID) return fail(BRS_EINVAL, "a device-side argument check failed (widths off the budget)");
  return ok();
}

}  // extern "C"
