/*
 * gdn.h - C ABI of the B200 (sm_100a) gated delta-rule decode library.
 *
 * One call advances the recurrent state of a batch of sequences by one token
 * (or a short suffix of tokens) and reads out one output row per token, for
 * every value head. The state of one (sequence, value head) is a K x V
 * matrix S kept in a caller-owned pool, indexed by slot or by page.
 *
 * Per token, with S right-acting (o = q S, rows of S index the key axis):
 *
 *     k^ = k / sqrt(sum k^2 + 1e-6)          (when use_qk_l2norm)
 *     q^ = q / sqrt(sum q^2 + 1e-6) * scale  (scale <= 0 selects 1/sqrt(K))
 *     S  <- diag(alpha) S                    (decay; scalar alpha for GDN)
 *     v_old = k^ S,  u = beta (v - v_old)    (what the key retrieves; residual)
 *     S  <- S + k^T u                        (delta write)
 *     o  = q^ S                              (readout from the updated state)
 *
 * GDN:  alpha = exp(-exp(A_log[hv]) * softplus(a + dt_bias[hv])),
 *       beta  = sigmoid(b).
 * KDA:  alpha[i] = exp(-exp(a_log[hv]) * softplus(raw_gate[i] + dt_bias[hv, i])),
 *       beta = sigmoid(beta_logits) or beta_logits as given.
 * Value head hv reads key head hv / (HV / H).
 *
 * Sources (page titles and sections): Circuit.LLM.Mixer, "Delta rule"
 * (deltaAttnStep) and "Gated memory" (gatedDeltaStep, kdaLiteStep);
 * flashinfer.gdn_paged.gated_delta_rule_decode_paged (description,
 * Parameters, Notes); max.nn.state_space.kda_decode (description,
 * Parameters, Raises); modelopt.torch.quantization.linear_attention.config
 * (LinearAttentionConfig state.block_v and the int8_hadamard32 decode codec,
 * LinearAttentionDecodeConfig readout and state_codec) and
 * ...linear_attention.decode (recurrent_decode: fp8_e4m3, block_v=64;
 * recurrent_decode_reference: an empty call performs no write).
 *
 * Conventions of every entry point:
 *  - Tensor pointers are DEVICE pointers owned by the caller; the library
 *    allocates nothing and keeps no state between calls. Every tensor is
 *    contiguous row-major with the shape given below. q, k, v, raw_gate,
 *    the KDA dt_bias, out and the pool data must be 16-byte aligned; every
 *    other pointer only to its element size. The library cannot see tensor
 *    extents: the shapes below are the caller's contract.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and runs asynchronously; a return of GDN_OK means the launch
 *    was enqueued, not that it finished.
 *  - The return value is a gdn_status. GDN_ERR_INVALID_ARG: a shape, dtype,
 *    enum value, pointer or struct_size is wrong (nothing is launched, like
 *    the ValueError of kda_decode). GDN_ERR_UNSUPPORTED: a known option that
 *    this library does not implement (nothing is launched). GDN_ERR_CUDA: the
 *    launch failed (cudaGetLastError after the launch).
 *  - Index VALUES (slots, pages, offsets) are not checked on the host, as the
 *    paged page says of precomputed slots. The kernel skips a unit whose
 *    index is out of range, writes zeros to its outputs, leaves the pool
 *    untouched and ORs a GDN_FLAG_* bit into *err_flags when err_flags is not
 *    NULL (a device int32 the caller zeroes). It never traps.
 *  - A negative slot index marks a padded sequence: its outputs are zero, no
 *    state is read or written, no flag is raised.
 *  - B == 0 (or no tokens) returns GDN_OK and launches nothing.
 *  - Preconditions that are not checked: the write slots/pages of one call
 *    are distinct, and no write page is another sequence's read page.
 */
#ifndef GDN_B200_GDN_H
#define GDN_B200_GDN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* gdn_stream_t;

typedef enum gdn_status {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = -1,
  GDN_ERR_UNSUPPORTED = -2,
  GDN_ERR_CUDA = -3
} gdn_status;

typedef enum gdn_dtype {
  GDN_F32 = 0,
  GDN_BF16 = 1,
  GDN_FP8_E4M3 = 2, /* state only: codes + one fp32 scale per [K, block_v] tile */
  GDN_INT8_H32 = 3  /* state only: int8_hadamard32, int8 codes of each
                       (key channel, 32 values) group rotated by H32/sqrt(32),
                       + one fp32 scale per group */
} gdn_dtype;

typedef enum gdn_index_dtype { GDN_I32 = 0, GDN_I64 = 1 } gdn_index_dtype;

/* Storage order of one [K, V] state. K_FIRST: [K][V], V contiguous.
 * V_FIRST: [V][K], K contiguous (the paged pool's [num_pages, HV, V, K]). */
typedef enum gdn_layout { GDN_K_FIRST = 0, GDN_V_FIRST = 1 } gdn_layout;

/* Which state o is read from when the state is stored in bf16, fp8 or int8:
 * WORKING = the fp32 state before it is rounded to its storage format,
 * STORED = the state after that rounding. Equal for fp32 states. */
typedef enum gdn_readout { GDN_READOUT_WORKING = 0, GDN_READOUT_STORED = 1 } gdn_readout;

typedef enum kda_gate_mode { KDA_GATE_ORIGINAL = 0, KDA_GATE_SAFE = 1 } kda_gate_mode;
typedef enum kda_beta_mode { KDA_BETA_LOGITS = 0, KDA_BETA_PROBABILITY = 1 } kda_beta_mode;

/* Bits ORed into *err_flags by the kernels. */
#define GDN_FLAG_SLOT_RANGE 1 /* a slot index >= num_slots */
#define GDN_FLAG_PAGE_RANGE 2 /* a page id outside [0, num_slots) or a CSR position outside [0, nnz) */
#define GDN_FLAG_PAGE_TABLE 4 /* empty page list, last_page_len outside [1, page_size], or a new page with no page before it */
#define GDN_FLAG_SEQLENS 8    /* cu_seqlens not non-decreasing within [0, total_tokens] */
#define GDN_FLAG_TIMEOUT 16   /* a bounded wait of a kernel (an MMA completion) gave up after 1 s; outputs of the call are incomplete */

/* The recurrent-state pool.
 *  data:      [num_slots, HV, K, V] logically, stored per `layout` in
 *             `dtype` (fp8: one uint8 E4M3 code per element; int8: one int8
 *             code per element).
 *  scales:    fp8: [num_slots, HV, V / block_v] fp32, one per [K, block_v]
 *             tile. int8_hadamard32: [num_slots, HV, V / 32, K] fp32, one
 *             per (32-value group, key channel), for either layout, 16-byte
 *             aligned. NULL otherwise.
 *  block_v:   fp8 tile width along V (64); ignored for the other dtypes.
 * fp8 states are decoded as code * scale when read and re-encoded with a
 * fresh scale (amax / 448) after every token.
 * int8_hadamard32 (ModelOpt linear-attention config: the decode codec whose
 * scales are fixed to one key channel and 32 values): for key channel k and
 * values 32g..32g+31, y = R x with R = H32 / sqrt(32) (Sylvester order,
 * symmetric, R R = I), s = amax|y| / 127, code = y / s rounded to nearest
 * even; decoding is R (code * s). Re-encoded after every token. Needs
 * V % 64 == 0 (else GDN_ERR_UNSUPPORTED). */
typedef struct gdn_state_pool {
  void* data;
  float* scales;
  int64_t num_slots;
  int32_t dtype;   /* gdn_dtype */
  int32_t layout;  /* gdn_layout */
  int32_t block_v;
  int32_t reserved;
} gdn_state_pool;

/* GDN decode on a slot pool: B sequences, T >= 1 tokens each.
 * Source: flashinfer.gdn_paged.gated_delta_rule_decode_paged, Parameters
 * (q, k, v, A_log, a, dt_bias, b, scale and use_qk_l2norm, which the page
 * defines by gated_delta_rule_decode_pretranspose), with the state addressed by slot
 * instead of by page; the step is Circuit.LLM.Mixer, "Gated memory"
 * (gatedDeltaStep); the per-token storage and readout of a T > 1 suffix are
 * modelopt...linear_attention.decode (recurrent_decode_reference: token
 * write events) and ...linear_attention.config
 * (LinearAttentionDecodeConfig: readout, state_codec).
 *  q, k     [B, T, H, K]   in_dtype (F32 or BF16)
 *  v        [B, T, HV, V]  in_dtype
 *  a, b     [B, T, HV]     in_dtype (gate and beta pre-activations)
 *  A_log    [HV] fp32, dt_bias [HV] fp32
 *  state_indices [B] (index_dtype): pool slot of each sequence; read and
 *                written in place after the last token.
 *  out      [B, T, HV, V]  out_dtype (F32 or BF16)
 * Constraints: HV % H == 0; K and V in {32, 64, 128, 256}; fp8 state needs
 * block_v == 64 and V % 64 == 0; int8_hadamard32 state needs V % 64 == 0.
 * T > 1 runs the tokens of each sequence in order with the state held on
 * chip (a short suffix); bf16/fp8/int8 states pass through their storage
 * format after every token. */
typedef struct gdn_decode_slots_params {
  int32_t struct_size; /* sizeof(gdn_decode_slots_params) */
  int32_t B, T, H, HV, K, V;
  int32_t in_dtype, out_dtype, index_dtype, readout, use_qk_l2norm;
  float scale;         /* <= 0 selects 1/sqrt(K) */
  const void* q;
  const void* k;
  const void* v;
  const void* a;
  const void* b;
  const float* A_log;
  const float* dt_bias;
  const void* state_indices;
  void* out;
  int32_t* err_flags;  /* may be NULL */
  gdn_state_pool pool;
} gdn_decode_slots_params;

int gdn_decode_slots(const gdn_decode_slots_params* p, gdn_stream_t stream);

/* GDN decode of the last T tokens of every sequence on a paged pool
 * (num_slots = num_pages); a page holds the state after its last token.
 * Source: flashinfer.gdn_paged.gated_delta_rule_decode_paged (the
 * description's copy-on-new-page rule; Parameters: state_pool
 * [num_pages, HV, V, K], page_indices / page_indptr CSR table,
 * last_page_len in [1, page_size] including the decoded token, slots not
 * checked against the table; Notes: a new-page sequence owns two pages).
 * T > 1 is this library's reading of the same rule for a short suffix
 * (modelopt...linear_attention.config, LinearAttentionDecodeConfig, which
 * runs the recurrence over a suffix after a per-sequence prefix).
 *  q, k [B, T, H, K]; v [B, T, HV, V]; a, b [B, T, HV]; A_log, dt_bias [HV];
 *  page_indices [nnz], page_indptr [B+1], last_page_len [B] (index_dtype):
 *    CSR page table; the decoded tokens are the last T tokens of their
 *    sequence and last_page_len counts the tokens of the last page,
 *    including them (in [1, page_size]).
 *  out [B, T, HV, V].
 * T == 1, copy-on-new-page: when last_page_len[b] == 1 the state is read
 * from the page before the last and written to the last page, so the
 * previous page (possibly shared) is not modified; otherwise the last page
 * is updated in place. A sequence that opens a page must own at least two
 * pages. page_size <= 0 disables the last_page_len upper-bound check.
 *  slots: optional [B, 2] int64 rows (read_page, write_page) as written by
 *    gdn_paged_decode_slots for the same table; used as given, not checked
 *    against the table. NULL: the kernel resolves the rows itself in its
 *    prologue (no extra launch).
 * T > 1 (a short suffix; page_size required, slots must be NULL): with
 * L = (pages - 1) * page_size + last_page_len tokens, the suffix is
 * positions L-T .. L-1 and at least one token must precede it. The state
 * is read from the page of position L-T-1; every page whose last position
 * falls inside the suffix receives the state after that position; the final
 * state goes to the last page. Pages before the read page are untouched. */
typedef struct gdn_decode_paged_params {
  int32_t struct_size; /* sizeof(gdn_decode_paged_params) */
  int32_t B, T, H, HV, K, V;
  int32_t in_dtype, out_dtype, index_dtype, readout, use_qk_l2norm;
  int32_t page_size;
  float scale;
  int64_t nnz;         /* length of page_indices */
  const void* q;
  const void* k;
  const void* v;
  const void* a;
  const void* b;
  const float* A_log;
  const float* dt_bias;
  const void* page_indices;
  const void* page_indptr;
  const void* last_page_len;
  const int64_t* slots; /* may be NULL */
  void* out;            /* [B, 1, HV, V] */
  int32_t* err_flags;   /* may be NULL */
  gdn_state_pool pool;
} gdn_decode_paged_params;

int gdn_decode_paged(const gdn_decode_paged_params* p, gdn_stream_t stream);

/* Prefill (or continued prefill) on a paged pool.
 * Source: flashinfer.gdn_paged.gated_delta_rule_decode_paged, Parameters
 * (the CSR page table is the one chunk_gated_delta_rule_paged takes); the
 * run is the scan of single steps, Circuit.LLM.Mixer, "Gated memory"
 * (gatedDeltaPrefill), computed in 64-token chunks where the state is fp32
 * (modelopt...linear_attention.config, LinearAttentionConfig: chunk_size 64,
 * exact solve).
 * Appends a varlen run of tokens to every sequence. Sequence b gets n = cu_seqlens[b+1] - cu_seqlens[b]
 * new tokens, the last n of its L = (pages - 1) * page_size + last_page_len
 * tokens (the page table already includes them). The run is the scan of
 * single steps over its tokens. The state starts at zero when the sequence
 * has no earlier token (L == n), else it is read from the page of position
 * L-n-1; every page that fills inside the run receives the state after its
 * last token and the final state goes to the last page. n == 0 leaves the
 * sequence untouched.
 *  q, k [total_tokens, H, K]; v [total_tokens, HV, V]; a, b [total_tokens, HV]
 *  (in_dtype); A_log, dt_bias [HV] fp32; cu_seqlens [B+1] int32;
 *  page_indices [nnz], page_indptr [B+1], last_page_len [B] (index_dtype);
 *  out [total_tokens, HV, V] (out_dtype). page_size > 0 is required. */
typedef struct gdn_prefill_paged_params {
  int32_t struct_size; /* sizeof(gdn_prefill_paged_params) */
  int32_t B, total_tokens, H, HV, K, V;
  int32_t in_dtype, out_dtype, index_dtype, readout, use_qk_l2norm;
  int32_t page_size;
  float scale;
  int64_t nnz;
  const void* q;
  const void* k;
  const void* v;
  const void* a;
  const void* b;
  const float* A_log;
  const float* dt_bias;
  const int32_t* cu_seqlens;
  const void* page_indices;
  const void* page_indptr;
  const void* last_page_len;
  void* out;
  int32_t* err_flags;  /* may be NULL */
  gdn_state_pool pool;
} gdn_prefill_paged_params;

int gdn_prefill_paged(const gdn_prefill_paged_params* p, gdn_stream_t stream);

/* Resolve the (read_page, write_page) rows of a paged decode once per step,
 * to be shared by every layer's gdn_decode_paged call.
 * Source: flashinfer.gdn_paged.gated_delta_rule_decode_paged, Parameters:
 * slots (rows computed once for a page table and reused by the layers of a
 * step; a decode given none computes them itself).
 *  page_indices [nnz], page_indptr [B+1], last_page_len [B] (index_dtype);
 *  slots_out [B, 2] int64 (device). Rows of malformed sequences are (-1, -1)
 *  and raise a GDN_FLAG_* bit. */
int gdn_paged_decode_slots(const void* page_indices, const void* page_indptr,
                           const void* last_page_len, int32_t index_dtype, int64_t nnz,
                           int32_t B, int64_t num_pages, int32_t page_size,
                           int64_t* slots_out, int32_t* err_flags, gdn_stream_t stream);

/* KDA (per-key-channel gate) over varlen sequences on a slot pool.
 * Source: max.nn.state_space.kda_decode (description, Parameters, Raises);
 * the step is Circuit.LLM.Mixer, "Gated memory" (kdaLiteStep).
 *  q, k        [total_tokens, Hk, K]  in_dtype
 *  v           [total_tokens, HV, V]  in_dtype
 *  raw_gate    [total_tokens, HV, K]  in_dtype (before dt_bias is added)
 *  beta_logits [total_tokens, HV]     in_dtype
 *  a_log [HV] fp32; dt_bias [HV, K] fp32
 *  cu_seqlens  [B+1] int32 exclusive prefix offsets into the token axis
 *  state_indices [B] int32
 *  out         [total_tokens, HV, V]  out_dtype
 * q and k are always L2-normalised and q scaled by 1/sqrt(K). A sequence of
 * zero tokens leaves its slot untouched. gate_mode KDA_GATE_SAFE returns
 * GDN_ERR_UNSUPPORTED (its lower bound is not defined by the source).
 * State dtypes: any gdn_dtype, with the pool rules above. */
typedef struct kda_decode_varlen_params {
  int32_t struct_size; /* sizeof(kda_decode_varlen_params) */
  int32_t B, total_tokens, Hk, HV, K, V;
  int32_t in_dtype, out_dtype, gate_mode, beta_mode, readout;
  const void* q;
  const void* k;
  const void* v;
  const void* raw_gate;
  const void* beta_logits;
  const float* a_log;
  const float* dt_bias;
  const int32_t* cu_seqlens;
  const int32_t* state_indices;
  void* out;
  int32_t* err_flags;  /* may be NULL */
  gdn_state_pool pool;
} kda_decode_varlen_params;

int kda_decode_varlen(const kda_decode_varlen_params* p, gdn_stream_t stream);

/* fp8 E4M3 tile codec over n_states states of [K, V] (stored per layout).
 * Source: modelopt...linear_attention.config, LinearAttentionConfig
 * (state.block_v: one dynamic scale per [Dk, block_v] tile) and
 * ...linear_attention.decode (recurrent_decode: state_format fp8_e4m3,
 * block_v=64).
 * Per [K, block_v] tile: amax = max|x|, s = amax / 448, r = 1 / s (fp32,
 * round to nearest), code = E4M3(x * r) rounded to nearest even and
 * saturated to +-448; a tile with amax == 0 (or r not finite) stores s = 0
 * and all codes 0. Decoding is value(code) * s.
 *  src/dst [n_states, K, V] or [n_states, V, K] fp32; codes same shape
 *  uint8; scales [n_states, V / block_v] fp32. block_v == 64. */
int gdn_state_quantize_fp8(const float* src, uint8_t* codes, float* scales, int64_t n_states,
                           int32_t K, int32_t V, int32_t block_v, int32_t layout,
                           gdn_stream_t stream);
int gdn_state_dequantize_fp8(const uint8_t* codes, const float* scales, float* dst,
                             int64_t n_states, int32_t K, int32_t V, int32_t block_v,
                             int32_t layout, gdn_stream_t stream);

/* int8_hadamard32 codec over n_states states of [K, V] (stored per layout).
 * Source: modelopt...linear_attention.config, LinearAttentionConfig (the
 * decode codec int8_hadamard32 fixes scales to one key channel and 32
 * values) and LinearAttentionDecodeConfig.state_codec.
 * The pool's code format on its own (see gdn_state_pool). Everything in
 * binary32 with one fixed rounding order, so results are reproducible bit
 * for bit: the 32 values of a group are rotated by the fast Walsh-Hadamard
 * butterflies of span 1, 2, 4, 8, 16 ((a, b) -> (a + b, a - b)), each then
 * multiplied by the binary32 nearest 1/sqrt(32); s = amax / 127 and
 * r = 1 / s round to nearest; code = y * r (rounded product) rounded to the
 * nearest integer, ties to even (clamped to +-127, which finite inputs
 * never reach). A group whose amax is 0, or whose r is not finite, stores
 * s = 0 and codes 0. Decoding multiplies code * s (rounded) and applies the
 * same butterflies and product.
 *  src/dst [n_states, K, V] or [n_states, V, K] fp32; codes same shape
 *  int8; scales [n_states, V / 32, K] fp32. All pointers 16-byte aligned. */
int gdn_state_quantize_int8h32(const float* src, int8_t* codes, float* scales, int64_t n_states,
                               int32_t K, int32_t V, int32_t layout, gdn_stream_t stream);
int gdn_state_dequantize_int8h32(const int8_t* codes, const float* scales, float* dst,
                                 int64_t n_states, int32_t K, int32_t V, int32_t layout,
                                 gdn_stream_t stream);

/* Static description of a status code (never NULL). */
const char* gdn_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* GDN_B200_GDN_H */
