// Device helpers shared by the decode kernels: state storage formats, vector
// loads and stores, the token prologue (activations, norms) and the
// resolution of a (sequence) unit to its pool slots or pages.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

// ---------------------------------------------------------------------------
// enums shared with the host side (values match include/gdn.h)
// ---------------------------------------------------------------------------
enum StateFmt : int { ST_F32 = 0, ST_BF16 = 1, ST_FP8 = 2, ST_I8H = 3 };
enum Layout : int { L_KFIRST = 0, L_VFIRST = 1 };
enum IndexMode : int { IDX_SLOTS = 0, IDX_PAGED = 1 };
enum GateKind : int { GATE_SCALAR = 0, GATE_VECTOR = 1 };

// run-time flags of one call
constexpr int F_IN_BF16 = 1;
constexpr int F_OUT_BF16 = 2;
constexpr int F_IDX64 = 4;
constexpr int F_L2NORM = 8;
constexpr int F_BETA_PROB = 16;
constexpr int F_READOUT_STORED = 32;
constexpr int F_VARLEN = 64;

// err_flags bits (GDN_FLAG_* in the public header)
constexpr int E_SLOT_RANGE = 1;
constexpr int E_PAGE_RANGE = 2;
constexpr int E_PAGE_TABLE = 4;
constexpr int E_SEQLENS = 8;

constexpr float kL2Eps = 1e-6f;
constexpr float kE4M3Max = 448.0f;
constexpr unsigned kFull = 0xffffffffu;

// Everything one launch needs. Token-major inputs: GDN [B, T, ...] is the
// token axis tok = b * T + t; KDA uses the varlen token axis directly.
struct StepParams {
  const void* q;        // [tok, H, K]
  const void* k;        // [tok, H, K]
  const void* v;        // [tok, HV, V]
  const void* gate;     // GDN a [tok, HV]; KDA raw_gate [tok, HV, K]
  const void* beta;     // [tok, HV]
  const float* A_log;   // [HV]
  const float* dt_bias; // GDN [HV]; KDA [HV, K]
  void* pool;           // [num_slots, HV, state]
  float* scales;        // fp8: [num_slots, HV, V / 64]; int8: [num_slots, HV, V / 32, K]
  const void* idx;      // slots: state_indices [B]; paged: page_indices [nnz]
  const void* indptr;   // paged: page_indptr [B+1]; varlen: cu_seqlens [B+1] int32
  const void* lastlen;  // paged: last_page_len [B]
  const int32_t* cu;    // paged prefill: cu_seqlens [B+1]
  const int64_t* rows;  // paged: precomputed (read, write) [B, 2] or null
  void* out;            // [tok, HV, V]
  int32_t* err;         // optional
  int64_t num_slots;
  int64_t nnz;
  int B, T, H, HV, V;
  int G;                // value heads per key head, HV / H
  int n_vtiles;
  int total_tokens;
  int page_size;
  float scale;
  int flags;
};

// ---------------------------------------------------------------------------
// state formats: 16 bytes hold EPL elements
// ---------------------------------------------------------------------------
template <int SDT> struct StateTraits;
template <> struct StateTraits<ST_F32> { static constexpr int EPL = 4, BYTES = 4; };
template <> struct StateTraits<ST_BF16> { static constexpr int EPL = 8, BYTES = 2; };
template <> struct StateTraits<ST_FP8> { static constexpr int EPL = 16, BYTES = 1; };
template <> struct StateTraits<ST_I8H> { static constexpr int EPL = 16, BYTES = 1; };

// Streaming 16-byte load/store: the state is touched once per launch, so it
// should not displace anything in L1/L2 ("evict first").
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void st_stream16(void* p, uint4 v) {
  __stcs(reinterpret_cast<uint4*>(p), v);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Round to the nearest bf16 (ties to even) and keep it as fp32.
__device__ __forceinline__ float round_bf16(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // one paired conversion
  return *reinterpret_cast<const uint32_t*>(&v);
}

// fp8 E4M3 codes: hardware conversions; decode is exact (through half),
// encode rounds to nearest even and saturates to 448.
// Four E4M3 bytes of a word (byte i = x[i]) <-> four floats, converting the
// word's two halves in place (no masking or shifting to extract them).
__device__ __forceinline__ void e4m3x4_to_float4(uint32_t w, float* x) {
  uint32_t h0, h1;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, lo;\n\tcvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
      : "=r"(h0), "=r"(h1)
      : "r"(w));
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h0));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&h1));
  x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}
__device__ __forceinline__ uint32_t float4_to_e4m3x4(float x0, float x1, float x2, float x3) {
  uint32_t w;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\tcvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(w)
      : "f"(x0), "f"(x1), "f"(x2), "f"(x3));
  return w;
}

// ---------------------------------------------------------------------------
// int8_hadamard32 codes: each (key channel, 32 values) group of the state is
// held rotated by R = H32 / sqrt(32) (Sylvester order), as int8 codes with one
// fp32 scale s = amax / 127 per group.
// ---------------------------------------------------------------------------
constexpr float kInt8Max = 127.0f;
// 1.5 * 2^23: adding it to |x| < 2^22 rounds x to an integer (ties to even)
// and leaves that integer in the low mantissa bits, two's complement.
constexpr float kRoundMagic = 12582912.0f;
// 2^23 + 128: a byte b placed under the exponent of 2^23 reads 2^23 + b.
constexpr float kByteBias = 8388736.0f;

// The binary32 nearest to 1/sqrt(32) (a quarter of the one nearest 1/sqrt(2)).
__device__ __forceinline__ float inv_sqrt32() { return __uint_as_float(0x3E3504F3u); }

// 4 int8 codes (one word, low byte first) -> their values as floats, exactly:
// flipping the sign bit of a byte gives code + 128.
__device__ __forceinline__ void i8x4_to_float(uint32_t w, float* x) {
  const uint32_t u = w ^ 0x80808080u;
  const float2 bias = make_float2(-kByteBias, -kByteBias);
  const float2 lo = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540)),
                                           __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541))), bias);
  const float2 hi = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542)),
                                           __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543))), bias);
  x[0] = lo.x; x[1] = lo.y; x[2] = hi.x; x[3] = hi.y;
}

// 4 floats already multiplied by the group's r (|x| <= 127.5 for finite
// states) -> 4 int8 codes, nearest integer with ties to even.
__device__ __forceinline__ uint32_t float_to_i8x4(float a, float b, float c, float d) {
  const float2 m = make_float2(kRoundMagic, kRoundMagic);
  const float2 ab = __fadd2_rn(make_float2(a, b), m);
  const float2 cd = __fadd2_rn(make_float2(c, d), m);
  const uint32_t lo = __byte_perm(__float_as_uint(ab.x), __float_as_uint(ab.y), 0x0040);
  const uint32_t hi = __byte_perm(__float_as_uint(cd.x), __float_as_uint(cd.y), 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

// Group scale from the group's amax: s = amax / 127 and r = 1 / s, both
// correctly rounded; a zero group (or one whose r overflows) stores s = 0
// and codes 0 (signalled by r = 0).
__device__ __forceinline__ void h32_scale_of(float amax, float& s, float& r) {
  s = __fdiv_rn(amax, kInt8Max);
  r = __frcp_rn(s);
  if (!(amax > 0.0f) || isinf(r)) { s = 0.0f; r = 0.0f; }
}

// Unnormalised 32-point Walsh-Hadamard transform of one value per lane
// (lane = position in the group): butterflies of span 1, 2, 4, 8, 16.
__device__ __forceinline__ float fwht_lanes(float x, int lane) {
#pragma unroll
  for (int span = 1; span < 32; span <<= 1) {
    const float p = __shfl_xor_sync(kFull, x, span);
    x = (lane & span) ? __fsub_rn(p, x) : __fadd_rn(x, p);
  }
  return x;
}

// The same transform of 32 values held by one thread, in the same stage
// order: stage `span` turns the pair at (i, i + span), i & span == 0, into
// (a + b, a - b).
__device__ __forceinline__ void fwht32_regs(float* x) {
#pragma unroll
  for (int span = 1; span < 32; span <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((i & span) == 0) {
        const float a = x[i], b = x[i + span];
        x[i] = __fadd_rn(a, b);
        x[i + span] = __fsub_rn(a, b);
      }
    }
  }
}

// Decode 16 stored bytes into EPL floats (fp8 and int8 codes are returned
// unscaled).
template <int SDT>
__device__ __forceinline__ void decode16(uint4 raw, float* x) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  if constexpr (SDT == ST_F32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = __uint_as_float(w[i]);
  } else if constexpr (SDT == ST_BF16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) { x[2 * i] = bf16_lo(w[i]); x[2 * i + 1] = bf16_hi(w[i]); }
  } else if constexpr (SDT == ST_I8H) {
#pragma unroll
    for (int i = 0; i < 4; ++i) i8x4_to_float(w[i], x + 4 * i);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) e4m3x4_to_float4(w[i], x + 4 * i);
  }
}

// Encode EPL floats into 16 stored bytes. For fp8 and int8 the caller passes
// x * r.
template <int SDT>
__device__ __forceinline__ uint4 encode16(const float* x) {
  uint32_t w[4];
  if constexpr (SDT == ST_F32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = __float_as_uint(x[i]);
  } else if constexpr (SDT == ST_BF16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
  } else if constexpr (SDT == ST_I8H) {
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = float_to_i8x4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = float4_to_e4m3x4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// 8 stored fp8 bytes <-> 8 floats (codes unscaled)
__device__ __forceinline__ void decode8_fp8(uint2 raw, float* x) {
  e4m3x4_to_float4(raw.x, x);
  e4m3x4_to_float4(raw.y, x + 4);
}
__device__ __forceinline__ uint2 encode8_fp8(const float* x) {
  return make_uint2(float4_to_e4m3x4(x[0], x[1], x[2], x[3]), float4_to_e4m3x4(x[4], x[5], x[6], x[7]));
}

// Running max of |x| (m >= 0): the absolute value is an operand modifier of
// the max, and the three-input max of sm_100 takes two elements at once.
__device__ __forceinline__ float absmax_acc(float m, float x) { return fmaxf(m, fabsf(x)); }
__device__ __forceinline__ float absmax_acc2(float m, float x, float y) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(m), "f"(fabsf(x)), "f"(fabsf(y)));
  return r;
}

// fp8 tile scale from the tile's amax: s = amax / 448 and r = 1 / s, both
// correctly rounded; a zero tile (or one whose r overflows) stores s = 0 and
// codes 0 (signalled by r = 0).
__device__ __forceinline__ void fp8_scale_of(float amax, float& s, float& r) {
  s = __fdiv_rn(amax, kE4M3Max);
  r = __frcp_rn(s);
  if (!(amax > 0.0f) || isinf(r)) { s = 0.0f; r = 0.0f; }
}
// The value handed to the E4M3 encoder: x * r, and +0 for a zero tile (so
// that negative inputs do not encode as -0).
__device__ __forceinline__ float fp8_prescale(float x, float r) {
  return r == 0.0f ? 0.0f : __fmul_rn(x, r);
}

// ---------------------------------------------------------------------------
// token inputs
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ld_in1(const void* base, int64_t i, bool bf16) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i])
              : reinterpret_cast<const float*>(base)[i];
}

// The 32-bit word holding input element i (bf16: the aligned pair), and the
// element read back out of it.
__device__ __forceinline__ const void* in_word(const void* base, int64_t i, bool bf16) {
  return bf16 ? static_cast<const void*>(reinterpret_cast<const uint32_t*>(base) + (i >> 1))
              : static_cast<const void*>(reinterpret_cast<const float*>(base) + i);
}
__device__ __forceinline__ float in_from_word(uint32_t w, int64_t i, bool bf16) {
  return bf16 ? ((i & 1) ? bf16_hi(w) : bf16_lo(w)) : __uint_as_float(w);
}

// N contiguous input elements starting at element i (i a multiple of N,
// base 16-byte aligned), widened to fp32.
template <int N>
__device__ __forceinline__ void ld_in_vec(const void* base, int64_t i, bool bf16, float* x) {
  if (bf16) {
    const __nv_bfloat16* p = reinterpret_cast<const __nv_bfloat16*>(base) + i;
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int c = 0; c < N / 8; ++c) {
        uint4 r = reinterpret_cast<const uint4*>(p)[c];
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) { x[8 * c + 2 * j] = bf16_lo(w[j]); x[8 * c + 2 * j + 1] = bf16_hi(w[j]); }
      }
    } else if constexpr (N == 4) {
      uint2 r = *reinterpret_cast<const uint2*>(p);
      x[0] = bf16_lo(r.x); x[1] = bf16_hi(r.x); x[2] = bf16_lo(r.y); x[3] = bf16_hi(r.y);
    } else if constexpr (N == 2) {
      uint32_t r = *reinterpret_cast<const uint32_t*>(p);
      x[0] = bf16_lo(r); x[1] = bf16_hi(r);
    } else {
#pragma unroll
      for (int j = 0; j < N; ++j) x[j] = __bfloat162float(p[j]);
    }
  } else {
    const float* p = reinterpret_cast<const float*>(base) + i;
    if constexpr (N % 4 == 0) {
#pragma unroll
      for (int c = 0; c < N / 4; ++c) {
        float4 r = reinterpret_cast<const float4*>(p)[c];
        x[4 * c] = r.x; x[4 * c + 1] = r.y; x[4 * c + 2] = r.z; x[4 * c + 3] = r.w;
      }
    } else if constexpr (N == 2) {
      float2 r = *reinterpret_cast<const float2*>(p);
      x[0] = r.x; x[1] = r.y;
    } else {
#pragma unroll
      for (int j = 0; j < N; ++j) x[j] = p[j];
    }
  }
}

__device__ __forceinline__ void st_out1(void* base, int64_t i, float x, bool bf16) {
  if (bf16) reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(x);
  else reinterpret_cast<float*>(base)[i] = x;
}

// ---------------------------------------------------------------------------
// activations (fp32)
// ---------------------------------------------------------------------------
__device__ __forceinline__ float softplus_f(float x) {
  return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}
// alpha = exp(-exp(A_log) * softplus(x)), x = gate pre-activation + dt_bias
__device__ __forceinline__ float decay_of(float exp_A_log, float x) {
  return expf(-exp_A_log * softplus_f(x));
}
__device__ __forceinline__ float sigmoid_f(float x) { return 1.0f / (1.0f + expf(-x)); }

template <int LANES>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int o = LANES / 2; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
  return x;
}
template <int LANES>
__device__ __forceinline__ float group_max(float x) {
#pragma unroll
  for (int o = LANES / 2; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, o));
  return x;
}

// ---------------------------------------------------------------------------
// unit resolution
// ---------------------------------------------------------------------------
enum UnitStatus : int { U_OK = 0, U_PAD = 1, U_SKIP = 2 };

struct Unit {
  int64_t src, dst;  // pool slot (or page) read and written
  int tok0, tok1;    // token range
  int status;
  int err;
  int64_t p0, L;     // paged suffix: first CSR position and tokens of the sequence
  int T;             // paged suffix: tokens of the run
  bool fresh;        // paged prefill of a sequence with no earlier token: S starts at 0
};

__device__ __forceinline__ int64_t ld_index(const void* base, int64_t i, bool i64) {
  return i64 ? reinterpret_cast<const int64_t*>(base)[i]
             : static_cast<int64_t>(reinterpret_cast<const int32_t*>(base)[i]);
}

// Copy-on-new-page rule of a paged decode (flashinfer gdn_paged, description):
// the decoded token sits in the sequence's last page; if it opens that page
// (last_page_len == 1) the state is read from the page before it, otherwise
// the last page is read and updated in place.
__device__ __forceinline__ void resolve_page_rows(const void* indices, const void* indptr,
                                                  const void* lastlen, bool i64, int64_t nnz,
                                                  int64_t num_pages, int page_size, int b,
                                                  int64_t& read, int64_t& write, int& err) {
  read = write = -1;
  const int64_t p0 = ld_index(indptr, b, i64);
  const int64_t p1 = ld_index(indptr, b + 1, i64);
  const int64_t len = ld_index(lastlen, b, i64);
  if (p0 < 0 || p1 > nnz) { err |= E_PAGE_RANGE; return; }
  if (p1 <= p0 || len < 1 || (page_size > 0 && len > page_size)) { err |= E_PAGE_TABLE; return; }
  if (len == 1 && p1 - 1 <= p0) { err |= E_PAGE_TABLE; return; }
  const int64_t w = ld_index(indices, p1 - 1, i64);
  const int64_t r = (len == 1) ? ld_index(indices, p1 - 2, i64) : w;
  if (w < 0 || w >= num_pages || r < 0 || r >= num_pages) { err |= E_PAGE_RANGE; return; }
  read = r;
  write = w;
}

// The last n tokens of a paged sequence: a page holds the state after its
// last token, so with L = (pages - 1) * page_size + last_page_len the state
// is read from the page of position L-n-1 and the final state goes to the
// last page (pages filled inside the run are written by the kernel's token
// loop, see suffix_snapshot_page). With allow_fresh, a sequence with no
// earlier token (L == n) starts from a zero state.
__device__ __forceinline__ void resolve_suffix(const StepParams& p, int b, int n, bool allow_fresh, Unit& u) {
  const bool i64 = (p.flags & F_IDX64) != 0;
  u.src = u.dst = -1;
  u.T = n;
  const int64_t p0 = ld_index(p.indptr, b, i64);
  const int64_t p1 = ld_index(p.indptr, b + 1, i64);
  const int64_t len = ld_index(p.lastlen, b, i64);
  if (p0 < 0 || p1 > p.nnz) { u.err |= E_PAGE_RANGE; return; }
  if (p1 <= p0 || len < 1 || len > p.page_size) { u.err |= E_PAGE_TABLE; return; }
  const int64_t L = (p1 - p0 - 1) * p.page_size + len;
  const bool fresh = allow_fresh && L == n;
  if (!fresh && L < n + 1) { u.err |= E_PAGE_TABLE; return; }
  const int64_t r = fresh ? 0 : ld_index(p.idx, p0 + (L - n - 1) / p.page_size, i64);
  const int64_t w = ld_index(p.idx, p1 - 1, i64);
  if (r < 0 || r >= p.num_slots || w < 0 || w >= p.num_slots) { u.err |= E_PAGE_RANGE; return; }
  u.src = fresh ? -1 : r;
  u.dst = w;
  u.p0 = p0;
  u.L = L;
  u.fresh = fresh;
}

// Page that receives the state after run token t (not the last one), or -1:
// the page whose last position is L-n+t, when that position closes a page.
__device__ __forceinline__ int64_t suffix_snapshot_page(const StepParams& p, const Unit& u, int t) {
  const int64_t pos = u.L - u.T + t;
  if (t >= u.T - 1 || (pos % p.page_size) != p.page_size - 1) return -1;
  return ld_index(p.idx, u.p0 + pos / p.page_size, (p.flags & F_IDX64) != 0);
}

template <int IDX>
__device__ __forceinline__ Unit resolve_unit(const StepParams& p, int b) {
  Unit u;
  u.status = U_OK;
  u.err = 0;
  u.p0 = 0;
  u.L = 0;
  u.T = 0;
  u.fresh = false;
  const bool i64 = (p.flags & F_IDX64) != 0;
  if constexpr (IDX == IDX_SLOTS) {
    if (p.flags & F_VARLEN) {
      const int32_t* cu = reinterpret_cast<const int32_t*>(p.indptr);
      u.tok0 = cu[b];
      u.tok1 = cu[b + 1];
      if (u.tok0 < 0 || u.tok1 < u.tok0 || u.tok1 > p.total_tokens) {
        u.err |= E_SEQLENS;
        u.status = U_SKIP;
        return u;
      }
    } else {
      u.tok0 = b * p.T;
      u.tok1 = u.tok0 + p.T;
    }
    const int64_t s = ld_index(p.idx, b, i64);
    u.src = u.dst = s;
    if (s < 0) u.status = U_PAD;
    else if (s >= p.num_slots) { u.status = U_PAD; u.err |= E_SLOT_RANGE; }
  } else if (p.flags & F_VARLEN) {
    // prefill: a varlen run appended to the sequence (see resolve_suffix)
    const int32_t* cu = reinterpret_cast<const int32_t*>(p.cu);
    u.tok0 = cu[b];
    u.tok1 = cu[b + 1];
    if (u.tok0 < 0 || u.tok1 < u.tok0 || u.tok1 > p.total_tokens) {
      u.err |= E_SEQLENS;
      u.status = U_SKIP;
      return u;
    }
    if (u.tok1 == u.tok0) return u;
    resolve_suffix(p, b, u.tok1 - u.tok0, true, u);
    if (u.err) u.status = U_PAD;
  } else if (p.T > 1) {
    // suffix of T tokens (see resolve_suffix)
    u.tok0 = b * p.T;
    u.tok1 = u.tok0 + p.T;
    resolve_suffix(p, b, p.T, false, u);
    if (u.err) u.status = U_PAD;
  } else {
    u.tok0 = b;
    u.tok1 = b + 1;
    if (p.rows != nullptr) {
      u.src = p.rows[2 * b];
      u.dst = p.rows[2 * b + 1];
      if (u.src < 0 || u.dst < 0) u.status = U_PAD;
      else if (u.src >= p.num_slots || u.dst >= p.num_slots) { u.status = U_PAD; u.err |= E_PAGE_RANGE; }
    } else {
      resolve_page_rows(p.idx, p.indptr, p.lastlen, i64, p.nnz, p.num_slots, p.page_size, b,
                        u.src, u.dst, u.err);
      if (u.err) u.status = U_PAD;
    }
  }
  return u;
}

__device__ __forceinline__ void raise_err(int32_t* err, int bits) {
  if (err != nullptr && bits != 0) atomicOr(err, bits);
}

}  // namespace gdn
