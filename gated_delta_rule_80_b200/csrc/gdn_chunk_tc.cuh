// Paged prefill of fp32 states on the tensor cores: the chunked form of the
// gated delta rule, 64 tokens per chunk, one CTA per (sequence, value head).
//
// Within a chunk (tokens t = 0..63 of the page-aligned chunk, g_t the
// inclusive prefix sum of log alpha, S0 the state before the chunk):
//     A_ts = beta_t (k^_t . k^_s) e^{g_t - g_s}      (s < t)
//     P_ts = (q^_t . k^_s) e^{g_t - g_s}             (s <= t)
//     R_t  = beta_t (v_t - e^{g_t} k^_t S0)
//     (I + A) U = R                                  (forward substitution)
//     o_t  = e^{g_t} q^_t S0 + sum_{s<=t} P_ts U_s
//     S_C  = e^{g_C} S0 + sum_t e^{g_C - g_t} k^_t U_t^T
// which is the scan of single steps (u_t = U_t) written for a block of
// tokens (Circuit.LLM.Mixer "Gated memory": a prefill is the steps in order).
//
// The state is kept transposed (rows = value index, the V_FIRST page row) in
// tensor memory as an fp32 accumulator. Three products run on tcgen05:
//     G1   = S0^T [K ; Q]^T     (128 x 128 x 128: k S0 and q S0 of all tokens)
//     Gram = [K ; Q] K^T        (128 x 64 x 128)
//     S_C^T += (diag(w) U)^T K  (128 x 128 x 64, w_t = |k_t|^-1 e^{g_C - g_t})
// with raw bf16 k and q rows as operands (their norms are applied to the
// results), the fp32 operands (diag(w) U)^T, U^T and P split into three bf16
// terms each (hi + mid + lo carries 24 bits) and S0^T into two (hi + lo, 16
// bits: S0 only enters k S0 and q S0, where that keeps outputs within about
// 2e-6 of the scan), so every product is exact and the accumulation is fp32.
// The splits use the paired hardware conversion (round to nearest even); the
// Gram, which needs only the chunk's rows, is issued as soon as they have
// landed. The small triangular work (A, P, the forward substitution, the
// outputs) runs on the CUDA cores: each of the two warpgroups has one thread
// per value column v and takes half of the columns, tokens or rows of every
// phase.
//
// Chunks are aligned to absolute token positions (multiples of 64), so with
// page_size a multiple of 64 every page end is a chunk end; slots of a chunk
// outside the run are padding (k = q = v = 0, alpha = 1, beta = 0), which
// leaves the state and the other tokens unchanged.
#pragma once

#include "gdn_device.cuh"
#include "gdn_umma.cuh"

namespace gdn {

struct ChunkTC {
  static constexpr int C = 64;    // tokens per chunk
  static constexpr int D = 128;   // K = V
  static constexpr int NT = 256;  // two warpgroups; thread v of each owns value column v / tensor-memory lane v
  // dynamic shared memory (bytes)
  static constexpr uint32_t KQ = 0;               // 2 x [128 rows (k then q tokens) x 128] bf16, K-major
  static constexpr uint32_t KQ_BYTES = 2 * C * D * 2;
  static constexpr uint32_t VB = 2 * KQ_BYTES;    // 2 x [64 tokens x 128] bf16 row-major
  static constexpr uint32_t V_BYTES = C * D * 2;
  static constexpr uint32_t S3 = VB + 2 * V_BYTES;  // 2 x [128 x 128] bf16, K-major: S0^T split (region of 3)
  static constexpr uint32_t S3_BYTES = D * D * 2;
  // after G1 the S3 region holds A (fp32, for the solve), then in its place
  // U^T and later (diag(w) U)^T (three bf16 terms each), K^T, and P (three
  // bf16 terms)
  static constexpr uint32_t UT3 = S3;                 // 3 x [128 x 64] bf16, K-major
  static constexpr uint32_t UT_BYTES = D * C * 2;
  static constexpr int AS = C + 4;                    // row stride of A (floats), staggers banks
  static constexpr uint32_t AM = S3;                  // [64 x AS] fp32, inside the UT3 area
  static constexpr uint32_t KT = UT3 + 3 * UT_BYTES;  // [128 x 64] bf16, K-major: K^T
  static constexpr uint32_t P3 = KT + UT_BYTES;       // 3 x [64 x 64] bf16, K-major: P split
  static constexpr uint32_t P_BYTES = C * C * 2;
  // the update operand (diag(w) U)^T in two bf16 terms (16 bits: the state
  // moves by about 5e-6), written beside U^T so that the output product and
  // the update are issued together
  // (starting in the S3 region's unused tail, after P)
  static constexpr uint32_t WU2 = P3 + 3 * P_BYTES;  // 2 x [128 x 64] bf16, K-major
  static constexpr uint32_t SMEM = WU2 + 2 * UT_BYTES;
  static_assert(AM + C * AS * 4 <= KT && SMEM >= S3 + 3 * S3_BYTES, "chunk operands fit in the S3 region");
  static_assert(SMEM + 4096 <= 227 * 1024, "dynamic plus static shared memory within one CTA's 227 KiB");
  // tensor memory columns
  // tensor memory columns: state, G1, Gram / outputs, and the page snapshot
  // of the chunk's initial state, stored to the pool a quarter at a time
  // over the chunk instead of in one burst (every CTA writing 64 KiB at the
  // same point stalled its warps on the stores)
  static constexpr uint32_t T_ST = 0, T_G1 = 128, T_GR = 256, T_SN = 320, T_COLS = 512;
};

// Splits of fp32 pairs into bf16 terms with the paired hardware conversion
// (round to nearest, ties to even), packed as the MMA operands want them
// (the first value in the low half). Each residual is exact in binary32, so
// x = hi + lo to 16 bits, and x = hi + mid + lo to 24.
__device__ __forceinline__ uint32_t bf16x2_rn(float x0, float x1) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float2 bf16x2_residual(float2 x, uint32_t h) {
  return __fadd2_rn(x, make_float2(-bf16_lo(h), -bf16_hi(h)));
}
__device__ __forceinline__ void split2_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = bf16x2_rn(x0, x1);
  const float2 r = bf16x2_residual(make_float2(x0, x1), hi);
  lo = bf16x2_rn(r.x, r.y);
}
__device__ __forceinline__ void split3_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& mid, uint32_t& lo) {
  hi = bf16x2_rn(x0, x1);
  const float2 r = bf16x2_residual(make_float2(x0, x1), hi);
  mid = bf16x2_rn(r.x, r.y);
  const float2 r2 = bf16x2_residual(r, mid);
  lo = bf16x2_rn(r2.x, r2.y);
}
// 8 values -> three 16-byte rows of bf16 terms
__device__ __forceinline__ void split3_bf16x8(const float* x, uint4& h, uint4& m, uint4& l) {
  uint32_t hw[4], mw[4], lw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) split3_bf16x2(x[2 * i], x[2 * i + 1], hw[i], mw[i], lw[i]);
  h = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  m = make_uint4(mw[0], mw[1], mw[2], mw[3]);
  l = make_uint4(lw[0], lw[1], lw[2], lw[3]);
}

// The token inputs of the chunk starting at absolute position `base` into
// input buffer `buf`: k rows and q rows into the [K ; Q] operand tile, v rows
// row-major; slots outside [pos_lo, pos_hi) are zero filled. Part `part` of
// kLoadParts (one cp.async group each): the next chunk's copies are issued
// in parts over the current chunk, because every CTA issuing its 48 KiB at
// the same point stalled on the memory system.
constexpr int kLoadParts = 4;
__device__ __forceinline__ void chunk_issue_loads(const StepParams& p, unsigned char* sm, int buf, int64_t base,
                                                  int64_t pos_lo, int64_t pos_hi, int64_t tok_lo, int h, int hv,
                                                  int part) {
  using CT = ChunkTC;
  unsigned char* kq = sm + CT::KQ + buf * CT::KQ_BYTES;
  unsigned char* vv = sm + CT::VB + buf * CT::V_BYTES;
  constexpr int PER = 3 * CT::C * 16 / kLoadParts;
  static_assert(PER % CT::NT == 0, "whole copies per thread and part");
  for (int id = part * PER + threadIdx.x; id < (part + 1) * PER; id += CT::NT) {
    const int which = id / (CT::C * 16), rem = id % (CT::C * 16), j = rem / 16, piece = rem % 16;
    const int64_t pos = base + j;
    const bool valid = pos >= pos_lo && pos < pos_hi;
    const int64_t tok = tok_lo + (pos - pos_lo);
    const char* src = reinterpret_cast<const char*>(p.q);  // any valid address; no bytes are read when zero filling
    unsigned char* dst;
    if (which < 2) {
      dst = kq + kmajor_offset(which * CT::C + j, 8 * piece, CT::D);
      if (valid) src = reinterpret_cast<const char*>(which == 0 ? p.k : p.q) + ((tok * p.H + h) * CT::D) * 2 + piece * 16;
    } else {
      dst = vv + j * (CT::D * 2) + piece * 16;
      if (valid) src = reinterpret_cast<const char*>(p.v) + ((tok * p.HV + hv) * CT::D) * 2 + piece * 16;
    }
    cp_async16(dst, src, valid);
  }
  cp_async_commit();
}

__global__ void __launch_bounds__(ChunkTC::NT, 1) prefill_chunk_tc(const StepParams p) {
  using CT = ChunkTC;
  constexpr int C = CT::C, D = CT::D;
  extern __shared__ __align__(1024) unsigned char sm[];
  // MMA completion: one barrier for the Gram, one for G1 and the update, so
  // that neither ever has more than one phase outstanding
  __shared__ __align__(8) uint64_t bar, bar_gr;
  __shared__ uint32_t s_tmem;
  __shared__ double s_g[C];
  __shared__ double s_wsum;
  __shared__ float s_beta[C], s_ik[C], s_iq[C];
  __shared__ float s_egk[C], s_egq[C], s_wc[C];  // e^{g_t} |k_t|^-1, e^{g_t} scale |q_t|^-1, |k_t|^-1 e^{g_C - g_t}
  __shared__ float s_eg[C], s_kinv[C];           // e^{g_t}; |k_t|^-1 e^{-g_t} (chunks with g_C > -80)
  __shared__ float s_nrm[D];                     // the second warpgroup's half of each row's sum of squares

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wg = tid >> 7;      // warpgroup: splits the columns, tokens or rows of each phase
  const int v = tid & (D - 1);  // value column, tensor-memory lane and tile row of this thread
  const int hv = blockIdx.x, b = blockIdx.y;
  const int h = hv / p.G;
  const bool in_bf16 = (p.flags & F_IN_BF16) != 0;
  const bool out_bf16 = (p.flags & F_OUT_BF16) != 0;

  const Unit u = resolve_unit<IDX_PAGED>(p, b);
  if (tid == 0) raise_err(p.err, u.err);
  if (u.status == U_SKIP || u.tok1 <= u.tok0) return;
  if (u.status == U_PAD) {
    if (wg == 0)
      for (int tok = u.tok0; tok < u.tok1; ++tok) st_out1(p.out, ((int64_t)tok * p.HV + hv) * D + v, 0.0f, out_bf16);
    return;
  }
  const int64_t n = u.tok1 - u.tok0;
  const int64_t pos_lo = u.L - n, pos_hi = u.L;
  const int64_t base0 = (pos_lo / C) * C;
  const int nchunks = static_cast<int>((pos_hi - base0 + C - 1) / C);
  const int64_t head = (int64_t)D * D;  // floats of one (page, head) state
  float* pool = reinterpret_cast<float*>(p.pool);

  if (tid == 0) {
    mbar_init(&bar, 1);
    mbar_init(&bar_gr, 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&s_tmem, CT::T_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = s_tmem;
  const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
  const uint32_t t_st = tmem + CT::T_ST + lane_base;
  const uint32_t t_g1 = tmem + CT::T_G1 + lane_base;
  const uint32_t t_gr = tmem + CT::T_GR + lane_base;
  const uint32_t t_sn = tmem + CT::T_SN + lane_base;
  uint32_t phase = 0, phase_gr = 0;
  bool aborted = false;
  // bounded wait for the oldest commit on `bar` (or on `bar_gr`), decided by the whole CTA
  auto wait_on = [&](uint64_t* br, uint32_t& ph) -> bool {
    const bool late = !mbar_wait(br, ph);
    ph ^= 1u;
    const bool any = __syncthreads_or(late) != 0;
    tc_fence_after_sync();
    return any;
  };
  auto wait_mma = [&]() -> bool { return wait_on(&bar, phase); };
  // a quarter (16 columns) of this warpgroup's half of the staged snapshot to
  // the pool; the snapshot page is the same for the whole CTA
  auto snap_piece = [&](int64_t page, int piece) {
    if (page < 0) return;
    // 16x256b loads: in each 16-lane half of the warp's 32 lanes, four
    // consecutive threads hold 8 consecutive columns of one lane (row), so
    // each 8-byte store fills whole 32-byte sectors of the page row (the
    // 32x32b shape gives each thread its own row: 16-byte pieces of 32
    // rows per store instruction)
    const int lane = tid & 31;
    const uint32_t sp = static_cast<uint32_t>(32 * ((tid >> 5) & 3));
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t r[8];
      tmem_ld16x256b_x2(tmem + CT::T_SN + ((sp + 16 * half) << 16) + 64 * wg + 16 * piece, r);
#pragma unroll
      for (int g = 0; g < 2; ++g)
#pragma unroll
        for (int hl = 0; hl < 2; ++hl) {
          const int row = sp + 16 * half + 8 * hl + (lane >> 2);
          const int col = 64 * wg + 16 * piece + 8 * g + 2 * (lane & 3);
          __stcs(reinterpret_cast<float2*>(pool + (page * p.HV + hv) * head + (int64_t)row * D + col),
                 make_float2(__uint_as_float(r[4 * g + 2 * hl]), __uint_as_float(r[4 * g + 2 * hl + 1])));
        }
    }
  };

  const float expA = expf(p.A_log[hv]);
  const float dtb = p.dt_bias[hv];
  float na = 0.f, nb = 0.f;  // raw gate and beta of the next chunk (threads < C)
  auto load_ab = [&](int64_t base) {
    if (tid < C) {
      const int64_t pos = base + tid;
      if (pos >= pos_lo && pos < pos_hi) {
        const int64_t tok = u.tok0 + (pos - pos_lo);
        na = ld_in1(p.gate, tok * p.HV + hv, in_bf16);
        nb = ld_in1(p.beta, tok * p.HV + hv, in_bf16);
      }
    }
  };
#pragma unroll 1
  for (int part = 0; part < kLoadParts; ++part) chunk_issue_loads(p, sm, 0, base0, pos_lo, pos_hi, u.tok0, h, hv, part);
  load_ab(base0);
  // part `part` of the next chunk's copies (they go to the other buffer,
  // free since the previous chunk ended)
  auto next_loads = [&](int c, int64_t base, int part) {
    if (c + 1 < nchunks) chunk_issue_loads(p, sm, (c & 1) ^ 1, base + C, pos_lo, pos_hi, u.tok0, h, hv, part);
  };

  for (int c = 0; c < nchunks && !aborted; ++c) {
    const int buf = c & 1;
    const int64_t base = base0 + (int64_t)c * C;
    const float ca = na, cb = nb;
    cp_async_wait<0>();
    fence_async_smem();  // this thread's copies, to the tensor core's proxy
    tc_fence_before_sync();
    __syncthreads();
    // Gram = [K ; Q] K^T on the tensor cores at once: it needs only this
    // chunk's rows, so it runs under the prologue and the state split
    if (tid == 0) {
      tc_fence_after_sync();
      const uint64_t dk = umma_desc_kmajor(sm + CT::KQ + buf * CT::KQ_BYTES, D);
      const uint32_t id_gr = umma_idesc_bf16(128, 64);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        umma_bf16(tmem + CT::T_GR, umma_desc_add(dk, ks * 256), umma_desc_add(dk, ks * 256), id_gr, ks > 0);
      umma_commit(&bar_gr);
    }
    next_loads(c, base, 0);
    if (c + 1 < nchunks) load_ab(base + C);
    const unsigned char* kq = sm + CT::KQ + buf * CT::KQ_BYTES;

    // ---- per-token scalars: log alpha prefix (double), beta, norms
    if (tid < C) {
      const int64_t pos = base + tid;
      const bool valid = pos >= pos_lo && pos < pos_hi;
      const float la = valid ? -expA * softplus_f(ca + dtb) : 0.0f;
      s_beta[tid] = valid ? ((p.flags & F_BETA_PROB) ? cb : sigmoid_f(cb)) : 0.0f;
      double x = static_cast<double>(la);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
      }
      s_g[tid] = x;
      if (tid == 31) s_wsum = x;
    }
    float ss = 0.f;  // row v of [K ; Q], this warpgroup's 64 columns
#pragma unroll
    for (int c8 = 0; c8 < D / 16; ++c8) {
      const uint4 w = *reinterpret_cast<const uint4*>(kq + kmajor_offset(v, 64 * wg + 8 * c8, D));
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = bf16_lo(ww[e]), hi = bf16_hi(ww[e]);
        ss = fmaf(lo, lo, ss);
        ss = fmaf(hi, hi, ss);
      }
    }
    if (wg == 1) s_nrm[v] = ss;
    __syncthreads();
    if (tid >= 32 && tid < C) s_g[tid] += s_wsum;
    if (wg == 0) {
      const float inv = (p.flags & F_L2NORM) ? rsqrtf(ss + s_nrm[v] + kL2Eps) : 1.0f;
      if (v < C) s_ik[v] = inv;
      else s_iq[v - C] = inv * p.scale;
    }
    __syncthreads();
    const double gC = s_g[C - 1];
    const float eC = expf(static_cast<float>(gC));
    if (tid < C) {
      const float eg = static_cast<float>(exp(s_g[tid]));  // double: the exponent is not rounded to fp32 first
      s_eg[tid] = eg;
      s_kinv[tid] = gC > -80.0 ? s_ik[tid] * static_cast<float>(exp(-s_g[tid])) : 0.0f;
      s_egk[tid] = eg * s_ik[tid];
      s_egq[tid] = eg * s_iq[tid];
      s_wc[tid] = s_ik[tid] * expf(static_cast<float>(gC - s_g[tid]));
    }

    // ---- the state: previous chunk's update done; snapshot, split, decay
    // (this warpgroup's 64 columns of row v)
    if (c > 0 && wait_mma()) {
      aborted = true;
      break;
    }
    int64_t snap = -1;  // page receiving the chunk's initial state, staged in tensor memory
    {
      if (c > 0) {
        const int64_t last = base - 1;  // last position of the previous chunk
        if (last >= pos_lo) snap = suffix_snapshot_page(p, u, static_cast<int>(last - pos_lo));
      }
      if (snap >= p.num_slots) {
        if (tid == 0) raise_err(p.err, E_PAGE_RANGE);
        snap = -1;
      }
      // both 32-column blocks of this warpgroup's half of row v are loaded
      // (and stored back) with one wait for the pair
      float x[2][32];
      if (c == 0) {
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const int kc = 2 * wg + kk;
          if (u.fresh) {
#pragma unroll
            for (int i = 0; i < 32; ++i) x[kk][i] = 0.0f;
          } else {
            const float4* src = reinterpret_cast<const float4*>(pool + (u.src * p.HV + hv) * head + (int64_t)v * D + 32 * kc);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 f = __ldcs(src + q);
              x[kk][4 * q] = f.x; x[kk][4 * q + 1] = f.y; x[kk][4 * q + 2] = f.z; x[kk][4 * q + 3] = f.w;
            }
          }
        }
      } else {
        uint32_t r0[32], r1[32];
        tmem_ld32_issue(t_st + 64 * wg, r0);
        tmem_ld32_issue(t_st + 64 * wg + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          x[0][i] = __uint_as_float(r0[i]);
          x[1][i] = __uint_as_float(r1[i]);
        }
      }
      if (snap >= 0) {
        tmem_st32_issue(t_sn + 64 * wg, x[0]);
        tmem_st32_issue(t_sn + 64 * wg + 32, x[1]);
      }
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int kc = 2 * wg + kk;
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) split2_bf16x2(x[kk][8 * q8 + 2 * i], x[kk][8 * q8 + 2 * i + 1], hw[i], lw[i]);
          const uint32_t off = kmajor_offset(v, 32 * kc + 8 * q8, D);
          *reinterpret_cast<uint4*>(sm + CT::S3 + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(sm + CT::S3 + CT::S3_BYTES + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) x[kk][i] *= eC;
      }
      tmem_st32_issue(t_st + 64 * wg, x[0]);
      tmem_st32_issue(t_st + 64 * wg + 32, x[1]);
      tmem_wait_st();
    }
    fence_async_smem();
    tc_fence_before_sync();
    __syncthreads();

    // ---- G1 = S0^T [K ; Q]^T on the tensor cores
    if (tid == 0) {
      tc_fence_after_sync();
      const uint32_t id_g1 = umma_idesc_bf16(128, 128);
      const uint64_t da = umma_desc_kmajor(sm + CT::S3, D), db = umma_desc_kmajor(kq, D);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          umma_bf16(tmem + CT::T_G1, umma_desc_add(da, i * CT::S3_BYTES + ks * 256), umma_desc_add(db, ks * 256), id_g1,
                    i > 0 || ks > 0);
      umma_commit(&bar);
    }
    // the Gram (issued first): A, P and K^T do not wait for G1
    if (wait_on(&bar_gr, phase_gr)) {
      aborted = true;
      break;
    }

    snap_piece(snap, 0);
    // ---- A and P rows from the Gram: thread (wg, r) takes columns 32 wg ..
    // 32 wg + 31 of row r (k row r < 64: A in fp32; q row r - 64: P as three
    // bf16 tiles, the B operand of the output product). A and K^T take space
    // of the S0 split that G1 is still reading, so they are held in
    // registers until G1 is done; P has a region of its own.
    const int t_row = v & (C - 1);
    const bool is_p = v >= C;
    float aw[32];
    {
      const int t = t_row;
      float gr[32];
      tmem_ld32(t_gr + 32 * wg, gr);
      const double gt = s_g[t];
      const float coef = is_p ? s_iq[t] : s_beta[t] * s_ik[t];
      const int lim = is_p ? t + 1 : t;  // columns s < lim are kept
      // e^{g_t - g_s} = e^{g_t} e^{-g_s} while e^{-g_C} stays finite; per pair otherwise
      const bool factored = gC > -80.0;
      const float ct = coef * (factored ? s_eg[t] : 1.0f);
#pragma unroll
      for (int s8 = 0; s8 < 32; s8 += 8) {
        float w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int sx = 32 * wg + s8 + e;
          const float d = factored ? s_kinv[sx] : s_ik[sx] * __expf(static_cast<float>(gt - s_g[sx]));
          w[e] = sx < lim ? ct * d * gr[s8 + e] : 0.0f;
        }
        if (is_p) {
          uint4 hh, mm, ll;
          split3_bf16x8(w, hh, mm, ll);
          const uint32_t off = kmajor_offset(t, 32 * wg + s8, C);
          *reinterpret_cast<uint4*>(sm + CT::P3 + off) = hh;
          *reinterpret_cast<uint4*>(sm + CT::P3 + CT::P_BYTES + off) = mm;
          *reinterpret_cast<uint4*>(sm + CT::P3 + 2 * CT::P_BYTES + off) = ll;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) aw[s8 + e] = w[e];
        }
      }
    }
    // ---- K^T for the update: thread (wg, k) gathers 32 tokens of column k
    uint4 ktw[4];
#pragma unroll
    for (int tt = 0; tt < 4; ++tt) {
      const int t8 = 4 * wg + tt;
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t lo = *reinterpret_cast<const uint16_t*>(kq + kmajor_offset(8 * t8 + 2 * i, v, D));
        const uint32_t hi = *reinterpret_cast<const uint16_t*>(kq + kmajor_offset(8 * t8 + 2 * i + 1, v, D));
        w[i] = lo | (hi << 16);
      }
      ktw[tt] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    snap_piece(snap, 1);
    next_loads(c, base, 1);
    if (wait_mma()) {  // G1; also orders P before the reads below
      aborted = true;
      break;
    }
    // A and K^T into the space of the S0 split (read by the solve after the
    // barrier that follows the residuals, and by the update product)
    if (!is_p) {
      float* arow = reinterpret_cast<float*>(sm + CT::AM) + t_row * CT::AS + 32 * wg;
#pragma unroll
      for (int s8 = 0; s8 < 32; s8 += 4)
        *reinterpret_cast<float4*>(arow + s8) = make_float4(aw[s8], aw[s8 + 1], aw[s8 + 2], aw[s8 + 3]);
    }
#pragma unroll
    for (int tt = 0; tt < 4; ++tt)
      *reinterpret_cast<uint4*>(sm + CT::KT + kmajor_offset(v, 8 * (4 * wg + tt), C)) = ktw[tt];
    // U lives in the chunk's [K ; Q] buffer from here on: Us[t][v]
    float* Us = reinterpret_cast<float*>(sm + CT::KQ + buf * CT::KQ_BYTES);
    // ---- residuals R_t = beta_t (v_t - e^{g_t} k^_t S0), tokens 32 wg .. 32 wg + 31
    {
      const __nv_bfloat16* vcol = reinterpret_cast<const __nv_bfloat16*>(sm + CT::VB + buf * CT::V_BYTES) + v;
      float x[32];
      tmem_ld32(t_g1 + 32 * wg, x);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int t = 32 * wg + i;
        Us[t * D + v] = s_beta[t] * (__bfloat162float(vcol[t * D]) - s_egk[t] * x[i]);
      }
    }
    __syncthreads();
    snap_piece(snap, 2);
    next_loads(c, base, 2);
    // ---- (I + A) U = R in two blocks of 32 tokens: each warpgroup takes 16
    // rows of the block for the part from the earlier block; the triangle
    // inside the block is finished by the first warpgroup, then by the second
    {
      constexpr int BS = 32, HB = BS / 2;
      const float* Am = reinterpret_cast<const float*>(sm + CT::AM);
#pragma unroll 1
      for (int bb = 0; bb < C / BS; ++bb) {
        const int t0 = BS * bb, r0 = t0 + HB * wg;
        float uu[HB];
#pragma unroll
        for (int i = 0; i < HB; ++i) uu[i] = Us[(r0 + i) * D + v];
#pragma unroll 1
        for (int s4 = 0; s4 < t0; s4 += 4) {
          float us[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) us[e] = Us[(s4 + e) * D + v];
#pragma unroll
          for (int i = 0; i < HB; ++i) {
            const float4 a = *reinterpret_cast<const float4*>(Am + (r0 + i) * CT::AS + s4);
            uu[i] = fmaf(-a.x, us[0], uu[i]);
            uu[i] = fmaf(-a.y, us[1], uu[i]);
            uu[i] = fmaf(-a.z, us[2], uu[i]);
            uu[i] = fmaf(-a.w, us[3], uu[i]);
          }
        }
        if (wg == 0) {
#pragma unroll
          for (int i = 1; i < HB; ++i)
#pragma unroll
            for (int j = 0; j < i; ++j) uu[i] = fmaf(-Am[(t0 + i) * CT::AS + t0 + j], uu[j], uu[i]);
#pragma unroll
          for (int i = 0; i < HB; ++i) Us[(t0 + i) * D + v] = uu[i];
        }
        __syncthreads();
        if (wg == 1) {
#pragma unroll
          for (int j4 = 0; j4 < HB; j4 += 4) {
            float lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) lo[e] = Us[(t0 + j4 + e) * D + v];
#pragma unroll
            for (int i = 0; i < HB; ++i) {
              const float4 a = *reinterpret_cast<const float4*>(Am + (r0 + i) * CT::AS + t0 + j4);
              uu[i] = fmaf(-a.x, lo[0], uu[i]);
              uu[i] = fmaf(-a.y, lo[1], uu[i]);
              uu[i] = fmaf(-a.z, lo[2], uu[i]);
              uu[i] = fmaf(-a.w, lo[3], uu[i]);
            }
          }
#pragma unroll
          for (int i = 1; i < HB; ++i)
#pragma unroll
            for (int j = 0; j < i; ++j) uu[i] = fmaf(-Am[(r0 + i) * CT::AS + r0 + j], uu[j], uu[i]);
#pragma unroll
          for (int i = 0; i < HB; ++i) Us[(r0 + i) * D + v] = uu[i];
        }
        __syncthreads();
      }
    }
    snap_piece(snap, 3);
    next_loads(c, base, 3);
    // ---- outputs o_t = e^{g_t} q^_t S0 + sum_{s<=t} P_ts U_s: U^T (three bf16
    // terms, replacing A) times P^T on the tensor cores (the six products of
    // the splits above the lowest order), then the state part added
#pragma unroll 1
    for (int tt = 0; tt < 4; ++tt) {
      const int t8 = 4 * wg + tt;
      float x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = Us[(8 * t8 + i) * D + v];
      uint4 hh, mm, ll;
      split3_bf16x8(x, hh, mm, ll);
      const uint32_t off = kmajor_offset(v, 8 * t8, C);
      *reinterpret_cast<uint4*>(sm + CT::UT3 + off) = hh;
      *reinterpret_cast<uint4*>(sm + CT::UT3 + CT::UT_BYTES + off) = mm;
      *reinterpret_cast<uint4*>(sm + CT::UT3 + 2 * CT::UT_BYTES + off) = ll;
      // the update operand (diag(w) U)^T, two terms
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        split2_bf16x2(s_wc[8 * t8 + 2 * i] * x[2 * i], s_wc[8 * t8 + 2 * i + 1] * x[2 * i + 1], hw[i], lw[i]);
      *reinterpret_cast<uint4*>(sm + CT::WU2 + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(sm + CT::WU2 + CT::UT_BYTES + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    fence_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after_sync();
      const uint32_t id_o = umma_idesc_bf16(128, 64);
      const uint64_t da = umma_desc_kmajor(sm + CT::UT3, C), db = umma_desc_kmajor(sm + CT::P3, C);
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int j = 0; i + j < 3; ++j)
#pragma unroll
          for (int ks = 0; ks < C / 16; ++ks)
            umma_bf16(tmem + CT::T_GR, umma_desc_add(da, i * CT::UT_BYTES + ks * 256),
                      umma_desc_add(db, j * CT::P_BYTES + ks * 256), id_o, i + j + ks > 0);
      umma_commit(&bar_gr);
      // ---- S^T += (diag(w) U)^T K on the tensor cores (the state was decayed
      // above); it completes while the outputs are stored
      const uint32_t id_up = umma_idesc_bf16(128, 128);
      const uint64_t dw = umma_desc_kmajor(sm + CT::WU2, C), dkt = umma_desc_kmajor(sm + CT::KT, C);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          umma_bf16(tmem + CT::T_ST, umma_desc_add(dw, i * CT::UT_BYTES + ks * 256), umma_desc_add(dkt, ks * 256), id_up,
                    true);
      umma_commit(&bar);
    }
    if (wait_on(&bar_gr, phase_gr)) {
      aborted = true;
      break;
    }
    {
      float pu[32], ob[32];
      tmem_ld32(t_gr + 32 * wg, pu);
      tmem_ld32(t_g1 + C + 32 * wg, ob);
      if (out_bf16) {
        // bf16 outputs go through the chunk's v buffer (consumed by now) and
        // leave as 16-byte rows after the next barrier
        __nv_bfloat16* ost = reinterpret_cast<__nv_bfloat16*>(sm + CT::VB + buf * CT::V_BYTES);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int t = 32 * wg + i;
          ost[t * D + v] = __float2bfloat16_rn(fmaf(s_egq[t], ob[i], pu[i]));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int t = 32 * wg + i;
          const int64_t pos = base + t;
          if (pos >= pos_lo && pos < pos_hi)
            st_out1(p.out, ((u.tok0 + (pos - pos_lo)) * p.HV + hv) * D + v, fmaf(s_egq[t], ob[i], pu[i]), false);
        }
      }
    }
    if (out_bf16) {
      // the staged bf16 outputs: 16 bytes (8 values of one token) per copy
      __syncthreads();
      const uint4* ost = reinterpret_cast<const uint4*>(sm + CT::VB + buf * CT::V_BYTES);
#pragma unroll
      for (int k = 0; k < C * D / 8 / CT::NT; ++k) {
        const int id = tid + CT::NT * k, t = id / (D / 8), piece = id % (D / 8);
        const int64_t pos = base + t;
        if (pos >= pos_lo && pos < pos_hi)
          __stcs(reinterpret_cast<uint4*>(p.out) + ((u.tok0 + (pos - pos_lo)) * p.HV + hv) * (D / 8) + piece, ost[id]);
      }
    }
  }

  // ---- the final state to the last page (this warpgroup's 64 columns of row v)
  if (!aborted) {
    if (wait_mma()) {
      aborted = true;
    } else {
      float4* dst = reinterpret_cast<float4*>(pool + (u.dst * p.HV + hv) * head + (int64_t)v * D);
#pragma unroll 1
      for (int kk = 0; kk < 2; ++kk) {
        const int kc = 2 * wg + kk;
        float x[32];
        tmem_ld32(t_st + 32 * kc, x);
#pragma unroll
        for (int q = 0; q < 8; ++q) __stcs(dst + 8 * kc + q, make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]));
      }
    }
  }
  if (aborted) {
    if (tid == 0) raise_err(p.err, E_TIMEOUT);
    // a bounded chance for the MMAs in flight to finish (the last commit on
    // each barrier; an already completed phase returns at once)
    (void)mbar_wait(&bar, phase ^ 1u);
    (void)mbar_wait(&bar_gr, phase_gr ^ 1u);
  }
  cp_async_wait<0>();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, CT::T_COLS);
  }
}

}  // namespace gdn
