// KDA over varlen runs on a slot pool, on the tensor cores: the chunked form
// of the gated delta rule with a decay per key channel, 32 tokens per chunk,
// one CTA per (sequence, value head).
//
// Within a chunk (tokens t = 0..31, G_t[i] the inclusive prefix sum of
// log alpha_t[i] over the chunk, S0 the state before it, k^ and q^ the
// normalised rows, q^ scaled by 1/sqrt(K)):
//     A_ts = beta_t sum_i k^_t[i] k^_s[i] e^{G_t[i] - G_s[i]}      (s < t)
//     P_ts = sum_i q^_t[i] k^_s[i] e^{G_t[i] - G_s[i]}             (s <= t)
//     R_t  = beta_t (v_t - K~_t S0),  K~_t = k^_t o e^{G_t}
//     (I + A) U = R                                               (forward substitution)
//     o_t  = Q~_t S0 + sum_{s<=t} P_ts U_s,  Q~_t = q^_t o e^{G_t}
//     S_C  = diag(e^{G_C}) S0 + sum_t K^_t^T U_t,  K^_t = k^_t o e^{G_C - G_t}
// which is the scan of single steps (u_t = U_t) of Circuit.LLM.Mixer,
// "Gated memory" (kdaLiteStep: each key row of S decays by its own alpha),
// written for a block of tokens. Every exponent above is <= 0, so no factor
// can overflow however strong the decay.
//
// The state is kept transposed (rows = value index) in tensor memory as an
// fp32 accumulator. Three products run on tcgen05 (bf16 x bf16 -> fp32):
//     G1  = S0^T [K~ ; Q~]^T   (128 x 64 x 128)
//     O^T = U^T P^T            (128 x 32 x 32)
//     S^T += U^T K^            (128 x 128 x 32)
// The operands are split into bf16 terms so that the products keep fp32
// accuracy: S0^T and the scaled rows K~, Q~, K^ in two terms (16 bits), U
// and P in three (24 bits); a numpy model of this kernel stays within 1e-5
// of the float64 scan over 200 tokens. A and P (exact per channel) and the
// solve run on the CUDA cores, A and P while G1 runs.
//
// Runs are cut into chunks from their first token; the slots of the last
// chunk past the run are padding (k = q = v = 0, alpha = 1, beta = 0),
// which leaves the state and the other tokens unchanged. A run of n tokens
// costs ceil(n / 32) chunks, so the caller sends only long runs here.
#pragma once

#include "gdn_chunk_tc.cuh"

namespace gdn {

struct KdaTC {
  static constexpr int C = 32;    // tokens per chunk
  static constexpr int D = 128;   // K = V
  static constexpr int NT = 256;  // two warpgroups; thread v of each owns value column v / tensor-memory lane v
  // dynamic shared memory (bytes)
  // two input buffers: k rows then q rows [64 x 128] (rows padded to RS
  // bytes, so that the pair loop's loads from eight rows hit distinct
  // banks), v rows [32 x 128] and raw gate rows [32 x 128], bf16 row-major
  static constexpr uint32_t RAW = 0;
  static constexpr int RS = D * 2 + 16;
  static constexpr uint32_t R_KQ = 0, R_V = 2 * C * RS, R_G = R_V + C * D * 2;
  static constexpr uint32_t RAW_BYTES = R_G + C * D * 2;
  static constexpr int GS = D + 4;                      // row stride (floats) of G, staggers banks
  static constexpr uint32_t GM = RAW + 2 * RAW_BYTES;   // [C x GS] fp32: G in log2 units
  static constexpr uint32_t KQT = GM + C * GS * 4;      // 2 terms x [64 x 128] bf16, K-major: [K~ ; Q~]
  static constexpr uint32_t KQT_BYTES = 2 * C * D * 2;
  static constexpr uint32_t KBT = KQT + 2 * KQT_BYTES;  // 2 terms x [128 x 32] bf16, K-major: K^ ^T
  static constexpr uint32_t KBT_BYTES = D * C * 2;
  static constexpr uint32_t AL = KBT + 2 * KBT_BYTES;   // [C x GS] fp32: alpha_t[i] = 2^(G_t - G_(t-1))
  static constexpr int AS = C + 4;                      // row stride (floats) of A
  static constexpr uint32_t AM = AL + C * GS * 4;       // [C x AS] fp32
  static constexpr uint32_t P3 = AM + C * AS * 4;       // 3 terms x [32 x 32] bf16, K-major: P
  static constexpr uint32_t P_BYTES = C * C * 2;
  // the S0^T split (2 terms x [128 x 128] bf16, K-major); once G1 is done
  // the same region holds U (fp32 [C x D], the solve) and the U^T split
  static constexpr uint32_t X = P3 + 3 * P_BYTES;
  static constexpr uint32_t S_BYTES = D * D * 2;
  static constexpr uint32_t US = X;
  static constexpr uint32_t UT3 = X + C * D * 4;        // 3 terms x [128 x 32] bf16, K-major
  static constexpr uint32_t UT_BYTES = D * C * 2;
  static constexpr uint32_t SMEM = X + 2 * S_BYTES;
  static_assert(UT3 + 3 * UT_BYTES <= SMEM, "U and its split fit where the S0 split was");
  static_assert(SMEM + 2048 <= 227 * 1024, "dynamic plus static shared memory within one CTA's 227 KiB");
  static_assert(KQT % 16 == 0 && KBT % 16 == 0 && AL % 16 == 0 && P3 % 16 == 0 && X % 16 == 0 && UT3 % 16 == 0,
                "16-byte tiles");
  // tensor memory columns: state, G1 (32 k columns then 32 q columns), O
  static constexpr uint32_t T_ST = 0, T_G1 = 128, T_O = 192, T_COLS = 256;
};

constexpr float kLog2e = 1.4426950408889634f;

// 2^x on the special-function unit (relative error about 2^-22; results
// below the smallest normal flush to zero).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// log2(x) on the special-function unit (relative error about 2^-22).
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// softplus(x) / ln 2 = max(x, 0) log2(e) + log2(1 + 2^(-|x| log2(e))): the
// decay exponent in log2 units. When 1 + 2^(...) rounds to 1 (x < -17) the
// term it drops is below 6e-8, which moves a decay factor by less than
// 1e-6 relative.
__device__ __forceinline__ float softplus_log2(float x) {
  return fmaxf(x, 0.0f) * kLog2e + lg2_approx(1.0f + ex2_approx(-fabsf(x) * kLog2e));
}

// one fp32 value into three bf16 terms (hi + mid + lo carries 24 bits)
__device__ __forceinline__ void split3_bf16(float x, uint16_t& h, uint16_t& m, uint16_t& l) {
  const __nv_bfloat16 bh = __float2bfloat16_rn(x);
  const float r = x - __bfloat162float(bh);
  const __nv_bfloat16 bm = __float2bfloat16_rn(r);
  const __nv_bfloat16 bl = __float2bfloat16_rn(r - __bfloat162float(bm));
  h = __bfloat16_as_ushort(bh);
  m = __bfloat16_as_ushort(bm);
  l = __bfloat16_as_ushort(bl);
}

template <int L>
__global__ void __launch_bounds__(KdaTC::NT, 1) kda_chunk_tc(const StepParams p) {
  using CT = KdaTC;
  constexpr int C = CT::C, D = CT::D;
  extern __shared__ __align__(1024) unsigned char sm[];
  __shared__ __align__(8) uint64_t bar, bar_o;  // G1 and the update; the output product
  __shared__ uint32_t s_tmem;
  __shared__ float s_beta[C], s_ik[C], s_iq[C];
  __shared__ float s_egc[D];  // e^{G_C[i]} per key channel
  __shared__ float s_tot[D];  // G of the chunk's first half, per key channel

  const int tid = threadIdx.x;
  const int wg = tid >> 7;      // warpgroup: takes half of the keys, tokens or rows of each phase
  const int v = tid & (D - 1);  // value column / tensor-memory lane; key channel in the prologue
  const int hv = blockIdx.x, b = blockIdx.y;
  const int h = hv / p.G;
  const bool out_bf16 = (p.flags & F_OUT_BF16) != 0;

  const Unit u = resolve_unit<IDX_SLOTS>(p, b);
  if (tid == 0) raise_err(p.err, u.err);
  if (u.status == U_SKIP || u.tok1 <= u.tok0) return;
  if (u.status == U_PAD) {
    for (int tok = u.tok0 + wg; tok < u.tok1; tok += 2) st_out1(p.out, ((int64_t)tok * p.HV + hv) * D + v, 0.0f, out_bf16);
    return;
  }
  const int n = u.tok1 - u.tok0;
  const int nchunks = (n + C - 1) / C;
  float* state = reinterpret_cast<float*>(p.pool) + (u.src * p.HV + hv) * (int64_t)(D * D);
  float* Gm = reinterpret_cast<float*>(sm + CT::GM);

  if (tid == 0) {
    mbar_init(&bar, 1);
    mbar_init(&bar_o, 1);
    mbar_fence_init();
  }
  if (tid < 32) {
    tmem_alloc(&s_tmem, CT::T_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = s_tmem;
  const uint32_t lane_base = static_cast<uint32_t>(32 * ((tid >> 5) & 3)) << 16;
  const uint32_t t_st = tmem + CT::T_ST + lane_base;
  const uint32_t t_g1 = tmem + CT::T_G1 + lane_base;
  const uint32_t t_o = tmem + CT::T_O + lane_base;
  uint32_t phase = 0, phase_o = 0;
  bool aborted = false;
  auto wait_on = [&](uint64_t* br, uint32_t& ph) -> bool {
    const bool late = !mbar_wait(br, ph);
    ph ^= 1u;
    const bool any = __syncthreads_or(late) != 0;
    tc_fence_after_sync();
    return any;
  };
  auto wait_mma = [&]() -> bool { return wait_on(&bar, phase); };

  const float expA = expf(p.A_log[hv]);
  const float dtb = p.dt_bias[(int64_t)hv * D + v];
  // the token inputs of chunk c into input buffer `buf` (zero past the run),
  // part `part` of four (one cp.async group each): the next chunk's copies
  // are spread over the current chunk rather than issued by every CTA at once
  constexpr int kParts = 4, PER = 4 * C * 16 / kParts;
  static_assert(PER % CT::NT == 0, "whole copies per thread and part");
  auto issue_loads = [&](int c, int buf, int part) {
    unsigned char* raw = sm + CT::RAW + buf * CT::RAW_BYTES;
    const int nv = min(C, n - c * C);
    const int64_t t0 = u.tok0 + (int64_t)c * C;
    for (int id = part * PER + tid; id < (part + 1) * PER; id += CT::NT) {
      const int which = id / (C * 16), rem = id % (C * 16), j = rem / 16, piece = rem % 16;
      const bool valid = j < nv;
      const int64_t tok = t0 + j;
      const char* src = reinterpret_cast<const char*>(p.q);  // any valid address; no bytes are read when zero filling
      unsigned char* dst;
      if (which < 2) {
        dst = raw + CT::R_KQ + (which * C + j) * CT::RS + piece * 16;
        if (valid) src = reinterpret_cast<const char*>(which == 0 ? p.k : p.q) + ((tok * p.H + h) * D) * 2 + piece * 16;
      } else {
        dst = raw + (which == 2 ? CT::R_V : CT::R_G) + j * (D * 2) + piece * 16;
        if (valid)
          src = reinterpret_cast<const char*>(which == 2 ? p.v : p.gate) + ((tok * p.HV + hv) * D) * 2 + piece * 16;
      }
      cp_async16(dst, src, valid);
    }
    cp_async_commit();
  };
  float nb = 0.f;  // beta input of the next chunk (threads < C)
  auto load_beta = [&](int c) {
    if (tid < C && c * C + tid < n) nb = ld_in1(p.beta, (u.tok0 + (int64_t)c * C + tid) * p.HV + hv, true);
  };
  // P past the diagonal (s > t) is never written by the pair loop: zero once
  for (int i = tid; i < 3 * CT::P_BYTES / 16; i += CT::NT)
    reinterpret_cast<uint4*>(sm + CT::P3)[i] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
  for (int part = 0; part < kParts; ++part) issue_loads(0, 0, part);
  load_beta(0);
  auto next_loads = [&](int c, int part) {
    if (c + 1 < nchunks) issue_loads(c + 1, (c & 1) ^ 1, part);
  };

  for (int c = 0; c < nchunks && !aborted; ++c) {
    const int buf = c & 1;
    const int nv = min(C, n - c * C);
    const float cb = nb;
    cp_async_wait<0>();
    __syncthreads();
    next_loads(c, 0);
    if (c + 1 < nchunks) load_beta(c + 1);
    const unsigned char* raw = sm + CT::RAW + buf * CT::RAW_BYTES;

    // ---- prologue: norms (4 threads per k or q row), beta, the decay prefix
    {
      const int row = tid >> 2, part = tid & 3;
      const uint4* rp = reinterpret_cast<const uint4*>(raw + CT::R_KQ + row * CT::RS + part * 64);
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 w = rp[i];
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float lo = bf16_lo(ww[e]), hi = bf16_hi(ww[e]);
          ss = fmaf(lo, lo, ss);
          ss = fmaf(hi, hi, ss);
        }
      }
      ss += __shfl_xor_sync(kFull, ss, 1);
      ss += __shfl_xor_sync(kFull, ss, 2);
      if (part == 0) {
        const float inv = rsqrtf(ss + kL2Eps);
        if (row < C) s_ik[row] = inv;
        else s_iq[row - C] = inv * p.scale;
      }
    }
    if (tid < C) s_beta[tid] = tid < nv ? ((p.flags & F_BETA_PROB) ? cb : sigmoid_f(cb)) : 0.0f;
    float gl[C / 2];  // G of tokens 16 wg .. 16 wg + 15 of key channel v
    {
      const __nv_bfloat16* gr = reinterpret_cast<const __nv_bfloat16*>(raw + CT::R_G) + v;
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < C / 2; ++j) {
        const int t = (C / 2) * wg + j;
        const float la = t < nv ? -expA * softplus_log2(__bfloat162float(gr[t * D]) + dtb) : 0.0f;
        acc += la;
        gl[j] = acc;
      }
      if (wg == 0) s_tot[v] = acc;
    }
    __syncthreads();
    {
      const float off = wg ? s_tot[v] : 0.0f;
      float* Al = reinterpret_cast<float*>(sm + CT::AL);
      float prev = off;
#pragma unroll
      for (int j = 0; j < C / 2; ++j) {
        gl[j] += off;
        Gm[((C / 2) * wg + j) * CT::GS + v] = gl[j];
        Al[((C / 2) * wg + j) * CT::GS + v] = ex2_approx(gl[j] - prev);
        prev = gl[j];
      }
      if (wg == 1) s_egc[v] = ex2_approx(gl[C / 2 - 1]);
    }
    __syncthreads();

    // ---- the scaled rows [K~ ; Q~] in two bf16 terms (the B operand of G1)
#pragma unroll 1
    for (int id = tid; id < 2 * C * 16; id += CT::NT) {
      // consecutive threads take consecutive rows of one 8-channel piece, so
      // their 16-byte stores into the K-major tile fill whole bank rows
      const int row = id & (2 * C - 1), piece = id >> 6, t = row & (C - 1);
      const float sc = row < C ? s_ik[t] : s_iq[t];
      const uint4 w = *reinterpret_cast<const uint4*>(raw + CT::R_KQ + row * CT::RS + piece * 16);
      const float4 g0 = *reinterpret_cast<const float4*>(Gm + t * CT::GS + 8 * piece);
      const float4 g1 = *reinterpret_cast<const float4*>(Gm + t * CT::GS + 8 * piece + 4);
      const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        split2_bf16x2(bf16_lo(ww[e]) * sc * ex2_approx(gg[2 * e]), bf16_hi(ww[e]) * sc * ex2_approx(gg[2 * e + 1]),
                      hw[e], lw[e]);
      const uint32_t off = kmajor_offset(row, 8 * piece, D);
      *reinterpret_cast<uint4*>(sm + CT::KQT + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(sm + CT::KQT + CT::KQT_BYTES + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    // ---- the state: previous chunk's update done; split S0^T, decay by
    // e^{G_C} per key channel (this warpgroup's 64 keys of row v)
    if (c > 0 && wait_mma()) {
      aborted = true;
      break;
    }
    // K^ ^T (the B operand of the update), now that the previous update,
    // which read the tile, is done
    {
      const float gC = Gm[(C - 1) * CT::GS + v];
      const __nv_bfloat16* kcol = reinterpret_cast<const __nv_bfloat16*>(raw + CT::R_KQ) + v;
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        const int t8 = 2 * wg + tt;
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = 8 * t8 + 2 * e;
          const float x0 = __bfloat162float(kcol[t * (CT::RS / 2)]) * s_ik[t] * ex2_approx(gC - Gm[t * CT::GS + v]);
          const float x1 =
              __bfloat162float(kcol[(t + 1) * (CT::RS / 2)]) * s_ik[t + 1] * ex2_approx(gC - Gm[(t + 1) * CT::GS + v]);
          split2_bf16x2(x0, x1, hw[e], lw[e]);
        }
        const uint32_t off = kmajor_offset(v, 8 * t8, C);
        *reinterpret_cast<uint4*>(sm + CT::KBT + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(sm + CT::KBT + CT::KBT_BYTES + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
    }

    {
      // both 32-key blocks of this warpgroup's half of row v are loaded (and
      // stored back) with one wait for the pair
      float x[2][32];
      if (c == 0) {
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const int kc = 2 * wg + kk;
          if constexpr (L == L_VFIRST) {
            const float4* src = reinterpret_cast<const float4*>(state + (int64_t)v * D + 32 * kc);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 f = __ldcs(src + q);
              x[kk][4 * q] = f.x; x[kk][4 * q + 1] = f.y; x[kk][4 * q + 2] = f.z; x[kk][4 * q + 3] = f.w;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) x[kk][j] = __ldcs(state + (int64_t)(32 * kc + j) * D + v);
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
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int kc = 2 * wg + kk;
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) split2_bf16x2(x[kk][8 * q8 + 2 * i], x[kk][8 * q8 + 2 * i + 1], hw[i], lw[i]);
          const uint32_t off = kmajor_offset(v, 32 * kc + 8 * q8, D);
          *reinterpret_cast<uint4*>(sm + CT::X + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(sm + CT::X + CT::S_BYTES + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) x[kk][i] *= s_egc[32 * kc + i];
      }
      tmem_st32_issue(t_st + 64 * wg, x[0]);
      tmem_st32_issue(t_st + 64 * wg + 32, x[1]);
      tmem_wait_st();
    }
    fence_async_smem();
    tc_fence_before_sync();
    __syncthreads();

    // ---- G1 = S0^T [K~ ; Q~]^T on the tensor cores (the three products of the
    // splits above the lowest order)
    if (tid == 0) {
      tc_fence_after_sync();
      const uint32_t id_g1 = umma_idesc_bf16(128, 2 * C);
      const uint64_t da = umma_desc_kmajor(sm + CT::X, D), db = umma_desc_kmajor(sm + CT::KQT, D);
#pragma unroll
      for (int ij = 0; ij < 3; ++ij) {
        const int i = ij == 2 ? 1 : 0, j = ij == 1 ? 1 : 0;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          umma_bf16(tmem + CT::T_G1, umma_desc_add(da, i * CT::S_BYTES + ks * 256),
                    umma_desc_add(db, j * CT::KQT_BYTES + ks * 256), id_g1, ij + ks > 0);
      }
      umma_commit(&bar);
    }

    next_loads(c, 1);
    // ---- A and P on the CUDA cores while G1 runs. The pairs (t, s <= t) of
    // row t come in groups of up to three consecutive s; group g goes to
    // thread g (187 groups), so the lanes of a warp share few t-rows and
    // their t-row loads broadcast. A group takes e^{G_t - G_s} at its largest s with one
    // exponential per key channel and steps down with
    // e^{G_t - G_(s-1)} = e^{G_t - G_s} alpha_s (every factor <= 1), so a
    // chunk needs about a third of the exponentials of one per pair.
    // Channels are taken in pairs with the paired fp32 instructions.
    {
      const int item = tid;
      int t = 0, rem = item;
      while (t < C && rem >= (t + 3) / 3) {
        rem -= (t + 3) / 3;
        ++t;
      }
      if (t < C) {
        const int s0 = 3 * rem;
        const int shi = min(s0 + 2, t);  // pairs shi, shi - 1, shi - 2 (those >= s0 are kept)
        const int sm1 = max(shi - 1, 0), sm2 = max(shi - 2, 0);
        const float* Al = reinterpret_cast<const float*>(sm + CT::AL);
        float2 a2[3], p2[3];
#pragma unroll
        for (int j = 0; j < 3; ++j) a2[j] = p2[j] = make_float2(0.f, 0.f);
        const unsigned char* krow = raw + CT::R_KQ;
#pragma unroll 4
        for (int i4 = 0; i4 < D; i4 += 4) {
          const float4 gt = *reinterpret_cast<const float4*>(Gm + t * CT::GS + i4);
          const float4 gs = *reinterpret_cast<const float4*>(Gm + shi * CT::GS + i4);
          const float4 al0 = *reinterpret_cast<const float4*>(Al + shi * CT::GS + i4);
          const float4 al1 = *reinterpret_cast<const float4*>(Al + sm1 * CT::GS + i4);
          const uint2 kw = *reinterpret_cast<const uint2*>(krow + t * CT::RS + i4 * 2);
          const uint2 qw = *reinterpret_cast<const uint2*>(krow + (C + t) * CT::RS + i4 * 2);
          const uint2 sw[3] = {*reinterpret_cast<const uint2*>(krow + shi * CT::RS + i4 * 2),
                               *reinterpret_cast<const uint2*>(krow + sm1 * CT::RS + i4 * 2),
                               *reinterpret_cast<const uint2*>(krow + sm2 * CT::RS + i4 * 2)};
          const float2 kt0 = make_float2(bf16_lo(kw.x), bf16_hi(kw.x)), kt1 = make_float2(bf16_lo(kw.y), bf16_hi(kw.y));
          const float2 qt0 = make_float2(bf16_lo(qw.x), bf16_hi(qw.x)), qt1 = make_float2(bf16_lo(qw.y), bf16_hi(qw.y));
          const float2 d0 = __fadd2_rn(make_float2(gt.x, gt.y), make_float2(-gs.x, -gs.y));
          const float2 d1 = __fadd2_rn(make_float2(gt.z, gt.w), make_float2(-gs.z, -gs.w));
          float2 e0 = make_float2(ex2_approx(d0.x), ex2_approx(d0.y));
          float2 e1 = make_float2(ex2_approx(d1.x), ex2_approx(d1.y));
#pragma unroll
          for (int j = 0; j < 3; ++j) {
            const float2 w0 = __fmul2_rn(make_float2(bf16_lo(sw[j].x), bf16_hi(sw[j].x)), e0);
            const float2 w1 = __fmul2_rn(make_float2(bf16_lo(sw[j].y), bf16_hi(sw[j].y)), e1);
            a2[j] = __ffma2_rn(kt0, w0, a2[j]);
            a2[j] = __ffma2_rn(kt1, w1, a2[j]);
            p2[j] = __ffma2_rn(qt0, w0, p2[j]);
            p2[j] = __ffma2_rn(qt1, w1, p2[j]);
            if (j == 0) {
              e0 = __fmul2_rn(e0, make_float2(al0.x, al0.y));
              e1 = __fmul2_rn(e1, make_float2(al0.z, al0.w));
            } else if (j == 1) {
              e0 = __fmul2_rn(e0, make_float2(al1.x, al1.y));
              e1 = __fmul2_rn(e1, make_float2(al1.z, al1.w));
            }
          }
        }
        float* arow = reinterpret_cast<float*>(sm + CT::AM) + t * CT::AS;
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          const int sx = shi - j;
          if (sx >= s0) {
            arow[sx] = sx < t ? s_beta[t] * s_ik[t] * s_ik[sx] * (a2[j].x + a2[j].y) : 0.0f;
            uint16_t ph, pm, pl;
            split3_bf16(s_iq[t] * s_ik[sx] * (p2[j].x + p2[j].y), ph, pm, pl);
            const uint32_t off = kmajor_offset(t, sx, C);
            *reinterpret_cast<uint16_t*>(sm + CT::P3 + off) = ph;
            *reinterpret_cast<uint16_t*>(sm + CT::P3 + CT::P_BYTES + off) = pm;
            *reinterpret_cast<uint16_t*>(sm + CT::P3 + 2 * CT::P_BYTES + off) = pl;
          }
        }
      }
    }
    if (wait_mma()) {  // G1; also orders A and P before the reads below
      aborted = true;
      break;
    }

    // ---- residuals R_t = beta_t (v_t - K~_t S0) (tokens 16 wg .. 16 wg + 15),
    // into U, where the S0 split was
    float* Us = reinterpret_cast<float*>(sm + CT::US);
    {
      const __nv_bfloat16* vcol = reinterpret_cast<const __nv_bfloat16*>(raw + CT::R_V) + v;
      float y[16];
      tmem_ld16(t_g1 + 16 * wg, y);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = 16 * wg + i;
        Us[t * D + v] = s_beta[t] * (__bfloat162float(vcol[t * D]) - y[i]);
      }
    }
    __syncthreads();
    next_loads(c, 2);
    // ---- (I + A) U = R: the first warpgroup solves rows 0..15, then the
    // second subtracts what they contribute to rows 16..31 and solves those
    {
      constexpr int RB = C / 2;
      const float* Am = reinterpret_cast<const float*>(sm + CT::AM);
      const int r0 = RB * wg;
      float uu[RB];
#pragma unroll
      for (int i = 0; i < RB; ++i) uu[i] = Us[(r0 + i) * D + v];
      if (wg == 0) {
#pragma unroll
        for (int i = 1; i < RB; ++i)
#pragma unroll
          for (int j = 0; j < i; ++j) uu[i] = fmaf(-Am[i * CT::AS + j], uu[j], uu[i]);
#pragma unroll
        for (int i = 0; i < RB; ++i) Us[i * D + v] = uu[i];
      }
      __syncthreads();
      if (wg == 1) {
#pragma unroll
        for (int j4 = 0; j4 < RB; j4 += 4) {
          float lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) lo[e] = Us[(j4 + e) * D + v];
#pragma unroll
          for (int i = 0; i < RB; ++i) {
            const float4 a = *reinterpret_cast<const float4*>(Am + (r0 + i) * CT::AS + j4);
            uu[i] = fmaf(-a.x, lo[0], uu[i]);
            uu[i] = fmaf(-a.y, lo[1], uu[i]);
            uu[i] = fmaf(-a.z, lo[2], uu[i]);
            uu[i] = fmaf(-a.w, lo[3], uu[i]);
          }
        }
#pragma unroll
        for (int i = 1; i < RB; ++i)
#pragma unroll
          for (int j = 0; j < i; ++j) uu[i] = fmaf(-Am[(r0 + i) * CT::AS + r0 + j], uu[j], uu[i]);
#pragma unroll
        for (int i = 0; i < RB; ++i) Us[(r0 + i) * D + v] = uu[i];
      }
      __syncthreads();
    }
    // ---- U^T in three bf16 terms: the A operand of both the output product
    // and the update (tokens 16 wg ..)
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      const int t8 = 2 * wg + tt;
      float x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = Us[(8 * t8 + i) * D + v];
      uint4 hh, mm, ll;
      split3_bf16x8(x, hh, mm, ll);
      const uint32_t off = kmajor_offset(v, 8 * t8, C);
      *reinterpret_cast<uint4*>(sm + CT::UT3 + off) = hh;
      *reinterpret_cast<uint4*>(sm + CT::UT3 + CT::UT_BYTES + off) = mm;
      *reinterpret_cast<uint4*>(sm + CT::UT3 + 2 * CT::UT_BYTES + off) = ll;
    }
    fence_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    // ---- O^T = U^T P^T (the six products above the lowest order) and
    // S^T += U^T K^ (U in three terms, K^ in two), on the tensor cores
    if (tid == 0) {
      tc_fence_after_sync();
      const uint32_t id_o = umma_idesc_bf16(128, C);
      const uint64_t du = umma_desc_kmajor(sm + CT::UT3, C), dp = umma_desc_kmajor(sm + CT::P3, C);
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int j = 0; i + j < 3; ++j)
#pragma unroll
          for (int ks = 0; ks < C / 16; ++ks)
            umma_bf16(tmem + CT::T_O, umma_desc_add(du, i * CT::UT_BYTES + ks * 256),
                      umma_desc_add(dp, j * CT::P_BYTES + ks * 256), id_o, i + j + ks > 0);
      umma_commit(&bar_o);
      const uint32_t id_up = umma_idesc_bf16(128, D);
      const uint64_t dk = umma_desc_kmajor(sm + CT::KBT, C);
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int j = 0; j < 2 && i + j < 3; ++j)
#pragma unroll
          for (int ks = 0; ks < C / 16; ++ks)
            umma_bf16(tmem + CT::T_ST, umma_desc_add(du, i * CT::UT_BYTES + ks * 256),
                      umma_desc_add(dk, j * CT::KBT_BYTES + ks * 256), id_up, true);
      umma_commit(&bar);
    }
    next_loads(c, 3);
    if (wait_on(&bar_o, phase_o)) {
      aborted = true;
      break;
    }
    // ---- outputs o_t = Q~_t S0 + (P U)_t (tokens 16 wg ..)
    {
      float yq[16], oo[16];
      tmem_ld16(t_g1 + C + 16 * wg, yq);
      tmem_ld16(t_o + 16 * wg, oo);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = 16 * wg + i;
        if (t < nv) st_out1(p.out, ((u.tok0 + (int64_t)c * C + t) * p.HV + hv) * D + v, yq[i] + oo[i], out_bf16);
      }
    }
  }

  // ---- the final state back to the slot (this warpgroup's 64 keys of row v)
  if (!aborted) {
    if (wait_mma()) {
      aborted = true;
    } else {
#pragma unroll 1
      for (int kk = 0; kk < 2; ++kk) {
        const int kc = 2 * wg + kk;
        float x[32];
        tmem_ld32(t_st + 32 * kc, x);
        if constexpr (L == L_VFIRST) {
          float4* dst = reinterpret_cast<float4*>(state + (int64_t)v * D + 32 * kc);
#pragma unroll
          for (int q = 0; q < 8; ++q) __stcs(dst + q, make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]));
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) __stcs(state + (int64_t)(32 * kc + j) * D + v, x[j]);
        }
      }
    }
  }
  if (aborted) {
    if (tid == 0) raise_err(p.err, E_TIMEOUT);
    // a bounded chance for the MMAs in flight to finish (the last commit on
    // each barrier; an already completed phase returns at once)
    (void)mbar_wait(&bar, phase ^ 1u);
    (void)mbar_wait(&bar_o, phase_o ^ 1u);
  }
  cp_async_wait<0>();
  tc_fence_before_sync();
  __syncthreads();
  if (tid < 32) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, CT::T_COLS);
  }
}

}  // namespace gdn
