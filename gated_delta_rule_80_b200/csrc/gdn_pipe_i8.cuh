// Single-token GDN decode on V_FIRST int8_hadamard32 pools: a persistent,
// warp-specialised pipeline.
//
// Work unit ("tile"): one 32-value scale group of one (sequence, value head),
// i.e. 32 stored rows of K int8 codes (contiguous in the pool), its K scales
// (contiguous in the [V/32, K] scale array) and the token's q and k rows and
// 32-value v slice. Each CTA takes a contiguous range of tiles. One producer
// warp resolves the sequence's slot (or pages) and streams every tile into a
// ring of NS shared-memory stages with bulk copies (cp.async.bulk, completed
// in bytes on the stage's "full" mbarrier); NWC consumer warps run the step
// from shared memory and store the new codes, scales and outputs straight to
// global memory, then hand the stage back on its "empty" mbarrier. Loads of
// later tiles are therefore always in flight while a tile is computed, with
// no registers held for them.
//
// The step itself (see also gdn_tile1.cuh for the plain-state version) runs
// in the rotated basis in which the pool keeps the state: with R = H32 /
// sqrt(32) acting on the 32 values of a group (symmetric, R R = I), the step
// commutes with R, so the tile is advanced as S R = code * scale with R v
// in place of v, and the output is rotated back once (o = R (R o)). The scale
// varies along the key axis of a stored row, so it is folded into the
// per-thread key vectors:
//     a_k = |k|^-1 sum_i (k_i s_i) c_i,   a_q = scale |q|^-1 sum_i (q_i s_i) c_i,
//     S'_i = (alpha s_i) c_i + k^_i u.
// New scales: the maximum over the group's 32 rows of every key channel
// (each thread's rows first, then the CTA's partial maxima in shared
// memory), s = amax / 127 and r = 1 / s, codes rint(S' r).
//
// Thread mapping of the consumers: a lane holds 8 codes (8 bytes) of a
// stored row, LPR = K / 8 lanes a row, RPW = 32 / LPR rows per warp
// instruction, NR = 4 rows per thread (2 for K = 32). The 2 NR partial dot
// products of a thread are finished by a reduce-scatter over the row's lanes.
#pragma once

#include "gdn_pipe.cuh"
#include "gdn_tile1.cuh"

namespace gdn {

template <int K>
struct PipeI8Shape {
  static constexpr int EPL = 8;                      // codes per lane vector
  static constexpr int LPR = K / EPL;                // lanes per stored row
  static constexpr int RPW = 32 / LPR;               // rows per warp instruction
  static constexpr int VT = 32;                      // rows per tile: one scale group
  static constexpr int NWC = (K == 32) ? 2 : K / 32; // consumer warps
  static constexpr int NR = VT / (NWC * RPW);        // rows per thread
  static constexpr int NS = 4;                       // pipeline stages
  static constexpr int NT = (NWC + 1) * 32;          // + the producer warp
  static constexpr int MIN_CTAS = (NT <= 160) ? 4 : 2;  // resident CTAs the registers are sized for
  // one stage: codes | scales | q | k | v (inputs sized for fp32)
  static constexpr int CODES = VT * K;
  static constexpr int SCALES = K * 4;
  static constexpr int QK = K * 4;
  static constexpr int VV = VT * 4;
  static constexpr int STAGE = CODES + SCALES + 2 * QK + VV;
  static constexpr int SMEM = NS * STAGE;            // dynamic shared memory
};

template <int K, int IDX>
__global__ void __launch_bounds__(PipeI8Shape<K>::NT, PipeI8Shape<K>::MIN_CTAS)
step_pipe_i8(const StepParams p, int64_t n_tiles) {
  using PS = PipeI8Shape<K>;
  constexpr int EPL = PS::EPL, LPR = PS::LPR, RPW = PS::RPW, VT = PS::VT;
  constexpr int NWC = PS::NWC, NR = PS::NR, NS = PS::NS;
  constexpr int NC = NWC * 32;                       // consumer threads
  constexpr int NV = 2 * NR;                         // k.S and q.S partial sums per thread
  static_assert(LPR >= 2 && LPR <= 32 && NR >= 1 && NR * NWC * RPW == VT, "tile split");
  static_assert(NV <= LPR, "one finished sum per lane");
  constexpr int REP = LPR / NV;
  constexpr int NP = 32 / NR;                        // partial maxima per key channel
  static_assert(NP == NWC * RPW, "one partial per (warp, row lane)");
  static_assert(PS::STAGE % 16 == 0, "bulk copies need 16-byte granules");

  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t full[NS], empty[NS];
  __shared__ int s_status[NS];
  __shared__ long long s_dst[NS];
  __shared__ float s_pro[5];                         // alpha, beta, q scale, k scale, q^.k^
  __shared__ float s_vt[VT];                         // R v
  __shared__ float s_ot[VT];                         // R o
  __shared__ __align__(16) float s_part[NP][K];
  __shared__ __align__(16) float s_sc[K];
  __shared__ __align__(16) float s_rc[K];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool in_bf16 = (p.flags & F_IN_BF16) != 0;
  const int in_b = in_bf16 ? 2 : 4;
  const int NVT = p.V / VT;
  const int64_t G32 = p.V / 32;
  const int64_t t_begin = n_tiles * blockIdx.x / gridDim.x;
  const int64_t t_end = n_tiles * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_fence_init();
  }
  __syncthreads();

  // ------------------------------------------------------------------ producer
  if (warp == NWC) {
    if (lane != 0) return;
    int cur_b = -1;
    Unit u{};
    int j = 0;
    bool ok = true;
    TileCursor c;
    c.init(t_begin, p.HV, NVT);
    for (int64_t t = t_begin; t < t_end; ++t, ++j, c.next(p.HV, NVT)) {
      const int s = j % NS;
      const int b = c.b, hv = c.hv, vt = c.vt;
      if (b != cur_b) {
        u = resolve_unit<IDX>(p, b);
        raise_err(p.err, u.err);
        cur_b = b;
      }
      if (j >= NS && !mbar_wait(&empty[s], ((j / NS) - 1) & 1)) {
        ok = false;
        break;
      }
      s_status[s] = u.status;
      s_dst[s] = u.dst;
      if (u.status == U_OK) {
        unsigned char* st = smem + s * PS::STAGE;
        const uint32_t qb = K * in_b, vb = VT * in_b;
        const int h = hv / p.G;
        mbar_arrive_tx(&full[s], PS::CODES + PS::SCALES + 2 * qb + vb);
        bulk_g2s(st, reinterpret_cast<const char*>(p.pool) + ((u.src * p.HV + hv) * K * (int64_t)p.V +
                                                              (int64_t)vt * VT * K),
                 PS::CODES, &full[s]);
        bulk_g2s(st + PS::CODES, p.scales + ((u.src * p.HV + hv) * G32 + vt) * K, PS::SCALES, &full[s]);
        bulk_g2s(st + PS::CODES + PS::SCALES,
                 reinterpret_cast<const char*>(p.q) + ((int64_t)b * p.H + h) * K * in_b, qb, &full[s]);
        bulk_g2s(st + PS::CODES + PS::SCALES + PS::QK,
                 reinterpret_cast<const char*>(p.k) + ((int64_t)b * p.H + h) * K * in_b, qb, &full[s]);
        bulk_g2s(st + PS::CODES + PS::SCALES + 2 * PS::QK,
                 reinterpret_cast<const char*>(p.v) + (((int64_t)b * p.HV + hv) * p.V + (int64_t)vt * VT) * in_b,
                 vb, &full[s]);
      } else {
        mbar_arrive(&full[s]);
      }
    }
    if (!ok) {
      raise_err(p.err, E_TIMEOUT);
      // let the copies already issued land before the CTA can retire
      for (int jj = (j >= NS ? j - NS : 0); jj < j; ++jj) (void)mbar_wait(&full[jj % NS], (jj / NS) & 1);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int li = lane % LPR;
  const int ri = lane / LPR;
  const int vidx = li / REP;
  const int myrow = vidx >> 1;
  const bool holds_q = (vidx & 1) != 0;
  const int grp = lane - li;
  const bool writer = !holds_q && (li % REP) == 0;
  const int kofs = li * EPL;
  const int row0 = warp * NR * RPW + ri;            // rows row0 + jj * RPW of the tile
  const int myrow_t = row0 + myrow * RPW;
  const int pid = warp * RPW + ri;
  const bool out_bf16 = (p.flags & F_OUT_BF16) != 0;
  const bool stored_readout = (p.flags & F_READOUT_STORED) != 0;

  // per-token scalars of a tile, loaded one tile ahead
  auto scalars = [&](const TileCursor& c, float* x) {
    const int b = c.b, hv = c.hv;
    x[0] = ld_in1(p.gate, (int64_t)b * p.HV + hv, in_bf16);
    x[1] = ld_in1(p.beta, (int64_t)b * p.HV + hv, in_bf16);
    x[2] = p.A_log[hv];
    x[3] = p.dt_bias[hv];
  };
  TileCursor c, cn;
  c.init(t_begin, p.HV, NVT);
  cn = c;
  float nx[4] = {0.f, 0.f, 0.f, 0.f};
  if (warp == 0 && lane == 0 && t_begin < t_end) scalars(c, nx);
  int pb = -1, phv = -1;  // the (sequence, head) whose scalars s_pro holds

  int j = 0;
  for (int64_t t = t_begin; t < t_end; ++t, ++j, c = cn) {
    const int s = j % NS;
    const int b = c.b, hv = c.hv, vt = c.vt;
    const int64_t out_row = ((int64_t)b * p.HV + hv) * p.V + (int64_t)vt * VT;
    float cur[4] = {nx[0], nx[1], nx[2], nx[3]};
    cn.next(p.HV, NVT);
    if (warp == 0 && lane == 0 && t + 1 < t_end) scalars(cn, nx);
    const bool new_head = (b != pb || hv != phv);
    pb = b;
    phv = hv;

    const bool late = !mbar_wait(&full[s], (j / NS) & 1);
    const int status = s_status[s];
    const int64_t dst_slot = s_dst[s];
    if (bar_or(1, NC, late)) {
      if (threadIdx.x == 0) raise_err(p.err, E_TIMEOUT);
      break;
    }
    if (status != U_OK) {
      if (threadIdx.x == 0) mbar_arrive(&empty[s]);
      if (status == U_PAD)
        for (int i = threadIdx.x; i < VT; i += NC) st_out1(p.out, out_row + i, 0.0f, out_bf16);
      continue;
    }
    const unsigned char* st = smem + s * PS::STAGE;
    const unsigned char* sq = st + PS::CODES + PS::SCALES;
    const unsigned char* sk = sq + PS::QK;
    const unsigned char* sv_in = sk + PS::QK;

    // the thread's codes, scales, q and k slices
    uint2 raw[NR];
#pragma unroll
    for (int jj = 0; jj < NR; ++jj) raw[jj] = *reinterpret_cast<const uint2*>(st + (row0 + jj * RPW) * K + kofs);
    float sv[EPL], qv[EPL], kv[EPL];
    {
      const float4* sp = reinterpret_cast<const float4*>(st + PS::CODES) + kofs / 4;
      const float4 f0 = sp[0], f1 = sp[1];
      sv[0] = f0.x; sv[1] = f0.y; sv[2] = f0.z; sv[3] = f0.w;
      sv[4] = f1.x; sv[5] = f1.y; sv[6] = f1.z; sv[7] = f1.w;
    }
    ld_in_vec<EPL>(sq, kofs, in_bf16, qv);
    ld_in_vec<EPL>(sk, kofs, in_bf16, kv);

    // token prologue: warp 0 the scalars (once per (sequence, head)), the
    // last warp the rotated v
    if (warp == 0 && new_head) {
      constexpr int KPL = K / 32;
      float qn[KPL], kn[KPL];
      ld_in_vec<KPL>(sq, lane * KPL, in_bf16, qn);
      ld_in_vec<KPL>(sk, lane * KPL, in_bf16, kn);
      float ssq = 0.f, ssk = 0.f, sqk = 0.f;
#pragma unroll
      for (int e = 0; e < KPL; ++e) {
        ssq = fmaf(qn[e], qn[e], ssq);
        ssk = fmaf(kn[e], kn[e], ssk);
        sqk = fmaf(qn[e], kn[e], sqk);
      }
      ssq = group_sum<32>(ssq);
      ssk = group_sum<32>(ssk);
      sqk = group_sum<32>(sqk);
      if (lane == 0) {
        float iq = p.scale, ik = 1.0f;
        if (p.flags & F_L2NORM) {
          iq *= rsqrtf(ssq + kL2Eps);
          ik = rsqrtf(ssk + kL2Eps);
        }
        s_pro[0] = decay_of(expf(cur[2]), cur[0] + cur[3]);
        s_pro[1] = (p.flags & F_BETA_PROB) ? cur[1] : sigmoid_f(cur[1]);
        s_pro[2] = iq;
        s_pro[3] = ik;
        s_pro[4] = sqk * iq * ik;
      }
    } else if (warp == NWC - 1) {
      const float x = ld_in1(sv_in, lane, in_bf16);
      s_vt[lane] = __fmul_rn(fwht_lanes(x, lane), inv_sqrt32());
    }
    bar_sync(2, NC);
    const float alpha = s_pro[0], beta = s_pro[1], iq = s_pro[2], ik = s_pro[3], qk = s_pro[4];

    // the per-key factors: k and q times the scale (dots), alpha times the
    // scale and the normalised k (update)
    float kw[EPL], qw[EPL], fa[EPL], kh[EPL];
#pragma unroll
    for (int e = 0; e < EPL; e += 2) {
      const float2 s2 = make_float2(sv[e], sv[e + 1]);
      const float2 k2 = make_float2(kv[e], kv[e + 1]);
      const float2 a = __fmul2_rn(k2, s2), bq = __fmul2_rn(make_float2(qv[e], qv[e + 1]), s2);
      const float2 f2 = __fmul2_rn(make_float2(alpha, alpha), s2), h2 = __fmul2_rn(k2, make_float2(ik, ik));
      kw[e] = a.x; kw[e + 1] = a.y;
      qw[e] = bq.x; qw[e + 1] = bq.y;
      fa[e] = f2.x; fa[e + 1] = f2.y;
      kh[e] = h2.x; kh[e + 1] = h2.y;
    }

    // partial k.S and q.S on the code values
    float C[NR][EPL];
    float x[NV];
#pragma unroll
    for (int jj = 0; jj < NR; ++jj) {
      i8x4_to_float(raw[jj].x, C[jj]);
      i8x4_to_float(raw[jj].y, C[jj] + 4);
      float2 ak = make_float2(0.f, 0.f), aq = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < EPL; e += 2) {
        const float2 c2 = make_float2(C[jj][e], C[jj][e + 1]);
        ak = __ffma2_rn(make_float2(kw[e], kw[e + 1]), c2, ak);
        aq = __ffma2_rn(make_float2(qw[e], qw[e + 1]), c2, aq);
      }
      x[2 * jj] = ak.x + ak.y;
      x[2 * jj + 1] = aq.x + aq.y;
    }
    const float mine = ReduceScatter<NV, LPR / 2>::run(x, li);
    const float other = __shfl_xor_sync(kFull, mine, REP);
    const float dk = (holds_q ? other : mine) * ik;
    const float dq = (holds_q ? mine : other) * iq;
    const float u_mine = beta * (s_vt[myrow_t] - alpha * dk);
    const float o_mine = fmaf(qk, u_mine, alpha * dq);

    // S' = (alpha s) c + k^ u and the thread's maxima per key channel
    float m[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) m[e] = 0.f;
#pragma unroll
    for (int jj = 0; jj < NR; ++jj) {
      const float uj = __shfl_sync(kFull, u_mine, grp + 2 * jj * REP);
      const float2 u2 = make_float2(uj, uj);
#pragma unroll
      for (int e = 0; e < EPL; e += 2) {
        const float2 y = __ffma2_rn(make_float2(kh[e], kh[e + 1]), u2,
                                    __fmul2_rn(make_float2(fa[e], fa[e + 1]), make_float2(C[jj][e], C[jj][e + 1])));
        C[jj][e] = y.x;
        C[jj][e + 1] = y.y;
      }
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
#pragma unroll
      for (int jj = 0; jj + 1 < NR; jj += 2) m[e] = absmax_acc2(m[e], C[jj][e], C[jj + 1][e]);
      if constexpr (NR % 2 != 0) m[e] = absmax_acc(m[e], C[NR - 1][e]);
    }
    {
      float4* dp = reinterpret_cast<float4*>(&s_part[pid][kofs]);
      dp[0] = make_float4(fabsf(m[0]), fabsf(m[1]), fabsf(m[2]), fabsf(m[3]));
      dp[1] = make_float4(fabsf(m[4]), fabsf(m[5]), fabsf(m[6]), fabsf(m[7]));
    }
    if (writer && !stored_readout) s_ot[myrow_t] = o_mine;
    bar_sync(3, NC);
    // every read of the stage is done: hand it back to the producer
    if (threadIdx.x == 0) mbar_arrive(&empty[s]);
    for (int i = threadIdx.x; i < K; i += NC) {
      float a = s_part[0][i];
#pragma unroll
      for (int pp = 1; pp < NP; ++pp) a = fmaxf(a, s_part[pp][i]);
      float sn, r;
      h32_scale_of(a, sn, r);
      s_sc[i] = sn;
      s_rc[i] = r;
    }
    bar_sync(4, NC);

    // re-encode; codes, scales and outputs go straight to global memory
    char* dst = reinterpret_cast<char*>(p.pool) + (dst_slot * p.HV + hv) * K * (int64_t)p.V +
                (int64_t)(vt * VT + row0) * K + kofs;
    {
      float rr[EPL];
      const float4 r0 = *reinterpret_cast<const float4*>(&s_rc[kofs]);
      const float4 r1 = *reinterpret_cast<const float4*>(&s_rc[kofs + 4]);
      rr[0] = r0.x; rr[1] = r0.y; rr[2] = r0.z; rr[3] = r0.w;
      rr[4] = r1.x; rr[5] = r1.y; rr[6] = r1.z; rr[7] = r1.w;
#pragma unroll
      for (int jj = 0; jj < NR; ++jj) {
        float y[EPL];
#pragma unroll
        for (int e = 0; e < EPL; e += 2) {
          const float2 tt = __fmul2_rn(make_float2(C[jj][e], C[jj][e + 1]), make_float2(rr[e], rr[e + 1]));
          y[e] = tt.x;
          y[e + 1] = tt.y;
        }
        const uint2 cw = make_uint2(float_to_i8x4(y[0], y[1], y[2], y[3]), float_to_i8x4(y[4], y[5], y[6], y[7]));
        __stcs(reinterpret_cast<uint2*>(dst + jj * RPW * K), cw);
        if (stored_readout) {  // code values of the stored state
          i8x4_to_float(cw.x, C[jj]);
          i8x4_to_float(cw.y, C[jj] + 4);
        }
      }
    }
    {
      float* dsc = p.scales + ((dst_slot * p.HV + hv) * G32 + vt) * K;
      for (int i = threadIdx.x; i < K; i += NC) dsc[i] = s_sc[i];
    }
    if (stored_readout) {
      // o from the stored state: q^.(c s) of every row through the same reduction
      float qs[EPL];
      ld_in_vec<EPL>(p.q, ((int64_t)b * p.H + hv / p.G) * K + kofs, in_bf16, qs);  // the stage is released
#pragma unroll
      for (int e = 0; e < EPL; ++e) qs[e] *= s_sc[kofs + e];
#pragma unroll
      for (int jj = 0; jj < NR; ++jj) {
        float y = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) y = fmaf(qs[e], C[jj][e], y);
        x[2 * jj] = y * iq;
        x[2 * jj + 1] = 0.f;
      }
      const float o_st = ReduceScatter<NV, LPR / 2>::run(x, li);
      if (writer) s_ot[myrow_t] = o_st;
      bar_sync(5, NC);
    }
    // the output back from the rotated basis
    if (warp == NWC / 2) {
      const float o = __fmul_rn(fwht_lanes(s_ot[lane], lane), inv_sqrt32());
      st_out1(p.out, out_row + lane, o, out_bf16);
    }
  }
}

}  // namespace gdn
