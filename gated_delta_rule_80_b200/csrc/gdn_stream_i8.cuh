// Single-token GDN decode on V_FIRST int8_hadamard32 pools: a persistent
// kernel streaming its tiles through a ring of shared-memory stages, in the
// scheme of step_stream_fp8 (gdn_stream_fp8.cuh).
//
// Work unit ("tile"): two 32-value scale groups of one (sequence, value
// head), i.e. 64 stored rows of K int8 codes (contiguous in the pool) and the
// groups' 2 K scales (contiguous in the [V/32, K] scale array). Every thread
// copies its own 16-byte chunks of the tile NS - 1 tiles ahead with
// cp.async; the remaining threads' chunks cover the scales, the v slice and
// (on a key-head change) the q and k rows, thread 0 the gate inputs.
//
// The step runs in the rotated basis in which the pool keeps the state: with
// R = H32 / sqrt(32) acting on the 32 values of a group (symmetric, R R = I)
// the step commutes with R, so the tile is advanced as S R = code * scale
// with R v in place of v, and the output is rotated back once (o = R (R o)).
// The scale varies along the key axis of a stored row (one per key channel
// and group); the decoded values S_i = c_i s_i enter the single-pass step of
// gdn_tile1.cuh unchanged:
//     a_k = |k|^-1 k.S,   a_q = scale |q|^-1 q.S,   S'_i = alpha S_i + k^_i u.
// New scales: the maximum over the group's 32 rows of every key channel
// (each thread's rows first, then the partial maxima of the group's threads
// in shared memory), s = amax / 127 and r = 1 / s, codes rint(S' r).
// A group's 32 rows belong to NW / 2 warps; every warp rotates its group's v
// slice itself (one 32-lane butterfly), so no barrier is spent on it.
//
// Per tile the CTA meets three times: when the copies have landed; when the
// partial maxima of every (group, key channel) and the rotated outputs are
// in shared memory (the new scales s = amax / 127, r = 1 / s are then formed,
// one (group, key channel) per thread, and the outputs rotated back by one
// warp per group); and when the scales are there for the re-encode. A stored
// readout takes a fourth.
#pragma once

#include "gdn_pipe.cuh"
#include "gdn_tile1.cuh"

namespace gdn {

template <int K>
struct StreamI8Shape {
  static constexpr int EPL = 16;                 // codes per lane vector (16 bytes)
  static constexpr int VT = 64;                  // rows per tile: two scale groups
  static constexpr int NW = (K == 256) ? 8 : 4;  // warps
  static constexpr int NT = NW * 32;
  static constexpr int LPR = K / EPL;            // lanes per stored row
  static constexpr int RPW = 32 / LPR;           // rows per warp instruction
  static constexpr int NR = VT / (NW * RPW);     // rows per thread
  static constexpr int WPG = NW / 2;             // warps per scale group
  static constexpr int NP = WPG * RPW;           // partial maxima per (group, key channel)
  static constexpr int NS = 4;                   // stages in the ring
  // one stage: codes | 2 K scales | q row | k row | v slice (inputs sized for
  // fp32) | header: gate and beta words, A_log, dt_bias, status, tile index
  // within the slot, write slot, change level, gate-index parity
  static constexpr int CODES = VT * K;
  static constexpr int SCB = 2 * K * 4;
  static constexpr int QK = K * 4;
  static constexpr int VV = VT * 4;
  static constexpr int O_SC = CODES, O_Q = O_SC + SCB, O_K = O_Q + QK, O_V = O_K + QK, O_HDR = O_V + VV;
  static constexpr int STAGE = O_HDR + 48;
  static constexpr int SMEM = NS * STAGE;        // dynamic shared memory
  static constexpr int MIN_CTAS = (NW == 8) ? 1 : 3;
  static_assert(STAGE % 16 == 0, "16-byte chunks");
  static_assert(NP * NR == 32, "a group's rows");
};

template <int K, int IDX>
__global__ void __launch_bounds__(StreamI8Shape<K>::NT, StreamI8Shape<K>::MIN_CTAS)
step_stream_i8(const StepParams p, int64_t n_tiles) {
  using PS = StreamI8Shape<K>;
  constexpr int EPL = PS::EPL, LPR = PS::LPR, RPW = PS::RPW, VT = PS::VT;
  constexpr int NW = PS::NW, NR = PS::NR, NS = PS::NS, NT = PS::NT, WPG = PS::WPG, NP = PS::NP;
  constexpr int NV = 2 * NR;           // k.S and q.S partial sums per thread
  static_assert(LPR >= 2 && LPR <= 32 && NR >= 1 && NR * NW * RPW == VT, "tile split");
  static_assert(NV <= LPR, "one finished sum per lane");
  constexpr int REP = LPR / NV;        // lanes that end with the same sum
  constexpr int ROWB = K;              // bytes of one stored row
  constexpr int TILEB = VT * K;        // bytes of one tile

  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float s_gate[2][2];       // alpha, beta of a tile, by tile parity
  __shared__ __align__(16) float s_part[2][NP][K];
  __shared__ __align__(16) float s_sc[2][K];
  __shared__ __align__(16) float s_rc[2][K];
  __shared__ float s_ot[VT];           // R o of the tile's rows

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int li = lane % LPR;
  const int ri = lane / LPR;
  const int vidx = li / REP;           // the sum this lane finishes
  const int myrow = vidx >> 1;         // ... belongs to this of the thread's rows
  const bool holds_q = (vidx & 1) != 0;
  const int grp = lane - li;
  const bool writer = !holds_q && (li % REP) == 0;
  const int kofs = li * EPL;
  const int row0r = warp * NR * RPW + ri;  // tile row of row jj: row0r + jj * RPW
  const int myrow_t = row0r + myrow * RPW;
  const int g = warp / WPG;            // the thread's scale group
  const int pid = (warp % WPG) * RPW + ri;
  const int my_off = row0r * ROWB + kofs;
  const bool in_bf16 = (p.flags & F_IN_BF16) != 0;
  const bool out_bf16 = (p.flags & F_OUT_BF16) != 0;
  const bool stored_readout = (p.flags & F_READOUT_STORED) != 0;
  const int in_b = in_bf16 ? 2 : 4;
  const int NVT = p.V / VT;
  const int64_t per_b = (int64_t)p.HV * NVT;        // tiles of one sequence
  const int64_t slot_bytes = per_b * TILEB;         // one slot (or page) of the pool
  const int64_t t_begin = n_tiles * blockIdx.x / gridDim.x;
  const int64_t t_end = n_tiles * (blockIdx.x + 1) / gridDim.x;
  const int n_my = static_cast<int>(t_end - t_begin);
  if (n_my <= 0) return;
  // input chunks: scales (nsc), q (nq), k (nq), v (nvv)
  const int nsc = PS::SCB / 16;
  const int nq = K * in_b / 16;
  const int nvv = VT * in_b / 16;
  const int n_in = nsc + 2 * nq + nvv;

  // ---- producer side: copies of tile t_begin + i into stage i % NS
  StreamCursor pc;
  pc.init(t_begin, p.HV, NVT, p.G);
  int pc_change = 3;                   // relative to the previous tile
  int64_t pc_src = 0, pc_dst = 0;
  int pc_status = U_SKIP;
  auto issue = [&](int i) {
    unsigned char* st = smem + (i % NS) * PS::STAGE;
    if (pc_change == 3) {
      const Unit u = resolve_unit<IDX>(p, pc.b);
      if (threadIdx.x == 0) raise_err(p.err, u.err);
      pc_src = u.src;
      pc_dst = u.dst;
      pc_status = u.status;
    }
    if (threadIdx.x == 0) {
      int* hdr = reinterpret_cast<int*>(st + PS::O_HDR);
      hdr[4] = pc_status;
      hdr[5] = pc.within;
      *reinterpret_cast<long long*>(hdr + 6) = pc_dst;
      hdr[8] = pc_change;
      hdr[9] = (pc.b * p.HV + pc.hv) & 1;
    }
    if (pc_status == U_OK) {
      const char* src = reinterpret_cast<const char*>(p.pool) + pc_src * slot_bytes + (int64_t)pc.within * TILEB + my_off;
#pragma unroll
      for (int jj = 0; jj < NR; ++jj) cp_async16(st + my_off + jj * RPW * ROWB, src + jj * RPW * ROWB, true);
      const int64_t t = t_begin + i;
      for (int c = threadIdx.x; c < n_in; c += NT) {
        if (c < nsc) {
          const char* base = reinterpret_cast<const char*>(p.scales + (pc_src * per_b + pc.within) * 2 * K);
          cp_async16(st + PS::O_SC + c * 16, base + c * 16, true);
        } else if (c < nsc + 2 * nq) {
          if (pc_change >= 2) {
            const bool isk = c >= nsc + nq;
            const int ch = c - nsc - (isk ? nq : 0);
            const char* base =
                reinterpret_cast<const char*>(isk ? p.k : p.q) + ((int64_t)pc.b * p.H + pc.h) * K * in_b;
            cp_async16(st + (isk ? PS::O_K : PS::O_Q) + ch * 16, base + ch * 16, true);
          }
        } else {
          const int ch = c - nsc - 2 * nq;
          cp_async16(st + PS::O_V + ch * 16, reinterpret_cast<const char*>(p.v) + t * VT * in_b + ch * 16, true);
        }
      }
      if (threadIdx.x == 0 && pc_change >= 1) {
        const int64_t gi = (int64_t)pc.b * p.HV + pc.hv;
        cp_async4(st + PS::O_HDR, in_word(p.gate, gi, in_bf16));
        cp_async4(st + PS::O_HDR + 4, in_word(p.beta, gi, in_bf16));
        cp_async4(st + PS::O_HDR + 8, p.A_log + pc.hv);
        cp_async4(st + PS::O_HDR + 12, p.dt_bias + pc.hv);
      }
    }
    cp_async_commit();
    pc_change = pc.next(p.HV, NVT, p.G);
  };

  // ---- consumer side: what it needs of a tile's position is in the header
  // thread 0: alpha and beta of tile i from its stage (thread 0 copied the
  // inputs and wrote the header itself, so its own wait suffices)
  auto gate_of = [&](int i) {
    const unsigned char* st = smem + (i % NS) * PS::STAGE;
    const int* hdr = reinterpret_cast<const int*>(st + PS::O_HDR);
    const int par = i & 1;
    if (hdr[8] >= 1) {
      const int gi = hdr[9];
      const float a = in_from_word(*reinterpret_cast<const uint32_t*>(st + PS::O_HDR), gi, in_bf16);
      const float b = in_from_word(*reinterpret_cast<const uint32_t*>(st + PS::O_HDR + 4), gi, in_bf16);
      const float alog = *reinterpret_cast<const float*>(st + PS::O_HDR + 8);
      const float dtb = *reinterpret_cast<const float*>(st + PS::O_HDR + 12);
      s_gate[par][0] = decay_of(expf(alog), a + dtb);
      s_gate[par][1] = (p.flags & F_BETA_PROB) ? b : sigmoid_f(b);
    } else {
      s_gate[par][0] = s_gate[par ^ 1][0];
      s_gate[par][1] = s_gate[par ^ 1][1];
    }
  };

#pragma unroll 1
  for (int i = 0; i < NS - 1; ++i) {
    if (i < n_my) issue(i);
    else cp_async_commit();
  }
  if (threadIdx.x == 0) {
    cp_async_wait<NS - 2>();
    gate_of(0);
  }

  float qv[EPL], kv[EPL];              // raw q and k of the current key head
  float iq = 0.f, ik = 0.f, qk = 0.f;

#pragma unroll 1
  for (int j = 0; j < n_my; ++j) {
    if (j + NS - 1 < n_my) issue(j + NS - 1);
    else cp_async_commit();
    // this thread's copies of tile j have landed; after the barrier everyone's
    cp_async_wait<NS - 1>();
    __syncthreads();

    const unsigned char* st = smem + (j % NS) * PS::STAGE;
    const int* hdr = reinterpret_cast<const int*>(st + PS::O_HDR);
    const int status = hdr[4];
    const int within = hdr[5];
    const int64_t dst_slot = *reinterpret_cast<const long long*>(hdr + 6);
    const int change = hdr[8];
    const int64_t out_row = (t_begin + j) * VT;
    float S[NR][EPL];
    float x[NV];
    if (status == U_OK) {
      if (change >= 2) {
        // q and k of the new key head: raw values and their norms
        ld_in_vec<EPL>(st + PS::O_Q, kofs, in_bf16, qv);
        ld_in_vec<EPL>(st + PS::O_K, kofs, in_bf16, kv);
        float2 sq = make_float2(0.f, 0.f), sk = sq, sqk = sq;
#pragma unroll
        for (int e = 0; e < EPL; e += 2) {
          const float2 q2 = make_float2(qv[e], qv[e + 1]), k2 = make_float2(kv[e], kv[e + 1]);
          sq = __ffma2_rn(q2, q2, sq);
          sk = __ffma2_rn(k2, k2, sk);
          sqk = __ffma2_rn(q2, k2, sqk);
        }
        const float nq2 = group_sum<LPR>(sq.x + sq.y);
        const float nk2 = group_sum<LPR>(sk.x + sk.y);
        const float dqk = group_sum<LPR>(sqk.x + sqk.y);
        iq = p.scale;
        ik = 1.0f;
        if (p.flags & F_L2NORM) {
          iq *= rsqrtf(nq2 + kL2Eps);
          ik = rsqrtf(nk2 + kL2Eps);
        }
        qk = dqk * iq * ik;
      }
      const float alpha = s_gate[j & 1][0], beta = s_gate[j & 1][1];
      // R v of the group (lane = position), then this lane's row of it
      const float vl = in_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(st + PS::O_V)[32 * g + lane])
                               : reinterpret_cast<const float*>(st + PS::O_V)[32 * g + lane];
      const float vr = __fmul_rn(fwht_lanes(vl, lane), inv_sqrt32());
      const float v_mine = __shfl_sync(kFull, vr, myrow_t & 31);

      // decoded state S = code * scale, and the partial k.S and q.S of every row
      {
        float sv[EPL];
        const float4* sp = reinterpret_cast<const float4*>(st + PS::O_SC + (g * K + kofs) * 4);
#pragma unroll
        for (int c4 = 0; c4 < EPL / 4; ++c4) {
          const float4 f = sp[c4];
          sv[4 * c4] = f.x; sv[4 * c4 + 1] = f.y; sv[4 * c4 + 2] = f.z; sv[4 * c4 + 3] = f.w;
        }
#pragma unroll
        for (int jj = 0; jj < NR; ++jj) {
          const uint4 raw = *reinterpret_cast<const uint4*>(st + my_off + jj * RPW * ROWB);
          i8x4_to_float(raw.x, S[jj]);
          i8x4_to_float(raw.y, S[jj] + 4);
          i8x4_to_float(raw.z, S[jj] + 8);
          i8x4_to_float(raw.w, S[jj] + 12);
          float2 ak = make_float2(0.f, 0.f), aq = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < EPL; e += 2) {
            const float2 s2 = __fmul2_rn(make_float2(S[jj][e], S[jj][e + 1]), make_float2(sv[e], sv[e + 1]));
            S[jj][e] = s2.x;
            S[jj][e + 1] = s2.y;
            ak = __ffma2_rn(make_float2(kv[e], kv[e + 1]), s2, ak);
            aq = __ffma2_rn(make_float2(qv[e], qv[e + 1]), s2, aq);
          }
          x[2 * jj] = ak.x + ak.y;
          x[2 * jj + 1] = aq.x + aq.y;
        }
      }
      const float mine = ReduceScatter<NV, LPR / 2>::run(x, li);
      const float other = __shfl_xor_sync(kFull, mine, REP);
      const float dk = (holds_q ? other : mine) * ik;
      const float dq = (holds_q ? mine : other) * iq;
      const float u_mine = beta * (v_mine - alpha * dk);
      if (writer && !stored_readout) s_ot[myrow_t] = fmaf(qk, u_mine, alpha * dq);

      // S' = alpha S + k (|k|^-1 u), and the thread's maxima per key channel
      const float2 a2 = make_float2(alpha, alpha);
      const float un = u_mine * ik;
#pragma unroll
      for (int jj = 0; jj < NR; ++jj) {
        const float uj = __shfl_sync(kFull, un, grp + 2 * jj * REP);
        const float2 u2 = make_float2(uj, uj);
#pragma unroll
        for (int e = 0; e < EPL; e += 2) {
          const float2 y =
              __ffma2_rn(make_float2(kv[e], kv[e + 1]), u2, __fmul2_rn(a2, make_float2(S[jj][e], S[jj][e + 1])));
          S[jj][e] = y.x;
          S[jj][e + 1] = y.y;
        }
      }
      float m[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        m[e] = 0.f;
#pragma unroll
        for (int jj = 0; jj + 1 < NR; jj += 2) m[e] = absmax_acc2(m[e], S[jj][e], S[jj + 1][e]);
        if constexpr (NR % 2 != 0) m[e] = absmax_acc(m[e], S[NR - 1][e]);
      }
      float4* dp = reinterpret_cast<float4*>(&s_part[g][pid][kofs]);
#pragma unroll
      for (int c4 = 0; c4 < EPL / 4; ++c4) dp[c4] = make_float4(m[4 * c4], m[4 * c4 + 1], m[4 * c4 + 2], m[4 * c4 + 3]);
    }
    __syncthreads();

    if (status == U_OK) {
      // new scales, one (group, key channel) at a time; stored at once
      float* dsc = p.scales + (dst_slot * per_b + within) * 2 * K;
      for (int c = threadIdx.x; c < 2 * K; c += NT) {
        const int gg = c / K, i = c - gg * K;
        float a = s_part[gg][0][i];
#pragma unroll
        for (int pp = 1; pp < NP; ++pp) a = fmaxf(a, s_part[gg][pp][i]);
        float sn, r;
        h32_scale_of(a, sn, r);
        s_sc[gg][i] = sn;
        s_rc[gg][i] = r;
        dsc[c] = sn;
      }
      // the outputs back from the rotated basis, one warp per group
      if (!stored_readout && warp % WPG == 0) {
        const float o = __fmul_rn(fwht_lanes(s_ot[32 * g + lane], lane), inv_sqrt32());
        st_out1(p.out, out_row + 32 * g + lane, o, out_bf16);
      }
    } else if (status == U_PAD) {
      if (writer) st_out1(p.out, out_row + myrow_t, 0.0f, out_bf16);
    }
    __syncthreads();

    if (status == U_OK) {
      // re-encode rint(S' r), four key channels (one code word per row) at a time
      uint32_t cw[NR][EPL / 4];
#pragma unroll
      for (int c4 = 0; c4 < EPL / 4; ++c4) {
        const float4 r4 = *reinterpret_cast<const float4*>(&s_rc[g][kofs + 4 * c4]);
#pragma unroll
        for (int jj = 0; jj < NR; ++jj) {
          const float2 lo = __fmul2_rn(make_float2(S[jj][4 * c4], S[jj][4 * c4 + 1]), make_float2(r4.x, r4.y));
          const float2 hi = __fmul2_rn(make_float2(S[jj][4 * c4 + 2], S[jj][4 * c4 + 3]), make_float2(r4.z, r4.w));
          cw[jj][c4] = float_to_i8x4(lo.x, lo.y, hi.x, hi.y);
        }
      }
      char* dst = reinterpret_cast<char*>(p.pool) + dst_slot * slot_bytes + (int64_t)within * TILEB + my_off;
#pragma unroll
      for (int jj = 0; jj < NR; ++jj)
        st_stream16(dst + jj * RPW * ROWB, make_uint4(cw[jj][0], cw[jj][1], cw[jj][2], cw[jj][3]));
      if (stored_readout) {
        // o from the stored state: q^.(c s) of every row through the same reduction
#pragma unroll
        for (int jj = 0; jj < NR; ++jj) x[2 * jj] = x[2 * jj + 1] = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < EPL / 4; ++c4) {
          const float4 s4 = *reinterpret_cast<const float4*>(&s_sc[g][kofs + 4 * c4]);
          const float qs[4] = {qv[4 * c4] * s4.x, qv[4 * c4 + 1] * s4.y, qv[4 * c4 + 2] * s4.z, qv[4 * c4 + 3] * s4.w};
#pragma unroll
          for (int jj = 0; jj < NR; ++jj) {
            float c[4];
            i8x4_to_float(cw[jj][c4], c);
#pragma unroll
            for (int e = 0; e < 4; ++e) x[2 * jj] = fmaf(qs[e], c[e], x[2 * jj]);
          }
        }
#pragma unroll
        for (int jj = 0; jj < NR; ++jj) x[2 * jj] *= iq;
        const float o_st = ReduceScatter<NV, LPR / 2>::run(x, li);
        if (writer) s_ot[myrow_t] = o_st;
      }
    }
    if (stored_readout) {
      __syncthreads();
      if (status == U_OK && warp % WPG == 0) {
        const float o = __fmul_rn(fwht_lanes(s_ot[32 * g + lane], lane), inv_sqrt32());
        st_out1(p.out, out_row + 32 * g + lane, o, out_bf16);
      }
    }

    // advance; thread 0 publishes the next tile's gate and beta (the next
    // tile's first barrier makes them visible)
    if (threadIdx.x == 0 && j + 1 < n_my) {
      cp_async_wait<NS - 2>();
      gate_of(j + 1);
    }
  }
  cp_async_wait<0>();
}

}  // namespace gdn
