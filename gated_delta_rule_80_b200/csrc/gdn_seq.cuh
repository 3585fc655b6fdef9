// Decode of T >= 1 tokens per unit (GDN short suffix, KDA varlen) and of
// K_FIRST pools: one CTA per (sequence, value head, V-tile) holding the
// tile in registers for all of the unit's tokens.
//
// Everything a token step needs that does not depend on the state (q and k
// normalised, q.k, the gate alpha -- a scalar for GDN, a K-vector for KDA --,
// beta and the v slice) is computed for a chunk of up to TC tokens in
// parallel, one warp per token, into shared memory, while the tile's loads
// are in flight. The token loop then only runs the state-dependent part of
// the single-pass step:
//     a_k = (alpha o k^).S, a_q = (alpha o q^).S, u = beta (v - a_k),
//     S' = diag(alpha) S + k^ u^T, o = a_q + (q^.k^) u
// (for GDN alpha is a scalar and multiplies the reduced sums instead).
//
// Thread mappings (reductions stay inside a warp; fp8 takes one CTA barrier
// per token for the tile amax, int8_hadamard32 two for its group scales):
//  * V_FIRST (tile = VC stored rows of K): LPR lanes hold one row in 16-byte
//    vectors, a thread holds NR rows; the 2 NR row sums are finished by a
//    reduce-scatter over the row's lanes.
//  * K_FIRST (tile = K rows x VC columns): a warp owns 16 columns of all K
//    rows; lanes are 8 row groups x 4 column quads (4 elements per lane), a
//    thread holds K/8 rows. The 8 column sums (k and q for 4 columns) are
//    finished by a reduce-scatter over the 8 row groups.
//
// int8_hadamard32 states are worked on in their rotated basis: with
// R = H32 / sqrt(32) acting on each 32-value group (symmetric, R R = I), the
// step commutes with the rotation -- S R advanced by R v gives S' R and reads
// out R o -- so the tile decodes to S R directly (code * scale), the token's
// v slice is rotated once in the prologue, the outputs are rotated back once
// per chunk, and the state itself is never transformed.
#pragma once

#include "gdn_tile1.cuh"

namespace gdn {

template <int N, int O, int STOP>
struct ReduceScatterS {
  // As ReduceScatter, over the lanes that differ in bits STOP..O of the lane id.
  __device__ __forceinline__ static float run(float* x, int lane) {
    if constexpr (N > 1) {
      const bool hi = (lane & O) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        const float keep = hi ? x[N / 2 + i] : x[i];
        const float send = hi ? x[i] : x[N / 2 + i];
        x[i] = keep + __shfl_xor_sync(kFull, send, O);
      }
      return ReduceScatterS<N / 2, O / 2, STOP>::run(x, lane);
    } else {
      float v = x[0];
#pragma unroll
      for (int o = O; o >= STOP; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
      return v;
    }
  }
};

template <int SDT, int LAYOUT, int K, int NW>
struct SeqShape {
  // tokens per prologue chunk (4 for int8 K=256, whose scale-group buffers
  // would otherwise push the static shared memory past 48 KiB; 16 for small
  // heads, whose runs are latency-bound and whose buffers are small)
  static constexpr int TC = (SDT == ST_I8H && K == 256) ? 4 : (K <= 64 ? 16 : 8);
  // V_FIRST: 16-byte vectors (32 for a K=256 fp32 row, so that it fits a warp)
  static constexpr int VB_V = (SDT == ST_F32 && K == 256) ? 32 : 16;
  // K_FIRST: 4 elements per lane, CPL lanes per row segment (16 columns per
  // warp; 8 for K = 256 so that a thread holds K/16 rows)
  static constexpr int CPL = (K == 256) ? 2 : 4;
  static constexpr int EPL = (LAYOUT == L_VFIRST) ? VB_V / StateTraits<SDT>::BYTES : 4;
  // fp8: the [K, 64] scale tile; int8_hadamard32: two 32-value scale groups
  static constexpr int VC = (LAYOUT == L_VFIRST) ? ((SDT == ST_FP8 || SDT == ST_I8H) ? 64 : (K == 256 ? 16 : 32))
                                                 : CPL * 4 * NW;
};

template <int SDT, int LAYOUT, int K, int GATE, int IDX, int NW>
__global__ void __launch_bounds__(NW * 32)
step_seq(const StepParams p) {
  using ST = StateTraits<SDT>;
  using SH = SeqShape<SDT, LAYOUT, K, NW>;
  constexpr int TC = SH::TC;
  constexpr int EPL = SH::EPL;
  constexpr int VC = SH::VC;
  constexpr int VB = EPL * ST::BYTES;  // bytes per lane vector
  static_assert(VB == 4 || VB == 8 || VB == 16 || VB == 32, "vector width");
  constexpr bool VF = (LAYOUT == L_VFIRST);
  constexpr int CPL = SH::CPL;        // K_FIRST lanes per row segment
  constexpr int RG = 32 / CPL;        // K_FIRST row groups
  // V_FIRST geometry
  constexpr int LPR = VF ? K / EPL : CPL;
  constexpr int RPW = 32 / LPR;
  constexpr int NR = VF ? VC / (NW * RPW) : K / RG;  // rows per thread
  static_assert(!VF || (LPR >= 2 && LPR <= 32 && NR >= 1 && NR * NW * RPW == VC), "V_FIRST tile split");
  static_assert(VF || (K % RG == 0 && VC == CPL * EPL * NW), "K_FIRST tile split");
  constexpr int NV = VF ? 2 * NR : 2 * EPL;  // partial sums per thread
  static_assert(!VF || NV <= LPR, "one finished sum per lane");
  static_assert(VF || NV <= RG, "one finished sum per lane");
  constexpr int REP = VF ? LPR / NV : 1;
  constexpr int KPL = K / 32;
  constexpr bool I8 = (SDT == ST_I8H);
  // int8_hadamard32: 32-value scale groups in the tile, and partial maxima
  // per (group, key channel): V_FIRST one per stored row a thread holds of
  // the group, K_FIRST one per 4-column lane vector
  constexpr int NG = I8 ? VC / 32 : 1;
  constexpr int NP = I8 ? (VF ? 32 / NR : 8) : 1;
  static_assert(!I8 || VC % 32 == 0, "whole scale groups per tile");
  static_assert(!I8 || !VF || 32 % (NR * RPW) == 0, "a warp's rows stay inside one scale group");

  // K_FIRST fp32 with a decay per key channel (KDA): a thread reads one key
  // row at a time, so the row's scalars sit in pairs, (alpha k^, alpha q^)
  // for the dots and (k^, alpha) for the update, one 8-byte load each (s_q
  // keeps q^ for a stored readout)
  constexpr bool KW = !VF && GATE == GATE_VECTOR && SDT == ST_F32;
  __shared__ __align__(16) float s_q[TC][K];
  __shared__ __align__(16) float s_k[TC][KW ? 1 : K];
  __shared__ __align__(16) float s_a[TC][(GATE == GATE_VECTOR && !KW) ? K : 1];
  __shared__ __align__(16) float2 s_wd[KW ? TC : 1][KW ? K : 1];
  __shared__ __align__(16) float2 s_wu[KW ? TC : 1][KW ? K : 1];
  __shared__ __align__(16) float s_v[TC][VC];
  __shared__ float s_b[TC], s_qk[TC];
  __shared__ float s_amax[2][NW];
  __shared__ __align__(16) float s_part[NG][NP][I8 ? K : 1];
  __shared__ __align__(16) float s_sc[NG][I8 ? K : 1];
  __shared__ __align__(16) float s_rc[NG][I8 ? K : 1];
  __shared__ float s_ot[I8 ? TC : 1][I8 ? VC : 1];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int tile = blockIdx.x;
  const int hv = blockIdx.y;
  const int b = blockIdx.z;
  const int h = hv / p.G;
  const int v0 = tile * VC;
  const int64_t V = p.V;
  const bool in_bf16 = (p.flags & F_IN_BF16) != 0;
  const bool out_bf16 = (p.flags & F_OUT_BF16) != 0;
  const bool stored_readout = (p.flags & F_READOUT_STORED) != 0;

  // ---- thread geometry
  // V_FIRST: rows row0 + jj * RPW, elements kofs..kofs+EPL of each row.
  // K_FIRST: rows g + RG j, columns c0..c0+3 (all relative to the tile).
  const int li = VF ? lane % LPR : lane % CPL;
  const int g = lane / CPL;  // K_FIRST row group
  const int kofs = li * EPL;
  const int row0 = VF ? warp * NR * RPW + lane / LPR : 0;
  const int c0 = VF ? 0 : warp * CPL * 4 + li * 4;
  // the sum a lane finishes: V_FIRST value index li / REP (row, k or q);
  // K_FIRST value index from lane bits 4..2 (column >> 1, k or q); for
  // CPL == 2, lane bit 1 is a replica
  const int vidx = VF ? li / REP : (lane >> 2) & 7;
  const bool holds_q = (vidx & 1) != 0;
  const int mycol = vidx >> 1;  // V_FIRST: row of the thread; K_FIRST: column in the lane's 4
  const int grp = VF ? lane - li : li;
  const bool writer = VF ? (!holds_q && (li % REP) == 0) : (!holds_q && (CPL == 4 || (lane & 2) == 0));
  // int8_hadamard32: the thread's scale group in the tile, and which partial
  // maximum of that group it writes
  [[maybe_unused]] const int tg = VF ? (warp * NR * RPW) / 32 : c0 / 32;
  [[maybe_unused]] const int pid =
      VF ? lane / LPR + RPW * (((warp * NR * RPW) % 32) / (NR * RPW)) : (c0 % 32) / 4;

  const Unit u = resolve_unit<IDX>(p, b);
  if (threadIdx.x == 0) raise_err(p.err, u.err);
  if (u.status == U_SKIP || u.tok1 <= u.tok0) return;
  // output position of the value this thread writes
  const int out_col = VF ? v0 + row0 + mycol * RPW : v0 + c0 + mycol;
  if (u.status == U_PAD) {
    if (writer)
      for (int tok = u.tok0; tok < u.tok1; ++tok) st_out1(p.out, ((int64_t)tok * p.HV + hv) * V + out_col, 0.0f, out_bf16);
    return;
  }

  // ---- state tile loads
  using SV = StateVec<SDT, (VB >= 16 ? VB : 8)>;
  const int64_t head_bytes = (int64_t)K * V * ST::BYTES;
  const char* src = reinterpret_cast<const char*>(p.pool) + ((u.fresh ? 0 : u.src) * p.HV + hv) * head_bytes;
  float S[NR][EPL];
  // element offset (within the head) of vector jj of this thread
  auto vec_off = [&](int jj) -> int64_t {
    if constexpr (VF) return (int64_t)(v0 + row0 + jj * RPW) * K + kofs;
    else return (int64_t)(g + RG * jj) * V + v0 + c0;
  };
  if (u.fresh) {  // a paged prefill with no earlier token: S starts at zero
#pragma unroll
    for (int jj = 0; jj < NR; ++jj)
#pragma unroll
      for (int e = 0; e < EPL; ++e) S[jj][e] = 0.0f;
  } else if constexpr (VB >= 8) {
    typename SV::T raw[NR];
#pragma unroll
    for (int jj = 0; jj < NR; ++jj) raw[jj] = SV::load(src + vec_off(jj) * ST::BYTES);
#pragma unroll
    for (int jj = 0; jj < NR; ++jj) SV::decode(raw[jj], S[jj]);
  } else {  // 4 fp8 or int8 codes
    uint32_t raw[NR];
#pragma unroll
    for (int jj = 0; jj < NR; ++jj) raw[jj] = __ldcs(reinterpret_cast<const unsigned int*>(src + vec_off(jj)));
#pragma unroll
    for (int jj = 0; jj < NR; ++jj) {
      if constexpr (I8) {
        i8x4_to_float(raw[jj], S[jj]);
      } else {
        e4m3x4_to_float4(raw[jj], S[jj]);
      }
    }
  }
  const int n_scale = p.V / 64;
  const int stile = v0 / 64;  // fp8: this CTA's scale tile
  if constexpr (SDT == ST_FP8) {
    const float sc = u.fresh ? 0.0f : p.scales[(u.src * p.HV + hv) * n_scale + stile];
#pragma unroll
    for (int jj = 0; jj < NR; ++jj)
#pragma unroll
      for (int e = 0; e < EPL; ++e) S[jj][e] = __fmul_rn(S[jj][e], sc);
  } else if constexpr (I8) {
    // code * scale of the element's (group, key channel): the state in the
    // rotated basis
    if (!u.fresh) {
      const float* sc = p.scales + ((u.src * p.HV + hv) * (int64_t)(V / 32) + v0 / 32 + tg) * K;
      if constexpr (VF) {
        float sv[EPL];
#pragma unroll
        for (int c = 0; c < EPL / 4; ++c) {
          const float4 f = reinterpret_cast<const float4*>(sc + kofs)[c];
          sv[4 * c] = f.x; sv[4 * c + 1] = f.y; sv[4 * c + 2] = f.z; sv[4 * c + 3] = f.w;
        }
#pragma unroll
        for (int jj = 0; jj < NR; ++jj)
#pragma unroll
          for (int e = 0; e < EPL; ++e) S[jj][e] = __fmul_rn(S[jj][e], sv[e]);
      } else {
#pragma unroll
        for (int jj = 0; jj < NR; ++jj) {
          const float sj = sc[g + RG * jj];
#pragma unroll
          for (int e = 0; e < EPL; ++e) S[jj][e] = __fmul_rn(S[jj][e], sj);
        }
      }
    }
  }

  const float expA = expf(p.A_log[hv]);
  [[maybe_unused]] float s_last = 0.0f;
  [[maybe_unused]] uint32_t codes[NR][EPL / 4];

  // store the tile (in its storage format) to pool slot/page `slot`
  auto store_tile = [&](int64_t slot) {
    char* dst = reinterpret_cast<char*>(p.pool) + (slot * p.HV + hv) * head_bytes;
    if constexpr (SDT == ST_FP8 || I8) {
#pragma unroll
      for (int jj = 0; jj < NR; ++jj) {
        char* a = dst + vec_off(jj);
        if constexpr (EPL == 16) st_stream16(a, make_uint4(codes[jj][0], codes[jj][1], codes[jj][2], codes[jj][3]));
        else if constexpr (EPL == 8) __stcs(reinterpret_cast<uint2*>(a), make_uint2(codes[jj][0], codes[jj][1]));
        else __stcs(reinterpret_cast<unsigned int*>(a), codes[jj][0]);
      }
      if constexpr (I8) {
        // the tile's groups are consecutive rows of the [V/32, K] scale array
        float* dsc = p.scales + ((slot * p.HV + hv) * (int64_t)(V / 32) + v0 / 32) * K;
        for (int i = threadIdx.x; i < NG * K; i += NW * 32) dsc[i] = s_sc[i / K][i % K];
      } else if (threadIdx.x == 0) {
        p.scales[(slot * p.HV + hv) * n_scale + stile] = s_last;
      }
    } else {
#pragma unroll
      for (int jj = 0; jj < NR; ++jj) SV::store(dst + vec_off(jj) * ST::BYTES, SV::encode(S[jj]));
    }
  };

  for (int t0 = u.tok0; t0 < u.tok1; t0 += TC) {
    const int nt = min(TC, u.tok1 - t0);
    // ---- prologue of the chunk: one warp per token
    for (int tt = warp; tt < nt; tt += NW) {
      const int tok = t0 + tt;
      const int64_t qrow = ((int64_t)tok * p.H + h) * K;
      float qn[KPL], kn[KPL];
      ld_in_vec<KPL>(p.q, qrow + lane * KPL, in_bf16, qn);
      ld_in_vec<KPL>(p.k, qrow + lane * KPL, in_bf16, kn);
      float sq = 0.f, sk = 0.f, sqk = 0.f;
#pragma unroll
      for (int e = 0; e < KPL; ++e) {
        sq = fmaf(qn[e], qn[e], sq);
        sk = fmaf(kn[e], kn[e], sk);
        sqk = fmaf(qn[e], kn[e], sqk);
      }
      sq = group_sum<32>(sq);
      sk = group_sum<32>(sk);
      sqk = group_sum<32>(sqk);
      float iq = p.scale, ik = 1.0f;
      if (p.flags & F_L2NORM) {
        iq *= rsqrtf(sq + kL2Eps);
        ik = rsqrtf(sk + kL2Eps);
      }
      if constexpr (KW) {
        float gv[KPL], db[KPL];
        ld_in_vec<KPL>(p.gate, ((int64_t)tok * p.HV + hv) * K + lane * KPL, in_bf16, gv);
        ld_in_vec<KPL>(p.dt_bias, (int64_t)hv * K + lane * KPL, false, db);
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
          const float a = decay_of(expA, gv[e] + db[e]);
          const float kh = kn[e] * ik, qh = qn[e] * iq;
          s_q[tt][lane * KPL + e] = qh;
          s_wd[tt][lane * KPL + e] = make_float2(a * kh, a * qh);
          s_wu[tt][lane * KPL + e] = make_float2(kh, a);
        }
      } else {
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
          s_q[tt][lane * KPL + e] = qn[e] * iq;
          s_k[tt][lane * KPL + e] = kn[e] * ik;
        }
        if constexpr (GATE == GATE_VECTOR) {
          float gv[KPL], db[KPL];
          ld_in_vec<KPL>(p.gate, ((int64_t)tok * p.HV + hv) * K + lane * KPL, in_bf16, gv);
          ld_in_vec<KPL>(p.dt_bias, (int64_t)hv * K + lane * KPL, false, db);
#pragma unroll
          for (int e = 0; e < KPL; ++e) s_a[tt][lane * KPL + e] = decay_of(expA, gv[e] + db[e]);
        }
      }
      for (int c = lane; c < VC; c += 32) {
        float x = ld_in1(p.v, ((int64_t)tok * p.HV + hv) * V + v0 + c, in_bf16);
        if constexpr (I8) x = __fmul_rn(fwht_lanes(x, lane), inv_sqrt32());  // R v of one group
        s_v[tt][c] = x;
      }
      if (lane == 0) {
        const float braw = ld_in1(p.beta, (int64_t)tok * p.HV + hv, in_bf16);
        s_b[tt] = (p.flags & F_BETA_PROB) ? braw : sigmoid_f(braw);
        s_qk[tt] = sqk * iq * ik;
        if constexpr (GATE == GATE_SCALAR)
          s_a[tt][0] = decay_of(expA, ld_in1(p.gate, (int64_t)tok * p.HV + hv, in_bf16) + p.dt_bias[hv]);
      }
    }
    __syncthreads();

    // ---- the state-dependent part, token by token
    for (int tt = 0; tt < nt; ++tt) {
      const int tok = t0 + tt;
      const bool last = (tok + 1 == u.tok1);
      const float beta = s_b[tt], qk = s_qk[tt];
      [[maybe_unused]] const float alpha = (GATE == GATE_SCALAR) ? s_a[tt][0] : 1.0f;
      float x[NV];
      float kw[VF ? EPL : NR];  // k^ of the thread's key positions (update)
      if constexpr (VF) {
        float qw[EPL], kk[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          kw[e] = s_k[tt][kofs + e];
          qw[e] = s_q[tt][kofs + e];
          kk[e] = kw[e];
          if constexpr (GATE == GATE_VECTOR) {
            const float a = s_a[tt][kofs + e];
            kk[e] *= a;
            qw[e] *= a;
          }
        }
#pragma unroll
        for (int jj = 0; jj < NR; ++jj) {
          float2 ak = make_float2(0.f, 0.f), aq = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < EPL; e += 2) {
            const float2 s2 = make_float2(S[jj][e], S[jj][e + 1]);
            ak = __ffma2_rn(make_float2(kk[e], kk[e + 1]), s2, ak);
            aq = __ffma2_rn(make_float2(qw[e], qw[e + 1]), s2, aq);
          }
          x[2 * jj] = ak.x + ak.y;
          x[2 * jj + 1] = aq.x + aq.y;
        }
      } else {
        float2 ak[EPL / 2], aq[EPL / 2];
#pragma unroll
        for (int c = 0; c < EPL / 2; ++c) { ak[c] = make_float2(0.f, 0.f); aq[c] = make_float2(0.f, 0.f); }
#pragma unroll
        for (int jj = 0; jj < NR; ++jj) {
          const int r = g + RG * jj;
          float wk, wq;
          if constexpr (KW) {
            const float2 w = s_wd[tt][r];
            wk = w.x;
            wq = w.y;
          } else {
            kw[jj] = s_k[tt][r];
            wk = kw[jj];
            wq = s_q[tt][r];
            if constexpr (GATE == GATE_VECTOR) {
              const float a = s_a[tt][r];
              wk *= a;
              wq *= a;
            }
          }
          const float2 wk2 = make_float2(wk, wk), wq2 = make_float2(wq, wq);
#pragma unroll
          for (int c = 0; c < EPL / 2; ++c) {
            const float2 s2 = make_float2(S[jj][2 * c], S[jj][2 * c + 1]);
            ak[c] = __ffma2_rn(wk2, s2, ak[c]);
            aq[c] = __ffma2_rn(wq2, s2, aq[c]);
          }
        }
#pragma unroll
        for (int c = 0; c < EPL / 2; ++c) {
          x[4 * c + 0] = ak[c].x;
          x[4 * c + 1] = aq[c].x;
          x[4 * c + 2] = ak[c].y;
          x[4 * c + 3] = aq[c].y;
        }
      }
      float mine;
      if constexpr (VF) mine = ReduceScatterS<NV, LPR / 2, 1>::run(x, lane);
      else mine = ReduceScatterS<NV, 16, CPL>::run(x, lane);
      constexpr int PAIR = VF ? REP : 4;  // lane offset between the k and q sums of one row/column
      const float other = __shfl_xor_sync(kFull, mine, PAIR);
      const float dk = holds_q ? other : mine;
      const float dq = holds_q ? mine : other;
      const float vval = VF ? s_v[tt][row0 + mycol * RPW] : s_v[tt][c0 + mycol];
      float u_mine, o_mine;
      if constexpr (GATE == GATE_SCALAR) {
        u_mine = beta * (vval - alpha * dk);
        o_mine = fmaf(qk, u_mine, alpha * dq);
      } else {
        u_mine = beta * (vval - dk);
        o_mine = fmaf(qk, u_mine, dq);
      }
      // u of every row (V_FIRST) / column (K_FIRST) the thread updates
      float uu[VF ? NR : EPL];
      if constexpr (VF) {
#pragma unroll
        for (int jj = 0; jj < NR; ++jj) uu[jj] = __shfl_sync(kFull, u_mine, grp + 2 * jj * REP);
      } else {
#pragma unroll
        for (int c = 0; c < EPL; ++c) uu[c] = __shfl_sync(kFull, u_mine, (2 * c) * 4 + grp);  // lane bit 1 = 0
      }
      // S' = diag(alpha) S + k^ u^T
#pragma unroll
      for (int jj = 0; jj < NR; ++jj) {
#pragma unroll
        for (int e = 0; e < EPL; e += 2) {
          float2 f2, k2, u2;
          if constexpr (VF) {
            k2 = make_float2(kw[e], kw[e + 1]);
            u2 = make_float2(uu[jj], uu[jj]);
            if constexpr (GATE == GATE_SCALAR) f2 = make_float2(alpha, alpha);
            else f2 = make_float2(s_a[tt][kofs + e], s_a[tt][kofs + e + 1]);
          } else {
            u2 = make_float2(uu[e], uu[e + 1]);
            if constexpr (KW) {
              const float2 w = s_wu[tt][g + RG * jj];
              k2 = make_float2(w.x, w.x);
              f2 = make_float2(w.y, w.y);
            } else {
              k2 = make_float2(kw[jj], kw[jj]);
              if constexpr (GATE == GATE_SCALAR) f2 = make_float2(alpha, alpha);
              else {
                const float a = s_a[tt][g + RG * jj];
                f2 = make_float2(a, a);
              }
            }
          }
          const float2 y = __ffma2_rn(k2, u2, __fmul2_rn(f2, make_float2(S[jj][e], S[jj][e + 1])));
          S[jj][e] = y.x;
          S[jj][e + 1] = y.y;
        }
      }
      // storage format after every token
      if constexpr (SDT == ST_BF16) {
#pragma unroll
        for (int jj = 0; jj < NR; ++jj)
#pragma unroll
          for (int e = 0; e < EPL; ++e) S[jj][e] = round_bf16(S[jj][e]);
      } else if constexpr (SDT == ST_FP8) {
        float m = 0.f;
#pragma unroll
        for (int jj = 0; jj < NR; ++jj)
#pragma unroll
          for (int e = 0; e < EPL; e += 2) m = absmax_acc2(m, S[jj][e], S[jj][e + 1]);
        m = group_max<32>(m);
        const int buf = (tok - u.tok0) & 1;
        if (lane == 0) s_amax[buf][warp] = m;
        __syncthreads();
        float amax = s_amax[buf][0];
#pragma unroll
        for (int w = 1; w < NW; ++w) amax = fmaxf(amax, s_amax[buf][w]);
        float sn, r;
        fp8_scale_of(amax, sn, r);
        s_last = sn;
        const float2 r2 = make_float2(r, r);
#pragma unroll
        for (int jj = 0; jj < NR; ++jj) {
#pragma unroll
          for (int w4 = 0; w4 < EPL / 4; ++w4) {
            float y[4];
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
              const float2 t2 = __fmul2_rn(make_float2(S[jj][4 * w4 + e], S[jj][4 * w4 + e + 1]), r2);
              y[e] = t2.x;
              y[e + 1] = t2.y;
            }
            const uint32_t cw = (r == 0.0f) ? 0u : float4_to_e4m3x4(y[0], y[1], y[2], y[3]);
            codes[jj][w4] = cw;
            if (!last || stored_readout) {
              float d[4];
              e4m3x4_to_float4(cw, d);
#pragma unroll
              for (int e = 0; e < 4; ++e) S[jj][4 * w4 + e] = __fmul_rn(d[e], sn);
            }
          }
        }
      } else if constexpr (I8) {
        // group maxima: the thread's part, then the CTA's
        if constexpr (VF) {
          float m[EPL];
#pragma unroll
          for (int e = 0; e < EPL; ++e) {
            float a = 0.f;
#pragma unroll
            for (int jj = 0; jj < NR; ++jj) a = absmax_acc(a, S[jj][e]);
            m[e] = fabsf(a);
          }
          float4* dp = reinterpret_cast<float4*>(&s_part[tg][pid][kofs]);
#pragma unroll
          for (int c = 0; c < EPL / 4; ++c) dp[c] = make_float4(m[4 * c], m[4 * c + 1], m[4 * c + 2], m[4 * c + 3]);
        } else {
#pragma unroll
          for (int jj = 0; jj < NR; ++jj) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) a = absmax_acc(a, S[jj][e]);
            s_part[tg][pid][g + RG * jj] = fabsf(a);
          }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < NG * K; i += NW * 32) {
          const int gi = i / K, kk = i % K;
          float a = s_part[gi][0][kk];
#pragma unroll
          for (int pp = 1; pp < NP; ++pp) a = fmaxf(a, s_part[gi][pp][kk]);
          float sn, r;
          h32_scale_of(a, sn, r);
          s_sc[gi][kk] = sn;
          s_rc[gi][kk] = r;
        }
        __syncthreads();
        // codes, and the stored state back (code * scale) where it is used again
        const bool keep = !last || stored_readout;
#pragma unroll
        for (int jj = 0; jj < NR; ++jj) {
#pragma unroll
          for (int w4 = 0; w4 < EPL / 4; ++w4) {
            float r4[4], s4[4];
            if constexpr (VF) {
              const float4 rv = *reinterpret_cast<const float4*>(&s_rc[tg][kofs + 4 * w4]);
              const float4 sv = *reinterpret_cast<const float4*>(&s_sc[tg][kofs + 4 * w4]);
              r4[0] = rv.x; r4[1] = rv.y; r4[2] = rv.z; r4[3] = rv.w;
              s4[0] = sv.x; s4[1] = sv.y; s4[2] = sv.z; s4[3] = sv.w;
            } else {
              const float rj = s_rc[tg][g + RG * jj], sj = s_sc[tg][g + RG * jj];
#pragma unroll
              for (int e = 0; e < 4; ++e) { r4[e] = rj; s4[e] = sj; }
            }
            const float2 y01 = __fmul2_rn(make_float2(S[jj][4 * w4], S[jj][4 * w4 + 1]), make_float2(r4[0], r4[1]));
            const float2 y23 = __fmul2_rn(make_float2(S[jj][4 * w4 + 2], S[jj][4 * w4 + 3]), make_float2(r4[2], r4[3]));
            codes[jj][w4] = float_to_i8x4(y01.x, y01.y, y23.x, y23.y);
            if (keep) {
              float c4[4];
              i8x4_to_float(codes[jj][w4], c4);
#pragma unroll
              for (int e = 0; e < 4; ++e) S[jj][4 * w4 + e] = __fmul_rn(c4[e], s4[e]);
            }
          }
        }
      }
      if constexpr (SDT != ST_F32) {
        if (stored_readout) {
          // o from the stored state: one more reduction of q^.S'
          if constexpr (VF) {
#pragma unroll
            for (int jj = 0; jj < NR; ++jj) {
              float y = 0.f;
#pragma unroll
              for (int e = 0; e < EPL; ++e) {
                const float qh = s_q[tt][kofs + e];
                y = fmaf(qh, S[jj][e], y);
              }
              x[2 * jj] = y;
              x[2 * jj + 1] = 0.f;
            }
            o_mine = ReduceScatterS<NV, LPR / 2, 1>::run(x, lane);
          } else {
            float y[EPL];
#pragma unroll
            for (int c = 0; c < EPL; ++c) y[c] = 0.f;
#pragma unroll
            for (int jj = 0; jj < NR; ++jj) {
              const float qh = s_q[tt][g + RG * jj];
#pragma unroll
              for (int c = 0; c < EPL; ++c) y[c] = fmaf(qh, S[jj][c], y[c]);
            }
#pragma unroll
            for (int c = 0; c < EPL; ++c) {
              x[2 * c] = y[c];
              x[2 * c + 1] = 0.f;
            }
            o_mine = ReduceScatterS<NV, 16, CPL>::run(x, lane);
          }
        }
      }
      if (writer) {
        if constexpr (I8) s_ot[tt][out_col - v0] = o_mine;  // R o; rotated back after the chunk
        else st_out1(p.out, ((int64_t)tok * p.HV + hv) * V + out_col, o_mine, out_bf16);
      }
      if constexpr (IDX == IDX_PAGED) {
        // a page that fills inside a multi-token suffix keeps this state
        if (u.T > 1) {
          const int64_t page = suffix_snapshot_page(p, u, tok - u.tok0);
          if (page >= p.num_slots) {
            if (threadIdx.x == 0) raise_err(p.err, E_PAGE_RANGE);
          } else if (page >= 0) {
            store_tile(page);
          }
        }
      }
    }
    __syncthreads();  // the next chunk's prologue overwrites the token buffers
    if constexpr (I8) {
      // the chunk's outputs back from the rotated basis: one warp per (token, group)
      for (int pr = warp; pr < nt * NG; pr += NW) {
        const int tt = pr / NG, gi = pr % NG;
        const float o = __fmul_rn(fwht_lanes(s_ot[tt][32 * gi + lane], lane), inv_sqrt32());
        st_out1(p.out, ((int64_t)(t0 + tt) * p.HV + hv) * V + v0 + 32 * gi + lane, o, out_bf16);
      }
    }
  }

  // ---- store the state once, after the last token
  store_tile(u.dst);
}

}  // namespace gdn
