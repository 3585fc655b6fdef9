// Decode kernels: one CTA per (sequence, value head, V-tile).
//
// Per token the step of the gated delta rule (Circuit.LLM.Mixer, "Delta
// rule" and "Gated memory") is evaluated in a single pass over the state:
// with a_k = k^T S and a_q = q^T S taken from the state BEFORE the decay,
//     GDN:  v_old = alpha a_k,  u = beta (v - v_old),
//           S' = alpha S + k u^T,  o = alpha a_q + (q.k) u
//     KDA:  a_k = (alpha o k)^T S, a_q = (alpha o q)^T S (alpha per key row),
//           S' = diag(alpha) S + k u^T,  o = a_q + (q.k) u
// which equals decay -> read -> write -> read-out from the updated state,
// but reads S once and writes it once. Both reductions are issued before any
// write. The state tile stays in registers for every token of the unit.
//
// Two thread mappings, chosen by the pool layout:
//  * V_FIRST ([V][K], K contiguous): a row of the stored state is one value
//    column S[:, v]; LPR = K / EPL lanes hold one row (EPL elements of 16
//    bytes each), so the K-reductions are shuffles inside that lane group.
//  * K_FIRST ([K][V], V contiguous): lanes run along V in 16-byte vectors and
//    rows of K are spread over lanes and warps; the K-reduction is in-thread
//    sums, shuffles across the lanes of a column group, and one pass through
//    shared memory across warps.
#pragma once

#include "gdn_device.cuh"

namespace gdn {

// Tile shape of a state format: V-tile width VT (for fp8 the scale tile,
// block_v = 64) and warps per CTA.
template <int SDT>
struct TileShape {
  static constexpr int VT = (SDT == ST_FP8) ? 64 : 32;
  static constexpr int NW = 4;
};

template <int N>
__device__ __forceinline__ void st_out_vec(void* base, int64_t i, const float* x, bool bf16) {
  if (bf16) {
    __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(base) + i;
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int c = 0; c < N / 8; ++c) {
        uint4 w;
        w.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
        w.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
        w.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
        w.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
        reinterpret_cast<uint4*>(p)[c] = w;
      }
    } else if constexpr (N == 4) {
      uint2 w;
      w.x = pack_bf16x2(x[0], x[1]);
      w.y = pack_bf16x2(x[2], x[3]);
      *reinterpret_cast<uint2*>(p) = w;
    } else {
#pragma unroll
      for (int j = 0; j < N; ++j) p[j] = __float2bfloat16_rn(x[j]);
    }
  } else {
    float* p = reinterpret_cast<float*>(base) + i;
    if constexpr (N % 4 == 0) {
#pragma unroll
      for (int c = 0; c < N / 4; ++c)
        reinterpret_cast<float4*>(p)[c] = make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < N; ++j) p[j] = x[j];
    }
  }
}

// ===========================================================================
// V_FIRST
// ===========================================================================
template <int SDT, int K, int GATE, int IDX>
__global__ void __launch_bounds__(TileShape<SDT>::NW * 32)
step_vfirst(const StepParams p) {
  using ST = StateTraits<SDT>;
  constexpr int EPL = ST::EPL;
  constexpr int LPR = K / EPL;  // lanes per stored row
  static_assert(K % EPL == 0 && LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "row must fit a warp");
  constexpr int RPW = 32 / LPR;  // rows per warp instruction
  constexpr int VT = TileShape<SDT>::VT;
  constexpr int NW = TileShape<SDT>::NW;
  constexpr int NR = VT / (NW * RPW);  // rows per thread
  static_assert(NR >= 1 && NR * NW * RPW == VT, "tile must split evenly");

  __shared__ float s_amax[2][NW];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int li = lane % LPR;
  const int ri = lane / LPR;
  int unit = blockIdx.x;
  const int tile = unit % p.n_vtiles;
  unit /= p.n_vtiles;
  const int hv = unit % p.HV;
  const int b = unit / p.HV;
  const int h = hv / (p.HV / p.H);
  const int kofs = li * EPL;
  const bool in_bf16 = (p.flags & F_IN_BF16) != 0;
  const bool out_bf16 = (p.flags & F_OUT_BF16) != 0;
  const int64_t V = p.V;

  int rows[NR];
#pragma unroll
  for (int j = 0; j < NR; ++j) rows[j] = tile * VT + (warp * NR + j) * RPW + ri;

  const Unit u = resolve_unit<IDX>(p, b);
  if (threadIdx.x == 0) raise_err(p.err, u.err);
  if (u.status == U_SKIP || u.tok1 <= u.tok0) return;
  if (u.status == U_PAD) {
    if (li == 0)
      for (int tok = u.tok0; tok < u.tok1; ++tok)
#pragma unroll
        for (int j = 0; j < NR; ++j) st_out1(p.out, ((int64_t)tok * p.HV + hv) * V + rows[j], 0.0f, out_bf16);
    return;
  }

  const int64_t head_elems = (int64_t)K * V;
  const char* src = reinterpret_cast<const char*>(p.pool) + (u.src * p.HV + hv) * head_elems * ST::BYTES;
  float S[NR][EPL];
#pragma unroll
  for (int j = 0; j < NR; ++j)
    decode16<SDT>(ld_stream16(src + ((int64_t)rows[j] * K + kofs) * ST::BYTES), S[j]);
  const int n_scale = p.V / VT;
  if constexpr (SDT == ST_FP8) {
    const float sc = p.scales[(u.src * p.HV + hv) * n_scale + tile];
#pragma unroll
    for (int j = 0; j < NR; ++j)
#pragma unroll
      for (int e = 0; e < EPL; ++e) S[j][e] = __fmul_rn(S[j][e], sc);
  }

  const float expA = expf(p.A_log[hv]);
  [[maybe_unused]] uint4 codes[NR];
  [[maybe_unused]] float s_last = 0.0f;

  for (int tok = u.tok0; tok < u.tok1; ++tok) {
    const bool last = (tok + 1 == u.tok1);
    float qv[EPL], kv[EPL];
    ld_in_vec<EPL>(p.q, ((int64_t)tok * p.H + h) * K + kofs, in_bf16, qv);
    ld_in_vec<EPL>(p.k, ((int64_t)tok * p.H + h) * K + kofs, in_bf16, kv);
    float vv[NR];
#pragma unroll
    for (int j = 0; j < NR; ++j) vv[j] = ld_in1(p.v, ((int64_t)tok * p.HV + hv) * V + rows[j], in_bf16);
    const float braw = ld_in1(p.beta, (int64_t)tok * p.HV + hv, in_bf16);

    // q/k norms and q.k over the K elements of one row group
    float sq = 0.f, sk = 0.f, sqk = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      sq = fmaf(qv[e], qv[e], sq);
      sk = fmaf(kv[e], kv[e], sk);
      sqk = fmaf(qv[e], kv[e], sqk);
    }
    sqk = group_sum<LPR>(sqk);
    float iq = p.scale, ik = 1.0f;
    if (p.flags & F_L2NORM) {
      sq = group_sum<LPR>(sq);
      sk = group_sum<LPR>(sk);
      iq *= rsqrtf(sq + kL2Eps);
      ik = rsqrtf(sk + kL2Eps);
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) { qv[e] *= iq; kv[e] *= ik; }
    const float qk = sqk * iq * ik;
    const float beta = (p.flags & F_BETA_PROB) ? braw : sigmoid_f(braw);

    // gate; for KDA fold alpha into the reduction weights
    [[maybe_unused]] float alpha = 1.0f;
    [[maybe_unused]] float al[EPL];
    float wk[EPL], wq[EPL];
    if constexpr (GATE == GATE_SCALAR) {
      alpha = decay_of(expA, ld_in1(p.gate, (int64_t)tok * p.HV + hv, in_bf16) + p.dt_bias[hv]);
#pragma unroll
      for (int e = 0; e < EPL; ++e) { wk[e] = kv[e]; wq[e] = qv[e]; }
    } else {
      float g[EPL], db[EPL];
      ld_in_vec<EPL>(p.gate, ((int64_t)tok * p.HV + hv) * K + kofs, in_bf16, g);
      ld_in_vec<EPL>(p.dt_bias, (int64_t)hv * K + kofs, false, db);
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        al[e] = decay_of(expA, g[e] + db[e]);
        wk[e] = al[e] * kv[e];
        wq[e] = al[e] * qv[e];
      }
    }

    // a_k, a_q per row: in-thread partial sums, then the row's lane group
    float dk[NR], dq[NR];
#pragma unroll
    for (int j = 0; j < NR; ++j) {
      float x = 0.f, y = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) { x = fmaf(wk[e], S[j][e], x); y = fmaf(wq[e], S[j][e], y); }
      dk[j] = x;
      dq[j] = y;
    }
#pragma unroll
    for (int j = 0; j < NR; ++j) { dk[j] = group_sum<LPR>(dk[j]); dq[j] = group_sum<LPR>(dq[j]); }

    float uu[NR], oo[NR];
#pragma unroll
    for (int j = 0; j < NR; ++j) {
      if constexpr (GATE == GATE_SCALAR) {
        uu[j] = beta * (vv[j] - alpha * dk[j]);
        oo[j] = fmaf(qk, uu[j], alpha * dq[j]);
      } else {
        uu[j] = beta * (vv[j] - dk[j]);
        oo[j] = fmaf(qk, uu[j], dq[j]);
      }
    }
    // S' = diag(alpha) S + k u^T
#pragma unroll
    for (int j = 0; j < NR; ++j)
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        if constexpr (GATE == GATE_SCALAR) S[j][e] = fmaf(kv[e], uu[j], alpha * S[j][e]);
        else S[j][e] = fmaf(kv[e], uu[j], al[e] * S[j][e]);
      }

    // the state's storage format after every token (a write event)
    const bool stored_readout = (p.flags & F_READOUT_STORED) != 0;
    if constexpr (SDT == ST_BF16) {
#pragma unroll
      for (int j = 0; j < NR; ++j)
#pragma unroll
        for (int e = 0; e < EPL; ++e) S[j][e] = round_bf16(S[j][e]);
    } else if constexpr (SDT == ST_FP8) {
      float m = 0.f;
#pragma unroll
      for (int j = 0; j < NR; ++j)
#pragma unroll
        for (int e = 0; e < EPL; ++e) m = absmax_acc(m, S[j][e]);
      m = group_max<32>(fabsf(m));
      const int buf = (tok - u.tok0) & 1;
      if (lane == 0) s_amax[buf][warp] = m;
      __syncthreads();
      float amax = s_amax[buf][0];
#pragma unroll
      for (int w = 1; w < NW; ++w) amax = fmaxf(amax, s_amax[buf][w]);
      float s, r;
      fp8_scale_of(amax, s, r);
      s_last = s;
#pragma unroll
      for (int j = 0; j < NR; ++j) {
        float y[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) y[e] = fp8_prescale(S[j][e], r);
        codes[j] = encode16<SDT>(y);
      }
      if (!last || stored_readout) {
#pragma unroll
        for (int j = 0; j < NR; ++j) {
          decode16<SDT>(codes[j], S[j]);
#pragma unroll
          for (int e = 0; e < EPL; ++e) S[j][e] = __fmul_rn(S[j][e], s);
        }
      }
    }
    if constexpr (SDT != ST_F32) {
      if (stored_readout) {
#pragma unroll
        for (int j = 0; j < NR; ++j) {
          float y = 0.f;
#pragma unroll
          for (int e = 0; e < EPL; ++e) y = fmaf(qv[e], S[j][e], y);
          oo[j] = group_sum<LPR>(y);
        }
      }
    }
    if (li == 0) {
#pragma unroll
      for (int j = 0; j < NR; ++j) st_out1(p.out, ((int64_t)tok * p.HV + hv) * V + rows[j], oo[j], out_bf16);
    }
  }

  char* dst = reinterpret_cast<char*>(p.pool) + (u.dst * p.HV + hv) * head_elems * ST::BYTES;
#pragma unroll
  for (int j = 0; j < NR; ++j) {
    void* a = dst + ((int64_t)rows[j] * K + kofs) * ST::BYTES;
    if constexpr (SDT == ST_FP8) st_stream16(a, codes[j]);
    else st_stream16(a, encode16<SDT>(S[j]));
  }
  if constexpr (SDT == ST_FP8) {
    if (threadIdx.x == 0) p.scales[(u.dst * p.HV + hv) * n_scale + tile] = s_last;
  }
}

// ===========================================================================
// K_FIRST
// ===========================================================================
template <int SDT, int K, int GATE, int IDX>
__global__ void __launch_bounds__(TileShape<SDT>::NW * 32)
step_kfirst(const StepParams p) {
  using ST = StateTraits<SDT>;
  constexpr int EPL = ST::EPL;
  constexpr int VT = TileShape<SDT>::VT;
  constexpr int NW = TileShape<SDT>::NW;
  constexpr int CPR = VT / EPL;  // lanes per row segment
  static_assert(CPR >= 1 && CPR <= 32 && 32 % CPR == 0, "row segment must fit a warp");
  constexpr int RPI = 32 / CPR;  // rows per warp instruction
  constexpr int RPC = NW * RPI;  // rows per CTA pass
  static_assert(K % RPC == 0, "K must split over the CTA");
  constexpr int KR = K / RPC;    // rows per thread
  constexpr int KPL = K / 32;    // elements per lane for the norms
  static_assert(K % 32 == 0, "K must be a multiple of 32");

  __shared__ float s_red[2][NW][2][VT];
  __shared__ float s_amax[2][NW];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int c = lane % CPR;
  const int rr = lane / CPR;
  int unit = blockIdx.x;
  const int tile = unit % p.n_vtiles;
  unit /= p.n_vtiles;
  const int hv = unit % p.HV;
  const int b = unit / p.HV;
  const int h = hv / (p.HV / p.H);
  const bool in_bf16 = (p.flags & F_IN_BF16) != 0;
  const bool out_bf16 = (p.flags & F_OUT_BF16) != 0;
  const int64_t V = p.V;
  const int col0 = tile * VT + c * EPL;
  const bool writer = (warp == 0) && (rr == 0);

  int krow[KR];
#pragma unroll
  for (int j = 0; j < KR; ++j) krow[j] = j * RPC + warp * RPI + rr;

  const Unit u = resolve_unit<IDX>(p, b);
  if (threadIdx.x == 0) raise_err(p.err, u.err);
  if (u.status == U_SKIP || u.tok1 <= u.tok0) return;
  if (u.status == U_PAD) {
    if (writer) {
      float z[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) z[e] = 0.0f;
      for (int tok = u.tok0; tok < u.tok1; ++tok)
        st_out_vec<EPL>(p.out, ((int64_t)tok * p.HV + hv) * V + col0, z, out_bf16);
    }
    return;
  }

  const int64_t head_elems = (int64_t)K * V;
  const char* src = reinterpret_cast<const char*>(p.pool) + (u.src * p.HV + hv) * head_elems * ST::BYTES;
  float S[KR][EPL];
#pragma unroll
  for (int j = 0; j < KR; ++j)
    decode16<SDT>(ld_stream16(src + ((int64_t)krow[j] * V + col0) * ST::BYTES), S[j]);
  const int n_scale = p.V / VT;
  if constexpr (SDT == ST_FP8) {
    const float sc = p.scales[(u.src * p.HV + hv) * n_scale + tile];
#pragma unroll
    for (int j = 0; j < KR; ++j)
#pragma unroll
      for (int e = 0; e < EPL; ++e) S[j][e] = __fmul_rn(S[j][e], sc);
  }

  const float expA = expf(p.A_log[hv]);
  [[maybe_unused]] uint4 codes[KR];
  [[maybe_unused]] float s_last = 0.0f;
  const bool stored_readout = (p.flags & F_READOUT_STORED) != 0;

  for (int tok = u.tok0; tok < u.tok1; ++tok) {
    const bool last = (tok + 1 == u.tok1);
    const int buf = (tok - u.tok0) & 1;
    const int64_t qk_base = ((int64_t)tok * p.H + h) * K;
    // warp-wide q/k norms and q.k
    float qn[KPL], kn[KPL];
    ld_in_vec<KPL>(p.q, qk_base + lane * KPL, in_bf16, qn);
    ld_in_vec<KPL>(p.k, qk_base + lane * KPL, in_bf16, kn);
    float sq = 0.f, sk = 0.f, sqk = 0.f;
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      sq = fmaf(qn[e], qn[e], sq);
      sk = fmaf(kn[e], kn[e], sk);
      sqk = fmaf(qn[e], kn[e], sqk);
    }
    sqk = group_sum<32>(sqk);
    float iq = p.scale, ik = 1.0f;
    if (p.flags & F_L2NORM) {
      sq = group_sum<32>(sq);
      sk = group_sum<32>(sk);
      iq *= rsqrtf(sq + kL2Eps);
      ik = rsqrtf(sk + kL2Eps);
    }
    const float qk = sqk * iq * ik;
    float kr[KR], qr[KR];
#pragma unroll
    for (int j = 0; j < KR; ++j) {
      kr[j] = ld_in1(p.k, qk_base + krow[j], in_bf16) * ik;
      qr[j] = ld_in1(p.q, qk_base + krow[j], in_bf16) * iq;
    }
    float vv[EPL];
    ld_in_vec<EPL>(p.v, ((int64_t)tok * p.HV + hv) * V + col0, in_bf16, vv);
    const float braw = ld_in1(p.beta, (int64_t)tok * p.HV + hv, in_bf16);
    const float beta = (p.flags & F_BETA_PROB) ? braw : sigmoid_f(braw);

    [[maybe_unused]] float alpha = 1.0f;
    [[maybe_unused]] float al[KR];
    float wk[KR], wq[KR];
    if constexpr (GATE == GATE_SCALAR) {
      alpha = decay_of(expA, ld_in1(p.gate, (int64_t)tok * p.HV + hv, in_bf16) + p.dt_bias[hv]);
#pragma unroll
      for (int j = 0; j < KR; ++j) { wk[j] = kr[j]; wq[j] = qr[j]; }
    } else {
#pragma unroll
      for (int j = 0; j < KR; ++j) {
        const float g = ld_in1(p.gate, ((int64_t)tok * p.HV + hv) * K + krow[j], in_bf16);
        al[j] = decay_of(expA, g + p.dt_bias[(int64_t)hv * K + krow[j]]);
        wk[j] = al[j] * kr[j];
        wq[j] = al[j] * qr[j];
      }
    }

    float dk[EPL], dq[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) { dk[e] = 0.f; dq[e] = 0.f; }
#pragma unroll
    for (int j = 0; j < KR; ++j)
#pragma unroll
      for (int e = 0; e < EPL; ++e) { dk[e] = fmaf(wk[j], S[j][e], dk[e]); dq[e] = fmaf(wq[j], S[j][e], dq[e]); }
#pragma unroll
    for (int o = CPR; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        dk[e] += __shfl_xor_sync(kFull, dk[e], o);
        dq[e] += __shfl_xor_sync(kFull, dq[e], o);
      }
    if (rr == 0) {
#pragma unroll
      for (int e = 0; e < EPL; ++e) { s_red[buf][warp][0][c * EPL + e] = dk[e]; s_red[buf][warp][1][c * EPL + e] = dq[e]; }
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      float x = 0.f, y = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) { x += s_red[buf][w][0][c * EPL + e]; y += s_red[buf][w][1][c * EPL + e]; }
      dk[e] = x;
      dq[e] = y;
    }

    float uu[EPL], oo[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      if constexpr (GATE == GATE_SCALAR) {
        uu[e] = beta * (vv[e] - alpha * dk[e]);
        oo[e] = fmaf(qk, uu[e], alpha * dq[e]);
      } else {
        uu[e] = beta * (vv[e] - dk[e]);
        oo[e] = fmaf(qk, uu[e], dq[e]);
      }
    }
#pragma unroll
    for (int j = 0; j < KR; ++j)
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        if constexpr (GATE == GATE_SCALAR) S[j][e] = fmaf(kr[j], uu[e], alpha * S[j][e]);
        else S[j][e] = fmaf(kr[j], uu[e], al[j] * S[j][e]);
      }

    if constexpr (SDT == ST_BF16) {
#pragma unroll
      for (int j = 0; j < KR; ++j)
#pragma unroll
        for (int e = 0; e < EPL; ++e) S[j][e] = round_bf16(S[j][e]);
    } else if constexpr (SDT == ST_FP8) {
      float m = 0.f;
#pragma unroll
      for (int j = 0; j < KR; ++j)
#pragma unroll
        for (int e = 0; e < EPL; ++e) m = absmax_acc(m, S[j][e]);
      m = group_max<32>(fabsf(m));
      if (lane == 0) s_amax[buf][warp] = m;
      __syncthreads();
      float amax = s_amax[buf][0];
#pragma unroll
      for (int w = 1; w < NW; ++w) amax = fmaxf(amax, s_amax[buf][w]);
      float s, r;
      fp8_scale_of(amax, s, r);
      s_last = s;
#pragma unroll
      for (int j = 0; j < KR; ++j) {
        float y[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) y[e] = fp8_prescale(S[j][e], r);
        codes[j] = encode16<SDT>(y);
      }
      if (!last || stored_readout) {
#pragma unroll
        for (int j = 0; j < KR; ++j) {
          decode16<SDT>(codes[j], S[j]);
#pragma unroll
          for (int e = 0; e < EPL; ++e) S[j][e] = __fmul_rn(S[j][e], s);
        }
      }
    }
    if constexpr (SDT != ST_F32) {
      if (stored_readout) {
        // o = q^T S from the stored state: one more K-reduction
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          float y = 0.f;
#pragma unroll
          for (int j = 0; j < KR; ++j) y = fmaf(qr[j], S[j][e], y);
          oo[e] = y;
        }
#pragma unroll
        for (int o = CPR; o < 32; o <<= 1)
#pragma unroll
          for (int e = 0; e < EPL; ++e) oo[e] += __shfl_xor_sync(kFull, oo[e], o);
        __syncthreads();  // every thread is done reading s_red[buf]
        if (rr == 0) {
#pragma unroll
          for (int e = 0; e < EPL; ++e) s_red[buf][warp][1][c * EPL + e] = oo[e];
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          float y = 0.f;
#pragma unroll
          for (int w = 0; w < NW; ++w) y += s_red[buf][w][1][c * EPL + e];
          oo[e] = y;
        }
      }
    }
    if (writer) st_out_vec<EPL>(p.out, ((int64_t)tok * p.HV + hv) * V + col0, oo, out_bf16);
  }

  char* dst = reinterpret_cast<char*>(p.pool) + (u.dst * p.HV + hv) * head_elems * ST::BYTES;
#pragma unroll
  for (int j = 0; j < KR; ++j) {
    void* a = dst + ((int64_t)krow[j] * V + col0) * ST::BYTES;
    if constexpr (SDT == ST_FP8) st_stream16(a, codes[j]);
    else st_stream16(a, encode16<SDT>(S[j]));
  }
  if constexpr (SDT == ST_FP8) {
    if (threadIdx.x == 0) p.scales[(u.dst * p.HV + hv) * n_scale + tile] = s_last;
  }
}

}  // namespace gdn
