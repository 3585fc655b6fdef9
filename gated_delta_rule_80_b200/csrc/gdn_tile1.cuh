// Single-token GDN decode on V_FIRST fp32 and bf16 pools: one short-lived CTA
// per (sequence, value head, V-tile), kept small in registers so that many
// CTAs per SM keep their state loads in flight. The reduce-scatter and the
// 16-byte state vectors below also serve the fp8 and int8 kernels.
//
// The state tile is VT rows of K contiguous elements (one value column of S
// per row), a contiguous block in the pool. A CTA of NW warps issues every
// 16-byte load of its tile at once, right after the (dependent) slot or page
// resolution; the token prologue is computed while the loads are in flight.
//
// Per row (value column v) the step needs a_k = k.S[:, v] and a_q = q.S[:, v]
// summed over the LPR lanes that hold the row. The 2 * NR partial sums of a
// thread go through a reduce-scatter (halving exchanges, then a plain
// butterfly), so each lane ends with one finished sum; k.S and q.S of a row
// meet with one more exchange, the lane computes u and o for that row, and u
// is broadcast back to the lanes that update the row. q and k are used raw
// in the dot products and their norms are applied to the reduced sums:
//     a_k = |k|^-1 (k.S),   a_q = scale |q|^-1 (q.S),   q^.k^ likewise,
// then (single pass, S read once, written once)
//     u = beta (v - alpha a_k),   o = alpha a_q + (q^.k^) u,
//     S' = alpha S + k^ u^T.
#pragma once

#include "gdn_device.cuh"

namespace gdn {

template <int SDT, int K>
struct Tile1Shape {
  // rows per tile: 16 KiB of fp32 state (8 KiB of bf16)
  static constexpr int VT = (K == 256) ? 16 : 32;
  static constexpr int NW = 4;
  // bytes one lane moves per row: a K=256 fp32 row needs 32 to fit a warp
  static constexpr int VB = (SDT == ST_F32 && K == 256) ? 32 : 16;
  static constexpr int MIN_CTAS = 8;  // resident CTAs per SM the registers are sized for
};

// Vector of VB stored bytes: load/store and decode/encode.
template <int SDT, int VB> struct StateVec;
template <int SDT> struct StateVec<SDT, 16> {
  using T = uint4;
  static constexpr int EPL = StateTraits<SDT>::EPL;
  __device__ __forceinline__ static T load(const char* p) { return ld_stream16(p); }
  __device__ __forceinline__ static void store(char* p, T v) { st_stream16(p, v); }
  __device__ __forceinline__ static void decode(T v, float* x) { decode16<SDT>(v, x); }
  __device__ __forceinline__ static T encode(const float* x) { return encode16<SDT>(x); }
  __device__ __forceinline__ static T zero() { return make_uint4(0u, 0u, 0u, 0u); }
};
template <int SDT> struct StateVec<SDT, 32> {
  struct T { uint4 a, b; };
  static constexpr int EPL = 2 * StateTraits<SDT>::EPL;
  __device__ __forceinline__ static T load(const char* p) { return T{ld_stream16(p), ld_stream16(p + 16)}; }
  __device__ __forceinline__ static void store(char* p, T v) {
    st_stream16(p, v.a);
    st_stream16(p + 16, v.b);
  }
  __device__ __forceinline__ static void decode(T v, float* x) {
    decode16<SDT>(v.a, x);
    decode16<SDT>(v.b, x + EPL / 2);
  }
  __device__ __forceinline__ static T encode(const float* x) { return T{encode16<SDT>(x), encode16<SDT>(x + EPL / 2)}; }
  __device__ __forceinline__ static T zero() { return T{make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)}; }
};
template <> struct StateVec<ST_BF16, 8> {
  using T = uint2;
  static constexpr int EPL = 4;
  __device__ __forceinline__ static T load(const char* p) { return __ldcs(reinterpret_cast<const uint2*>(p)); }
  __device__ __forceinline__ static void store(char* p, T v) { __stcs(reinterpret_cast<uint2*>(p), v); }
  __device__ __forceinline__ static void decode(T v, float* x) {
    x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x); x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
  }
  __device__ __forceinline__ static T encode(const float* x) {
    return make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
  }
  __device__ __forceinline__ static T zero() { return make_uint2(0u, 0u); }
};
template <> struct StateVec<ST_FP8, 8> {
  using T = uint2;
  static constexpr int EPL = 8;
  __device__ __forceinline__ static T load(const char* p) { return __ldcs(reinterpret_cast<const uint2*>(p)); }
  __device__ __forceinline__ static void store(char* p, T v) { __stcs(reinterpret_cast<uint2*>(p), v); }
  __device__ __forceinline__ static void decode(T v, float* x) { decode8_fp8(v, x); }
  __device__ __forceinline__ static T encode(const float* x) { return encode8_fp8(x); }
  __device__ __forceinline__ static T zero() { return make_uint2(0u, 0u); }
};

// Reduce-scatter of N values over the lanes of a row group: each halving
// stage (offset O) sends half of the kept values to the partner lane and
// keeps the other half, the upper half where (li & O) != 0; once one value is
// left the remaining stages are a plain butterfly. A lane ends with the full
// group sum of value number li / (LPR / N0).
template <int N, int O>
struct ReduceScatter {
  __device__ __forceinline__ static float run(float* x, int li) {
    if constexpr (N > 1) {
      const bool hi = (li & O) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        const float keep = hi ? x[N / 2 + i] : x[i];
        const float send = hi ? x[i] : x[N / 2 + i];
        x[i] = keep + __shfl_xor_sync(kFull, send, O);
      }
      return ReduceScatter<N / 2, O / 2>::run(x, li);
    } else {
      float v = x[0];
#pragma unroll
      for (int o = O; o >= 1; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
      return v;
    }
  }
};

// fp32 and bf16 states (fp8 pools use step_stream_fp8 in gdn_stream_fp8.cuh).
template <int SDT, int K, int IDX>
__global__ void __launch_bounds__(Tile1Shape<SDT, K>::NW * 32, Tile1Shape<SDT, K>::MIN_CTAS)
step_tile1(const StepParams p) {
  static_assert(SDT == ST_F32 || SDT == ST_BF16, "plain states only");
  using ST = StateTraits<SDT>;
  using TS = Tile1Shape<SDT, K>;
  using SV = StateVec<SDT, TS::VB>;
  constexpr int EPL = SV::EPL;
  constexpr int LPR = K / EPL;  // lanes per stored row
  static_assert(K % EPL == 0 && LPR >= 2 && LPR <= 32 && 32 % LPR == 0, "row must fit a warp");
  constexpr int RPW = 32 / LPR;  // rows per warp instruction
  constexpr int VT = TS::VT;
  constexpr int NW = TS::NW;
  constexpr int NR = VT / (NW * RPW);  // rows per thread
  static_assert(NR >= 1 && NR * NW * RPW == VT, "tile must split evenly");
  constexpr int NV = 2 * NR;           // k.S and q.S partial sums per thread
  static_assert(NV <= LPR, "one finished sum per lane");
  constexpr int REP = LPR / NV;        // lanes that end with the same sum
  constexpr int ROWB = K * ST::BYTES;  // bytes of one stored row

  __shared__ float s_pro[5];           // alpha, beta, q scale, k scale, q^.k^

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int li = lane % LPR;
  const int ri = lane / LPR;
  const int vidx = li / REP;           // the sum this lane finishes
  const int myrow = vidx >> 1;         // ... belongs to this of the thread's rows
  const bool holds_q = (vidx & 1) != 0;
  const int grp = lane - li;
  const bool writer = !holds_q && (li % REP) == 0;
  const int tile = blockIdx.x;
  const int hv = blockIdx.y;
  const int b = blockIdx.z;            // T == 1: the token of sequence b is b
  const int h = hv / p.G;
  const int kofs = li * EPL;
  const bool in_bf16 = (p.flags & F_IN_BF16) != 0;
  const int row0r = warp * NR * RPW + ri;   // tile row of row jj: row0r + jj * RPW

  const Unit u = resolve_unit<IDX>(p, b);
  if (threadIdx.x == 0) raise_err(p.err, u.err);
  if (u.status == U_SKIP) return;
  if (u.status == U_PAD) {
    if (writer)
      st_out1(p.out, ((int64_t)b * p.HV + hv) * p.V + tile * VT + row0r + myrow * RPW, 0.0f,
              (p.flags & F_OUT_BF16) != 0);
    return;
  }

  // all state loads first
  const int64_t head_bytes = (int64_t)K * p.V * ST::BYTES;
  const char* src = reinterpret_cast<const char*>(p.pool) + (u.src * p.HV + hv) * head_bytes +
                    (int64_t)(tile * VT + row0r) * ROWB + kofs * ST::BYTES;
  typename SV::T raw[NR];
#pragma unroll
  for (int jj = 0; jj < NR; ++jj) raw[jj] = SV::load(src + jj * RPW * ROWB);

  // token prologue while the tile is in flight: warp 0 computes the
  // per-token scalars, every lane loads its own q/k/v entries
  float qv[EPL], kv[EPL];
  ld_in_vec<EPL>(p.q, ((int64_t)b * p.H + h) * K + kofs, in_bf16, qv);
  ld_in_vec<EPL>(p.k, ((int64_t)b * p.H + h) * K + kofs, in_bf16, kv);
  const float v_mine = ld_in1(p.v, ((int64_t)b * p.HV + hv) * p.V + tile * VT + row0r + myrow * RPW, in_bf16);
  if (warp == 0) {
    constexpr int KPL = K / 32;
    float qn[KPL], kn[KPL];
    ld_in_vec<KPL>(p.q, ((int64_t)b * p.H + h) * K + lane * KPL, in_bf16, qn);
    ld_in_vec<KPL>(p.k, ((int64_t)b * p.H + h) * K + lane * KPL, in_bf16, kn);
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
    if (lane == 0) {
      float iq = p.scale, ik = 1.0f;
      if (p.flags & F_L2NORM) {
        iq *= rsqrtf(sq + kL2Eps);
        ik = rsqrtf(sk + kL2Eps);
      }
      const float a_in = ld_in1(p.gate, (int64_t)b * p.HV + hv, in_bf16) + p.dt_bias[hv];
      const float b_in = ld_in1(p.beta, (int64_t)b * p.HV + hv, in_bf16);
      s_pro[0] = decay_of(expf(p.A_log[hv]), a_in);
      s_pro[1] = (p.flags & F_BETA_PROB) ? b_in : sigmoid_f(b_in);
      s_pro[2] = iq;
      s_pro[3] = ik;
      s_pro[4] = sqk * iq * ik;
    }
  }
  __syncthreads();
  const float alpha = s_pro[0], beta = s_pro[1], iq = s_pro[2], ik = s_pro[3], qk = s_pro[4];

  // partial k.S and q.S of every row (raw q, k)
  float S[NR][EPL];
  float x[NV];
#pragma unroll
  for (int jj = 0; jj < NR; ++jj) {
    SV::decode(raw[jj], S[jj]);
    float2 ak = make_float2(0.f, 0.f), aq = make_float2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < EPL; e += 2) {
      const float2 s2 = make_float2(S[jj][e], S[jj][e + 1]);
      ak = __ffma2_rn(make_float2(kv[e], kv[e + 1]), s2, ak);
      aq = __ffma2_rn(make_float2(qv[e], qv[e + 1]), s2, aq);
    }
    x[2 * jj] = ak.x + ak.y;
    x[2 * jj + 1] = aq.x + aq.y;
  }
  const float mine = ReduceScatter<NV, LPR / 2>::run(x, li);
  const float other = __shfl_xor_sync(kFull, mine, REP);
  const float dk = (holds_q ? other : mine) * ik;
  const float dq = (holds_q ? mine : other) * iq;
  const float u_mine = beta * (v_mine - alpha * dk);
  float o_mine = fmaf(qk, u_mine, alpha * dq);

  // S' = alpha S + k^ u^T (u of each row from the lane that finished it)
  float kh[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) kh[e] = kv[e] * ik;
  const float2 f2 = make_float2(alpha, alpha);
#pragma unroll
  for (int jj = 0; jj < NR; ++jj) {
    const float uj = __shfl_sync(kFull, u_mine, grp + 2 * jj * REP);
    const float2 u2 = make_float2(uj, uj);
#pragma unroll
    for (int e = 0; e < EPL; e += 2) {
      const float2 y = __ffma2_rn(make_float2(kh[e], kh[e + 1]), u2, __fmul2_rn(f2, make_float2(S[jj][e], S[jj][e + 1])));
      S[jj][e] = y.x;
      S[jj][e + 1] = y.y;
    }
  }

  // storage format and store
  const int row0 = tile * VT + row0r;
  const int64_t out_at = ((int64_t)b * p.HV + hv) * p.V + row0 + myrow * RPW;
  char* dst = reinterpret_cast<char*>(p.pool) + (u.dst * p.HV + hv) * head_bytes + (int64_t)row0 * ROWB +
              kofs * ST::BYTES;
#pragma unroll
  for (int jj = 0; jj < NR; ++jj) {
    if constexpr (SDT == ST_BF16) {
#pragma unroll
      for (int e = 0; e < EPL; ++e) S[jj][e] = round_bf16(S[jj][e]);
    }
    SV::store(dst + jj * RPW * ROWB, SV::encode(S[jj]));
  }
  if constexpr (SDT == ST_BF16) {
    if (p.flags & F_READOUT_STORED) {
      // o from the stored state: q^.S' of every row through the same reduction
#pragma unroll
      for (int jj = 0; jj < NR; ++jj) {
        float y = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) y = fmaf(qv[e], S[jj][e], y);
        x[2 * jj] = y * iq;
        x[2 * jj + 1] = 0.f;
      }
      o_mine = ReduceScatter<NV, LPR / 2>::run(x, li);
    }
  }
  if (writer) st_out1(p.out, out_at, o_mine, (p.flags & F_OUT_BF16) != 0);
}

}  // namespace gdn
