// Single-token GDN decode on V_FIRST fp8 E4M3 pools: a persistent kernel
// that streams its tiles through a ring of shared-memory stages.
//
// Work unit ("tile"): TPU consecutive [K, 64] scale tiles of one (sequence,
// value head), i.e. 64 TPU stored rows of K codes, contiguous in the pool
// (two where the head's V allows, so that the per-unit bookkeeping, the
// copies' barrier and the gate are shared by both; each scale tile keeps its
// own amax barrier). Each CTA takes a
// contiguous range of tiles. Every thread copies its own 16-byte chunks of
// the tile NS - 1 tiles ahead with cp.async (global -> shared, no registers
// held while the copy is in flight), together with a few threads that copy
// the token's q and k rows (when the key head changes), the tile's v slice
// and its scale. A thread therefore always has the next NS - 1 tiles in
// flight while it runs the step of the current one, whose codes it reads
// back from the chunks it copied itself.
//
// The step is that of step_tile1 (same thread mapping and single-pass
// algebra, see gdn_tile1.cuh): per row the two dot products k.S and q.S
// finished by a reduce-scatter over the row's lanes, u and o from them,
// S' = alpha s c + k^ u with c the code values and s the tile scale, the
// tile amax through shared memory, s' = amax / 448 and the new codes.
//
// Per tile the CTA meets twice: once when the tile's copies have landed
// (after which every thread may read what the others copied, and the stage
// of the previous tile is free for the next copy) and once for the amax.
// Thread 0 derives the gate and beta of the next tile, loaded one tile
// ahead, after the second barrier; each warp takes the norms of q and k from
// the rows in shared memory whenever the key head changes.
#pragma once

#include "gdn_pipe.cuh"
#include "gdn_tile1.cuh"

namespace gdn {

template <int K, int TPU = 1>
struct StreamFp8Shape {
  static constexpr int EPL = 16;                 // codes per lane vector (16 bytes)
  static constexpr int VS = 64;                  // rows of one scale tile
  static constexpr int VT = VS * TPU;            // rows per unit: TPU scale tiles of one head
  static constexpr int NW = (K == 256) ? 8 : 4;  // warps
  static constexpr int NT = NW * 32;
  static constexpr int LPR = K / EPL;            // lanes per stored row
  static constexpr int RPW = 32 / LPR;           // rows per warp instruction
  static constexpr int NR = VS / (NW * RPW);     // rows per thread and scale tile
  static constexpr int NS = (TPU == 1) ? 4 : 3;  // stages in the ring
  // one stage: codes | q row | k row | v slice (inputs sized for fp32) |
  // header: first tile scale, gate and beta words, A_log, dt_bias, status,
  // write slot, second tile scale
  static constexpr int CODES = VT * K;
  static constexpr int QK = K * 4;
  static constexpr int VV = VT * 4;
  static constexpr int O_Q = CODES, O_K = CODES + QK, O_V = CODES + 2 * QK, O_HDR = O_V + VV;
  static constexpr int STAGE = O_HDR + 48;
  static constexpr int SMEM = NS * STAGE;        // dynamic shared memory
  static constexpr int MIN_CTAS = (NW == 8) ? 2 : 4;
  static_assert(STAGE % 16 == 0, "16-byte chunks");
};

// FL: the call's input dtype and readout fixed at compile time (bit 0: bf16
// inputs, bit 1: stored readout), so that the unrolled loops carry no test of
// them; -1 reads both from the flags at run time.
template <int K, int IDX, int TPU, int FL = -1>
__global__ void __launch_bounds__(StreamFp8Shape<K, TPU>::NT, StreamFp8Shape<K, TPU>::MIN_CTAS)
step_stream_fp8(const StepParams p, int64_t n_tiles) {
  using PS = StreamFp8Shape<K, TPU>;
  using SV = StateVec<ST_FP8, 16>;
  constexpr int EPL = PS::EPL, LPR = PS::LPR, RPW = PS::RPW, VT = PS::VT, VS = PS::VS;
  constexpr int NW = PS::NW, NR = PS::NR, NS = PS::NS;
  constexpr int NV = 2 * NR;           // k.S and q.S partial sums per thread
  static_assert(LPR >= 2 && LPR <= 32 && NR >= 1 && NR * NW * RPW == VS, "tile split");
  static_assert(NV <= LPR, "one finished sum per lane");
  constexpr int REP = LPR / NV;        // lanes that end with the same sum
  constexpr int ROWB = K;              // bytes of one stored row
  constexpr int TILEB = VT * K;        // bytes of one unit
  constexpr int SUBB = VS * K;         // bytes of one scale tile

  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float s_gate[2][2];       // alpha, beta of a tile, by tile parity
  __shared__ float s_amax[TPU][NW];

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
  const int my_off = row0r * ROWB + kofs;  // this thread's first chunk in a tile
  const bool in_bf16 = FL < 0 ? (p.flags & F_IN_BF16) != 0 : (FL & 1) != 0;
  const bool out_bf16 = (p.flags & F_OUT_BF16) != 0;
  const bool stored_readout = FL < 0 ? (p.flags & F_READOUT_STORED) != 0 : (FL & 2) != 0;
  const int in_b = in_bf16 ? 2 : 4;
  const int NVT = p.V / VT;
  const int64_t per_b = (int64_t)p.HV * NVT;        // units of one sequence
  const int64_t slot_bytes = per_b * TILEB;         // one slot (or page) of the pool
  const int64_t t_begin = n_tiles * blockIdx.x / gridDim.x;
  const int64_t t_end = n_tiles * (blockIdx.x + 1) / gridDim.x;
  const int n_my = static_cast<int>(t_end - t_begin);
  if (n_my <= 0) return;
  // input chunks: q (nq), k (nq), v (nvv), then the scale; at most one per thread
  const int nq = K * in_b / 16;
  const int nvv = VT * in_b / 16;
  const int c_in = threadIdx.x;

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
      *reinterpret_cast<int*>(st + PS::O_HDR + 20) = pc_status;
      *reinterpret_cast<long long*>(st + PS::O_HDR + 24) = pc_dst;
    }
    if (pc_status == U_OK) {
      const char* src = reinterpret_cast<const char*>(p.pool) + pc_src * slot_bytes + (int64_t)pc.within * TILEB + my_off;
#pragma unroll
      for (int sub = 0; sub < TPU; ++sub)
#pragma unroll
        for (int jj = 0; jj < NR; ++jj)
          cp_async16(st + sub * SUBB + my_off + jj * RPW * ROWB, src + sub * SUBB + jj * RPW * ROWB, true);
      const int64_t t = t_begin + i;
      if (c_in < 2 * nq) {
        if (pc_change >= 2) {
          const bool isk = c_in >= nq;
          const int ch = isk ? c_in - nq : c_in;
          const char* base = reinterpret_cast<const char*>(isk ? p.k : p.q) + ((int64_t)pc.b * p.H + pc.h) * K * in_b;
          cp_async16(st + (isk ? PS::O_K : PS::O_Q) + ch * 16, base + ch * 16, true);
        }
      } else if (c_in < 2 * nq + nvv) {
        const int ch = c_in - 2 * nq;
        cp_async16(st + PS::O_V + ch * 16, reinterpret_cast<const char*>(p.v) + t * VT * in_b + ch * 16, true);
      } else if (c_in >= 2 * nq + nvv && c_in < 2 * nq + nvv + TPU) {
        const int sub = c_in - 2 * nq - nvv;
        cp_async4(st + PS::O_HDR + 32 * sub, p.scales + (pc_src * per_b + pc.within) * TPU + sub);
      }
      if (threadIdx.x == 0 && pc_change >= 1) {
        const int64_t gi = (int64_t)pc.b * p.HV + pc.hv;
        cp_async4(st + PS::O_HDR + 4, in_word(p.gate, gi, in_bf16));
        cp_async4(st + PS::O_HDR + 8, in_word(p.beta, gi, in_bf16));
        cp_async4(st + PS::O_HDR + 12, p.A_log + pc.hv);
        cp_async4(st + PS::O_HDR + 16, p.dt_bias + pc.hv);
      }
    }
    cp_async_commit();
    pc_change = pc.next(p.HV, NVT, p.G);
  };

  // ---- consumer side
  StreamCursor cc;
  cc.init(t_begin, p.HV, NVT, p.G);
  int cc_change = 3;
  // thread 0: alpha and beta of tile i from its stage (thread 0 copied the
  // inputs itself, so its own wait suffices)
  auto gate_of = [&](int i, int change) {
    const unsigned char* st = smem + (i % NS) * PS::STAGE;
    const int par = i & 1;
    if (change >= 1) {
      const int64_t gi = (int64_t)cc.b * p.HV + cc.hv;
      const float a = in_from_word(*reinterpret_cast<const uint32_t*>(st + PS::O_HDR + 4), gi, in_bf16);
      const float b = in_from_word(*reinterpret_cast<const uint32_t*>(st + PS::O_HDR + 8), gi, in_bf16);
      const float alog = *reinterpret_cast<const float*>(st + PS::O_HDR + 12);
      const float dtb = *reinterpret_cast<const float*>(st + PS::O_HDR + 16);
      s_gate[par][0] = decay_of(expf(alog), a + dtb);
      s_gate[par][1] = (p.flags & F_BETA_PROB) ? b : sigmoid_f(b);
    } else {
      s_gate[par][0] = s_gate[par ^ 1][0];
      s_gate[par][1] = s_gate[par ^ 1][1];
    }
  };

  // fill the ring with tiles 0 .. NS - 2
#pragma unroll 1
  for (int i = 0; i < NS - 1; ++i) {
    if (i < n_my) issue(i);
    else cp_async_commit();
  }
  if (threadIdx.x == 0) {
    cp_async_wait<NS - 2>();
    gate_of(0, 3);
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
    const int status = *reinterpret_cast<const int*>(st + PS::O_HDR + 20);
    const int64_t dst_slot = *reinterpret_cast<const long long*>(st + PS::O_HDR + 24);
    if (status == U_OK && cc_change >= 2) {
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

#pragma unroll 1
    for (int sub = 0; sub < TPU; ++sub) {
      const int64_t out_row = (t_begin + j) * VT + sub * VS;
      const unsigned char* sst = st + sub * SUBB;  // this scale tile's codes
      float S[NR][EPL];
      float o_mine = 0.f;
      if (status == U_OK) {
        const float alpha = s_gate[j & 1][0], beta = s_gate[j & 1][1];
        const float sc_in = *reinterpret_cast<const float*>(st + PS::O_HDR + 32 * sub);
        const float v_mine = in_bf16
                                 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(st + PS::O_V)[sub * VS + myrow_t])
                                 : reinterpret_cast<const float*>(st + PS::O_V)[sub * VS + myrow_t];

        // partial k.S and q.S of every row on the code values
        float x[NV];
#pragma unroll
        for (int jj = 0; jj < NR; ++jj) {
          const uint4 raw = *reinterpret_cast<const uint4*>(sst + my_off + jj * RPW * ROWB);
          SV::decode(raw, S[jj]);
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
        const float dk = (holds_q ? other : mine) * (ik * sc_in);
        const float dq = (holds_q ? mine : other) * (iq * sc_in);
        const float u_mine = beta * (v_mine - alpha * dk);
        o_mine = fmaf(qk, u_mine, alpha * dq);

        // S' = (alpha s) c + k (|k|^-1 u): the norm rides on u
        const float f = __fmul_rn(alpha, sc_in);
        const float2 f2 = make_float2(f, f);
        const float un = u_mine * ik;
#pragma unroll
        for (int jj = 0; jj < NR; ++jj) {
          const float uj = __shfl_sync(kFull, un, grp + 2 * jj * REP);
          const float2 u2 = make_float2(uj, uj);
#pragma unroll
          for (int e = 0; e < EPL; e += 2) {
            const float2 y =
                __ffma2_rn(make_float2(kv[e], kv[e + 1]), u2, __fmul2_rn(f2, make_float2(S[jj][e], S[jj][e + 1])));
            S[jj][e] = y.x;
            S[jj][e + 1] = y.y;
          }
        }
        // one partial maximum per row (independent chains), then their maximum
        float mj[NR];
#pragma unroll
        for (int jj = 0; jj < NR; ++jj) {
          mj[jj] = 0.f;
#pragma unroll
          for (int e = 0; e < EPL; e += 2) mj[jj] = absmax_acc2(mj[jj], S[jj][e], S[jj][e + 1]);
        }
        float m = mj[0];
#pragma unroll
        for (int jj = 1; jj < NR; ++jj) m = fmaxf(m, mj[jj]);
        m = group_max<32>(m);
        if (lane == 0) s_amax[sub][warp] = m;
      }
      __syncthreads();

      if (status == U_OK) {
        float amax = s_amax[sub][0];
#pragma unroll
        for (int w = 1; w < NW; ++w) amax = fmaxf(amax, s_amax[sub][w]);
        float sn, r;
        fp8_scale_of(amax, sn, r);
        char* dst = reinterpret_cast<char*>(p.pool) + dst_slot * slot_bytes + (int64_t)cc.within * TILEB + sub * SUBB +
                    my_off;
        if (r != 0.0f) {
          const float2 r2 = make_float2(r, r);
#pragma unroll
          for (int jj = 0; jj < NR; ++jj) {
            float y[EPL];
#pragma unroll
            for (int e = 0; e < EPL; e += 2) {
              const float2 tt = __fmul2_rn(make_float2(S[jj][e], S[jj][e + 1]), r2);
              y[e] = tt.x;
              y[e + 1] = tt.y;
            }
            const uint4 c = SV::encode(y);
            SV::store(dst + jj * RPW * ROWB, c);
            if (stored_readout) {
              SV::decode(c, S[jj]);
#pragma unroll
              for (int e = 0; e < EPL; ++e) S[jj][e] = __fmul_rn(S[jj][e], sn);
            }
          }
        } else {
          // a zero tile stores +0 codes (no -0 from negative inputs)
#pragma unroll
          for (int jj = 0; jj < NR; ++jj) {
            SV::store(dst + jj * RPW * ROWB, SV::zero());
#pragma unroll
            for (int e = 0; e < EPL; ++e) S[jj][e] = 0.0f;
          }
        }
        if (threadIdx.x == 0) p.scales[(dst_slot * per_b + cc.within) * TPU + sub] = sn;
        if (stored_readout) {
          // o from the stored state: q^.S' of every row through the same reduction
          float x[NV];
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
        if (writer) st_out1(p.out, out_row + myrow_t, o_mine, out_bf16);
      } else if (status == U_PAD) {
        if (writer) st_out1(p.out, out_row + myrow_t, 0.0f, out_bf16);
      }

    }

    // advance; thread 0 publishes the next tile's gate and beta (the next
    // tile's first barrier makes them visible)
    cc_change = cc.next(p.HV, NVT, p.G);
    if (threadIdx.x == 0 && j + 1 < n_my) {
      cp_async_wait<NS - 2>();
      gate_of(j + 1, cc_change);
    }
  }
  cp_async_wait<0>();
}

}  // namespace gdn
