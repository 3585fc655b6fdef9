// Single-token GDN decode on V_FIRST int8_hadamard32 pools with K = 128: one
// warp per scale group, every warp on its own.
//
// Work unit: one 32-value scale group of one (sequence, value head), i.e. 32
// stored rows of 128 int8 codes (4 KiB, contiguous in the pool) and the
// group's 128 scales (one per key channel, contiguous in the [V/32, K] scale
// array). A CTA is one warp; it takes a contiguous range of groups and
// streams them through its own ring of shared-memory stages with per-lane
// cp.async copies, NS - 1 groups ahead. Nothing is shared between warps, so
// the kernel has no CTA barrier: the warp meets only itself (__syncwarp).
//
// Lane l = 8 rb + cc holds rows 8 rb .. 8 rb + 7 of the group and key
// channels 16 cc .. 16 cc + 15 of each (128 state values):
//   - the amax of a key channel runs over the group's 32 rows, i.e. over the
//     lane's own 8 rows and the 4 lanes of the same cc (through a 2.5 KiB
//     buffer in the consumed stage);
//   - the dot products k.S and q.S of a row run over the 8 lanes of the same
//     rb; their reduce-scatter leaves row l's pair on lane l, which is where
//     the 32-lane rotation of v and of the output wants it.
//
// Arithmetic, in the rotated basis in which the pool keeps the state (with
// R = H32 / sqrt(32) on the 32 values of a group, R R = I, the step
// commutes with R; see gdn_stream_i8.cuh):
//   pass 1:  a_k = (k s) . c,  a_q = (q s) . c      (c the code values, s the
//            group's scales of the lane's channels)
//   row l:   u = beta (R v - alpha |k|^-1 a_k),  R o = alpha iq a_q + (q^.k^) u
//   pass 2:  S' = (alpha s) c + k (|k|^-1 u)        (codes decoded again from
//            the stage, S' held in registers)
//   scales:  amax per key channel, s' = amax / 127, r' = 1 / s' (correctly
//            rounded), codes rint(S' r')
//   o = R (R o) by one 32-lane butterfly.
#pragma once

#include "gdn_pipe.cuh"
#include "gdn_tile1.cuh"

namespace gdn {

struct GroupI8Shape {
  static constexpr int K = 128;
  static constexpr int VT = 32;                  // rows per unit: one scale group
  static constexpr int EPL = 16;                 // codes per lane vector (16 bytes)
  static constexpr int LPR = K / EPL;            // lanes per stored row (8)
  static constexpr int RB = 32 / LPR;            // row blocks (4)
  static constexpr int NR = VT / RB;             // rows per lane (8)
  static constexpr int NT = 32;                  // one warp
  static constexpr int NS = 3;                   // stages in the ring
  // one stage: codes | K scales | q row | k row | v slice (inputs sized for
  // fp32) | header: gate and beta words, A_log, dt_bias, status, unit index
  // within the slot, write slot, change level, gate-index parity.
  // Per-channel vectors that every lane reads in its 16-channel block (the
  // scales, k, and later r' and s') are padded by 16 bytes per block, so that
  // the 8 blocks of a row fall in distinct banks: block b starts at
  // b (16 w + 16) for elements of w bytes (pad16_ofs).
  static constexpr int CODES = VT * K;
  static constexpr int PADV = K * 4 + (K / EPL) * 16;   // a padded vector of fp32
  static constexpr int O_SC = CODES, O_Q = O_SC + PADV, O_K = O_Q + K * 4, O_V = O_K + PADV;
  static constexpr int O_HDR = O_V + VT * 4;
  static constexpr int STAGE = O_HDR + 48;
  static constexpr int SMEM = NS * STAGE;        // dynamic shared memory
  // after pass 2 the stage's code area holds the partial maxima [RB][K], the
  // new r' and (for a stored readout) the new s', all padded
  static constexpr int O_MX = 0, O_R = RB * PADV, O_S = O_R + PADV;
  static constexpr int MIN_CTAS = 12;
  static_assert(STAGE % 16 == 0 && O_S + PADV <= CODES, "stage layout");
  static_assert(MIN_CTAS * (SMEM + 1024) <= 233472, "the ring of 12 warps fits one SM's shared memory");
  static_assert(NR == LPR, "the reduce-scatter of 2 NR sums over LPR lanes leaves one row's pair per lane");
};

// Reduce-scatter of 2 N sums (the k and q partial dots of N rows, row r at
// x[2r], x[2r + 1]) over N lanes (offsets O = N/2 .. 1): each stage keeps the
// half whose row index bit matches the lane's, so lane cc ends with row cc.
template <int N, int O>
__device__ __forceinline__ float2 rs_row_pairs(float* x, int cc) {
  if constexpr (N == 1) {
    return make_float2(x[0], x[1]);
  } else {
    const bool hi = (cc & O) != 0;
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const float keep = hi ? x[N + i] : x[i];
      const float send = hi ? x[i] : x[N + i];
      x[i] = keep + __shfl_xor_sync(kFull, send, O);
    }
    return rs_row_pairs<N / 2, O / 2>(x, cc);
  }
}

// Byte offset of 16-byte chunk c of a vector stored with a 16-byte pad after
// every `cpb` chunks (one lane block of 16 channels).
__device__ __forceinline__ int pad16_ofs(int c, int cpb) { return 16 * c + 16 * (c / cpb); }

// 16 int8 codes (16 bytes) -> their values as floats
__device__ __forceinline__ void decode_i8x16(uint4 raw, float* c) {
  i8x4_to_float(raw.x, c);
  i8x4_to_float(raw.y, c + 4);
  i8x4_to_float(raw.z, c + 8);
  i8x4_to_float(raw.w, c + 12);
}
// 16 floats from shared memory (16-byte aligned)
__device__ __forceinline__ void ld_vec16_f32(const unsigned char* p, float* x) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4) {
    const float4 f = q[c4];
    x[4 * c4] = f.x; x[4 * c4 + 1] = f.y; x[4 * c4 + 2] = f.z; x[4 * c4 + 3] = f.w;
  }
}
// input elements i, i + 1 (i even) widened to fp32
__device__ __forceinline__ float2 ld_in_pair(const unsigned char* base, int i, bool bf16) {
  if (bf16) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(base + 2 * i);
    return make_float2(bf16_lo(w), bf16_hi(w));
  }
  return *reinterpret_cast<const float2*>(base + 4 * i);
}

// IN_BF16: bf16 token inputs (else fp32); STORED: the output is read from the
// stored state (else from the working state). Both are fixed per call, so
// they are template parameters and the unrolled loops carry no test of them.
template <int IDX, bool IN_BF16, bool STORED>
__global__ void __launch_bounds__(GroupI8Shape::NT, GroupI8Shape::MIN_CTAS)
step_group_i8(const StepParams p, int64_t n_units) {
  using PS = GroupI8Shape;
  constexpr int K = PS::K, EPL = PS::EPL, NR = PS::NR, NS = PS::NS, VT = PS::VT;
  constexpr int ROWB = K;              // bytes of one stored row
  constexpr int UNITB = VT * K;        // bytes of one group

  extern __shared__ __align__(128) unsigned char smem[];

  const int lane = threadIdx.x;
  const int cc = lane & (PS::LPR - 1);
  const int rb = lane / PS::LPR;
  const int row0 = rb * NR;            // the lane's first row; its rows are row0 .. row0 + NR - 1
  const int my_off = row0 * ROWB + cc * EPL;
  constexpr bool in_bf16 = IN_BF16;
  const bool out_bf16 = (p.flags & F_OUT_BF16) != 0;
  constexpr bool stored_readout = STORED;
  constexpr int in_b = in_bf16 ? 2 : 4;
  const int NVG = p.V / VT;
  const int64_t per_b = (int64_t)p.HV * NVG;        // groups of one sequence
  const int64_t slot_bytes = per_b * UNITB;         // one slot (or page) of the pool
  const int64_t u_begin = n_units * blockIdx.x / gridDim.x;
  const int64_t u_end = n_units * (blockIdx.x + 1) / gridDim.x;
  const int n_my = static_cast<int>(u_end - u_begin);
  if (n_my <= 0) return;
  const int nqk = K * in_b / 16;       // 16-byte chunks of a q (or k) row
  const int kblk = 16 * in_b + 16;     // a lane block of the padded k row (bytes)
  constexpr int FBLK = EPL * 4 + 16;   // ... of a padded fp32 vector
  const int nvv = VT * in_b / 16;      // ... of the v slice

  // ---- producer side: copies of unit u_begin + i into stage i % NS
  StreamCursor pc;
  pc.init(u_begin, p.HV, NVG, p.G);
  int pc_change = 3;                   // relative to the previous unit
  int64_t pc_src = 0, pc_dst = 0;
  int pc_status = U_SKIP;
  auto issue = [&](int i) {
    unsigned char* st = smem + (i % NS) * PS::STAGE;
    if (pc_change == 3) {
      const Unit u = resolve_unit<IDX>(p, pc.b);
      if (lane == 0) raise_err(p.err, u.err);
      pc_src = u.src;
      pc_dst = u.dst;
      pc_status = u.status;
    }
    if (lane == 0) {
      int* hdr = reinterpret_cast<int*>(st + PS::O_HDR);
      hdr[4] = pc_status;
      hdr[5] = pc.within;
      *reinterpret_cast<long long*>(hdr + 6) = pc_dst;
      hdr[8] = pc_change;
      hdr[9] = (pc.b * p.HV + pc.hv) & 1;
    }
    if (pc_status == U_OK) {
      const char* src = reinterpret_cast<const char*>(p.pool) + pc_src * slot_bytes + (int64_t)pc.within * UNITB + my_off;
#pragma unroll
      for (int r = 0; r < NR; ++r) cp_async16(st + my_off + r * ROWB, src + r * ROWB, true);
      const char* scb = reinterpret_cast<const char*>(p.scales + (pc_src * per_b + pc.within) * K);
      cp_async16(st + PS::O_SC + pad16_ofs(lane, 4), scb + lane * 16, true);
      const int64_t qk_row = ((int64_t)pc.b * p.H + pc.h) * K * in_b;
      for (int c = lane; c < 2 * nqk; c += 32) {
        const bool isk = c >= nqk;
        const int ch = c - (isk ? nqk : 0);
        cp_async16(st + (isk ? PS::O_K + pad16_ofs(ch, in_b) : PS::O_Q + ch * 16),
                   reinterpret_cast<const char*>(isk ? p.k : p.q) + qk_row + ch * 16, true);
      }
      if (lane < nvv)
        cp_async16(st + PS::O_V + lane * 16,
                   reinterpret_cast<const char*>(p.v) + (u_begin + i) * VT * in_b + lane * 16, true);
      if (lane == 0 && pc_change >= 1) {
        const int64_t gi = (int64_t)pc.b * p.HV + pc.hv;
        cp_async4(st + PS::O_HDR, in_word(p.gate, gi, in_bf16));
        cp_async4(st + PS::O_HDR + 4, in_word(p.beta, gi, in_bf16));
        cp_async4(st + PS::O_HDR + 8, p.A_log + pc.hv);
        cp_async4(st + PS::O_HDR + 12, p.dt_bias + pc.hv);
      }
    }
    cp_async_commit();
    pc_change = pc.next(p.HV, NVG, p.G);
  };

#pragma unroll 1
  for (int i = 0; i < NS - 1; ++i) {
    if (i < n_my) issue(i);
    else cp_async_commit();
  }

  float alpha = 0.f, beta = 0.f;       // gate of the current value head
  float iq = 0.f, ik = 0.f, qk = 0.f;  // norms of the current key head

#pragma unroll 1
  for (int j = 0; j < n_my; ++j) {
    // every lane is done with the stage the next copies go to
    __syncwarp();
    if (j + NS - 1 < n_my) issue(j + NS - 1);
    else cp_async_commit();
    cp_async_wait<NS - 1>();
    __syncwarp();

    unsigned char* st = smem + (j % NS) * PS::STAGE;
    const int* hdr = reinterpret_cast<const int*>(st + PS::O_HDR);
    const int status = hdr[4];
    const int within = hdr[5];
    const int64_t dst_slot = *reinterpret_cast<const long long*>(hdr + 6);
    const int change = hdr[8];
    const int64_t out_row = (u_begin + j) * VT;
    if (status == U_PAD) {
      st_out1(p.out, out_row + lane, 0.0f, out_bf16);
      continue;
    }
    if (status != U_OK) continue;

    if (change >= 1) {
      const int gp = hdr[9];
      const float a = in_from_word(*reinterpret_cast<const uint32_t*>(st + PS::O_HDR), gp, in_bf16);
      const float b = in_from_word(*reinterpret_cast<const uint32_t*>(st + PS::O_HDR + 4), gp, in_bf16);
      const float alog = *reinterpret_cast<const float*>(st + PS::O_HDR + 8);
      const float dtb = *reinterpret_cast<const float*>(st + PS::O_HDR + 12);
      alpha = decay_of(expf(alog), a + dtb);
      beta = (p.flags & F_BETA_PROB) ? b : sigmoid_f(b);
    }
    float x[2 * NR];
    {
      float qv[EPL], kv[EPL], sv[EPL];
      ld_in_vec<EPL>(st + PS::O_Q, cc * EPL, in_bf16, qv);
      ld_in_vec<EPL>(st + PS::O_K + cc * kblk, 0, in_bf16, kv);
      if (change >= 2) {
        float2 sq = make_float2(0.f, 0.f), sk = sq, sqk = sq;
#pragma unroll
        for (int e = 0; e < EPL; e += 2) {
          const float2 q2 = make_float2(qv[e], qv[e + 1]), k2 = make_float2(kv[e], kv[e + 1]);
          sq = __ffma2_rn(q2, q2, sq);
          sk = __ffma2_rn(k2, k2, sk);
          sqk = __ffma2_rn(q2, k2, sqk);
        }
        const float nq2 = group_sum<PS::LPR>(sq.x + sq.y);
        const float nk2 = group_sum<PS::LPR>(sk.x + sk.y);
        const float dqk = group_sum<PS::LPR>(sqk.x + sqk.y);
        iq = p.scale;
        ik = 1.0f;
        if (p.flags & F_L2NORM) {
          iq *= rsqrtf(nq2 + kL2Eps);
          ik = rsqrtf(nk2 + kL2Eps);
        }
        qk = dqk * iq * ik;
      }
      ld_vec16_f32(st + PS::O_SC + cc * FBLK, sv);
      // the scales ride on k and q for the dots
#pragma unroll
      for (int e = 0; e < EPL; e += 2) {
        const float2 s2 = make_float2(sv[e], sv[e + 1]);
        const float2 k2 = __fmul2_rn(make_float2(kv[e], kv[e + 1]), s2);
        const float2 q2 = __fmul2_rn(make_float2(qv[e], qv[e + 1]), s2);
        kv[e] = k2.x; kv[e + 1] = k2.y;
        qv[e] = q2.x; qv[e + 1] = q2.y;
      }
      // pass 1: partial k.S and q.S of every row on the code values
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        const uint4 raw = *reinterpret_cast<const uint4*>(st + my_off + r * ROWB);
        float c[EPL];
        decode_i8x16(raw, c);
        float2 ak = make_float2(0.f, 0.f), aq = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < EPL; e += 2) {
          const float2 c2 = make_float2(c[e], c[e + 1]);
          ak = __ffma2_rn(make_float2(kv[e], kv[e + 1]), c2, ak);
          aq = __ffma2_rn(make_float2(qv[e], qv[e + 1]), c2, aq);
        }
        x[2 * r] = ak.x + ak.y;
        x[2 * r + 1] = aq.x + aq.y;
      }
    }
    // row `lane`: its dots, R v, u and R o
    const float2 d = rs_row_pairs<NR, NR / 2>(x, cc);
    const float vl = in_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(st + PS::O_V)[lane])
                             : reinterpret_cast<const float*>(st + PS::O_V)[lane];
    const float vr = __fmul_rn(fwht_lanes(vl, lane), inv_sqrt32());
    const float u = beta * (vr - alpha * (d.x * ik));
    float o_rot = fmaf(qk, u, alpha * (d.y * iq));
    const float un = u * ik;

    // pass 2: the rows' codes decoded again, then S' = (alpha s) c + k (|k|^-1 u)
    // one key-channel pair at a time (k and s read from the stage as they are
    // needed, so that only S' stays in registers), with the pair's maxima
    float S[NR][EPL];
    float un_r[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      un_r[r] = __shfl_sync(kFull, un, row0 + r);
      decode_i8x16(*reinterpret_cast<const uint4*>(st + my_off + r * ROWB), S[r]);
    }
    // every lane has its codes: the code area takes the maxima
    __syncwarp();
    {
      const float2 a2 = make_float2(alpha, alpha);
      float4* mx = reinterpret_cast<float4*>(st + PS::O_MX + rb * PS::PADV + cc * FBLK);
#pragma unroll
      for (int c4 = 0; c4 < EPL / 4; ++c4) {
        float m[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int e = 4 * c4 + 2 * h;
          const float2 k2 = ld_in_pair(st + PS::O_K + cc * kblk, e, in_bf16);
          const float2 f2 = __fmul2_rn(a2, *reinterpret_cast<const float2*>(st + PS::O_SC + cc * FBLK + e * 4));
#pragma unroll
          for (int r = 0; r < NR; ++r) {
            const float2 y = __ffma2_rn(f2, make_float2(S[r][e], S[r][e + 1]),
                                        __fmul2_rn(k2, make_float2(un_r[r], un_r[r])));
            S[r][e] = y.x;
            S[r][e + 1] = y.y;
          }
          float m0 = 0.f, m1 = 0.f;
#pragma unroll
          for (int r = 0; r < NR; r += 2) {
            m0 = absmax_acc2(m0, S[r][e], S[r + 1][e]);
            m1 = absmax_acc2(m1, S[r][e + 1], S[r + 1][e + 1]);
          }
          m[2 * h] = m0;
          m[2 * h + 1] = m1;
        }
        mx[c4] = make_float4(m[0], m[1], m[2], m[3]);
      }
    }
    // the maxima per key channel over the 4 lanes of the lane's channels
    __syncwarp();
    {
      // lane l: key channels 4 l .. 4 l + 3
      const unsigned char* mx = st + PS::O_MX + pad16_ofs(lane, 4);
      float4 a = *reinterpret_cast<const float4*>(mx);
#pragma unroll
      for (int b = 1; b < PS::RB; ++b) {
        const float4 t = *reinterpret_cast<const float4*>(mx + b * PS::PADV);
        a = make_float4(fmaxf(a.x, t.x), fmaxf(a.y, t.y), fmaxf(a.z, t.z), fmaxf(a.w, t.w));
      }
      float4 s4, r4;
      h32_scale_of(a.x, s4.x, r4.x);
      h32_scale_of(a.y, s4.y, r4.y);
      h32_scale_of(a.z, s4.z, r4.z);
      h32_scale_of(a.w, s4.w, r4.w);
      float* dsc = p.scales + (dst_slot * per_b + within) * K;
      st_stream16(dsc + 4 * lane, make_uint4(__float_as_uint(s4.x), __float_as_uint(s4.y), __float_as_uint(s4.z),
                                             __float_as_uint(s4.w)));
      *reinterpret_cast<float4*>(st + PS::O_R + pad16_ofs(lane, 4)) = r4;
      if (stored_readout) *reinterpret_cast<float4*>(st + PS::O_S + pad16_ofs(lane, 4)) = s4;
    }
    __syncwarp();

    // re-encode rint(S' r'), four key channels (one code word per row) at a
    // time, so that S' leaves the registers as the codes come in
    {
      uint32_t cw[NR][EPL / 4];
#pragma unroll
      for (int c4 = 0; c4 < EPL / 4; ++c4) {
        const float4 r4 = *reinterpret_cast<const float4*>(st + PS::O_R + cc * FBLK + 16 * c4);
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          const float2 lo = __fmul2_rn(make_float2(S[r][4 * c4], S[r][4 * c4 + 1]), make_float2(r4.x, r4.y));
          const float2 hi = __fmul2_rn(make_float2(S[r][4 * c4 + 2], S[r][4 * c4 + 3]), make_float2(r4.z, r4.w));
          cw[r][c4] = float_to_i8x4(lo.x, lo.y, hi.x, hi.y);
        }
      }
      char* dst = reinterpret_cast<char*>(p.pool) + dst_slot * slot_bytes + (int64_t)within * UNITB + my_off;
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        st_stream16(dst + r * ROWB, make_uint4(cw[r][0], cw[r][1], cw[r][2], cw[r][3]));
        if (stored_readout) {
          // o from the stored state: q^.(c' s') of every row through the same
          // reduction, q and s' read from the stage four channels at a time
          float y = 0.f;
#pragma unroll
          for (int c4 = 0; c4 < EPL / 4; ++c4) {
            float c[4], q4[4];
            i8x4_to_float(cw[r][c4], c);
            ld_in_vec<4>(st + PS::O_Q, cc * EPL + 4 * c4, in_bf16, q4);
            const float4 s4 = *reinterpret_cast<const float4*>(st + PS::O_S + cc * FBLK + 16 * c4);
            y = fmaf(q4[0] * s4.x, c[0], y);
            y = fmaf(q4[1] * s4.y, c[1], y);
            y = fmaf(q4[2] * s4.z, c[2], y);
            y = fmaf(q4[3] * s4.w, c[3], y);
          }
          x[2 * r] = y;
          x[2 * r + 1] = 0.f;
        }
      }
      if (stored_readout) o_rot = rs_row_pairs<NR, NR / 2>(x, cc).x * iq;
    }
    // the output back from the rotated basis
    const float o = __fmul_rn(fwht_lanes(o_rot, lane), inv_sqrt32());
    st_out1(p.out, out_row + lane, o, out_bf16);
  }
  cp_async_wait<0>();
}

}  // namespace gdn
