// C ABI of the decode library: host-side validation, launch selection and
// the small auxiliary kernels (paged slot rows, fp8 tile codec,
// int8_hadamard32 codec).
//
// Validation runs before any CUDA call, so a rejected call touches neither
// the device nor the stream. The device is taken from the state pool's
// pointer: this library links its own CUDA runtime, whose current device is
// independent of the caller's.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <initializer_list>
#include <utility>

#include "../../include/gdn.h"
#include "gdn_seq.cuh"
#include "gdn_stream_fp8.cuh"
#include "gdn_stream_i8.cuh"
#include "gdn_group_i8.cuh"
#include "gdn_chunk_tc.cuh"
#include "gdn_kda_chunk.cuh"

using namespace gdn;

namespace {

bool aligned(const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) & (n - 1)) == 0; }
bool aligned16(const void* p) { return aligned(p, 16); }
uintptr_t io_size(int dtype) { return dtype == GDN_BF16 ? 2 : 4; }
uintptr_t index_size(int dtype) { return dtype == GDN_I64 ? 8 : 4; }

// Vector-loaded tensors need 16-byte alignment, scalar-loaded ones only
// their element size.
bool ptrs_ok(std::initializer_list<const void*> vec16, std::initializer_list<std::pair<const void*, uintptr_t>> scal) {
  for (const void* x : vec16)
    if (x == nullptr || !aligned16(x)) return false;
  for (const auto& x : scal)
    if (x.first == nullptr || !aligned(x.first, x.second)) return false;
  return true;
}
bool head_dim_ok(int x) { return x == 32 || x == 64 || x == 128 || x == 256; }
bool io_dtype_ok(int d) { return d == GDN_F32 || d == GDN_BF16; }
bool state_dtype_ok(int d) { return d == GDN_F32 || d == GDN_BF16 || d == GDN_FP8_E4M3 || d == GDN_INT8_H32; }
bool layout_ok(int l) { return l == GDN_K_FIRST || l == GDN_V_FIRST; }

// Checks of a state pool shared by every entry point.
int check_pool(const gdn_state_pool& pool, int V) {
  if (pool.data == nullptr || !aligned16(pool.data)) return GDN_ERR_INVALID_ARG;
  if (pool.num_slots < 0) return GDN_ERR_INVALID_ARG;
  if (!state_dtype_ok(pool.dtype) || !layout_ok(pool.layout)) return GDN_ERR_INVALID_ARG;
  if (pool.dtype == GDN_FP8_E4M3) {
    if (pool.scales == nullptr || !aligned(pool.scales, 4)) return GDN_ERR_INVALID_ARG;
    const int bv = pool.block_v == 0 ? 64 : pool.block_v;
    if (bv <= 0 || V % bv != 0) return GDN_ERR_INVALID_ARG;
    if (bv != 64) return GDN_ERR_UNSUPPORTED;
  }
  if (pool.dtype == GDN_INT8_H32) {
    if (pool.scales == nullptr || !aligned16(pool.scales)) return GDN_ERR_INVALID_ARG;
    if (V % 64 != 0) return GDN_ERR_UNSUPPORTED;  // the kernels' tile is two scale groups
  }
  return GDN_OK;
}

// Make the pool's device current for this library's runtime.
int select_device(const void* dev_ptr) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, dev_ptr) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) return GDN_ERR_INVALID_ARG;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != attr.device) {
    if (cudaSetDevice(attr.device) != cudaSuccess) {
      cudaGetLastError();
      return GDN_ERR_CUDA;
    }
  }
  return GDN_OK;
}

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// Single-token GDN decode on a V_FIRST fp32 or bf16 pool: one small CTA per tile.
template <int SDT, int K, int IDX>
int launch_tile1(StepParams p, int B, cudaStream_t s) {
  using TS = Tile1Shape<SDT, K>;
  p.n_vtiles = p.V / TS::VT;
  const dim3 grid(p.n_vtiles, p.HV, B);
  step_tile1<SDT, K, IDX><<<grid, TS::NW * 32, 0, s>>>(p);
  return launch_status();
}

// Single-token GDN decode on a V_FIRST fp8 or int8_hadamard32 pool:
// persistent CTAs (as many as fit on the device at once) over the (sequence,
// value head, tile) units. One instantiation per kernel, so that each
// kernel's shared-memory attribute and occupancy are set and cached for it.
template <class PS, auto KERNEL>
int launch_pipe(StepParams p, int B, cudaStream_t s) {
  static int resident[64] = {0};  // CTAs per SM, per device
  const auto kernel = KERNEL;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  if (resident[dev] == 0) {
    int n = 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PS::SMEM) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, PS::NT, PS::SMEM) != cudaSuccess || n < 1) {
      cudaGetLastError();
      return GDN_ERR_CUDA;
    }
    resident[dev] = n;
  }
  const int64_t n_tiles = (int64_t)B * p.HV * (p.V / PS::VT);
  const int64_t grid = std::min<int64_t>(n_tiles, (int64_t)sms * resident[dev]);
  kernel<<<static_cast<unsigned>(grid), PS::NT, PS::SMEM, s>>>(p, n_tiles);
  return launch_status();
}

// Paged prefill on the tensor cores (fp32 V_FIRST pages, K = V = 128, bf16
// token inputs, page_size a multiple of 64): one CTA per (value head, sequence).
int launch_prefill_tc(StepParams p, int B, cudaStream_t s) {
  static bool ready[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  if (!ready[dev]) {
    if (cudaFuncSetAttribute(prefill_chunk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, ChunkTC::SMEM) !=
        cudaSuccess) {
      cudaGetLastError();
      return GDN_ERR_CUDA;
    }
    ready[dev] = true;
  }
  if (B > 65535) return GDN_ERR_INVALID_ARG;  // grid y
  p.G = p.HV / p.H;
  prefill_chunk_tc<<<dim3(p.HV, B), ChunkTC::NT, ChunkTC::SMEM, s>>>(p);
  return launch_status();
}

// KDA varlen on the tensor cores (fp32 pools of either layout, K = V = 128,
// bf16 token inputs): one CTA per (value head, sequence), 32-token chunks.
// Runs shorter than a chunk are padded, so kda_decode_varlen sends a call
// here only when its runs average at least kKdaChunkMinMean tokens.
constexpr int kKdaChunkMinMean = 32;

template <int L>
int launch_kda_tc_l(StepParams p, int B, cudaStream_t s) {
  static bool ready[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  if (!ready[dev]) {
    if (cudaFuncSetAttribute(kda_chunk_tc<L>, cudaFuncAttributeMaxDynamicSharedMemorySize, KdaTC::SMEM) !=
        cudaSuccess) {
      cudaGetLastError();
      return GDN_ERR_CUDA;
    }
    ready[dev] = true;
  }
  if (B > 65535) return GDN_ERR_INVALID_ARG;  // grid y
  p.G = p.HV / p.H;
  kda_chunk_tc<L><<<dim3(p.HV, B), KdaTC::NT, KdaTC::SMEM, s>>>(p);
  return launch_status();
}

int launch_kda_tc(const StepParams& p, int layout, int B, cudaStream_t s) {
  return layout == GDN_V_FIRST ? launch_kda_tc_l<L_VFIRST>(p, B, s) : launch_kda_tc_l<L_KFIRST>(p, B, s);
}

// T >= 1 tokens per unit, either layout: the chunked-prologue kernel.
template <int L, int SDT, int K, int GATE, int IDX, int NW>
int launch_seq_nw(StepParams p, int B, cudaStream_t s) {
  using SH = SeqShape<SDT, L, K, NW>;
  p.n_vtiles = p.V / SH::VC;
  const dim3 grid(p.n_vtiles, p.HV, B);
  step_seq<SDT, L, K, GATE, IDX, NW><<<grid, NW * 32, 0, s>>>(p);
  return launch_status();
}

template <int L, int SDT, int K, int GATE, int IDX>
int launch_one(StepParams p, int B, cudaStream_t s) {
  p.G = p.HV / p.H;
  if (B > 65535) return GDN_ERR_INVALID_ARG;  // grid z
  constexpr bool CODED = (SDT == ST_FP8 || SDT == ST_I8H);
  if constexpr (L == L_VFIRST && GATE == GATE_SCALAR) {
    if (p.T == 1) {
      if constexpr (SDT == ST_I8H) {
        if constexpr (K == 128) {
          const bool bf = (p.flags & F_IN_BF16) != 0, st = (p.flags & F_READOUT_STORED) != 0;
          if (bf) return st ? launch_pipe<GroupI8Shape, step_group_i8<IDX, true, true>>(p, B, s)
                            : launch_pipe<GroupI8Shape, step_group_i8<IDX, true, false>>(p, B, s);
          return st ? launch_pipe<GroupI8Shape, step_group_i8<IDX, false, true>>(p, B, s)
                    : launch_pipe<GroupI8Shape, step_group_i8<IDX, false, false>>(p, B, s);
        }
        else return launch_pipe<StreamI8Shape<K>, step_stream_i8<K, IDX>>(p, B, s);
      }
      else if constexpr (SDT == ST_FP8) {
        if constexpr (K == 128) {
          // the configured width: input dtype and readout fixed per instantiation
          if (p.V % 128 == 0) {
            const int fl = ((p.flags & F_IN_BF16) ? 1 : 0) | ((p.flags & F_READOUT_STORED) ? 2 : 0);
            switch (fl) {
              case 0: return launch_pipe<StreamFp8Shape<K, 2>, step_stream_fp8<K, IDX, 2, 0>>(p, B, s);
              case 1: return launch_pipe<StreamFp8Shape<K, 2>, step_stream_fp8<K, IDX, 2, 1>>(p, B, s);
              case 2: return launch_pipe<StreamFp8Shape<K, 2>, step_stream_fp8<K, IDX, 2, 2>>(p, B, s);
              default: return launch_pipe<StreamFp8Shape<K, 2>, step_stream_fp8<K, IDX, 2, 3>>(p, B, s);
            }
          }
        }
        if (p.V % 128 == 0) return launch_pipe<StreamFp8Shape<K, 2>, step_stream_fp8<K, IDX, 2>>(p, B, s);
        return launch_pipe<StreamFp8Shape<K, 1>, step_stream_fp8<K, IDX, 1>>(p, B, s);
      }
      else return launch_tile1<SDT, K, IDX>(p, B, s);
    }
  }
  if constexpr (L == L_KFIRST) {
    constexpr int VTW = (K == 256) ? 8 : 16;  // columns per warp
    if constexpr (CODED) {
      return launch_seq_nw<L, SDT, K, GATE, IDX, 64 / VTW>(p, B, s);  // 64-column tiles of scale groups
    } else {
      if (p.V % (4 * VTW) != 0) return launch_seq_nw<L, SDT, K, GATE, IDX, 2>(p, B, s);
      return launch_seq_nw<L, SDT, K, GATE, IDX, 4>(p, B, s);
    }
  } else {
    // eight warps for wide int8/fp8 rows, and for fp32 K = 32 (one row per
    // thread: the shortest per-token chain for the latency-bound small heads)
    return launch_seq_nw<L, SDT, K, GATE, IDX, ((CODED && K == 256) || (SDT == ST_F32 && K == 32)) ? 8 : 4>(p, B, s);
  }
}

template <int L, int SDT, int GATE, int IDX>
int launch_k(const StepParams& p, int K, int B, cudaStream_t s) {
  switch (K) {
    case 32: return launch_one<L, SDT, 32, GATE, IDX>(p, B, s);
    case 64: return launch_one<L, SDT, 64, GATE, IDX>(p, B, s);
    case 128: return launch_one<L, SDT, 128, GATE, IDX>(p, B, s);
    case 256: return launch_one<L, SDT, 256, GATE, IDX>(p, B, s);
    default: return GDN_ERR_INVALID_ARG;
  }
}

template <int L, int GATE, int IDX>
int launch_sdt(const StepParams& p, int sdt, int K, int B, cudaStream_t s) {
  switch (sdt) {
    case GDN_F32: return launch_k<L, ST_F32, GATE, IDX>(p, K, B, s);
    case GDN_BF16: return launch_k<L, ST_BF16, GATE, IDX>(p, K, B, s);
    case GDN_FP8_E4M3: return launch_k<L, ST_FP8, GATE, IDX>(p, K, B, s);
    case GDN_INT8_H32: return launch_k<L, ST_I8H, GATE, IDX>(p, K, B, s);
    default: return GDN_ERR_INVALID_ARG;
  }
}

template <int GATE, int IDX>
int launch_step(const StepParams& p, const gdn_state_pool& pool, int K, int B, cudaStream_t s) {
  if (pool.layout == GDN_V_FIRST) return launch_sdt<L_VFIRST, GATE, IDX>(p, pool.dtype, K, B, s);
  return launch_sdt<L_KFIRST, GATE, IDX>(p, pool.dtype, K, B, s);
}

float default_scale(float scale, int K) {
  return scale > 0.0f ? scale : 1.0f / std::sqrt(static_cast<float>(K));
}

// --------------------------------------------------------------------------
// auxiliary kernels
// --------------------------------------------------------------------------
__global__ void paged_rows_kernel(const void* indices, const void* indptr, const void* lastlen, bool i64,
                                  int64_t nnz, int B, int64_t num_pages, int page_size, int64_t* rows,
                                  int32_t* err) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  int64_t r, w;
  int e = 0;
  resolve_page_rows(indices, indptr, lastlen, i64, nnz, num_pages, page_size, b, r, w, e);
  rows[2 * b] = r;
  rows[2 * b + 1] = w;
  raise_err(err, e);
}

// One CTA per [K, 64] tile of one state. Thread t owns 16-element chunks
// t, t + NT, ...; a chunk is 16 consecutive elements of one stored row.
template <int K, int LAYOUT>
__global__ void __launch_bounds__(K == 256 ? 256 : 128) fp8_quantize_kernel(const float* src, uint8_t* codes,
                                                                            float* scales, int V) {
  constexpr int NT = (K == 256) ? 256 : 128, BV = 64, CHUNKS = K * BV / 16, PER = CHUNKS / NT;
  static_assert(CHUNKS % NT == 0, "tile must split over the CTA");
  __shared__ float s_amax[NT / 32];
  const int n_tiles = V / BV;
  const int64_t n = blockIdx.x / n_tiles;
  const int tile = blockIdx.x % n_tiles;
  const int64_t base = n * (int64_t)K * V;
  int64_t off[PER];
  float x[PER][16];
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int ch = threadIdx.x + i * NT;
    if constexpr (LAYOUT == L_VFIRST) {
      const int row = tile * BV + ch / (K / 16);
      off[i] = base + (int64_t)row * K + (ch % (K / 16)) * 16;
    } else {
      const int row = ch / (BV / 16);
      off[i] = base + (int64_t)row * V + tile * BV + (ch % (BV / 16)) * 16;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float4 f = reinterpret_cast<const float4*>(src + off[i])[c];
      x[i][4 * c] = f.x; x[i][4 * c + 1] = f.y; x[i][4 * c + 2] = f.z; x[i][4 * c + 3] = f.w;
    }
#pragma unroll
    for (int e = 0; e < 16; e += 2) m = absmax_acc2(m, x[i][e], x[i][e + 1]);
  }
  m = group_max<32>(m);
  if ((threadIdx.x & 31) == 0) s_amax[threadIdx.x >> 5] = m;
  __syncthreads();
  float amax = s_amax[0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) amax = fmaxf(amax, s_amax[w]);
  float s, r;
  fp8_scale_of(amax, s, r);
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    float y[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) y[e] = fp8_prescale(x[i][e], r);
    *reinterpret_cast<uint4*>(codes + off[i]) = encode16<ST_FP8>(y);
  }
  if (threadIdx.x == 0) scales[n * n_tiles + tile] = s;
}

template <int LAYOUT>
__global__ void fp8_dequantize_kernel(const uint8_t* codes, const float* scales, float* dst, int64_t n_chunks,
                                      int K, int V) {
  const int64_t ch = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (ch >= n_chunks) return;
  const int64_t per_state = (int64_t)K * V / 16;
  const int64_t n = ch / per_state;
  const int64_t within = ch % per_state;
  int col;  // the V coordinate of the chunk's first element
  if constexpr (LAYOUT == L_VFIRST) col = static_cast<int>(within / (K / 16));
  else col = static_cast<int>((within % (V / 16)) * 16);
  const float s = scales[n * (V / 64) + col / 64];
  float x[16];
  decode16<ST_FP8>(*reinterpret_cast<const uint4*>(codes + ch * 16), x);
  float4* o = reinterpret_cast<float4*>(dst + ch * 16);
#pragma unroll
  for (int c = 0; c < 4; ++c)
    o[c] = make_float4(__fmul_rn(x[4 * c], s), __fmul_rn(x[4 * c + 1], s), __fmul_rn(x[4 * c + 2], s),
                       __fmul_rn(x[4 * c + 3], s));
}

template <int LAYOUT>
int launch_quantize(const float* src, uint8_t* codes, float* scales, int64_t n, int K, int V, cudaStream_t s) {
  const int64_t blocks = n * (V / 64);
  if (blocks > INT_MAX) return GDN_ERR_INVALID_ARG;
  const unsigned g = static_cast<unsigned>(blocks);
  switch (K) {
    case 32: fp8_quantize_kernel<32, LAYOUT><<<g, 128, 0, s>>>(src, codes, scales, V); break;
    case 64: fp8_quantize_kernel<64, LAYOUT><<<g, 128, 0, s>>>(src, codes, scales, V); break;
    case 128: fp8_quantize_kernel<128, LAYOUT><<<g, 128, 0, s>>>(src, codes, scales, V); break;
    case 256: fp8_quantize_kernel<256, LAYOUT><<<g, 256, 0, s>>>(src, codes, scales, V); break;
    default: return GDN_ERR_INVALID_ARG;
  }
  return launch_status();
}

// int8_hadamard32 codec: one thread per (state, 32-value group, key
// channel), consecutive threads on consecutive key channels. The 32 values
// are rotated in registers by the butterfly order of fwht32_regs, scaled by
// the binary32 nearest 1/sqrt(32), and coded against amax / 127.
template <int LAYOUT>
__global__ void __launch_bounds__(128) h32_quantize_kernel(const float* src, int8_t* codes, float* scales, int K,
                                                           int V, int64_t n_items) {
  const int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (it >= n_items) return;
  const int G = V / 32;
  const int k = static_cast<int>(it % K);
  const int64_t ng = it / K;
  const int g = static_cast<int>(ng % G);
  const int64_t base = (ng / G) * (int64_t)K * V;
  float x[32];
  if constexpr (LAYOUT == L_VFIRST) {
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = src[base + (int64_t)(32 * g + j) * K + k];
  } else {
    const float4* p4 = reinterpret_cast<const float4*>(src + base + (int64_t)k * V + 32 * g);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 f = p4[c];
      x[4 * c] = f.x; x[4 * c + 1] = f.y; x[4 * c + 2] = f.z; x[4 * c + 3] = f.w;
    }
  }
  fwht32_regs(x);
  float m = 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    x[j] = __fmul_rn(x[j], inv_sqrt32());
    m = absmax_acc(m, x[j]);
  }
  float s, r;
  h32_scale_of(fabsf(m), s, r);
  uint32_t w[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) y[e] = fminf(fmaxf(__fmul_rn(x[4 * c + e], r), -kInt8Max), kInt8Max);
    w[c] = float_to_i8x4(y[0], y[1], y[2], y[3]);
  }
  if constexpr (LAYOUT == L_VFIRST) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      codes[base + (int64_t)(32 * g + j) * K + k] = static_cast<int8_t>((w[j / 4] >> (8 * (j % 4))) & 0xffu);
  } else {
    uint4* c4 = reinterpret_cast<uint4*>(codes + base + (int64_t)k * V + 32 * g);
    c4[0] = make_uint4(w[0], w[1], w[2], w[3]);
    c4[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
  scales[ng * K + k] = s;
}

template <int LAYOUT>
__global__ void __launch_bounds__(128) h32_dequantize_kernel(const int8_t* codes, const float* scales, float* dst,
                                                             int K, int V, int64_t n_items) {
  const int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (it >= n_items) return;
  const int G = V / 32;
  const int k = static_cast<int>(it % K);
  const int64_t ng = it / K;
  const int g = static_cast<int>(ng % G);
  const int64_t base = (ng / G) * (int64_t)K * V;
  const float s = scales[ng * K + k];
  float x[32];
  if constexpr (LAYOUT == L_VFIRST) {
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = static_cast<float>(codes[base + (int64_t)(32 * g + j) * K + k]);
  } else {
    const uint4* c4 = reinterpret_cast<const uint4*>(codes + base + (int64_t)k * V + 32 * g);
    const uint4 a = c4[0], b = c4[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int c = 0; c < 8; ++c) i8x4_to_float(w[c], x + 4 * c);
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) x[j] = __fmul_rn(x[j], s);
  fwht32_regs(x);
#pragma unroll
  for (int j = 0; j < 32; ++j) x[j] = __fmul_rn(x[j], inv_sqrt32());
  if constexpr (LAYOUT == L_VFIRST) {
#pragma unroll
    for (int j = 0; j < 32; ++j) dst[base + (int64_t)(32 * g + j) * K + k] = x[j];
  } else {
    float4* d4 = reinterpret_cast<float4*>(dst + base + (int64_t)k * V + 32 * g);
#pragma unroll
    for (int c = 0; c < 8; ++c) d4[c] = make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
  }
}

// Shared checks of the two int8_hadamard32 codec calls; n_items out = threads.
int h32_codec_args(const void* a, const void* b, const void* c, int64_t n_states, int K, int V, int layout,
                   int64_t& n_items) {
  if (n_states < 0 || !head_dim_ok(K) || !head_dim_ok(V) || !layout_ok(layout)) return GDN_ERR_INVALID_ARG;
  n_items = n_states * (V / 32) * K;
  if (n_states == 0) return GDN_OK;
  if (a == nullptr || b == nullptr || c == nullptr) return GDN_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(b) || !aligned16(c)) return GDN_ERR_INVALID_ARG;
  if ((n_items + 127) / 128 > INT_MAX) return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

}  // namespace

// ==========================================================================
// entry points
// ==========================================================================
extern "C" {

const char* gdn_status_string(int status) {
  switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG: a shape, dtype, enum, pointer or struct_size is invalid";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: option not implemented by this library";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA: the CUDA launch failed";
    default: return "unknown gdn status";
  }
}

int gdn_decode_slots(const gdn_decode_slots_params* p, gdn_stream_t stream) {
  if (p == nullptr || p->struct_size != static_cast<int32_t>(sizeof(gdn_decode_slots_params)))
    return GDN_ERR_INVALID_ARG;
  if (p->B < 0 || p->T < 0 || p->H <= 0 || p->HV <= 0 || p->HV % p->H != 0) return GDN_ERR_INVALID_ARG;
  if (!head_dim_ok(p->K) || !head_dim_ok(p->V)) return GDN_ERR_INVALID_ARG;
  if (!io_dtype_ok(p->in_dtype) || !io_dtype_ok(p->out_dtype)) return GDN_ERR_INVALID_ARG;
  if (p->index_dtype != GDN_I32 && p->index_dtype != GDN_I64) return GDN_ERR_INVALID_ARG;
  if (p->readout != GDN_READOUT_WORKING && p->readout != GDN_READOUT_STORED) return GDN_ERR_INVALID_ARG;
  if (const int rc = check_pool(p->pool, p->V)) return rc;
  if (p->B == 0 || p->T == 0) return GDN_OK;
  const uintptr_t es = io_size(p->in_dtype);
  if (!ptrs_ok({p->q, p->k, p->v, p->out},
               {{p->a, es}, {p->b, es}, {p->A_log, 4}, {p->dt_bias, 4}, {p->state_indices, index_size(p->index_dtype)}}))
    return GDN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(p->B) * p->T > INT_MAX) return GDN_ERR_INVALID_ARG;
  if (const int rc = select_device(p->pool.data)) return rc;

  StepParams k{};
  k.q = p->q; k.k = p->k; k.v = p->v; k.gate = p->a; k.beta = p->b;
  k.A_log = p->A_log; k.dt_bias = p->dt_bias;
  k.pool = p->pool.data; k.scales = p->pool.scales;
  k.idx = p->state_indices; k.out = p->out; k.err = p->err_flags;
  k.num_slots = p->pool.num_slots;
  k.B = p->B; k.T = p->T; k.H = p->H; k.HV = p->HV; k.V = p->V;
  k.total_tokens = p->B * p->T;
  k.scale = default_scale(p->scale, p->K);
  k.flags = (p->in_dtype == GDN_BF16 ? F_IN_BF16 : 0) | (p->out_dtype == GDN_BF16 ? F_OUT_BF16 : 0) |
            (p->index_dtype == GDN_I64 ? F_IDX64 : 0) | (p->use_qk_l2norm ? F_L2NORM : 0) |
            (p->readout == GDN_READOUT_STORED ? F_READOUT_STORED : 0);
  return launch_step<GATE_SCALAR, IDX_SLOTS>(k, p->pool, p->K, p->B, reinterpret_cast<cudaStream_t>(stream));
}

int gdn_decode_paged(const gdn_decode_paged_params* p, gdn_stream_t stream) {
  if (p == nullptr || p->struct_size != static_cast<int32_t>(sizeof(gdn_decode_paged_params)))
    return GDN_ERR_INVALID_ARG;
  if (p->B < 0 || p->T < 0 || p->H <= 0 || p->HV <= 0 || p->HV % p->H != 0 || p->nnz < 0)
    return GDN_ERR_INVALID_ARG;
  if (p->T > 1 && (p->page_size <= 0 || p->slots != nullptr)) return GDN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(p->B) * p->T > INT_MAX) return GDN_ERR_INVALID_ARG;
  if (!head_dim_ok(p->K) || !head_dim_ok(p->V)) return GDN_ERR_INVALID_ARG;
  if (!io_dtype_ok(p->in_dtype) || !io_dtype_ok(p->out_dtype)) return GDN_ERR_INVALID_ARG;
  if (p->index_dtype != GDN_I32 && p->index_dtype != GDN_I64) return GDN_ERR_INVALID_ARG;
  if (p->readout != GDN_READOUT_WORKING && p->readout != GDN_READOUT_STORED) return GDN_ERR_INVALID_ARG;
  if (const int rc = check_pool(p->pool, p->V)) return rc;
  if (p->B == 0 || p->T == 0) return GDN_OK;
  const uintptr_t es = io_size(p->in_dtype), is = index_size(p->index_dtype);
  if (!ptrs_ok({p->q, p->k, p->v, p->out}, {{p->a, es}, {p->b, es}, {p->A_log, 4}, {p->dt_bias, 4}}))
    return GDN_ERR_INVALID_ARG;
  if (p->slots == nullptr) {
    if (!ptrs_ok({}, {{p->page_indices, is}, {p->page_indptr, is}, {p->last_page_len, is}}))
      return GDN_ERR_INVALID_ARG;
  } else if (!aligned(p->slots, 8)) {
    return GDN_ERR_INVALID_ARG;
  }
  if (const int rc = select_device(p->pool.data)) return rc;

  StepParams k{};
  k.q = p->q; k.k = p->k; k.v = p->v; k.gate = p->a; k.beta = p->b;
  k.A_log = p->A_log; k.dt_bias = p->dt_bias;
  k.pool = p->pool.data; k.scales = p->pool.scales;
  k.idx = p->page_indices; k.indptr = p->page_indptr; k.lastlen = p->last_page_len; k.rows = p->slots;
  k.out = p->out; k.err = p->err_flags;
  k.num_slots = p->pool.num_slots; k.nnz = p->nnz;
  k.B = p->B; k.T = p->T; k.H = p->H; k.HV = p->HV; k.V = p->V;
  k.total_tokens = p->B * p->T;
  k.page_size = p->page_size;
  k.scale = default_scale(p->scale, p->K);
  k.flags = (p->in_dtype == GDN_BF16 ? F_IN_BF16 : 0) | (p->out_dtype == GDN_BF16 ? F_OUT_BF16 : 0) |
            (p->index_dtype == GDN_I64 ? F_IDX64 : 0) | (p->use_qk_l2norm ? F_L2NORM : 0) |
            (p->readout == GDN_READOUT_STORED ? F_READOUT_STORED : 0);
  return launch_step<GATE_SCALAR, IDX_PAGED>(k, p->pool, p->K, p->B, reinterpret_cast<cudaStream_t>(stream));
}

int gdn_prefill_paged(const gdn_prefill_paged_params* p, gdn_stream_t stream) {
  if (p == nullptr || p->struct_size != static_cast<int32_t>(sizeof(gdn_prefill_paged_params)))
    return GDN_ERR_INVALID_ARG;
  if (p->B < 0 || p->total_tokens < 0 || p->H <= 0 || p->HV <= 0 || p->HV % p->H != 0 || p->nnz < 0)
    return GDN_ERR_INVALID_ARG;
  if (p->page_size <= 0) return GDN_ERR_INVALID_ARG;
  if (!head_dim_ok(p->K) || !head_dim_ok(p->V)) return GDN_ERR_INVALID_ARG;
  if (!io_dtype_ok(p->in_dtype) || !io_dtype_ok(p->out_dtype)) return GDN_ERR_INVALID_ARG;
  if (p->index_dtype != GDN_I32 && p->index_dtype != GDN_I64) return GDN_ERR_INVALID_ARG;
  if (p->readout != GDN_READOUT_WORKING && p->readout != GDN_READOUT_STORED) return GDN_ERR_INVALID_ARG;
  if (const int rc = check_pool(p->pool, p->V)) return rc;
  if (p->B == 0 || p->total_tokens == 0) return GDN_OK;
  const uintptr_t es = io_size(p->in_dtype), is = index_size(p->index_dtype);
  if (!ptrs_ok({p->q, p->k, p->v, p->out},
               {{p->a, es}, {p->b, es}, {p->A_log, 4}, {p->dt_bias, 4}, {p->cu_seqlens, 4},
                {p->page_indices, is}, {p->page_indptr, is}, {p->last_page_len, is}}))
    return GDN_ERR_INVALID_ARG;
  if (const int rc = select_device(p->pool.data)) return rc;

  StepParams k{};
  k.q = p->q; k.k = p->k; k.v = p->v; k.gate = p->a; k.beta = p->b;
  k.A_log = p->A_log; k.dt_bias = p->dt_bias;
  k.pool = p->pool.data; k.scales = p->pool.scales;
  k.idx = p->page_indices; k.indptr = p->page_indptr; k.lastlen = p->last_page_len; k.cu = p->cu_seqlens;
  k.out = p->out; k.err = p->err_flags;
  k.num_slots = p->pool.num_slots; k.nnz = p->nnz;
  k.B = p->B; k.T = 0; k.H = p->H; k.HV = p->HV; k.V = p->V;
  k.total_tokens = p->total_tokens;
  k.page_size = p->page_size;
  k.scale = default_scale(p->scale, p->K);
  k.flags = (p->in_dtype == GDN_BF16 ? F_IN_BF16 : 0) | (p->out_dtype == GDN_BF16 ? F_OUT_BF16 : 0) |
            (p->index_dtype == GDN_I64 ? F_IDX64 : 0) | (p->use_qk_l2norm ? F_L2NORM : 0) | F_VARLEN |
            (p->readout == GDN_READOUT_STORED ? F_READOUT_STORED : 0);
  if (p->pool.dtype == GDN_F32 && p->pool.layout == GDN_V_FIRST && p->K == ChunkTC::D && p->V == ChunkTC::D &&
      p->in_dtype == GDN_BF16 && p->page_size % ChunkTC::C == 0)
    return launch_prefill_tc(k, p->B, reinterpret_cast<cudaStream_t>(stream));
  return launch_step<GATE_SCALAR, IDX_PAGED>(k, p->pool, p->K, p->B, reinterpret_cast<cudaStream_t>(stream));
}

int gdn_paged_decode_slots(const void* page_indices, const void* page_indptr, const void* last_page_len,
                           int32_t index_dtype, int64_t nnz, int32_t B, int64_t num_pages, int32_t page_size,
                           int64_t* slots_out, int32_t* err_flags, gdn_stream_t stream) {
  if (B < 0 || nnz < 0 || num_pages < 0) return GDN_ERR_INVALID_ARG;
  if (index_dtype != GDN_I32 && index_dtype != GDN_I64) return GDN_ERR_INVALID_ARG;
  if (B == 0) return GDN_OK;
  const uintptr_t is = index_size(index_dtype);
  if (!ptrs_ok({}, {{page_indices, is}, {page_indptr, is}, {last_page_len, is}, {slots_out, 8}}))
    return GDN_ERR_INVALID_ARG;
  if (const int rc = select_device(slots_out)) return rc;
  const int threads = 128;
  paged_rows_kernel<<<(B + threads - 1) / threads, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      page_indices, page_indptr, last_page_len, index_dtype == GDN_I64, nnz, B, num_pages, page_size, slots_out,
      err_flags);
  return launch_status();
}

int kda_decode_varlen(const kda_decode_varlen_params* p, gdn_stream_t stream) {
  if (p == nullptr || p->struct_size != static_cast<int32_t>(sizeof(kda_decode_varlen_params)))
    return GDN_ERR_INVALID_ARG;
  if (p->B < 0 || p->total_tokens < 0 || p->Hk <= 0 || p->HV <= 0 || p->HV % p->Hk != 0) return GDN_ERR_INVALID_ARG;
  if (!head_dim_ok(p->K) || !head_dim_ok(p->V)) return GDN_ERR_INVALID_ARG;
  if (!io_dtype_ok(p->in_dtype) || !io_dtype_ok(p->out_dtype)) return GDN_ERR_INVALID_ARG;
  if (p->gate_mode != KDA_GATE_ORIGINAL && p->gate_mode != KDA_GATE_SAFE) return GDN_ERR_INVALID_ARG;
  if (p->beta_mode != KDA_BETA_LOGITS && p->beta_mode != KDA_BETA_PROBABILITY) return GDN_ERR_INVALID_ARG;
  if (p->readout != GDN_READOUT_WORKING && p->readout != GDN_READOUT_STORED) return GDN_ERR_INVALID_ARG;
  if (const int rc = check_pool(p->pool, p->V)) return rc;
  if (p->gate_mode == KDA_GATE_SAFE) return GDN_ERR_UNSUPPORTED;
  if (p->B == 0 || p->total_tokens == 0) return GDN_OK;
  const uintptr_t es = io_size(p->in_dtype);
  if (!ptrs_ok({p->q, p->k, p->v, p->raw_gate, p->dt_bias, p->out},
               {{p->beta_logits, es}, {p->a_log, 4}, {p->cu_seqlens, 4}, {p->state_indices, 4}}))
    return GDN_ERR_INVALID_ARG;
  if (const int rc = select_device(p->pool.data)) return rc;

  StepParams k{};
  k.q = p->q; k.k = p->k; k.v = p->v; k.gate = p->raw_gate; k.beta = p->beta_logits;
  k.A_log = p->a_log; k.dt_bias = p->dt_bias;
  k.pool = p->pool.data; k.scales = p->pool.scales;
  k.idx = p->state_indices; k.indptr = p->cu_seqlens; k.out = p->out; k.err = p->err_flags;
  k.num_slots = p->pool.num_slots;
  k.B = p->B; k.T = 0; k.H = p->Hk; k.HV = p->HV; k.V = p->V;
  k.total_tokens = p->total_tokens;
  k.scale = 1.0f / std::sqrt(static_cast<float>(p->K));
  k.flags = (p->in_dtype == GDN_BF16 ? F_IN_BF16 : 0) | (p->out_dtype == GDN_BF16 ? F_OUT_BF16 : 0) | F_L2NORM |
            F_VARLEN | (p->beta_mode == KDA_BETA_PROBABILITY ? F_BETA_PROB : 0) |
            (p->readout == GDN_READOUT_STORED ? F_READOUT_STORED : 0);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (p->pool.dtype == GDN_F32 && p->K == 128 && p->V == 128 && p->in_dtype == GDN_BF16 &&
      static_cast<int64_t>(p->total_tokens) >= static_cast<int64_t>(kKdaChunkMinMean) * p->B)
    return launch_kda_tc(k, p->pool.layout, p->B, s);
  return launch_step<GATE_VECTOR, IDX_SLOTS>(k, p->pool, p->K, p->B, s);
}

int gdn_state_quantize_fp8(const float* src, uint8_t* codes, float* scales, int64_t n_states, int32_t K, int32_t V,
                           int32_t block_v, int32_t layout, gdn_stream_t stream) {
  if (n_states < 0 || !head_dim_ok(K) || !head_dim_ok(V) || !layout_ok(layout)) return GDN_ERR_INVALID_ARG;
  if (block_v <= 0 || V % block_v != 0) return GDN_ERR_INVALID_ARG;
  if (block_v != 64) return GDN_ERR_UNSUPPORTED;
  if (n_states == 0) return GDN_OK;
  if (src == nullptr || codes == nullptr || scales == nullptr) return GDN_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(codes)) return GDN_ERR_INVALID_ARG;
  if (const int rc = select_device(src)) return rc;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return layout == GDN_V_FIRST ? launch_quantize<L_VFIRST>(src, codes, scales, n_states, K, V, s)
                               : launch_quantize<L_KFIRST>(src, codes, scales, n_states, K, V, s);
}

int gdn_state_dequantize_fp8(const uint8_t* codes, const float* scales, float* dst, int64_t n_states, int32_t K,
                             int32_t V, int32_t block_v, int32_t layout, gdn_stream_t stream) {
  if (n_states < 0 || !head_dim_ok(K) || !head_dim_ok(V) || !layout_ok(layout)) return GDN_ERR_INVALID_ARG;
  if (block_v <= 0 || V % block_v != 0) return GDN_ERR_INVALID_ARG;
  if (block_v != 64) return GDN_ERR_UNSUPPORTED;
  if (n_states == 0) return GDN_OK;
  if (codes == nullptr || scales == nullptr || dst == nullptr) return GDN_ERR_INVALID_ARG;
  if (!aligned16(dst) || !aligned16(codes)) return GDN_ERR_INVALID_ARG;
  if (const int rc = select_device(dst)) return rc;
  const int64_t n_chunks = n_states * K * V / 16;
  const int threads = 256;
  const int64_t blocks = (n_chunks + threads - 1) / threads;
  if (blocks > INT_MAX) return GDN_ERR_INVALID_ARG;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (layout == GDN_V_FIRST)
    fp8_dequantize_kernel<L_VFIRST><<<static_cast<unsigned>(blocks), threads, 0, s>>>(codes, scales, dst, n_chunks, K, V);
  else
    fp8_dequantize_kernel<L_KFIRST><<<static_cast<unsigned>(blocks), threads, 0, s>>>(codes, scales, dst, n_chunks, K, V);
  return launch_status();
}

int gdn_state_quantize_int8h32(const float* src, int8_t* codes, float* scales, int64_t n_states, int32_t K,
                               int32_t V, int32_t layout, gdn_stream_t stream) {
  int64_t n = 0;
  if (const int rc = h32_codec_args(src, codes, scales, n_states, K, V, layout, n)) return rc;
  if (n_states == 0) return GDN_OK;
  if (const int rc = select_device(src)) return rc;
  const unsigned blocks = static_cast<unsigned>((n + 127) / 128);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (layout == GDN_V_FIRST) h32_quantize_kernel<L_VFIRST><<<blocks, 128, 0, s>>>(src, codes, scales, K, V, n);
  else h32_quantize_kernel<L_KFIRST><<<blocks, 128, 0, s>>>(src, codes, scales, K, V, n);
  return launch_status();
}

int gdn_state_dequantize_int8h32(const int8_t* codes, const float* scales, float* dst, int64_t n_states, int32_t K,
                                 int32_t V, int32_t layout, gdn_stream_t stream) {
  int64_t n = 0;
  if (const int rc = h32_codec_args(codes, scales, dst, n_states, K, V, layout, n)) return rc;
  if (n_states == 0) return GDN_OK;
  if (const int rc = select_device(dst)) return rc;
  const unsigned blocks = static_cast<unsigned>((n + 127) / 128);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (layout == GDN_V_FIRST) h32_dequantize_kernel<L_VFIRST><<<blocks, 128, 0, s>>>(codes, scales, dst, K, V, n);
  else h32_dequantize_kernel<L_KFIRST><<<blocks, 128, 0, s>>>(codes, scales, dst, K, V, n);
  return launch_status();
}

}  // extern "C"
