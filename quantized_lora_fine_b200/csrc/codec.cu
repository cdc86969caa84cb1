// NF4 quantizer, dequantizer and the small elementwise / reduction kernels of
// the LoRA path. All HBM-bound: 128-bit loads and stores, warp shuffles.
#include <algorithm>
#include <cfloat>
#include <cstdlib>
#include <cstring>
#include <cuda_bf16.h>

#include <mutex>

#include "internal.cuh"
#include "nf4_device.cuh"
#include "ptx.cuh"

namespace qlb {

// ------------------------------------------------------------------ quantize
//
// One CTA of 256 threads per group of 256 blocks (16384 elements). In each of 8
// slices, lane l of warp w handles elements [8*(l%8), 8*(l%8)+8) of block
// (slice*32 + 4*w + l/8): a warp reads 512 contiguous bytes of bf16 per slice.

template <typename T>
__device__ __forceinline__ void load8(const T* W, int64_t e0, int64_t numel, float (&w)[8]);

template <>
__device__ __forceinline__ void load8<uint16_t>(const uint16_t* W, int64_t e0, int64_t numel, float (&w)[8]) {
  if (e0 + 8 <= numel) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(W + e0));
    uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) { w[2 * i] = bf16_lo(u[i]); w[2 * i + 1] = bf16_hi(u[i]); }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = (e0 + i < numel) ? __uint_as_float(uint32_t(W[e0 + i]) << 16) : 0.f;
  }
}

template <>
__device__ __forceinline__ void load8<float>(const float* W, int64_t e0, int64_t numel, float (&w)[8]) {
  if (e0 + 8 <= numel) {
    float4 a = __ldg(reinterpret_cast<const float4*>(W + e0));
    float4 b = __ldg(reinterpret_cast<const float4*>(W + e0 + 4));
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = (e0 + i < numel) ? W[e0 + i] : 0.f;
  }
}

// Shared tail of both quantizer variants: double quantization of the group's
// 256 absmax values held in s_amax.
__device__ __forceinline__ void dq_group(const float* s_amax, float* s_red, int64_t nb, int64_t g,
                                         uint8_t* __restrict__ absmax_q, float* __restrict__ absmax2) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __syncthreads();
  const int64_t nblk_g = (int64_t(kDQBlock) < nb - g * kDQBlock ? int64_t(kDQBlock) : nb - g * kDQBlock);
  float v = (tid < nblk_g) ? s_amax[tid] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  float G = s_red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) G = fmaxf(G, s_red[i]);
  if (tid < nblk_g) {
    uint8_t q = 0;
    if (G > 0.f) {
      const float inv = __fdiv_rn(448.f, G);
      q = f32_to_e4m3_satfinite(__fmul_rn(s_amax[tid], inv));
    }
    absmax_q[g * kDQBlock + tid] = q;
  }
  if (tid == 0) absmax2[g] = (G > 0.f) ? __fdiv_rn(G, 448.f) : 0.f;
}

// bf16 weights. One CTA of 256 threads per group of 256 blocks (16384 elements, the
// double-quant group); thread t owns block t. The group's weights (up to 32 KB)
// reach shared memory by one bulk copy (an odd tail of fewer than 8 elements by
// plain loads); thread t reads its block as eight 16-byte pieces, piece j ^ (t mod 8)
// at step j, so that the 8 lanes of a quarter warp touch 8 different bank groups.
// Per block: absmax over packed bf16 pairs and one reciprocal r = RN(1/a). Per
// element pair: one packed fp32 multiply n~ = RN(w r). For every pair of bf16
// values with |w| <= a, n~ lies on the same side of every code midpoint as the
// IEEE quotient RN(w / a) (an exhaustive check over all significand pairs and
// exponent gaps; the GPU tests repeat it through this kernel), so n~ picks the
// same code. Per element the code index comes from a 32-cell lookup held in the
// warp's registers: cell = floor(15.75 n~ + 16) from the bits of an RZ multiply-add,
// the cell's base index B and the midpoint above it by two warp shuffles, s =
// sat(n~ 2^36 + T) in {0, 1}, and bits(B + s) carry the index; a multiply-add chain
// packs 8 of them into a code word. Three exchange stages put the thread's 8 code
// words back in order, and the block's 32 bytes leave in two 16-byte stores.
// The matrices one launch quantizes: a single one (QuantOne, one CTA per group) or
// up to kMaxQuantBatch of them (QuantBatch; the CTA's matrix is found by a binary
// search over first_group).
struct QuantOne {
  const uint16_t* W;
  int64_t numel;
  uint8_t* codes;
  float* absmax;
  uint8_t* absmax_q;
  float* absmax2;
};
constexpr int kMaxQuantBatch = 512;
struct QuantBatch {
  const uint16_t* W[kMaxQuantBatch];
  int64_t numel[kMaxQuantBatch];
  uint8_t* codes[kMaxQuantBatch];
  float* absmax[kMaxQuantBatch];   // may be null with double quant
  uint8_t* absmax_q[kMaxQuantBatch];
  float* absmax2[kMaxQuantBatch];
  int32_t first_group[kMaxQuantBatch + 1];
  int32_t n;
};
static_assert(sizeof(QuantBatch) <= 32000, "kernel parameter limit");

__device__ __forceinline__ QuantOne quant_target(const QuantOne& t, int64_t cta, int64_t& g) {
  g = cta;
  return t;
}
__device__ __forceinline__ QuantOne quant_target(const QuantBatch& t, int64_t cta, int64_t& g) {
  int lo = 0, hi = t.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (t.first_group[mid] <= cta) lo = mid; else hi = mid - 1;
  }
  g = cta - t.first_group[lo];
  return QuantOne{t.W[lo], t.numel[lo], t.codes[lo], t.absmax[lo], t.absmax_q[lo], t.absmax2[lo]};
}

// With RELOAD each thread reads its eight pieces from shared memory twice (for the
// absmax, then for the codes) instead of holding them in registers, so more CTAs fit
// an SM.
template <bool DQ, class Tab, bool RELOAD = false>
__global__ void __launch_bounds__(256, RELOAD ? 6 : 4) nf4_quantize_bf16_kernel(const __grid_constant__ Tab tab,
                                                                                int* status) {
  __shared__ __align__(128) uint32_t s_w[kChunkBytes / 4];   // the group's bf16 pairs
  __shared__ float s_amax[kDQBlock];
  __shared__ float s_red[8];
  __shared__ __align__(8) uint64_t s_bar;
  const int tid = threadIdx.x;
  const uint32_t bar = smem_u32(&s_bar);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbarrier_init();
  }
  const LaneTables lt = lane_tables(tid & 31);
  int64_t g;
  const QuantOne q = quant_target(tab, blockIdx.x, g);
  const uint16_t* __restrict__ W = q.W;
  const int64_t numel = q.numel;
  uint8_t* __restrict__ codes = q.codes;
  float* __restrict__ absmax = q.absmax;
  uint8_t* __restrict__ absmax_q = q.absmax_q;
  float* __restrict__ absmax2 = q.absmax2;
  const int64_t nb = (numel + kBlock - 1) / kBlock;
  const int64_t e_g = g * int64_t(kDQBlock * kBlock);                 // first element of the group
  const int n_g = int(min(int64_t(kDQBlock * kBlock), numel - e_g));  // its elements (even, > 0)
  const int nblk = (n_g + kBlock - 1) / kBlock;
  const uint32_t bulk = uint32_t(n_g * 2) & ~15u;                     // bytes the bulk copy moves
  __syncthreads();
  pdl_wait();
  pdl_launch();
  if (bulk > 0) {
    if (tid == 0) {
      mbar_arrive_expect_tx(bar, bulk);
      bulk_load(smem_u32(s_w), W + e_g, bulk, bar);
    }
    const bool landed = mbar_wait(bar, 0);
    if (!__syncthreads_and(landed)) {   // every thread leaves together
      if (tid == 0) set_status(status, QLORA_ERR_TIMEOUT);
      if (!landed) mbar_wait(bar, 0, 20000000000ull);   // the copy must land before the CTA's memory is released
      return;
    }
  }
  // the last block of a ragged group: elements past the bulk copy by plain loads
  // (whole bf16 pairs: numel is even), zeros to the end of the block
  const int tail0 = int(bulk / 2);
  if (tail0 < nblk * kBlock && tid == tail0 / kBlock) {
    for (int e = tail0; e < nblk * kBlock; e += 2)
      s_w[e / 2] = (e < n_g) ? __ldg(reinterpret_cast<const uint32_t*>(W + e_g + e)) : 0u;
  }
  const bool valid = tid < nblk;
  const uint32_t rot = uint32_t(tid & 7);
  const uint32_t src = smem_u32(s_w) + uint32_t(tid) * 128u + rot * 16u;
  uint32_t u[RELOAD ? 1 : 8][4];
  uint32_t m = 0u;
  if constexpr (RELOAD) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t v[4] = {0u, 0u, 0u, 0u};
      if (valid) lds_u4(src ^ (uint32_t(j) << 4), v);
      m = bf16x2_maxabs(m, v[0]);
      m = bf16x2_maxabs(m, v[1]);
      m = bf16x2_maxabs(m, v[2]);
      m = bf16x2_maxabs(m, v[3]);
    }
  } else {
    if (valid) {
#pragma unroll
      for (int j = 0; j < 8; ++j) lds_u4(src ^ (uint32_t(j) << 4), u[j]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) u[j][0] = u[j][1] = u[j][2] = u[j][3] = 0u;
    }
    m = bf16x2_maxabs(u[0][0], u[0][1]);
#pragma unroll
    for (int k = 2; k < 32; ++k) m = bf16x2_maxabs(m, u[k >> 2][k & 3]);
  }
  m &= 0x7FFF7FFFu;
  const uint32_t amb = max(m >> 16, m & 0xFFFFu);
  const bool bad = amb >= 0x7F80u;
  const float am = __uint_as_float(amb << 16);
  if (valid) {
    if constexpr (DQ) s_amax[tid] = am;
    if (absmax != nullptr) absmax[g * kDQBlock + tid] = am;
  }
  // Every lane runs the lookup (it holds warp shuffles). Lanes without a live block
  // (past the group, all-zero or non-finite) run it on zeros with a = 1, which keeps
  // every quotient finite; their code words are the zero code (a non-finite block
  // sets the status word).
  const bool live = am > 0.f && !bad;
  if constexpr (!RELOAD) {
    if (bad) {
#pragma unroll
      for (int j = 0; j < 8; ++j) u[j][0] = u[j][1] = u[j][2] = u[j][3] = 0u;
    }
  }
  const CellScale cs(live ? am : 1.f);
  uint32_t cw[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t x[8];
    if constexpr (RELOAD) {
      u[0][0] = u[0][1] = u[0][2] = u[0][3] = 0u;
      if (valid && !bad) lds_u4(src ^ (uint32_t(j) << 4), u[0]);
      piece_index_bits(u[0], cs, lt, x);
    } else {
      piece_index_bits(u[j], cs, lt, x);
    }
    cw[j] = live ? pack_code_word(x) : 0x77777777u;
  }
  if (valid) {
    unrotate8(cw, rot);
    // the block's 32 code bytes (fewer in a ragged last block)
    const int cb = min(32, n_g / 2 - 32 * tid);
    uint8_t* dst = codes + e_g / 2 + 32 * tid;
    if (cb == 32) {
      reinterpret_cast<uint4*>(dst)[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      reinterpret_cast<uint4*>(dst)[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
    } else {
#pragma unroll
      for (int b = 0; b < 32; ++b)   // static indices keep cw in registers
        if (b < cb) dst[b] = uint8_t(cw[b >> 2] >> (8 * (b & 3)));
    }
  }
  if (bad) set_status(status, QLORA_ERR_NONFINITE);
  if constexpr (DQ) dq_group(s_amax, s_red, nb, g, absmax_q, absmax2);
}

// fp32 weights: IEEE division per element, linear midpoint count (kept simple:
// the workloads quantize bf16 weights).
template <bool DQ>
__global__ void __launch_bounds__(256) nf4_quantize_f32_kernel(const float* __restrict__ W, int64_t numel,
                                                               uint8_t* __restrict__ codes,
                                                               float* __restrict__ absmax,
                                                               uint8_t* __restrict__ absmax_q,
                                                               float* __restrict__ absmax2, int* status) {
  __shared__ float s_amax[256];
  __shared__ float s_red[8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t nb = (numel + kBlock - 1) / kBlock;
  const int64_t g = blockIdx.x;
  bool bad = false;
#pragma unroll 1
  for (int it = 0; it < 8; ++it) {
    const int bi = it * 32 + warp * 4 + (lane >> 3);
    const int64_t blk = g * kDQBlock + bi;
    const int64_t e0 = blk * kBlock + (lane & 7) * 8;
    float w[8];
    const bool live = blk < nb && e0 < numel;
    if (live) load8<float>(W, e0, numel, w);
    else {
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = 0.f;
    }
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float aw = fabsf(w[i]);
      bad |= !(aw <= FLT_MAX);
      am = fmaxf(am, aw);
    }
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
    if ((lane & 7) == 0) {
      s_amax[bi] = am;
      if (blk < nb && absmax != nullptr) absmax[blk] = am;
    }
    if (live) {
      uint32_t idx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) idx[i] = (am > 0.f) ? nf4_index(__fdiv_rn(w[i], am)) : 7u;
      if (e0 + 8 <= numel) {
        uint32_t word = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) word |= ((idx[2 * k] << 4) | idx[2 * k + 1]) << (8 * k);
        *reinterpret_cast<uint32_t*>(codes + e0 / 2) = word;
      } else {
        for (int k = 0; 2 * k < numel - e0; ++k) codes[e0 / 2 + k] = uint8_t((idx[2 * k] << 4) | idx[2 * k + 1]);
      }
    }
  }
  if (bad) set_status(status, QLORA_ERR_NONFINITE);
  if constexpr (DQ) dq_group(s_amax, s_red, nb, g, absmax_q, absmax2);
}

// Quantizer variant: each thread reads its block from shared memory twice (more CTAs
// per SM), unless QLORA_B200_QUANT_RELOAD=0 (read on every call).
static bool quant_reload() {
  const char* e = std::getenv("QLORA_B200_QUANT_RELOAD");
  return !(e && std::strcmp(e, "0") == 0);
}

qlora_status launch_quantize(const void* W, int w_dtype, int64_t numel, bool dq, uint8_t* codes, float* absmax,
                             uint8_t* absmax_q, float* absmax2, int* status, cudaStream_t s) {
  const int64_t nb = (numel + kBlock - 1) / kBlock;
  const int64_t groups = (nb + kDQBlock - 1) / kDQBlock;
  if (groups <= 0) return QLORA_OK;
  dim3 grid(static_cast<unsigned>(groups));
  if (w_dtype == QLORA_DTYPE_BF16) {
    const uint16_t* Wb = static_cast<const uint16_t*>(W);
    const QuantOne one{Wb, numel, codes, absmax, absmax_q, absmax2};
    if (quant_reload()) {
      if (dq) launch_pdl(nf4_quantize_bf16_kernel<true, QuantOne, true>, grid, dim3(256), 0, s, one, status);
      else launch_pdl(nf4_quantize_bf16_kernel<false, QuantOne, true>, grid, dim3(256), 0, s, one, status);
    } else {
      if (dq) launch_pdl(nf4_quantize_bf16_kernel<true, QuantOne>, grid, dim3(256), 0, s, one, status);
      else launch_pdl(nf4_quantize_bf16_kernel<false, QuantOne>, grid, dim3(256), 0, s, one, status);
    }
  } else {
    if (dq) nf4_quantize_f32_kernel<true><<<grid, 256, 0, s>>>((const float*)W, numel, codes, absmax, absmax_q, absmax2, status);
    else nf4_quantize_f32_kernel<false><<<grid, 256, 0, s>>>((const float*)W, numel, codes, absmax, absmax_q, absmax2, status);
  }
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status launch_quantize_batch(int n, const uint16_t* const* W, const int64_t* numel, bool dq,
                                   uint8_t* const* codes, float* const* absmax, uint8_t* const* absmax_q,
                                   float* const* absmax2, int* status, cudaStream_t s) {
  if (n < 1 || n > kMaxQuantBatch) return QLORA_ERR_SHAPE;
  static std::mutex mu;
  static QuantBatch tab;   // host staging of the by-value parameter
  std::lock_guard<std::mutex> lock(mu);
  tab.n = n;
  int64_t c = 0;
  for (int i = 0; i < n; ++i) {
    tab.W[i] = W[i];
    tab.numel[i] = numel[i];
    tab.codes[i] = codes[i];
    tab.absmax[i] = absmax ? absmax[i] : nullptr;
    tab.absmax_q[i] = dq ? absmax_q[i] : nullptr;
    tab.absmax2[i] = dq ? absmax2[i] : nullptr;
    tab.first_group[i] = int32_t(c);
    const int64_t nb = (numel[i] + kBlock - 1) / kBlock;
    c += (nb + kDQBlock - 1) / kDQBlock;
    if (c > (int64_t(1) << 31) - 1) return QLORA_ERR_SHAPE;
  }
  tab.first_group[n] = int32_t(c);
  const dim3 grid(static_cast<unsigned>(c));
  const bool rl = quant_reload();
  const cudaError_t e =
      dq ? (rl ? launch_pdl(nf4_quantize_bf16_kernel<true, QuantBatch, true>, grid, dim3(256), 0, s, tab, status)
               : launch_pdl(nf4_quantize_bf16_kernel<true, QuantBatch>, grid, dim3(256), 0, s, tab, status))
         : (rl ? launch_pdl(nf4_quantize_bf16_kernel<false, QuantBatch, true>, grid, dim3(256), 0, s, tab, status)
               : launch_pdl(nf4_quantize_bf16_kernel<false, QuantBatch>, grid, dim3(256), 0, s, tab, status));
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? QLORA_OK : QLORA_ERR_CUDA;
}

// ---------------------------------------------------------------- dequantize
//
// Each thread turns 16 code bytes (32 elements, half a block) into 64 bytes of
// bf16 through the per-block product table.

__device__ __forceinline__ float block_scale(int64_t blk, const float* absmax, const uint8_t* absmax_q,
                                             const float* absmax2, bool dq) {
  if (!dq) return __ldg(absmax + blk);
  return __fmul_rn(e4m3_to_f32(__ldg(absmax_q + blk)), __ldg(absmax2 + blk / kDQBlock));
}

__global__ void __launch_bounds__(256) nf4_dequantize_kernel(const uint8_t* __restrict__ codes,
                                                             const float* __restrict__ absmax,
                                                             const uint8_t* __restrict__ absmax_q,
                                                             const float* __restrict__ absmax2, int dq,
                                                             int64_t numel, uint16_t* __restrict__ out) {
  const int64_t n_units = (numel + 31) / 32;
  for (int64_t u = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; u < n_units; u += int64_t(gridDim.x) * blockDim.x) {
    const int64_t e0 = u * 32;
    const int64_t blk = e0 / kBlock;
    const float a = block_scale(blk, absmax, absmax_q, absmax2, dq != 0);
    const NF4Lut t = nf4_make_lut(a);
    if (e0 + 32 <= numel) {
      const uint4 c = __ldg(reinterpret_cast<const uint4*>(codes + e0 / 2));
      const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
      uint4* dst = reinterpret_cast<uint4*>(out + e0);
#pragma unroll
      for (int k = 0; k < 4; ++k) dst[k] = nf4_dequant_word(cw[k], t);
    } else {
      for (int64_t e = e0; e < numel; ++e) {
        const uint8_t b = codes[e / 2];
        const uint32_t j = (e & 1) ? (b & 0xF) : (b >> 4);
        const float v = __fmul_rn(nf4_code(j), a);
        __nv_bfloat16 h = __float2bfloat16_rn(v);
        out[e] = *reinterpret_cast<uint16_t*>(&h);
      }
    }
  }
}

qlora_status launch_dequantize(const uint8_t* codes, const float* absmax, const uint8_t* absmax_q,
                               const float* absmax2, bool dq, int64_t numel, uint16_t* out, cudaStream_t s) {
  const int64_t n_units = (numel + 31) / 32;
  if (n_units == 0) return QLORA_OK;
  const int64_t blocks = std::min<int64_t>((n_units + 255) / 256, int64_t(num_sms()) * 16);
  nf4_dequantize_kernel<<<unsigned(blocks), 256, 0, s>>>(codes, absmax, absmax_q, absmax2, dq ? 1 : 0, numel, out);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// ------------------------------------------------------------------ LoRA merge
//
// W_out = bf16_rn(W_hat + s (L1 L2)^T) in the stored out x in layout, W_hat the
// dequantized NF4 weight (or the protected bf16 one). The rank-r product is summed in
// fp64 (the products of bf16 values are exact there, and so are the sums for weights
// and adapters of ordinary ranges) and rounded to bf16 once.
//
// Tiles of 128 x 64 (rows n, columns k; each tile row is one NF4 block); thread
// (tn, tk) = (tid / 8, tid % 8) owns rows 4 tn .. 4 tn + 3 and columns 8 tk .. 8 tk + 7,
// so the 8 lanes of a block are 8 consecutive lanes of one warp. The adapter slices
// of a tile go through shared memory 16 ranks at a time, as fp64: L1 as [q][k], L2
// as [q][n]. Per rank a thread reads its 8 L1 values as four 16-byte pieces and its
// 4 L2 values as two; the pieces of each 8-column group are stored rotated by
// (group / 2) so that the 8 groups a warp reads at once sit in 8 different 16-byte
// bank groups (no conflicts), and the 4 row groups of a warp read 64 contiguous
// bytes. 32 fp64 FMAs per 6 shared loads.
//
// Persistent: two CTAs per SM walk the work items (tile, 16-rank chunk) of their
// tiles. While item i is converted to fp64, summed and (after a tile's last chunk)
// written out, the raw bf16 adapter slices of item i + 1 and, at a tile's first
// chunk, the tile's weight rows (32 code bytes or 128 bf16 bytes per row) arrive by
// cp.async in the other buffer. Buffer reuse is ordered by the two barriers of each
// item: staging buffer (i + 1) % 2 was last read by the conversion of item i - 1,
// and weight slot j % 2 (j = the CTA's tile count) by the epilogue of tile j - 2;
// both precede the first barrier of item i, after which the copies are issued.
// Block scales are read into registers at a tile's first chunk and used in its
// epilogue.
//
// QUANT epilogue: the merged block is NF4-quantized in place of the bf16 store, with
// the quantizer's rule (absmax over the block's 64 merged bf16 values by shuffles
// among its 8 lanes; the code the IEEE quotient selects, found as the quantizer finds
// it; element 2k in the high nibble of byte k); codes always use the exact fp32
// absmax, which goes to `q_absmax` for the double-quant pass.
constexpr int kMergeRows = 128, kMergeCols = 64, kMergeQ = 16;
constexpr int kMergeStageBytes = kMergeCols * kMergeQ * 2 + kMergeQ * kMergeRows * 2;   // raw L1 + L2 chunk
template <bool BF16W>
__host__ __device__ constexpr int merge_w_bytes() { return kMergeRows * (BF16W ? kMergeCols * 2 : kMergeCols / 2); }
template <bool BF16W>
__host__ __device__ constexpr int merge_smem_bytes() {
  return (kMergeQ * kMergeCols + kMergeQ * kMergeRows) * 8 + 2 * kMergeStageBytes + 2 * merge_w_bytes<BF16W>();
}

struct MergeArgs {
  const uint8_t* codes;
  const float* absmax;
  const uint8_t* absmax_q;
  const float* absmax2;
  int dq;
  const uint16_t* Wbf;        // protected bf16 weight, or null
  int64_t out, in;
  const uint16_t* L1;         // in x r
  const uint16_t* L2;         // r x out
  int r;
  double s;
  uint16_t* W_out;            // bf16 out x in (bf16 epilogue)
  uint8_t* q_codes;           // NF4 codes out (QUANT epilogue)
  float* q_absmax;            // fp32 absmax out (QUANT epilogue)
  int* status;
};

__device__ __forceinline__ double bf16_to_f64(uint16_t b) { return double(__uint_as_float(uint32_t(b) << 16)); }

// Position of column k of an 8-column group inside its shared-memory row: the four
// 2-column pieces of group g are stored rotated by g / 2.
__device__ __forceinline__ int merge_col_slot(int k) {
  const int g = k >> 3, p = (k >> 1) & 3;
  return (g << 3) | (((p + (g >> 1)) & 3) << 1) | (k & 1);
}

template <bool BF16W, bool QUANT>
__global__ void __launch_bounds__(256, 2) lora_merge_kernel(const __grid_constant__ MergeArgs m) {
  extern __shared__ __align__(16) uint8_t smem[];
  double(*s_a)[kMergeCols] = reinterpret_cast<double(*)[kMergeCols]>(smem);                       // [q][slot(k)]
  double(*s_b)[kMergeRows] = reinterpret_cast<double(*)[kMergeRows]>(smem + kMergeQ * kMergeCols * 8);  // [q][n]
  uint8_t* const stage0 = smem + (kMergeQ * kMergeCols + kMergeQ * kMergeRows) * 8;    // 2 x {L1 [k][16], L2 [16][n]}
  uint8_t* const wbuf0 = stage0 + 2 * kMergeStageBytes;                                // 2 x weight rows
  constexpr int kRowBytes = merge_w_bytes<BF16W>() / kMergeRows;
  pdl_wait();
  pdl_launch();
  const int tid = threadIdx.x, tn = tid >> 3, tk = tid & 7;
  const int r = m.r;
  const int nchunk = (r + kMergeQ - 1) / kMergeQ;
  const int64_t tiles_k = m.in / kMergeCols, tiles_n = (m.out + kMergeRows - 1) / kMergeRows;
  const int64_t my_tiles = (tiles_k * tiles_n - blockIdx.x + gridDim.x - 1) / gridDim.x;
  const int64_t n_items = my_tiles * nchunk;
  // 16-byte copies need 16-byte aligned rows: L1 rows are r bf16 long, L2 rows out bf16
  const bool l1_async = (r % 8) == 0 && (reinterpret_cast<uintptr_t>(m.L1) & 15) == 0;
  const bool l2_async = (m.out % 8) == 0 && (reinterpret_cast<uintptr_t>(m.L2) & 15) == 0;

  // Copies for item `it` into staging buffer it % 2 (and, at a first chunk, the tile's
  // weight rows into slot (it / nchunk) % 2); one commit group per item.
  auto issue = [&](int64_t it) {
    const int64_t j = it / nchunk;
    const int c = int(it % nchunk);
    const int64_t t = blockIdx.x + j * gridDim.x;
    const int64_t n0 = (t / tiles_k) * kMergeRows, k0 = (t % tiles_k) * kMergeCols;
    const int q0 = c * kMergeQ, qn = min(kMergeQ, r - q0);
    uint8_t* st = stage0 + (it & 1) * kMergeStageBytes;
    uint16_t* st_l1 = reinterpret_cast<uint16_t*>(st);                       // [k][16]
    uint16_t* st_l2 = reinterpret_cast<uint16_t*>(st + kMergeCols * kMergeQ * 2);   // [16][n]
    if (l1_async) {
      // row k: qn ranks = qn / 8 pieces of 16 bytes
      const int pieces = qn / 8;
      for (int i = tid; i < kMergeCols * pieces; i += 256) {
        const int k = i / pieces, pc = i % pieces;
        cp_async16(smem_u32(st_l1 + k * kMergeQ + pc * 8), m.L1 + (k0 + k) * r + q0 + pc * 8);
      }
    } else {
      for (int i = tid; i < kMergeCols * kMergeQ; i += 256) {
        const int k = i >> 4, q = i & 15;
        if (q < qn) st_l1[k * kMergeQ + q] = m.L1[(k0 + k) * r + q0 + q];
      }
    }
    const int64_t ncols = min(int64_t(kMergeRows), m.out - n0);
    if (l2_async) {
      const int pieces = int(ncols / 8);                                      // per L2 row
      for (int i = tid; i < qn * pieces; i += 256) {
        const int q = i / pieces, pc = i % pieces;
        cp_async16(smem_u32(st_l2 + q * kMergeRows + pc * 8), m.L2 + int64_t(q0 + q) * m.out + n0 + pc * 8);
      }
    } else {
      for (int i = tid; i < kMergeQ * kMergeRows; i += 256) {
        const int q = i >> 7, n = i & 127;
        if (q < qn && n < ncols) st_l2[q * kMergeRows + n] = m.L2[int64_t(q0 + q) * m.out + n0 + n];
      }
    }
    if (c == 0) {
      constexpr int kPieces = kRowBytes / 16;   // 16-byte pieces per weight row: 8 (bf16) or 2 (codes)
      uint8_t* wb = wbuf0 + (j & 1) * merge_w_bytes<BF16W>();
      const uint8_t* src = BF16W ? reinterpret_cast<const uint8_t*>(m.Wbf) : m.codes;
#pragma unroll
      for (int u = 0; u < kMergeRows * kPieces / 256; ++u) {
        const int i = tid + 256 * u, row = i / kPieces, piece = i % kPieces;
        if (n0 + row < m.out)
          cp_async16(smem_u32(wb + row * kRowBytes + piece * 16),
                     src + ((n0 + row) * m.in + k0) * kRowBytes / kMergeCols + piece * 16);
      }
    }
    cp_async_commit();
  };

  double acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
  float scale[4] = {0.f, 0.f, 0.f, 0.f};
  bool bad = false;
  if (n_items > 0) issue(0);
  for (int64_t it = 0; it < n_items; ++it) {
    const int64_t j = it / nchunk;
    const int c = int(it % nchunk);
    const int64_t t = blockIdx.x + j * gridDim.x;
    const int64_t n0 = (t / tiles_k) * kMergeRows, k0 = (t % tiles_k) * kMergeCols;
    const int q0 = c * kMergeQ, qn = min(kMergeQ, r - q0);
    cp_async_wait_all();
    __syncthreads();                                           // item it has landed; item it - 1 is done
    if (it + 1 < n_items) issue(it + 1);
    if constexpr (!BF16W) {
      if (c == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int64_t n = n0 + 4 * tn + i;
          scale[i] = n < m.out ? block_scale((n * m.in + k0) / kBlock, m.absmax, m.absmax_q, m.absmax2, m.dq != 0)
                               : 0.f;
        }
      }
    }
    {
      const uint8_t* st = stage0 + (it & 1) * kMergeStageBytes;
      const uint16_t* st_l1 = reinterpret_cast<const uint16_t*>(st);
      const uint16_t* st_l2 = reinterpret_cast<const uint16_t*>(st + kMergeCols * kMergeQ * 2);
      const int64_t ncols = min(int64_t(kMergeRows), m.out - n0);
#pragma unroll
      for (int u = 0; u < kMergeQ * kMergeCols / 256; ++u) {
        const int i = tid + 256 * u, q = i >> 6, k = i & 63;
        s_a[q][merge_col_slot(k)] = (q < qn) ? bf16_to_f64(st_l1[k * kMergeQ + q]) : 0.0;
      }
#pragma unroll
      for (int u = 0; u < kMergeQ * kMergeRows / 256; ++u) {
        const int i = tid + 256 * u, q = i >> 7, n = i & 127;
        s_b[q][n] = (q < qn && n < ncols) ? bf16_to_f64(st_l2[q * kMergeRows + n]) : 0.0;
      }
    }
    __syncthreads();                                           // fp64 slices ready
    const double2* ra = reinterpret_cast<const double2*>(&s_a[0][8 * tk]);
    const double2* rb = reinterpret_cast<const double2*>(&s_b[0][4 * tn]);
    const int rot = tk >> 1;
    auto rank_step = [&](int q) {
      double a[8];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const double2 v = ra[q * (kMergeCols / 2) + ((p + rot) & 3)];
        a[2 * p] = v.x;
        a[2 * p + 1] = v.y;
      }
      const double2 b01 = rb[q * (kMergeRows / 2)], b23 = rb[q * (kMergeRows / 2) + 1];
      const double b[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) acc[i][jj] = fma(a[jj], b[i], acc[i][jj]);
    };
    if (qn == kMergeQ) {   // a full chunk, unrolled so that the next rank's loads overlap this rank's FMAs
#pragma unroll
      for (int q = 0; q < kMergeQ; ++q) rank_step(q);
    } else {
      for (int q = 0; q < qn; ++q) rank_step(q);
    }
    if (c != nchunk - 1) continue;
    // ---- epilogue of tile t: its weight rows are in slot j % 2
    const uint8_t* wb = wbuf0 + (j & 1) * merge_w_bytes<BF16W>();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = 4 * tn + i;
      const int64_t n = n0 + row;
      const bool live = n < m.out;                              // same for the 8 lanes of a block
      const int64_t e = n * m.in + k0 + 8 * tk;                 // first of this thread's 8 elements
      uint4 wv = make_uint4(0u, 0u, 0u, 0u);
      if (live) {
        if constexpr (BF16W) {
          wv = *reinterpret_cast<const uint4*>(wb + row * kRowBytes + 16 * tk);
        } else {
          wv = nf4_dequant_word(*reinterpret_cast<const uint32_t*>(wb + row * kRowBytes + 4 * tk),
                                nf4_make_lut(scale[i]));
        }
      }
      const uint32_t wh[4] = {wv.x, wv.y, wv.z, wv.w};
      uint32_t o[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        uint16_t lo, hi;
        const double v0 = double(__uint_as_float(wh[p] << 16)) + m.s * acc[i][2 * p];
        const double v1 = double(__uint_as_float(wh[p] & 0xFFFF0000u)) + m.s * acc[i][2 * p + 1];
        asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(lo) : "d"(v0));
        asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(hi) : "d"(v1));
        o[p] = live ? (uint32_t(lo) | (uint32_t(hi) << 16)) : 0u;
        acc[i][2 * p] = 0.0;
        acc[i][2 * p + 1] = 0.0;
      }
      if constexpr (!QUANT) {
        if (live) *reinterpret_cast<uint4*>(m.W_out + e) = make_uint4(o[0], o[1], o[2], o[3]);
      } else {
        float w[8];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          w[2 * p] = bf16_lo(o[p]);
          w[2 * p + 1] = bf16_hi(o[p]);
        }
        float am = 0.f;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const float aw = fabsf(w[jj]);
          bad |= !(aw <= FLT_MAX);
          am = fmaxf(am, aw);
        }
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
        // the quantizer's code lookup (cell of the one-multiply quotient, then two lane
        // table shuffles); every lane runs it, for a dead row too
        const bool use = am > 0.f && am <= FLT_MAX;
        uint32_t x[8];
        piece_index_bits(o, CellScale(use ? am : 1.f), lane_tables(tid & 31), x);
        if (live) {
          const uint32_t word = use ? pack_code_word(x) : 0x77777777u;
          *reinterpret_cast<uint32_t*>(m.q_codes + e / 2) = word;
          if (tk == 0) m.q_absmax[e / kBlock] = am;
        }
      }
    }
  }
  if constexpr (QUANT) {
    if (bad) set_status(m.status, QLORA_ERR_NONFINITE);
  }
}

// Double quantization of a finished absmax array: one CTA of 256 threads per group
// of 256 scales, the same arithmetic as the quantizer's own double-quant tail.
__global__ void __launch_bounds__(256) dq_scales_kernel(const float* __restrict__ absmax, int64_t nb,
                                                        uint8_t* __restrict__ absmax_q,
                                                        float* __restrict__ absmax2) {
  __shared__ float s_amax[kDQBlock];
  __shared__ float s_red[8];
  pdl_wait();
  pdl_launch();
  const int64_t g = blockIdx.x;
  const int64_t b = g * kDQBlock + threadIdx.x;
  s_amax[threadIdx.x] = b < nb ? absmax[b] : 0.f;
  dq_group(s_amax, s_red, nb, g, absmax_q, absmax2);
}

template <bool BF16W, bool QUANT>
static cudaError_t launch_merge_cfg(const MergeArgs& m, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    const cudaError_t e = cudaFuncSetAttribute(lora_merge_kernel<BF16W, QUANT>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, merge_smem_bytes<BF16W>());
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int64_t tiles = (m.in / kMergeCols) * ((m.out + kMergeRows - 1) / kMergeRows);
  const int grid = int(std::max<int64_t>(1, std::min<int64_t>(tiles, int64_t(num_sms()) * 2)));
  return launch_pdl(lora_merge_kernel<BF16W, QUANT>, dim3(unsigned(grid)), dim3(256), merge_smem_bytes<BF16W>(), st, m);
}

qlora_status launch_lora_merge(const uint8_t* codes, const float* absmax, const uint8_t* absmax_q,
                               const float* absmax2, bool dq, const uint16_t* Wbf, int64_t out, int64_t in,
                               const uint16_t* L1, const uint16_t* L2, int r, double s, uint16_t* W_out,
                               uint8_t* q_codes, float* q_absmax, int* status, cudaStream_t st) {
  const MergeArgs m{codes, absmax, absmax_q, absmax2, dq ? 1 : 0, Wbf, out, in, L1, L2, r, s, W_out,
                    q_codes, q_absmax, status};
  const bool quant = q_codes != nullptr;
  cudaError_t e;
  if (Wbf)
    e = quant ? launch_merge_cfg<true, true>(m, st) : launch_merge_cfg<true, false>(m, st);
  else
    e = quant ? launch_merge_cfg<false, true>(m, st) : launch_merge_cfg<false, false>(m, st);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status launch_dq_scales(const float* absmax, int64_t nb, uint8_t* absmax_q, float* absmax2, cudaStream_t st) {
  const int64_t groups = (nb + kDQBlock - 1) / kDQBlock;
  if (groups <= 0) return QLORA_OK;
  const cudaError_t e = launch_pdl(dq_scales_kernel, dim3(unsigned(groups)), dim3(256), 0, st, absmax, nb, absmax_q,
                                   absmax2);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? QLORA_OK : QLORA_ERR_CUDA;
}

// ------------------------------------------------- residual NF4 second stage
//
// A protected layer may be stored as two NF4 stages instead of bf16: the second
// quantizes what the first missed, R = fp32_rn(w - fp32_rn(c1 a1)), with the fp32
// quantizer; the GEMM then consumes bf16_rn(fp32_rn(v1 + v2)), vi = fp32_rn(ci ai).
// Both kernels: one thread per 8 elements (one code word), grid-stride, the 16 code
// values in shared memory; numel % 64 == 0.
struct NF4Stage {
  const uint8_t* codes;
  const float* absmax;
  const uint8_t* absmax_q;
  const float* absmax2;
  int dq;
};

__global__ void __launch_bounds__(256) nf4_residual_kernel(const uint16_t* __restrict__ W, const NF4Stage s1,
                                                           int64_t numel, float* __restrict__ R) {
  __shared__ float s_code[16];
  pdl_wait();
  pdl_launch();
  if (threadIdx.x < 16) s_code[threadIdx.x] = nf4_code(int(threadIdx.x));
  __syncthreads();
  const int64_t units = numel / 8;
  for (int64_t u = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; u < units; u += int64_t(gridDim.x) * blockDim.x) {
    const int64_t e = u * 8;
    const float a = block_scale(e / kBlock, s1.absmax, s1.absmax_q, s1.absmax2, s1.dq != 0);
    const uint32_t cw = *reinterpret_cast<const uint32_t*>(s1.codes + e / 2);
    const uint4 wv = *reinterpret_cast<const uint4*>(W + e);
    const uint32_t wh[4] = {wv.x, wv.y, wv.z, wv.w};
    float r[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {   // byte k: element 2k in the high nibble
      const uint32_t b = (cw >> (8 * k)) & 0xFFu;
      r[2 * k] = __fsub_rn(bf16_lo(wh[k]), __fmul_rn(s_code[b >> 4], a));
      r[2 * k + 1] = __fsub_rn(bf16_hi(wh[k]), __fmul_rn(s_code[b & 15u], a));
    }
    float4* dst = reinterpret_cast<float4*>(R + e);
    dst[0] = make_float4(r[0], r[1], r[2], r[3]);
    dst[1] = make_float4(r[4], r[5], r[6], r[7]);
  }
}

__global__ void __launch_bounds__(256) nf4_dequantize2_kernel(const NF4Stage s1, const NF4Stage s2, int64_t numel,
                                                              uint16_t* __restrict__ out) {
  __shared__ float s_code[16];
  pdl_wait();
  pdl_launch();
  if (threadIdx.x < 16) s_code[threadIdx.x] = nf4_code(int(threadIdx.x));
  __syncthreads();
  const int64_t units = numel / 8;
  for (int64_t u = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; u < units; u += int64_t(gridDim.x) * blockDim.x) {
    const int64_t e = u * 8;
    const float a1 = block_scale(e / kBlock, s1.absmax, s1.absmax_q, s1.absmax2, s1.dq != 0);
    const float a2 = block_scale(e / kBlock, s2.absmax, s2.absmax_q, s2.absmax2, s2.dq != 0);
    const uint32_t c1 = *reinterpret_cast<const uint32_t*>(s1.codes + e / 2);
    const uint32_t c2 = *reinterpret_cast<const uint32_t*>(s2.codes + e / 2);
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t b1 = (c1 >> (8 * k)) & 0xFFu, b2 = (c2 >> (8 * k)) & 0xFFu;
      const float even = __fadd_rn(__fmul_rn(s_code[b1 >> 4], a1), __fmul_rn(s_code[b2 >> 4], a2));
      const float odd = __fadd_rn(__fmul_rn(s_code[b1 & 15u], a1), __fmul_rn(s_code[b2 & 15u], a2));
      o[k] = pack_bf16x2(even, odd);
    }
    *reinterpret_cast<uint4*>(out + e) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

qlora_status launch_nf4_residual(const uint16_t* W, const uint8_t* codes, const float* absmax,
                                 const uint8_t* absmax_q, const float* absmax2, bool dq, int64_t numel, float* R,
                                 cudaStream_t st) {
  const NF4Stage s1{codes, absmax, absmax_q, absmax2, dq ? 1 : 0};
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((numel / 8 + 255) / 256, int64_t(num_sms()) * 8));
  const cudaError_t e = launch_pdl(nf4_residual_kernel, dim3(unsigned(blocks)), dim3(256), 0, st, W, s1, numel, R);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status launch_dequantize_two_stage(const uint8_t* codes1, const float* absmax1, const uint8_t* absmax_q1,
                                         const float* absmax2_1, bool dq1, const uint8_t* codes2,
                                         const float* absmax_2, const uint8_t* absmax_q2, const float* absmax2_2,
                                         bool dq2, int64_t numel, uint16_t* out, cudaStream_t st) {
  const NF4Stage s1{codes1, absmax1, absmax_q1, absmax2_1, dq1 ? 1 : 0};
  const NF4Stage s2{codes2, absmax_2, absmax_q2, absmax2_2, dq2 ? 1 : 0};
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((numel / 8 + 255) / 256, int64_t(num_sms()) * 8));
  const cudaError_t e =
      launch_pdl(nf4_dequantize2_kernel, dim3(unsigned(blocks)), dim3(256), 0, st, s1, s2, numel, out);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? QLORA_OK : QLORA_ERR_CUDA;
}

// ------------------------------------------------------- expanded GEMM scales

__global__ void expand_scales_kernel(const float* __restrict__ absmax, const uint8_t* __restrict__ absmax_q,
                                     const float* __restrict__ absmax2, int dq, int64_t out, int64_t nbr,
                                     float* __restrict__ scales_t) {
  // scales_t[kb][o] = scale of block (o, kb)
  __shared__ float tile[32][33];
  pdl_wait();
  pdl_launch();
  const int64_t o0 = int64_t(blockIdx.x) * 32, k0 = int64_t(blockIdx.y) * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  for (int j = ty; j < 32; j += 8) {
    const int64_t o = o0 + j, kb = k0 + tx;
    float v = 0.f;
    if (o < out && kb < nbr) v = block_scale(o * nbr + kb, absmax, absmax_q, absmax2, dq != 0);
    tile[j][tx] = v;
  }
  __syncthreads();
  for (int j = ty; j < 32; j += 8) {
    const int64_t kb = k0 + j, o = o0 + tx;
    if (o < out && kb < nbr) scales_t[kb * out + o] = tile[tx][j];
  }
}

qlora_status launch_expand_scales(const uint8_t*, const float* absmax, const uint8_t* absmax_q,
                                  const float* absmax2, bool dq, int64_t out, int64_t in, float* scales_t,
                                  cudaStream_t s) {
  const int64_t nbr = in / kBlock;
  dim3 grid(unsigned((out + 31) / 32), unsigned((nbr + 31) / 32));
  launch_pdl(expand_scales_kernel, grid, dim3(32, 8), 0, s, absmax, absmax_q, absmax2, dq ? 1 : 0, out, nbr, scales_t);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// ---------------------------------------------------------- LoRA prep / reduce

__global__ void scale_lora_kernel(const uint16_t* __restrict__ src, int64_t rows, int64_t cols, float scale,
                                  int transpose, uint16_t* __restrict__ dst) {
  pdl_wait();
  pdl_launch();
  const int64_t n = rows * cols;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    // non-transposed: dst[i] = s*src[i]; transposed: src is rows x cols, dst is cols x rows
    int64_t d = i;
    if (transpose) {
      const int64_t rr = i / cols, cc = i % cols;
      d = cc * rows + rr;
    }
    const float v = __fmul_rn(__uint_as_float(uint32_t(src[i]) << 16), scale);
    __nv_bfloat16 h = __float2bfloat16_rn(v);
    dst[d] = *reinterpret_cast<uint16_t*>(&h);
  }
}

qlora_status launch_scale_lora(const uint16_t* src, int64_t rows, int64_t cols, float scale, bool transpose,
                               uint16_t* dst, cudaStream_t s) {
  const int64_t n = rows * cols;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 4096);
  launch_pdl(scale_lora_kernel, dim3(unsigned(blocks)), dim3(256), 0, s, src, rows, cols, scale, transpose ? 1 : 0, dst);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qlb
