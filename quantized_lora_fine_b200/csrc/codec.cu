// NF4 quantizer, dequantizer and the small elementwise / reduction kernels of
// the LoRA path. All HBM-bound: 128-bit loads and stores, warp shuffles.
#include <algorithm>
#include <cfloat>
#include <cuda_bf16.h>

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

// bf16 weights. One CTA of 256 threads per group of 256 blocks (16384 elements);
// in each of 4 passes a thread takes 16 consecutive elements (4 threads per block,
// a CTA covers 8 KB contiguous per pass), loading the next pass while it codes the
// current one. Per block: integer absmax on packed bf16 pairs (4-lane shuffle
// max) and one IEEE reciprocal. Per element pair: Markstein division in packed
// fp32 (exact RN(w / a) for bf16 operands); per element the code index comes from
// the 33-cell table on the FMA pipe (cell address by RZ multiply-add, one
// shared-memory load, a saturating FMA for the midpoint test) and is accumulated
// as fp32 nibble weights.
__device__ __forceinline__ void quant_load16(const uint16_t* __restrict__ W, int64_t e, int64_t numel,
                                             uint4 (&r)[2]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t eh = e + 8 * h;
    if (eh + 8 <= numel) {
      r[h] = __ldg(reinterpret_cast<const uint4*>(W + eh));
    } else {
      uint32_t t0 = 0, t1 = 0, t2 = 0, t3 = 0;
      if (eh + 0 < numel) t0 |= uint32_t(W[eh + 0]);
      if (eh + 1 < numel) t0 |= uint32_t(W[eh + 1]) << 16;
      if (eh + 2 < numel) t1 |= uint32_t(W[eh + 2]);
      if (eh + 3 < numel) t1 |= uint32_t(W[eh + 3]) << 16;
      if (eh + 4 < numel) t2 |= uint32_t(W[eh + 4]);
      if (eh + 5 < numel) t2 |= uint32_t(W[eh + 5]) << 16;
      if (eh + 6 < numel) t3 |= uint32_t(W[eh + 6]);
      if (eh + 7 < numel) t3 |= uint32_t(W[eh + 7]) << 16;
      r[h] = make_uint4(t0, t1, t2, t3);
    }
  }
}

// Codes of 16 bf16 weights (8 packed pairs) of a block with absmax am > 0, as two
// words in storage order (byte k = idx[2k] << 4 | idx[2k + 1]).
__device__ __forceinline__ uint2 quant16_bf16(const uint32_t (&u)[8], float am, uint32_t tbl) {
  float a = am;
  uint64_t wp[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) wp[i] = f2_from_bf16x2(u[i]);
  if (am < 0x1p-100f) {   // tiny block: rescale by 2^64 (exact) so that 1/a stays normal
    a = am * 0x1p64f;
    const uint64_t s64 = f2_splat(0x1p64f);
#pragma unroll
    for (int i = 0; i < 8; ++i) wp[i] = f2_mul(wp[i], s64);
  }
  const uint64_t r2 = f2_splat(__frcp_rn(a)), na2 = f2_splat(-a);
  uint32_t word[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    // within a 16-bit half the 4 elements weigh 16, 1, 4096, 256 (storage order)
    float acc[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint64_t q = f2_div_by_recip(wp[4 * h + i], na2, r2);
      const float n0 = f2_lo(q), n1 = f2_hi(q);
      const uint64_t cells = coarse_cells2(q);
      const float2 t0 = lds_f2(coarse_addr_bits<8>(uint32_t(cells), tbl));
      const float2 t1 = lds_f2(coarse_addr_bits<8>(uint32_t(cells >> 32), tbl));
      const float w0 = (i & 1) ? 4096.f : 16.f, w1 = (i & 1) ? 256.f : 1.f;
      acc[i >> 1] = __fmaf_rn(t0.y + sat_fma(n0, 0x1p100f, t0.x), w0, acc[i >> 1]);
      acc[i >> 1] = __fmaf_rn(t1.y + sat_fma(n1, 0x1p100f, t1.x), w1, acc[i >> 1]);
    }
    word[h] = prmt(nibbles_from_f32(acc[0]), nibbles_from_f32(acc[1]), 0x5410u);
  }
  return make_uint2(word[0], word[1]);
}

template <bool DQ>
__global__ void __launch_bounds__(256) nf4_quantize_bf16_kernel(const uint16_t* __restrict__ W, int64_t numel,
                                                                uint8_t* __restrict__ codes,
                                                                float* __restrict__ absmax,
                                                                uint8_t* __restrict__ absmax_q,
                                                                float* __restrict__ absmax2, int* status) {
  __shared__ __align__(16) float2 s_tbl[33];
  __shared__ float s_amax[256];
  __shared__ float s_red[8];
  pdl_wait();
  pdl_launch();
  const int tid = threadIdx.x, lane = tid & 31;
  if (tid < 33) s_tbl[tid] = make_float2(__uint_as_float(kNF4CoarseQ[2 * tid]), __uint_as_float(kNF4CoarseQ[2 * tid + 1]));
  const uint32_t tbl = static_cast<uint32_t>(__cvta_generic_to_shared(s_tbl));
  __syncthreads();
  const int64_t nb = (numel + kBlock - 1) / kBlock;
  const int64_t g = blockIdx.x;
  const int64_t g0 = g * int64_t(kDQBlock * kBlock);   // first element of the group
  uint32_t bad = 0;
  uint4 cur[2], nxt[2];
  quant_load16(W, g0 + int64_t(tid) * 16, numel, cur);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (k < 3) quant_load16(W, g0 + int64_t((k + 1) * 256 + tid) * 16, numel, nxt);
    const int bi = (k * 256 + tid) >> 2;               // block within the group
    const int64_t blk = g * kDQBlock + bi;
    const int64_t e0 = g0 + int64_t(k * 256 + tid) * 16;
    const uint32_t u[8] = {cur[0].x, cur[0].y, cur[0].z, cur[0].w, cur[1].x, cur[1].y, cur[1].z, cur[1].w};
    uint32_t m = __vmaxu2(u[0] & 0x7FFF7FFFu, u[1] & 0x7FFF7FFFu);
#pragma unroll
    for (int i = 2; i < 8; ++i) m = __vmaxu2(m, u[i] & 0x7FFF7FFFu);
    uint32_t amb = max(m >> 16, m & 0xFFFFu);
    amb = max(amb, __shfl_xor_sync(0xffffffffu, amb, 1));
    amb = max(amb, __shfl_xor_sync(0xffffffffu, amb, 2));
    bad |= amb >= 0x7F80u;
    const float am = __uint_as_float(amb << 16);
    if ((lane & 3) == 0) {
      if constexpr (DQ) s_amax[bi] = am;
      if (absmax != nullptr && blk < nb) absmax[blk] = am;
    }
    if (e0 < numel) {
      const uint2 word = (am > 0.f) ? quant16_bf16(u, am, tbl) : make_uint2(0x77777777u, 0x77777777u);
      if (e0 + 16 <= numel) {
        *reinterpret_cast<uint2*>(codes + e0 / 2) = word;
      } else {
        const uint64_t both = (uint64_t(word.y) << 32) | word.x;
        for (int kb = 0; 2 * kb < numel - e0; ++kb) codes[e0 / 2 + kb] = uint8_t(both >> (8 * kb));
      }
    }
    if (k < 3) { cur[0] = nxt[0]; cur[1] = nxt[1]; }
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

qlora_status launch_quantize(const void* W, int w_dtype, int64_t numel, bool dq, uint8_t* codes, float* absmax,
                             uint8_t* absmax_q, float* absmax2, int* status, cudaStream_t s) {
  const int64_t nb = (numel + kBlock - 1) / kBlock;
  const int64_t groups = (nb + kDQBlock - 1) / kDQBlock;
  if (groups <= 0) return QLORA_OK;
  dim3 grid(static_cast<unsigned>(groups));
  if (w_dtype == QLORA_DTYPE_BF16) {
    const uint16_t* Wb = static_cast<const uint16_t*>(W);
    if (dq) launch_pdl(nf4_quantize_bf16_kernel<true>, grid, dim3(256), 0, s, Wb, numel, codes, absmax, absmax_q, absmax2, status);
    else launch_pdl(nf4_quantize_bf16_kernel<false>, grid, dim3(256), 0, s, Wb, numel, codes, absmax, absmax_q, absmax2, status);
  } else {
    if (dq) nf4_quantize_f32_kernel<true><<<grid, 256, 0, s>>>((const float*)W, numel, codes, absmax, absmax_q, absmax2, status);
    else nf4_quantize_f32_kernel<false><<<grid, 256, 0, s>>>((const float*)W, numel, codes, absmax, absmax_q, absmax2, status);
  }
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
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
