// AQLoRA allocation pass on the GPU: per-layer NF4 reconstruction error
// (relative Frobenius norm), then ranking and the top-K keep mask.
//
// Pass 1: one CTA per chunk of 256 blocks (16384 elements) of some layer;
//         quantizes, dequantizes and accumulates sum (w - w_hat)^2 and sum w^2
//         in fp64; writes one partial pair per chunk.
// Pass 2: per layer, sums its chunk partials in chunk order -> err.
// Pass 3: one CTA ranks all layers by (err desc, id asc).
// The workspace entry point runs all three in one launch (the last chunk CTA of a
// layer does pass 2 for it, the last layer's finisher does pass 3); the
// allocation-free entry point, which has no counters, launches them separately.
#include <cfloat>
#include <cuda_bf16.h>

#include <mutex>

#include "internal.cuh"
#include "nf4_device.cuh"
#include "ptx.cuh"

namespace qlb {

constexpr int kMaxLayers = 1024;

struct LayerTable {
  static constexpr bool kWrite = false;
  const uint16_t* ptr[kMaxLayers];
  int64_t numel[kMaxLayers];
  int32_t first_chunk[kMaxLayers + 1];
  int32_t n_layers;
};

// The fused pass also writes every layer's NF4 storage; its table (a by-value
// kernel parameter, at most 32 KB) holds fewer layers.
constexpr int kMaxFusedLayers = 512;
struct FusedTable {
  static constexpr bool kWrite = true;
  const uint16_t* ptr[kMaxFusedLayers];
  int64_t numel[kMaxFusedLayers];
  uint8_t* codes[kMaxFusedLayers];
  float* absmax[kMaxFusedLayers];       // may be null with double quant
  uint8_t* absmax_q[kMaxFusedLayers];   // double quant only
  float* absmax2[kMaxFusedLayers];      // double quant only
  int32_t first_chunk[kMaxFusedLayers + 1];
  int32_t n_layers;
};
static_assert(sizeof(FusedTable) <= 32000, "kernel parameter limit");

// Error contribution of 16 bf16 weights (8 packed pairs) of one block: codes
// from the exact absmax a (same arithmetic as the quantizer), reconstruction
// w_hat = bf16(fp32(code * ahat)) with ahat = a, or the double-quantized scale.
// Squares are summed per pair lane in fp32 (8 terms) before the fp64 total.
// With kCodes, also the 16 codes in storage order (byte k = idx[2k] << 4 |
// idx[2k + 1]): idx = base + sat(n 2^100 + T) from the quantizer's {T, base}
// table (tbl_base), the four indices of a 16-bit half accumulated as fp32
// nibble weights.
template <bool kTiny, bool kCodes>
__device__ __forceinline__ void err16_core(const uint32_t (&u)[8], float a, float ahat, uint32_t tbl,
                                           uint32_t tbl_base, double& sd, double& sw, uint2& codes) {
  float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  // tiny blocks: the division operands are rescaled by 2^64 (exact) so 1/a stays normal
  const float as = kTiny ? a * 0x1p64f : a;
  const uint64_t r2 = f2_splat(__frcp_rn(as)), na2 = f2_splat(-as), ah2 = f2_splat(ahat);
  uint64_t sd2 = 0, sw2 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint64_t w = f2_from_bf16x2(u[i]);
    const uint64_t q = f2_div_by_recip(kTiny ? f2_mul(w, f2_splat(0x1p64f)) : w, na2, r2);
    // cell entries {code[base], code[base + 1] - code[base]}; RN(2 lo + diff) is twice
    // the cell's midpoint, so s = sat(n 2^100 - RN(2 lo + diff) 2^99) tests n > m
    const uint64_t cells = coarse_cells2(q);
    const uint64_t n2 = f2_mul(q, 0x7180000071800000ull);   // n * 2^100, both lanes
    const float2 e0 = lds_f2(coarse_addr_bits<8>(uint32_t(cells), tbl));
    const float2 e1 = lds_f2(coarse_addr_bits<8>(uint32_t(cells >> 32), tbl));
    const float s0 = sat_fma(__fmaf_rn(e0.x, 2.f, e0.y), -0x1p99f, f2_lo(n2));
    const float s1 = sat_fma(__fmaf_rn(e1.x, 2.f, e1.y), -0x1p99f, f2_hi(n2));
    const float c0 = __fmaf_rn(s0, e0.y, e0.x);   // code value (exact)
    const float c1 = __fmaf_rn(s1, e1.y, e1.x);
    if constexpr (kCodes) {
      // the index needs the midpoint test of the quantizer's table: in a cell
      // without a midpoint s above may be 1 (harmless for the value, not for idx)
      const float2 t0 = lds_f2(coarse_addr_bits<8>(uint32_t(cells), tbl_base));
      const float2 t1 = lds_f2(coarse_addr_bits<8>(uint32_t(cells >> 32), tbl_base));
      const float i0 = t0.y + sat_fma(f2_lo(q), 0x1p100f, t0.x);
      const float i1 = t1.y + sat_fma(f2_hi(q), 0x1p100f, t1.x);
      const int h = i >> 2, j = i & 3;
      acc[h][j >> 1] = __fmaf_rn(i0, (j & 1) ? 4096.f : 16.f, acc[h][j >> 1]);
      acc[h][j >> 1] = __fmaf_rn(i1, (j & 1) ? 256.f : 1.f, acc[h][j >> 1]);
    }
    const uint64_t p = f2_mul((uint64_t(__float_as_uint(c1)) << 32) | __float_as_uint(c0), ah2);
    const uint64_t wh = f2_from_bf16x2(pack_bf16x2(f2_lo(p), f2_hi(p)));
    const uint64_t d = f2_sub(w, wh);
    sd2 = f2_fma(d, d, sd2);
    sw2 = f2_fma(w, w, sw2);
  }
  sd += double(f2_lo(sd2)) + double(f2_hi(sd2));
  sw += double(f2_lo(sw2)) + double(f2_hi(sw2));
  if constexpr (kCodes) {
    codes.x = prmt(nibbles_from_f32(acc[0][0]), nibbles_from_f32(acc[0][1]), 0x5410u);
    codes.y = prmt(nibbles_from_f32(acc[1][0]), nibbles_from_f32(acc[1][1]), 0x5410u);
  }
}

template <bool kCodes>
__device__ __forceinline__ void err16_bf16(const uint32_t (&u)[8], float a, float ahat, uint32_t tbl,
                                           uint32_t tbl_base, double& sd, double& sw, uint2& codes) {
  if (!(a > 0.f)) {   // all-zero block: every w and w_hat is 0, every code the zero code
    codes = make_uint2(0x77777777u, 0x77777777u);
    return;
  }
  if (a < 0x1p-100f) err16_core<true, kCodes>(u, a, ahat, tbl, tbl_base, sd, sw, codes);
  else err16_core<false, kCodes>(u, a, ahat, tbl, tbl_base, sd, sw, codes);
}

// absmax (bf16 bits) of 16 weights, over the 4 lanes that share the block
__device__ __forceinline__ uint32_t absmax16_lanes(const uint32_t (&u)[8]) {
  uint32_t m = __vmaxu2(u[0] & 0x7FFF7FFFu, u[1] & 0x7FFF7FFFu);
#pragma unroll
  for (int i = 2; i < 8; ++i) m = __vmaxu2(m, u[i] & 0x7FFF7FFFu);
  uint32_t amb = max(m >> 16, m & 0xFFFFu);
  amb = max(amb, __shfl_xor_sync(0xffffffffu, amb, 1));
  amb = max(amb, __shfl_xor_sync(0xffffffffu, amb, 2));
  return amb;
}

__device__ __forceinline__ void finish_layer(const double2* __restrict__ partial, int c0, int c1,
                                             double* __restrict__ err_out);

// Pass 1 (and, with counters, passes 2-3 fused): one CTA per chunk of 256 blocks
// of some layer; in each of 4 passes a thread takes 16 consecutive weights (4
// threads per block). The chunk's (sum d^2, sum w^2) goes to partial[chunk]. With
// counters (zero on entry, left zero): the last chunk CTA of a layer sums that
// layer's partials in chunk order into err[layer], and the last layer to finish
// ranks all layers and writes order / keep.
template <bool DQ, class Tab>
__global__ void __launch_bounds__(256) layer_error_chunk_kernel(const __grid_constant__ Tab tab,
                                                                double2* __restrict__ partial, int* status,
                                                                int* counters, double* __restrict__ err, int K,
                                                                int32_t* __restrict__ order, uint8_t* __restrict__ keep) {
  constexpr bool kW = Tab::kWrite;
  __shared__ __align__(16) float2 s_tbl[33];
  __shared__ __align__(16) float2 s_base[33];
  __shared__ float s_amax[256];
  __shared__ float s_ahat[256];
  __shared__ float s_red[8];
  __shared__ double s_sum[2][8];
  __shared__ int s_flag;
  pdl_wait();
  pdl_launch();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < 33) {
    s_tbl[tid] = make_float2(__uint_as_float(kNF4CoarseD[2 * tid]), __uint_as_float(kNF4CoarseD[2 * tid + 1]));
    if constexpr (kW)
      s_base[tid] = make_float2(__uint_as_float(kNF4CoarseQ[2 * tid]), __uint_as_float(kNF4CoarseQ[2 * tid + 1]));
  }
  const uint32_t tbl = static_cast<uint32_t>(__cvta_generic_to_shared(s_tbl));
  const uint32_t tbl_base = static_cast<uint32_t>(__cvta_generic_to_shared(s_base));
  const int chunk = blockIdx.x;
  int lo = 0, hi = tab.n_layers - 1;  // layer owning this chunk
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab.first_chunk[mid] <= chunk) lo = mid; else hi = mid - 1;
  }
  const int layer = lo;
  const uint16_t* W = tab.ptr[layer];
  const int64_t nb = tab.numel[layer] / kBlock;
  const int64_t g = chunk - tab.first_chunk[layer];
  // task k of this thread: weights [16 (tid & 3), +16) of block 64 k + tid / 4
  auto load_task = [&](int k, uint32_t (&u)[8]) {
    const int64_t blk = g * kDQBlock + ((k * 256 + tid) >> 2);
    const uint16_t* src = W + blk * kBlock + (tid & 3) * 16;
    const uint4 z = make_uint4(0, 0, 0, 0);
    const uint4 v0 = (blk < nb) ? __ldg(reinterpret_cast<const uint4*>(src)) : z;
    const uint4 v1 = (blk < nb) ? __ldg(reinterpret_cast<const uint4*>(src + 8)) : z;
    u[0] = v0.x; u[1] = v0.y; u[2] = v0.z; u[3] = v0.w; u[4] = v1.x; u[5] = v1.y; u[6] = v1.z; u[7] = v1.w;
  };
  __syncthreads();   // the table is in place
  uint32_t bad = 0;
  double sd = 0.0, sw = 0.0;
  float am_k[4];
  uint32_t cur[8], nxt[8];
  load_task(0, cur);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (k < 3) load_task(k + 1, nxt);
    const uint32_t amb = absmax16_lanes(cur);
    bad |= amb >= 0x7F80u;
    const float am = __uint_as_float(amb << 16);
    am_k[k] = am;
    const int64_t blk = g * kDQBlock + ((k * 256 + tid) >> 2);
    if constexpr (DQ) {
      if ((tid & 3) == 0) s_amax[(k * 256 + tid) >> 2] = am;
      if constexpr (kW) {
        if ((tid & 3) == 0 && blk < nb && tab.absmax[layer] != nullptr) tab.absmax[layer][blk] = am;
      }
    } else {
      uint2 cw;
      err16_bf16<kW>(cur, am, am, tbl, tbl_base, sd, sw, cw);
      if constexpr (kW) {
        if (blk < nb) {
          if ((tid & 3) == 0) tab.absmax[layer][blk] = am;
          *reinterpret_cast<uint2*>(tab.codes[layer] + blk * (kBlock / 2) + (tid & 3) * 8) = cw;
        }
      }
    }
    if (k < 3) {
#pragma unroll
      for (int i = 0; i < 8; ++i) cur[i] = nxt[i];
    }
  }
  if (bad && status) set_status(status, QLORA_ERR_NONFINITE);
  if constexpr (DQ) {
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
    float ah = 0.f;
    if (G > 0.f && tid < nblk_g) {
      const float inv = __fdiv_rn(448.f, G);
      const uint8_t q = f32_to_e4m3_satfinite(__fmul_rn(s_amax[tid], inv));
      ah = __fmul_rn(e4m3_to_f32(q), __fdiv_rn(G, 448.f));
    }
    s_ahat[tid] = ah;
    if constexpr (kW) {
      if (tid < nblk_g) tab.absmax_q[layer][g * kDQBlock + tid] =
          (G > 0.f) ? f32_to_e4m3_satfinite(__fmul_rn(s_amax[tid], __fdiv_rn(448.f, G))) : uint8_t(0);
      if (tid == 0) tab.absmax2[layer][g] = (G > 0.f) ? __fdiv_rn(G, 448.f) : 0.f;
    }
    __syncthreads();
    // second pass over the chunk (from L2): codes use the exact absmax, the
    // reconstruction the double-quantized scale
    load_task(0, cur);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (k < 3) load_task(k + 1, nxt);
      uint2 cw;
      err16_bf16<kW>(cur, am_k[k], s_ahat[(k * 256 + tid) >> 2], tbl, tbl_base, sd, sw, cw);
      if constexpr (kW) {
        const int64_t blk = g * kDQBlock + ((k * 256 + tid) >> 2);
        if (blk < nb) *reinterpret_cast<uint2*>(tab.codes[layer] + blk * (kBlock / 2) + (tid & 3) * 8) = cw;
      }
      if (k < 3) {
#pragma unroll
        for (int i = 0; i < 8; ++i) cur[i] = nxt[i];
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sd += __shfl_xor_sync(0xffffffffu, sd, o);
    sw += __shfl_xor_sync(0xffffffffu, sw, o);
  }
  if (lane == 0) { s_sum[0][warp] = sd; s_sum[1][warp] = sw; }
  __syncthreads();
  if (tid == 0) {
    double a = 0.0, b = 0.0;
    for (int i = 0; i < 8; ++i) { a += s_sum[0][i]; b += s_sum[1][i]; }
    partial[chunk] = make_double2(a, b);
  }
  if (counters == nullptr) return;
  // ---- fused finish: last chunk of the layer -> err[layer]; last layer -> ranks
  if (tid == 0) {
    __threadfence();
    const int nchunks = tab.first_chunk[layer + 1] - tab.first_chunk[layer];
    const int done = atomicAdd(counters + 1 + layer, 1);
    s_flag = (done == nchunks - 1);
    if (s_flag) atomicExch(counters + 1 + layer, 0);
  }
  __syncthreads();
  if (!s_flag) return;
  __threadfence();
  finish_layer(partial, tab.first_chunk[layer], tab.first_chunk[layer + 1], err + layer);
  if (tid == 0) {
    __threadfence();
    const int done = atomicAdd(counters, 1);
    s_flag = (done == tab.n_layers - 1);
    if (s_flag) atomicExch(counters, 0);
  }
  __syncthreads();
  if (!s_flag) return;
  __threadfence();
  const int n = tab.n_layers;
  for (int l = tid; l < n; l += 256) {
    const double e = __ldcg(err + l);
    int rank = 0;
    for (int j = 0; j < n; ++j) {
      const double f = __ldcg(err + j);
      rank += (f > e || (f == e && j < l)) ? 1 : 0;
    }
    order[rank] = l;
    keep[l] = rank < K ? 1 : 0;
  }
}

// One CTA per layer: thread t sums chunks first+t, first+t+256, ... in order, then a
// fixed-shape tree combines the 256 partials -- deterministic for a given layout.
__device__ __forceinline__ void finish_layer(const double2* __restrict__ partial, int c0, int c1,
                                             double* __restrict__ err_out) {
  __shared__ double s_a[256], s_b[256];
  double a = 0.0, b = 0.0;
  for (int c = c0 + threadIdx.x; c < c1; c += 256) {
    const double2 v = __ldcg(partial + c);
    a += v.x;
    b += v.y;
  }
  s_a[threadIdx.x] = a;
  s_b[threadIdx.x] = b;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) { s_a[threadIdx.x] += s_a[threadIdx.x + o]; s_b[threadIdx.x] += s_b[threadIdx.x + o]; }
    __syncthreads();
  }
  if (threadIdx.x == 0) *err_out = (s_b[0] > 0.0) ? sqrt(s_a[0] / s_b[0]) : 0.0;
}

__global__ void __launch_bounds__(1024) rank_topk_kernel(const double* __restrict__ err, int n_layers, int K,
                                                         int32_t* __restrict__ order, uint8_t* __restrict__ keep) {
  __shared__ double s_err[kMaxLayers];
  for (int i = threadIdx.x; i < n_layers; i += blockDim.x) s_err[i] = err[i];
  __syncthreads();
  for (int l = threadIdx.x; l < n_layers; l += blockDim.x) {
    const double e = s_err[l];
    int rank = 0;
    for (int j = 0; j < n_layers; ++j) {
      const double f = s_err[j];
      rank += (f > e || (f == e && j < l)) ? 1 : 0;
    }
    order[rank] = l;
    keep[l] = rank < K ? 1 : 0;
  }
}

__global__ void __launch_bounds__(256) layer_error_finish_table_kernel(const double2* __restrict__ partial,
                                                                       const __grid_constant__ LayerTable tab,
                                                                       double* __restrict__ err);

static int32_t chunks_of(int64_t numel) {
  const int64_t nb = numel / kBlock;
  return static_cast<int32_t>((nb + kDQBlock - 1) / kDQBlock);
}

size_t layer_error_ws_bytes(int n_layers, const int64_t* numel) {
  int64_t chunks = 0;
  for (int i = 0; i < n_layers; ++i) chunks += chunks_of(numel[i]);
  return kReservedBytes + size_t(chunks) * sizeof(double2);
}

qlora_status launch_layer_error_rank(int n_layers, const uint16_t* const* W_ptrs, const int64_t* numel, bool dq,
                                     int K, double* err, int32_t* order, uint8_t* keep, void* ws, size_t ws_bytes,
                                     int* status, cudaStream_t s) {
  // The chunk table travels as a by-value kernel parameter (no host-to-device
  // copy), so this call can be captured into a CUDA graph.
  static std::mutex mu;
  static LayerTable tab;
  std::lock_guard<std::mutex> lock(mu);
  tab.n_layers = n_layers;
  int32_t c = 0;
  for (int i = 0; i < n_layers; ++i) {
    tab.ptr[i] = W_ptrs[i];
    tab.numel[i] = numel[i];
    tab.first_chunk[i] = c;
    c += chunks_of(numel[i]);
  }
  tab.first_chunk[n_layers] = c;
  if (layer_error_ws_bytes(n_layers, numel) > ws_bytes) return QLORA_ERR_WORKSPACE;
  double2* partial = reinterpret_cast<double2*>(static_cast<char*>(ws) + kReservedBytes);
  int* counters = reinterpret_cast<int*>(static_cast<char*>(ws) + kStatusBytes);   // 1 + n_layers, zero
  if (dq) launch_pdl(layer_error_chunk_kernel<true, LayerTable>, dim3(unsigned(c)), dim3(256), 0, s, tab, partial, status, counters, err, K, order, keep);
  else launch_pdl(layer_error_chunk_kernel<false, LayerTable>, dim3(unsigned(c)), dim3(256), 0, s, tab, partial, status, counters, err, K, order, keep);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status launch_quantize_error_rank(int n_layers, const uint16_t* const* W_ptrs, const int64_t* numel, bool dq,
                                       int K, uint8_t* const* codes, float* const* absmax, uint8_t* const* absmax_q,
                                       float* const* absmax2, double* err, int32_t* order, uint8_t* keep, void* ws,
                                       size_t ws_bytes, int* status, cudaStream_t s) {
  if (n_layers > kMaxFusedLayers) return QLORA_ERR_SHAPE;
  static std::mutex mu;
  static FusedTable tab;
  std::lock_guard<std::mutex> lock(mu);
  tab.n_layers = n_layers;
  int32_t c = 0;
  for (int i = 0; i < n_layers; ++i) {
    tab.ptr[i] = W_ptrs[i];
    tab.numel[i] = numel[i];
    tab.codes[i] = codes[i];
    tab.absmax[i] = absmax ? absmax[i] : nullptr;
    tab.absmax_q[i] = dq ? absmax_q[i] : nullptr;
    tab.absmax2[i] = dq ? absmax2[i] : nullptr;
    tab.first_chunk[i] = c;
    c += chunks_of(numel[i]);
  }
  tab.first_chunk[n_layers] = c;
  if (layer_error_ws_bytes(n_layers, numel) > ws_bytes) return QLORA_ERR_WORKSPACE;
  double2* partial = reinterpret_cast<double2*>(static_cast<char*>(ws) + kReservedBytes);
  int* counters = reinterpret_cast<int*>(static_cast<char*>(ws) + kStatusBytes);
  cudaError_t e;
  if (dq)
    e = launch_pdl(layer_error_chunk_kernel<true, FusedTable>, dim3(unsigned(c)), dim3(256), 0, s, tab, partial, status,
                   counters, err, K, order, keep);
  else
    e = launch_pdl(layer_error_chunk_kernel<false, FusedTable>, dim3(unsigned(c)), dim3(256), 0, s, tab, partial,
                   status, counters, err, K, order, keep);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? QLORA_OK : QLORA_ERR_CUDA;
}

// ------------------------------------------------------------------------
// Allocation-free variant.
//
// Same three passes, but the per-chunk partial sums live in a file-scope device
// array instead of a caller workspace, and the chunk table reaches the finish
// pass as a kernel parameter, so a call needs no device memory beyond its
// inputs and outputs. The array is 16 MiB (2^20 chunks of 16384 weights, i.e.
// up to 2^34 weights per call); every GPU that loads the library keeps it
// until the process exits. All calls share it: calls that overlap on the GPU
// (two streams, two host threads) race on it. Each call overwrites every
// partial it reads, so nothing has to be cleared between calls.

constexpr int64_t kNoAllocMaxChunks = int64_t(1) << 20;
static __device__ __align__(256) double2 g_noalloc_partials[kNoAllocMaxChunks];

__global__ void __launch_bounds__(256) layer_error_finish_table_kernel(const double2* __restrict__ partial,
                                                                       const __grid_constant__ LayerTable tab,
                                                                       double* __restrict__ err) {
  const int l = blockIdx.x;
  if (l >= tab.n_layers) return;
  finish_layer(partial, tab.first_chunk[l], tab.first_chunk[l + 1], err + l);
}

namespace {
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoAllocMaxDevices] = {};
LayerTable g_noalloc_tab;  // host staging of the by-value parameter, guarded by g_noalloc_mu
}  // namespace

int64_t noalloc_chunks(int n_layers, const int64_t* numel) {
  int64_t c = 0;
  for (int i = 0; i < n_layers; ++i) c += chunks_of(numel[i]);
  return c;
}

qlora_status launch_layer_error_rank_noalloc(int n_layers, const uint16_t* const* W_ptrs, const int64_t* numel,
                                             bool dq, int K, double* err, int32_t* order, uint8_t* keep,
                                             cudaStream_t s) {
  if (noalloc_chunks(n_layers, numel) > kNoAllocMaxChunks) return QLORA_ERR_SHAPE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return QLORA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    // One-time set-up on this device (the current one): the host-side name of the
    // array is only a stand-in, the kernels need its device address.
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_partials) != cudaSuccess || ptr == nullptr) return QLORA_ERR_CUDA;
    g_noalloc_addr[dev] = ptr;
  }
  double2* partial = static_cast<double2*>(g_noalloc_addr[dev]);
  LayerTable& tab = g_noalloc_tab;
  tab.n_layers = n_layers;
  int32_t c = 0;
  for (int i = 0; i < n_layers; ++i) {
    tab.ptr[i] = W_ptrs[i];
    tab.numel[i] = numel[i];
    tab.first_chunk[i] = c;
    c += chunks_of(numel[i]);
  }
  tab.first_chunk[n_layers] = c;
  if (dq) layer_error_chunk_kernel<true, LayerTable><<<unsigned(c), 256, 0, s>>>(tab, partial, nullptr, nullptr, err, K, order, keep);
  else layer_error_chunk_kernel<false, LayerTable><<<unsigned(c), 256, 0, s>>>(tab, partial, nullptr, nullptr, err, K, order, keep);
  if (cudaGetLastError() != cudaSuccess) return QLORA_ERR_CUDA;
  layer_error_finish_table_kernel<<<n_layers, 256, 0, s>>>(partial, tab, err);
  rank_topk_kernel<<<1, 1024, 0, s>>>(err, n_layers, K, order, keep);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qlb
