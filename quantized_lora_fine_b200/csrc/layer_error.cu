// AQLoRA allocation pass on the GPU: per-layer NF4 reconstruction error
// (relative Frobenius norm), then ranking and the top-K keep mask.
//
// Pass 1: one CTA per chunk of 256 blocks (16384 elements) of some layer;
//         quantizes, dequantizes and accumulates sum (w - w_hat)^2 and sum w^2
//         in fp64; writes one partial pair per chunk (nothing else is written).
// Pass 2: per layer, sums its chunk partials in chunk order -> err.
// Pass 3: one CTA ranks all layers by (err desc, id asc).
#include <cfloat>
#include <cuda_bf16.h>

#include <mutex>

#include "internal.cuh"
#include "nf4_device.cuh"

namespace qlb {

constexpr int kMaxLayers = 1024;

struct LayerTable {
  const uint16_t* ptr[kMaxLayers];
  int64_t numel[kMaxLayers];
  int32_t first_chunk[kMaxLayers + 1];
  int32_t n_layers;
};

// Error contribution of 8 bf16 weights of one block: codes from the exact absmax
// a, reconstruction with ahat (= a, or the double-quantized scale). w and w_hat
// are bf16 values within a small exponent range of each other (or w_hat = 0),
// so d = w - w_hat and the squares d^2, w^2 are exact in fp32; the 8-term
// partial sums carry at most 8 roundings before they are added in fp64.
__device__ __forceinline__ void err8_bf16(uint4 v, float a, float ahat, const NF4CellSmem& cells, const float* s_code,
                                          float& sd8, float& sw8) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  uint32_t idx[8];
  if (a > 0.f) quant8_bf16(v, a, cells, idx);
  else {
#pragma unroll
    for (int i = 0; i < 8; ++i) idx[i] = 7u;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float w = (i & 1) ? __uint_as_float(u[i >> 1] & 0xFFFF0000u) : __uint_as_float(u[i >> 1] << 16);
    const float wh = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s_code[idx[i]], ahat)));
    const float d = __fsub_rn(w, wh);
    sd8 = __fmaf_rn(d, d, sd8);
    sw8 = __fmaf_rn(w, w, sw8);
  }
}

template <bool DQ>
__global__ void __launch_bounds__(256) layer_error_chunk_kernel(const __grid_constant__ LayerTable tab,
                                                                double2* __restrict__ partial, int* status) {
  __shared__ float s_amax[256];
  __shared__ float s_ahat[256];
  __shared__ float s_red[8];
  __shared__ float s_code[16];
  __shared__ double s_sum[2][8];
  __shared__ NF4CellSmem s_cells;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  nf4_cells_load(s_cells, tid);
  if (tid < 16) s_code[tid] = nf4_code(tid);
  const int chunk = blockIdx.x;
  int lo = 0, hi = tab.n_layers - 1;  // layer owning this chunk
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab.first_chunk[mid] <= chunk) lo = mid; else hi = mid - 1;
  }
  const uint16_t* W = tab.ptr[lo];
  const int64_t nb = tab.numel[lo] / kBlock;
  const int64_t g = chunk - tab.first_chunk[lo];
  auto load = [&](int it) -> uint4 {
    const int64_t blk = g * kDQBlock + it * 32 + warp * 4 + (lane >> 3);
    return (blk < nb) ? __ldg(reinterpret_cast<const uint4*>(W + blk * kBlock + (lane & 7) * 8)) : make_uint4(0, 0, 0, 0);
  };
  uint4 raw[8];
#pragma unroll
  for (int it = 0; it < 8; ++it) raw[it] = load(it);
  __syncthreads();
  uint32_t bad = 0;
  double sd = 0.0, sw = 0.0;
  float am_slice[8];
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int bi = it * 32 + warp * 4 + (lane >> 3);
    const uint32_t amb = block_max8_lanes(absmax8_bf16_bits(raw[it]));
    bad |= amb >= 0x7F80u;
    const float am = __uint_as_float(amb << 16);
    am_slice[it] = am;
    if constexpr (DQ) {
      if ((lane & 7) == 0) s_amax[bi] = am;
    } else {
      float sd8 = 0.f, sw8 = 0.f;
      err8_bf16(raw[it], am, am, s_cells, s_code, sd8, sw8);
      sd += double(sd8);
      sw += double(sw8);
    }
  }
  if (bad) set_status(status, QLORA_ERR_NONFINITE);
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
    __syncthreads();
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int bi = it * 32 + warp * 4 + (lane >> 3);
      float sd8 = 0.f, sw8 = 0.f;
      err8_bf16(raw[it], am_slice[it], s_ahat[bi], s_cells, s_code, sd8, sw8);
      sd += double(sd8);
      sw += double(sw8);
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
}

// One CTA per layer: thread t sums chunks first+t, first+t+256, ... in order, then a
// fixed-shape tree combines the 256 partials -- deterministic for a given layout.
__device__ __forceinline__ void finish_layer(const double2* __restrict__ partial, int c0, int c1,
                                             double* __restrict__ err_out) {
  __shared__ double s_a[256], s_b[256];
  double a = 0.0, b = 0.0;
  for (int c = c0 + threadIdx.x; c < c1; c += 256) { a += partial[c].x; b += partial[c].y; }
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
  if (dq) layer_error_chunk_kernel<true><<<unsigned(c), 256, 0, s>>>(tab, partial, status);
  else layer_error_chunk_kernel<false><<<unsigned(c), 256, 0, s>>>(tab, partial, status);
  if (cudaGetLastError() != cudaSuccess) return QLORA_ERR_CUDA;
  layer_error_finish_table_kernel<<<n_layers, 256, 0, s>>>(partial, tab, err);
  rank_topk_kernel<<<1, 1024, 0, s>>>(err, n_layers, K, order, keep);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
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
  if (dq) layer_error_chunk_kernel<true><<<unsigned(c), 256, 0, s>>>(tab, partial, nullptr);
  else layer_error_chunk_kernel<false><<<unsigned(c), 256, 0, s>>>(tab, partial, nullptr);
  if (cudaGetLastError() != cudaSuccess) return QLORA_ERR_CUDA;
  layer_error_finish_table_kernel<<<n_layers, 256, 0, s>>>(partial, tab, err);
  rank_topk_kernel<<<1, 1024, 0, s>>>(err, n_layers, K, order, keep);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qlb
