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

template <bool DQ>
__global__ void __launch_bounds__(256) layer_error_chunk_kernel(const __grid_constant__ LayerTable tab,
                                                                double2* __restrict__ partial, int* status) {
  __shared__ float s_amax[256];
  __shared__ float s_ahat[256];
  __shared__ float s_red[8];
  __shared__ float s_code[16];
  __shared__ double s_sum[2][8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = blockIdx.x;
  // find the layer owning this chunk
  int lo = 0, hi = tab.n_layers - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab.first_chunk[mid] <= chunk) lo = mid; else hi = mid - 1;
  }
  const int layer = lo;
  const uint16_t* W = tab.ptr[layer];
  const int64_t numel = tab.numel[layer];
  const int64_t g = chunk - tab.first_chunk[layer];
  const int64_t nb = numel / kBlock;
  if (tid < 16) s_code[tid] = nf4_code(tid);

  uint4 raw[8];
  float am_slice[8];
  bool bad = false;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int bi = it * 32 + warp * 4 + (lane >> 3);
    const int64_t blk = g * kDQBlock + bi;
    raw[it] = make_uint4(0, 0, 0, 0);
    if (blk < nb) raw[it] = __ldg(reinterpret_cast<const uint4*>(W + blk * kBlock + (lane & 7) * 8));
    const uint32_t u[4] = {raw[it].x, raw[it].y, raw[it].z, raw[it].w};
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a0 = fabsf(bf16_lo(u[i])), a1 = fabsf(bf16_hi(u[i]));
      bad |= !(a0 <= FLT_MAX) || !(a1 <= FLT_MAX);
      am = fmaxf(am, fmaxf(a0, a1));
    }
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
    am_slice[it] = am;
    if ((lane & 7) == 0) s_amax[bi] = am;
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
  }
  __syncthreads();
  double sd = 0.0, sw = 0.0;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int bi = it * 32 + warp * 4 + (lane >> 3);
    const float a = am_slice[it];
    const float ahat = DQ ? s_ahat[bi] : a;
    const uint32_t u[4] = {raw[it].x, raw[it].y, raw[it].z, raw[it].w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float w = (i & 1) ? bf16_hi(u[i >> 1]) : bf16_lo(u[i >> 1]);
      const uint32_t j = (a > 0.f) ? nf4_index(__fdiv_rn(w, a)) : 7u;
      const float wh = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s_code[j], ahat)));
      const double d = double(w) - double(wh);
      sd = fma(d, d, sd);
      sw = fma(double(w), double(w), sw);
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

__global__ void layer_error_finish_kernel(const double2* __restrict__ partial, const int32_t* __restrict__ first,
                                          int n_layers, double* __restrict__ err) {
  const int l = blockIdx.x * blockDim.x + threadIdx.x;
  if (l >= n_layers) return;
  double sd = 0.0, sw = 0.0;
  for (int c = first[l]; c < first[l + 1]; ++c) { sd += partial[c].x; sw += partial[c].y; }
  err[l] = (sw > 0.0) ? sqrt(sd / sw) : 0.0;
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

static int32_t chunks_of(int64_t numel) {
  const int64_t nb = numel / kBlock;
  return static_cast<int32_t>((nb + kDQBlock - 1) / kDQBlock);
}

size_t layer_error_ws_bytes(int n_layers, const int64_t* numel) {
  int64_t chunks = 0;
  for (int i = 0; i < n_layers; ++i) chunks += chunks_of(numel[i]);
  return kStatusBytes + size_t(chunks) * sizeof(double2) + size_t(n_layers + 1) * sizeof(int32_t) + 256;
}

qlora_status launch_layer_error_rank(int n_layers, const uint16_t* const* W_ptrs, const int64_t* numel, bool dq,
                                     int K, double* err, int32_t* order, uint8_t* keep, void* ws, size_t ws_bytes,
                                     int* status, cudaStream_t s) {
  static LayerTable tab;  // host staging of the by-value kernel parameter
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
  char* base = static_cast<char*>(ws) + kStatusBytes;
  double2* partial = reinterpret_cast<double2*>(base);
  int32_t* first_dev = reinterpret_cast<int32_t*>(base + size_t(c) * sizeof(double2));
  if (cudaMemcpyAsync(first_dev, tab.first_chunk, size_t(n_layers + 1) * sizeof(int32_t), cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return QLORA_ERR_CUDA;
  if (dq) layer_error_chunk_kernel<true><<<unsigned(c), 256, 0, s>>>(tab, partial, status);
  else layer_error_chunk_kernel<false><<<unsigned(c), 256, 0, s>>>(tab, partial, status);
  if (cudaGetLastError() != cudaSuccess) return QLORA_ERR_CUDA;
  layer_error_finish_kernel<<<(n_layers + 255) / 256, 256, 0, s>>>(partial, first_dev, n_layers, err);
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

__global__ void layer_error_finish_table_kernel(const double2* __restrict__ partial,
                                                const __grid_constant__ LayerTable tab, double* __restrict__ err) {
  const int l = blockIdx.x * blockDim.x + threadIdx.x;
  if (l >= tab.n_layers) return;
  double sd = 0.0, sw = 0.0;
  for (int c = tab.first_chunk[l]; c < tab.first_chunk[l + 1]; ++c) { sd += partial[c].x; sw += partial[c].y; }
  err[l] = (sw > 0.0) ? sqrt(sd / sw) : 0.0;
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
  layer_error_finish_table_kernel<<<(n_layers + 255) / 256, 256, 0, s>>>(partial, tab, err);
  rank_topk_kernel<<<1, 1024, 0, s>>>(err, n_layers, K, order, keep);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qlb
