// AQLoRA allocation pass on the GPU: per-layer NF4 reconstruction error
// (relative Frobenius norm), then ranking and the top-K keep mask.
//
// Pass 1: one CTA per chunk of 256 blocks (16384 elements) of some layer;
//         quantizes, dequantizes and accumulates sum (w - w_hat)^2 and sum w^2
//         in fp64; writes one partial pair per chunk (the fused entry also
//         writes the codes and scales).
// Pass 2: one warp per layer sums its chunk partials in chunk order -> err.
// Pass 3: one CTA ranks all layers by (err desc, id asc).
// The three kernels follow each other on the stream with programmatic dependent
// launch: each waits for its predecessor's memory before reading it.
#include <cfloat>
#include <cstdlib>
#include <cstring>
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

// Chunk ranges of the layers, for the finish pass (a by-value kernel parameter).
struct ChunkRanges {
  int32_t first_chunk[kMaxLayers + 1];
  int32_t n_layers;
};


// Chunk c of the table: its layer (binary search over first_chunk), index within
// the layer and number of blocks.
template <class Tab>
struct ChunkRef {
  int layer;
  int64_t g;
  int nblk;
  __device__ __forceinline__ ChunkRef(const Tab& tab, int64_t c) {
    int lo = 0, hi = tab.n_layers - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tab.first_chunk[mid] <= c) lo = mid; else hi = mid - 1;
    }
    layer = lo;
    g = c - tab.first_chunk[lo];
    const int64_t nb = tab.numel[lo] / kBlock;
    nblk = int(min(int64_t(kDQBlock), nb - g * kDQBlock));
  }
};

// Pass 1: one CTA per chunk of 256 blocks
// (16384 weights, the double-quant group) of some layer; thread t owns block t. The
// chunk's bf16 weights reach shared memory by one bulk copy; thread t reads its
// block as eight 16-byte pieces, piece j ^ (t mod 8) at step j (the 8 lanes of a
// quarter warp touch 8 different bank groups). Per block: absmax over packed bf16
// pairs; with double quant the chunk's max G of the absmax values gives the
// reconstruction scale ahat = e4m3(a 448 / G) G / 448 (the codes use the exact a).
// Per element: the code index from the one-multiply quotient and the shuffle lookup
// (as the quantizer), the code value by one more warp shuffle from the lane that
// holds it (lane l holds code[l mod 16]; the index bits select the lane),
// w_hat = bf16(fp32(code ahat)), and (w_hat - w)^2 (a mixed bf16 - fp32
// subtraction), w^2 summed in packed fp32 (16 terms per accumulator) before the
// fp64 chunk total. With Tab::kWrite (the fused pass) the thread's 8 code words go
// back in order and out in two 16-byte stores, with the scales. Warp 0 sums the
// 256 per-thread totals in a fixed order into partial[chunk]; the other warps
// leave as soon as their totals are in shared memory.
// With RELOAD the thread reads its pieces from shared memory twice (once for the
// absmax, once in the element loop) instead of holding all eight in registers, so
// six CTAs fit an SM instead of four.
template <bool DQ, class Tab, bool RELOAD = false>
__global__ void __launch_bounds__(256, RELOAD ? 6 : 4) layer_error_chunk_kernel(const __grid_constant__ Tab tab,
                                                                                double2* __restrict__ partial,
                                                                                int* status, uint64_t copy_wait_ns) {
  constexpr bool kW = Tab::kWrite;
  __shared__ __align__(128) uint32_t s_w[kChunkBytes / 4];
  __shared__ double2 s_part[256];
  __shared__ float s_red[8];
  __shared__ int s_ref[3];
  __shared__ __align__(8) uint64_t s_bar;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t bar = smem_u32(&s_bar);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbarrier_init();
  }
  const LaneTables lt = lane_tables(lane);
  const int64_t chunk = blockIdx.x;
  if (tid == 0) {   // the chunk's layer, by one thread
    const ChunkRef<Tab> cr(tab, chunk);
    s_ref[0] = cr.layer;
    s_ref[1] = cr.nblk;
    s_ref[2] = int(cr.g);
  }
  __syncthreads();   // barrier and chunk reference in place
  const int layer = s_ref[0], nblk = s_ref[1];
  const int64_t g = s_ref[2];
  pdl_wait();
  pdl_launch();
  if (tid == 0) {
    const uint32_t bytes = uint32_t(nblk) * kBlock * 2u;
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load(smem_u32(s_w), tab.ptr[layer] + g * (kDQBlock * kBlock), bytes, bar);
  }
  // the chunk's copy must land within copy_wait_ns (0: one non-blocking check)
  const bool landed = copy_wait_ns ? mbar_wait(bar, 0, copy_wait_ns) : mbar_test_wait(bar, 0);
  if (!__syncthreads_and(landed)) {   // every thread leaves together
    if (tid == 0) {
      if (status) set_status(status, QLORA_ERR_TIMEOUT);
      // the chunk's partial still gets written: NaN, so the layer's error shows the
      // failure instead of a sum left over from an earlier call
      partial[chunk] = make_double2(__longlong_as_double(0x7FF8000000000000ll),
                                    __longlong_as_double(0x7FF8000000000000ll));
    }
    if (!landed) mbar_wait(bar, 0, 20000000000ull);   // the copy must land before the CTA's memory is released
    return;
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
  const int64_t blk = g * kDQBlock + tid;
  float ahat = am;
  if constexpr (DQ) {
    float v = valid ? am : 0.f;   // max over the chunk (NaN blocks compare false and drop out)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) s_red[warp] = v;
    __syncthreads();
    float G = s_red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) G = fmaxf(G, s_red[i]);
    uint8_t q8 = 0;
    ahat = 0.f;
    if (G > 0.f) {
      q8 = f32_to_e4m3_satfinite(__fmul_rn(am, __fdiv_rn(448.f, G)));
      ahat = __fmul_rn(e4m3_to_f32(q8), __fdiv_rn(G, 448.f));
    }
    if constexpr (kW) {
      if (valid) {
        tab.absmax_q[layer][blk] = q8;
        if (tab.absmax[layer] != nullptr) tab.absmax[layer][blk] = am;
      }
      if (tid == 0) tab.absmax2[layer][g] = (G > 0.f) ? __fdiv_rn(G, 448.f) : 0.f;
    }
  } else if constexpr (kW) {
    if (valid) tab.absmax[layer][blk] = am;
  }
  // Every lane runs the element loop (it holds warp shuffles). Lanes without a live
  // block (past the chunk, all-zero or non-finite) run it on zeros with a = 1, which
  // keeps every quotient finite and adds nothing to the sums; their code words are
  // the zero code.
  const bool live = valid && am > 0.f && !bad;
  if constexpr (!RELOAD) {
    if (bad) {
#pragma unroll
      for (int j = 0; j < 8; ++j) u[j][0] = u[j][1] = u[j][2] = u[j][3] = 0u;
    }
  }
  const CellScale cs(live ? am : 1.f);
  const uint64_t ah2 = f2_splat(ahat);
  uint64_t sd2[2] = {0ull, 0ull}, sw2[2] = {0ull, 0ull};
  uint32_t cw[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t x[8];
    uint32_t* uj = u[RELOAD ? 0 : j];
    if constexpr (RELOAD) {
      uj[0] = uj[1] = uj[2] = uj[3] = 0u;
      if (valid && !bad) lds_u4(src ^ (uint32_t(j) << 4), u[0]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint64_t w = f2_from_bf16x2(uj[i]);
      const uint64_t q = f2_mul(w, cs.r2);
      const uint64_t c = cells2(q, cs.cmul2);
      x[2 * i] = index_bits(f2_lo(q), uint32_t(c), cs.M, lt);
      x[2 * i + 1] = index_bits(f2_hi(q), uint32_t(c >> 32), cs.M, lt);
      const float c0 = code_value(x[2 * i], lt), c1 = code_value(x[2 * i + 1], lt);
      const uint64_t p = f2_mul((uint64_t(__float_as_uint(c1)) << 32) | __float_as_uint(c0), ah2);
      const uint64_t d = f2_bf16x2_minus(pack_bf16x2(f2_lo(p), f2_hi(p)), w);
      sd2[j >> 2] = f2_fma(d, d, sd2[j >> 2]);
      sw2[j >> 2] = f2_fma(w, w, sw2[j >> 2]);
    }
    if constexpr (kW) cw[j] = live ? pack_code_word(x) : 0x77777777u;
  }
  if constexpr (kW) {
    if (valid) {
      unrotate8(cw, rot);
      uint4* dst = reinterpret_cast<uint4*>(tab.codes[layer] + blk * (kBlock / 2));
      dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
    }
  }
  if (bad && status) set_status(status, QLORA_ERR_NONFINITE);
  double sd = 0.0, sw = 0.0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    sd += double(f2_lo(sd2[h])) + double(f2_hi(sd2[h]));
    sw += double(f2_lo(sw2[h])) + double(f2_hi(sw2[h]));
  }
  if (bad && !status) {
    // without a status word the non-finite block is reported through the sums:
    // NaN reaches the chunk's partial and the layer's error
    sd = __longlong_as_double(0x7FF8000000000000ll);
    sw = sd;
  }
  s_part[tid] = make_double2(sd, sw);
  __syncthreads();
  if (warp != 0) return;
  // ---- warp 0: the chunk total in a fixed order
  double a = 0.0, b = 0.0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const double2 v = s_part[lane * 8 + k];
    a += v.x;
    b += v.y;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  if (lane == 0) partial[chunk] = make_double2(a, b);
}

// One warp per layer: lane l sums chunks first+l, first+l+32, ... in order; the 32
// lane sums combine by a fixed shuffle pattern, so the result is deterministic for
// a given layout.
__device__ __forceinline__ void finish_layer_warp(const double2* __restrict__ partial, int c0, int c1,
                                                  double* __restrict__ err_out) {
  const int lane = threadIdx.x & 31;
  double a = 0.0, b = 0.0;
  for (int c = c0 + lane; c < c1; c += 32) {
    const double2 v = __ldcg(partial + c);
    a += v.x;
    b += v.y;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  // an all-zero layer has error 0; a NaN sum (non-finite block or timed-out copy on
  // the path without a status word) gives NaN
  if (lane == 0) *err_out = (b == 0.0) ? 0.0 : sqrt(a / b);
}

// Position of layer l in the order (error descending, index ascending). A NaN
// error (only the path without a status word produces one) ranks ahead of every
// number, NaN layers among themselves by index, so the order stays a permutation.
__device__ __forceinline__ int rank_of(const double* s_err, int n_layers, int l) {
  const double e = s_err[l];
  const bool en = isnan(e);
  int rank = 0;
  for (int j = 0; j < n_layers; ++j) {
    const double f = s_err[j];
    const bool fn = isnan(f);
    const bool before = (fn != en) ? fn : (en ? (j < l) : (f > e || (f == e && j < l)));
    rank += before ? 1 : 0;
  }
  return rank;
}

__global__ void __launch_bounds__(1024) rank_topk_kernel(const double* __restrict__ err, int n_layers, int K,
                                                         int32_t* __restrict__ order, uint8_t* __restrict__ keep) {
  pdl_wait();
  pdl_launch();
  __shared__ double s_err[kMaxLayers];
  for (int i = threadIdx.x; i < n_layers; i += blockDim.x) s_err[i] = err[i];
  __syncthreads();
  for (int l = threadIdx.x; l < n_layers; l += blockDim.x) {
    const int rank = rank_of(s_err, n_layers, l);
    order[rank] = l;
    keep[l] = rank < K ? 1 : 0;
  }
}

// Keep rule by memory budget: the longest prefix of the order whose added bytes
// (cost[l]: what keeping layer l in bf16 adds to its NF4 storage, always > 0) sum
// to at most `budget`. One thread per layer (n_layers <= 1024 = block size):
// costs are placed at their rank, an inclusive prefix sum runs in shared memory,
// and since the prefixes grow, K is the number of them within the budget.
struct BudgetTable {
  int64_t cost[kMaxLayers];
  int64_t budget;
};

__global__ void __launch_bounds__(1024) rank_budget_kernel(const double* __restrict__ err, int n_layers,
                                                           const __grid_constant__ BudgetTable bt,
                                                           int32_t* __restrict__ order, uint8_t* __restrict__ keep,
                                                           int32_t* __restrict__ K_out) {
  pdl_wait();
  pdl_launch();
  __shared__ double s_err[kMaxLayers];
  __shared__ int64_t s_pre[kMaxLayers];
  __shared__ int32_t s_rank[kMaxLayers];
  const int t = threadIdx.x;
  if (t < n_layers) s_err[t] = err[t];
  __syncthreads();
  if (t < n_layers) {
    const int rank = rank_of(s_err, n_layers, t);
    s_rank[t] = rank;
    order[rank] = t;
    s_pre[rank] = bt.cost[t];
  }
  __syncthreads();
  for (int off = 1; off < n_layers; off <<= 1) {
    const int64_t v = (t < n_layers && t >= off) ? s_pre[t - off] : 0;
    __syncthreads();
    if (t < n_layers) s_pre[t] += v;
    __syncthreads();
  }
  const int K = __syncthreads_count(t < n_layers && s_pre[t] <= bt.budget);
  if (t < n_layers) keep[t] = s_rank[t] < K ? 1 : 0;
  if (t == 0) *K_out = K;
}

// Pass 2: one warp per layer.
__global__ void __launch_bounds__(32) layer_error_finish_kernel(const double2* __restrict__ partial,
                                                                const __grid_constant__ ChunkRanges r,
                                                                double* __restrict__ err) {
  pdl_wait();
  pdl_launch();
  const int l = blockIdx.x;
  if (l >= r.n_layers) return;
  finish_layer_warp(partial, r.first_chunk[l], r.first_chunk[l + 1], err + l);
}

// Passes 2 and 3 in one CTA for a few layers (the allocation pass of one matrix, or
// of a layer's handful): all 1024 threads sum a layer's chunk partials (thread t
// takes chunks first + t, first + t + 1024, ...; warps then the 32 warp sums
// combine by a fixed shuffle pattern, so the result is deterministic for a given
// layout), then every thread ranks layers as rank_topk_kernel does.
constexpr int kSmallLayers = 16;
__global__ void __launch_bounds__(1024) finish_rank_small_kernel(const double2* __restrict__ partial,
                                                                 const __grid_constant__ ChunkRanges r,
                                                                 double* __restrict__ err, int K,
                                                                 int32_t* __restrict__ order,
                                                                 uint8_t* __restrict__ keep) {
  pdl_wait();
  pdl_launch();
  __shared__ double s_a[32], s_b[32];
  __shared__ double s_err[kSmallLayers];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = r.n_layers;
  for (int l = 0; l < n; ++l) {
    double a = 0.0, b = 0.0;
    for (int c = r.first_chunk[l] + tid; c < r.first_chunk[l + 1]; c += 1024) {
      const double2 v = __ldcg(partial + c);
      a += v.x;
      b += v.y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      b += __shfl_xor_sync(0xffffffffu, b, o);
    }
    if (lane == 0) {
      s_a[warp] = a;
      s_b[warp] = b;
    }
    __syncthreads();
    if (warp == 0) {
      a = s_a[lane];
      b = s_b[lane];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
      }
      // as finish_layer_warp: an all-zero layer has error 0, a NaN sum gives NaN
      if (lane == 0) {
        const double e = (b == 0.0) ? 0.0 : sqrt(a / b);
        s_err[l] = e;
        err[l] = e;
      }
    }
    __syncthreads();
  }
  for (int l = tid; l < n; l += blockDim.x) {
    const int rank = rank_of(s_err, n, l);
    order[rank] = l;
    keep[l] = rank < K ? 1 : 0;
  }
}

// Limit of the chunk kernel's wait for its bulk copy: 2 s, or QLORA_B200_COPY_WAIT_NS
// (read on every call; 0 = one non-blocking check). A limit that runs out records
// QLORA_ERR_TIMEOUT (or a NaN error without a status word) and the kernel still waits
// for its copy to land before it exits; the failure-detection tests use 0.
static uint64_t copy_wait_ns() {
  const char* e = std::getenv("QLORA_B200_COPY_WAIT_NS");
  if (!e) return 2000000000ull;
  return std::strtoull(e, nullptr, 10);
}

static int32_t chunks_of(int64_t numel) {
  const int64_t nb = numel / kBlock;
  return static_cast<int32_t>((nb + kDQBlock - 1) / kDQBlock);
}

// Bytes of one NF4 matrix as stored: packed codes plus fp32 scales, or with double
// quant one E4M3 byte per block plus one fp32 factor per 256 blocks.
int64_t nf4_storage_bytes(int64_t numel, bool dq) {
  const int64_t nb = (numel + kBlock - 1) / kBlock;
  return (numel + 1) / 2 + (dq ? nb + 4 * ((nb + kDQBlock - 1) / kDQBlock) : 4 * nb);
}

size_t layer_error_ws_bytes(int n_layers, const int64_t* numel) {
  int64_t chunks = 0;
  for (int i = 0; i < n_layers; ++i) chunks += chunks_of(numel[i]);
  return kReservedBytes + size_t(chunks) * sizeof(double2);
}

// Chunk kernel variant: six CTAs per SM, each thread reading its pieces twice, unless
// QLORA_B200_ERR_RELOAD=0 (four CTAs, pieces held in registers; read on every call).
// On the 224-matrix stack: error pass 3.51 against 3.38 TB/s, fused quantize + error
// 4.02 against 3.78 TB/s.
static bool err_reload() {
  const char* e = std::getenv("QLORA_B200_ERR_RELOAD");
  return !(e && std::strcmp(e, "0") == 0);
}

// The three passes on stream s. tab.first_chunk / n_layers are filled in; the chunk
// and rank kernels need nothing else from the host. With pdl, each kernel may start
// while its predecessor drains (the allocation-free entry launches plainly).
template <bool DQ, class Tab>
static qlora_status launch_passes(const Tab& tab, double2* partial, int* status, double* err, int K,
                                  int32_t* order, uint8_t* keep, cudaStream_t s, bool pdl,
                                  const BudgetTable* budget = nullptr, int32_t* K_out = nullptr) {
  static std::mutex mu;
  static ChunkRanges r;   // host staging of the by-value parameter
  std::lock_guard<std::mutex> lock(mu);
  const int n = tab.n_layers;
  r.n_layers = n;
  for (int i = 0; i <= n; ++i) r.first_chunk[i] = tab.first_chunk[i];
  const unsigned c = unsigned(tab.first_chunk[n]);
  cudaError_t e;
  if (pdl) {
    e = err_reload() ? launch_pdl(layer_error_chunk_kernel<DQ, Tab, true>, dim3(c), dim3(256), 0, s, tab, partial,
                                  status, copy_wait_ns())
                     : launch_pdl(layer_error_chunk_kernel<DQ, Tab>, dim3(c), dim3(256), 0, s, tab, partial, status,
                                  copy_wait_ns());
    if (e == cudaSuccess && !budget && n <= kSmallLayers) {
      e = launch_pdl(finish_rank_small_kernel, dim3(1), dim3(1024), 0, s, partial, r, err, K, order, keep);
    } else {
      if (e == cudaSuccess)
        e = launch_pdl(layer_error_finish_kernel, dim3(unsigned(n)), dim3(32), 0, s, partial, r, err);
      if (e == cudaSuccess)
        e = budget ? launch_pdl(rank_budget_kernel, dim3(1), dim3(1024), 0, s, err, n, *budget, order, keep, K_out)
                   : launch_pdl(rank_topk_kernel, dim3(1), dim3(1024), 0, s, err, n, K, order, keep);
    }
  } else {
    if (err_reload())
      layer_error_chunk_kernel<DQ, Tab, true><<<c, 256, 0, s>>>(tab, partial, status, copy_wait_ns());
    else
      layer_error_chunk_kernel<DQ, Tab><<<c, 256, 0, s>>>(tab, partial, status, copy_wait_ns());
    if (!budget && n <= kSmallLayers) {
      finish_rank_small_kernel<<<1, 1024, 0, s>>>(partial, r, err, K, order, keep);
    } else {
      layer_error_finish_kernel<<<unsigned(n), 32, 0, s>>>(partial, r, err);
      if (budget)
        rank_budget_kernel<<<1, 1024, 0, s>>>(err, n, *budget, order, keep, K_out);
      else
        rank_topk_kernel<<<1, 1024, 0, s>>>(err, n, K, order, keep);
    }
    e = cudaSuccess;
  }
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status launch_layer_error_rank(int n_layers, const uint16_t* const* W_ptrs, const int64_t* numel, bool dq,
                                     int K, double* err, int32_t* order, uint8_t* keep, void* ws, size_t ws_bytes,
                                     int* status, cudaStream_t s, int64_t budget_bytes, int32_t* K_out) {
  // The chunk table travels as a by-value kernel parameter (no host-to-device
  // copy), so this call can be captured into a CUDA graph.
  static std::mutex mu;
  static LayerTable tab;
  std::lock_guard<std::mutex> lock(mu);
  if (layer_error_ws_bytes(n_layers, numel) > ws_bytes) return QLORA_ERR_WORKSPACE;
  tab.n_layers = n_layers;
  int32_t c = 0;
  for (int i = 0; i < n_layers; ++i) {
    tab.ptr[i] = W_ptrs[i];
    tab.numel[i] = numel[i];
    tab.first_chunk[i] = c;
    c += chunks_of(numel[i]);
  }
  tab.first_chunk[n_layers] = c;
  double2* partial = reinterpret_cast<double2*>(static_cast<char*>(ws) + kReservedBytes);
  if (K_out) {   // keep rule by memory budget
    static BudgetTable bt;
    for (int i = 0; i < n_layers; ++i) bt.cost[i] = 2 * numel[i] - nf4_storage_bytes(numel[i], dq);
    bt.budget = budget_bytes;
    return dq ? launch_passes<true>(tab, partial, status, err, 0, order, keep, s, true, &bt, K_out)
              : launch_passes<false>(tab, partial, status, err, 0, order, keep, s, true, &bt, K_out);
  }
  return dq ? launch_passes<true>(tab, partial, status, err, K, order, keep, s, true)
            : launch_passes<false>(tab, partial, status, err, K, order, keep, s, true);
}

qlora_status launch_rank_errors(int n, const double* err, int K, int32_t* order, uint8_t* keep, cudaStream_t s) {
  const cudaError_t e = launch_pdl(rank_topk_kernel, dim3(1), dim3(1024), 0, s, err, n, K, order, keep);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status launch_quantize_error_rank(int n_layers, const uint16_t* const* W_ptrs, const int64_t* numel, bool dq,
                                       int K, uint8_t* const* codes, float* const* absmax, uint8_t* const* absmax_q,
                                       float* const* absmax2, double* err, int32_t* order, uint8_t* keep, void* ws,
                                       size_t ws_bytes, int* status, cudaStream_t s) {
  if (n_layers > kMaxFusedLayers) return QLORA_ERR_SHAPE;
  static std::mutex mu;
  static FusedTable tab;
  std::lock_guard<std::mutex> lock(mu);
  if (layer_error_ws_bytes(n_layers, numel) > ws_bytes) return QLORA_ERR_WORKSPACE;
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
  double2* partial = reinterpret_cast<double2*>(static_cast<char*>(ws) + kReservedBytes);
  return dq ? launch_passes<true>(tab, partial, status, err, K, order, keep, s, true)
            : launch_passes<false>(tab, partial, status, err, K, order, keep, s, true);
}

// ------------------------------------------------------------------------
// Allocation-free variant.
//
// Same three passes, but the per-chunk partial sums live in a file-scope device
// array instead of a caller workspace, so a call needs no device memory beyond
// its inputs and outputs. The array is 16 MiB (2^20 chunks of 16384 weights, i.e.
// up to 2^34 weights per call); every GPU that loads the library keeps it
// until the process exits. All calls share it: calls that overlap on the GPU
// (two streams, two host threads) race on it. Each call overwrites every
// partial it reads (a chunk whose copy timed out writes NaN), so nothing has to be
// cleared between calls. There is no status word on this path: a non-finite block
// or a timed-out copy turns its chunk's partial, and so the layer's error, into NaN.

constexpr int64_t kNoAllocMaxChunks = int64_t(1) << 20;
static __device__ __align__(256) double2 g_noalloc_partials[kNoAllocMaxChunks];

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
  return dq ? launch_passes<true>(tab, partial, nullptr, err, K, order, keep, s, false)
            : launch_passes<false>(tab, partial, nullptr, err, K, order, keep, s, false);
}

}  // namespace qlb
