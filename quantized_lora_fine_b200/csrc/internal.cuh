// Internal declarations shared by the translation units of libqlora_b200.so.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/qlora_b200.h"

namespace qlb {

constexpr int kBlock = 64;        // NF4 block (elements per absmax)
constexpr int kDQBlock = 256;     // absmax values per second-level scale
constexpr size_t kStatusBytes = 256;
// Workspace layout shared by every entry point: [0, 256) status word,
// [256, 256 + 64 KiB) split-K tile counters and the next 1 KiB of pair-GEMM tile
// counters (only ever used as counters, which the kernels return to zero), then
// per-call scratch.
constexpr size_t kCounterBytes = 65536;
// then 4 KiB of pair-GEMM counters and flags (the split last round's tile counters and
// the fused forward's per-block T flags; also left at zero)
constexpr size_t kGemmCounterBytes = 4096;
constexpr size_t kReservedBytes = kStatusBytes + kCounterBytes + kGemmCounterBytes;
constexpr int64_t kMaxCounterTiles = int64_t(kCounterBytes / 4);

// Launch with programmatic dependent launch allowed (unless QLORA_B200_PDL=0):
// the kernel may begin while the previous kernel in the stream finishes, so every
// kernel launched this way calls pdl_wait() before it touches global memory.
bool pdl_enabled();

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = at;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

int num_sms();

// The quantizer and the error pass stage one chunk of 256 blocks (32 KB of bf16,
// the double-quant group) per CTA in shared memory.
constexpr uint32_t kChunkBytes = uint32_t(kDQBlock) * kBlock * 2u;

__device__ __forceinline__ void set_status(int* st, int code) {
  if (st) atomicCAS(st, 0, code);
}

// Records the first error and, next to it, which wait gave up (a site number
// chosen by the kernel), for diagnosing a stalled pipeline.
__device__ __forceinline__ void set_status_site(int* st, int code, int site) {
  if (st && atomicCAS(st, 0, code) == 0) atomicExch(st + 1, site);
}

// ---- codec.cu
qlora_status launch_quantize(const void* W, int w_dtype, int64_t numel, bool dq, uint8_t* codes, float* absmax,
                             uint8_t* absmax_q, float* absmax2, int* status, cudaStream_t s);
// Up to 512 bf16 matrices in one launch (same double-quant setting for all).
qlora_status launch_quantize_batch(int n, const uint16_t* const* W, const int64_t* numel, bool dq,
                                   uint8_t* const* codes, float* const* absmax, uint8_t* const* absmax_q,
                                   float* const* absmax2, int* status, cudaStream_t s);
qlora_status launch_dequantize(const uint8_t* codes, const float* absmax, const uint8_t* absmax_q,
                               const float* absmax2, bool dq, int64_t numel, uint16_t* out, cudaStream_t s);
// Scales of an out x in NF4 weight, expanded to fp32 and laid out [in/64][out].
qlora_status launch_expand_scales(const uint8_t* unused, const float* absmax, const uint8_t* absmax_q,
                                  const float* absmax2, bool dq, int64_t out, int64_t in, float* scales_t,
                                  cudaStream_t s);
// dst[i][q] = bf16(s * src[i][q]), rows x r  (transpose = 0)
// dst[n][q] = bf16(s * src[q][n]), src r x cols (transpose = 1)
qlora_status launch_scale_lora(const uint16_t* src, int64_t rows, int64_t cols, float scale, bool transpose,
                               uint16_t* dst, cudaStream_t s);
// W_out = bf16(W_hat + s (L1 L2)^T) (stored layout; W_hat from the NF4 fields, or Wbf
// when it is non-null); in % 64 == 0. With q_codes non-null the merged weight is
// NF4-quantized instead of stored: codes to q_codes, exact fp32 absmax to q_absmax,
// non-finite merged values set QLORA_ERR_NONFINITE in *status.
qlora_status launch_lora_merge(const uint8_t* codes, const float* absmax, const uint8_t* absmax_q,
                               const float* absmax2, bool dq, const uint16_t* Wbf, int64_t out, int64_t in,
                               const uint16_t* L1, const uint16_t* L2, int r, double s, uint16_t* W_out,
                               uint8_t* q_codes, float* q_absmax, int* status, cudaStream_t st);
// R = fp32_rn(w - fp32_rn(c1 a1)) for the first NF4 stage (codes, scales); numel % 64 == 0.
qlora_status launch_nf4_residual(const uint16_t* W, const uint8_t* codes, const float* absmax,
                                 const uint8_t* absmax_q, const float* absmax2, bool dq, int64_t numel, float* R,
                                 cudaStream_t st);
// out = bf16_rn(fp32_rn(v1 + v2)) of two NF4 stages; numel % 64 == 0.
qlora_status launch_dequantize_two_stage(const uint8_t* codes1, const float* absmax1, const uint8_t* absmax_q1,
                                         const float* absmax2_1, bool dq1, const uint8_t* codes2,
                                         const float* absmax_2, const uint8_t* absmax_q2, const float* absmax2_2,
                                         bool dq2, int64_t numel, uint16_t* out, cudaStream_t st);
// Double-quantize a finished fp32 absmax array (nb scales, groups of 256).
qlora_status launch_dq_scales(const float* absmax, int64_t nb, uint8_t* absmax_q, float* absmax2, cudaStream_t st);
// ---- layer_error.cu
size_t layer_error_ws_bytes(int n_layers, const int64_t* numel);
qlora_status launch_quantize_error_rank(int n_layers, const uint16_t* const* W_ptrs, const int64_t* numel, bool dq,
                                       int K, uint8_t* const* codes, float* const* absmax, uint8_t* const* absmax_q,
                                       float* const* absmax2, double* err, int32_t* order, uint8_t* keep, void* ws,
                                       size_t ws_bytes, int* status, cudaStream_t s);
// With K_out non-null the keep rule is the memory budget (K ignored): the longest
// prefix of the order whose added bf16 bytes fit in budget_bytes; K goes to *K_out.
qlora_status launch_layer_error_rank(int n_layers, const uint16_t* const* W_ptrs, const int64_t* numel, bool dq,
                                     int K, double* err, int32_t* order, uint8_t* keep, void* ws, size_t ws_bytes,
                                     int* status, cudaStream_t s, int64_t budget_bytes = 0,
                                     int32_t* K_out = nullptr);
// The ranking alone over errors already on the device (1 <= n <= 1024).
qlora_status launch_rank_errors(int n, const double* err, int K, int32_t* order, uint8_t* keep, cudaStream_t s);
// Stored bytes of one NF4 matrix (codes + scales; double quant as configured).
int64_t nf4_storage_bytes(int64_t numel, bool dq);

// Allocation-free variant: partial sums in a file-scope device array (see layer_error.cu).
int64_t noalloc_chunks(int n_layers, const int64_t* numel);
qlora_status launch_layer_error_rank_noalloc(int n_layers, const uint16_t* const* W_ptrs, const int64_t* numel,
                                             bool dq, int K, double* err, int32_t* order, uint8_t* keep,
                                             cudaStream_t s);

// ---- gemm.cu
int last_pair_clusters();
// SMs a pair GEMM over num_tiles 256 x 256 tiles leaves free (see pairs_for).
int pair_spare_sms(bool dx, int num_tiles);
// The same for the 512 x 256 pair kernel over num_tiles tiles of `steps` K steps.
int pair2_spare_sms(bool dx, int num_tiles, int steps);
// Operand descriptions for the tcgen05 GEMM engine.
struct GemmPlan;
}  // namespace qlb
