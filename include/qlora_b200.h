/*
 * qlora_b200.h -- C ABI of the NF4-LoRA hot path for NVIDIA B200 (sm_100a).
 *
 * The operations and the pages that define them:
 *   nf4_quantize / nf4_dequantize
 *       "QLoRA: How to fine-tune large language models with less memory",
 *       sections "1. NormalFloat" (16 normal-shaped 4-bit codes, one scale per
 *       block of weights, dequantized to BFloat16 before the matmul) and
 *       "2. Double quantization" (8-bit first-level scales, a higher-precision
 *       scale per group of 256); AQLoRA summary page, section 3.1 (64-element
 *       blocks).
 *   qlora_linear_fwd
 *       Same QLoRA page, "The algebra", eq. (3): Y = X W + s X L1 L2, with the
 *       scaling s = alpha / r of "LoRA: Fine-tuning a model by learning a small
 *       update", eq. (3).
 *   qlora_linear_bwd
 *       Gradients of eq. (3) with the base frozen: gradient reaches X through
 *       the dequantized W, no gradient is formed for W ("Lesson 17. What QLoRA
 *       Actually Costs", warm-up; QLoRA page, "One training step").
 *   nf4_layer_error_rank
 *       AQLoRA summary page, sections 3.1-3.2: per-layer NF4 reconstruction
 *       error, ranking, top-K kept in 16-bit.
 *
 * Conventions (all entry points):
 *   - Every tensor is dense, row-major, and lives in device memory owned by the
 *     caller. The library never allocates device memory on these calls; scratch
 *     comes from a caller workspace sized by the matching *_workspace_size().
 *   - bf16 tensors are passed as uint16_t* (bit patterns).
 *   - Weights are stored out x in (nn.Linear layout): W_s = W^T of eq. (3).
 *     Quantization blocks of 64 run along `in` (the flattened row-major order).
 *   - Work is enqueued on `stream` and runs asynchronously; pointers must stay
 *     valid until it completes. Host-side argument checks run before any
 *     launch and return an error without touching device memory.
 *   - Device-side conditions (non-finite weights, an internal wait that ran
 *     out) are recorded in an int32 status word at the start of the
 *     workspace. The word is sticky: it keeps the first error until
 *     qlora_reset_status(). A fresh workspace must be zeroed (or reset) once.
 *   - One workspace may serve every entry point on a stream: its first 256
 *     bytes hold the status word, the next 64 KiB + 4 KiB split-K tile
 *     counters and the forward GEMM's per-row-block flags, which must be zero
 *     when a call starts and which every call that ends with status 0 leaves
 *     zero; a call's other scratch comes after them. Zeroing a workspace once
 *     keeps this true for any sequence of successful calls; after an error,
 *     qlora_reset_workspace() restores it.
 *   - No call aborts the process or throws.
 */
#ifndef QLORA_B200_H
#define QLORA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* qlora_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_NULL = 1,        /* a required pointer is NULL                         */
  QLORA_ERR_SHAPE = 2,       /* a size or a size combination is not supported      */
  QLORA_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned                   */
  QLORA_ERR_DTYPE = 4,       /* unknown dtype code                                 */
  QLORA_ERR_UNSUPPORTED = 5, /* device is not sm_100, or a config value unsupported */
  QLORA_ERR_CUDA = 6,        /* a CUDA runtime/driver call failed                  */
  QLORA_ERR_WORKSPACE = 7,   /* workspace NULL, misaligned or too small            */
  QLORA_ERR_NONFINITE = 8,   /* device: a weight was NaN or +-Inf                  */
  QLORA_ERR_TIMEOUT = 9      /* device: a pipeline wait exceeded its limit         */
} qlora_status;

enum { QLORA_DTYPE_BF16 = 0, QLORA_DTYPE_F32 = 1 };

/* Quantization config: blocksize must be 64 and dq_blocksize 256 (the values
 * the pages give); double_quant is 0 or 1. */
typedef struct {
  int32_t blocksize;
  int32_t double_quant;
  int32_t dq_blocksize;
} nf4_qconfig;

/* Descriptor of one frozen linear weight, stored out x in.
 *   is_bf16 = 0: NF4 storage.
 *     codes    uint8 [out*in/2]; byte k holds element 2k in its high nibble and
 *              element 2k+1 in its low nibble; a nibble is the index (0..15) of
 *              the code in the ascending NF4 table.
 *     absmax   fp32 [out*in/64]          (double_quant = 0)
 *     absmax_q uint8 [out*in/64], E4M3   (double_quant = 1)
 *     absmax2  fp32 [ceil(out*in/64/256)] (double_quant = 1)
 *   is_bf16 = 1: a protected layer kept in 16-bit (AQLoRA section 3.2);
 *     w_bf16 bf16 [out*in]; the NF4 fields are ignored.
 */
typedef struct {
  int64_t out;
  int64_t in;
  nf4_qconfig q;
  int32_t is_bf16;
  const uint8_t* codes;
  const float* absmax;
  const uint8_t* absmax_q;
  const float* absmax2;
  const uint16_t* w_bf16;
} qlora_weight;

/* ------------------------------------------------------------------ status */

const char* qlora_status_str(qlora_status s);

/* Synchronizes `stream` and returns the device status word in `workspace`
 * (QLORA_OK if no device-side error was recorded). */
qlora_status qlora_read_status(const void* workspace, qlora_stream_t stream);

/* Clears the device status word (stream-ordered). */
qlora_status qlora_reset_status(void* workspace, qlora_stream_t stream);

/* Clears the status word and the tile counters and block flags that follow it
 * (the workspace's first min(workspace_bytes, 256 + 64 KiB + 4 KiB) bytes;
 * stream-ordered). A call that ended with a nonzero status may have stopped
 * between setting and clearing those, so reset this way (not only the status
 * word) before the workspace serves a GEMM again. QLORA_ERR_WORKSPACE when
 * workspace is NULL or smaller than 256 bytes. */
qlora_status qlora_reset_workspace(void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/* Checks that device `device` is an sm_100 (B200-class) part. */
qlora_status qlora_device_check(int device);

/* Profiling aid (not part of the method): when set, cudaEvent_t handles that
 * the library records on the caller's stream right before and right after the
 * main tensor-core GEMM of qlora_linear_fwd (fwd_*) and of qlora_linear_bwd
 * (dx_*). Pass NULL to disable. Process-wide; not thread-safe. */
qlora_status qlora_profile_events(void* fwd_begin, void* fwd_end, void* dx_begin, void* dx_end);

/* Diagnostic (not part of the method): the number of 2-SM CTA pairs the last NF4
 * GEMM launch used (0 before any). The 256 x 256 output tiles are spread over
 * them, so a part that co-schedules fewer pairs takes more rounds of tiles. */
int32_t qlora_pair_clusters(void);

/* Diagnostic, host only (no device work): the schedule the NF4 pair GEMM (512 x 256
 * tiles) uses for `tiles` tiles of `steps` K steps (K / 64 plus the LoRA steps), the
 * first `aux_tiles` of them the T or U tiles (0 when the LoRA product is computed
 * apart), over `pairs` co-resident CTA pairs (1..80):
 *   out[0] P = pairs, out[1] R = whole rounds (pair p takes tiles p + r P, r < R),
 *   out[2] L = steps per pair in the remaining tiles (0: none remain), out[3] W =
 *   their total steps, out[4] base = R P (tail step s is step s % steps of tile
 *   base + s / steps), out[5] pairs launched, out[6] A and out[7] La: pair p < A (one
 *   that ran an aux tile, about half a tile's work) takes tail steps [p La, (p + 1)
 *   La), pair p >= A takes [A La + (p - A) L, + L), all clipped to W (A = 0: every
 *   pair [p L, (p + 1) L)).
 * A tile cut into parts is finished by the pair holding its first step.
 * QLORA_ERR_SHAPE unless tiles >= 1, 0 <= aux_tiles <= tiles, steps >= 1 and
 * 1 <= pairs <= 80; QLORA_ERR_NULL when out is NULL. */
qlora_status qlora_pair_schedule(int32_t tiles, int32_t aux_tiles, int32_t steps, int32_t pairs, int32_t* out);

/* ------------------------------------------------------------ NF4 codec */

/* Bytes of workspace nf4_quantize needs (the status word only). */
size_t nf4_quantize_workspace_size(int64_t numel);

/* Blockwise NF4 quantization of W (numel = out*in elements, any even count up to
 * 2^40, else QLORA_ERR_SHAPE; a short last block uses the elements present).
 *   W        device, bf16 (w_dtype QLORA_DTYPE_BF16) or fp32, 16-byte aligned
 *   codes    device out, uint8 [numel/2]
 *   absmax   device out, fp32 [ceil(numel/64)]; required when double_quant = 0,
 *            optional (may be NULL) when double_quant = 1
 *   absmax_q device out, uint8 [ceil(numel/64)]      (double_quant = 1)
 *   absmax2  device out, fp32 [ceil(numel/64/256)]   (double_quant = 1)
 * Per block b: a_b = max|w| (fp32); n = w / a_b (IEEE fp32 division); code =
 * #{j : n > m_j} over the 15 fp32 midpoints of adjacent codes. With double
 * quantization, per group of 256 scales: G = max a_b, q_b =
 * E4M3_rn_satfinite(a_b * fp32(448/G)), absmax2 = fp32(G/448); codes always use
 * the exact a_b. A NaN/Inf weight sets QLORA_ERR_NONFINITE in the status word
 * (codes of that block are then unspecified; the call still completes). */
qlora_status nf4_quantize(const void* W, int32_t w_dtype, int64_t out, int64_t in, nf4_qconfig q,
                          uint8_t* codes, float* absmax, uint8_t* absmax_q, float* absmax2,
                          void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/* The same quantization for n bf16 matrices in one launch (a whole model at
 * load time): matrix i is W_ptrs[i] (numel[i] elements, even, <= 2^40) with its own
 * codes[i], absmax[i] / absmax_q[i], absmax2[i] laid out as for nf4_quantize;
 * every bit is the one nf4_quantize gives that matrix alone.
 *   n        1 <= n <= 512
 *   W_ptrs, numel, codes, absmax, absmax_q, absmax2   HOST arrays of n entries
 *            (device pointers inside; absmax may be NULL or hold NULLs with
 *            double quant, absmax_q / absmax2 may be NULL without it)
 *   w_dtype  QLORA_DTYPE_BF16
 * Errors and workspace as nf4_quantize. */
qlora_status nf4_quantize_batch(int32_t n, const uint16_t* const* W_ptrs, const int64_t* numel, int32_t w_dtype,
                                nf4_qconfig q, uint8_t* const* codes, float* const* absmax,
                                uint8_t* const* absmax_q, float* const* absmax2, void* workspace,
                                size_t workspace_bytes, qlora_stream_t stream);

/* Dequantization to bf16: W_out[i] = bf16_rn(fp32_rn(code[idx_i] * a)) with a the
 * block's absmax, or with double quantization a = fp32_rn(fp32(q_b) * absmax2[g]).
 *   w      host pointer to a descriptor with is_bf16 = 0 (device buffers inside);
 *          out * in even and at most 2^40
 *   W_out  device out, bf16 [out*in], 16-byte aligned */
qlora_status nf4_dequantize(const qlora_weight* w, uint16_t* W_out, qlora_stream_t stream);

/* ------------------------------------------ residual NF4 second stage */

/* A protected layer stored as two NF4 stages instead of bf16 ("AQLoRA: A
 * Zero-Search Recipe for Fast Quantized LoRA Fine-Tuning", "Additional controls"
 * and section 8: a second NF4 stage over the protected layers' residuals matched
 * 16-bit protection at +3.6 % step time). The second stage quantizes
 *   R = fp32_rn(w - fp32_rn(c1 * a1))
 * (w the original bf16 weight, c1 * a1 the first stage's value) exactly as
 * nf4_quantize quantizes an fp32 tensor (config q, its own double-quant setting).
 *   W        device bf16 [out x in], 16-byte aligned: the weight the first stage
 *            was made from
 *   w1       host pointer to the first stage's descriptor (is_bf16 = 0);
 *            out, in <= 2^30, out * in % 64 == 0 and out * in <= 2^40
 *   codes, absmax, absmax_q, absmax2   device outs for the second stage, laid out
 *            as nf4_quantize's
 *   workspace  nf4_quantize_residual_workspace_size(out * in) bytes, 16-byte
 *            aligned (status word, counters, then R) */
size_t nf4_quantize_residual_workspace_size(int64_t numel);
qlora_status nf4_quantize_residual(const uint16_t* W, const qlora_weight* w1, nf4_qconfig q, uint8_t* codes,
                                   float* absmax, uint8_t* absmax_q, float* absmax2, void* workspace,
                                   size_t workspace_bytes, qlora_stream_t stream);

/* The two-stage reconstruction the GEMM consumes:
 *   W_out[i] = bf16_rn(fp32_rn(fp32_rn(c1 * a1) + fp32_rn(c2 * a2)))
 *   w1, w2   host pointers to the two stages' descriptors (same out, in)
 *   W_out    device out, bf16 [out x in], 16-byte aligned
 * A layer stored this way runs the linear through the protected-layer (bf16)
 * path on W_out. */
qlora_status nf4_dequantize_two_stage(const qlora_weight* w1, const qlora_weight* w2, uint16_t* W_out,
                                      qlora_stream_t stream);

/* ------------------------------------------------------------ LoRA merge */

/* Merging the adapter into the frozen weight after training ("LoRA: Fine-tuning a
 * model by learning a small update", section "Serving models and switching tasks":
 * W_merged = W_0 + (alpha / r) B A, no extra inference latency; "QLoRA: How to
 * fine-tune large language models with less memory", eq. (3)), in the stored
 * out x in layout:
 *   W_out = bf16_rn(W_hat + s (L1 L2)^T)
 * with W_hat the dequantized NF4 weight (bf16_rn(fp32_rn(code * scale)), as
 * nf4_dequantize) or the protected bf16 one. The rank-r product is summed in fp64
 * and the sum rounded to bf16 once (exact for bf16 adapters and weights of ordinary
 * ranges: every product is exact in fp64). A negative scale unmerges.
 *   w      host pointer to the weight descriptor; in % 64 == 0
 *   L1     device bf16 [in x r]     L2 device bf16 [r x out]     1 <= r <= 256
 *   W_out  device out, bf16 [out x in], 16-byte aligned
 * qlora_lora_merge_requantize NF4-quantizes the merged bf16 weight exactly as
 * nf4_quantize would (codes / scales laid out as there; config q) without storing
 * it: each 64-block is quantized where it is merged, then the scales are
 * double-quantized when q.double_quant is set. absmax (fp32 [out*in/64]) may be
 * NULL with double quant; the exact scales then live in the workspace
 * (qlora_lora_merge_requantize_workspace_size bytes, 16-byte aligned; its first
 * bytes are the status word, which gets QLORA_ERR_NONFINITE if a merged value is
 * not finite). */
qlora_status qlora_lora_merge(const qlora_weight* w, const uint16_t* L1, const uint16_t* L2, int32_t r, float scale,
                              uint16_t* W_out, qlora_stream_t stream);
size_t qlora_lora_merge_requantize_workspace_size(int64_t out, int64_t in);
qlora_status qlora_lora_merge_requantize(const qlora_weight* w, const uint16_t* L1, const uint16_t* L2, int32_t r,
                                         float scale, nf4_qconfig q, uint8_t* codes, float* absmax,
                                         uint8_t* absmax_q, float* absmax2, void* workspace,
                                         size_t workspace_bytes, qlora_stream_t stream);

/* --------------------------------------------------------- NF4-LoRA linear */

/* Shape rules for the linear: in % 256 == 0, out % 256 == 0, 1 <= M <= 2^20
 * and in, out <= 2^20, r % 8 == 0 and 8 <= r <= 256; every pointer 16-byte
 * aligned. The workspace holds, after the status word, 64 KiB of split-K tile
 * counters that the kernels leave at zero: zero a fresh workspace once before
 * its first use. A workspace serves one call at a time: calls that may run at
 * the same time (on different streams) need different workspaces. */
size_t qlora_fwd_workspace_size(int64_t M, int64_t out, int64_t in, int32_t r);
size_t qlora_bwd_workspace_size(int64_t M, int64_t out, int64_t in, int32_t r);

/* Forward, eq. (3) in stored layout:
 *   T = X L1             (M x r; fp32 accumulation, rounded once to bf16)
 *   Y = X W_s^T + s T L2 (M x out; fp32 accumulation in tensor memory, one bf16
 *                         rounding at the end)
 *   w       host pointer to the weight descriptor (NF4 or protected bf16)
 *   X       device bf16 [M x in]     L1 device bf16 [in x r]   L2 device bf16 [r x out]
 *   scale   s (alpha / r, or any value)
 *   Y       device out, bf16 [M x out]
 *   T_save  device out, bf16 [M x r] (T, unscaled), or NULL to keep it in the
 *           workspace only.
 * The NF4 weight is dequantized tile by tile inside the GEMM; no dequantized
 * copy of W is written to memory. With an NF4 weight (and M <= 110592) T is
 * computed inside the same GEMM, in one leading tile per 512 rows of X whose rows
 * the LoRA step of the output tiles waits for (QLORA_B200_FUSED_T=0: as its own
 * pass); a protected weight computes T as its own pass. The two ways sum the fp32
 * products in different orders, so T may differ in the last bf16 bit. */
qlora_status qlora_linear_fwd(const qlora_weight* w, const uint16_t* X, int64_t M,
                              const uint16_t* L1, const uint16_t* L2, int32_t r, float scale,
                              uint16_t* Y, uint16_t* T_save,
                              void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/* The forward in two parts, for callers that overlap T = X L1 with other work
 * (e.g. the weight's quantization on another stream):
 *   qlora_lora_down    T = X L1 (M x r, fp32 accumulation, rounded once to bf16),
 *                      the LoRA down-projection of eq. (3) on its own. Shapes as for
 *                      the linear (in % 256 == 0, r % 8 == 0, 8 <= r <= 256);
 *                      workspace of qlora_lora_down_workspace_size bytes, zeroed
 *                      once before first use (status word + split-K counters).
 *                      X device bf16 [M x in], L1 device bf16 [in x r], T device out
 *                      bf16 [M x r]; all 16-byte aligned.
 *   qlora_linear_fwd_t Y = X W_s^T + s T L2 with T supplied (device bf16 [M x r],
 *                      from qlora_lora_down or the caller); otherwise as
 *                      qlora_linear_fwd (same workspace size). Gives the bits of
 *                      qlora_linear_fwd when T is the same (as it is when that
 *                      call computes T as its own pass). */
size_t qlora_lora_down_workspace_size(int64_t M, int64_t in, int32_t r);
qlora_status qlora_lora_down(const uint16_t* X, int64_t M, int64_t in, const uint16_t* L1, int32_t r,
                             uint16_t* T, void* workspace, size_t workspace_bytes, qlora_stream_t stream);
qlora_status qlora_linear_fwd_t(const qlora_weight* w, const uint16_t* X, int64_t M, const uint16_t* T,
                                const uint16_t* L2, int32_t r, float scale, uint16_t* Y,
                                void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/* Backward of the forward above (no gradient for W):
 *   U   = dY L2^T                 (M x r, bf16 after fp32 accumulation)
 *   dX  = dY W_s + s U L1^T       (M x in, bf16)          -- skipped if dX == NULL
 *   dL2 = s T^T dY                (r x out, fp32)
 *   dL1 = s X^T U                 (in x r, fp32)
 *   T_saved  device bf16 [M x r] from the forward, or NULL to recompute T = X L1.
 * dX == NULL expresses an early backward stop below the lowest adapted layer
 * (AQLoRA section 3.3). dL1/dL2 are overwritten, not accumulated. Their
 * reductions run in a fixed order, so repeated calls give identical bits. With an
 * NF4 weight, U (and s U, the dX LoRA step's operand) can be computed inside the
 * dX GEMM, in one leading tile per 512 rows of dY: by default when in >= 8192 (32
 * column tiles of the output), QLORA_B200_FUSED_U=1 always, =0 never; U may then
 * differ in the last bf16 bit from U as its own pass, and dX and dL1 with it. */
qlora_status qlora_linear_bwd(const qlora_weight* w, const uint16_t* X, const uint16_t* dY, int64_t M,
                              const uint16_t* L1, const uint16_t* L2, int32_t r, float scale,
                              const uint16_t* T_saved, uint16_t* dX, float* dL1, float* dL2,
                              void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/* ------------------------------------------------------ AQLoRA allocation */

/* Workspace for nf4_layer_error_rank over n_layers matrices of the given
 * element counts (host array). */
size_t nf4_layer_error_rank_workspace_size(int32_t n_layers, const int64_t* numel);

/* Per-layer NF4 reconstruction error, ranking and top-K selection.
 *   W_ptrs   HOST array of n_layers DEVICE pointers, each a bf16 matrix
 *            (w_dtype must be QLORA_DTYPE_BF16), 16-byte aligned
 *   numel    HOST array of element counts (each a positive multiple of 64, at
 *            most 2^40; at most 2^31 - 1 chunks of 16384 in all)
 *   q        quantization config used for every layer (double_quant 0 or 1)
 *   K        number of layers to keep (0 <= K <= n_layers)
 *   err      device out, fp64 [n_layers]: e = sqrt(sum (w - w_hat)^2 / sum w^2)
 *            with w_hat the bf16 dequantized weight (0 for an all-zero matrix)
 *            A NaN or +-Inf weight sets QLORA_ERR_NONFINITE in the status word and
 *            leaves that layer's err unspecified (NaN errors rank first, by id).
 *   order    device out, int32 [n_layers]: layer ids by (err desc, id asc)
 *   keep     device out, uint8 [n_layers]: 1 for the first K of `order`
 * 1 <= n_layers <= 1024. Sums run in fp64 in a fixed order (deterministic). */
qlora_status nf4_layer_error_rank(int32_t n_layers, const uint16_t* const* W_ptrs, const int64_t* numel,
                                  int32_t w_dtype, nf4_qconfig q, int32_t K,
                                  double* err, int32_t* order, uint8_t* keep,
                                  void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/* The same pass with K taken from a memory budget ("AQLoRA: A Zero-Search Recipe
 * for Fast Quantized LoRA Fine-Tuning", section 3.2: the top-K layers are kept in
 * 16-bit under a memory budget). Keeping layer l in bf16 adds
 *   cost_l = 2 numel_l - (NF4 bytes of layer l: numel_l / 2 code bytes plus
 *            4 numel_l / 64 scale bytes, or with double quant numel_l / 64 E4M3
 *            bytes plus 4 ceil(numel_l / 16384) bytes)
 * to the all-NF4 model. K is the largest count such that the first K layers of
 * `order` add at most budget_bytes in total (0 <= budget_bytes; the budget is
 * inclusive).
 *   K_out    device out, int32 [1]
 * Other arguments, the workspace and the errors as for nf4_layer_error_rank;
 * numel_l <= 2^40. */
qlora_status nf4_layer_error_rank_budget(int32_t n_layers, const uint16_t* const* W_ptrs, const int64_t* numel,
                                         int32_t w_dtype, nf4_qconfig q, int64_t budget_bytes, double* err,
                                         int32_t* order, uint8_t* keep, int32_t* K_out, void* workspace,
                                         size_t workspace_bytes, qlora_stream_t stream);

/* The ranking step alone ("AQLoRA: A Zero-Search Recipe for Fast Quantized LoRA
 * Fine-Tuning", section 3.2: layers ranked by their error, the top K kept in 16-bit)
 * over errors already on the device, e.g. gathered from several GPUs that each
 * scored their own matrices:
 *   err    device fp64 [n_layers] (NaN ranks ahead of every number, by id)
 *   order  device out, int32 [n_layers]: layer ids by (err desc, id asc)
 *   keep   device out, uint8 [n_layers]: 1 for the first K of `order`
 * 1 <= n_layers <= 1024, 0 <= K <= n_layers. Deterministic: every caller with the
 * same errors gets the same order. No workspace. */
qlora_status nf4_rank_errors(int32_t n_layers, const double* err, int32_t K, int32_t* order, uint8_t* keep,
                             qlora_stream_t stream);

/* K from a protection fraction rho = num / den of n_layers layers (same page,
 * section 3.2, where rho = 0.2 of 144 linear layers keeps 29): round half up of
 * rho * n_layers, in exact integer arithmetic. Host only (no device work).
 *   0 <= num <= den, 0 < den <= 2^31, 0 <= n_layers <= 2^30; K host out. */
qlora_status nf4_k_from_fraction(int64_t num, int64_t den, int32_t n_layers, int32_t* K);

/* The allocation pass fused with the quantization it measures ("AQLoRA: A
 * Zero-Search Recipe for Fast Quantized LoRA Fine-Tuning", section 3.1-3.2: one
 * pass quantizes every linear layer to NF4 and scores its reconstruction error;
 * "QLoRA: How to fine-tune large language models with less memory", sections
 * "1. NormalFloat" and "2. Double quantization", for the storage). One read of
 * every matrix gives err / order / keep exactly as nf4_layer_error_rank and the
 * NF4 storage exactly as nf4_quantize, so the layers that are not kept need no
 * second pass.
 *   codes     HOST array of n_layers DEVICE pointers, uint8 [numel / 2] each,
 *             16-byte aligned
 *   absmax    HOST array of DEVICE pointers, fp32 [numel / 64]: required without
 *             double quant; with it the array, or any entry, may be NULL
 *   absmax_q, absmax2   HOST arrays of DEVICE pointers, E4M3 [numel / 64] and fp32
 *             [ceil(numel / 16384)]: required with double quant, else ignored
 * Other arguments, the workspace (nf4_layer_error_rank_workspace_size) and the
 * errors as for nf4_layer_error_rank; 1 <= n_layers <= 512 (the per-layer
 * pointers travel as one kernel parameter). */
qlora_status nf4_quantize_error_rank(int32_t n_layers, const uint16_t* const* W_ptrs, const int64_t* numel,
                                     int32_t w_dtype, nf4_qconfig q, int32_t K, uint8_t* const* codes,
                                     float* const* absmax, uint8_t* const* absmax_q, float* const* absmax2,
                                     double* err, int32_t* order, uint8_t* keep, void* workspace,
                                     size_t workspace_bytes, qlora_stream_t stream);

/* Allocation-free variant of nf4_layer_error_rank (the paper has no
 * counterpart; this is a convenience of the library).
 *
 * For callers that cannot allocate device memory at the point of the call:
 * runtimes that hand out device memory only from a fixed pool fixed at start-up
 * (so a workspace of this size may not exist), code running in a host callback
 * or an allocator hook where cudaMalloc is not allowed, and pipelines that
 * cannot afford cudaMalloc/cudaFree because those calls synchronize the device.
 * It takes the same inputs and outputs as nf4_layer_error_rank and no
 * workspace: the per-chunk partial sums live in a 16 MiB array inside the
 * library (one per GPU, kept until the process exits).
 *
 * Limits and behaviour:
 *   - at most 2^20 chunks of 16384 weights per call (sum over layers of
 *     ceil(numel/16384) <= 1048576, about 1.7e10 weights); larger calls return
 *     QLORA_ERR_SHAPE before any device work;
 *   - the first call on a device looks up the array's device address (with that
 *     device current) and caches it; make that first call before capturing any
 *     stream;
 *   - every call on a device uses the same array, so calls that overlap on the
 *     GPU (different streams or host threads) race and must be serialized by the
 *     caller; nothing needs clearing between calls;
 *   - there is no device status word. A layer that contains NaN or +-Inf, or a
 *     chunk of it whose bulk copy into shared memory timed out, gets err = NaN;
 *     NaN errors rank ahead of every finite error (among themselves by layer
 *     id), so `order` stays a permutation and such layers are the first kept.
 * Allocates no device memory and calls no allocating routine. */
qlora_status nf4_layer_error_rank_noalloc(int32_t n_layers, const uint16_t* const* W_ptrs, const int64_t* numel,
                                          int32_t w_dtype, nf4_qconfig q, int32_t K,
                                          double* err, int32_t* order, uint8_t* keep, qlora_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_B200_H */
