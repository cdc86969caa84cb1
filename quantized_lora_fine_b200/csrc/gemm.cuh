// Host-side interface of the tcgen05 GEMM engine (gemm.cu).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/qlora_b200.h"

namespace qlb {

struct GemmParams {
  int M;                  // rows of D
  int N;                  // columns of D (valid columns; partial tiles are predicated)
  int num_k_main;         // main K steps of 64
  int num_k_ext;          // LoRA extension K steps of 64 (only used when splits == 1)
  int tiles_m, tiles_n;   // tile grid
  int splits;             // split-K factor (fp32 partial output when > 1 or OUT_F32)
  int ksteps_per_split;   // main K steps per split
  int bn;                 // tile N (set by the launcher)
  void* out;              // bf16 [M x ld] or fp32 partials [splits][M x ld]
  int64_t ld_out;
  int64_t split_stride;   // elements between split partials
  int* status;            // device status word
  // Fused split-K reduction (thin products): when counters != nullptr, the last
  // CTA to finish a tile sums the split partials in split order and writes
  //   fin_mode 0: bf16 [M x N]            fin_mode 1: fp32 [M x N] * fin_scale
  //   fin_mode 2: fp32 [N x M] * fin_scale (transposed)
  // Counters (one int per M tile) must start at zero; the kernel leaves them zero.
  int* counters;
  void* fin_out;
  int fin_mode;       // 3: bf16 [M x N] to fin_out and bf16(fin_scale * that) to fin_out2
  float fin_scale;
  void* fin_out2;
  // CTA-pair NF4 kernel: packed codes [out x in/2] and expanded block scales S_t
  // [in/64 x out] (S_t[j][n] = scale of weight row n, block j), read directly by
  // the dequantizer warps (coalesced in both orientations)
  const uint8_t* codes;
  int64_t codes_ld;   // bytes between code rows (in / 2)
  const float* scales;
  int64_t scales_ld;  // floats between S_t rows (out)
  // Schedule of the 512 x 256 pair kernel (set by its launcher): sk_R rounds of whole
  // tiles (pair p takes tiles p + r sk_P), then the remaining tiles' steps as ranges of
  // sk_L steps, pair p taking [p sk_L, min((p + 1) sk_L, sk_W)) of the sk_W tail steps
  // (tail tile u is tile sk_base + u). A tile split over several pairs is finished by
  // the pair that holds its first step: it adds the others' fp32 partials (sk_part,
  // one slot per pair) in pair order once their counter (sk_count, two per tail tile,
  // left at zero) says they are written. With sk_A > 0 the first sk_A pairs (those
  // whose first round was an aux tile, about half a tile's work) take tail ranges of
  // sk_La steps instead: pair p < sk_A takes [p sk_La, (p + 1) sk_La), pair p >= sk_A
  // [sk_A sk_La + (p - sk_A) sk_L, + sk_L), all clipped to sk_W.
  int sk_P, sk_R, sk_L, sk_W, sk_base, sk_A, sk_La;
  float* sk_part;
  int* sk_count;
  // Forward of the 512 x 256 pair kernel with T = X L1 fused in: aux_tiles leading
  // "T tiles" (one per 512-row block, tile id = block) multiply the block's X rows by
  // L1 (loaded by TMA in place of a dequantized B) and store T (t_chunks 64-column
  // chunks) before raising the block's flag in t_flags; a main tile's first LoRA step
  // waits (bounded) for its block's flag. t_flags holds [flag, readers] per block and
  // CTA rank, left at zero (the last reader clears them). aux_tiles = 0: no T tiles.
  // The dX kernel's aux tiles are "U tiles" the same way: U = dY L2^T of the block
  // (A = the dY rows, B = L2 [r x out] read K-major), stored as U and, with aux_dual,
  // also as bf16(aux_scale * bf16(U)) to the second aux output (the LoRA step's A).
  int aux_tiles, t_chunks;
  int* t_flags;
  int aux_dual;
  float aux_scale;
};

struct GemmOperands {
  CUtensorMap A, B, codes, scales, Ax, Bx, Y, L1, Tout, Tout2;
};

enum class GemmKind {
  FwdNF4,   // A = X (K-major), B = dequantized W (K-major), + LoRA extension, bf16 out
  DxNF4,    // A = dY (K-major), B = dequantized W (MN-major), + LoRA extension, bf16 out
  FwdBF16,  // as FwdNF4 with a bf16 W loaded by TMA
  DxBF16,   // as DxNF4 with a bf16 W loaded by TMA
  ThinKK,   // fp32 partials, A K-major, B K-major
  ThinKM,   // fp32 partials, A K-major, B MN-major
  ThinMM,   // fp32 partials, A MN-major, B MN-major
};

enum class TmapType { BF16, U8, F32 };

// 2-D tensor map: `inner` elements per row (contiguous), `outer` rows,
// `row_bytes` between rows; box of box_inner x box_outer elements.
bool make_tmap_2d(CUtensorMap* m, const void* base, TmapType type, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128);
// Same with an explicit swizzle: 0 none, 32, 64 or 128 (bytes).
bool make_tmap_2d_sw(CUtensorMap* m, const void* base, TmapType type, uint64_t inner, uint64_t outer,
                     uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, int swizzle_bytes);

qlora_status launch_gemm(GemmKind kind, int bn, const GemmOperands& o, const GemmParams& p, cudaStream_t s);

// Fused NF4 GEMM on CTA pairs (256 x 256 tiles). Operands: A (box 64 x 128),
// codes (fwd: box 32 B x 128 rows; dX: box 64 B x 64 rows, 64-byte swizzle),
// scales (fwd: box 128 x 1; dX: box 64 x 2), Ax (box 64 x 128), Bx (box 64 x 128).
// Requires N % 256 == 0.
qlora_status launch_gemm_pair(bool dx, const GemmOperands& o, const GemmParams& p, cudaStream_t s);

// Fused NF4 GEMM on CTA pairs with 512 x 256 tiles (two M = 256 accumulators per
// decoded B stage) and a split last round. Operands as launch_gemm_pair plus Y (the
// output, box 64 x 128, 128-byte swizzle, written by TMA). The caller provides
// p.sk_part (pair2_partial_bytes(...) bytes) and p.sk_count (pair2_counter_ints(...)
// ints, zero); requires N % 256 == 0.
qlora_status launch_gemm_pair2(bool dx, const GemmOperands& o, GemmParams p, cudaStream_t s);
// The schedule over `pairs` co-resident pairs: {P, R, L, W, base, launch, A, La} (host only).
void pair2_schedule_of(int tiles, int aux_tiles, int steps, int pairs, int32_t* out);
// Upper bounds of the split-round scratch for a D[M x N] product (host only).
size_t pair2_partial_bytes(int64_t M, int64_t N);
constexpr int kPair2MaxPairs = 80;                 // pairs launched at most
constexpr int kPair2CounterInts = 2 * kPair2MaxPairs;   // two per split tile
// T fused into the forward: 4 ints per 512-row block after the split-tile counters, so
// at most this many blocks (M <= 110592 tokens); larger M runs T as its own pass.
constexpr int kPair2MaxTBlocks = 216;

}  // namespace qlb
