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
};

struct GemmOperands {
  CUtensorMap A, B, codes, scales, Ax, Bx;
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

qlora_status launch_gemm(GemmKind kind, int bn, const GemmOperands& o, const GemmParams& p, cudaStream_t s);

}  // namespace qlb
