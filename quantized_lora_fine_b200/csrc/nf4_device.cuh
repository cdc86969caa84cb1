// Device-side NF4 helpers shared by the codec, error-pass and GEMM kernels.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "nf4_constants.cuh"

namespace qlb {

__device__ __forceinline__ float nf4_code(int j) { return __uint_as_float(kNF4CodeBits[j]); }

// Index of the nearest code for a normalised value n: #{j : n > m_j}.
__device__ __forceinline__ uint32_t nf4_index(float n) {
  uint32_t idx = 0;
#pragma unroll
  for (int j = 0; j < 15; ++j) idx += (n > __uint_as_float(kNF4MidBits[j])) ? 1u : 0u;
  return idx;
}

// Shared-memory copy of the cell tables (64 thresholds + 64 base indices).
struct NF4CellSmem {
  float thr[64];
  uint32_t base[64];
};

__device__ __forceinline__ void nf4_cells_load(NF4CellSmem& t, int tid) {
  if (tid < 64) {
    t.thr[tid] = __uint_as_float(kNF4CellThrBits[tid]);
    t.base[tid] = kNF4CellBase[tid];
  }
}

// Same result as nf4_index(n) for every fp32 n (NaN maps to some index; callers
// flag non-finite input separately): the cell of n holds at most one midpoint.
__device__ __forceinline__ uint32_t nf4_index_cell(float n, const NF4CellSmem& t) {
  const uint32_t c = (__float_as_uint(__fadd_rn(n, 3.0f)) >> 18) & 63u;
  return t.base[c] + ((n > t.thr[c]) ? 1u : 0u);
}

// Correctly rounded w / a from r = RN(1/a) with one residual correction
// (Markstein's division step: q0 = RN(w r), e = w - q0 a exactly by FMA,
// q = RN(q0 + e r)). Requires a normal, finite a with 1/a normal; the callers
// rescale tiny blocks by 2^64 first. Checked against IEEE division for every
// (bf16 w, bf16 a) significand / exponent-gap combination by the GPU tests.
__device__ __forceinline__ float div_by_recip(float w, float a, float r) {
  const float q0 = __fmul_rn(w, r);
  const float e = __fmaf_rn(-q0, a, w);
  return __fmaf_rn(e, r, q0);
}

// Normalised value n = RN(w / a) for a block with absmax a > 0. bf16 inputs take
// the reciprocal path (exact for every bf16 pair, see div_by_recip); fp32 inputs
// use IEEE division directly.
template <typename T>
struct BlockDiv {
  float a, r;
  __device__ __forceinline__ BlockDiv(float am) {
    // Tiny blocks: rescale by 2^64 (exact) so that 1/a stays a normal number.
    a = (am < 0x1p-100f) ? am * 0x1p64f : am;
    r = __frcp_rn(a);
  }
  __device__ __forceinline__ float operator()(float w, float am) const {
    if constexpr (sizeof(T) == 2) {
      return div_by_recip((am < 0x1p-100f) ? w * 0x1p64f : w, a, r);
    } else {
      return __fdiv_rn(w, am);
    }
  }
};

// bf16 bit pattern of max |w| over 8 elements held as 4 packed bf16 pairs.
// Comparing magnitudes as unsigned integers orders +Inf and NaN above every
// finite value, so a result >= 0x7F80 flags a non-finite element.
__device__ __forceinline__ uint32_t absmax8_bf16_bits(uint4 v) {
  const uint32_t a = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
  const uint32_t b = __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu);
  const uint32_t m = __vmaxu2(a, b);
  return max(m >> 16, m & 0xFFFFu);
}

// Max over the 8 lanes (l ^ 1, l ^ 2, l ^ 4) that share one 64-element block.
__device__ __forceinline__ uint32_t block_max8_lanes(uint32_t v) {
  v = max(v, __shfl_xor_sync(0xffffffffu, v, 1));
  v = max(v, __shfl_xor_sync(0xffffffffu, v, 2));
  v = max(v, __shfl_xor_sync(0xffffffffu, v, 4));
  return v;
}

// Codes of 8 bf16 weights (4 packed pairs) of a block with absmax a > 0, packed in
// storage order (byte k = idx[2k] << 4 | idx[2k + 1]).
__device__ __forceinline__ uint32_t quant8_bf16(uint4 v, float a, const NF4CellSmem& cells, uint32_t (&idx)[8]) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  float w[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) { w[2 * i] = __uint_as_float(u[i] << 16); w[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u); }
  float as = a;
  if (a < 0x1p-100f) {  // tiny block: rescale by 2^64 (exact) so that 1/a stays normal
    as = a * 0x1p64f;
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] *= 0x1p64f;
  }
  const float r = __frcp_rn(as);
#pragma unroll
  for (int i = 0; i < 8; ++i) idx[i] = nf4_index_cell(div_by_recip(w[i], as, r), cells);
  // byte k = idx[2k] << 4 | idx[2k+1]; integer multiply-adds keep this off the ALU pipe
  uint32_t word = idx[1];
  word = idx[0] * 16u + word;
  word = idx[3] * 256u + word;
  word = idx[2] * 4096u + word;
  word = idx[5] * 65536u + word;
  word = idx[4] * 1048576u + word;
  word = idx[7] * 16777216u + word;
  word = idx[6] * 268435456u + word;
  return word;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t bitselect(uint32_t a, uint32_t b, uint32_t m) {
  // (a & ~m) | (b & m); lut 0xCA = (x & y) | (~x & z) with x = m, y = b, z = a
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xCA;" : "=r"(d) : "r"(m), "r"(b), "r"(a));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic: two IEEE fp32 operations in one
// instruction, round to nearest, subnormals kept)
__device__ __forceinline__ uint64_t f2_from_bf16x2(uint32_t u) {
  // (element 0, element 1) of a bf16 pair as a packed fp32 pair
  return (uint64_t(u & 0xFFFF0000u) << 32) | uint64_t(u << 16);
}
__device__ __forceinline__ uint64_t f2_splat(float x) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float(uint32_t(v)); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float(uint32_t(v >> 32)); }
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// RN(w / a) for both elements of a pair, from r = RN(1/a) and na = -a (Markstein
// step, as div_by_recip).
__device__ __forceinline__ uint64_t f2_div_by_recip(uint64_t w, uint64_t na, uint64_t r) {
  const uint64_t q0 = f2_mul(w, r);
  const uint64_t e = f2_fma(q0, na, w);
  return f2_fma(e, r, q0);
}

// ---- fine-cell code lookup, evaluated on the FMA pipe
// Cell c = bits(n) >> 21 (2048 cells of 1/4 binade; each holds at most one
// midpoint). s = sat(n * 2^100 + T_c) is exactly 1.0 when n is above the cell's
// midpoint and 0.0 otherwise; the code index is base_c + s.
__device__ __forceinline__ float sat_fma(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float2 fine_q_entry(const float2* tbl, float n) {
  return tbl[__float_as_uint(n) >> 21];
}
// Coarse cell c = floor(16 (n + 1)) for n in [-1, 1], as a shared-memory address
// without integer ALU work: bits(RZ(16 n + 16 + 2^23)) = 0x4B000000 + c, and one
// integer multiply-add (mod 2^32) turns that into tbl + c * entry_bytes.
template <uint32_t kEntryBytes>
__device__ __forceinline__ uint32_t coarse_addr(float n, uint32_t tbl) {
  float v;
  asm("fma.rz.f32 %0, %1, 0f41800000, 0f4B000010;" : "=f"(v) : "f"(n));   // 16 n + (2^23 + 16)
  return __float_as_uint(v) * kEntryBytes + (tbl - 0x4B000000u * kEntryBytes);
}
// Both cells of a packed pair: bits of RZ(16 n + 16 + 2^23) per lane.
__device__ __forceinline__ uint64_t coarse_cells2(uint64_t n2) {
  uint64_t v;
  asm("fma.rz.f32x2 %0, %1, %2, %3;" : "=l"(v) : "l"(n2), "l"(0x4180000041800000ull), "l"(0x4B0000104B000010ull));
  return v;
}
template <uint32_t kEntryBytes>
__device__ __forceinline__ uint32_t coarse_addr_bits(uint32_t cell_bits, uint32_t tbl) {
  return cell_bits * kEntryBytes + (tbl - 0x4B000000u * kEntryBytes);
}
__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}
// Four code indices accumulated as sum idx_p * 16^p in fp32 (exact below 2^16)
// turn into integer bits through the 2^23 bias: low 16 bits of bits(h + 2^23).
__device__ __forceinline__ uint32_t nibbles_from_f32(float h) {
  return __float_as_uint(__fadd_rn(h, 8388608.0f));
}

// Per-block dequantization table: the 16 products bf16_rn(fp32_rn(c_j * a)) split
// into a low-byte table (lo[0..3], byte j = low byte of entry j) and a high-byte
// table (hi[0..3]).
struct NF4Lut {
  uint32_t lo[4];
  uint32_t hi[4];
};

__device__ __forceinline__ NF4Lut nf4_make_lut(float a) {
  uint32_t p[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) p[j] = pack_bf16x2(nf4_code(2 * j) * a, nf4_code(2 * j + 1) * a);
  NF4Lut t;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    t.lo[q] = prmt(p[2 * q], p[2 * q + 1], 0x6420u);
    t.hi[q] = prmt(p[2 * q], p[2 * q + 1], 0x7531u);
  }
  return t;
}

// Dequantize 8 packed codes (one little-endian 32-bit word = 4 code bytes; byte k
// holds element 2k in its high nibble) into 8 bf16 values (a 16-byte chunk, element
// 0 in the lowest half-word).
__device__ __forceinline__ uint4 nf4_dequant_word(uint32_t w, const NF4Lut& t) {
  const uint32_t s = w & 0x77777777u;                                   // table index within a half
  const uint32_t sm = (w & 0x88888888u) | ((w >> 3) & 0x11111111u);      // sign-replicate selector
  uint32_t out[4];
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const uint32_t sg = g ? (s >> 16) : s;
    const uint32_t mg = g ? (sm >> 16) : sm;
    const uint32_t m = prmt(0x00008000u, 0u, mg);   // byte i = 0xFF iff nibble i >= 8
    const uint32_t lo = bitselect(prmt(t.lo[0], t.lo[1], sg), prmt(t.lo[2], t.lo[3], sg), m);
    const uint32_t hi = bitselect(prmt(t.hi[0], t.hi[1], sg), prmt(t.hi[2], t.hi[3], sg), m);
    // nibble order within a byte pair is (odd, even); reorder to (even, odd)
    out[2 * g] = prmt(lo, hi, 0x4051u);
    out[2 * g + 1] = prmt(lo, hi, 0x6273u);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// fp32 value of an E4M3 scale byte (exact).
__device__ __forceinline__ float e4m3_to_f32(uint8_t q) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(q), __NV_E4M3);
  return __half2float(__half(h));
}

__device__ __forceinline__ uint8_t f32_to_e4m3_satfinite(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

}  // namespace qlb
