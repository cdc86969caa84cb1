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

// max(|a|, |b|) per bf16 lane (the sign bit holds the xor of the operands' signs);
// a NaN operand gives NaN, so the masked magnitude of a chain flags any NaN or Inf
// by being >= 0x7F80.
__device__ __forceinline__ uint32_t bf16x2_maxabs(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
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
// ---- code index of a normalised value: FMA-pipe arithmetic and warp shuffles
// A block with absmax a is processed with a power-of-two scale sc (1, or 2^64 /
// 2^-64 for tiny / huge blocks) so that r = RN(1/(a sc)) is a normal number; a
// weight's scaled quotient is n_s = RN(w r) = n~ / sc with n~ = RN(w RN(1/a)).
// Cell c = floor(15.75 n~ + 16) in [0, 31] of both elements of a pair: the low 5
// bits of RZ(n_s (15.75 sc) + 2^23 + 16).
__device__ __forceinline__ uint64_t cells2(uint64_t ns2, uint64_t cmul2) {
  uint64_t v;
  asm("fma.rz.f32x2 %0, %1, %2, %3;" : "=l"(v) : "l"(ns2), "l"(cmul2), "l"(0x4B0000104B000010ull));
  return v;
}
__device__ __forceinline__ float sat_fma(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// This lane's entries of the lookup tables: lane l holds cell l's B and T and
// code[l mod 16] (a kernel loads the ones it uses).
struct LaneTables {
  float B, T, code;
};
__device__ __forceinline__ LaneTables lane_tables(int lane) {
  LaneTables t;
  t.B = __uint_as_float(kNF4LaneB[lane]);
  t.T = __uint_as_float(kNF4LaneT[lane]);
  t.code = __uint_as_float(kNF4CodeBits[lane & 15]);
  return t;
}
// Index bits 0x4B000000 + idx of one element from its scaled quotient and cell bits:
// b = B[cell] and t = T[cell] by two independent shuffles (a shuffle uses the low 5
// bits of its lane operand), s = sat(n_s M + t) in {0, 1} with M = 2^36 sc, bits(b + s).
// Every lane of the warp must call it.
__device__ __forceinline__ uint32_t index_bits(float ns, uint32_t cell_bits, float M, const LaneTables& lt) {
  const float b = __shfl_sync(0xffffffffu, lt.B, int(cell_bits));
  const float t = __shfl_sync(0xffffffffu, lt.T, int(cell_bits));
  return __float_as_uint(b + sat_fma(ns, M, t));
}
// Code value of index bits x (lane x mod 32 holds code[x mod 16]).
__device__ __forceinline__ float code_value(uint32_t x, const LaneTables& lt) {
  return __shfl_sync(0xffffffffu, lt.code, int(x));
}
// Per-block constants of the lookup: r = RN(1/(a sc)) and the two multipliers.
struct CellScale {
  uint64_t r2, cmul2;
  float M;
  __device__ __forceinline__ explicit CellScale(float a) {
    const float sc = (a < 0x1p-100f) ? 0x1p64f : (a > 0x1p100f) ? 0x1p-64f : 1.f;
    r2 = f2_splat(__frcp_rn(a * sc));
    cmul2 = f2_splat(15.75f * sc);
    M = 0x1p36f * sc;
  }
};
// The 8 elements of a piece (4 packed bf16 pairs, storage order) -> index bits x[k].
// Every lane of the warp must call it.
__device__ __forceinline__ void piece_index_bits(const uint32_t (&u)[4], const CellScale& cs, const LaneTables& lt,
                                                 uint32_t (&x)[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint64_t q = f2_mul(f2_from_bf16x2(u[i]), cs.r2);
    const uint64_t c = cells2(q, cs.cmul2);
    x[2 * i] = index_bits(f2_lo(q), uint32_t(c), cs.M, lt);
    x[2 * i + 1] = index_bits(f2_hi(q), uint32_t(c >> 32), cs.M, lt);
  }
}
// {bf16 lo(h) - a.x, bf16 hi(h) - a.y} in fp32: the bf16 halves enter exactly
// (mixed-precision subtraction), one rounding each.
__device__ __forceinline__ uint64_t f2_bf16x2_minus(uint32_t h, uint64_t a) {
  uint64_t d;
  asm("{\n\t.reg .b16 l, u;\n\t.reg .f32 a0, a1, d0, d1;\n\t"
      "mov.b32 {l, u}, %1;\n\tmov.b64 {a0, a1}, %2;\n\t"
      "sub.rn.f32.bf16 d0, l, a0;\n\tsub.rn.f32.bf16 d1, u, a1;\n\t"
      "mov.b64 %0, {d0, d1};\n\t}"
      : "=l"(d) : "r"(h), "l"(a));
  return d;
}
// Undo a thread's piece rotation: word j was computed for position j ^ rot; after
// this, w[p] holds position p (three conditional exchange stages, one per bit).
__device__ __forceinline__ void unrotate8(uint32_t (&w)[8], uint32_t rot) {
#pragma unroll
  for (int b = 0; b < 3; ++b) {
    const bool sw = (rot >> b) & 1u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i & (1 << b)) continue;
      const uint32_t x = w[i], y = w[i | (1 << b)];
      w[i] = sw ? y : x;
      w[i | (1 << b)] = sw ? x : y;
    }
  }
}
// Code word of a piece (byte k = idx[2k] << 4 | idx[2k + 1]) from its index bits by a
// multiply-add chain mod 2^32: the 0x4B000000 of each term survives only from the
// last two terms (0x4B000000 + 0xB0000000), which the final add cancels.
__device__ __forceinline__ uint32_t pack_code_word(const uint32_t (&x)[8]) {
  uint32_t acc = x[6];
  acc = acc * 16u + x[7];
  acc = acc * 16u + x[4];
  acc = acc * 16u + x[5];
  acc = acc * 16u + x[2];
  acc = acc * 16u + x[3];
  acc = acc * 16u + x[0];
  acc = acc * 16u + x[1];
  return acc + 0x05000000u;
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
