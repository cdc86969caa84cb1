// tcgen05 GEMM engine for sm_100a.
//
//   D[M x N] = A[M x K] * B[N x K]^T  (+ A_ext[M x r] * B_ext[N x r]^T)
//
// Tiles of 128 x BN x 64 (bf16 in, fp32 accumulate in tensor memory), a
// persistent grid, warp-specialised roles:
//   warp 0      TMA producer (one elected lane): A tiles, and either B tiles
//               (bf16 operand) or packed NF4 codes + expanded scales
//   warp 1      TMEM allocator and MMA issuer (one elected lane)
//   warps 2-5   epilogue: tcgen05.ld -> registers -> global (bf16 or fp32)
//   warps 6-13  (NF4 operand only) dequantizers: packed codes in shared memory
//               -> bf16 B tile in the 128-byte-swizzled UMMA layout, through a
//               per-block 16-entry product table (prmt byte lookups)
// Stage hand-off uses mbarriers; MMA completion is signalled with
// tcgen05.commit; the accumulator is double-buffered in TMEM so that the
// epilogue of one tile overlaps the mainloop of the next.
//
// Operand layouts in shared memory (all 128-byte swizzle, 1024-byte aligned):
//   K-major  : rows x 64 elements (128 B per row); 8-row groups 1024 B apart.
//   MN-major : [MN/64 chunks][64 K rows][64 elements]; chunk stride 8 KB.
// The LoRA term is appended as extra K steps whose A and B tiles are loaded by
// TMA (T or U, and the scaled L2^T or L1), zero-filled beyond r.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "gemm.cuh"
#include "internal.cuh"
#include "nf4_device.cuh"
#include "ptx.cuh"

namespace qlb {

// --------------------------------------------------------------- config

template <int BN_, bool A_MN_, bool B_MN_, bool NF4_, bool OUT_F32_, int STAGES_>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64, BN = BN_;
  static constexpr bool A_MN = A_MN_, B_MN = B_MN_, NF4 = NF4_, OUT_F32 = OUT_F32_;
  static constexpr int STAGES = STAGES_;
  static constexpr int kA = BM * BK * 2;
  static constexpr int kB = BN * BK * 2;
  static constexpr int kCodes = NF4 ? BN * BK / 2 : 0;
  static constexpr int kScales = NF4 ? BN * 4 : 0;  // fwd: BN scales; dX: 64 rows x BN/64 blocks
  static constexpr int kCodesOff = kA + kB;
  static constexpr int kScalesOff = kCodesOff + ((kCodes + 1023) / 1024) * 1024;
  static constexpr int kStage = kScalesOff + ((kScales + 1023) / 1024) * 1024;
  static constexpr int kDequantWarps = NF4 ? 8 : 0;
  static constexpr int kThreads = (6 + kDequantWarps) * 32;
  static constexpr int kTmemCols = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                   : (2 * BN <= 256) ? 256 : 512;
  static constexpr int kBarBytes = 8 * (3 * STAGES + 5) + 16;
  static constexpr int kSmem = STAGES * kStage + kBarBytes + 1024;  // + alignment slack
  static_assert(BN % 16 == 0 && BN <= 256, "tcgen05 M=128 needs N % 16 == 0, N <= 256");
  static_assert(!B_MN || BN % 64 == 0, "MN-major B tiles are 64-element chunks");
  static_assert(!NF4 || BN == 256, "dequant mapping assumes BN = 256");
  static_assert(kSmem <= 232448, "shared memory budget");
};

// --------------------------------------------------------------- tile decode

struct TileInfo {
  int m0, n0, split, kb, ke;  // main k-step range [kb, ke)
  int n_ext;
};

__device__ __forceinline__ TileInfo decode_tile(const GemmParams& p, int t) {
  TileInfo ti;
  const int per_split = p.tiles_m * p.tiles_n;
  ti.split = t / per_split;
  const int r = t - ti.split * per_split;
  const int mb = r / p.tiles_n, nb = r - mb * p.tiles_n;
  ti.m0 = mb * 128;
  ti.n0 = nb * p.bn;
  ti.kb = ti.split * p.ksteps_per_split;
  ti.ke = min(p.num_k_main, ti.kb + p.ksteps_per_split);
  ti.n_ext = (p.splits == 1) ? p.num_k_ext : 0;
  return ti;
}

// --------------------------------------------------------------- dequant stage

// fwd (K-major B): thread t owns B row n = t (one 64-element block per stage).
// dX  (MN-major B): thread t owns K row (t % 64) and 64-column chunk (t / 64).
template <bool B_MN>
__device__ __forceinline__ void dequant_stage(uint32_t t, const uint8_t* codes_s, const float* scales_s,
                                              uint32_t b_tile) {
  uint32_t row, chunk, code_off0, code_off1;
  float a;
  if constexpr (!B_MN) {
    row = t;
    chunk = 0;
    code_off0 = t * 32;
    code_off1 = t * 32 + 16;
    a = scales_s[t];
  } else {
    row = t & 63u;
    chunk = t >> 6;
    const uint32_t sw = row & 7u;
    code_off0 = row * 128 + (((2 * chunk) ^ sw) << 4);
    code_off1 = row * 128 + (((2 * chunk + 1) ^ sw) << 4);
    a = scales_s[chunk * 64 + row];
  }
  const uint4 c0 = *reinterpret_cast<const uint4*>(codes_s + code_off0);
  const uint4 c1 = *reinterpret_cast<const uint4*>(codes_s + code_off1);
  const NF4Lut lut = nf4_make_lut(a);
  const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const uint32_t sw = row & 7u;
  const uint32_t row_base = b_tile + (B_MN ? chunk * 8192u : 0u) + (row >> 3) * 1024u + sw * 128u;
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c) {
    const uint4 v = nf4_dequant_word(words[c], lut);
    const uint32_t addr = row_base + ((c ^ sw) << 4);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
  }
}

// --------------------------------------------------------------- kernel

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmCodes, const __grid_constant__ CUtensorMap tmScales,
                   const __grid_constant__ CUtensorMap tmAx, const __grid_constant__ CUtensorMap tmBx,
                   const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t smem_base = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::kStage);
  const uint32_t bar_base = smem_u32(bars);
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto deq_bar = [&](int s) { return bar_base + 8u * (C::STAGES + s); };
  auto empty_bar = [&](int s) { return bar_base + 8u * (2 * C::STAGES + s); };
  auto tfull_bar = [&](int a) { return bar_base + 8u * (3 * C::STAGES + a); };
  auto tempty_bar = [&](int a) { return bar_base + 8u * (3 * C::STAGES + 2 + a); };
  const uint32_t drain_bar = bar_base + 8u * (3 * C::STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * C::STAGES + 5);

  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ uint32_t s_last;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(deq_bar(s), C::kDequantWarps > 0 ? C::kDequantWarps : 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4);
    }
    mbar_init(drain_bar, 1);
    fence_mbarrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_launch();

  const int num_tiles = p.tiles_m * p.tiles_n * p.splits;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      if (!C::NF4) tma_prefetch_desc(&tmB);
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const TileInfo ti = decode_tile(p, t);
        const int nsteps = (ti.ke - ti.kb) + ti.n_ext;
        for (int j = 0; j < nsteps; ++j, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1u;
          if (!mbar_wait(empty_bar(s), ph ^ 1u)) { set_status_site(p.status, QLORA_ERR_TIMEOUT, 1); ok = false; break; }
          const uint32_t st = smem_base + s * C::kStage;
          const uint32_t a_s = st, b_s = st + C::kA;
          if (j < ti.ke - ti.kb) {
            const int ks = ti.kb + j;
            const int k0 = ks * 64;
            const uint32_t bytes = C::kA + (C::NF4 ? (C::kCodes + C::kScales) : C::kB);
            mbar_arrive_expect_tx(full_bar(s), bytes);
            if constexpr (!C::A_MN) {
              tma_load_2d(a_s, &tmA, full_bar(s), k0, ti.m0);
            } else {
              tma_load_2d(a_s, &tmA, full_bar(s), ti.m0, k0);
              tma_load_2d(a_s + 8192, &tmA, full_bar(s), ti.m0 + 64, k0);
            }
            if constexpr (C::NF4) {
              if constexpr (!C::B_MN) {
                tma_load_2d(st + C::kCodesOff, &tmCodes, full_bar(s), k0 / 2, ti.n0);
                tma_load_2d(st + C::kScalesOff, &tmScales, full_bar(s), ti.n0, ks);
              } else {
                tma_load_2d(st + C::kCodesOff, &tmCodes, full_bar(s), ti.n0 / 2, k0);
                tma_load_2d(st + C::kScalesOff, &tmScales, full_bar(s), k0, ti.n0 / 64);
              }
            } else {
              if constexpr (!C::B_MN) {
                tma_load_2d(b_s, &tmB, full_bar(s), k0, ti.n0);
              } else {
#pragma unroll
                for (int c = 0; c < C::BN / 64; ++c) tma_load_2d(b_s + c * 8192, &tmB, full_bar(s), ti.n0 + 64 * c, k0);
              }
            }
          } else {
            const int kx = (j - (ti.ke - ti.kb)) * 64;
            mbar_arrive_expect_tx(full_bar(s), C::kA + C::kB);
            tma_load_2d(a_s, &tmAx, full_bar(s), kx, ti.m0);
            tma_load_2d(b_s, &tmBx, full_bar(s), kx, ti.n0);
          }
        }
      }
      // Do not leave while copies this thread issued may still be landing.
      if (it > 0) {
        const uint32_t last = it - 1;
        for (int k = 0; k < C::STAGES && k <= int(last); ++k) {
          const uint32_t i2 = last - k;
          mbar_wait(full_bar(i2 % C::STAGES), (i2 / C::STAGES) & 1u, 100000000ull);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_main = make_idesc_bf16(128, C::BN, C::A_MN ? 1 : 0, C::B_MN ? 1 : 0);
      constexpr uint32_t idesc_ext = make_idesc_bf16(128, C::BN, 0, 0);
      // K advance per 16-element MMA step: 32 B inside a K-major row; 2 x 8-row
      // groups (2048 B) in an MN-major tile.
      constexpr uint32_t a_adv = C::A_MN ? 2048u : 32u;
      constexpr uint32_t b_adv = C::B_MN ? 2048u : 32u;
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++tcount) {
        const TileInfo ti = decode_tile(p, t);
        const int nsteps = (ti.ke - ti.kb) + ti.n_ext;
        const uint32_t acc = tcount & 1u, tph = (tcount >> 1) & 1u;
        if (!mbar_wait(tempty_bar(acc), tph ^ 1u)) { set_status_site(p.status, QLORA_ERR_TIMEOUT, 2); ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * C::BN;
        for (int j = 0; j < nsteps; ++j, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1u;
          if (!mbar_wait(full_bar(s), ph)) { set_status_site(p.status, QLORA_ERR_TIMEOUT, 3); ok = false; break; }
          if (C::NF4 && !mbar_wait(deq_bar(s), ph)) { set_status_site(p.status, QLORA_ERR_TIMEOUT, 4); ok = false; break; }
          tc_fence_after();
          const uint32_t st = smem_base + s * C::kStage;
          const bool ext = j >= ti.ke - ti.kb;
          const uint32_t a_lbo = (!ext && C::A_MN) ? 8192u : 16u;
          const uint32_t b_lbo = (!ext && C::B_MN) ? 8192u : 16u;
          const uint64_t adesc = make_smem_desc(st, a_lbo, 1024u, kSwizzle128B);
          const uint64_t bdesc = make_smem_desc(st + C::kA, b_lbo, 1024u, kSwizzle128B);
          const uint32_t aadv = ext ? 32u : a_adv, badv = ext ? 32u : b_adv;
          const uint32_t idesc = ext ? idesc_ext : idesc_main;
#pragma unroll
          for (uint32_t kk = 0; kk < 4; ++kk) {
            tc_mma_bf16(d_tmem, adesc + uint64_t((kk * aadv) >> 4), bdesc + uint64_t((kk * badv) >> 4), idesc,
                        (j > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(empty_bar(s));
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));
      }
      // all MMAs issued by this thread are complete once drain_bar flips
      tc_commit(drain_bar);
      mbar_wait(drain_bar, 0, 100000000ull);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const uint32_t q = warp & 3u;
    const uint32_t row = q * 32 + lane;
    uint32_t tcount = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++tcount) {
      const TileInfo ti = decode_tile(p, t);
      const uint32_t acc = tcount & 1u, tph = (tcount >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(tfull_bar(acc), tph))) {
        set_status_site(p.status, QLORA_ERR_TIMEOUT, 5); break;
      }
      tc_fence_after();
      const int grow = ti.m0 + int(row);
      const uint32_t tbase = tmem_base + ((q * 32u) << 16) + acc * C::BN;
#pragma unroll 1
      for (int c = 0; c < C::BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + c * 32, v);
        tmem_ld_wait();
        const int col0 = ti.n0 + c * 32;
        if (grow < p.M) {
          if constexpr (C::OUT_F32) {
            float* dst = reinterpret_cast<float*>(p.out) + int64_t(ti.split) * p.split_stride +
                         int64_t(grow) * p.ld_out + col0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              if (col0 + 4 * i + 4 <= p.N)
                reinterpret_cast<float4*>(dst)[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                                __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            }
          } else {
            uint16_t* dst = reinterpret_cast<uint16_t*>(p.out) + int64_t(grow) * p.ld_out + col0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (col0 + 8 * i + 8 <= p.N) {
                uint4 o;
                o.x = pack_bf16x2(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]));
                o.y = pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]));
                o.z = pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]));
                o.w = pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]));
                reinterpret_cast<uint4*>(dst)[i] = o;
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      if constexpr (C::OUT_F32) {
        if (p.counters != nullptr) {
          // Split-K finish: the last of the `splits` CTAs of this M tile reduces.
          const int mt = t % (p.tiles_m * p.tiles_n);
          __threadfence();
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (warp == 2 && lane == 0) s_last = (atomicAdd(p.counters + mt, 1) == p.splits - 1) ? 1u : 0u;
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (s_last) {
            __threadfence();
            if (grow < p.M) {
              const float* src = reinterpret_cast<const float*>(p.out) + int64_t(grow) * p.ld_out;
              for (int c4 = 0; c4 < p.N; c4 += 4) {
                float4 acc4 = *reinterpret_cast<const float4*>(src + c4);
                for (int sp = 1; sp < p.splits; ++sp) {
                  const float4 v4 = *reinterpret_cast<const float4*>(src + int64_t(sp) * p.split_stride + c4);
                  acc4.x += v4.x; acc4.y += v4.y; acc4.z += v4.z; acc4.w += v4.w;
                }
                if (p.fin_mode == 0) {
                  uint2 o2;
                  o2.x = pack_bf16x2(acc4.x, acc4.y);
                  o2.y = pack_bf16x2(acc4.z, acc4.w);
                  *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(p.fin_out) + int64_t(grow) * p.N + c4) = o2;
                } else if (p.fin_mode == 3) {
                  uint2 o2;
                  o2.x = pack_bf16x2(acc4.x, acc4.y);
                  o2.y = pack_bf16x2(acc4.z, acc4.w);
                  *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(p.fin_out) + int64_t(grow) * p.N + c4) = o2;
                  // the same bf16 values times the LoRA scale, rounded once more to bf16
                  uint2 s2;
                  s2.x = pack_bf16x2(__fmul_rn(__uint_as_float(o2.x << 16), p.fin_scale),
                                     __fmul_rn(__uint_as_float(o2.x & 0xFFFF0000u), p.fin_scale));
                  s2.y = pack_bf16x2(__fmul_rn(__uint_as_float(o2.y << 16), p.fin_scale),
                                     __fmul_rn(__uint_as_float(o2.y & 0xFFFF0000u), p.fin_scale));
                  *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(p.fin_out2) + int64_t(grow) * p.N + c4) = s2;
                } else if (p.fin_mode == 1) {
                  float* d = reinterpret_cast<float*>(p.fin_out) + int64_t(grow) * p.N + c4;
                  *reinterpret_cast<float4*>(d) = make_float4(__fmul_rn(acc4.x, p.fin_scale), __fmul_rn(acc4.y, p.fin_scale),
                                                              __fmul_rn(acc4.z, p.fin_scale), __fmul_rn(acc4.w, p.fin_scale));
                } else {
                  float* d = reinterpret_cast<float*>(p.fin_out);
                  d[int64_t(c4 + 0) * p.M + grow] = __fmul_rn(acc4.x, p.fin_scale);
                  d[int64_t(c4 + 1) * p.M + grow] = __fmul_rn(acc4.y, p.fin_scale);
                  d[int64_t(c4 + 2) * p.M + grow] = __fmul_rn(acc4.z, p.fin_scale);
                  d[int64_t(c4 + 3) * p.M + grow] = __fmul_rn(acc4.w, p.fin_scale);
                }
              }
            }
            if (warp == 2 && lane == 0) p.counters[mt] = 0;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ dequantizers
    if constexpr (C::NF4) {
      const uint32_t dt = threadIdx.x - 192;
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const TileInfo ti = decode_tile(p, t);
        const int nsteps = (ti.ke - ti.kb) + ti.n_ext;
        for (int j = 0; j < nsteps; ++j, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1u;
          if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), ph))) {
            set_status_site(p.status, QLORA_ERR_TIMEOUT, 6); ok = false; break;
          }
          if (j < ti.ke - ti.kb) {
            uint8_t* st = smem + s * C::kStage;
            dequant_stage<C::B_MN>(dt, st + C::kCodesOff, reinterpret_cast<const float*>(st + C::kScalesOff),
                                   smem_base + s * C::kStage + C::kA);
            fence_proxy_async_smem();
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(deq_bar(s));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// =============================================================== CTA-pair kernel
//
// Fused NF4 GEMM on a pair of CTAs (cluster of 2, tcgen05 cta_group::2).
// One pair tile is 256 (M) x 256 (N), one M = 256, N = 256 accumulator (double
// buffered in TMEM). Each CTA stages its 128 rows of A by TMA and dequantizes its
// 128-wide half of B; every MMA reads 4 KB of A and 4 KB of B per CTA per 128
// tensor cycles, and each A byte fetched from L2 feeds 256 output columns.
//
// Shared memory per CTA: S slots, each holding A (this CTA's 128 rows, or the
// LoRA T/U rows in the extension steps) and this CTA's bf16 half of B (128 rows
// fwd, K-major / 128 columns dX, MN-major in two 64-column chunks). Slot s of
// step `it` is it % S. Every slot has exactly one writer per role (the A producer
// for A; the two dequantizer warps that own slot it % S for B, which also issue
// the TMA of the LoRA steps' B half) and all writers wait for the slot's previous
// round to be consumed, so a parity wait never matches a phase two rounds old.
// The dequantizers read packed codes and scales from global memory (L2) into
// registers one owned step ahead; shared memory holds only the MMA operands.
//
// Barriers (same offsets in both CTAs):
//   ready[s]  even CTA only: one arrival from the even A producer, which also
//             posts every byte the step needs (both CTAs' A tiles, loaded with
//             2-SM TMA that signals the even CTA; the LoRA steps' B halves; a
//             4-byte st.async from each odd slot owner), plus one arrival per
//             even slot owner. The odd owners' st.async completes on the even
//             barrier with release semantics at cluster scope once their B rows
//             are written and fenced for the async proxy.
//   empty[s]  one multicast tcgen05.commit per step from the even CTA's MMA
//   tfull[b] / tempty[b]  accumulator double buffer
// Warp roles: 0 A producer, 1 MMA issuer (even CTA) and TMEM allocation, 2-5
// epilogue, 6.. dequantizers (kWarpsPerSlot warps per slot).

template <bool B_MN_>
struct PairCfg {
  static constexpr bool B_MN = B_MN_;
  static constexpr int S = 7;                   // ring slots (one K step each)
  static constexpr int kA = 128 * 64 * 2;       // this CTA's 128 A rows: 16 KB
  static constexpr int kB = 128 * 64 * 2;       // this CTA's B half: 16 KB
  static constexpr int kSlot = kA + kB;         // 32 KB
  static constexpr int kBarOff = S * kSlot;
  static constexpr int kWarpsPerSlot = 2;       // each thread dequantizes two 64-element blocks
  static constexpr int kDeqWarps = S * kWarpsPerSlot;
  static constexpr int kFirstDeqWarp = 6;       // 0 A producer, 1 MMA, 2-5 epilogue
  static constexpr int kThreads = (kFirstDeqWarp + kDeqWarps) * 32;
  static constexpr int kTmemCols = 512;         // 2 buffers x 256 columns
  static constexpr int kNumBars = 2 * S + 5;
  static constexpr int kSigOff = kBarOff + 8 * kNumBars + 16;   // 4 bytes per dequantizer warp
  static constexpr int kSigBytes = 4;
  static constexpr int kSmem = kSigOff + kDeqWarps * kSigBytes + 1024;
  static_assert(kSmem <= 232448, "shared memory budget");
};

// One thread turns two 64-element blocks of this CTA's B half into bf16.
//   fwd (K-major B, 128 rows x 64 K): blocks are B rows t and t + 64 (weight rows
//     nc0 + t, nc0 + t + 64 at K block j).
//   dX (MN-major B, 64 K rows x 128 columns): blocks are K row t (weight row
//     64 j + t) of the column chunks 0 and 1 (weight columns nc0 .. nc0 + 127).
// The packed codes and expanded scales are read straight from global memory (L2)
// into registers one owned step ahead, so they are in place when the slot frees;
// the product tables are built after the slot wait. (Reading the E4M3 scales in
// place instead was measured slower: the per-row scale bytes are 64 bytes apart,
// so every warp load touches 32 sectors.)
struct PairRaw {
  uint4 c[2][2];   // 32 code bytes per block
  float a[2];      // block scales
};

template <bool B_MN>
__device__ __forceinline__ void pair_load_raw(const GemmParams& p, uint32_t t, int j, int nc0, PairRaw& r) {
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    const uint8_t* cp;
    const float* sp;
    if constexpr (!B_MN) {
      const int64_t n = nc0 + int64_t(t) + 64 * b;
      cp = p.codes + n * p.codes_ld + int64_t(j) * 32;
      sp = p.scales + int64_t(j) * p.scales_ld + n;
    } else {
      const int64_t kr = int64_t(j) * 64 + t;
      cp = p.codes + kr * p.codes_ld + (nc0 + 64 * b) / 2;
      sp = p.scales + int64_t(nc0 / 64 + b) * p.scales_ld + kr;
    }
    r.c[b][0] = __ldg(reinterpret_cast<const uint4*>(cp));
    r.c[b][1] = __ldg(reinterpret_cast<const uint4*>(cp + 16));
    r.a[b] = __ldg(sp);
  }
}

// Writes block `blk` of thread t as one 128-byte swizzled row of the B half.
template <bool B_MN>
__device__ __forceinline__ void pair_store_block(uint32_t t, uint32_t blk, const PairRaw& r, uint32_t b_tile) {
  const NF4Lut lut = nf4_make_lut(r.a[blk]);
  const uint32_t w[8] = {r.c[blk][0].x, r.c[blk][0].y, r.c[blk][0].z, r.c[blk][0].w,
                         r.c[blk][1].x, r.c[blk][1].y, r.c[blk][1].z, r.c[blk][1].w};
  const uint32_t row = B_MN ? t : t + 64u * blk;
  const uint32_t sw = row & 7u;
  const uint32_t row_base = b_tile + (B_MN ? blk * 8192u : 0u) + (row >> 3) * 1024u + sw * 128u;
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c) {
    const uint4 v = nf4_dequant_word(w[c], lut);
    const uint32_t addr = row_base + ((c ^ sw) << 4);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
  }
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    tc_gemm_nf4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAx,
                            const __grid_constant__ CUtensorMap tmBx, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_base + C::kBarOff;
  auto ready = [&](int i) { return bar_base + 8u * i; };
  auto empty = [&](int i) { return bar_base + 8u * (C::S + i); };
  const int kT0 = 2 * C::S;
  auto tfull = [&](int b) { return bar_base + 8u * (kT0 + b); };
  auto tempty = [&](int b) { return bar_base + 8u * (kT0 + 2 + b); };
  const uint32_t drain_bar = bar_base + 8u * (kT0 + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 8 * C::kNumBars);
  auto slot = [&](uint32_t i) { return smem_base + (i % C::S) * C::kSlot; };          // A | B half

  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::S; ++i) {
      mbar_init(ready(i), 1 + C::kWarpsPerSlot);   // used in the even CTA only
      mbar_init(empty(i), 1);
    }
    for (int b = 0; b < 2; ++b) { mbar_init(tfull(b), 1); mbar_init(tempty(b), 8); }
    mbar_init(drain_bar, 1);
    fence_mbarrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_launch();

  const int num_tiles = p.tiles_m * p.tiles_n;   // tiles of 256 x 256
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int nsteps = p.num_k_main + p.num_k_ext;

  if (warp == 0) {
    // ------------------------------------------------------------ A producer (both CTAs)
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      uint32_t it = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += npairs) {
        const int m0 = (t / p.tiles_n) * 256 + int(rank) * 128;
        for (int j = 0; j < nsteps; ++j, ++it) {
          if (!mbar_wait(empty(it % C::S), ((it / C::S) & 1u) ^ 1u)) {
            set_status_site(p.status, QLORA_ERR_TIMEOUT, 101); ok = false; break;
          }
          const bool main_step = j < p.num_k_main;
          const uint32_t dst = slot(it), bar = ready(it % C::S);
          const CUtensorMap* m = main_step ? &tmA : &tmAx;
          const int kx = (main_step ? j : j - p.num_k_main) * 64;
          if (rank == 0) {
            // bytes of the whole step: both CTAs' A tiles and, in LoRA steps, B halves
            mbar_arrive_expect_tx(bar, 2 * C::kA + (main_step ? uint32_t(C::kWarpsPerSlot * C::kSigBytes)
                                                          : uint32_t(2 * C::kB)));
            tma_load_2d(dst, m, bar, kx, m0);
          } else {
            tma_load_2d_pair(dst, m, mapa_shared(bar, 0), kx, m0);
          }
        }
      }
      // let the last copies land before leaving
      mbar_wait(empty(it % C::S), ((it / C::S) & 1u) ^ 1u, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc_main = make_idesc_bf16(256, 256, 0, C::B_MN ? 1 : 0);
      // the LoRA steps' B is K-major in both directions ([N x r] rows)
      constexpr uint32_t idesc_ext = make_idesc_bf16(256, 256, 0, 0);
      constexpr uint32_t b_adv = C::B_MN ? (2048u >> 4) : (32u >> 4);
      constexpr uint32_t b_adv_ext = 32u >> 4;
      // descriptors are linear in the start address (bits 0..13 hold addr >> 4);
      // the MN-major B half is two 64-column chunks 8 KB apart (leading offset),
      // which a K-major operand ignores
      const uint64_t da_base = make_smem_desc(slot(0), 16u, 1024u, kSwizzle128B);
      const uint64_t db_base = make_smem_desc(slot(0) + C::kA, 8192u, 1024u, kSwizzle128B);
      constexpr uint64_t kSlotAdv = uint64_t(C::kSlot >> 4);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += npairs, ++tcount) {
        const uint32_t buf = tcount & 1u, tph = (tcount >> 1) & 1u;
        if (!mbar_wait_cluster(tempty(buf), tph ^ 1u)) { set_status_site(p.status, QLORA_ERR_TIMEOUT, 104); ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + buf * 256u;
        for (int j = 0; j < nsteps; ++j, ++it) {
          const uint32_t si = it % C::S;
          if (!mbar_wait_cluster(ready(si), (it / C::S) & 1u)) {
            set_status_site(p.status, QLORA_ERR_TIMEOUT, 105); ok = false; break;
          }
          tc_fence_after();
          const bool ext = j >= p.num_k_main;
          const uint64_t ad = da_base + si * kSlotAdv, bd = db_base + si * kSlotAdv;
          const uint32_t badv = ext ? b_adv_ext : b_adv;
          const uint32_t idesc = ext ? idesc_ext : idesc_main;
#pragma unroll
          for (uint32_t kk = 0; kk < 4; ++kk)
            tc_mma_bf16_pair(d, ad + 2 * kk, bd + kk * badv, idesc, (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit_pair_mc(empty(si), 0x3);
        }
        if (!ok) break;
        tc_commit_pair_mc(tfull(buf), 0x3);
      }
      tc_commit_pair_mc(drain_bar, 0x1);
      mbar_wait(drain_bar, 0, 100000000ull);
    }
  } else if (warp < uint32_t(C::kFirstDeqWarp)) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const uint32_t q = warp & 3u;
    const uint32_t row = q * 32 + lane;
    const uint32_t tempty_remote0 = mapa_shared(tempty(0), 0), tempty_remote1 = mapa_shared(tempty(1), 0);
    uint32_t tcount = 0;
    for (int t = pair; t < num_tiles; t += npairs, ++tcount) {
      const int mb = t / p.tiles_n, nb = t - mb * p.tiles_n;
      const uint32_t buf = tcount & 1u, tph = (tcount >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(tfull(buf), tph))) {
        set_status_site(p.status, QLORA_ERR_TIMEOUT, 107); break;
      }
      tc_fence_after();
      {
        const int grow = mb * 256 + int(rank) * 128 + int(row);
        const uint32_t tbase = tmem_base + ((q * 32u) << 16) + buf * 256u;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tbase + c * 32, v);
          tmem_ld_wait();
          if (grow < p.M) {
            uint16_t* dst = reinterpret_cast<uint16_t*>(p.out) + int64_t(grow) * p.ld_out + nb * 256 + c * 32;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]));
              o.y = pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]));
              o.z = pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]));
              o.w = pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]));
              reinterpret_cast<uint4*>(dst)[i] = o;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(buf ? tempty_remote1 : tempty_remote0);
    }
  } else {
    // ------------------------------------------------------------ dequantizers (both CTAs)
    const uint32_t dw = warp - uint32_t(C::kFirstDeqWarp);
    const uint32_t own = dw / C::kWarpsPerSlot;   // slot this warp fills
    const uint32_t sub = dw % C::kWarpsPerSlot;   // threads t in [32 sub, 32 sub + 32)
    const uint32_t row = sub * 32 + lane;
    const uint32_t ready_even = mapa_shared(ready(own), 0);
    const uint32_t sig_even = mapa_shared(smem_base + C::kSigOff + dw * C::kSigBytes, 0);
    // this pair's steps are numbered it = (tile of the pair) * nsteps + j; this
    // warp owns it = own, own + S, ...
    const uint32_t total = uint32_t((num_tiles - pair + npairs - 1) / npairs) * uint32_t(nsteps);
    auto tile_of = [&](uint32_t i) { return pair + int(i / uint32_t(nsteps)) * npairs; };
    auto nc0_of = [&](int t) { return (t % p.tiles_n) * 256 + int(rank) * 128; };
    PairRaw raw;
    if (own < total && int(own % uint32_t(nsteps)) < p.num_k_main)
      pair_load_raw<C::B_MN>(p, row, int(own % uint32_t(nsteps)), nc0_of(tile_of(own)), raw);
    for (uint32_t it = own; it < total; it += C::S) {
      const int t = tile_of(it), j = int(it % uint32_t(nsteps));
      const uint32_t round = it / C::S;
      const uint32_t b_tile = slot(it) + C::kA;
      if (!__all_sync(0xffffffffu, mbar_wait(empty(own), (round & 1u) ^ 1u))) {
        set_status_site(p.status, QLORA_ERR_TIMEOUT, 118);
        break;
      }
      if (j < p.num_k_main) {
        pair_store_block<C::B_MN>(row, 0, raw, b_tile);
        pair_store_block<C::B_MN>(row, 1, raw, b_tile);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0) mbar_arrive(ready(own));
          else st_async_signal(sig_even, ready_even);
        }
      } else if (lane == 0) {
        // LoRA step: B half by TMA; its bytes were posted by the even A producer
        const int kx = (j - p.num_k_main) * 64, n0 = nc0_of(t);
        const uint32_t bar = rank == 0 ? ready(own) : ready_even;
        if (sub == 0) {   // [N x r] rows n0.. (s.L2^T for the forward pass, L1 for dX)
          if (rank == 0) tma_load_2d(b_tile, &tmBx, bar, kx, n0);
          else tma_load_2d_pair(b_tile, &tmBx, bar, kx, n0);
        }
        if (rank == 0) mbar_arrive(ready(own));
      }
      // codes of this warp's next step, in flight while it waits for that slot
      const uint32_t nx = it + C::S;
      if (nx < total && int(nx % uint32_t(nsteps)) < p.num_k_main)
        pair_load_raw<C::B_MN>(p, row, int(nx % uint32_t(nsteps)), nc0_of(tile_of(nx)), raw);
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

// =============================================================== CTA-pair kernel, 512-row tiles
//
// Same pair MMA (cluster of 2, tcgen05 cta_group::2, M = 256, N = 256) as above, but a
// pair tile is 512 (M) x 256 (N): each K step stages two 128-row A sub-tiles per CTA
// and issues two pair MMAs per 16-wide K slice against the same dequantized B half,
// into two accumulators (TMEM columns 0-255: rows m0 .. m0 + 255 of the tile, columns
// 256-511: rows m0 + 256 .. m0 + 511). Every decoded weight therefore meets 512 token
// rows instead of 256: the dequantizers' ALU work and shared-memory stores per MMA
// are halved. The two accumulators fill TMEM, so there is no second buffer: the MMA
// issuer commits accumulator 0 before the last step's accumulator-1 MMAs, the
// epilogue drains it first (TMEM -> registers -> bf16 in a swizzled staging buffer ->
// TMA store), and the next tile's first MMAs wait only for accumulator 0.
//
// Schedule (GemmParams::sk_*): sk_R rounds of whole tiles, then the remaining tiles'
// steps cut into ranges of sk_L steps, one range per pair (so a part that can co-run
// fewer pairs than a multiple of the tile count does not idle through a last partial
// round). A tile cut into parts is finished by the pair holding its first step, which
// is the last range of that pair: the other parts (the first range of their pairs,
// done before it) write fp32 partials and count themselves in; the finishing pair
// waits for the count (bounded), adds the partials in pair order to its accumulator
// and writes the tile.
//
// Aux tiles (GemmParams::aux_tiles): the LoRA product the output tiles' LoRA step
// reads can be computed in the same launch, one leading tile per 512-row block: the
// forward's T = X L1 (B = L1 by TMA) or the dX pass's U = dY L2^T (B = L2 by TMA,
// stored as U and s.U). An aux tile takes A like an output tile, stores through the
// same staging, then releases a per-block flag; an output tile's producer acquires
// that flag before its LoRA step loads the aux rows. Aux tiles wait on nothing and
// come first in every pair's order, so no wait closes a cycle.
//
// Shared memory per CTA: S ring slots of 48 KB (the A rows 128 rank + {0, 256} +
// 0..127 of the tile, and this CTA's B half) and kNumStage 16 KB epilogue staging
// buffers (128 rows x 64 bf16 columns, 128-byte swizzle, written out by TMA store),
// barriers. The epilogue's stores leave the SM slowly while every pair drains at
// once (a store held its buffer about 2000 cycles before it had read it), so the
// default gives the staging a whole accumulator (3 slots, 4 buffers).
// Warp roles: 0 A producer, 1 MMA issuer (even CTA) and TMEM allocation, 2-5
// epilogue, then the dequantizers (two per ring slot).

template <bool B_MN_, int S_, int NST_>
struct Pair2Cfg {
  static constexpr bool B_MN = B_MN_;
  static constexpr int S = S_;                    // ring slots (one K step each)
  static constexpr int kNumStage = NST_;          // epilogue staging buffers of 16 KB
  static constexpr int kA = 128 * 64 * 2;         // one 128-row A sub-tile: 16 KB
  static constexpr int kB = 128 * 64 * 2;         // this CTA's B half: 16 KB
  static constexpr int kSlot = 2 * kA + kB;       // 48 KB
  static constexpr int kStageOff = S * kSlot;     // epilogue staging
  static constexpr int kStageBytes = 128 * 64 * 2;   // 128 rows x 64 bf16 columns
  static constexpr int kBarOff = kStageOff + kNumStage * kStageBytes;
  static constexpr int kWarpsPerSlot = 2;
  static constexpr int kDeqWarps = S * kWarpsPerSlot;
  static constexpr int kFirstDeqWarp = 6;
  static constexpr int kThreads = (kFirstDeqWarp + kDeqWarps) * 32;
  static constexpr int kTmemCols = 512;
  static constexpr int kNumBars = 2 * S + 5;      // ready, empty, tfull[2], tempty[2], drain
  static constexpr int kTmemSlotOff = kBarOff + 8 * kNumBars;
  static constexpr int kSigOff = kTmemSlotOff + 8;                 // 4 bytes per dequantizer warp
  static constexpr int kSigBytes = 4;
  static constexpr int kSmem = kSigOff + kDeqWarps * kSigBytes + 1024;
  static constexpr int kEpiThreads = 128;
  static_assert(kSmem <= 232448, "shared memory budget");
  static_assert(kStageOff % 1024 == 0, "swizzled staging must be 1024-byte aligned");
};

// Tail range of pair `pr`: its first tail step and length (see GemmParams::sk_*).
__device__ __forceinline__ int sk_tail_begin(const GemmParams& p, int pr) {
  return pr < p.sk_A ? pr * p.sk_La : p.sk_A * p.sk_La + (pr - p.sk_A) * p.sk_L;
}
__device__ __forceinline__ int sk_tail_len(const GemmParams& p, int pr) {
  return pr < p.sk_A ? p.sk_La : p.sk_L;
}
// The pair whose tail range holds tail step s (s < sk_W).
__device__ __forceinline__ int sk_pair_of(const GemmParams& p, int s) {
  const int a = p.sk_A * p.sk_La;
  return s < a ? s / p.sk_La : p.sk_A + (s - a) / p.sk_L;
}
// Steps of pair `pr` and the (tile, k step) of its step i (see GemmParams::sk_*).
__device__ __forceinline__ uint32_t sk_num_steps(const GemmParams& p, int pr) {
  const int S = p.num_k_main + p.num_k_ext;
  uint32_t n = uint32_t(p.sk_R) * uint32_t(S);
  const int b = sk_tail_begin(p, pr), e = min(b + sk_tail_len(p, pr), p.sk_W);
  if (e > b) n += uint32_t(e - b);
  return n;
}
__device__ __forceinline__ void sk_step(const GemmParams& p, int pr, uint32_t i, int& tile, int& k) {
  const int S = p.num_k_main + p.num_k_ext;
  const uint32_t dp = uint32_t(p.sk_R) * uint32_t(S);
  if (i < dp) {
    const int r = int(i / uint32_t(S));
    tile = pr + r * p.sk_P;
    k = int(i) - r * S;
  } else {
    const int ti = sk_tail_begin(p, pr) + int(i - dp);
    const int u = ti / S;
    tile = p.sk_base + u;
    k = ti - u * S;
  }
}

// Block and column tile of a tile id: the aux_tiles leading aux tiles (T or U;
// block = id, column -1), then the output tiles row-block-major.
__device__ __forceinline__ void sk_tile(const GemmParams& p, int tile, int& mb, int& nb) {
  if (tile < p.aux_tiles) {
    mb = tile;
    nb = -1;
  } else {
    const int t2 = tile - p.aux_tiles;
    mb = t2 / p.tiles_n;
    nb = t2 - mb * p.tiles_n;
  }
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    tc_gemm_nf4_pair2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAx,
                             const __grid_constant__ CUtensorMap tmBx, const __grid_constant__ CUtensorMap tmY,
                             const __grid_constant__ CUtensorMap tmL1, const __grid_constant__ CUtensorMap tmT,
                             const __grid_constant__ CUtensorMap tmT2, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_base + C::kBarOff;
  auto ready = [&](int i) { return bar_base + 8u * i; };
  auto empty = [&](int i) { return bar_base + 8u * (C::S + i); };
  const int kT0 = 2 * C::S;
  auto tfull = [&](int h) { return bar_base + 8u * (kT0 + h); };
  auto tempty = [&](int h) { return bar_base + 8u * (kT0 + 2 + h); };
  const uint32_t drain_bar = bar_base + 8u * (kT0 + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kTmemSlotOff);
  auto slot = [&](uint32_t i) { return smem_base + (i % C::S) * C::kSlot; };   // A0 | A1 | B half

  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::S; ++i) {
      mbar_init(ready(i), 1 + C::kWarpsPerSlot);   // used in the even CTA only
      mbar_init(empty(i), 1);
    }
    for (int h = 0; h < 2; ++h) { mbar_init(tfull(h), 1); mbar_init(tempty(h), 8); }
    mbar_init(drain_bar, 1);
    fence_mbarrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_launch();

  const int pr = int(blockIdx.x >> 1);
  const int S = p.num_k_main + p.num_k_ext;
  const uint32_t nsteps = sk_num_steps(p, pr);
  const uint32_t dp_steps = uint32_t(p.sk_R) * uint32_t(S);
  // MMA width of the aux tiles: 128 columns hold r <= 128, else 256
  const int t_n = p.t_chunks <= 2 ? 128 : 256;

  if (warp == 0) {
    // ------------------------------------------------------------ A producer (both CTAs)
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmAx);
      uint32_t it = 0;
      for (; it < nsteps; ++it) {
        int tile, k;
        sk_step(p, pr, it, tile, k);
        if (!mbar_wait(empty(it % C::S), ((it / C::S) & 1u) ^ 1u)) {
          set_status_site(p.status, QLORA_ERR_TIMEOUT, 201);
          break;
        }
        int mb, nb;
        sk_tile(p, tile, mb, nb);
        const bool ttile = nb < 0;
        const int m0 = mb * 512 + int(rank) * 128;
        const bool main_step = k < p.num_k_main;
        const uint32_t dst = slot(it), bar = ready(it % C::S);
        // an aux tile reads A (X or dY) in every step (its extra step starts past the K
        // extent: zeros)
        const bool x_step = main_step || ttile;
        const CUtensorMap* m = x_step ? &tmA : &tmAx;
        const int kx = (x_step ? k : k - p.num_k_main) * 64;
        if (!x_step && p.aux_tiles > 0 && k == p.num_k_main) {
          // the first LoRA step of an output tile needs its block's T (or s.U): wait for
          // the flag
          int* fl = p.t_flags + (mb * 2 + int(rank)) * 2;
          if (ld_acquire_gpu(fl) == 0) {
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_gpu(fl) == 0) {
              if (globaltimer_ns() - t0 > 2000000000ull) {
                set_status_site(p.status, QLORA_ERR_TIMEOUT, 202);
                break;
              }
            }
          }
          fence_proxy_async_global();
          // the block's last reader clears the flag for the next call
          if (atomicAdd(fl + 1, 1) == p.tiles_n - 1) {
            fl[1] = 0;
            fl[0] = 0;
          }
        }
        if (rank == 0) {
          // bytes of the whole step: both CTAs' two A sub-tiles and, in LoRA steps and aux
          // tiles, B halves by TMA (an aux tile's B is its MMA width t_n x 64 K, split
          // over the pair)
          mbar_arrive_expect_tx(bar, 4 * C::kA + (main_step && !ttile ? uint32_t(C::kWarpsPerSlot * C::kSigBytes)
                                                  : ttile             ? uint32_t(t_n * 128)
                                                                      : uint32_t(2 * C::kB)));
          tma_load_2d(dst, m, bar, kx, m0);
          tma_load_2d(dst + C::kA, m, bar, kx, m0 + 256);
        } else {
          const uint32_t bar0 = mapa_shared(bar, 0);
          tma_load_2d_pair(dst, m, bar0, kx, m0);
          tma_load_2d_pair(dst + C::kA, m, bar0, kx, m0 + 256);
        }
      }
      // let the last copies land before leaving
      if (it > 0) mbar_wait(empty(it % C::S), ((it / C::S) & 1u) ^ 1u, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc_main = make_idesc_bf16(256, 256, 0, C::B_MN ? 1 : 0);
      constexpr uint32_t idesc_ext = make_idesc_bf16(256, 256, 0, 0);   // LoRA B is [N x r], K-major
      // aux tiles, N = t_n: forward T tiles read L1 [K x r] (MN-major), dX U tiles L2
      // [r x K] (K-major)
      constexpr uint32_t t_bmn = C::B_MN ? 0u : 1u;
      const uint32_t idesc_t = t_n == 128 ? make_idesc_bf16(256, 128, 0, t_bmn) : make_idesc_bf16(256, 256, 0, t_bmn);
      constexpr uint32_t b_adv_t = C::B_MN ? (32u >> 4) : (2048u >> 4);
      constexpr uint32_t b_adv = C::B_MN ? (2048u >> 4) : (32u >> 4);
      constexpr uint32_t b_adv_ext = 32u >> 4;
      const uint64_t da_base = make_smem_desc(slot(0), 16u, 1024u, kSwizzle128B);
      const uint64_t db_base = make_smem_desc(slot(0) + 2 * C::kA, 8192u, 1024u, kSwizzle128B);
      constexpr uint64_t kSlotAdv = uint64_t(C::kSlot >> 4);
      constexpr uint64_t kA1 = uint64_t(C::kA >> 4);
      uint32_t seg = 0;
      for (uint32_t it = 0; it < nsteps; ++it) {
        int tile, k;
        sk_step(p, pr, it, tile, k);
        const bool first = (k == 0) || (it == dp_steps);
        const bool last = (k == S - 1) || (it + 1 == nsteps);
        const uint32_t par = (seg & 1u) ^ 1u;
        if (first) {
          if (!mbar_wait_cluster(tempty(0), par)) { set_status_site(p.status, QLORA_ERR_TIMEOUT, 204); break; }
          tc_fence_after();
        }
        const uint32_t si = it % C::S;
        if (!mbar_wait_cluster(ready(si), (it / C::S) & 1u)) {
          set_status_site(p.status, QLORA_ERR_TIMEOUT, 205);
          break;
        }
        tc_fence_after();
        const bool ext = k >= p.num_k_main;
        const uint64_t ad = da_base + si * kSlotAdv, bd = db_base + si * kSlotAdv;
        // an aux tile's B is the same operand in every step
        const bool ttile = tile < p.aux_tiles;
        const uint32_t badv = ttile ? b_adv_t : ext ? b_adv_ext : b_adv;
        const uint32_t idesc = ttile ? idesc_t : ext ? idesc_ext : idesc_main;
#pragma unroll
        for (uint32_t kk = 0; kk < 4; ++kk)
          tc_mma_bf16_pair(tmem_base, ad + 2 * kk, bd + kk * badv, idesc, (!first || kk > 0) ? 1u : 0u);
        if (last) tc_commit_pair_mc(tfull(0), 0x3);
        if (first) {
          if (!mbar_wait_cluster(tempty(1), par)) { set_status_site(p.status, QLORA_ERR_TIMEOUT, 206); break; }
          tc_fence_after();
        }
#pragma unroll
        for (uint32_t kk = 0; kk < 4; ++kk)
          tc_mma_bf16_pair(tmem_base + 256u, ad + kA1 + 2 * kk, bd + kk * badv, idesc, (!first || kk > 0) ? 1u : 0u);
        tc_commit_pair_mc(empty(si), 0x3);
        if (last) {
          tc_commit_pair_mc(tfull(1), 0x3);
          ++seg;
        }
      }
      tc_commit_pair_mc(drain_bar, 0x1);
      mbar_wait(drain_bar, 0, 100000000ull);
    }
  } else if (warp < uint32_t(C::kFirstDeqWarp)) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const uint32_t q = warp & 3u;
    const uint32_t row = q * 32 + lane;              // TMEM lane = row of this CTA's sub-tiles
    const bool leader = (warp == 2 && lane == 0);    // issues the TMA stores and counts in
    const uint32_t tempty_remote[2] = {mapa_shared(tempty(0), 0), mapa_shared(tempty(1), 0)};
    const uint32_t stage0 = smem_base + C::kStageOff;
    const uint32_t tl = tmem_base + ((q * 32u) << 16);
    constexpr size_t kRankFloats = size_t(2) * 256 * 128;   // one rank's partial: 2 halves x 256 cols x 128 rows
    // Every epilogue warp walks the same segments and named barriers even after a
    // wait has timed out (ok = false then skips the remaining waits), so no warp is
    // left alone at a barrier.
    uint32_t seg = 0, chunk = 0;
    bool ok = true;
    auto wait_full = [&](int h, uint32_t par, int site) {
      if (ok && !__all_sync(0xffffffffu, mbar_wait_cluster(tfull(h), par))) {
        set_status_site(p.status, QLORA_ERR_TIMEOUT, site);
        ok = false;
      }
    };
    for (uint32_t i = 0; i < nsteps;) {
      int tile, kb;
      sk_step(p, pr, i, tile, kb);
      const int len = (i < dp_steps) ? S : min(S - kb, int(nsteps - i));
      i += uint32_t(len);
      const int ke = kb + len;
      int mb, nb;
      sk_tile(p, tile, mb, nb);
      const bool ttile = nb < 0;                         // an aux tile: T or U of block mb
      const int nchunks = ttile ? p.t_chunks : 4;        // 64-column chunks written
      const uint32_t par = seg & 1u;
      ++seg;
      int extra = 0, pf1 = 0;     // partials of later parts to add, from pair slots pf1, pf1 + 1, ...
      if (kb > 0 || ke < S) {
        // ---- a tile cut into parts (pairs pf .. pl, in step order)
        const int u = tile - p.sk_base;
        const int pf = sk_pair_of(p, u * S), pl = sk_pair_of(p, (u + 1) * S - 1);
        int* counter = p.sk_count + 2 * u + int(rank);
        if (kb > 0) {
          // a later part: fp32 partial to this pair's slot (column-major in 128-row
          // columns, so every warp store is one 128-byte line), then count in
          float* dst = p.sk_part + (size_t(pr) * 2 + rank) * kRankFloats + row;
          for (int h = 0; h < 2; ++h) {
            wait_full(h, par, 207);
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 8; ++c) {
              uint32_t v[32];
              tmem_ld_32x32b_x32(tl + uint32_t(h) * 256u + uint32_t(c) * 32u, v);
              tmem_ld_wait();
              float* d = dst + (size_t(h) * 256 + c * 32) * 128;
#pragma unroll
              for (int j = 0; j < 32; ++j) __stcg(d + size_t(j) * 128, __uint_as_float(v[j]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_remote[h]);
          }
          __threadfence();
          named_bar_sync(1, C::kEpiThreads);
          if (leader) atomicAdd(counter, 1);
          continue;
        }
        // the first part: wait (bounded) until the pl - pf later parts have counted in
        extra = pl - pf;
        pf1 = pf + 1;
        if (ok && ld_acquire_gpu(counter) < extra) {
          const uint64_t t0 = globaltimer_ns();
          while (ld_acquire_gpu(counter) < extra) {
            if (globaltimer_ns() - t0 > 2000000000ull) {
              set_status_site(p.status, QLORA_ERR_TIMEOUT, 208);
              break;
            }
          }
        }
      }
      for (int h = 0; h < 2; ++h) {
        wait_full(h, par, 209);
        tc_fence_after();
        const int y = mb * 512 + h * 256 + int(rank) * 128;   // first output row of this store box
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
          uint32_t v[64];
          tmem_ld_32x32b_x32(tl + uint32_t(h) * 256u + uint32_t(c) * 64u, *reinterpret_cast<uint32_t(*)[32]>(v));
          tmem_ld_32x32b_x32(tl + uint32_t(h) * 256u + uint32_t(c) * 64u + 32u,
                             *reinterpret_cast<uint32_t(*)[32]>(v + 32));
          tmem_ld_wait();
          if (c == nchunks - 1) {
            // the accumulator is in registers: the next tile's MMAs may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_remote[h]);
          }
          for (int e = 0; e < extra; ++e) {
            const float* src = p.sk_part + (size_t(pf1 + e) * 2 + rank) * kRankFloats +
                               (size_t(h) * 256 + c * 64) * 128 + row;
#pragma unroll
            for (int j = 0; j < 64; ++j)
              v[j] = __float_as_uint(__uint_as_float(v[j]) + __ldcg(src + size_t(j) * 128));
          }
          // a U tile writes the chunk twice: U, then bf16(aux_scale * bf16(U))
          const int npass = (ttile && p.aux_dual) ? 2 : 1;
#pragma unroll 1
          for (int pass = 0; pass < npass; ++pass) {
            const uint32_t buf = chunk++ % uint32_t(C::kNumStage);
            // the store that used this staging buffer kNumStage uses ago must have read it
            if (leader) bulk_wait_group_read<C::kNumStage - 1>();
            named_bar_sync(1, C::kEpiThreads);
            const uint32_t sbase = stage0 + buf * C::kStageBytes + row * 128u;
            const uint32_t sw = row & 7u;
            auto pk = [&](uint32_t x0, uint32_t x1) {
              const uint32_t a = pack_bf16x2(__uint_as_float(x0), __uint_as_float(x1));
              if (pass == 0) return a;
              return pack_bf16x2(__fmul_rn(__uint_as_float(a << 16), p.aux_scale),
                                 __fmul_rn(__uint_as_float(a & 0xFFFF0000u), p.aux_scale));
            };
#pragma unroll
            for (uint32_t j = 0; j < 8; ++j) {
              const uint32_t a0 = pk(v[8 * j + 0], v[8 * j + 1]);
              const uint32_t a1 = pk(v[8 * j + 2], v[8 * j + 3]);
              const uint32_t a2 = pk(v[8 * j + 4], v[8 * j + 5]);
              const uint32_t a3 = pk(v[8 * j + 6], v[8 * j + 7]);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sbase + ((j ^ sw) << 4)), "r"(a0),
                           "r"(a1), "r"(a2), "r"(a3)
                           : "memory");
            }
            fence_proxy_async_smem();
            named_bar_sync(1, C::kEpiThreads);
            if (leader && y < p.M) {   // rows past M are clipped by the store; a box wholly past M is skipped
              const uint32_t sb = stage0 + buf * C::kStageBytes;
              if (!ttile) tma_store_2d(&tmY, sb, nb * 256 + c * 64, y);
              else if (pass == 0) tma_store_2d(&tmT, sb, c * 64, y);   // columns past r clipped
              else tma_store_2d(&tmT2, sb, c * 64, y);
            }
            if (leader) bulk_commit_group();
          }
        }
      }
      if (extra > 0 && leader) {
        // every later part has been read: the counter goes back to zero for the next call
        p.sk_count[2 * (tile - p.sk_base) + int(rank)] = 0;
      }
      if (ttile && leader) {
        // this CTA's aux rows of the block are in global memory: raise its flag for the
        // output tiles' LoRA steps (they read them with TMA after an acquire of the flag)
        bulk_wait_group<0>();
        fence_proxy_async_global();
        __threadfence();
        st_release_gpu(p.t_flags + (mb * 2 + int(rank)) * 2, 1);
      }
    }
    if (leader) bulk_wait_group<0>();
  } else {
    // ------------------------------------------------------------ dequantizers (both CTAs)
    const uint32_t dw = warp - uint32_t(C::kFirstDeqWarp);
    const uint32_t own = dw / C::kWarpsPerSlot;   // ring slot this warp fills
    const uint32_t sub = dw % C::kWarpsPerSlot;   // threads t in [32 sub, 32 sub + 32)
    const uint32_t row = sub * 32 + lane;
    const uint32_t ready_even = mapa_shared(ready(own), 0);
    const uint32_t sig_even = mapa_shared(smem_base + C::kSigOff + dw * C::kSigBytes, 0);
    auto nc0_of = [&](int t) { return ((t - p.aux_tiles) % p.tiles_n) * 256 + int(rank) * 128; };
    PairRaw raw;
    if (own < nsteps) {
      int t, k;
      sk_step(p, pr, own, t, k);
      if (k < p.num_k_main && t >= p.aux_tiles) pair_load_raw<C::B_MN>(p, row, k, nc0_of(t), raw);
    }
    for (uint32_t it = own; it < nsteps; it += C::S) {
      int t, k;
      sk_step(p, pr, it, t, k);
      const uint32_t round = it / C::S;
      const uint32_t b_tile = slot(it) + 2 * C::kA;
      if (!__all_sync(0xffffffffu, mbar_wait(empty(own), (round & 1u) ^ 1u))) {
        set_status_site(p.status, QLORA_ERR_TIMEOUT, 218);
        break;
      }
      if (t < p.aux_tiles) {
        if (lane == 0) {
          // T tile: this CTA's B half is L1 rows 64 k.. (zeros past the K extent), columns
          // (t_n / 2) rank .. + t_n / 2 - 1 (zeros past r), as MN-major 64-column chunks by
          // TMA; the even A producer posted its bytes
          // (a U tile: L2 rows (t_n / 2) rank .. + t_n / 2 - 1, K columns 64 k.., one
          // K-major box)
          const uint32_t bar = rank == 0 ? ready(own) : ready_even;
          if (sub == 0) {
            if constexpr (!C::B_MN) {
              for (int c = 0; c < t_n / 128; ++c) {
                const int x = int(rank) * (t_n / 2) + 64 * c;
                if (rank == 0) tma_load_2d(b_tile + c * 8192, &tmL1, bar, x, k * 64);
                else tma_load_2d_pair(b_tile + c * 8192, &tmL1, bar, x, k * 64);
              }
            } else {
              const int y = int(rank) * (t_n / 2);
              if (rank == 0) tma_load_2d(b_tile, &tmL1, bar, k * 64, y);
              else tma_load_2d_pair(b_tile, &tmL1, bar, k * 64, y);
            }
          }
          if (rank == 0) mbar_arrive(ready(own));
        }
      } else if (k < p.num_k_main) {
        pair_store_block<C::B_MN>(row, 0, raw, b_tile);
        pair_store_block<C::B_MN>(row, 1, raw, b_tile);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0) mbar_arrive(ready(own));
          else st_async_signal(sig_even, ready_even);
        }
      } else if (lane == 0) {
        // LoRA step: B half by TMA; its bytes were posted by the even A producer
        const int kx = (k - p.num_k_main) * 64, n0 = nc0_of(t);
        const uint32_t bar = rank == 0 ? ready(own) : ready_even;
        if (sub == 0) {   // [N x r] rows n0.. (s.L2^T for the forward pass, L1 for dX)
          if (rank == 0) tma_load_2d(b_tile, &tmBx, bar, kx, n0);
          else tma_load_2d_pair(b_tile, &tmBx, bar, kx, n0);
        }
        if (rank == 0) mbar_arrive(ready(own));
      }
      // codes of this warp's next step, in flight while it waits for that slot
      const uint32_t nx = it + C::S;
      if (nx < nsteps) {
        int t2, k2;
        sk_step(p, pr, nx, t2, k2);
        if (k2 < p.num_k_main && t2 >= p.aux_tiles) pair_load_raw<C::B_MN>(p, row, k2, nc0_of(t2), raw);
      }
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

// --------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

bool make_tmap_2d(CUtensorMap* m, const void* base, TmapType type, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
  return make_tmap_2d_sw(m, base, type, inner, outer, row_bytes, box_inner, box_outer, swizzle128 ? 128 : 0);
}

bool make_tmap_2d_sw(CUtensorMap* m, const void* base, TmapType type, uint64_t inner, uint64_t outer,
                     uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, int swizzle_bytes) {
  auto fn = encode_fn();
  if (!fn) return false;
  CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (type == TmapType::U8) dt = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  if (type == TmapType::F32) dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                  : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                  : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <class C>
static qlora_status launch_cfg(const GemmOperands& o, GemmParams p, int ctas_per_sm, cudaStream_t s) {
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(tc_gemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) !=
        cudaSuccess)
      return QLORA_ERR_CUDA;
    attr_set = true;
  }
  p.bn = C::BN;
  const int num_tiles = p.tiles_m * p.tiles_n * p.splits;
  const int grid = std::max(1, std::min(num_tiles, num_sms() * ctas_per_sm));
  if (launch_pdl(tc_gemm_kernel<C>, dim3(grid), dim3(C::kThreads), C::kSmem, s, o.A, o.B, o.codes, o.scales, o.Ax,
                 o.Bx, p) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// CTA pairs of the last pair launch (0 before any): the co-resident 2-SM clusters the
// occupancy calculator reports for the kernel (74 on a 148-SM part when every GPC can
// pair all of its SMs), capped by the tile count.
static int g_last_pairs = 0;
int last_pair_clusters() { return g_last_pairs; }

// Co-resident 2-SM clusters of the pair kernel (occupancy calculator; sets the
// kernel's shared-memory limit on first use), 0 on failure.
template <class C>
static int pair_max_clusters() {
  static int max_pairs = -1;
  if (max_pairs < 0) {
    if (cudaFuncSetAttribute(tc_gemm_nf4_pair_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) !=
        cudaSuccess)
      return 0;
    cudaLaunchConfig_t qc = {};
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    qc.gridDim = dim3(2 * 74, 1, 1);
    qc.blockDim = dim3(C::kThreads, 1, 1);
    qc.dynamicSmemBytes = C::kSmem;
    qc.attrs = qa;
    qc.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, tc_gemm_nf4_pair_kernel<C>, &qc) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = num_sms() / 2;
    }
    max_pairs = n;
  }
  return max_pairs;
}

// The fewest pairs that still finish num_tiles tiles in the least number of rounds:
// the same time for the GEMM, and the SMs left over stay free for concurrent work.
static int pairs_for(int num_tiles, int max_pairs) {
  const int rounds = (num_tiles + max_pairs - 1) / max_pairs;
  return std::max(1, (num_tiles + rounds - 1) / rounds);
}

int pair_spare_sms(bool dx, int num_tiles) {
  const int mp = dx ? pair_max_clusters<PairCfg<true>>() : pair_max_clusters<PairCfg<false>>();
  if (mp <= 0) return 0;
  return num_sms() - 2 * pairs_for(num_tiles, mp);
}

template <class C>
static qlora_status launch_pair_cfg(const GemmOperands& o, GemmParams p, cudaStream_t s) {
  const int max_pairs = pair_max_clusters<C>();
  if (max_pairs <= 0) return QLORA_ERR_CUDA;
  p.bn = 256;
  const int num_tiles = p.tiles_m * p.tiles_n;
  const int pairs = pairs_for(num_tiles, max_pairs);
  g_last_pairs = pairs;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  if (cudaLaunchKernelEx(&cfg, tc_gemm_nf4_pair_kernel<C>, o.A, o.Ax, o.Bx, p) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// ---- 512 x 256 pair kernel

template <class C>
static int pair2_max_clusters() {
  static int max_pairs = -1;
  if (max_pairs < 0) {
    if (cudaFuncSetAttribute(tc_gemm_nf4_pair2_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) !=
        cudaSuccess)
      return 0;
    cudaLaunchConfig_t qc = {};
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    qc.gridDim = dim3(2 * 74, 1, 1);
    qc.blockDim = dim3(C::kThreads, 1, 1);
    qc.dynamicSmemBytes = C::kSmem;
    qc.attrs = qa;
    qc.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, tc_gemm_nf4_pair2_kernel<C>, &qc) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = num_sms() / 2;
    }
    max_pairs = n;
  }
  return max_pairs;
}

// QLORA_B200_MAX_PAIRS=n caps the pairs of the 512 x 256 kernel (read on every call, so
// tests can force a given schedule of whole rounds and split tiles on any part).
static int pair2_pair_cap() {
  const char* e = std::getenv("QLORA_B200_MAX_PAIRS");
  if (!e) return kPair2MaxPairs;
  const int v = std::atoi(e);
  return (v >= 1 && v <= kPair2MaxPairs) ? v : kPair2MaxPairs;
}

// Schedule over P co-resident pairs: R = T / P rounds of whole tiles, then the
// remaining T - R P tiles' W steps in ranges of L = ceil(W / P) steps (at least a
// third of a tile, so a tile has at most four parts). When cutting saves less than a
// twentieth of a tile, L = S: the remaining tiles run whole, one per pair.
struct Pair2Sched {
  int P, R, L, W, base, launch, A, La;
};
// T tiles (the first A of them aux tiles) of S steps over P pairs. When the aux tiles
// all fall in the first of at least one whole round, the pairs that ran one (about
// half an output tile's work: the same A bytes, half the MMA width) take tail
// ranges longer by 9/20 of a tile, so all pairs end together.
static Pair2Sched pair2_schedule(int T, int S, int P, int A = 0) {
  Pair2Sched sc;
  sc.P = P;
  sc.R = T / P;
  const int Tr = T - sc.R * P;
  sc.base = sc.R * P;
  sc.W = Tr * S;
  sc.L = 0;
  sc.A = 0;
  sc.La = 0;
  const int min_range = (S + 2) / 3;   // at most four parts per tile
  if (Tr > 0) {
    int L = std::max((sc.W + P - 1) / P, min_range);
    if (L >= S || (S - L) * 20 < S) L = S;
    sc.L = L;
    // (only where the others' ranges stay at least a third of a tile; else even ranges)
    const int e = (9 * S) / 20;
    if (A > 0 && A <= P && sc.R >= 1 && L < S && e > 0) {
      const int Ln = (sc.W - A * e + P - 1) / P;
      if (Ln >= min_range) {
        sc.A = A;
        sc.La = Ln + e;
        sc.L = Ln;
      }
    }
  }
  sc.launch = sc.R > 0 ? P : (sc.L > 0 ? (sc.W + sc.L - 1) / sc.L : 0);
  return sc;
}

void pair2_schedule_of(int tiles, int aux_tiles, int steps, int pairs, int32_t* out) {
  const Pair2Sched sc = pair2_schedule(tiles, steps, pairs, aux_tiles);
  out[0] = sc.P;
  out[1] = sc.R;
  out[2] = sc.L;
  out[3] = sc.W;
  out[4] = sc.base;
  out[5] = sc.launch;
  out[6] = sc.A;
  out[7] = sc.La;
}

size_t pair2_partial_bytes(int64_t M, int64_t N) {
  const int64_t T = ((M + 511) / 512) * (N / 256 + 1);   // with the aux tiles
  const int64_t slots = std::min<int64_t>(kPair2MaxPairs, 4 * T);
  return size_t(slots) * (size_t(2) * 2 * 256 * 128 * sizeof(float));
}

// Longer tail ranges for the pairs that ran an aux tile, unless QLORA_B200_AUX_BALANCE=0
// (read on every call).
static bool aux_balance() {
  const char* e = std::getenv("QLORA_B200_AUX_BALANCE");
  return !(e && std::strcmp(e, "0") == 0);
}

template <class C>
static qlora_status launch_pair2_cfg(const GemmOperands& o, GemmParams p, cudaStream_t s) {
  const int max_pairs = std::min(pair2_max_clusters<C>(), pair2_pair_cap());
  if (max_pairs <= 0) return QLORA_ERR_CUDA;
  p.bn = 256;
  const int T = p.aux_tiles + p.tiles_m * p.tiles_n;
  const int S = p.num_k_main + p.num_k_ext;
  if (p.aux_tiles > 0 && (p.aux_tiles != p.tiles_m || p.aux_tiles > kPair2MaxTBlocks || !p.t_flags ||
                          p.t_chunks < 1 || p.t_chunks > 4))
    return QLORA_ERR_CUDA;
  if (T <= 0 || S <= 0) return QLORA_OK;
  const Pair2Sched sc = pair2_schedule(T, S, max_pairs, aux_balance() ? p.aux_tiles : 0);
  p.sk_P = sc.P;
  p.sk_R = sc.R;
  p.sk_L = sc.L;
  p.sk_W = sc.W;
  p.sk_base = sc.base;
  p.sk_A = sc.A;
  p.sk_La = sc.La;
  const bool may_split = sc.W > 0 && (sc.A > 0 || (sc.L > 0 && sc.L < S));
  if (sc.launch > kPair2MaxPairs || (may_split && (!p.sk_part || !p.sk_count))) return QLORA_ERR_CUDA;
  g_last_pairs = sc.launch;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(2 * sc.launch, 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  if (cudaLaunchKernelEx(&cfg, tc_gemm_nf4_pair2_kernel<C>, o.A, o.Ax, o.Bx, o.Y, o.L1, o.Tout, o.Tout2, p) !=
      cudaSuccess)
    return QLORA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// Ring and staging: 3 slots and 4 staging buffers by default (64 KB of staging holds a
// whole accumulator's bf16 rows, so accumulator 0 leaves TMEM without waiting for any
// store); QLORA_B200_PAIR2=4x2 selects 4 slots and 2 buffers (read on every call, for
// measurement). On the q_proj workload 3 x 4 ran the forward and dX GEMMs in 198 and
// 199 us against 214 and 217 us for 4 x 2 on the same B200.
static bool pair2_shallow_stage() {
  const char* e = std::getenv("QLORA_B200_PAIR2");
  return e && std::strcmp(e, "4x2") == 0;
}
using Pair2Fwd = Pair2Cfg<false, 3, 4>;
using Pair2Dx = Pair2Cfg<true, 3, 4>;

qlora_status launch_gemm_pair2(bool dx, const GemmOperands& o, GemmParams p, cudaStream_t s) {
  if (pair2_shallow_stage()) {
    if (!dx) return launch_pair2_cfg<Pair2Cfg<false, 4, 2>>(o, p, s);
    return launch_pair2_cfg<Pair2Cfg<true, 4, 2>>(o, p, s);
  }
  if (!dx) return launch_pair2_cfg<Pair2Fwd>(o, p, s);
  return launch_pair2_cfg<Pair2Dx>(o, p, s);
}

int pair2_spare_sms(bool dx, int num_tiles, int steps) {
  const int mp = std::min(dx ? pair2_max_clusters<Pair2Dx>() : pair2_max_clusters<Pair2Fwd>(), pair2_pair_cap());
  if (mp <= 0) return 0;
  return num_sms() - 2 * pair2_schedule(num_tiles, steps, mp).launch;
}

qlora_status launch_gemm_pair(bool dx, const GemmOperands& o, const GemmParams& p, cudaStream_t s) {
  if (!dx) return launch_pair_cfg<PairCfg<false>>(o, p, s);
  return launch_pair_cfg<PairCfg<true>>(o, p, s);
}

qlora_status launch_gemm(GemmKind kind, int bn, const GemmOperands& o, const GemmParams& p, cudaStream_t s) {
  switch (kind) {
    case GemmKind::FwdNF4: return launch_cfg<GemmCfg<256, false, false, true, false, 3>>(o, p, 1, s);
    case GemmKind::DxNF4: return launch_cfg<GemmCfg<256, false, true, true, false, 3>>(o, p, 1, s);
    case GemmKind::FwdBF16: return launch_cfg<GemmCfg<256, false, false, false, false, 4>>(o, p, 1, s);
    case GemmKind::DxBF16: return launch_cfg<GemmCfg<256, false, true, false, false, 4>>(o, p, 1, s);
    // thin products: one CTA per SM, split-K; a 4-stage ring (96 KB of shared memory)
    // for r <= 64 so that the products the backward runs side by side (U and dL2), and
    // T beside the allocation pass, can share SMs (measured: the step 8 us shorter)
    case GemmKind::ThinKK:  // A K-major, B K-major, fp32 partials
      if (bn <= 64) return launch_cfg<GemmCfg<64, false, false, false, true, 4>>(o, p, 1, s);
      if (bn <= 128) return launch_cfg<GemmCfg<128, false, false, false, true, 6>>(o, p, 1, s);
      return launch_cfg<GemmCfg<256, false, false, false, true, 4>>(o, p, 1, s);
    case GemmKind::ThinKM:  // A K-major, B MN-major
      if (bn <= 64) return launch_cfg<GemmCfg<64, false, true, false, true, 4>>(o, p, 1, s);
      if (bn <= 128) return launch_cfg<GemmCfg<128, false, true, false, true, 6>>(o, p, 1, s);
      return launch_cfg<GemmCfg<256, false, true, false, true, 4>>(o, p, 1, s);
    case GemmKind::ThinMM:  // A MN-major, B MN-major
      if (bn <= 64) return launch_cfg<GemmCfg<64, true, true, false, true, 4>>(o, p, 1, s);
      if (bn <= 128) return launch_cfg<GemmCfg<128, true, true, false, true, 6>>(o, p, 1, s);
      return launch_cfg<GemmCfg<256, true, true, false, true, 4>>(o, p, 1, s);
  }
  return QLORA_ERR_UNSUPPORTED;
}

}  // namespace qlb
