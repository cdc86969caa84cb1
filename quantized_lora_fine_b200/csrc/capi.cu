// C entry points: host-side validation, workspace carving and the launch
// sequence of each operation. Every compute step runs in this library's kernels.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "gemm.cuh"
#include "internal.cuh"

using namespace qlb;

namespace {

constexpr int kThinTargetCtas = 148;  // split-K target for the thin LoRA products, about one CTA per SM
                                      // (fixed: results do not depend on the device's SM count)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// out x in matrices of the codec entry points: both positive and at most 2^40
// elements in all (the grids count chunks of 16384 elements in 32 bits, and
// every byte count stays far inside 64 bits).
constexpr int64_t kMaxCodecNumel = int64_t(1) << 40;
inline bool codec_dims_ok(int64_t out, int64_t in) {
  return out > 0 && in > 0 && out <= kMaxCodecNumel && in <= kMaxCodecNumel / out;
}
inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
inline cudaStream_t S(qlora_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

qlora_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  static int checked_dev = -1;
  static qlora_status cached = QLORA_OK;
  if (checked_dev == dev) return cached;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return QLORA_ERR_CUDA;
  cached = (major == 10 && minor == 0) ? QLORA_OK : QLORA_ERR_UNSUPPORTED;
  checked_dev = dev;
  return cached;
}

bool qconfig_ok(const nf4_qconfig& q) {
  return q.blocksize == 64 && q.dq_blocksize == 256 && (q.double_quant == 0 || q.double_quant == 1);
}

struct ThinSplit {
  int tiles, splits, kps;
};

ThinSplit thin_split(int64_t rows, int64_t ksteps) {
  ThinSplit t;
  t.tiles = int((rows + 127) / 128);
  static const int target = [] {
    const char* e = std::getenv("QLORA_B200_THIN_CTAS");
    const int v = e ? std::atoi(e) : 0;
    return v > 0 ? v : kThinTargetCtas;
  }();
  int sp = std::max(1, int(target / t.tiles));  // one wave of CTAs
  sp = int(std::min<int64_t>(sp, ksteps));
  t.kps = int((ksteps + sp - 1) / sp);
  t.splits = int((ksteps + t.kps - 1) / t.kps);
  return t;
}

int thin_bn(int r) { return r <= 64 ? 64 : (r <= 128 ? 128 : 256); }

// ---- workspace layouts

static_assert(size_t(kPair2CounterInts + 4 * kPair2MaxTBlocks) * sizeof(int) <= kGemmCounterBytes,
              "pair-GEMM counters and T flags fit their region");

struct FwdLayout {
  size_t scales, l2t, t, part, gpart, counters, total;
};

FwdLayout fwd_layout(int64_t M, int64_t out, int64_t in, int32_t r) {
  FwdLayout L;
  L.counters = kStatusBytes;
  size_t off = kReservedBytes;
  L.scales = off; off += up256(size_t(out) * size_t(in / 64) * 4);
  L.l2t = off;    off += up256(size_t(out) * r * 2);
  L.t = off;      off += up256(size_t(M) * r * 2);
  const ThinSplit ts = thin_split(M, in / 64);
  L.part = off;   off += up256(size_t(ts.splits) * size_t(M) * r * 4);
  L.gpart = off;  off += up256(pair2_partial_bytes(M, out));   // pair GEMM: split last round
  L.total = off;
  return L;
}

struct BwdLayout {
  size_t scales, l1s, t, u, su, part, part2, gpart, counters, total;
};

BwdLayout bwd_layout(int64_t M, int64_t out, int64_t in, int32_t r) {
  BwdLayout L;
  L.counters = kStatusBytes;
  size_t off = kReservedBytes;
  L.scales = off; off += up256(size_t(out) * size_t(in / 64) * 4);
  L.l1s = off;    off += up256(size_t(in) * r * 2);
  L.t = off;      off += up256(size_t(M) * r * 2);
  L.u = off;      off += up256(size_t(M) * r * 2);
  L.su = off;     off += up256(size_t(M) * r * 2);
  const ThinSplit a = thin_split(M, in / 64), b = thin_split(M, out / 64);
  const ThinSplit c = thin_split(out, (M + 63) / 64), d = thin_split(in, (M + 63) / 64);
  size_t part = std::max({size_t(a.splits) * M * r, size_t(b.splits) * M * r, size_t(c.splits) * out * r,
                          size_t(d.splits) * in * r}) * 4;
  L.part = off;   off += up256(part);
  L.part2 = off;  off += up256(size_t(c.splits) * out * r * 4);   // dL2 partials on the side stream
  L.gpart = off;  off += up256(pair2_partial_bytes(M, in));         // pair GEMM: split last round
  L.total = off;
  return L;
}

qlora_status check_linear(const qlora_weight* w, int64_t M, int32_t r) {
  if (!w) return QLORA_ERR_NULL;
  if (w->out <= 0 || w->in <= 0 || M <= 0) return QLORA_ERR_SHAPE;
  if (w->in % 256 || w->out % 256) return QLORA_ERR_SHAPE;
  if (w->in > (int64_t(1) << 30) || w->out > (int64_t(1) << 30) || M > (int64_t(1) << 30)) return QLORA_ERR_SHAPE;
  // split-K tile counters: one per 128 rows of M, out or in; the backward runs two
  // products at once, each on its own half of the counters
  if ((std::max({M, w->out, w->in}) + 127) / 128 > kMaxCounterTiles / 2) return QLORA_ERR_SHAPE;
  if (r < 8 || r > 256 || r % 8) return QLORA_ERR_SHAPE;
  if (w->is_bf16) {
    if (!w->w_bf16) return QLORA_ERR_NULL;
    if (!aligned16(w->w_bf16)) return QLORA_ERR_ALIGN;
  } else {
    if (!qconfig_ok(w->q)) return QLORA_ERR_UNSUPPORTED;
    if (!w->codes) return QLORA_ERR_NULL;
    if (!aligned16(w->codes)) return QLORA_ERR_ALIGN;
    if (w->q.double_quant) {
      if (!w->absmax_q || !w->absmax2) return QLORA_ERR_NULL;
    } else if (!w->absmax) {
      return QLORA_ERR_NULL;
    }
  }
  return QLORA_OK;
}

// thin product into fp32 partials then a reduction
struct Thin {
  GemmKind kind;
  const void* a; int64_t a_inner, a_outer;  // A tensor as stored: inner x outer (row-major)
  const void* b; int64_t b_inner, b_outer;
  int64_t rows;        // D rows
  int64_t ksteps;      // K / 64 (ceil)
  int r;
};

qlora_status run_thin(const Thin& t, float* part, int* counters, void* fin_out, int fin_mode, float fin_scale,
                      int* status, cudaStream_t s, void* fin_out2 = nullptr) {
  const ThinSplit ts = thin_split(t.rows, t.ksteps);
  const int bn = thin_bn(t.r);
  GemmOperands o;
  std::memset(&o, 0, sizeof(o));
  const bool a_mn = t.kind == GemmKind::ThinMM;
  const bool b_mn = t.kind != GemmKind::ThinKK;
  if (!make_tmap_2d(&o.A, t.a, TmapType::BF16, t.a_inner, t.a_outer, t.a_inner * 2, 64, a_mn ? 64 : 128, true))
    return QLORA_ERR_CUDA;
  if (!make_tmap_2d(&o.B, t.b, TmapType::BF16, t.b_inner, t.b_outer, t.b_inner * 2, 64, b_mn ? 64 : bn, true))
    return QLORA_ERR_CUDA;
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = int(t.rows);
  p.N = t.r;
  p.num_k_main = int(t.ksteps);
  p.num_k_ext = 0;
  p.tiles_m = ts.tiles;
  p.tiles_n = 1;
  p.splits = ts.splits;
  p.ksteps_per_split = ts.kps;
  p.out = part;
  p.ld_out = t.r;
  p.split_stride = t.rows * t.r;
  p.status = status;
  p.counters = counters;
  p.fin_out = fin_out;
  p.fin_mode = fin_mode;
  p.fin_scale = fin_scale;
  p.fin_out2 = fin_out2;
  return launch_gemm(t.kind, bn, o, p, s);
}

#define QLB_TRY(x)                         \
  do {                                     \
    qlora_status _st = (x);                \
    if (_st != QLORA_OK) return _st;       \
  } while (0)

cudaEvent_t g_prof[4] = {nullptr, nullptr, nullptr, nullptr};

// Profiling events are recorded as timestamp nodes when the stream is being
// captured into a CUDA graph.
void record_prof(cudaEvent_t e, cudaStream_t s) {
  if (!e) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  else
    cudaEventRecord(e, s);
}

}  // namespace

namespace qlb {
// Programmatic dependent launch is on unless QLORA_B200_PDL=0 (kept switchable for
// measurement: the results are the same either way).
bool pdl_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("QLORA_B200_PDL");
    v = (e && std::strcmp(e, "0") == 0) ? 0 : 1;
  }
  return v == 1;
}
}  // namespace qlb

namespace {

// The NF4 GEMMs run on the CTA-pair kernel unless QLORA_B200_GEMM=1cta selects
// the single-CTA kernel (both compute the same values; kept side by side for
// measurement).
// Backward schedule: QLORA_B200_BWD=beside or =serial forces one of the two (read on
// every call, so tests can cover both on any part); otherwise it follows the SMs the
// dX GEMM leaves free.
int bwd_schedule_override() {
  const char* e = std::getenv("QLORA_B200_BWD");
  if (!e) return 0;
  if (std::strcmp(e, "beside") == 0) return 1;
  if (std::strcmp(e, "serial") == 0) return 2;
  return 0;
}

// NF4 GEMM engine: 2 = CTA pairs with 512 x 256 tiles (default), 1 = CTA pairs with
// 256 x 256 tiles (QLORA_B200_GEMM=pair256), 0 = single CTAs (QLORA_B200_GEMM=1cta).
// All compute the same products within rounding; the others are kept for measurement.
int gemm_engine() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("QLORA_B200_GEMM");
    v = (e && std::strcmp(e, "1cta") == 0) ? 0 : (e && std::strcmp(e, "pair256") == 0) ? 1 : 2;
  }
  return v;
}
bool use_pair_kernel() { return gemm_engine() >= 1; }
// T = X L1 inside the forward GEMM unless QLORA_B200_FUSED_T=0 (read on every call; the
// separate T pass is kept for measurement).
bool fused_t_enabled() {
  const char* e = std::getenv("QLORA_B200_FUSED_T");
  return !(e && std::strcmp(e, "0") == 0);
}
// U = dY L2^T inside the dX GEMM: QLORA_B200_FUSED_U=1 always, =0 never, unset when
// the output has at least 32 column tiles of 256 (read on every call). A U tile
// takes a whole tile's turn in the schedule but does about half its MMA work, so it
// pays where its share of the tiles is small: on q_proj (16 column tiles) the dX
// GEMM took 233.5 us with U tiles against 218.8 us, and the backward 280.6 us
// against 277.1 us with U as its own pass.
bool fused_u_wanted(int64_t n_cols) {
  const char* e = std::getenv("QLORA_B200_FUSED_U");
  if (e && std::strcmp(e, "0") == 0) return false;
  if (e && std::strcmp(e, "1") == 0) return true;
  return n_cols / 256 >= 32;
}

// Fused NF4 GEMM on CTA pairs (256 x 256 tiles): out = A . W' + Ax . Bx^T, where
// the LoRA step reads Bx as [N x r] rows: Ax = T with Bx = s.L2^T (fwd), or
// Ax = s.U with Bx = L1 as stored (dX). Codes are read in place, scales from S_t.
// (An MN-major LoRA B read straight from L2 [r x out] was measured 12 us slower
// per forward GEMM on the q_proj workload than this transposed copy.)
// With aux_out (512 x 256 engine) the GEMM also computes the LoRA product its
// output tiles' LoRA step reads, in its own aux tiles before them: forward, T = X L1
// into aux_out (aux_b = L1; Ax must be aux_out); dX, U = dY L2^T into aux_out and
// bf16(aux_scale * U) into aux_out2 (aux_b = L2; Ax must be aux_out2).
qlora_status run_pair(bool dx, const qlora_weight* w, const uint16_t* A, int64_t M, const uint16_t* Ax,
                      const uint16_t* Bx, int32_t r, const float* scales_t, uint16_t* out, int* status,
                      float* gpart, int* gcount, cudaStream_t s, const uint16_t* aux_b = nullptr,
                      uint16_t* aux_out = nullptr, uint16_t* aux_out2 = nullptr, float aux_scale = 0.f) {
  const int64_t o_ = w->out, h = w->in;
  const int64_t Kdim = dx ? o_ : h;
  const int64_t Ndim = dx ? h : o_;
  GemmOperands pp;
  std::memset(&pp, 0, sizeof(pp));
  if (!make_tmap_2d(&pp.A, A, TmapType::BF16, Kdim, M, Kdim * 2, 64, 128, true)) return QLORA_ERR_CUDA;
  if (!make_tmap_2d(&pp.Ax, Ax, TmapType::BF16, r, M, int64_t(r) * 2, 64, 128, true)) return QLORA_ERR_CUDA;
  if (!make_tmap_2d(&pp.Bx, Bx, TmapType::BF16, r, Ndim, int64_t(r) * 2, 64, 128, true)) return QLORA_ERR_CUDA;
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = int(M);
  p.N = int(Ndim);
  p.num_k_main = int(Kdim / 64);
  p.num_k_ext = (r + 63) / 64;
  p.tiles_m = int((M + 255) / 256);
  p.tiles_n = int(Ndim / 256);
  p.splits = 1;
  p.ksteps_per_split = p.num_k_main;
  p.out = out;
  p.ld_out = Ndim;
  p.status = status;
  p.codes = w->codes;
  p.codes_ld = h / 2;
  p.scales = scales_t;
  p.scales_ld = o_;
  if (gemm_engine() == 2) {
    p.tiles_m = int((M + 511) / 512);
    p.sk_part = gpart;
    p.sk_count = gcount;
    // output written by TMA: 128-row x 64-column boxes, 128-byte swizzle
    if (!make_tmap_2d(&pp.Y, out, TmapType::BF16, Ndim, M, Ndim * 2, 64, 128, true)) return QLORA_ERR_CUDA;
    if (aux_out) {
      p.aux_tiles = p.tiles_m;
      p.t_chunks = (r + 63) / 64;
      p.t_flags = gcount + kPair2CounterInts;
      const int t_n = p.t_chunks <= 2 ? 128 : 256;   // the aux tiles' MMA width (as the kernel)
      if (!dx) {
        // T tiles: B = L1 [in x r] as MN-major 64 x 64 chunks
        if (!make_tmap_2d(&pp.L1, aux_b, TmapType::BF16, r, h, int64_t(r) * 2, 64, 64, true)) return QLORA_ERR_CUDA;
      } else {
        // U tiles: B = L2 [r x out] K-major, one box of t_n / 2 rows per CTA
        if (!make_tmap_2d(&pp.L1, aux_b, TmapType::BF16, o_, r, o_ * 2, 64, t_n / 2, true)) return QLORA_ERR_CUDA;
        if (!aux_out2) return QLORA_ERR_CUDA;
        if (!make_tmap_2d(&pp.Tout2, aux_out2, TmapType::BF16, r, M, int64_t(r) * 2, 64, 128, true))
          return QLORA_ERR_CUDA;
        p.aux_dual = 1;
        p.aux_scale = aux_scale;
      }
      // T or U [M x r] stored in 128 x 64 boxes
      if (!make_tmap_2d(&pp.Tout, aux_out, TmapType::BF16, r, M, int64_t(r) * 2, 64, 128, true)) return QLORA_ERR_CUDA;
    }
  }
  record_prof(g_prof[dx ? 2 : 0], s);
  const qlora_status st = gemm_engine() == 2 ? launch_gemm_pair2(dx, pp, p, s) : launch_gemm_pair(dx, pp, p, s);
  record_prof(g_prof[dx ? 3 : 1], s);
  return st;
}

// main GEMM with NF4 or bf16 weight and the LoRA extension
qlora_status run_main(bool dx, const qlora_weight* w, const uint16_t* A, int64_t M, const uint16_t* Ax,
                      const uint16_t* Bx, int32_t r, const float* scales_t, uint16_t* out, int* status,
                      cudaStream_t s) {
  const int64_t o_ = w->out, h = w->in;
  const int64_t Kdim = dx ? o_ : h;   // reduction length
  const int64_t Ndim = dx ? h : o_;   // output columns
  GemmOperands op;
  std::memset(&op, 0, sizeof(op));
  if (!make_tmap_2d(&op.A, A, TmapType::BF16, Kdim, M, Kdim * 2, 64, 128, true)) return QLORA_ERR_CUDA;
  if (!make_tmap_2d(&op.Ax, Ax, TmapType::BF16, r, M, int64_t(r) * 2, 64, 128, true)) return QLORA_ERR_CUDA;
  if (!make_tmap_2d(&op.Bx, Bx, TmapType::BF16, r, Ndim, int64_t(r) * 2, 64, 256, true)) return QLORA_ERR_CUDA;
  GemmKind kind;
  if (w->is_bf16) {
    if (!dx) {
      if (!make_tmap_2d(&op.B, w->w_bf16, TmapType::BF16, h, o_, h * 2, 64, 256, true)) return QLORA_ERR_CUDA;
      kind = GemmKind::FwdBF16;
    } else {
      if (!make_tmap_2d(&op.B, w->w_bf16, TmapType::BF16, h, o_, h * 2, 64, 64, true)) return QLORA_ERR_CUDA;
      kind = GemmKind::DxBF16;
    }
  } else {
    if (!dx) {
      if (!make_tmap_2d(&op.codes, w->codes, TmapType::U8, h / 2, o_, h / 2, 32, 256, false)) return QLORA_ERR_CUDA;
      if (!make_tmap_2d(&op.scales, scales_t, TmapType::F32, o_, h / 64, o_ * 4, 256, 1, false)) return QLORA_ERR_CUDA;
      kind = GemmKind::FwdNF4;
    } else {
      if (!make_tmap_2d(&op.codes, w->codes, TmapType::U8, h / 2, o_, h / 2, 128, 64, true)) return QLORA_ERR_CUDA;
      if (!make_tmap_2d(&op.scales, scales_t, TmapType::F32, o_, h / 64, o_ * 4, 64, 4, false)) return QLORA_ERR_CUDA;
      kind = GemmKind::DxNF4;
    }
  }
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = int(M);
  p.N = int(Ndim);
  p.num_k_main = int(Kdim / 64);
  p.num_k_ext = (r + 63) / 64;
  p.tiles_m = int((M + 127) / 128);
  p.tiles_n = int(Ndim / 256);
  p.splits = 1;
  p.ksteps_per_split = p.num_k_main;
  p.out = out;
  p.ld_out = Ndim;
  p.split_stride = 0;
  p.status = status;
  record_prof(g_prof[dx ? 2 : 0], s);
  const qlora_status st = launch_gemm(kind, 256, op, p, s);
  record_prof(g_prof[dx ? 3 : 1], s);
  return st;
}


// ---- side stream for independent small kernels (fork / join with events)
//
// One non-blocking stream and two events per device, created on first use. A
// call records `fork` on the caller's stream, makes the side stream wait on it,
// launches independent work there, records `join` on the side stream and makes
// the caller's stream wait on it before the dependent work. Works inside CUDA
// graph capture (the side stream joins the capture through the event). Calls
// from several host threads serialize on the mutex while they enqueue.
struct SideStream {
  cudaStream_t stream = nullptr;   // default priority: small independent kernels
  cudaStream_t hi = nullptr;       // highest priority: a GEMM that shares the GPU
  cudaEvent_t fork = nullptr, mid = nullptr, join = nullptr;
};
constexpr int kMaxSideDevices = 64;
std::mutex g_side_mu;
SideStream g_side[kMaxSideDevices];

// Returns nullptr (run everything on the caller's stream) when no side stream
// can be made.
SideStream* side_stream() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxSideDevices) return nullptr;
  SideStream& ss = g_side[dev];
  if (!ss.stream) {
    // hi: when its tensor-core GEMM and a caller-stream kernel become ready together,
    // the GEMM's CTAs are placed first
    int least = 0, greatest = 0;
    cudaDeviceGetStreamPriorityRange(&least, &greatest);
    if (cudaStreamCreateWithFlags(&ss.stream, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithPriority(&ss.hi, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.mid, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      ss = SideStream();
      return nullptr;
    }
  }
  return &ss;
}

// side waits for the work enqueued on s so far (side = ss->stream by default, or ss->hi)
qlora_status fork_to(SideStream* ss, cudaStream_t s, cudaStream_t side = nullptr) {
  if (cudaEventRecord(ss->fork, s) != cudaSuccess ||
      cudaStreamWaitEvent(side ? side : ss->stream, ss->fork, 0) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
}

// A second fork point: side waits for the work enqueued on s so far.
qlora_status handoff_to(SideStream* ss, cudaStream_t s, cudaStream_t side) {
  if (cudaEventRecord(ss->mid, s) != cudaSuccess || cudaStreamWaitEvent(side, ss->mid, 0) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
}

// s waits for everything enqueued on side (ss->stream by default, or ss->hi)
qlora_status join_from(SideStream* ss, cudaStream_t s, cudaStream_t side = nullptr) {
  if (cudaEventRecord(ss->join, side ? side : ss->stream) != cudaSuccess ||
      cudaStreamWaitEvent(s, ss->join, 0) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
}

}  // namespace

extern "C" {

const char* qlora_status_str(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_NULL: return "null pointer";
    case QLORA_ERR_SHAPE: return "unsupported shape";
    case QLORA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case QLORA_ERR_DTYPE: return "unknown dtype";
    case QLORA_ERR_UNSUPPORTED: return "unsupported device or configuration";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case QLORA_ERR_NONFINITE: return "non-finite weight";
    case QLORA_ERR_TIMEOUT: return "device pipeline wait timed out";
  }
  return "unknown status";
}

int32_t qlora_pair_clusters(void) { return last_pair_clusters(); }

qlora_status qlora_pair_schedule(int32_t tiles, int32_t aux_tiles, int32_t steps, int32_t pairs, int32_t* out) {
  if (!out) return QLORA_ERR_NULL;
  if (tiles < 1 || aux_tiles < 0 || aux_tiles > tiles || steps < 1 || pairs < 1 || pairs > kPair2MaxPairs)
    return QLORA_ERR_SHAPE;
  pair2_schedule_of(tiles, aux_tiles, steps, pairs, out);
  return QLORA_OK;
}

qlora_status qlora_profile_events(void* fwd_begin, void* fwd_end, void* dx_begin, void* dx_end) {
  g_prof[0] = static_cast<cudaEvent_t>(fwd_begin);
  g_prof[1] = static_cast<cudaEvent_t>(fwd_end);
  g_prof[2] = static_cast<cudaEvent_t>(dx_begin);
  g_prof[3] = static_cast<cudaEvent_t>(dx_end);
  return QLORA_OK;
}

qlora_status qlora_device_check(int device) {
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return (major == 10 && minor == 0) ? QLORA_OK : QLORA_ERR_UNSUPPORTED;
}

qlora_status qlora_read_status(const void* workspace, qlora_stream_t stream) {
  if (!workspace) return QLORA_ERR_WORKSPACE;
  int v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, S(stream)) != cudaSuccess)
    return QLORA_ERR_CUDA;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return QLORA_ERR_CUDA;
  return static_cast<qlora_status>(v);
}

qlora_status qlora_reset_status(void* workspace, qlora_stream_t stream) {
  if (!workspace) return QLORA_ERR_WORKSPACE;
  return cudaMemsetAsync(workspace, 0, sizeof(int), S(stream)) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_reset_workspace(void* workspace, size_t workspace_bytes, qlora_stream_t stream) {
  if (!workspace || workspace_bytes < kStatusBytes) return QLORA_ERR_WORKSPACE;
  const size_t n = std::min(workspace_bytes, kReservedBytes);
  return cudaMemsetAsync(workspace, 0, n, S(stream)) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

size_t nf4_quantize_workspace_size(int64_t) { return kStatusBytes; }

qlora_status nf4_quantize(const void* W, int32_t w_dtype, int64_t out, int64_t in, nf4_qconfig q, uint8_t* codes,
                          float* absmax, uint8_t* absmax_q, float* absmax2, void* workspace, size_t workspace_bytes,
                          qlora_stream_t stream) {
  if (w_dtype != QLORA_DTYPE_BF16 && w_dtype != QLORA_DTYPE_F32) return QLORA_ERR_DTYPE;
  if (!qconfig_ok(q)) return QLORA_ERR_UNSUPPORTED;
  if (!codec_dims_ok(out, in)) return QLORA_ERR_SHAPE;
  const int64_t numel = out * in;
  if (numel % 2) return QLORA_ERR_SHAPE;
  if (!W || !codes) return QLORA_ERR_NULL;
  if (q.double_quant ? (!absmax_q || !absmax2) : !absmax) return QLORA_ERR_NULL;
  if (!aligned16(W)) return QLORA_ERR_ALIGN;
  if (!aligned16(codes)) return QLORA_ERR_ALIGN;
  if (!workspace || workspace_bytes < kStatusBytes || !aligned16(workspace)) return QLORA_ERR_WORKSPACE;
  QLB_TRY(check_device());
  return launch_quantize(W, w_dtype, numel, q.double_quant != 0, codes, absmax, absmax_q, absmax2,
                         static_cast<int*>(workspace), S(stream));
}

qlora_status nf4_quantize_batch(int32_t n, const uint16_t* const* W_ptrs, const int64_t* numel, int32_t w_dtype,
                                nf4_qconfig q, uint8_t* const* codes, float* const* absmax,
                                uint8_t* const* absmax_q, float* const* absmax2, void* workspace,
                                size_t workspace_bytes, qlora_stream_t stream) {
  if (w_dtype != QLORA_DTYPE_BF16) return QLORA_ERR_DTYPE;
  if (!qconfig_ok(q)) return QLORA_ERR_UNSUPPORTED;
  if (n < 1 || n > 512) return QLORA_ERR_SHAPE;
  if (!W_ptrs || !numel || !codes) return QLORA_ERR_NULL;
  const bool dq = q.double_quant != 0;
  if (dq ? (!absmax_q || !absmax2) : !absmax) return QLORA_ERR_NULL;
  for (int i = 0; i < n; ++i) {
    if (!W_ptrs[i] || !codes[i]) return QLORA_ERR_NULL;
    if (dq ? (!absmax_q[i] || !absmax2[i]) : !absmax[i]) return QLORA_ERR_NULL;
    if (numel[i] <= 0 || numel[i] % 2 || numel[i] > kMaxCodecNumel) return QLORA_ERR_SHAPE;
    if (!aligned16(W_ptrs[i]) || !aligned16(codes[i])) return QLORA_ERR_ALIGN;
  }
  if (!workspace || workspace_bytes < kStatusBytes || !aligned16(workspace)) return QLORA_ERR_WORKSPACE;
  QLB_TRY(check_device());
  return launch_quantize_batch(n, W_ptrs, numel, dq, codes, absmax, absmax_q, absmax2,
                               static_cast<int*>(workspace), S(stream));
}

namespace {
qlora_status check_merge(const qlora_weight* w, const uint16_t* L1, const uint16_t* L2, int32_t r) {
  if (!w || !L1 || !L2) return QLORA_ERR_NULL;
  if (w->out <= 0 || w->in <= 0 || w->in % 64) return QLORA_ERR_SHAPE;
  if (w->in > (int64_t(1) << 30) || w->out > (int64_t(1) << 30)) return QLORA_ERR_SHAPE;
  if (w->in / 64 > 65535 * int64_t(1) || (w->out + 63) / 64 > 65535) return QLORA_ERR_SHAPE;
  if (r < 1 || r > 256) return QLORA_ERR_SHAPE;
  if (w->is_bf16) {
    if (!w->w_bf16) return QLORA_ERR_NULL;
    if (!aligned16(w->w_bf16)) return QLORA_ERR_ALIGN;
  } else {
    if (!qconfig_ok(w->q)) return QLORA_ERR_UNSUPPORTED;
    if (!w->codes || (w->q.double_quant ? (!w->absmax_q || !w->absmax2) : !w->absmax)) return QLORA_ERR_NULL;
    if (!aligned16(w->codes)) return QLORA_ERR_ALIGN;
  }
  return QLORA_OK;
}

qlora_status merge_into(const qlora_weight* w, const uint16_t* L1, const uint16_t* L2, int32_t r, float scale,
                        uint16_t* W_out, uint8_t* q_codes, float* q_absmax, int* status, cudaStream_t s) {
  return launch_lora_merge(w->codes, w->absmax, w->absmax_q, w->absmax2, w->q.double_quant != 0,
                           w->is_bf16 ? w->w_bf16 : nullptr, w->out, w->in, L1, L2, r, double(scale), W_out, q_codes,
                           q_absmax, status, s);
}
}  // namespace

qlora_status qlora_lora_merge(const qlora_weight* w, const uint16_t* L1, const uint16_t* L2, int32_t r, float scale,
                              uint16_t* W_out, qlora_stream_t stream) {
  QLB_TRY(check_merge(w, L1, L2, r));
  if (!W_out) return QLORA_ERR_NULL;
  if (!aligned16(W_out)) return QLORA_ERR_ALIGN;
  QLB_TRY(check_device());
  return merge_into(w, L1, L2, r, scale, W_out, nullptr, nullptr, nullptr, S(stream));
}

size_t qlora_lora_merge_requantize_workspace_size(int64_t out, int64_t in) {
  if (out <= 0 || in <= 0) return 0;
  return kReservedBytes + up256(size_t(out) * size_t(in / 64) * sizeof(float));
}

qlora_status qlora_lora_merge_requantize(const qlora_weight* w, const uint16_t* L1, const uint16_t* L2, int32_t r,
                                         float scale, nf4_qconfig q, uint8_t* codes, float* absmax,
                                         uint8_t* absmax_q, float* absmax2, void* workspace,
                                         size_t workspace_bytes, qlora_stream_t stream) {
  QLB_TRY(check_merge(w, L1, L2, r));
  if (!qconfig_ok(q)) return QLORA_ERR_UNSUPPORTED;
  if (!codes || (q.double_quant ? (!absmax_q || !absmax2) : !absmax)) return QLORA_ERR_NULL;
  if (!aligned16(codes)) return QLORA_ERR_ALIGN;
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < qlora_lora_merge_requantize_workspace_size(w->out, w->in))
    return QLORA_ERR_WORKSPACE;
  QLB_TRY(check_device());
  // the exact fp32 scales go to the caller's absmax when given, else to the workspace
  // (scratch after the split-K counters, which other calls on this workspace expect to find zero)
  float* amax = absmax ? absmax : reinterpret_cast<float*>(static_cast<char*>(workspace) + kReservedBytes);
  QLB_TRY(merge_into(w, L1, L2, r, scale, nullptr, codes, amax, static_cast<int*>(workspace), S(stream)));
  if (q.double_quant) return launch_dq_scales(amax, w->out * (w->in / 64), absmax_q, absmax2, S(stream));
  return QLORA_OK;
}

namespace {
qlora_status check_stage(const qlora_weight* w) {
  if (!w) return QLORA_ERR_NULL;
  if (w->is_bf16) return QLORA_ERR_UNSUPPORTED;
  if (!qconfig_ok(w->q)) return QLORA_ERR_UNSUPPORTED;
  if (w->out <= 0 || w->in <= 0 || w->out > (int64_t(1) << 30) || w->in > (int64_t(1) << 30)) return QLORA_ERR_SHAPE;
  if (!codec_dims_ok(w->out, w->in)) return QLORA_ERR_SHAPE;
  if ((w->out * w->in) % 64) return QLORA_ERR_SHAPE;
  if (!w->codes || (w->q.double_quant ? (!w->absmax_q || !w->absmax2) : !w->absmax)) return QLORA_ERR_NULL;
  if (!aligned16(w->codes)) return QLORA_ERR_ALIGN;
  return QLORA_OK;
}
}  // namespace

size_t nf4_quantize_residual_workspace_size(int64_t numel) {
  if (numel <= 0) return 0;
  return kReservedBytes + up256(size_t(numel) * sizeof(float));
}

qlora_status nf4_quantize_residual(const uint16_t* W, const qlora_weight* w1, nf4_qconfig q, uint8_t* codes,
                                   float* absmax, uint8_t* absmax_q, float* absmax2, void* workspace,
                                   size_t workspace_bytes, qlora_stream_t stream) {
  QLB_TRY(check_stage(w1));
  if (!W) return QLORA_ERR_NULL;
  if (!aligned16(W)) return QLORA_ERR_ALIGN;
  if (!qconfig_ok(q)) return QLORA_ERR_UNSUPPORTED;
  if (!codes || (q.double_quant ? (!absmax_q || !absmax2) : !absmax)) return QLORA_ERR_NULL;
  if (!aligned16(codes)) return QLORA_ERR_ALIGN;
  const int64_t numel = w1->out * w1->in;
  if (!workspace || !aligned16(workspace) || workspace_bytes < nf4_quantize_residual_workspace_size(numel))
    return QLORA_ERR_WORKSPACE;
  QLB_TRY(check_device());
  // R after the split-K counters, which other calls on this workspace expect to find zero
  float* R = reinterpret_cast<float*>(static_cast<char*>(workspace) + kReservedBytes);
  QLB_TRY(launch_nf4_residual(W, w1->codes, w1->absmax, w1->absmax_q, w1->absmax2, w1->q.double_quant != 0, numel, R,
                              S(stream)));
  return launch_quantize(R, QLORA_DTYPE_F32, numel, q.double_quant != 0, codes, absmax, absmax_q, absmax2,
                         static_cast<int*>(workspace), S(stream));
}

qlora_status nf4_dequantize_two_stage(const qlora_weight* w1, const qlora_weight* w2, uint16_t* W_out,
                                      qlora_stream_t stream) {
  QLB_TRY(check_stage(w1));
  QLB_TRY(check_stage(w2));
  if (w1->out != w2->out || w1->in != w2->in) return QLORA_ERR_SHAPE;
  if (!W_out) return QLORA_ERR_NULL;
  if (!aligned16(W_out)) return QLORA_ERR_ALIGN;
  QLB_TRY(check_device());
  return launch_dequantize_two_stage(w1->codes, w1->absmax, w1->absmax_q, w1->absmax2, w1->q.double_quant != 0,
                                     w2->codes, w2->absmax, w2->absmax_q, w2->absmax2, w2->q.double_quant != 0,
                                     w1->out * w1->in, W_out, S(stream));
}

qlora_status nf4_dequantize(const qlora_weight* w, uint16_t* W_out, qlora_stream_t stream) {
  if (!w || !W_out) return QLORA_ERR_NULL;
  if (w->is_bf16) return QLORA_ERR_UNSUPPORTED;
  if (!qconfig_ok(w->q)) return QLORA_ERR_UNSUPPORTED;
  if (!codec_dims_ok(w->out, w->in)) return QLORA_ERR_SHAPE;
  const int64_t numel = w->out * w->in;
  if (numel % 2) return QLORA_ERR_SHAPE;
  if (!w->codes) return QLORA_ERR_NULL;
  if (w->q.double_quant ? (!w->absmax_q || !w->absmax2) : !w->absmax) return QLORA_ERR_NULL;
  if (!aligned16(w->codes) || !aligned16(W_out)) return QLORA_ERR_ALIGN;
  QLB_TRY(check_device());
  return launch_dequantize(w->codes, w->absmax, w->absmax_q, w->absmax2, w->q.double_quant != 0, numel, W_out,
                           S(stream));
}

size_t qlora_fwd_workspace_size(int64_t M, int64_t out, int64_t in, int32_t r) {
  if (M <= 0 || out <= 0 || in <= 0 || r <= 0) return 0;
  return fwd_layout(M, out, in, r).total;
}

size_t qlora_bwd_workspace_size(int64_t M, int64_t out, int64_t in, int32_t r) {
  if (M <= 0 || out <= 0 || in <= 0 || r <= 0) return 0;
  return bwd_layout(M, out, in, r).total;
}

namespace {
// The forward with T either computed here (T_in == NULL: T = X L1 into T_save or
// the workspace) or supplied by the caller.
qlora_status linear_fwd_impl(const qlora_weight* w, const uint16_t* X, int64_t M, const uint16_t* L1,
                             const uint16_t* T_in, const uint16_t* L2, int32_t r, float scale, uint16_t* Y,
                             uint16_t* T_save, void* workspace, size_t workspace_bytes, cudaStream_t s) {
  const FwdLayout L = fwd_layout(M, w->out, w->in, r);
  if (workspace_bytes < L.total) return QLORA_ERR_WORKSPACE;
  QLB_TRY(check_device());
  char* ws = static_cast<char*>(workspace);
  int* status = reinterpret_cast<int*>(ws);
  float* scales_t = reinterpret_cast<float*>(ws + L.scales);
  uint16_t* l2t = reinterpret_cast<uint16_t*>(ws + L.l2t);
  float* part = reinterpret_cast<float*>(ws + L.part);
  const int64_t h = w->in, o_ = w->out;
  int* counters = reinterpret_cast<int*>(ws + L.counters);
  // T = X L1 inside the NF4 GEMM (its T tiles read X while it is in L2), unless T is
  // given, the weight is protected, another engine runs, or M has too many row blocks
  const bool fuse_t = !T_in && !w->is_bf16 && gemm_engine() == 2 && fused_t_enabled() &&
                      (M + 511) / 512 <= kPair2MaxTBlocks;
  const bool thin_t = !T_in && !fuse_t;
  // The scale expansion and s.L2^T are independent of T and of each other: the
  // expansion runs on the side stream, s.L2^T beside it on this stream, or beside T
  // when T = X L1 runs here as its own pass (A = X K-major, B = L1 [h x r] MN-major)
  std::lock_guard<std::mutex> lock(g_side_mu);
  SideStream* ss = side_stream();
  cudaStream_t aux = s;
  if (ss) {
    QLB_TRY(fork_to(ss, s));
    aux = ss->stream;
  }
  if (!w->is_bf16)
    QLB_TRY(launch_expand_scales(w->codes, w->absmax, w->absmax_q, w->absmax2, w->q.double_quant != 0, o_, h,
                                 scales_t, aux));
  QLB_TRY(launch_scale_lora(L2, r, o_, scale, /*transpose=*/true, l2t, thin_t ? aux : s));
  const uint16_t* T = T_in;
  uint16_t* Tw = T_save ? T_save : reinterpret_cast<uint16_t*>(ws + L.t);
  if (thin_t) {
    Thin tt{GemmKind::ThinKM, X, h, M, L1, r, h, M, h / 64, r};
    QLB_TRY(run_thin(tt, part, counters, Tw, 0, 1.f, status, s));
    T = Tw;
  }
  if (ss) QLB_TRY(join_from(ss, s));
  if (fuse_t)
    return run_pair(false, w, X, M, Tw, l2t, r, scales_t, Y, status, reinterpret_cast<float*>(ws + L.gpart),
                    reinterpret_cast<int*>(ws + kStatusBytes + kCounterBytes), s, L1, Tw);
  if (!w->is_bf16 && use_pair_kernel())
    return run_pair(false, w, X, M, T, l2t, r, scales_t, Y, status, reinterpret_cast<float*>(ws + L.gpart),
                    reinterpret_cast<int*>(ws + kStatusBytes + kCounterBytes), s);
  return run_main(false, w, X, M, T, l2t, r, scales_t, Y, status, s);
}

bool lora_shape_ok(int64_t M, int64_t in, int32_t r) {
  return M > 0 && in > 0 && in % 256 == 0 && in <= (int64_t(1) << 30) && M <= (int64_t(1) << 30) &&
         (std::max(M, in) + 127) / 128 <= kMaxCounterTiles && r >= 8 && r <= 256 && r % 8 == 0;
}
}  // namespace

qlora_status qlora_linear_fwd(const qlora_weight* w, const uint16_t* X, int64_t M, const uint16_t* L1,
                              const uint16_t* L2, int32_t r, float scale, uint16_t* Y, uint16_t* T_save,
                              void* workspace, size_t workspace_bytes, qlora_stream_t stream) {
  QLB_TRY(check_linear(w, M, r));
  if (!X || !L1 || !L2 || !Y) return QLORA_ERR_NULL;
  if (!aligned16(X) || !aligned16(L1) || !aligned16(L2) || !aligned16(Y) || (T_save && !aligned16(T_save)))
    return QLORA_ERR_ALIGN;
  if (!workspace || !aligned16(workspace)) return QLORA_ERR_WORKSPACE;
  return linear_fwd_impl(w, X, M, L1, nullptr, L2, r, scale, Y, T_save, workspace, workspace_bytes, S(stream));
}

qlora_status qlora_linear_fwd_t(const qlora_weight* w, const uint16_t* X, int64_t M, const uint16_t* T,
                                const uint16_t* L2, int32_t r, float scale, uint16_t* Y, void* workspace,
                                size_t workspace_bytes, qlora_stream_t stream) {
  QLB_TRY(check_linear(w, M, r));
  if (!X || !T || !L2 || !Y) return QLORA_ERR_NULL;
  if (!aligned16(X) || !aligned16(T) || !aligned16(L2) || !aligned16(Y)) return QLORA_ERR_ALIGN;
  if (!workspace || !aligned16(workspace)) return QLORA_ERR_WORKSPACE;
  return linear_fwd_impl(w, X, M, nullptr, T, L2, r, scale, Y, nullptr, workspace, workspace_bytes, S(stream));
}

size_t qlora_lora_down_workspace_size(int64_t M, int64_t in, int32_t r) {
  if (!lora_shape_ok(M, in, r)) return 0;
  const ThinSplit ts = thin_split(M, in / 64);
  return kReservedBytes + up256(size_t(ts.splits) * size_t(M) * r * 4);
}

qlora_status qlora_lora_down(const uint16_t* X, int64_t M, int64_t in, const uint16_t* L1, int32_t r, uint16_t* T,
                             void* workspace, size_t workspace_bytes, qlora_stream_t stream) {
  if (!lora_shape_ok(M, in, r)) return QLORA_ERR_SHAPE;
  if (!X || !L1 || !T) return QLORA_ERR_NULL;
  if (!aligned16(X) || !aligned16(L1) || !aligned16(T)) return QLORA_ERR_ALIGN;
  if (!workspace || !aligned16(workspace)) return QLORA_ERR_WORKSPACE;
  if (workspace_bytes < qlora_lora_down_workspace_size(M, in, r)) return QLORA_ERR_WORKSPACE;
  QLB_TRY(check_device());
  char* ws = static_cast<char*>(workspace);
  Thin tt{GemmKind::ThinKM, X, in, M, L1, r, in, M, in / 64, r};
  return run_thin(tt, reinterpret_cast<float*>(ws + kReservedBytes), reinterpret_cast<int*>(ws + kStatusBytes), T, 0,
                  1.f, reinterpret_cast<int*>(ws), S(stream));
}

qlora_status qlora_linear_bwd(const qlora_weight* w, const uint16_t* X, const uint16_t* dY, int64_t M,
                              const uint16_t* L1, const uint16_t* L2, int32_t r, float scale,
                              const uint16_t* T_saved, uint16_t* dX, float* dL1, float* dL2, void* workspace,
                              size_t workspace_bytes, qlora_stream_t stream) {
  QLB_TRY(check_linear(w, M, r));
  if (!X || !dY || !L1 || !L2 || !dL1 || !dL2) return QLORA_ERR_NULL;
  if (!aligned16(X) || !aligned16(dY) || !aligned16(L1) || !aligned16(L2) || !aligned16(dL1) || !aligned16(dL2) ||
      (dX && !aligned16(dX)) || (T_saved && !aligned16(T_saved)))
    return QLORA_ERR_ALIGN;
  if (!workspace || !aligned16(workspace)) return QLORA_ERR_WORKSPACE;
  const BwdLayout L = bwd_layout(M, w->out, w->in, r);
  if (workspace_bytes < L.total) return QLORA_ERR_WORKSPACE;
  QLB_TRY(check_device());
  cudaStream_t s = S(stream);
  char* ws = static_cast<char*>(workspace);
  int* status = reinterpret_cast<int*>(ws);
  float* scales_t = reinterpret_cast<float*>(ws + L.scales);
  uint16_t* l1s = reinterpret_cast<uint16_t*>(ws + L.l1s);
  uint16_t* U = reinterpret_cast<uint16_t*>(ws + L.u);
  float* part = reinterpret_cast<float*>(ws + L.part);
  const int64_t h = w->in, o_ = w->out;
  const int64_t mk = (M + 63) / 64;
  int* counters = reinterpret_cast<int*>(ws + L.counters);
  const uint16_t* T = T_saved;
  if (!T) {
    uint16_t* Tw = reinterpret_cast<uint16_t*>(ws + L.t);
    Thin tt{GemmKind::ThinKM, X, h, M, L1, r, h, M, h / 64, r};
    QLB_TRY(run_thin(tt, part, counters, Tw, 0, 1.f, status, s));
    T = Tw;
  }
  // U = dY L2^T (A = dY K-major, B = L2 [r x out] K-major; with the pair engine also
  // s.U, the dX LoRA step's A), dL1 = s X^T U and dL2 = s (dY^T T)^T (A = dY^T
  // MN-major, B = T MN-major, K = M, written transposed) are thin HBM-bound products;
  // dX is the tensor-core GEMM. dL2 uses its own partial buffer and counter range so
  // it can run beside the others. Two schedules:
  //  * the pair GEMM leaves SMs free (its pair count is the fewest that keeps its
  //    number of rounds of tiles, see pair_spare_sms): U, then dX on the side stream
  //    (highest priority) while dL1 and dL2 run on the caller's stream on the free
  //    SMs and, later, on the GEMM's idle SMs in its last round;
  //  * otherwise dL2 and the scale expansion run on the side stream beside U and dL1,
  //    and dX follows on the caller's stream.
  const bool pair = !w->is_bf16 && use_pair_kernel();
  uint16_t* sU = reinterpret_cast<uint16_t*>(ws + L.su);
  float* part2 = reinterpret_cast<float*>(ws + L.part2);
  std::lock_guard<std::mutex> lock(g_side_mu);
  SideStream* ss = ((M + 127) / 128 <= kMaxCounterTiles / 2 && (o_ + 127) / 128 <= kMaxCounterTiles / 2)
                       ? side_stream() : nullptr;
  const int forced = bwd_schedule_override();
  const int spare = !pair ? 0
                    : gemm_engine() == 2 ? pair2_spare_sms(true, int((M + 511) / 512) * int(h / 256),
                                                           int(o_ / 64) + (r + 63) / 64)
                                         : pair_spare_sms(true, int((M + 255) / 256) * int(h / 256));
  const bool beside_gemm = ss && dX && pair && forced != 2 && (forced == 1 || spare >= 16);
  // With every pair busy in the dX GEMM, U = dY L2^T (and s.U) is computed inside it
  // (its U tiles, before the output tiles' LoRA steps read s.U), and dL1 and dL2 follow
  // side by side on the two streams.
  const bool fuse_u = !beside_gemm && ss && dX && pair && forced == 0 && gemm_engine() == 2 && fused_u_wanted(h) &&
                      (M + 511) / 512 <= kPair2MaxTBlocks;
  float* gpart = reinterpret_cast<float*>(ws + L.gpart);
  int* gcount = reinterpret_cast<int*>(ws + kStatusBytes + kCounterBytes);
  cudaStream_t aux = s;
  int* counters2 = counters;
  if (ss) {
    aux = beside_gemm ? ss->hi : ss->stream;
    QLB_TRY(fork_to(ss, s, aux));
    counters2 = counters + kMaxCounterTiles / 2;
  }
  float* part_b = ss ? part2 : part;
  Thin tu{GemmKind::ThinKK, dY, o_, M, L2, o_, r, M, o_ / 64, r};
  Thin t1{GemmKind::ThinMM, X, h, M, U, r, M, h, mk, r};
  Thin t2{GemmKind::ThinMM, dY, o_, M, T, r, M, o_, mk, r};
  if (dX && !w->is_bf16)
    QLB_TRY(launch_expand_scales(w->codes, w->absmax, w->absmax_q, w->absmax2, w->q.double_quant != 0, o_, h,
                                 scales_t, aux));
  if (fuse_u) {
    QLB_TRY(join_from(ss, s, aux));    // the GEMM reads the expanded scales
    QLB_TRY(run_pair(true, w, dY, M, sU, L1, r, scales_t, dX, status, gpart, gcount, s, L2, U, sU, scale));
    QLB_TRY(handoff_to(ss, s, aux));   // dL2 (T, dY) beside dL1 (X, U), after the GEMM
    QLB_TRY(run_thin(t2, part_b, counters2, dL2, 2, scale, status, aux));
    QLB_TRY(run_thin(t1, part, counters, dL1, 1, scale, status, s));
    return join_from(ss, s, aux);
  }
  if (beside_gemm) {
    QLB_TRY(run_thin(tu, part, counters, U, 3, scale, status, s, sU));
    QLB_TRY(handoff_to(ss, s, aux));   // the GEMM needs s.U
    QLB_TRY(run_pair(true, w, dY, M, sU, L1, r, scales_t, dX, status, gpart, gcount, aux));
    QLB_TRY(run_thin(t1, part, counters, dL1, 1, scale, status, s));
    QLB_TRY(run_thin(t2, part_b, counters2, dL2, 2, scale, status, s));
    return join_from(ss, s, aux);
  }
  QLB_TRY(run_thin(t2, part_b, counters2, dL2, 2, scale, status, aux));
  if (pair && dX) QLB_TRY(run_thin(tu, part, counters, U, 3, scale, status, s, sU));
  else QLB_TRY(run_thin(tu, part, counters, U, 0, 1.f, status, s));
  QLB_TRY(run_thin(t1, part, counters, dL1, 1, scale, status, s));
  if (ss) QLB_TRY(join_from(ss, s));
  if (dX && pair) return run_pair(true, w, dY, M, sU, L1, r, scales_t, dX, status, gpart, gcount, s);
  if (dX) {
    QLB_TRY(launch_scale_lora(L1, h, r, scale, /*transpose=*/false, l1s, s));
    QLB_TRY(run_main(true, w, dY, M, U, l1s, r, scales_t, dX, status, s));
  }
  return QLORA_OK;
}

size_t nf4_layer_error_rank_workspace_size(int32_t n_layers, const int64_t* numel) {
  if (n_layers <= 0 || !numel) return 0;
  return layer_error_ws_bytes(n_layers, numel);
}

qlora_status nf4_layer_error_rank(int32_t n_layers, const uint16_t* const* W_ptrs, const int64_t* numel,
                                  int32_t w_dtype, nf4_qconfig q, int32_t K, double* err, int32_t* order,
                                  uint8_t* keep, void* workspace, size_t workspace_bytes, qlora_stream_t stream) {
  if (w_dtype != QLORA_DTYPE_BF16) return QLORA_ERR_DTYPE;
  if (!qconfig_ok(q)) return QLORA_ERR_UNSUPPORTED;
  if (n_layers < 1 || n_layers > 1024 || K < 0 || K > n_layers) return QLORA_ERR_SHAPE;
  if (!W_ptrs || !numel || !err || !order || !keep) return QLORA_ERR_NULL;
  for (int i = 0; i < n_layers; ++i) {
    if (!W_ptrs[i]) return QLORA_ERR_NULL;
    if (numel[i] <= 0 || numel[i] % 64 || numel[i] > kMaxCodecNumel) return QLORA_ERR_SHAPE;
    if (!aligned16(W_ptrs[i])) return QLORA_ERR_ALIGN;
  }
  if (noalloc_chunks(n_layers, numel) > int64_t(INT32_MAX)) return QLORA_ERR_SHAPE;   // chunk ids are 32-bit
  if (!workspace || !aligned16(workspace)) return QLORA_ERR_WORKSPACE;
  QLB_TRY(check_device());
  return launch_layer_error_rank(n_layers, W_ptrs, numel, q.double_quant != 0, K, err, order, keep, workspace,
                                 workspace_bytes, static_cast<int*>(workspace), S(stream));
}

qlora_status nf4_layer_error_rank_budget(int32_t n_layers, const uint16_t* const* W_ptrs, const int64_t* numel,
                                         int32_t w_dtype, nf4_qconfig q, int64_t budget_bytes, double* err,
                                         int32_t* order, uint8_t* keep, int32_t* K_out, void* workspace,
                                         size_t workspace_bytes, qlora_stream_t stream) {
  if (w_dtype != QLORA_DTYPE_BF16) return QLORA_ERR_DTYPE;
  if (!qconfig_ok(q)) return QLORA_ERR_UNSUPPORTED;
  if (n_layers < 1 || n_layers > 1024 || budget_bytes < 0) return QLORA_ERR_SHAPE;
  if (!W_ptrs || !numel || !err || !order || !keep || !K_out) return QLORA_ERR_NULL;
  for (int i = 0; i < n_layers; ++i) {
    if (!W_ptrs[i]) return QLORA_ERR_NULL;
    if (numel[i] <= 0 || numel[i] % 64 || numel[i] > (int64_t(1) << 40)) return QLORA_ERR_SHAPE;
    if (!aligned16(W_ptrs[i])) return QLORA_ERR_ALIGN;
  }
  if (noalloc_chunks(n_layers, numel) > int64_t(INT32_MAX)) return QLORA_ERR_SHAPE;   // chunk ids are 32-bit
  if (!workspace || !aligned16(workspace)) return QLORA_ERR_WORKSPACE;
  QLB_TRY(check_device());
  return launch_layer_error_rank(n_layers, W_ptrs, numel, q.double_quant != 0, 0, err, order, keep, workspace,
                                 workspace_bytes, static_cast<int*>(workspace), S(stream), budget_bytes, K_out);
}

qlora_status nf4_rank_errors(int32_t n_layers, const double* err, int32_t K, int32_t* order, uint8_t* keep,
                            qlora_stream_t stream) {
  if (n_layers < 1 || n_layers > 1024 || K < 0 || K > n_layers) return QLORA_ERR_SHAPE;
  if (!err || !order || !keep) return QLORA_ERR_NULL;
  QLB_TRY(check_device());
  return launch_rank_errors(n_layers, err, K, order, keep, S(stream));
}

qlora_status nf4_k_from_fraction(int64_t num, int64_t den, int32_t n_layers, int32_t* K) {
  if (!K) return QLORA_ERR_NULL;
  if (den <= 0 || num < 0 || num > den || den > (int64_t(1) << 31) || n_layers < 0 || n_layers > (1 << 30))
    return QLORA_ERR_SHAPE;
  *K = int32_t((2 * num * n_layers + den) / (2 * den));   // floor(num L / den + 1/2)
  return QLORA_OK;
}

qlora_status nf4_quantize_error_rank(int32_t n_layers, const uint16_t* const* W_ptrs, const int64_t* numel,
                                    int32_t w_dtype, nf4_qconfig q, int32_t K, uint8_t* const* codes,
                                    float* const* absmax, uint8_t* const* absmax_q, float* const* absmax2,
                                    double* err, int32_t* order, uint8_t* keep, void* workspace,
                                    size_t workspace_bytes, qlora_stream_t stream) {
  if (w_dtype != QLORA_DTYPE_BF16) return QLORA_ERR_DTYPE;
  if (!qconfig_ok(q)) return QLORA_ERR_UNSUPPORTED;
  if (n_layers < 1 || n_layers > 512 || K < 0 || K > n_layers) return QLORA_ERR_SHAPE;
  if (!W_ptrs || !numel || !err || !order || !keep || !codes) return QLORA_ERR_NULL;
  const bool dq = q.double_quant != 0;
  if (dq && (!absmax_q || !absmax2)) return QLORA_ERR_NULL;
  if (!dq && !absmax) return QLORA_ERR_NULL;
  for (int i = 0; i < n_layers; ++i) {
    if (!W_ptrs[i] || !codes[i]) return QLORA_ERR_NULL;
    if (dq && (!absmax_q[i] || !absmax2[i])) return QLORA_ERR_NULL;
    if (!dq && !absmax[i]) return QLORA_ERR_NULL;
    if (numel[i] <= 0 || numel[i] % 64 || numel[i] > kMaxCodecNumel) return QLORA_ERR_SHAPE;
    if (!aligned16(W_ptrs[i]) || !aligned16(codes[i])) return QLORA_ERR_ALIGN;
  }
  if (noalloc_chunks(n_layers, numel) > int64_t(INT32_MAX)) return QLORA_ERR_SHAPE;   // chunk ids are 32-bit
  if (!workspace || !aligned16(workspace)) return QLORA_ERR_WORKSPACE;
  QLB_TRY(check_device());
  return launch_quantize_error_rank(n_layers, W_ptrs, numel, dq, K, codes, absmax, absmax_q, absmax2, err, order,
                                    keep, workspace, workspace_bytes, static_cast<int*>(workspace), S(stream));
}

qlora_status nf4_layer_error_rank_noalloc(int32_t n_layers, const uint16_t* const* W_ptrs, const int64_t* numel,
                                          int32_t w_dtype, nf4_qconfig q, int32_t K, double* err, int32_t* order,
                                          uint8_t* keep, qlora_stream_t stream) {
  if (w_dtype != QLORA_DTYPE_BF16) return QLORA_ERR_DTYPE;
  if (!qconfig_ok(q)) return QLORA_ERR_UNSUPPORTED;
  if (n_layers < 1 || n_layers > 1024 || K < 0 || K > n_layers) return QLORA_ERR_SHAPE;
  if (!W_ptrs || !numel || !err || !order || !keep) return QLORA_ERR_NULL;
  for (int i = 0; i < n_layers; ++i) {
    if (!W_ptrs[i]) return QLORA_ERR_NULL;
    if (numel[i] <= 0 || numel[i] % 64 || numel[i] > kMaxCodecNumel) return QLORA_ERR_SHAPE;
    if (!aligned16(W_ptrs[i])) return QLORA_ERR_ALIGN;
  }
  if (noalloc_chunks(n_layers, numel) > (int64_t(1) << 20)) return QLORA_ERR_SHAPE;
  QLB_TRY(check_device());
  return launch_layer_error_rank_noalloc(n_layers, W_ptrs, numel, q.double_quant != 0, K, err, order, keep,
                                         S(stream));
}

}  // extern "C"
