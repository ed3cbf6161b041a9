// C ABI of the static FP8 W8A8 Linear-block library (declared in fp8ws.h).
//
// One translation unit: the kernels are included here so that the device
// status word has a single definition without relocatable device code.
// Host code validates every argument before enqueueing anything, builds the
// TMA tensor maps of each GEMM on the host (they travel as kernel
// parameters, so the calls stay free of device allocations and host syncs),
// picks the GEMM tile width from the problem shape and records every launch
// in a small ring for tests and benchmarks.
#include "../../include/fp8ws.h"

#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "elementwise.cuh"
#include "gemm_dual_sm100.cuh"
#include "gemm_pair_sm100.cuh"
#include "gemm_sm100.cuh"

namespace fp8ws {
namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kWaitLimitNs = 4ull * 1000 * 1000 * 1000;  // bounded mbarrier waits

// ---------------------------------------------------------------- launch log
std::mutex g_log_mu;
fp8ws_launch_record g_log[FP8WS_LOG_CAPACITY];
int64_t g_log_head = 0;  // records written since the last clear
int64_t g_launch_total = 0;

// One record per problem of a launch (member 0, 1, ... of a grouped launch);
// the launch itself is counted once, with member 0.
void log_launch(int kind, const void *in0, const void *in1, const void *out, int member = 0) {
  std::lock_guard<std::mutex> lk(g_log_mu);
  fp8ws_launch_record &r = g_log[g_log_head % FP8WS_LOG_CAPACITY];
  r.kind = kind;
  r.member = member;
  r.in0 = in0;
  r.in1 = in1;
  r.out = out;
  ++g_log_head;
  if (member == 0) ++g_launch_total;
}

enum { kKindQuant = 1, kKindGemm = 2, kKindSwiglu = 3, kKindCalib = 4, kKindDual = 5 };

// --------------------------------------------------------------- device info
// Per-device state, written once under g_dev_mu and read without it: the
// flags are atomics released after the values they publish.
struct DeviceInfo {
  std::atomic<int> checked{0};  // 0 unknown, 1 sm_100, -1 other
  int sms = 0;                  // set before `checked` is released
  int64_t l2_bytes = 0;         // likewise
  // bit per kernel whose attributes were set on this device: 0-2 one-CTA GEMMs,
  // 3/5/6/7 pair GEMM scale modes (+16 direct-store), 9 five-stage pair GEMM,
  // 4 dual (+8 variant, +16 direct variant, +24 direct plain), 8 per-token SwiGLU,
  // 10 staged quantizer
  std::atomic<unsigned> gemm_attr_set{0};
  std::atomic<int> pair_clusters{0};  // CTA pairs of the pair GEMM resident at once
  std::atomic<int> dual_clusters{0};  // CTA pairs of the gate/up dual GEMM resident at once
  // (the same for every epilogue variant: one CTA per SM either way)
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// First-use set-up of kernel `bit` on this device, once across threads:
// `setup` runs under g_dev_mu, and the bit is published after it succeeded.
template <typename F>
int once_per_device(DeviceInfo *d, int bit, F setup) {
  if (d->gemm_attr_set.load(std::memory_order_acquire) & (1u << bit)) return 0;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (d->gemm_attr_set.load(std::memory_order_relaxed) & (1u << bit)) return 0;
  const int rc = setup();
  if (rc == 0) d->gemm_attr_set.fetch_or(1u << bit, std::memory_order_release);
  return rc;
}

int current_device(int *dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return FP8WS_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return FP8WS_ERR_UNSUPPORTED;
  return FP8WS_OK;
}

int device_info(DeviceInfo **out) {
  int dev;
  int st = current_device(&dev);
  if (st) return st;
  DeviceInfo &d = g_dev[dev];
  if (d.checked.load(std::memory_order_acquire) == 0) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (d.checked.load(std::memory_order_relaxed) == 0) {
      int major = 0, minor = 0, sms = 0, l2 = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess)
        return FP8WS_ERR_CUDA;
      d.sms = sms;
      d.l2_bytes = l2;
      d.checked.store((major == 10 && minor == 0) ? 1 : -1, std::memory_order_release);
    }
  }
  if (d.checked.load(std::memory_order_acquire) != 1) return FP8WS_ERR_UNSUPPORTED;
  *out = &d;
  return FP8WS_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// The wide form of the streaming kernels loads 32 bytes at a time.
bool aligned32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// Which form of the two-input SwiGLU kernels runs on numel elements, G and U
// 32-byte aligned.  Timed on B200 with L2 flushed before each launch: the wide
// form is faster on short launches (up to 2^24 elements: fewer memory
// instructions, a shorter ramp; 12-14% at 8M-12M elements) and when the FP8
// output is larger than L2, so that write-backs stream during the kernel (6-8%
// at 134M-235M elements).  In between the output stays in L2, the launch is
// read-bound, and the 16-byte loads stream the reads 5-9% faster.  (The
// quantizer, with half the bytes read per element and no transcendental math,
// was as fast or faster in the wide form at every length from 3M to 201M
// elements, and takes it whenever its input is aligned.)
constexpr int64_t kWideShortElems = int64_t{1} << 24;
bool swiglu_wide_form(const DeviceInfo *d, int64_t numel) {
  return numel <= kWideShortElems || numel >= d->l2_bytes;
}

int launch_status() {
  return cudaGetLastError() == cudaSuccess ? FP8WS_OK : FP8WS_ERR_CUDA;
}

cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// Grid of a streaming kernel: enough blocks for every vector to be visited
// once by an unrolled iteration, capped at what all SMs hold at once (the
// kernels loop over the rest with a grid stride).
// The kernel is a template argument, so each kernel has its own count.
template <auto Kern>
int ew_grid(const DeviceInfo *d, int64_t nvec) {
  // blocks per SM, the same on every B200; found once per kernel (thread-safe
  // initialisation of a function-local static)
  static const int resident = [] {
    int r = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&r, Kern, kEwThreads, 0) != cudaSuccess ||
        r < 1)
      r = 1;
    return r;
  }();
  int64_t per_block = static_cast<int64_t>(kEwThreads) * kEwUnroll;
  int64_t want = (nvec + per_block - 1) / per_block;
  int64_t cap = static_cast<int64_t>(d->sms) * resident;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  return static_cast<int>(want);
}

// Kernels are launched with programmatic stream serialization: the next
// kernel on the stream may be scheduled while this one finishes, and waits in
// griddepcontrol.wait before touching memory.  FP8WS_PDL=0 turns it off.
bool use_pdl() {
  static const bool v = [] {
    const char *e = getenv("FP8WS_PDL");
    return !(e && e[0] == '0');
  }();
  return v;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      int cluster_x, Args... args) {
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (use_pdl()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// A streaming kernel in its wide form (BF16 inputs 32-byte aligned) or its
// 16-byte form, on a grid sized by ew_grid for nvec 8-element vectors.
template <auto KWide, auto KNarrow, typename... Args>
cudaError_t ew_launch(const DeviceInfo *d, bool wide, int64_t nvec, cudaStream_t st,
                      Args... args) {
  if (wide)
    return launch_ex(KWide, dim3(ew_grid<KWide>(d, nvec)), dim3(kEwThreads), 0, st, 1, args...);
  return launch_ex(KNarrow, dim3(ew_grid<KNarrow>(d, nvec)), dim3(kEwThreads), 0, st, 1, args...);
}

// ------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major [rows, cols] matrix, swizzled boxes of box_cols x box_rows (the
// box's rows are 128 bytes for the 128-byte swizzle, 64 for the 64-byte one).
int make_map_2d(CUtensorMap *map, CUtensorMapDataType dt, int elem_bytes, const void *base,
                int64_t rows, int64_t cols, int box_cols, int box_rows, bool for_load,
                CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return FP8WS_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * elem_bytes};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  for_load ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8WS_OK : FP8WS_ERR_CUDA;
}

// ------------------------------------------------------------------- GEMM
template <int BN, int STAGES, int BIT>
int launch_gemm_cfg(DeviceInfo *d, const uint8_t *xq, const uint8_t *wq, int M, int N, int K,
                    const float *s_in, const float *s_w, uint16_t *y, cudaStream_t st) {
  using C = GemmCfg<BN, STAGES>;
  auto kern = fp8_gemm_kernel<BN, STAGES>;
  int rc0 = once_per_device(d, BIT, [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::SMEM_BYTES) == cudaSuccess
               ? FP8WS_OK
               : FP8WS_ERR_CUDA;
  });
  if (rc0) return rc0;
  CUtensorMap ma, mb, md;
  int rc = make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, xq, M, K, kGemmBK, kGemmBM, true);
  if (!rc) rc = make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, wq, N, K, kGemmBK, BN, true);
  if (!rc)
    rc = make_map_2d(&md, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, M, N, C::EPI_COLS, 32, false);
  if (rc) return rc;
  const int tiles = ((M + kGemmBM - 1) / kGemmBM) * ((N + BN - 1) / BN);
  const int grid = tiles < d->sms ? tiles : d->sms;
  if (launch_ex(kern, dim3(grid), dim3(kGemmThreads), C::SMEM_BYTES, st, 1, ma, mb, md, s_in, s_w,
                M, N, K, kWaitLimitNs) != cudaSuccess)
    return FP8WS_ERR_CUDA;
  log_launch(kKindGemm, xq, wq, y);
  return launch_status();
}

// With M == 0 there is nothing to read or write, so xq and y may be NULL
// (an empty tensor's data pointer).
// CTA-pair GEMM: one cluster of two CTAs per TPC, persistent over 256 x 256
// tiles.  The grid holds as many pairs as can be resident at once.
// Split-K scratch of the CTA-pair GEMM, laid out independently of the device:
// kSplitkSlots slots of 2 x 128 x 256 fp32 (one per split unit) followed by
// one counter per (remainder tile, CTA, epilogue warp) for up to
// kSplitkTiles remainder tiles.  Plans never need more.
constexpr int kSplitkSlots = 148;
constexpr int kSplitkTiles = 128;
constexpr int kSplitkCounterWords = kSplitkTiles * 2 * 4;
size_t splitk_slot_bytes() { return static_cast<size_t>(2) * 128 * kPairTile * sizeof(float); }
int splitk_max_slots(int pairs) { return 2 * pairs < kSplitkSlots ? 2 * pairs : kSplitkSlots; }
size_t splitk_bytes() {
  return kSplitkSlots * splitk_slot_bytes() + ((kSplitkCounterWords * sizeof(int) + 255) & ~255ul);
}
int *splitk_counters(void *splitk) {
  return reinterpret_cast<int *>(static_cast<uint8_t *>(splitk) + kSplitkSlots * splitk_slot_bytes());
}

// Remainder tiles (those past the last full wave) split over S K ranges, S in
// 1..4 minimising waves-of-units x (1/S) of a tile's time, with at most two
// waves of units and at least two K steps per range.  No scratch: no split.
// A split pays only when it takes enough K steps off the critical path to cover
// its fixed cost (the fp32 partial stores, the wait for the last split, its
// reduction).  Timed on B200: splitting the ragged wave 4 ways saved 9 us at
// K = 12288 (96 K steps per tile) and cost 6 us at K = 3072 (24 K steps).
// Otherwise, when the remainder would fill at most half a wave, each of its
// tiles runs as two 256 x 128 halves instead (no scratch needed): the last
// wave then takes a half tile's time, not a whole one's.
constexpr int kSplitkMinKb = 64;

// FP8WS_TAIL_HALVES=0 keeps ragged last waves whole (timing comparisons).
bool tail_halves_enabled() {
  static const bool v = [] {
    const char *e = getenv("FP8WS_TAIL_HALVES");
    return !(e && e[0] == '0');
  }();
  return v;
}

SplitPlan make_split_plan(int tiles, int pairs, int num_kb, float *partials, int *counters,
                          bool halves_allowed = true) {
  SplitPlan p{tiles, 0, 1, num_kb, nullptr, nullptr, 1};
  if (pairs < 1 || tiles % pairs == 0) return p;
  const int R = tiles % pairs;
  const bool k_split_possible = partials && num_kb >= kSplitkMinKb && R <= kSplitkTiles;
  if (!k_split_possible) {
    if (halves_allowed && 2 * R <= pairs) {
      p.dp_tiles = tiles - R;
      p.split_tiles = R;
      p.halves = 2;
    }
    return p;
  }
  int best_s = 1;
  double best = 1.0;
  for (int S = 2; S <= 4; ++S) {
    const int kbs = (num_kb + S - 1) / S;
    if (kbs < 2 || (S - 1) * kbs >= num_kb || R * S > splitk_max_slots(pairs)) continue;
    const double t = static_cast<double>((R * S + pairs - 1) / pairs) / S;
    if (t < best - 1e-9) {
      best = t;
      best_s = S;
    }
  }
  if (best_s == 1) return p;
  p.dp_tiles = tiles - R;
  p.split_tiles = R;
  p.splits = best_s;
  p.kb_per_split = (num_kb + best_s - 1) / best_s;
  p.partials = partials;
  p.counters = counters;
  return p;
}

// One problem of a grouped CTA-pair launch: Y[M,N] from A[M,K] and B[N,K].
// b2 and s_w2 (the up weight) and s_down are read by the dual gate/up kernel
// only; out is Y (BF16) for the GEMM and H (FP8) for the dual kernel.  Every
// problem has M >= 1.
struct PairProblem {
  const uint8_t *a;
  const uint8_t *b;
  const uint8_t *b2;
  void *out;
  int M;
  int N;
  const float *s_in;
  const float *s_w;
  const float *s_w2;
  const float *s_down;
};

// The grouped gated MLP's overlap of the next call's input prefetch with its
// down GEMM's tail (late dependent launch + L2 prefetch); FP8WS_LATE_TRIGGER=0
// turns it off.
bool late_trigger_enabled() {
  static const bool v = [] {
    const char *e = getenv("FP8WS_LATE_TRIGGER");
    return !(e && e[0] == '0');
  }();
  return v;
}

// L2 prefetch of the quantizers' inputs before they wait for the kernel
// before them; FP8WS_PREFETCH=0 turns it off (timing comparisons).
bool prefetch_enabled() {
  static const bool v = [] {
    const char *e = getenv("FP8WS_PREFETCH");
    return !(e && e[0] == '0');
  }();
  return v;
}

// L2 eviction hints on the GEMM operand loads; FP8WS_L2_HINTS=0 turns them off
// (every load then takes the normal policy).
bool use_l2_hints() {
  static const bool v = [] {
    const char *e = getenv("FP8WS_L2_HINTS");
    return !(e && e[0] == '0');
  }();
  return v;
}

// Kernel-side description of a group whose tiles are tile_m x tile_n.
PairGroup make_pair_group(const PairProblem *pp, int np, int tile_m, int tile_n) {
  PairGroup G = {};
  G.n = np;
  int total = 0;
  for (int p = 0; p < kMaxGroup; ++p) {
    const PairProblem &q = pp[p < np ? p : 0];
    G.M[p] = q.M;
    G.N[p] = q.N;
    G.num_m[p] = (q.M + tile_m - 1) / tile_m;
    G.num_n[p] = (q.N + tile_n - 1) / tile_n;
    // Tile order.  When A (M x K) is larger than B (N x K; both weights for
    // the gate/up kernel), the tiles run row by row: a wave sweeps every
    // column of a few row blocks, so each A row block leaves DRAM once and B,
    // the smaller operand, is re-read from L2.  Otherwise they run column by
    // column within groups of kGroupM row blocks: each B column block is read
    // once per group and A is re-read from L2.
    G.group_m[p] = q.M > static_cast<int64_t>(q.N) * (q.b2 ? 2 : 1) ? 1 : kGroupM;
    // Row by row, each A row block is consumed within a wave and B is read
    // again by every wave; column by column within row groups, the other way
    // round.  The operand consumed within a wave is loaded evict-first.
    G.hint[p] = !use_l2_hints() ? kHintNone : (G.group_m[p] == 1 ? kHintAFirst : kHintBFirst);
    G.s_in[p] = q.s_in;
    G.s_w[p] = q.s_w;
    G.s_w2[p] = q.s_w2;
    G.s_down[p] = q.s_down;
    G.out[p] = q.out;
    G.tile_start[p] = p < np ? total : INT_MAX;
    if (p < np) total += G.num_m[p] * G.num_n[p];
  }
  G.tiles = total;
  return G;
}

// Grid of a CTA-pair kernel: as many clusters of two as can be resident at
// once, found by the occupancy query on the first launch of each variant.
template <typename Kernel>
int pair_clusters(DeviceInfo *d, Kernel kern, int threads, int smem, int bit,
                  std::atomic<int> *clusters_out) {
  return once_per_device(d, bit, [&] {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return FP8WS_ERR_CUDA;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (d->sms / 2));
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1)
      return FP8WS_ERR_CUDA;
    clusters_out->store(clusters, std::memory_order_relaxed);
    return FP8WS_OK;
  });
}

template <int STAGES, int BIT, int SCALE_MODE = 0, bool DIRECT = false>
int launch_gemm_pair_cfg(DeviceInfo *d, const PairProblem *pp, int np, int K, cudaStream_t st,
                         void *splitk = nullptr, bool late_trigger = false) {
  using C = PairCfg<STAGES, DIRECT>;
  auto kern = fp8_gemm_pair_kernel<STAGES, SCALE_MODE, DIRECT>;
  int rc = pair_clusters(d, kern, kGemmThreads, C::SMEM_BYTES, BIT, &d->pair_clusters);
  if (rc) return rc;
  // B is mapped twice: 128-row boxes for whole tiles, 64-row boxes for the
  // 256 x 128 halves of a ragged last wave
  CUtensorMap ma[kMaxGroup], mb[kMaxGroup], mbh[kMaxGroup], md[kMaxGroup];
  for (int p = 0; p < np && !rc; ++p) {
    const PairProblem &q = pp[p];
    rc = make_map_2d(&ma[p], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q.a, q.M, K, kGemmBK, 128, true);
    if (!rc)
      rc = make_map_2d(&mb[p], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q.b, q.N, K, kGemmBK, 128, true);
    if (!rc)
      rc = make_map_2d(&mbh[p], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q.b, q.N, K, kGemmBK, 64, true);
    if (!rc)
      rc = make_map_2d(&md[p], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q.out, q.M, q.N, C::EPI_COLS,
                       32, false);
  }
  if (rc) return rc;
  for (int p = np; p < kMaxGroup; ++p) {  // absent problems: copies, never used
    ma[p] = ma[0];
    mb[p] = mb[0];
    mbh[p] = mbh[0];
    md[p] = md[0];
  }
  const PairGroup G = make_pair_group(pp, np, kPairTile, kPairTile);
  const int tiles = G.tiles;
  float *partials = static_cast<float *>(splitk);
  int *counters = splitk ? splitk_counters(splitk) : nullptr;
  SplitPlan plan = make_split_plan(tiles, d->pair_clusters.load(std::memory_order_relaxed),
                                   (K + kGemmBK - 1) / kGemmBK, partials, counters,
                                   tail_halves_enabled());
  plan.late_trigger = late_trigger ? 1 : 0;
  const int units = plan.dp_tiles + plan.split_tiles * plan.splits * plan.halves;
  const int resident = d->pair_clusters.load(std::memory_order_relaxed);
  const int clusters = units < resident ? units : resident;
  if (launch_ex(kern, dim3(2 * clusters), dim3(kGemmThreads), C::SMEM_BYTES, st, 2, ma[0], ma[1],
                ma[2], mb[0], mb[1], mb[2], mbh[0], mbh[1], mbh[2], md[0], md[1], md[2], G, K,
                kWaitLimitNs, plan) != cudaSuccess)
    return FP8WS_ERR_CUDA;
  for (int p = 0; p < np; ++p) log_launch(kKindGemm, pp[p].a, pp[p].b, pp[p].out, p);
  return launch_status();
}

// Epilogue of the CTA-pair kernels: TMA stores from shared-memory tiles with
// six pipeline stages (default), or 16-byte global stores from registers with
// seven stages (FP8WS_EPILOGUE=direct).
bool direct_epilogue() {
  static const bool v = [] {
    const char *e = getenv("FP8WS_EPILOGUE");
    return e && e[0] == 'd';
  }();
  return v;
}

// FP8WS_PAIR_STAGES=5: the CTA-pair GEMM with a five-stage ring instead of six
// (per-tensor scales only), to see how the K step depends on the ring depth.
bool five_stages() {
  static const bool v = [] {
    const char *e = getenv("FP8WS_PAIR_STAGES");
    return e && e[0] == '5';
  }();
  return v;
}

template <int BIT, int SCALE_MODE = 0>
int launch_gemm_pair(DeviceInfo *d, const PairProblem *pp, int np, int K, cudaStream_t st,
                     void *splitk = nullptr, bool late_trigger = false) {
  if (SCALE_MODE == 0 && five_stages())
    return launch_gemm_pair_cfg<5, 9, 0, false>(d, pp, np, K, st, splitk, late_trigger);
  if (direct_epilogue())
    return launch_gemm_pair_cfg<7, BIT + 16, SCALE_MODE, true>(d, pp, np, K, st, splitk,
                                                                late_trigger);
  return launch_gemm_pair_cfg<6, BIT, SCALE_MODE, false>(d, pp, np, K, st, splitk,
                                                         late_trigger);
}

template <int BIT, int SCALE_MODE = 0>
int launch_gemm_pair(DeviceInfo *d, const uint8_t *xq, const uint8_t *wq, int M, int N, int K,
                     const float *s_in, const float *s_w, uint16_t *y, cudaStream_t st,
                     void *splitk = nullptr) {
  const PairProblem p = {xq, wq, nullptr, y, M, N, s_in, s_w, nullptr, nullptr};
  return launch_gemm_pair<BIT, SCALE_MODE>(d, &p, 1, K, st, splitk);
}

// Gate/up dual GEMM with the SwiGLU-quant epilogue, on CTA pairs.
template <int STAGES, int BIT, bool DIRECT, bool VARIANT>
int launch_dual_swiglu_cfg(DeviceInfo *d, const PairProblem *pp, int np, int N, int K,
                           SwigluParams act, cudaStream_t st) {
  using C = DualCfg<STAGES, DIRECT>;
  auto kern = fp8_dual_swiglu_pair_kernel<STAGES, DIRECT, VARIANT>;
  int rc = pair_clusters(d, kern, kDualThreads, C::SMEM_BYTES, BIT, &d->dual_clusters);
  if (rc) return rc;
  CUtensorMap ma[kMaxDualGroup], mg[kMaxDualGroup], mu[kMaxDualGroup], mh[kMaxDualGroup];
  for (int p = 0; p < np && !rc; ++p) {
    const PairProblem &q = pp[p];
    rc = make_map_2d(&ma[p], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q.a, q.M, K, kGemmBK, 128, true);
    if (!rc) rc = make_map_2d(&mg[p], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q.b, N, K, kGemmBK, 128, true);
    if (!rc)
      rc = make_map_2d(&mu[p], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q.b2, N, K, kGemmBK, 128, true);
    if (!rc)
      rc = make_map_2d(&mh[p], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q.out, q.M, N, C::EPI_COLS, 32,
                       false, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  if (rc) return rc;
  if (np == 1) {
    ma[1] = ma[0];
    mg[1] = mg[0];
    mu[1] = mu[0];
    mh[1] = mh[0];
  }
  const PairGroup G = make_pair_group(pp, np, kDualTileM, kDualTileN);
  const int tiles = G.tiles;
  const int resident = d->dual_clusters.load(std::memory_order_relaxed);
  const int clusters = tiles < resident ? tiles : resident;
  if (launch_ex(kern, dim3(2 * clusters), dim3(kDualThreads), C::SMEM_BYTES, st, 2, ma[0], mg[0],
                mu[0], mh[0], ma[1], mg[1], mu[1], mh[1], G, act, N, K,
                kWaitLimitNs) != cudaSuccess)
    return FP8WS_ERR_CUDA;
  for (int p = 0; p < np; ++p) log_launch(kKindDual, pp[p].a, pp[p].b, pp[p].out, p);
  return launch_status();
}

int launch_dual_swiglu(DeviceInfo *d, const PairProblem *pp, int np, int N, int K,
                       SwigluParams act, cudaStream_t st) {
  constexpr int BIT = 4;
  // the plain activation (alpha 1, no offset, no clamp) takes the kernel
  // without the variant's per-element tests
  const bool variant = act.alpha != 1.0f || act.beta != 0.0f || act.has_limit;
  if (direct_epilogue()) {
    if (variant) return launch_dual_swiglu_cfg<7, BIT + 16, true, true>(d, pp, np, N, K, act, st);
    return launch_dual_swiglu_cfg<7, BIT + 24, true, false>(d, pp, np, N, K, act, st);
  }
  if (variant) return launch_dual_swiglu_cfg<6, BIT + 8, false, true>(d, pp, np, N, K, act, st);
  return launch_dual_swiglu_cfg<6, BIT, false, false>(d, pp, np, N, K, act, st);
}

int launch_dual_swiglu(DeviceInfo *d, const uint8_t *xq, const uint8_t *wg, const uint8_t *wu,
                       int M, int N, int K, const float *s_in, const float *s_wg,
                       const float *s_wu, const float *s_down, SwigluParams act, uint8_t *h,
                       cudaStream_t st) {
  const PairProblem p = {xq, wg, wu, h, M, N, s_in, s_wg, s_wu, s_down};
  return launch_dual_swiglu(d, &p, 1, N, K, act, st);
}

int check_gemm_args(const void *xq, const void *wq, int64_t M, int64_t N, int64_t K,
                    const float *s_in, const float *s_w, const void *y) {
  if (!wq || !s_in || !s_w || (M != 0 && (!xq || !y))) return FP8WS_ERR_NULL;
  if (M < 0 || N < 8 || K < 16 || (N % 8) != 0 || (K % 16) != 0) return FP8WS_ERR_SHAPE;
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return FP8WS_ERR_SHAPE;
  if (!aligned16(xq) || !aligned16(wq) || !aligned16(y)) return FP8WS_ERR_ALIGN;
  return FP8WS_OK;
}

// Tile shape from a cost model: time ~ waves x (output area per SM per tile)
// / efficiency, where waves = ceil(tiles / tiles resident at once).  The
// efficiencies are the measured throughput of each configuration on large
// problems relative to the CTA-pair kernel: narrower one-CTA tiles move more
// operand bytes per tensor cycle and become L2-bandwidth bound.
std::atomic<int> g_forced_gemm_config{0};  // fp8ws_set_gemm_config: 0 = cost model

// 1 = CTA pair 256 x 256, 2 = one CTA 128 x 256, 3 = 128 x 128, 4 = 128 x 64,
// for the np problems M[p] x N[p] that one launch would cover.
// The cost model alone: the configuration (1 CTA pairs, 2/3/4 one CTA with
// 128x256, 128x128, 128x64 tiles) for np problems on `sms` SMs holding `pairs`
// CTA pairs at once.
int gemm_cost_choice(int sms, int pairs, const int64_t *M, const int64_t *N, int np) {
  auto waves = [](int64_t tiles, int64_t slots) { return (tiles + slots - 1) / slots; };
  int64_t t_pair = 0, t_256 = 0, t_128 = 0, t_64 = 0;
  for (int p = 0; p < np; ++p) {
    const int64_t m128 = (M[p] + 127) / 128, m256 = (M[p] + 255) / 256;
    t_pair += m256 * ((N[p] + 255) / 256);
    t_256 += m128 * ((N[p] + 255) / 256);
    t_128 += m128 * ((N[p] + 127) / 128);
    t_64 += m128 * ((N[p] + 63) / 64);
  }
  // CTA pairs: the full waves, then a ragged remainder that fills at most half
  // a wave runs as 256 x 128 halves, taken at 0.7 of a whole tile's time (a
  // half tile moves 3/4 of a whole tile's operand bytes per K step)
  const int64_t rem = t_pair % pairs;
  const double pair_waves = static_cast<double>(t_pair / pairs) +
                            (rem == 0 ? 0.0 : (2 * rem <= pairs ? 0.7 : 1.0));
  const double est_pair = pair_waves * (128.0 * 256) / 1.0;
  const double est_256 = waves(t_256, sms) * (128.0 * 256) / 0.85;
  const double est_128 = waves(t_128, sms) * (128.0 * 128) / 0.45;
  const double est_64 = waves(t_64, sms) * (128.0 * 64) / 0.25;
  const double best = fmin(fmin(est_pair, est_256), fmin(est_128, est_64));
  if (est_pair == best) return 1;
  if (est_256 == best) return 2;
  if (est_128 == best) return 3;
  return 4;
}

int gemm_choice(const DeviceInfo *d, const int64_t *M, const int64_t *N, int np) {
  const int forced = g_forced_gemm_config.load(std::memory_order_relaxed);
  if (forced) return forced;
  const int resident = d->pair_clusters.load(std::memory_order_relaxed);
  return gemm_cost_choice(d->sms, resident > 0 ? resident : d->sms / 2, M, N, np);
}

int gemm_dispatch(DeviceInfo *d, const uint8_t *xq, const uint8_t *wq, int64_t M, int64_t N,
                  int64_t K, const float *s_in, const float *s_w, uint16_t *y, cudaStream_t st,
                  void *splitk = nullptr) {
  if (M == 0) return FP8WS_OK;
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  switch (gemm_choice(d, &M, &N, 1)) {
    case 1: return launch_gemm_pair<3>(d, xq, wq, m, n, k, s_in, s_w, y, st, splitk);
    case 2: return launch_gemm_cfg<256, 4, 0>(d, xq, wq, m, n, k, s_in, s_w, y, st);
    case 3: return launch_gemm_cfg<128, 6, 1>(d, xq, wq, m, n, k, s_in, s_w, y, st);
    default: return launch_gemm_cfg<64, 8, 2>(d, xq, wq, m, n, k, s_in, s_w, y, st);
  }
}

// A group of up to kMaxGroup GEMMs sharing K: one CTA-pair launch over all
// their tiles when the cost model picks CTA pairs for the group, else one
// launch each.  Problems with M == 0 are skipped.
int gemm_group_dispatch(DeviceInfo *d, const PairProblem *pp, int np, int K, cudaStream_t st,
                        void *splitk = nullptr, bool late_trigger = false) {
  PairProblem live[kMaxGroup];
  int64_t rows[kMaxGroup], cols[kMaxGroup];
  int n = 0;
  for (int p = 0; p < np; ++p)
    if (pp[p].M > 0) {
      live[n] = pp[p];
      rows[n] = pp[p].M;
      cols[n++] = pp[p].N;
    }
  if (n == 0) return FP8WS_OK;
  if (gemm_choice(d, rows, cols, n) == 1)
    return launch_gemm_pair<3>(d, live, n, K, st, splitk, late_trigger);
  int rc = FP8WS_OK;
  for (int p = 0; p < n && !rc; ++p)
    rc = gemm_dispatch(d, live[p].a, live[p].b, live[p].M, live[p].N, K, live[p].s_in,
                       live[p].s_w, static_cast<uint16_t *>(live[p].out), st, splitk);
  return rc;
}

// Any number of GEMMs sharing K, in grouped launches of up to kMaxGroup.
int gemm_groups(DeviceInfo *d, const PairProblem *pp, int np, int K, cudaStream_t st,
                void *splitk) {
  int rc = FP8WS_OK;
  for (int p = 0; p < np && !rc; p += kMaxGroup)
    rc = gemm_group_dispatch(d, pp + p, np - p < kMaxGroup ? np - p : kMaxGroup, K, st, splitk);
  return rc;
}

// ----------------------------------------------------------- elementwise
// The quantizer's form, set by fp8ws_set_quant_form: 0 chooses by size
// (default), 1 the staged kernel, 2 the streaming kernels; FP8WS_QUANT=staged
// or =stream sets the starting value (timing comparisons).  All give the same
// codes.  Timed on B200, back to back: the streaming kernels are faster up to
// an input about as large as L2 (9.4 against 11.6 us for 4096 + 1024 rows x
// 3072, 4.6 against 5.7 us for 2048 x 3072, 35.8 against 37.4 us for 8192 x
// 8192, 134 MB); from 1.5 times L2 up the staged kernel's steady stream of
// reads wins (56.2 against 64.7 us for 12288 x 8192, 78 against 90 us for
// 16384 x 8192).
std::atomic<int> g_quant_form{-1};
bool staged_quant(const DeviceInfo *d, int64_t numel) {
  int f = g_quant_form.load(std::memory_order_relaxed);
  if (f < 0) {
    const char *e = getenv("FP8WS_QUANT");
    int want = !e ? 0 : (strcmp(e, "staged") == 0 ? 1 : (strcmp(e, "stream") == 0 ? 2 : 0));
    // keep a form set meanwhile by fp8ws_set_quant_form
    if (!g_quant_form.compare_exchange_strong(f, want, std::memory_order_relaxed)) want = f;
    f = want;
  }
  if (f == 0) return numel * 4 >= d->l2_bytes * 3;  // BF16 input >= 1.5 x L2
  return f == 1;
}

// One or two runs (b.numel = 0 for one) through quant_staged_kernel: one CTA
// per SM, or one per chunk when there are fewer chunks than SMs.
int quant_staged_launch(DeviceInfo *d, const QuantSeg &a, const QuantSeg &b, cudaStream_t st,
                        int *zero_words, int n_zero) {
  int rc = once_per_device(d, 10, [] {
    return cudaFuncSetAttribute(quant_staged_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kStagedSmem) == cudaSuccess
               ? FP8WS_OK
               : FP8WS_ERR_CUDA;
  });
  if (rc) return rc;
  const int64_t chunks = staged_chunks(a.numel) + staged_chunks(b.numel);
  const int grid = chunks >= d->sms ? d->sms : (chunks > 0 ? static_cast<int>(chunks) : 1);
  if (launch_ex(quant_staged_kernel, dim3(grid), dim3(kStagedThreads), kStagedSmem, st, 1, a, b,
                zero_words, n_zero, prefetch_enabled() ? 1 : 0, kWaitLimitNs) != cudaSuccess)
    return FP8WS_ERR_CUDA;
  return FP8WS_OK;
}

int quant_launch(DeviceInfo *d, const uint16_t *x, int64_t numel, const float *s, uint8_t *xq,
                 cudaStream_t st, int *zero_words = nullptr, int n_zero = 0) {
  if (numel == 0) return FP8WS_OK;
  if (staged_quant(d, numel)) {
    const int rc = quant_staged_launch(d, QuantSeg{x, numel, s, xq},
                                       QuantSeg{nullptr, 0, nullptr, nullptr}, st, zero_words,
                                       n_zero);
    if (rc) return rc;
    log_launch(kKindQuant, x, nullptr, xq);
    return launch_status();
  }
  // The pair kernel with an empty second run (every block on x): its 46
  // registers allow five blocks per SM where a single-run kernel of its own
  // compiled to 57 (four), 4.4 against 4.6 us at 2048 x 3072.  Its first
  // blocks prefetch x into L2 while the previous kernel drains.
  const bool wide = aligned32(x);
  const int grid = wide ? ew_grid<quant_static_pair_kernel<true>>(d, numel >> 3)
                        : ew_grid<quant_static_pair_kernel<false>>(d, numel >> 3);
  const QuantSeg a{x, numel, s, xq}, none{nullptr, 0, nullptr, nullptr};
  if (launch_ex(wide ? quant_static_pair_kernel<true> : quant_static_pair_kernel<false>,
                dim3(grid), dim3(kEwThreads), 0, st, 1, a, none, grid, zero_words, n_zero,
                prefetch_enabled() ? d->sms : 0) != cudaSuccess)
    return FP8WS_ERR_CUDA;
  log_launch(kKindQuant, x, nullptr, xq);
  return launch_status();
}

// Two activations in one launch, the blocks shared in proportion to their
// sizes; a single non-empty one goes to quant_launch.
// The first d->sms blocks prefetch both inputs into L2 while the previous
// kernel drains (see quant_static_pair_kernel).
int quant_pair_launch(DeviceInfo *d, const QuantSeg *q, int nq, cudaStream_t st,
                      int *zero_words = nullptr, int n_zero = 0) {
  const int prefetch_blocks = prefetch_enabled() ? d->sms : 0;
  QuantSeg live[2];
  int n = 0;
  for (int i = 0; i < nq; ++i)
    if (q[i].numel > 0) live[n++] = q[i];
  if (n == 0) return FP8WS_OK;
  if (n == 1)
    return quant_launch(d, live[0].x, live[0].numel, live[0].s_in, live[0].xq, st, zero_words,
                        n_zero);
  if (staged_quant(d, live[0].numel + live[1].numel)) {
    const int rc = quant_staged_launch(d, live[0], live[1], st, zero_words, n_zero);
    if (rc) return rc;
    log_launch(kKindQuant, live[0].x, nullptr, live[0].xq, 0);
    log_launch(kKindQuant, live[1].x, nullptr, live[1].xq, 1);
    return launch_status();
  }
  const int64_t total = live[0].numel + live[1].numel;
  const bool wide = aligned32(live[0].x) && aligned32(live[1].x);
  int grid = wide ? ew_grid<quant_static_pair_kernel<true>>(d, total >> 3)
                  : ew_grid<quant_static_pair_kernel<false>>(d, total >> 3);
  if (grid < 2) grid = 2;
  int split = static_cast<int>((static_cast<double>(grid) * live[0].numel) / total + 0.5);
  split = split < 1 ? 1 : (split > grid - 1 ? grid - 1 : split);
  if (launch_ex(wide ? quant_static_pair_kernel<true> : quant_static_pair_kernel<false>,
                dim3(grid), dim3(kEwThreads), 0, st, 1, live[0], live[1], split, zero_words,
                n_zero, prefetch_blocks) != cudaSuccess)
    return FP8WS_ERR_CUDA;
  log_launch(kKindQuant, live[0].x, nullptr, live[0].xq, 0);
  log_launch(kKindQuant, live[1].x, nullptr, live[1].xq, 1);
  return launch_status();
}

int silu_launch(DeviceInfo *d, const uint16_t *g, const uint16_t *u, int64_t numel,
                const float *s, uint8_t *h, cudaStream_t st) {
  if (numel == 0) return FP8WS_OK;
  const bool wide = aligned32(g) && aligned32(u) && swiglu_wide_form(d, numel);
  if (ew_launch<silu_mul_2in_kernel<true>, silu_mul_2in_kernel<false>>(d, wide, numel >> 3, st, g,
                                                                        u, numel, s, h) !=
      cudaSuccess)
    return FP8WS_ERR_CUDA;
  log_launch(kKindSwiglu, g, u, h);
  return launch_status();
}

size_t round256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// Workspace byte counts are formed in 128 bits from sizes below 2^63 and
// saturate at SIZE_MAX, so that no shape wraps a count into a small number (a
// SIZE_MAX workspace cannot be allocated).  ws_region(a, b, c) is one region of
// a * b * c bytes (c: element size, at most 4) rounded up to 256.
using u128 = unsigned __int128;
// Factors are clamped at 2^40 (a region that large saturates anyway), so a
// sum of a few regions stays far below 2^128.
u128 ws_region(int64_t a, int64_t b, int c = 1) {
  const int64_t cap = int64_t(1) << 40;
  const u128 x = static_cast<u128>(a < cap ? a : cap) * static_cast<u128>(b < cap ? b : cap) *
                 static_cast<u128>(c);
  return (x + 255) & ~static_cast<u128>(255);
}
size_t ws_saturate(u128 v) { return v > SIZE_MAX ? SIZE_MAX : static_cast<size_t>(v); }

// Self-test of the bounded wait (fp8ws_selftest_bounded_wait): lane 0 of warp 0
// waits on an mbarrier that nothing arrives at.  Mode 0: the wait runs out
// after limit_ns and records kSiteSelfTest in the status word.  Mode 1: warp 1
// raises the abort flag after a quarter of the limit and the wait returns
// then, recording nothing.  Either way the kernel returns; the time the wait
// took goes to g_selftest_elapsed_ns.
__device__ long long g_selftest_elapsed_ns = 0;

__global__ void selftest_wait_kernel(uint64_t limit_ns, int mode) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = global_timer_ns();
    const bool ok = mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns);
    const uint64_t t1 = global_timer_ns();
    if (!ok && mode == 0) record_timeout(kSiteSelfTest);
    g_selftest_elapsed_ns = static_cast<long long>(t1 - t0);
    mbar_arrive(&bar);  // complete the phase before the block exits
  } else if (threadIdx.x == 32 && mode == 1) {
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < limit_ns / 4) {
    }
    abort_flag = 1;
  }
}

// NULL = plain SwiGLU (alpha 1, no offset, no clamp).
int swiglu_params(const fp8ws_swiglu *act, SwigluParams *p) {
  p->alpha = 1.0f;
  p->beta = 0.0f;
  p->limit = 0.0f;
  p->has_limit = 0;
  if (!act) return FP8WS_OK;
  if (!isfinite(act->alpha) || !isfinite(act->beta)) return FP8WS_ERR_BAD_SCALE;
  if (act->has_limit && !(act->limit > 0.0f)) return FP8WS_ERR_BAD_SCALE;
  p->alpha = act->alpha;
  p->beta = act->beta;
  p->limit = act->limit;
  p->has_limit = act->has_limit ? 1 : 0;
  return FP8WS_OK;
}

}  // namespace
}  // namespace fp8ws

using namespace fp8ws;

extern "C" {

int fp8_quant_static(const uint16_t *x, int64_t numel, const float *s_in, uint8_t *xq,
                     void *stream) {
  if (numel < 0) return FP8WS_ERR_SHAPE;
  if (numel == 0) return FP8WS_OK;  // empty tensors may carry NULL pointers
  if (!x || !s_in || !xq) return FP8WS_ERR_NULL;
  if (!aligned16(x) || !aligned16(xq)) return FP8WS_ERR_ALIGN;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  return quant_launch(d, x, numel, s_in, xq, as_stream(stream));
}

int fp8_linear_static(const uint8_t *xq, const uint8_t *wq, int64_t M, int64_t N, int64_t K,
                      const float *s_in, const float *s_w, uint16_t *y, void *stream) {
  int rc = check_gemm_args(xq, wq, M, N, K, s_in, s_w, y);
  if (rc) return rc;
  DeviceInfo *d;
  rc = device_info(&d);
  if (rc) return rc;
  return gemm_dispatch(d, xq, wq, M, N, K, s_in, s_w, y, as_stream(stream));
}

int silu_mul_2in_fp8(const uint16_t *g, const uint16_t *u, int64_t numel, const float *s_down,
                     uint8_t *h, void *stream) {
  if (numel < 0) return FP8WS_ERR_SHAPE;
  if (numel == 0) return FP8WS_OK;  // empty tensors may carry NULL pointers
  if (!g || !u || !s_down || !h) return FP8WS_ERR_NULL;
  if (!aligned16(g) || !aligned16(u) || !aligned16(h)) return FP8WS_ERR_ALIGN;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  return silu_launch(d, g, u, numel, s_down, h, as_stream(stream));
}

int swiglu_2in_fp8(const uint16_t *g, const uint16_t *u, int64_t numel, const float *s_down,
                   const fp8ws_swiglu *act, uint8_t *h, void *stream) {
  if (numel < 0) return FP8WS_ERR_SHAPE;
  SwigluParams ap;
  int rc = swiglu_params(act, &ap);
  if (rc) return rc;
  if (numel == 0) return FP8WS_OK;
  if (!g || !u || !s_down || !h) return FP8WS_ERR_NULL;
  if (!aligned16(g) || !aligned16(u) || !aligned16(h)) return FP8WS_ERR_ALIGN;
  DeviceInfo *d;
  rc = device_info(&d);
  if (rc) return rc;
  cudaStream_t st = as_stream(stream);
  const bool wide = aligned32(g) && aligned32(u) && swiglu_wide_form(d, numel);
  if (ew_launch<swiglu_2in_kernel<true>, swiglu_2in_kernel<false>>(d, wide, numel >> 3, st, g, u,
                                                                    numel, s_down, ap, h) !=
      cudaSuccess)
    return FP8WS_ERR_CUDA;
  log_launch(kKindSwiglu, g, u, h);
  return launch_status();
}

size_t gated_mlp_static_fp8_workspace(int64_t M, int64_t d, int64_t I) {
  if (M < 0 || d < 0 || I < 0) return 0;
  return ws_saturate(ws_region(M, d) + 2 * ws_region(M, I, 2) + ws_region(M, I));
}

int gated_mlp_static_fp8(const uint16_t *x, int64_t M, int64_t dm, int64_t I, const float *s_in,
                         const uint8_t *Wg, const float *s_wg, const uint8_t *Wu,
                         const float *s_wu, const float *s_down, const uint8_t *Wd,
                         const float *s_wd, void *workspace, uint16_t *y, void *stream) {
  if (!s_in || !Wg || !s_wg || !Wu || !s_wu || !s_down || !Wd || !s_wd ||
      (M != 0 && (!x || !y)))
    return FP8WS_ERR_NULL;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FP8WS_ERR_WORKSPACE;
  if (!aligned16(x)) return FP8WS_ERR_ALIGN;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const size_t m = static_cast<size_t>(M < 0 ? 0 : M);
  uint8_t *xq = ws;
  uint16_t *G = reinterpret_cast<uint16_t *>(ws + round256(m * dm));
  uint16_t *U = reinterpret_cast<uint16_t *>(reinterpret_cast<uint8_t *>(G) + round256(m * I * 2));
  uint8_t *H = reinterpret_cast<uint8_t *>(U) + round256(m * I * 2);
  int rc = check_gemm_args(xq, Wg, M, I, dm, s_in, s_wg, G);
  if (!rc) rc = check_gemm_args(xq, Wu, M, I, dm, s_in, s_wu, U);
  if (!rc) rc = check_gemm_args(H, Wd, M, dm, I, s_down, s_wd, y);
  if (rc) return rc;
  DeviceInfo *d;
  rc = device_info(&d);
  if (rc) return rc;
  if (M == 0) return FP8WS_OK;
  cudaStream_t st = as_stream(stream);
  rc = quant_launch(d, x, M * dm, s_in, xq, st);
  if (!rc) rc = gemm_dispatch(d, xq, Wg, M, I, dm, s_in, s_wg, G, st);
  if (!rc) rc = gemm_dispatch(d, xq, Wu, M, I, dm, s_in, s_wu, U, st);
  if (!rc) rc = silu_launch(d, G, U, M * I, s_down, H, st);
  if (!rc) rc = gemm_dispatch(d, H, Wd, M, dm, I, s_down, s_wd, y, st);
  return rc;
}

size_t qkv_shared_quant_workspace(int64_t M, int64_t d) {
  return fp8_shared_quant_linears_workspace(M, d);
}

int qkv_shared_quant(const uint16_t *x, int64_t M, int64_t dm, const float *s_in,
                     const uint8_t *Wq, int64_t Nq, const float *s_wq, const uint8_t *Wk,
                     int64_t Nk, const float *s_wk, const uint8_t *Wv, int64_t Nv,
                     const float *s_wv, void *workspace, uint16_t *q, uint16_t *k, uint16_t *v,
                     void *stream) {
  const uint8_t *W[3] = {Wq, Wk, Wv};
  const int64_t N[3] = {Nq, Nk, Nv};
  const float *s_w[3] = {s_wq, s_wk, s_wv};
  uint16_t *y[3] = {q, k, v};
  return fp8_shared_quant_linears(x, M, dm, s_in, 3, W, N, s_w, y, workspace, stream);
}

int fp8_gate_up_swiglu_static(const uint8_t *xq, const uint8_t *Wg, const uint8_t *Wu,
                              int64_t M, int64_t I, int64_t K, const float *s_in,
                              const float *s_wg, const float *s_wu, const float *s_down,
                              const fp8ws_swiglu *act, uint8_t *h, void *stream) {
  if (!s_down || !Wu || !s_wu) return FP8WS_ERR_NULL;
  int rc = check_gemm_args(xq, Wg, M, I, K, s_in, s_wg, h);
  if (rc) return rc;
  SwigluParams ap;
  rc = swiglu_params(act, &ap);
  if (rc) return rc;
  if (I % 16 != 0) return FP8WS_ERR_SHAPE;  // FP8 rows of H must be 16-byte multiples
  if (!aligned16(Wu)) return FP8WS_ERR_ALIGN;
  DeviceInfo *d;
  rc = device_info(&d);
  if (rc) return rc;
  if (M == 0) return FP8WS_OK;
  return launch_dual_swiglu(d, xq, Wg, Wu, static_cast<int>(M), static_cast<int>(I),
                                  static_cast<int>(K), s_in, s_wg, s_wu, s_down, ap, h,
                                  as_stream(stream));
}

size_t gated_mlp_static_fp8_fused_workspace(int64_t M, int64_t d, int64_t I) {
  if (M < 0 || d < 0 || I < 0) return 0;
  return ws_saturate(ws_region(M, d) + ws_region(M, I));
}

int gated_mlp_static_fp8_fused(const uint16_t *x, int64_t M, int64_t dm, int64_t I,
                               const float *s_in, const uint8_t *Wg, const float *s_wg,
                               const uint8_t *Wu, const float *s_wu, const float *s_down,
                               const fp8ws_swiglu *act, const uint8_t *Wd, const float *s_wd,
                               void *workspace, uint16_t *y, void *stream) {
  if (!s_in || !Wg || !s_wg || !Wu || !s_wu || !s_down || !Wd || !s_wd ||
      (M != 0 && (!x || !y)))
    return FP8WS_ERR_NULL;
  SwigluParams ap;
  int rca = swiglu_params(act, &ap);
  if (rca) return rca;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FP8WS_ERR_WORKSPACE;
  if (!aligned16(x) || !aligned16(Wu)) return FP8WS_ERR_ALIGN;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const size_t m = static_cast<size_t>(M < 0 ? 0 : M);
  uint8_t *xq = ws;
  uint8_t *H = ws + round256(m * dm);
  int rc = check_gemm_args(xq, Wg, M, I, dm, s_in, s_wg, H);
  if (!rc) rc = check_gemm_args(H, Wd, M, dm, I, s_down, s_wd, y);
  if (rc) return rc;
  if (I % 16 != 0) return FP8WS_ERR_SHAPE;
  DeviceInfo *d;
  rc = device_info(&d);
  if (rc) return rc;
  if (M == 0) return FP8WS_OK;
  cudaStream_t st = as_stream(stream);
  rc = quant_launch(d, x, M * dm, s_in, xq, st);
  if (!rc)
    rc = launch_dual_swiglu(d, xq, Wg, Wu, static_cast<int>(M), static_cast<int>(I),
                                  static_cast<int>(dm), s_in, s_wg, s_wu, s_down, ap, H, st);
  if (!rc) rc = gemm_dispatch(d, H, Wd, M, dm, I, s_down, s_wd, y, st);
  return rc;
}

size_t fp8_linear_static_ws_bytes(void) { return splitk_bytes(); }

int fp8_linear_static_ws(const uint8_t *xq, const uint8_t *wq, int64_t M, int64_t N, int64_t K,
                         const float *s_in, const float *s_w, uint16_t *y, void *workspace,
                         size_t workspace_bytes, void *stream) {
  int rc = check_gemm_args(xq, wq, M, N, K, s_in, s_w, y);
  if (rc) return rc;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < splitk_bytes())
    return FP8WS_ERR_WORKSPACE;
  DeviceInfo *d;
  rc = device_info(&d);
  if (rc) return rc;
  if (M == 0) return FP8WS_OK;
  cudaStream_t st = as_stream(stream);
  if (cudaMemsetAsync(splitk_counters(workspace), 0, kSplitkCounterWords * sizeof(int), st) !=
      cudaSuccess)
    return FP8WS_ERR_CUDA;
  return gemm_dispatch(d, xq, wq, M, N, K, s_in, s_w, y, st, workspace);
}

int fp8_quant_static_group(const fp8ws_quant_problem *problems, int count, void *stream) {
  if (count < 1 || count > FP8WS_MAX_GROUP) return FP8WS_ERR_SHAPE;
  if (!problems) return FP8WS_ERR_NULL;
  QuantSeg seg[FP8WS_MAX_GROUP];
  for (int p = 0; p < count; ++p) {
    const fp8ws_quant_problem &q = problems[p];
    if (q.numel < 0) return FP8WS_ERR_SHAPE;
    if (q.numel > 0) {
      if (!q.x || !q.s_in || !q.xq) return FP8WS_ERR_NULL;
      if (!aligned16(q.x) || !aligned16(q.xq)) return FP8WS_ERR_ALIGN;
    }
    seg[p] = QuantSeg{q.x, q.numel, q.s_in, q.xq};
  }
  if (seg[0].numel == 0 && (count < 2 || seg[1].numel == 0)) return FP8WS_OK;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  return quant_pair_launch(d, seg, count, as_stream(stream));
}

int fp8_linear_static_group(const fp8ws_linear_problem *problems, int count, int64_t N,
                            int64_t K, void *workspace, size_t workspace_bytes, void *stream) {
  if (count < 1 || count > FP8WS_MAX_GROUP) return FP8WS_ERR_SHAPE;
  if (!problems) return FP8WS_ERR_NULL;
  PairProblem pp[FP8WS_MAX_GROUP];
  int64_t rows = 0;
  for (int p = 0; p < count; ++p) {
    const fp8ws_linear_problem &q = problems[p];
    const int rc = check_gemm_args(q.xq, q.wq, q.M, N, K, q.s_in, q.s_w, q.y);
    if (rc) return rc;
    pp[p] = PairProblem{q.xq, q.wq, nullptr, q.y, static_cast<int>(q.M), static_cast<int>(N),
                        q.s_in, q.s_w, nullptr, nullptr};
    rows += q.M;
  }
  if (workspace && ((reinterpret_cast<uintptr_t>(workspace) & 255u) ||
                    workspace_bytes < splitk_bytes()))
    return FP8WS_ERR_WORKSPACE;
  if (rows == 0) return FP8WS_OK;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  cudaStream_t st = as_stream(stream);
  if (workspace &&
      cudaMemsetAsync(splitk_counters(workspace), 0, kSplitkCounterWords * sizeof(int), st) !=
          cudaSuccess)
    return FP8WS_ERR_CUDA;
  return gemm_group_dispatch(d, pp, count, static_cast<int>(K), st, workspace);
}

int fp8_gate_up_swiglu_static_group(const fp8ws_gate_up_problem *problems, int count,
                                    int64_t I, int64_t K, const fp8ws_swiglu *act,
                                    void *stream) {
  if (count < 1 || count > FP8WS_MAX_GROUP) return FP8WS_ERR_SHAPE;
  if (!problems) return FP8WS_ERR_NULL;
  SwigluParams ap;
  int rc = swiglu_params(act, &ap);
  if (rc) return rc;
  PairProblem live[FP8WS_MAX_GROUP];
  int n = 0;
  for (int p = 0; p < count; ++p) {
    const fp8ws_gate_up_problem &q = problems[p];
    if (!q.s_down || !q.Wu || !q.s_wu) return FP8WS_ERR_NULL;
    rc = check_gemm_args(q.xq, q.Wg, q.M, I, K, q.s_in, q.s_wg, q.h);
    if (rc) return rc;
    if (!aligned16(q.Wu)) return FP8WS_ERR_ALIGN;
    if (q.M > 0)
      live[n++] = PairProblem{q.xq, q.Wg, q.Wu, q.h, static_cast<int>(q.M), static_cast<int>(I),
                              q.s_in, q.s_wg, q.s_wu, q.s_down};
  }
  if (I % 16 != 0) return FP8WS_ERR_SHAPE;  // FP8 rows of H must be 16-byte multiples
  if (n == 0) return FP8WS_OK;
  DeviceInfo *d;
  rc = device_info(&d);
  if (rc) return rc;
  return launch_dual_swiglu(d, live, n, static_cast<int>(I), static_cast<int>(K), ap,
                            as_stream(stream));
}

size_t gated_mlp_static_fp8_group_workspace(const int64_t *M, int count, int64_t d, int64_t I) {
  if (!M || count < 1 || count > FP8WS_MAX_GROUP || d < 0 || I < 0) return 0;
  u128 total = splitk_bytes();
  for (int p = 0; p < count; ++p) {
    if (M[p] < 0) return 0;
    total += ws_region(M[p], d) + ws_region(M[p], I);
  }
  return ws_saturate(total);
}

int gated_mlp_static_fp8_group(const fp8ws_mlp_tower *towers, int count, int64_t dm, int64_t I,
                               const fp8ws_swiglu *act, void *workspace, size_t workspace_bytes,
                               void *stream) {
  if (count < 1 || count > FP8WS_MAX_GROUP) return FP8WS_ERR_SHAPE;
  if (!towers) return FP8WS_ERR_NULL;
  SwigluParams ap;
  int rc = swiglu_params(act, &ap);
  if (rc) return rc;
  int64_t rows[FP8WS_MAX_GROUP];
  for (int p = 0; p < count; ++p) {
    const fp8ws_mlp_tower &t = towers[p];
    if (t.M < 0) return FP8WS_ERR_SHAPE;
    rows[p] = t.M;
    if (!t.s_in || !t.Wg || !t.s_wg || !t.Wu || !t.s_wu || !t.s_down || !t.Wd || !t.s_wd ||
        (t.M != 0 && (!t.x || !t.y)))
      return FP8WS_ERR_NULL;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < gated_mlp_static_fp8_group_workspace(rows, count, dm, I))
    return FP8WS_ERR_WORKSPACE;
  // workspace: Xq_0, H_0, Xq_1, H_1 (each 256-byte aligned), then the split-K scratch
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  QuantSeg qs[FP8WS_MAX_GROUP];
  PairProblem up[FP8WS_MAX_GROUP], down[FP8WS_MAX_GROUP];
  int n = 0;
  for (int p = 0; p < count; ++p) {
    const fp8ws_mlp_tower &t = towers[p];
    const size_t m = static_cast<size_t>(t.M);
    uint8_t *xq = ws;
    uint8_t *H = ws + round256(m * dm);
    ws += gated_mlp_static_fp8_fused_workspace(t.M, dm, I);
    if (!aligned16(t.x) || !aligned16(t.Wu)) return FP8WS_ERR_ALIGN;
    rc = check_gemm_args(xq, t.Wg, t.M, I, dm, t.s_in, t.s_wg, H);
    if (!rc) rc = check_gemm_args(H, t.Wd, t.M, dm, I, t.s_down, t.s_wd, t.y);
    if (rc) return rc;
    if (t.M == 0) continue;
    qs[n] = QuantSeg{t.x, t.M * dm, t.s_in, xq};
    up[n] = PairProblem{xq, t.Wg, t.Wu, H, static_cast<int>(t.M), static_cast<int>(I), t.s_in,
                        t.s_wg, t.s_wu, t.s_down};
    down[n] = PairProblem{H, t.Wd, nullptr, t.y, static_cast<int>(t.M), static_cast<int>(dm),
                          t.s_down, t.s_wd, nullptr, nullptr};
    ++n;
  }
  if (I % 16 != 0) return FP8WS_ERR_SHAPE;
  if (n == 0) return FP8WS_OK;  // no rows: nothing to do, nothing launched
  DeviceInfo *d;
  rc = device_info(&d);
  if (rc) return rc;
  cudaStream_t st = as_stream(stream);
  void *splitk = ws;  // 256-byte aligned: every region above is a multiple of 256 bytes
  // The quantizer prefetches both towers' X into L2 before it waits for the
  // kernel before it; the down GEMM lets the next kernel on the stream (the
  // next layer's quantizer, in a stack of these calls) launch only as its CTAs
  // start their last tiles, so that such a prefetch overlaps the GEMM's tail.
  rc = quant_pair_launch(d, qs, n, st, splitk_counters(splitk), kSplitkCounterWords);
  if (!rc) rc = launch_dual_swiglu(d, up, n, static_cast<int>(I), static_cast<int>(dm), ap, st);
  if (!rc)
    rc = gemm_group_dispatch(d, down, n, static_cast<int>(I), st, splitk,
                             late_trigger_enabled());
  return rc;
}

}  // extern "C"

// Scratch area of gated_mlp_static_fp8_noalloc, for callers that cannot
// allocate device memory per call.  Reserved in every GPU's memory when the
// library's module is loaded there and kept until the process exits.  Host
// code must not pass the array's name to a kernel: on the host it is only a
// stand-in, and the real device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FP8WS_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[fp8ws::kMaxDevices];  // device address per device, looked up once

// Bytes of scratch gated_mlp_static_fp8 would use for this shape, or SIZE_MAX
// for a shape it refuses (d or I not a positive multiple of 16, or a size of
// 2^31 or more), checked before the size is formed.  The size itself
// saturates rather than wraps (gated_mlp_static_fp8_workspace).
size_t noalloc_bytes(int64_t M, int64_t d, int64_t I) {
  const int64_t lim = int64_t(1) << 31;
  if (M < 0 || d < 16 || I < 16 || d % 16 != 0 || I % 16 != 0 || M >= lim || d >= lim ||
      I >= lim)
    return SIZE_MAX;
  return gated_mlp_static_fp8_workspace(M, d, I);
}

// Device address of the scratch area on the current device; the first call
// per device looks it up with that device current.
int noalloc_scratch(void **out) {
  int dev;
  int rc = fp8ws::current_device(&dev);
  if (rc) return rc;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FP8WS_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return FP8WS_OK;
}
}  // namespace

extern "C" {

int gated_mlp_static_fp8_noalloc(const uint16_t *x, int64_t M, int64_t d, int64_t I,
                                 const float *s_in, const uint8_t *Wg, const float *s_wg,
                                 const uint8_t *Wu, const float *s_wu, const float *s_down,
                                 const uint8_t *Wd, const float *s_wd, uint16_t *y, void *stream) {
  if (noalloc_bytes(M, d, I) > FP8WS_NOALLOC_SCRATCH_BYTES) return FP8WS_ERR_SHAPE;
  void *scratch = nullptr;
  int rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  return gated_mlp_static_fp8(x, M, d, I, s_in, Wg, s_wg, Wu, s_wu, s_down, Wd, s_wd, scratch, y,
                              stream);
}

size_t fp8_shared_quant_linears_workspace(int64_t M, int64_t d) {
  if (M < 0 || d < 0) return 0;
  return ws_saturate(ws_region(M, d) + splitk_bytes());
}

int fp8_shared_quant_linears(const uint16_t *x, int64_t M, int64_t dm, const float *s_in, int n,
                             const uint8_t *const *W, const int64_t *N, const float *const *s_w,
                             uint16_t *const *y, void *workspace, void *stream) {
  if (n < 1 || n > FP8WS_MAX_PROJECTIONS) return FP8WS_ERR_SHAPE;
  if (!W || !N || !s_w || !y || !s_in || (M != 0 && !x)) return FP8WS_ERR_NULL;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FP8WS_ERR_WORKSPACE;
  if (!aligned16(x)) return FP8WS_ERR_ALIGN;
  uint8_t *xq = static_cast<uint8_t *>(workspace);
  void *splitk = xq + round256(static_cast<size_t>(M < 0 ? 0 : M) * static_cast<size_t>(dm));
  int rc = FP8WS_OK;
  PairProblem pp[FP8WS_MAX_PROJECTIONS];
  for (int i = 0; i < n && !rc; ++i) {
    rc = check_gemm_args(xq, W[i], M, N[i], dm, s_in, s_w[i], y[i]);
    pp[i] = PairProblem{xq, W[i], nullptr, y[i], static_cast<int>(M), static_cast<int>(N[i]),
                        s_in, s_w[i], nullptr, nullptr};
  }
  if (rc) return rc;
  DeviceInfo *d;
  rc = device_info(&d);
  if (rc) return rc;
  if (M == 0) return FP8WS_OK;
  cudaStream_t st = as_stream(stream);
  // the quantizer also clears the split-K counters of the GEMMs that follow
  rc = quant_launch(d, x, M * dm, s_in, xq, st, splitk_counters(splitk), kSplitkCounterWords);
  if (!rc) rc = gemm_groups(d, pp, n, static_cast<int>(dm), st, splitk);
  return rc;
}

int fp8_linears_static(const uint8_t *xq, int64_t M, int64_t K, const float *s_in, int n,
                       const uint8_t *const *W, const int64_t *N, const float *const *s_w,
                       uint16_t *const *y, void *workspace, size_t workspace_bytes,
                       void *stream) {
  if (n < 1 || n > FP8WS_MAX_PROJECTIONS) return FP8WS_ERR_SHAPE;
  if (!W || !N || !s_w || !y) return FP8WS_ERR_NULL;
  if (workspace && ((reinterpret_cast<uintptr_t>(workspace) & 255u) ||
                    workspace_bytes < splitk_bytes()))
    return FP8WS_ERR_WORKSPACE;
  PairProblem pp[FP8WS_MAX_PROJECTIONS];
  for (int i = 0; i < n; ++i) {
    const int rc = check_gemm_args(xq, W[i], M, N[i], K, s_in, s_w[i], y[i]);
    if (rc) return rc;
    pp[i] = PairProblem{xq, W[i], nullptr, y[i], static_cast<int>(M), static_cast<int>(N[i]), s_in,
                        s_w[i], nullptr, nullptr};
  }
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  if (M == 0) return FP8WS_OK;
  cudaStream_t st = as_stream(stream);
  if (workspace &&
      cudaMemsetAsync(splitk_counters(workspace), 0, kSplitkCounterWords * sizeof(int), st) !=
          cudaSuccess)
    return FP8WS_ERR_CUDA;
  return gemm_groups(d, pp, n, static_cast<int>(K), st, workspace);
}

size_t cross_attention_qkv_static_fp8_workspace(int64_t Mq, int64_t Mkv, int64_t d) {
  if (Mq < 0 || Mkv < 0 || d < 0) return 0;
  return ws_saturate(ws_region(Mq, d) + ws_region(Mkv, d) + splitk_bytes());
}

int cross_attention_qkv_static_fp8(const uint16_t *x, int64_t Mq, const uint16_t *ctx,
                                   int64_t Mkv, int64_t dm, const float *s_q, const uint8_t *Wq,
                                   int64_t Nq, const float *s_wq, const float *s_kv,
                                   const uint8_t *Wk, int64_t Nk, const float *s_wk,
                                   const uint8_t *Wv, int64_t Nv, const float *s_wv,
                                   void *workspace, uint16_t *q, uint16_t *k, uint16_t *v,
                                   void *stream) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FP8WS_ERR_WORKSPACE;
  if (Mq < 0 || Mkv < 0 || dm < 0) return FP8WS_ERR_SHAPE;
  uint8_t *ws_kv = static_cast<uint8_t *>(workspace) + round256(static_cast<size_t>(Mq) * dm);
  // validate both halves before enqueueing either
  uint8_t *probe = static_cast<uint8_t *>(workspace);
  int rc = check_gemm_args(probe, Wq, Mq, Nq, dm, s_q, s_wq, q);
  if (!rc) rc = check_gemm_args(ws_kv, Wk, Mkv, Nk, dm, s_kv, s_wk, k);
  if (!rc) rc = check_gemm_args(ws_kv, Wv, Mkv, Nv, dm, s_kv, s_wv, v);
  if (!rc && ((Mq != 0 && !x) || (Mkv != 0 && !ctx))) rc = FP8WS_ERR_NULL;
  if (!rc && (!aligned16(x) || !aligned16(ctx))) rc = FP8WS_ERR_ALIGN;
  if (rc) return rc;
  DeviceInfo *d;
  rc = device_info(&d);
  if (rc) return rc;
  if (Mq == 0 && Mkv == 0) return FP8WS_OK;
  cudaStream_t st = as_stream(stream);
  // Q quantized from x at s_q; K and V share one quantization of ctx at s_kv
  // (sharing between Q and K/V must not engage: they read different tensors)
  void *splitk = ws_kv + round256(static_cast<size_t>(Mkv) * dm);
  const QuantSeg qs[2] = {QuantSeg{x, Mq * dm, s_q, probe}, QuantSeg{ctx, Mkv * dm, s_kv, ws_kv}};
  rc = quant_pair_launch(d, qs, 2, st, splitk_counters(splitk), kSplitkCounterWords);
  const PairProblem pp[3] = {
      PairProblem{probe, Wq, nullptr, q, static_cast<int>(Mq), static_cast<int>(Nq), s_q, s_wq,
                  nullptr, nullptr},
      PairProblem{ws_kv, Wk, nullptr, k, static_cast<int>(Mkv), static_cast<int>(Nk), s_kv, s_wk,
                  nullptr, nullptr},
      PairProblem{ws_kv, Wv, nullptr, v, static_cast<int>(Mkv), static_cast<int>(Nv), s_kv, s_wv,
                  nullptr, nullptr}};
  if (!rc) rc = gemm_groups(d, pp, 3, static_cast<int>(dm), st, splitk);
  return rc;
}

int fp8_quant_per_token(const uint16_t *x, int64_t rows, int64_t K, float *s, uint8_t *xq,
                        void *stream) {
  if (rows < 0 || K < 0 || K % 8 != 0 || rows >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return FP8WS_ERR_SHAPE;
  if (rows == 0 || K == 0) return FP8WS_OK;
  if (!x || !s || !xq) return FP8WS_ERR_NULL;
  if (!aligned16(x) || !aligned16(xq)) return FP8WS_ERR_ALIGN;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  cudaStream_t st = as_stream(stream);
  // rows of up to 3072 elements hold 3 vectors per thread, up to 4096 hold 4
  // (fewer registers, more rows in flight per SM: 9.7 against 10.6 us at 4096 x
  // 3072 with 3), up to 8192 hold 8, longer rows are read twice
  auto kern = K <= 3072 ? quant_rows_kernel<3>
                        : (K <= 4096 ? quant_rows_kernel<4> : quant_rows_kernel<8>);
  if (launch_ex(kern,
                dim3(static_cast<unsigned>(rows)), dim3(kQuantRowThreads), 0, st, 1, x,
                static_cast<int>(K), s, xq) != cudaSuccess)
    return FP8WS_ERR_CUDA;
  log_launch(kKindQuant, x, nullptr, xq);
  return launch_status();
}

int fp8_linear_scaled(const uint8_t *xq, const uint8_t *wq, int64_t M, int64_t N, int64_t K,
                      const float *s_x, int x_per_row, const float *s_w, int w_per_col,
                      uint16_t *y, void *stream) {
  int rc = check_gemm_args(xq, wq, M, N, K, s_x, s_w, y);
  if (rc) return rc;
  DeviceInfo *d;
  rc = device_info(&d);
  if (rc) return rc;
  if (M == 0) return FP8WS_OK;
  cudaStream_t st = as_stream(stream);
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  const int mode = (x_per_row ? kScaleRowVec : 0) | (w_per_col ? kScaleColVec : 0);
  switch (mode) {
    case 0: return launch_gemm_pair<3, 0>(d, xq, wq, m, n, k, s_x, s_w, y, st);
    case 1: return launch_gemm_pair<5, 1>(d, xq, wq, m, n, k, s_x, s_w, y, st);
    case 2: return launch_gemm_pair<6, 2>(d, xq, wq, m, n, k, s_x, s_w, y, st);
    default: return launch_gemm_pair<7, 3>(d, xq, wq, m, n, k, s_x, s_w, y, st);
  }
}

int silu_mul_2in_fp8_per_token(const uint16_t *g, const uint16_t *u, int64_t rows, int64_t I,
                               float *s, uint8_t *h, void *stream) {
  if (rows < 0 || I < 0 || I % 8 != 0 || I > kMaxRowI || rows >= (int64_t(1) << 31))
    return FP8WS_ERR_SHAPE;
  if (rows == 0 || I == 0) return FP8WS_OK;
  if (!g || !u || !s || !h) return FP8WS_ERR_NULL;
  if (!aligned16(g) || !aligned16(u) || !aligned16(h)) return FP8WS_ERR_ALIGN;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  const size_t smem = static_cast<size_t>(I) * sizeof(float);
  rc = once_per_device(d, 8, [] {
    const size_t max_smem = kMaxRowI * sizeof(float);
    return cudaFuncSetAttribute(silu_mul_rows_kernel<4>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                max_smem) == cudaSuccess &&
                   cudaFuncSetAttribute(silu_mul_rows_kernel<6>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        max_smem) == cudaSuccess
               ? FP8WS_OK
               : FP8WS_ERR_CUDA;
  });
  if (rc) return rc;
  cudaStream_t st = as_stream(stream);
  // one memory round trip per row where 5 or 6 vector pairs per thread cover it
  // (timed at 4096 x 12288: 41.1 against 52.0 us with 4 per batch; at I = 8192
  // and 14336 the batch of 4 is faster)
  const int64_t per_thread = (I / 8 + kRowThreads - 1) / kRowThreads;
  auto kern = (per_thread == 5 || per_thread == 6) ? silu_mul_rows_kernel<6>
                                                    : silu_mul_rows_kernel<4>;
  if (launch_ex(kern, dim3(static_cast<unsigned>(rows)), dim3(kRowThreads), smem, st, 1, g, u,
                static_cast<int>(I), s, h) != cudaSuccess)
    return FP8WS_ERR_CUDA;
  log_launch(kKindSwiglu, g, u, h);
  return launch_status();
}

size_t gated_mlp_per_token_fp8_workspace(int64_t M, int64_t d, int64_t I) {
  if (M < 0 || d < 0 || I < 0) return 0;
  return ws_saturate(ws_region(M, d) + ws_region(M, 4) + 2 * ws_region(M, I, 2) +
                     ws_region(M, I) + ws_region(M, 4));
}

int gated_mlp_per_token_fp8(const uint16_t *x, int64_t M, int64_t dm, int64_t I,
                            const uint8_t *Wg, const float *s_wg, const uint8_t *Wu,
                            const float *s_wu, const uint8_t *Wd, const float *s_wd,
                            void *workspace, uint16_t *y, void *stream) {
  if (!Wg || !s_wg || !Wu || !s_wu || !Wd || !s_wd || (M != 0 && (!x || !y))) return FP8WS_ERR_NULL;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FP8WS_ERR_WORKSPACE;
  if (M < 0 || dm % 16 != 0 || I % 16 != 0 || I > kMaxRowI) return FP8WS_ERR_SHAPE;
  if (!aligned16(x)) return FP8WS_ERR_ALIGN;
  const size_t m = static_cast<size_t>(M);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  uint8_t *xq = ws;
  float *sx = reinterpret_cast<float *>(ws + round256(m * dm));
  uint16_t *G = reinterpret_cast<uint16_t *>(reinterpret_cast<uint8_t *>(sx) + round256(m * 4));
  uint16_t *U = reinterpret_cast<uint16_t *>(reinterpret_cast<uint8_t *>(G) + round256(m * I * 2));
  uint8_t *H = reinterpret_cast<uint8_t *>(U) + round256(m * I * 2);
  float *sh = reinterpret_cast<float *>(H + round256(m * I));
  int rc = check_gemm_args(xq, Wg, M, I, dm, sx, s_wg, G);
  if (!rc) rc = check_gemm_args(xq, Wu, M, I, dm, sx, s_wu, U);
  if (!rc) rc = check_gemm_args(H, Wd, M, dm, I, sh, s_wd, y);
  if (rc) return rc;
  if (M == 0) return FP8WS_OK;
  DeviceInfo *d;
  rc = device_info(&d);
  if (rc) return rc;
  rc = fp8_quant_per_token(x, M, dm, sx, xq, stream);
  // gate and up share one launch (row and column scale vectors in the epilogue)
  const PairProblem gu[2] = {
      PairProblem{xq, Wg, nullptr, G, static_cast<int>(M), static_cast<int>(I), sx, s_wg, nullptr,
                  nullptr},
      PairProblem{xq, Wu, nullptr, U, static_cast<int>(M), static_cast<int>(I), sx, s_wu, nullptr,
                  nullptr}};
  if (!rc) rc = launch_gemm_pair<7, kScaleRowVec | kScaleColVec>(d, gu, 2, static_cast<int>(dm),
                                                                as_stream(stream));
  if (!rc) rc = silu_mul_2in_fp8_per_token(G, U, M, I, sh, H, stream);
  if (!rc) rc = fp8_linear_scaled(H, Wd, M, dm, I, sh, 1, s_wd, 1, y, stream);
  return rc;
}

int fp8_check_shared_input_scale(const float *const *d_scales, int n, void *stream) {
  if (!d_scales) return FP8WS_ERR_NULL;
  if (n < 1 || n > 4096) return FP8WS_ERR_SHAPE;
  for (int i = 0; i < n; ++i)
    if (!d_scales[i]) return FP8WS_ERR_NULL;
  cudaStream_t st = as_stream(stream);
  float vals[4096];
  for (int i = 0; i < n; ++i)
    if (cudaMemcpyAsync(&vals[i], d_scales[i], sizeof(float), cudaMemcpyDeviceToHost, st) !=
        cudaSuccess)
      return FP8WS_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return FP8WS_ERR_CUDA;
  for (int i = 0; i < n; ++i)
    if (!isfinite(vals[i]) || !(vals[i] > 0.0f)) return FP8WS_ERR_BAD_SCALE;
  uint32_t b0;
  memcpy(&b0, &vals[0], 4);
  for (int i = 1; i < n; ++i) {
    uint32_t bi;
    memcpy(&bi, &vals[i], 4);
    if (bi != b0) return FP8WS_ERR_SCALE_MISMATCH;
  }
  return FP8WS_OK;
}

int fp8_absmax_bf16(const uint16_t *x, int64_t numel, float *amax, void *stream) {
  if (!amax || (numel != 0 && !x)) return FP8WS_ERR_NULL;
  if (numel < 0) return FP8WS_ERR_SHAPE;
  if (!aligned16(x)) return FP8WS_ERR_ALIGN;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  cudaStream_t st = as_stream(stream);
  if (cudaMemsetAsync(amax, 0, sizeof(float), st) != cudaSuccess) return FP8WS_ERR_CUDA;
  if (numel == 0) return FP8WS_OK;
  absmax_bf16_kernel<<<ew_grid<absmax_bf16_kernel>(d, numel >> 3), kEwThreads, 0, st>>>(
      x, numel, reinterpret_cast<unsigned int *>(amax));
  log_launch(kKindCalib, x, nullptr, amax);
  return launch_status();
}

int fp8_silu_mul_absmax(const uint16_t *g, const uint16_t *u, int64_t numel, float *amax,
                        void *stream) {
  if (!amax || (numel != 0 && (!g || !u))) return FP8WS_ERR_NULL;
  if (numel < 0) return FP8WS_ERR_SHAPE;
  if (!aligned16(g) || !aligned16(u)) return FP8WS_ERR_ALIGN;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  cudaStream_t st = as_stream(stream);
  if (cudaMemsetAsync(amax, 0, sizeof(float), st) != cudaSuccess) return FP8WS_ERR_CUDA;
  if (numel == 0) return FP8WS_OK;
  silu_mul_absmax_kernel<<<ew_grid<silu_mul_absmax_kernel>(d, numel >> 3), kEwThreads, 0, st>>>(
      g, u, numel, reinterpret_cast<unsigned int *>(amax));
  log_launch(kKindCalib, g, u, amax);
  return launch_status();
}

int fp8_observer_scale(const float *amaxes, int nbatch, double c, float *scale, void *stream) {
  if (!amaxes || !scale) return FP8WS_ERR_NULL;
  if (nbatch < 1) return FP8WS_ERR_SHAPE;
  if (!isfinite(c)) return FP8WS_ERR_BAD_SCALE;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  observer_scale_kernel<<<1, 32, 0, as_stream(stream)>>>(amaxes, nbatch, c, scale);
  log_launch(kKindCalib, amaxes, nullptr, scale);
  return launch_status();
}

int fp8_rtn_quantize_weight(const uint16_t *w, int64_t numel, float *s_w, uint8_t *wq,
                            void *stream) {
  if (!w || !s_w || !wq) return FP8WS_ERR_NULL;
  if (numel < 1) return FP8WS_ERR_SHAPE;
  if (!aligned16(w) || !aligned16(wq)) return FP8WS_ERR_ALIGN;
  int rc = fp8_absmax_bf16(w, numel, s_w, stream);
  if (rc) return rc;
  cudaStream_t st = as_stream(stream);
  rtn_scale_kernel<<<1, 32, 0, st>>>(s_w);
  log_launch(kKindCalib, s_w, nullptr, s_w);
  rc = launch_status();
  if (rc) return rc;
  return fp8_quant_static(w, numel, s_w, wq, stream);
}

const char *fp8ws_status_string(int status) {
  switch (status) {
    case FP8WS_OK: return "ok";
    case FP8WS_ERR_NULL: return "null pointer";
    case FP8WS_ERR_SHAPE: return "unsupported size";
    case FP8WS_ERR_ALIGN: return "pointer not 16-byte aligned";
    case FP8WS_ERR_SCALE_MISMATCH: return "group input scales differ";
    case FP8WS_ERR_BAD_SCALE: return "scale not finite or not positive";
    case FP8WS_ERR_CUDA: return "CUDA runtime error";
    case FP8WS_ERR_DEVICE_TIMEOUT: return "bounded wait in a kernel ran out";
    case FP8WS_ERR_UNSUPPORTED: return "device is not sm_100";
    case FP8WS_ERR_WORKSPACE: return "workspace NULL or not 256-byte aligned";
    default: return "unknown status";
  }
}

int fp8ws_selftest_bounded_wait(int64_t limit_ns, int mode, int64_t *elapsed_ns, void *stream) {
  if (!elapsed_ns) return FP8WS_ERR_NULL;
  if (limit_ns <= 0 || limit_ns > static_cast<int64_t>(kWaitLimitNs) || (mode != 0 && mode != 1))
    return FP8WS_ERR_SHAPE;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  cudaStream_t st = as_stream(stream);
  selftest_wait_kernel<<<1, 64, 0, st>>>(static_cast<uint64_t>(limit_ns), mode);
  if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
    return FP8WS_ERR_CUDA;
  long long v = 0;
  if (cudaMemcpyFromSymbol(&v, g_selftest_elapsed_ns, sizeof(v)) != cudaSuccess)
    return FP8WS_ERR_CUDA;
  *elapsed_ns = v;
  return FP8WS_OK;
}

int fp8ws_device_check(void) {
  DeviceInfo *d;
  return device_info(&d);
}

int fp8ws_device_status(int *status, int *where) {
  if (!status || !where) return FP8WS_ERR_NULL;
  if (cudaDeviceSynchronize() != cudaSuccess) return FP8WS_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return FP8WS_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return FP8WS_ERR_CUDA;
  *where = v;
  *status = v ? FP8WS_ERR_DEVICE_TIMEOUT : FP8WS_OK;
  return FP8WS_OK;
}

int fp8ws_set_gemm_config(int config) {
  if (config < 0 || config > 4) return FP8WS_ERR_SHAPE;
  g_forced_gemm_config.store(config, std::memory_order_relaxed);
  return FP8WS_OK;
}

int fp8ws_set_quant_form(int form) {
  if (form < 0 || form > 2) return FP8WS_ERR_SHAPE;
  g_quant_form.store(form, std::memory_order_relaxed);
  return FP8WS_OK;
}

int fp8ws_gemm_plan(int sms, int pairs, const int64_t *M, const int64_t *N, int count,
                    int *config) {
  if (!M || !N || !config) return FP8WS_ERR_NULL;
  if (sms < 1 || pairs < 1 || count < 1 || count > kMaxGroup) return FP8WS_ERR_SHAPE;
  for (int p = 0; p < count; ++p)
    if (M[p] < 0 || N[p] < 1) return FP8WS_ERR_SHAPE;
  *config = gemm_cost_choice(sms, pairs, M, N, count);
  return FP8WS_OK;
}

int fp8ws_split_plan(int tiles, int pairs, int num_kb, int has_scratch, int *dp_tiles,
                     int *split_tiles, int *splits, int *kb_per_split, int *halves) {
  if (!dp_tiles || !split_tiles || !splits || !kb_per_split || !halves) return FP8WS_ERR_NULL;
  if (tiles < 0 || pairs < 1 || num_kb < 1) return FP8WS_ERR_SHAPE;
  // the plan only needs to know whether scratch exists; it is not dereferenced here
  float scratch_tag = 0.0f;
  const SplitPlan p =
      make_split_plan(tiles, pairs, num_kb, has_scratch ? &scratch_tag : nullptr, nullptr);
  *dp_tiles = p.dp_tiles;
  *split_tiles = p.split_tiles;
  *splits = p.splits;
  *kb_per_split = p.kb_per_split;
  *halves = p.halves;
  return FP8WS_OK;
}

int64_t fp8ws_launch_count(void) {
  std::lock_guard<std::mutex> lk(g_log_mu);
  return g_launch_total;
}

int fp8ws_launch_log(fp8ws_launch_record *out, int max) {
  if (!out || max <= 0) return 0;
  std::lock_guard<std::mutex> lk(g_log_mu);
  int64_t n = g_log_head < FP8WS_LOG_CAPACITY ? g_log_head : FP8WS_LOG_CAPACITY;
  if (n > max) n = max;
  for (int64_t i = 0; i < n; ++i) out[i] = g_log[(g_log_head - n + i) % FP8WS_LOG_CAPACITY];
  return static_cast<int>(n);
}

void fp8ws_launch_log_clear(void) {
  std::lock_guard<std::mutex> lk(g_log_mu);
  g_log_head = 0;
}

}  // extern "C"
