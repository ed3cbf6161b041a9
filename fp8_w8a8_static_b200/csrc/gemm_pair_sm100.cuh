// FP8 E4M3 W8A8 GEMM on CTA pairs (tcgen05 cta_group::2), for sm_100a.
//
//   Y_p[M_p,N_p] = bf16( (s_in_p * s_w_p) * Xq_p[M_p,K] . Wq_p[N_p,K]^T ),  fp32 accumulation
//
// for a group of up to three problems p that share K (the two towers of a
// Mixture-of-Transformers layer; the Q, K and V projections of one shared
// quantized activation), in one persistent launch.  256 x 256 output
// tiles are computed by a cluster of two CTAs on the two SMs of a TPC.  Each
// CTA loads 128 rows of A and 128 rows of B per 128-byte K step (32 KB instead
// of 48 KB per SM for the same tensor work), both CTAs' loads count on the
// leader CTA's barrier, and the leader issues one M=256, N=256 tcgen05.mma over
// both CTAs' shared memory.  Each CTA's TMEM holds the accumulator of its own
// 128 rows; both CTAs run the epilogue on their own rows.
//   warp 0      TMA producer (both CTAs; no cluster multicast)
//   warp 1      TMEM allocation (both CTAs, cta_group::2); MMA issue (leader)
//   warps 2..5  epilogue (both CTAs)
// The tiles of the group form one sequence (problem 0's, then problem 1's,
// ...), dealt round-robin to the clusters, so each problem fills the ragged
// last wave of the one before.  What remains past the last full wave may be
// split over K (SplitPlan) or, when it would fill at most half a wave, cut
// into 256 x 128 halves (an N = 128 MMA over 64 rows of B per CTA), so that
// the last wave runs twice as many, shorter, units.  Bounded waits as in
// fp8_gemm_kernel.  Both CTAs always reach the final cluster barrier, so
// neither leaves while its peer may still touch its shared memory or TMEM.
#pragma once

#include "common.cuh"
#include "gemm_sm100.cuh"

namespace fp8ws {

constexpr int kPairTile = 256;  // output rows and columns per CTA pair
constexpr int kMaxGroup = 3;    // problems per grouped launch

// The problems of one launch.  Problem p owns global tiles tile_start[p] ..
// tile_start[p + 1] - 1 (tile_start of absent problems: INT_MAX); tiles is
// the total.  s_w2 and s_down are read by the dual gate/up kernel only; out[p]
// is Y_p (BF16) or H_p (FP8) for the register-store epilogues.
struct PairGroup {
  int n;
  int tiles;
  int tile_start[kMaxGroup];
  int M[kMaxGroup];
  int N[kMaxGroup];
  int num_m[kMaxGroup];
  int num_n[kMaxGroup];
  int group_m[kMaxGroup];  // raster: row blocks per column-major group (1 = row-major)
  int hint[kMaxGroup];     // L2 policy of the loads: kHintNone, kHintAFirst or kHintBFirst
  const float *s_in[kMaxGroup];
  const float *s_w[kMaxGroup];
  const float *s_w2[kMaxGroup];
  const float *s_down[kMaxGroup];
  void *out[kMaxGroup];
};

// L2 eviction priority of a problem's operand loads.  The operand that the
// tile order consumes within one wave (A when the tiles run row by row, B
// when they run column by column within row groups) is loaded evict-first,
// so that it leaves L2 before the operand the next waves read again.
constexpr int kHintNone = 0;
constexpr int kHintAFirst = 1;
constexpr int kHintBFirst = 2;

struct GroupTile {
  int p;
  TileCoord tc;
};

// Member p of a group array, by selection rather than indexing, so that the
// kernel parameter block is not copied to local memory.
template <typename T>
__device__ __forceinline__ T pick(const T (&a)[kMaxGroup], int p) {
  return p == 2 ? a[2] : (p == 1 ? a[1] : a[0]);
}

__device__ __forceinline__ GroupTile group_tile(int g, const PairGroup &G) {
  const int p = (g >= G.tile_start[1]) + (g >= G.tile_start[2]);
  return GroupTile{p, tile_coord(g - pick(G.tile_start, p), pick(G.num_m, p), pick(G.num_n, p),
                                 pick(G.group_m, p))};
}

// Split-K of the remainder tiles.  Units 0 .. dp_tiles-1 are whole tiles (the
// full waves); the last split_tiles tiles are each cut into `splits` K ranges
// of kb_per_split 128-byte K steps, one unit per range.  Every split writes
// its fp32 partial (this CTA's 128 x 256) to its own slot of `partials`; the
// last split of a tile to finish, told apart by a per-warp counter in
// `counters` (zero before the launch, reset to zero by that last split), adds
// the partials in split order and runs the epilogue.  splits == 1: no split.
// halves == 2 (then splits == 1): the last split_tiles tiles are each cut
// into two 256 x 128 units over the full K instead (no partials).
struct SplitPlan {
  int dp_tiles;
  int split_tiles;
  int splits;
  int kb_per_split;
  float *partials;  // [split_tiles * splits] slots, see partial_index
  int *counters;    // [split_tiles][2][4]
  int halves;       // 1, or 2: the remainder tiles run as 256 x 128 halves
  // 1: let the next kernel on the stream launch only when this CTA starts its
  // last unit (the next kernel prefetches its input meanwhile), not at once
  int late_trigger;
};

struct UnitRange {
  int tile, kb0, kb1, split, slot;  // split < 0: a whole tile
  int half;                         // -1: all 256 columns; 0 / 1: columns 0-127 / 128-255
};

// A slot holds one CTA pair's 2 x 128 x 256 fp32 partial as float4s indexed
// [CTA][32-column chunk][float4 within the chunk][row], so that the 32 lanes
// of an epilogue warp (32 consecutive rows) touch 512 contiguous bytes.
__device__ __forceinline__ size_t partial_index(int slot, int rank, int chunk, int q4, int row) {
  return (((static_cast<size_t>(slot) * 2 + rank) * 8 + chunk) * 8 + q4) * 128 + row;
}

__device__ __forceinline__ UnitRange unit_range(int u, const SplitPlan &p, int num_kb) {
  if (u < p.dp_tiles) return UnitRange{u, 0, num_kb, -1, -1, -1};
  const int j = u - p.dp_tiles;
  if (p.halves == 2) return UnitRange{p.dp_tiles + (j >> 1), 0, num_kb, -1, -1, j & 1};
  const int sp = j % p.splits;
  const int kb0 = sp * p.kb_per_split;
  const int kb1 = min(kb0 + p.kb_per_split, num_kb);
  return UnitRange{p.dp_tiles + j / p.splits, kb0, kb1, sp, j, -1};
}

__device__ __forceinline__ int plan_units(const SplitPlan &p) {
  return p.dp_tiles + p.split_tiles * p.splits * p.halves;
}

// First output column of a unit, and whether it has any column inside N (the
// second half of a tile in the last, ragged column block may have none; every
// role skips such a unit alike).
__device__ __forceinline__ int unit_col0(const UnitRange &ur, const GroupTile &gt) {
  return gt.tc.n * kPairTile + (ur.half > 0 ? kPairTile / 2 : 0);
}
__device__ __forceinline__ bool unit_live(const UnitRange &ur, const GroupTile &gt,
                                          const PairGroup &G) {
  return ur.half <= 0 || unit_col0(ur, gt) < pick(G.N, gt.p);
}

// Scale modes of the epilogue: bit 0 = one activation scale per row
// (s_in[M], per token), bit 1 = one weight scale per column (s_w[N], per
// channel); 0 = the static per-tensor scalars.
constexpr int kScaleRowVec = 1;
constexpr int kScaleColVec = 2;

// DIRECT_: the epilogue writes Y with 16-byte global stores from registers
// instead of staging 32 x 64 tiles in shared memory for TMA stores; the 32 KB
// this frees hold a seventh pipeline stage.
template <int STAGES_, bool DIRECT_ = false>
struct PairCfg {
  static constexpr int STAGES = STAGES_;
  static constexpr bool DIRECT = DIRECT_;
  static constexpr int A_BYTES = 128 * kGemmBK;   // this CTA's half of A
  static constexpr int B_BYTES = 128 * kGemmBK;   // this CTA's half of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TX_BYTES = 2 * STAGE_BYTES;  // both CTAs, counted at the leader
  static constexpr int TX_HALF_BYTES = 2 * (A_BYTES + B_BYTES / 2);  // a 256 x 128 unit
  static constexpr int EPI_COLS = 64;
  static constexpr int EPI_BUF_BYTES = 32 * EPI_COLS * 2;
  static constexpr int EPI_BYTES = DIRECT ? 0 : 4 * 2 * EPI_BUF_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;  // two 256-column accumulators
  static_assert((2 * STAGES + 5) * 8 + 8 <= BAR_BYTES, "barrier area");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <int STAGES, int SCALE_MODE, bool DIRECT>
__global__ void __launch_bounds__(kGemmThreads, 1)
    fp8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a0,
                         const __grid_constant__ CUtensorMap tm_a1,
                         const __grid_constant__ CUtensorMap tm_a2,
                         const __grid_constant__ CUtensorMap tm_b0,
                         const __grid_constant__ CUtensorMap tm_b1,
                         const __grid_constant__ CUtensorMap tm_b2,
                         const __grid_constant__ CUtensorMap tm_bh0,
                         const __grid_constant__ CUtensorMap tm_bh1,
                         const __grid_constant__ CUtensorMap tm_bh2,
                         const __grid_constant__ CUtensorMap tm_d0,
                         const __grid_constant__ CUtensorMap tm_d1,
                         const __grid_constant__ CUtensorMap tm_d2, const PairGroup G, int K,
                         uint64_t timeout_ns, SplitPlan plan) {
  using C = PairCfg<STAGES, DIRECT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * C::A_BYTES;
  uint8_t *sEpi = sB + STAGES * C::B_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sEpi + C::EPI_BYTES);
  uint64_t *full = bars;              // leader: both CTAs' loads of a stage landed
  uint64_t *empty = bars + STAGES;    // both: the leader's MMAs finished with a stage
  uint64_t *tfull = bars + 2 * STAGES;  // both: an accumulator is complete
  uint64_t *tempty = tfull + 2;       // leader: both CTAs' epilogues read an accumulator
  uint64_t *drain = tempty + 2;       // leader: every MMA retired
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  const int num_kb = (K + kGemmBK - 1) / kGemmBK;
  const int num_units = plan_units(plan);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_a0);
    tma_prefetch_desc(&tm_b0);
    tma_prefetch_desc(&tm_d0);
    if (G.n > 1) {
      tma_prefetch_desc(&tm_a1);
      tma_prefetch_desc(&tm_b1);
      tma_prefetch_desc(&tm_d1);
    }
    if (G.n > 2) {
      tma_prefetch_desc(&tm_a2);
      tma_prefetch_desc(&tm_b2);
      tma_prefetch_desc(&tm_d2);
    }
    if (plan.halves == 2) {
      tma_prefetch_desc(&tm_bh0);
      if (G.n > 1) tma_prefetch_desc(&tm_bh1);
      if (G.n > 2) tma_prefetch_desc(&tm_bh2);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (!plan.late_trigger) pdl_launch_dependents();
  pdl_wait();  // the previous kernel's outputs (our inputs) are complete from here on
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      const uint64_t pol_first = l2_policy_evict_first();
      const uint64_t pol_normal = l2_policy_evict_normal();
      for (int u = cluster; u < num_units && ok; u += nclusters) {
        if (plan.late_trigger && u + nclusters >= num_units) pdl_launch_dependents();
        const UnitRange ur = unit_range(u, plan, num_kb);
        const GroupTile gt = group_tile(ur.tile, G);
        if (!unit_live(ur, gt, G)) continue;
        const bool half = ur.half >= 0;
        const CUtensorMap *tm_a = gt.p == 2 ? &tm_a2 : (gt.p ? &tm_a1 : &tm_a0);
        const CUtensorMap *tm_b = half ? (gt.p == 2 ? &tm_bh2 : (gt.p ? &tm_bh1 : &tm_bh0))
                                       : (gt.p == 2 ? &tm_b2 : (gt.p ? &tm_b1 : &tm_b0));
        const int hint = pick(G.hint, gt.p);
        const uint64_t pol_a = hint == kHintAFirst ? pol_first : pol_normal;
        const uint64_t pol_b = hint == kHintBFirst ? pol_first : pol_normal;
        const int a_row = gt.tc.m * kPairTile + static_cast<int>(rank) * 128;
        // a half unit: 64 rows of B per CTA (N = 128 over the pair)
        const int b_row = unit_col0(ur, gt) + static_cast<int>(rank) * (half ? 64 : 128);
        const uint32_t tx = half ? C::TX_HALF_BYTES : C::TX_BYTES;
        for (int kb = ur.kb0; kb < ur.kb1; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, timeout_ns)) {
            record_timeout(kSiteProducerEmpty);
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t full_leader = map_shared_rank(smem_u32(&full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], tx);
          tma_load_2d_pair_hint(sA + stage * C::A_BYTES, tm_a, full_leader, kb * kGemmBK, a_row,
                                pol_a);
          tma_load_2d_pair_hint(sB + stage * C::B_BYTES, tm_b, full_leader, kb * kGemmBK, b_row,
                                pol_b);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && leader) {
        // Let the loads of the rounds this CTA started land before leaving.
        int zero = 0;
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s))
            mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, &zero, timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------- MMA issue (leader)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc_full = idesc_e4m3_f32(kPairTile, kPairTile);
      constexpr uint32_t idesc_half = idesc_e4m3_f32(kPairTile, kPairTile / 2);
      uint32_t stage = 0, phase = 0;
      uint32_t it = 0;
      bool ok = true;
      for (int u = cluster; u < num_units && ok; u += nclusters) {
        const UnitRange ur = unit_range(u, plan, num_kb);
        if (!unit_live(ur, group_tile(ur.tile, G), G)) continue;
        const uint32_t idesc = ur.half >= 0 ? idesc_half : idesc_full;
        const uint32_t acc = it & 1u;
        const uint32_t acc_phase = (it >> 1) & 1u;
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, timeout_ns)) {
          record_timeout(kSiteMmaTmemEmpty);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kPairTile;
        for (int kb = ur.kb0; kb < ur.kb1; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, timeout_ns)) {
            record_timeout(kSiteMmaFull);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < kGemmBK / 32; ++k) {
            umma_f8_pair(d_tmem, smem_desc_k_sw128(a_addr + k * 32),
                         smem_desc_k_sw128(b_addr + k * 32), idesc,
                         (kb != ur.kb0 || k != 0) ? 1u : 0u);
          }
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit_pair(&tfull[acc], 0x3);
        ++it;
      }
      umma_commit_pair(drain, 0x1);
      int zero = 0;
      if (!mbar_wait_bounded(drain, 0, &zero, timeout_ns)) record_timeout(kSiteDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue (both CTAs)
    const int ew = warp - 2;
    const int quarter = warp & 3;
    uint32_t it = 0, chunk = 0;
    for (int u = cluster; u < num_units; u += nclusters) {
      const UnitRange ur = unit_range(u, plan, num_kb);
      const GroupTile gt = group_tile(ur.tile, G);
      if (!unit_live(ur, gt, G)) continue;
      const TileCoord tc = gt.tc;
      const int M = pick(G.M, gt.p);
      const int N = pick(G.N, gt.p);
      const CUtensorMap *tm_d = gt.p == 2 ? &tm_d2 : (gt.p ? &tm_d1 : &tm_d0);
      const float *s_in = pick(G.s_in, gt.p);
      const float *s_w = pick(G.s_w, gt.p);
      uint16_t *y_out = static_cast<uint16_t *>(pick(G.out, gt.p));
      const uint32_t acc = it & 1u;
      const uint32_t acc_phase = (it >> 1) & 1u;
      ++it;
      if (!mbar_wait_bounded_warp(&tfull[acc], acc_phase, abort_flag, timeout_ns)) {
        if (lane == 0) {
          record_timeout(kSiteEpiTmemFull);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int row0 = tc.m * kPairTile + static_cast<int>(rank) * 128 + quarter * 32;
      const uint32_t t_acc =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * kPairTile;
      // Split unit: publish this partial; only the tile's last split goes on.
      int last_split = -1;  // >= 0: this warp sums the partials of all splits
      if (ur.split >= 0) {
        float4 *slots = reinterpret_cast<float4 *>(plan.partials);
        const int prow = quarter * 32 + lane;
#pragma unroll 1
        for (int c = 0; c < kPairTile / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_acc + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            __stcg(slots + partial_index(ur.slot, static_cast<int>(rank), c, q4, prow),
                   make_float4(__uint_as_float(r[4 * q4]), __uint_as_float(r[4 * q4 + 1]),
                               __uint_as_float(r[4 * q4 + 2]), __uint_as_float(r[4 * q4 + 3])));
        }
        __threadfence();
        __syncwarp();
        int *cnt = plan.counters + ((ur.tile - plan.dp_tiles) * 2 + static_cast<int>(rank)) * 4 +
                   quarter;
        int old = 0;
        if (lane == 0) old = atomicAdd(cnt, 1);
        old = __shfl_sync(0xFFFFFFFFu, old, 0);
        if (old != plan.splits - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(map_shared_rank(smem_u32(&tempty[acc]), 0));
          continue;
        }
        __threadfence();
        if (lane == 0) atomicExch(cnt, 0);  // ready for the next launch
        last_split = ur.split;
      }
      const float scale = (SCALE_MODE == 0) ? __ldg(s_in) * __ldg(s_w) : 0.0f;
      float row_scale = 0.0f;  // this thread's row factor (row0 + lane)
      if (SCALE_MODE != 0) {
        const int my_row = row0 + lane;
        row_scale = (SCALE_MODE & kScaleRowVec) ? (my_row < M ? __ldg(s_in + my_row) : 0.0f)
                                                : __ldg(s_in);
        if (!(SCALE_MODE & kScaleColVec)) row_scale *= __ldg(s_w);
      }
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * kPairTile;
      // 64-column chunks of this unit: 4 for a whole tile, 2 for a half
      const int nchunk = (ur.half >= 0 ? kPairTile / 2 : kPairTile) / C::EPI_COLS;
#pragma unroll 1
      for (int c = 0; c < nchunk; ++c) {
        uint32_t r0[32], r1[32];
        tmem_ld_32x32b_x32(t_row + c * C::EPI_COLS, r0);
        tmem_ld_32x32b_x32(t_row + c * C::EPI_COLS + 32, r1);
        tmem_ld_wait();
        if (last_split >= 0) {
          // sum the tile's partials in split order (this split's from TMEM)
          const float4 *slots = reinterpret_cast<const float4 *>(plan.partials);
          const int prow = quarter * 32 + lane;
          const int first_slot = ur.slot - last_split;
          float v[64];
#pragma unroll
          for (int e = 0; e < 64; ++e) v[e] = 0.0f;
          for (int sp = 0; sp < plan.splits; ++sp) {
            if (sp == last_split) {
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                v[e] += __uint_as_float(r0[e]);
                v[32 + e] += __uint_as_float(r1[e]);
              }
            } else {
#pragma unroll
              for (int q4 = 0; q4 < 16; ++q4) {
                // 64 columns of this chunk = 32-column chunks 2c and 2c + 1
                const float4 w = __ldcg(slots + partial_index(first_slot + sp,
                                                              static_cast<int>(rank),
                                                              2 * c + q4 / 8, q4 % 8, prow));
                v[4 * q4] += w.x;
                v[4 * q4 + 1] += w.y;
                v[4 * q4 + 2] += w.z;
                v[4 * q4 + 3] += w.w;
              }
            }
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            r0[e] = __float_as_uint(v[e]);
            r1[e] = __float_as_uint(v[32 + e]);
          }
        }
        if (c == nchunk - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(map_shared_rank(smem_u32(&tempty[acc]), 0));
        }
        const int col0 = unit_col0(ur, gt) + c * C::EPI_COLS;
        if (col0 >= N || row0 >= M) continue;  // whole chunk outside Y
        // per-column scales of this chunk: lane l holds columns l and 32 + l
        float cs0 = 0.0f, cs1 = 0.0f;
        if (SCALE_MODE & kScaleColVec) {
          cs0 = col0 + lane < N ? __ldg(s_w + col0 + lane) : 0.0f;
          cs1 = col0 + 32 + lane < N ? __ldg(s_w + col0 + 32 + lane) : 0.0f;
        }
        uint8_t *buf = sEpi + (ew * 2 + (chunk & 1u)) * C::EPI_BUF_BYTES;
        if (!DIRECT) {
          if (lane == 0) tma_store_wait_read<1>();
          __syncwarp();
        }
        uint8_t *row = buf + lane * 128;
        // direct stores: this thread's row of Y, 64 columns from col0
        uint16_t *yrow = y_out + static_cast<int64_t>(row0 + lane) * N + col0;
        const bool row_ok = row0 + lane < M;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t *src = (j < 4) ? &r0[j * 8] : &r1[(j - 4) * 8];
          float sc[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (SCALE_MODE == 0) {
              sc[e] = scale;
            } else if (SCALE_MODE & kScaleColVec) {
              const int cc = j * 8 + e;  // column within the chunk
              sc[e] = row_scale * __shfl_sync(0xFFFFFFFFu, cc < 32 ? cs0 : cs1, cc & 31);
            } else {
              sc[e] = row_scale;
            }
          }
          uint4 v;
          __nv_bfloat162 p0 = __floats2bfloat162_rn(__uint_as_float(src[0]) * sc[0],
                                                    __uint_as_float(src[1]) * sc[1]);
          __nv_bfloat162 p1 = __floats2bfloat162_rn(__uint_as_float(src[2]) * sc[2],
                                                    __uint_as_float(src[3]) * sc[3]);
          __nv_bfloat162 p2 = __floats2bfloat162_rn(__uint_as_float(src[4]) * sc[4],
                                                    __uint_as_float(src[5]) * sc[5]);
          __nv_bfloat162 p3 = __floats2bfloat162_rn(__uint_as_float(src[6]) * sc[6],
                                                    __uint_as_float(src[7]) * sc[7]);
          v.x = *reinterpret_cast<uint32_t *>(&p0);
          v.y = *reinterpret_cast<uint32_t *>(&p1);
          v.z = *reinterpret_cast<uint32_t *>(&p2);
          v.w = *reinterpret_cast<uint32_t *>(&p3);
          if (DIRECT) {
            if (row_ok && col0 + j * 8 < N) *reinterpret_cast<uint4 *>(yrow + j * 8) = v;
          } else {
            *reinterpret_cast<uint4 *>(row + ((j ^ (lane & 7)) << 4)) = v;
          }
        }
        if (!DIRECT) {
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(tm_d, buf, col0, row0);
            tma_store_commit();
          }
        }
        ++chunk;
      }
    }
    if (lane == 0) tma_store_wait_all<0>();
  }

  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace fp8ws
