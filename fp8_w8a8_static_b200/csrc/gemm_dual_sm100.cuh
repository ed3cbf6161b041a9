// Gate/up dual FP8 GEMM with the two-input SwiGLU and the FP8 quantization of
// its result in the epilogue, on CTA pairs (tcgen05 cta_group::2), sm_100a.
//
//   G = bf16((s_in*s_wg) * Xq . Wg^T),  U = bf16((s_in*s_wu) * Xq . Wu^T)
//   H = E4M3_satRNE( SiLU(G) * U * (1/s_down) )            [M, I] FP8
//   (or the alpha/beta/limit SwiGLU variant of swiglu_mul)
//
// The BF16 rounding of G and U and the fp32 SwiGLU arithmetic are the very
// operations of fp8_gemm_kernel's epilogue followed by silu_mul_2in_kernel, so
// H is bit-identical to the unfused path, while G and U never leave the chip.
//
// A cluster of two CTAs computes a 256 x 128 tile of both G and U with one
// M=256, N=256 tcgen05.mma per K slice: the B operand's 256 rows are 128 rows
// of Wg held by the leader CTA and the same 128 rows of Wu held by the peer, so
// accumulator columns 0..127 are G and 128..255 are U.  Each CTA loads 128
// rows of Xq and 128 rows of its weight per 128-byte K step (32 KB per SM, the
// same operand traffic per flop as the plain CTA-pair GEMM).  TMEM per CTA
// holds two buffers of (G 128 columns | U 128 columns), so the epilogue of a
// tile overlaps the main loop of the next.  Eight warps share the epilogue:
// two per TMEM lane quarter (a warp may only read the 32 lanes of quarter
// warp % 4), each taking 64 of the tile's 128 columns, which keeps each
// warp's share of the SwiGLU work per tile small beside the main loop.  A warp reads 32 columns of G and of U per
// step, writes 32 FP8 codes of each row into a 64-byte swizzled row and
// TMA-stores 32 x 64-byte boxes.  Roles, bounded waits and teardown
// follow fp8_gemm_pair_kernel, and so does the problem group: one launch can
// cover the gate/up projections of both towers of a Mixture-of-Transformers
// layer (shared d and I, per-tower rows, weights and scales), their tiles
// dealt as one sequence.
#pragma once

#include "common.cuh"
#include "elementwise.cuh"
#include "gemm_pair_sm100.cuh"

namespace fp8ws {

constexpr int kDualTileM = 256;  // rows per CTA pair
constexpr int kDualTileN = 128;  // columns of G and of U per tile
constexpr int kMaxDualGroup = 2; // problems per grouped launch (the two towers)
constexpr int kDualEpiWarps = 8;                        // two per TMEM lane quarter
constexpr int kDualThreads = (2 + kDualEpiWarps) * 32;  // producer, MMA, epilogue

// DIRECT_: H written with 16-byte global stores from registers instead of
// TMA stores of shared-memory tiles; the freed 32 KB hold a seventh stage.
template <int STAGES_, bool DIRECT_ = false>
struct DualCfg {
  static constexpr int STAGES = STAGES_;
  static constexpr bool DIRECT = DIRECT_;
  static constexpr int A_BYTES = 128 * kGemmBK;   // this CTA's 128 rows of Xq
  static constexpr int B_BYTES = 128 * kGemmBK;   // 128 rows of Wg (leader) or Wu (peer)
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TX_BYTES = 2 * STAGE_BYTES;
  static constexpr int EPI_COLS = kDualTileN / 2;      // columns of H per epilogue warp
  static constexpr int EPI_BUF_BYTES = 32 * EPI_COLS;  // 32 rows x 64 FP8 codes
  static constexpr int EPI_BYTES = DIRECT ? 0 : kDualEpiWarps * 2 * EPI_BUF_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;
  static constexpr uint32_t ACC_COLS = 2 * kDualTileN;  // G | U
  static constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;   // two buffers
  static_assert((2 * STAGES + 5) * 8 + 8 <= BAR_BYTES, "barrier area");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(TMEM_COLS == 512, "tmem");
};

template <int STAGES, bool DIRECT, bool VARIANT>
__global__ void __launch_bounds__(kDualThreads, 1)
    fp8_dual_swiglu_pair_kernel(const __grid_constant__ CUtensorMap tm_a0,
                                const __grid_constant__ CUtensorMap tm_bg0,
                                const __grid_constant__ CUtensorMap tm_bu0,
                                const __grid_constant__ CUtensorMap tm_h0,
                                const __grid_constant__ CUtensorMap tm_a1,
                                const __grid_constant__ CUtensorMap tm_bg1,
                                const __grid_constant__ CUtensorMap tm_bu1,
                                const __grid_constant__ CUtensorMap tm_h1, const PairGroup G,
                                SwigluParams act, int N, int K, uint64_t timeout_ns) {
  using C = DualCfg<STAGES, DIRECT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * C::A_BYTES;
  uint8_t *sEpi = sB + STAGES * C::B_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sEpi + C::EPI_BYTES);
  uint64_t *full = bars;
  uint64_t *empty = bars + STAGES;
  uint64_t *tfull = bars + 2 * STAGES;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  const int num_tiles = G.tiles;
  const int num_kb = (K + kGemmBK - 1) / kGemmBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * kDualEpiWarps);  // every epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_a0);
    tma_prefetch_desc(leader ? &tm_bg0 : &tm_bu0);
    tma_prefetch_desc(&tm_h0);
    if (G.n > 1) {
      tma_prefetch_desc(&tm_a1);
      tma_prefetch_desc(leader ? &tm_bg1 : &tm_bu1);
      tma_prefetch_desc(&tm_h1);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  pdl_launch_dependents();
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
      for (int t = cluster; t < num_tiles && ok; t += nclusters) {
        const GroupTile gt = group_tile(t, G);
        const int a_row = gt.tc.m * kDualTileM + static_cast<int>(rank) * 128;
        const int b_row = gt.tc.n * kDualTileN;
        const CUtensorMap *tm_a = gt.p ? &tm_a1 : &tm_a0;
        const CUtensorMap *tm_b =
            gt.p ? (leader ? &tm_bg1 : &tm_bu1) : (leader ? &tm_bg0 : &tm_bu0);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, timeout_ns)) {
            record_timeout(kSiteProducerEmpty);
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t full_leader = map_shared_rank(smem_u32(&full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], C::TX_BYTES);
          tma_load_2d_pair(sA + stage * C::A_BYTES, tm_a, full_leader, kb * kGemmBK, a_row);
          tma_load_2d_pair(sB + stage * C::B_BYTES, tm_b, full_leader, kb * kGemmBK, b_row);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && leader) {
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
      constexpr uint32_t idesc = idesc_e4m3_f32(kDualTileM, 2 * kDualTileN);
      uint32_t stage = 0, phase = 0;
      uint32_t it = 0;
      bool ok = true;
      for (int t = cluster; t < num_tiles && ok; t += nclusters, ++it) {
        const uint32_t acc = it & 1u;
        const uint32_t acc_phase = (it >> 1) & 1u;
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, timeout_ns)) {
          record_timeout(kSiteMmaTmemEmpty);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_gu = tmem_base + acc * C::ACC_COLS;
        for (int kb = 0; kb < num_kb; ++kb) {
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
            umma_f8_pair(d_gu, smem_desc_k_sw128(a_addr + k * 32),
                         smem_desc_k_sw128(b_addr + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit_pair(&tfull[acc], 0x3);
      }
      umma_commit_pair(drain, 0x1);
      int zero = 0;
      if (!mbar_wait_bounded(drain, 0, &zero, timeout_ns)) record_timeout(kSiteDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue (both CTAs)
    const int ew = warp - 2;                      // 0 .. kDualEpiWarps - 1
    const int quarter = warp & 3;                 // the TMEM lanes this warp may read
    const int cbase = (ew >> 2) * C::EPI_COLS;    // this warp's 64 of the tile's columns
    float scale_g[kMaxDualGroup], scale_u[kMaxDualGroup], inv_s[kMaxDualGroup];
#pragma unroll
    for (int p = 0; p < kMaxDualGroup; ++p) {
      const int q = p < G.n ? p : 0;
      scale_g[p] = __ldg(pick(G.s_in, q)) * __ldg(pick(G.s_w, q));
      scale_u[p] = __ldg(pick(G.s_in, q)) * __ldg(pick(G.s_w2, q));
      inv_s[p] = __frcp_rn(__ldg(pick(G.s_down, q)));
    }
    uint32_t it = 0;
    for (int t = cluster; t < num_tiles; t += nclusters, ++it) {
      const GroupTile gt = group_tile(t, G);
      const TileCoord tc = gt.tc;
      const int M = pick(G.M, gt.p);
      const float sg = gt.p ? scale_g[1] : scale_g[0];
      const float su = gt.p ? scale_u[1] : scale_u[0];
      const float is = gt.p ? inv_s[1] : inv_s[0];
      const CUtensorMap *tm_h = gt.p ? &tm_h1 : &tm_h0;
      uint8_t *h_out = static_cast<uint8_t *>(pick(G.out, gt.p));
      const uint32_t acc = it & 1u;
      const uint32_t acc_phase = (it >> 1) & 1u;
      if (!mbar_wait_bounded_warp(&tfull[acc], acc_phase, abort_flag, timeout_ns)) {
        if (lane == 0) {
          record_timeout(kSiteEpiTmemFull);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int row0 = tc.m * kDualTileM + static_cast<int>(rank) * 128 + quarter * 32;
      const int col0 = tc.n * kDualTileN + cbase;
      const bool store = row0 < M && col0 < N;
      const uint32_t t_g =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * C::ACC_COLS + cbase;
      uint8_t *buf = sEpi + (ew * 2 + (it & 1u)) * C::EPI_BUF_BYTES;
      if (!DIRECT) {
        if (lane == 0) tma_store_wait_read<1>();  // this buffer's previous store has read it
        __syncwarp();
      }
      uint8_t *row = buf + lane * C::EPI_COLS;
      uint8_t *hrow = h_out + static_cast<int64_t>(row0 + lane) * N + col0;
      const bool row_ok = row0 + lane < M;
#pragma unroll 1
      for (int c = 0; c < C::EPI_COLS / 32; ++c) {
        uint32_t g[32], u[32];
        tmem_ld_32x32b_x32(t_g + c * 32, g);
        tmem_ld_32x32b_x32(t_g + kDualTileN + c * 32, u);
        tmem_ld_wait();
        if (c == C::EPI_COLS / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(map_shared_rank(smem_u32(&tempty[acc]), 0));
        }
        uint32_t q[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float h[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float gv = __bfloat162float(__float2bfloat16_rn(__uint_as_float(g[4 * j + e]) * sg));
            const float uv = __bfloat162float(__float2bfloat16_rn(__uint_as_float(u[4 * j + e]) * su));
            h[e] = VARIANT ? swiglu_mul_scaled(gv, uv, is, act) : silu_mul_scaled(gv, uv, is);
          }
          q[j] = pack4(cvt_e4m3x2(h[0], h[1]), cvt_e4m3x2(h[2], h[3]));
        }
        if (DIRECT) {
          // columns col0 + 32c .. +31 of this thread's row (N % 16 == 0)
          if (row_ok && col0 + 32 * c < N)
            *reinterpret_cast<uint4 *>(hrow + 32 * c) = make_uint4(q[0], q[1], q[2], q[3]);
          if (row_ok && col0 + 32 * c + 16 < N)
            *reinterpret_cast<uint4 *>(hrow + 32 * c + 16) = make_uint4(q[4], q[5], q[6], q[7]);
        } else {
          // 32 codes = 16-byte units 2c and 2c + 1 of this 64-byte row, placed
          // as the 64-byte swizzle of the store map expects: unit k of row r
          // at ((k ^ ((r >> 1) & 3)) << 4)
          const int sw = (lane >> 1) & 3;
          *reinterpret_cast<uint4 *>(row + (((2 * c) ^ sw) << 4)) =
              make_uint4(q[0], q[1], q[2], q[3]);
          *reinterpret_cast<uint4 *>(row + (((2 * c + 1) ^ sw) << 4)) =
              make_uint4(q[4], q[5], q[6], q[7]);
        }
      }
      if (!DIRECT) {
        fence_async_shared();
        __syncwarp();
        if (lane == 0 && store) {
          tma_store_2d(tm_h, buf, col0, row0);
        }
        if (lane == 0) tma_store_commit();
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
