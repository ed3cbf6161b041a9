// FP8 E4M3 W8A8 GEMM with the per-tensor dequant in the epilogue, for sm_100a.
//
//   Y[M,N] = bf16( (s_in * s_w) * Xq[M,K] . Wq[N,K]^T ),  fp32 accumulation
//
// Persistent, warp-specialised kernel, one CTA per SM:
//   warp 0      TMA producer: A (128 x 128 B) and B (BN x 128 B) K-major tiles
//               with the 128-byte swizzle into a STAGES-deep shared ring.
//   warp 1      allocates TMEM and issues tcgen05.mma (kind::f8f6f4, M=128,
//               N=BN, K=32 per instruction) from one thread into one of two
//               TMEM accumulators (2 x BN fp32 columns), so the epilogue of a
//               tile overlaps the main loop of the next.
//   warps 2..5  epilogue: tcgen05.ld of 32 lanes x 32 columns, multiply by
//               s_in*s_w, round to BF16, write a 32 x 64 swizzled tile to
//               shared memory and TMA-store it (double buffered per warp).
// Each CTA loads its own tiles (no cluster multicast).  Ragged M, N and K are
// handled by TMA: loads past the tensor read zeros, stores past it are clipped.
// Every mbarrier wait is bounded in time; on a timeout the kernel records the
// site in the device status word, lets in-flight copies and MMAs finish, frees
// its TMEM and returns.
#pragma once

#include "common.cuh"

namespace fp8ws {

constexpr int kGemmThreads = 192;
constexpr int kGemmBM = 128;
constexpr int kGemmBK = 128;  // bytes of K per stage = one 128-byte swizzle row
constexpr int kGroupM = 16;   // M-tiles per raster group (L2 reuse of B tiles)

template <int BN_, int STAGES_>
struct GemmCfg {
  static constexpr int BN = BN_;
  static constexpr int STAGES = STAGES_;
  static constexpr int A_BYTES = kGemmBM * kGemmBK;
  static constexpr int B_BYTES = BN * kGemmBK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_COLS = 64;                // BF16 columns per store box (128 B)
  static constexpr int EPI_BUF_BYTES = 32 * EPI_COLS * 2;
  static constexpr int EPI_BYTES = 4 * 2 * EPI_BUF_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
  static_assert((2 * STAGES + 5) * 8 + 8 <= BAR_BYTES, "barrier area");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(TMEM_COLS >= 32 && TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0, "tmem");
};

struct TileCoord {
  int m, n;
};

// Tile t of a num_m x num_n grid: column by column within groups of group_m
// row blocks (group_m = 1: row by row).
__device__ __forceinline__ TileCoord tile_coord(int t, int num_m, int num_n,
                                                int group_m = kGroupM) {
  const int per_group = group_m * num_n;
  const int group = t / per_group;
  const int first_m = group * group_m;
  const int gsize = min(num_m - first_m, group_m);
  const int r = t - group * per_group;
  return TileCoord{first_m + r % gsize, r / gsize};
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_d, const float *__restrict__ s_in,
                    const float *__restrict__ s_w, int M, int N, int K, uint64_t timeout_ns) {
  using C = GemmCfg<BN, STAGES>;
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
  const int num_m = (M + kGemmBM - 1) / kGemmBM;
  const int num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (K + kGemmBK - 1) / kGemmBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_d);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_launch_dependents();
  pdl_wait();  // the previous kernel's outputs (our inputs) are complete from here on
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;  // per stage: filled once / parity of last fill
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const TileCoord tc = tile_coord(t, num_m, num_n);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, timeout_ns)) {
            record_timeout(kSiteProducerEmpty);
            *abort_flag = 1;
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d(sA + stage * C::A_BYTES, &tm_a, &full[stage], kb * kGemmBK, tc.m * kGemmBM);
          tma_load_2d(sB + stage * C::B_BYTES, &tm_b, &full[stage], kb * kGemmBK, tc.n * BN);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let every load already issued land before the CTA leaves.
        int zero = 0;
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s))
            mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, &zero, timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3_f32(kGemmBM, BN);
      uint32_t stage = 0, phase = 0;
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++it) {
        const uint32_t acc = it & 1u;
        const uint32_t acc_phase = (it >> 1) & 1u;
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, timeout_ns)) {
          record_timeout(kSiteMmaTmemEmpty);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
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
            umma_f8(d_tmem, smem_desc_k_sw128(a_addr + k * 32), smem_desc_k_sw128(b_addr + k * 32),
                    idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(&tfull[acc]);
      }
      // Every MMA issued above has retired once this barrier flips.
      umma_commit(drain);
      int zero = 0;
      if (!mbar_wait_bounded(drain, 0, &zero, timeout_ns)) record_timeout(kSiteDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;        // 0..3: which epilogue warp
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const float scale = __ldg(s_in) * __ldg(s_w);
    uint32_t it = 0, chunk = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      const TileCoord tc = tile_coord(t, num_m, num_n);
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
      const int row0 = tc.m * kGemmBM + quarter * 32;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN;
      constexpr int NCHUNK = BN / C::EPI_COLS;
#pragma unroll 1
      for (int c = 0; c < NCHUNK; ++c) {
        uint32_t r0[32], r1[32];
        tmem_ld_32x32b_x32(t_row + c * C::EPI_COLS, r0);
        tmem_ld_32x32b_x32(t_row + c * C::EPI_COLS + 32, r1);
        tmem_ld_wait();
        if (c == NCHUNK - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        const int col0 = tc.n * BN + c * C::EPI_COLS;
        if (col0 >= N || row0 >= M) continue;  // whole chunk outside Y
        uint8_t *buf = sEpi + (ew * 2 + (chunk & 1u)) * C::EPI_BUF_BYTES;
        if (lane == 0) tma_store_wait_read<1>();
        __syncwarp();
        uint8_t *row = buf + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t *src = (j < 4) ? &r0[j * 8] : &r1[(j - 4) * 8];
          uint4 v;
          __nv_bfloat162 p0 = __floats2bfloat162_rn(__uint_as_float(src[0]) * scale,
                                                    __uint_as_float(src[1]) * scale);
          __nv_bfloat162 p1 = __floats2bfloat162_rn(__uint_as_float(src[2]) * scale,
                                                    __uint_as_float(src[3]) * scale);
          __nv_bfloat162 p2 = __floats2bfloat162_rn(__uint_as_float(src[4]) * scale,
                                                    __uint_as_float(src[5]) * scale);
          __nv_bfloat162 p3 = __floats2bfloat162_rn(__uint_as_float(src[6]) * scale,
                                                    __uint_as_float(src[7]) * scale);
          v.x = *reinterpret_cast<uint32_t *>(&p0);
          v.y = *reinterpret_cast<uint32_t *>(&p1);
          v.z = *reinterpret_cast<uint32_t *>(&p2);
          v.w = *reinterpret_cast<uint32_t *>(&p3);
          *reinterpret_cast<uint4 *>(row + ((j ^ (lane & 7)) << 4)) = v;
        }
        fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_d, buf, col0, row0);
          tma_store_commit();
        }
        ++chunk;
      }
    }
    if (lane == 0) tma_store_wait_all<0>();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace fp8ws
