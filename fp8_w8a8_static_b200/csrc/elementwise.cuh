// HBM-bound kernels of the static FP8 path: the activation quantizer, the
// two-input SwiGLU with FP8 output, and the calibration reductions.
//
// All of them stream flat contiguous runs: each thread moves 16-byte vectors
// (8 BF16 values) with several vectors in flight, grids are sized to fill every
// SM, and the ragged tail (numel not a multiple of 8) is finished by the first
// threads of the grid one element at a time.  The hot ones (the quantizer and
// the two-input SwiGLU) also have a wide form: 32-byte loads (16 values) and
// 16-byte stores of the codes, half the memory instructions per byte.  The host
// chooses it for 32-byte-aligned inputs (for the SwiGLU kernels also by length:
// swiglu_wide_form in fp8ws.cu).
#pragma once

#include "common.cuh"

namespace fp8ws {

constexpr int kEwThreads = 256;  // threads per block of the streaming kernels
constexpr int kEwUnroll = 4;     // 16-byte vectors in flight per thread and input
constexpr int kEwWideUnroll = 2; // 32-byte vectors in flight per thread and input (wide form)

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two fp32 values -> two E4M3 codes (first value in the low byte), rounded to
// nearest even with saturation to +-448 (NaN stays NaN).
__device__ __forceinline__ uint32_t cvt_e4m3x2(float a, float b) {
  return static_cast<uint32_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ uint32_t pack4(uint32_t p01, uint32_t p23) {
  return (p01 & 0xFFFFu) | (p23 << 16);
}

// Streaming loads/stores: every byte is touched once.
__device__ __forceinline__ uint4 ld_stream(const uint4 *p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(uint2 *p, uint2 v) { __stcs(p, v); }
__device__ __forceinline__ void st_stream(uint4 *p, uint4 v) { __stcs(p, v); }

// 32-byte streaming load (the 8 x 32-bit vector form of ld.global on
// sm_100): 16 BF16 values, the first 8 in lo.  p must be 32-byte aligned.
__device__ __forceinline__ void ld_stream_wide(const uint16_t *p, uint4 &lo, uint4 &hi) {
  asm volatile("ld.global.cs.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y),
                 "=r"(hi.z), "=r"(hi.w)
               : "l"(p));
}

__device__ __forceinline__ uint4 join(uint2 a, uint2 b) { return make_uint4(a.x, a.y, b.x, b.y); }

// The streaming loops.  Threads tid = 0 .. nthreads - 1 of a range visit its
// vectors with a stride of nthreads, kEwUnroll (kEwWideUnroll) vectors per
// input in flight; op8(v...) maps 8 BF16 values per input to 8 codes.  The
// return value is the number of leading elements covered by whole vectors; the
// caller finishes the rest (fewer than 16) one element per thread.
template <bool WIDE, typename Op8>
__device__ __forceinline__ int64_t stream1(const uint16_t *__restrict__ x, int64_t numel,
                                           uint8_t *__restrict__ out, int64_t tid,
                                           int64_t nthreads, Op8 op8) {
  if constexpr (WIDE) {
    const int64_t nw = numel >> 4;
    uint4 *ov = reinterpret_cast<uint4 *>(out);
    int64_t i = tid;
    for (; i + (kEwWideUnroll - 1) * nthreads < nw; i += kEwWideUnroll * nthreads) {
      uint4 lo[kEwWideUnroll], hi[kEwWideUnroll];
#pragma unroll
      for (int k = 0; k < kEwWideUnroll; ++k)
        ld_stream_wide(x + (i + k * nthreads) * 16, lo[k], hi[k]);
#pragma unroll
      for (int k = 0; k < kEwWideUnroll; ++k)
        st_stream(ov + i + k * nthreads, join(op8(lo[k]), op8(hi[k])));
    }
    for (; i < nw; i += nthreads) {
      uint4 lo, hi;
      ld_stream_wide(x + i * 16, lo, hi);
      st_stream(ov + i, join(op8(lo), op8(hi)));
    }
    return nw << 4;
  } else {
    const int64_t nvec = numel >> 3;
    const uint4 *xv = reinterpret_cast<const uint4 *>(x);
    uint2 *ov = reinterpret_cast<uint2 *>(out);
    int64_t i = tid;
    for (; i + (kEwUnroll - 1) * nthreads < nvec; i += kEwUnroll * nthreads) {
      uint4 v[kEwUnroll];
#pragma unroll
      for (int k = 0; k < kEwUnroll; ++k) v[k] = ld_stream(xv + i + k * nthreads);
#pragma unroll
      for (int k = 0; k < kEwUnroll; ++k) st_stream(ov + i + k * nthreads, op8(v[k]));
    }
    for (; i < nvec; i += nthreads) st_stream(ov + i, op8(ld_stream(xv + i)));
    return nvec << 3;
  }
}

template <bool WIDE, typename Op8>
__device__ __forceinline__ int64_t stream2(const uint16_t *__restrict__ a,
                                           const uint16_t *__restrict__ b, int64_t numel,
                                           uint8_t *__restrict__ out, int64_t tid,
                                           int64_t nthreads, Op8 op8) {
  if constexpr (WIDE) {
    const int64_t nw = numel >> 4;
    uint4 *ov = reinterpret_cast<uint4 *>(out);
    int64_t i = tid;
    for (; i + (kEwWideUnroll - 1) * nthreads < nw; i += kEwWideUnroll * nthreads) {
      uint4 a0[kEwWideUnroll], a1[kEwWideUnroll], b0[kEwWideUnroll], b1[kEwWideUnroll];
#pragma unroll
      for (int k = 0; k < kEwWideUnroll; ++k) {
        ld_stream_wide(a + (i + k * nthreads) * 16, a0[k], a1[k]);
        ld_stream_wide(b + (i + k * nthreads) * 16, b0[k], b1[k]);
      }
#pragma unroll
      for (int k = 0; k < kEwWideUnroll; ++k)
        st_stream(ov + i + k * nthreads, join(op8(a0[k], b0[k]), op8(a1[k], b1[k])));
    }
    for (; i < nw; i += nthreads) {
      uint4 a0, a1, b0, b1;
      ld_stream_wide(a + i * 16, a0, a1);
      ld_stream_wide(b + i * 16, b0, b1);
      st_stream(ov + i, join(op8(a0, b0), op8(a1, b1)));
    }
    return nw << 4;
  } else {
    const int64_t nvec = numel >> 3;
    const uint4 *av = reinterpret_cast<const uint4 *>(a);
    const uint4 *bv = reinterpret_cast<const uint4 *>(b);
    uint2 *ov = reinterpret_cast<uint2 *>(out);
    int64_t i = tid;
    for (; i + (kEwUnroll - 1) * nthreads < nvec; i += kEwUnroll * nthreads) {
      uint4 va[kEwUnroll], vb[kEwUnroll];
#pragma unroll
      for (int k = 0; k < kEwUnroll; ++k) {
        va[k] = ld_stream(av + i + k * nthreads);
        vb[k] = ld_stream(bv + i + k * nthreads);
      }
#pragma unroll
      for (int k = 0; k < kEwUnroll; ++k) st_stream(ov + i + k * nthreads, op8(va[k], vb[k]));
    }
    for (; i < nvec; i += nthreads) st_stream(ov + i, op8(ld_stream(av + i), ld_stream(bv + i)));
    return nvec << 3;
  }
}

// ------------------------------------------------------------- quantize
// q = E4M3_satRNE(fl32(x / s)), the code of the IEEE fp32 quotient.
//
// The code only depends on which E4M3 rounding interval fl32(x / s) falls in.
// With r = fl32(1/s), t = fl32(x * r) = (x/s)(1 + d) with |d| <= 2^-23 + 2^-48,
// and fl32(x/s) = (x/s)(1 + e) with |e| <= 2^-24, so the two differ by less
// than 3 ulp of t (an ulp is at least 2^-24 |t|).  Rounding to E4M3 is
// monotone, so when the floats 4 ulp below and above t (adjacent bit
// patterns, across a binade boundary too) give the same code, that is the
// code of the quotient.  Otherwise (t near an E4M3 rounding boundary, near
// zero, or not finite) the quotient is computed with IEEE division.
// r for the tests below: fl32(1/s) when that is a normal fp32 number, else 0.
// With r = 0 every test fails (the bits 4 ulp below +-0 are a NaN), so a scale
// whose reciprocal overflows or is subnormal sends each value to IEEE
// division: 0 * inf would otherwise give the NaN code for x = 0.
__device__ __forceinline__ float quant_recip(float s) {
  const float r = __frcp_rn(s);
  return (r >= 0x1p-126f && r <= 0x1p126f) ? r : 0.0f;
}

__device__ __forceinline__ uint32_t quant1(float x, float s, float r) {
  const float t = x * r;
  const uint32_t b = __float_as_uint(t);
  const uint32_t lohi = cvt_e4m3x2(__uint_as_float(b - 4u), __uint_as_float(b + 4u));
  if ((lohi & 0xFFu) == (lohi >> 8)) return lohi & 0xFFu;
  return cvt_e4m3x2(__fdiv_rn(x, s), 0.0f) & 0xFFu;
}

// The vector kernels test 8 values at once with a cheaper bracket (quant1
// above serves the values past the last whole vector): with
// rl = fl32(r (1 - 2^-20)) and rh = fl32(r (1 + 2^-20)) (r = fl32(1/s)
// normal), the products x rl and x rh bracket the IEEE quotient fl32(x / s)
// in magnitude while they are normal fp32 numbers: r, rl or rh and the product
// each add a relative error of at most 2^-24, about 3 * 2^-24 in all, far
// inside the 2^-20 offset, and fl32(x / s) is within 2^-24 of x / s.  Rounding
// to E4M3 is monotone, so equal codes at both ends are the quotient's code.
// Quotients below the fp32 normal range give the code +-0, as do both
// products; overflowing ones saturate at both ends.  A pair of values takes
// one packed f32x2 multiply per end.  Any other scale (1/s overflowing,
// subnormal, zero, negative or NaN) gets rl = 0 and rh = inf, whose codes
// never agree unless x is a NaN, so every value goes to IEEE division.
struct QuantBracket {
  uint64_t lo, hi;  // rl, rh in both halves of an f32x2
  float s;
};

__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}

__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// E4M3 codes of the two halves of an f32x2, the low half in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return cvt_e4m3x2(lo, hi);
}

__device__ __forceinline__ QuantBracket quant_bracket(float s) {
  const float r = __frcp_rn(s);
  const bool ok = r >= 0x1p-126f && r <= 0x1p126f;
  const float rl = ok ? __fmul_rn(r, 1.0f - 0x1p-20f) : 0.0f;
  const float rh = ok ? __fmul_rn(r, 1.0f + 0x1p-20f) : __int_as_float(0x7F800000);
  return QuantBracket{f32x2(rl, rl), f32x2(rh, rh), s};
}

// The pairs whose two ends disagree, by IEEE division; out of line so that
// the common path keeps few registers.
__device__ __noinline__ uint2 quant8_divide(uint4 v, float s, uint2 lo, uint2 hi) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t c[4] = {lo.x & 0xFFFFu, lo.x >> 16, lo.y & 0xFFFFu, lo.y >> 16};
  const uint32_t h[4] = {hi.x & 0xFFFFu, hi.x >> 16, hi.y & 0xFFFFu, hi.y >> 16};
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (c[k] != h[k]) c[k] = cvt_e4m3x2(__fdiv_rn(bf16_lo(w[k]), s), __fdiv_rn(bf16_hi(w[k]), s));
  return make_uint2(pack4(c[0], c[1]), pack4(c[2], c[3]));
}

__device__ __forceinline__ uint2 quant8_bracket(uint4 v, const QuantBracket &q) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t lo[4], hi[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint64_t x = f32x2(bf16_lo(w[k]), bf16_hi(w[k]));
    lo[k] = cvt_e4m3x2(mul_f32x2(x, q.lo));
    hi[k] = cvt_e4m3x2(mul_f32x2(x, q.hi));
  }
  const uint2 a = make_uint2(pack4(lo[0], lo[1]), pack4(lo[2], lo[3]));
  const uint2 b = make_uint2(pack4(hi[0], hi[1]), pack4(hi[2], hi[3]));
  if (a.x == b.x && a.y == b.y) return a;
  return quant8_divide(v, q.s, a, b);
}

// zero_words / n_zero: an optional int array cleared by block 0 (the split-K
// counters of the GEMMs that follow on the stream).
// The blocks block0 .. block0 + nblocks - 1 of a launch quantize x, each
// vector visited by one thread with a stride of the blocks' thread count.
template <bool WIDE>
__device__ __forceinline__ void quant_static_range(const uint16_t *__restrict__ x, int64_t numel,
                                                   const float *__restrict__ s_in,
                                                   uint8_t *__restrict__ xq, int block,
                                                   int nblocks) {
  if (numel <= 0) return;
  const float s = __ldg(s_in);
  const QuantBracket q = quant_bracket(s);
  const int64_t tid = static_cast<int64_t>(block) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(nblocks) * blockDim.x;
  const int64_t done =
      stream1<WIDE>(x, numel, xq, tid, nthreads, [&q](uint4 v) { return quant8_bracket(v, q); });
  const int64_t t = done + tid;
  if (t < numel) {
    float a = __uint_as_float(static_cast<uint32_t>(x[t]) << 16);
    xq[t] = static_cast<uint8_t>(quant1(a, s, quant_recip(s)));
  }
}

// Two activations, each with its own scale, quantized by one launch (the two
// towers of a layer): blocks 0 .. split - 1 take the first, the rest the
// second; one activation is the case of an empty second one and split equal
// to the grid.  Block 0 also clears n_zero words at zero_words (split-K
// counters of a later kernel).
struct QuantSeg {
  const uint16_t *x;
  int64_t numel;
  const float *s_in;
  uint8_t *xq;
};

// Thread 0 of block `blk` of the first `nblk` blocks prefetches its share of
// the n bytes at p into L2 (in 32 KB bulk prefetches; a tail of fewer than 16
// bytes is left to the loads).
__device__ __forceinline__ void prefetch_share_l2(const void *p, int64_t n, int blk, int nblk) {
  if (n <= 0 || blk >= nblk) return;
  const int64_t share = ((n + nblk - 1) / nblk + 15) & ~int64_t{15};
  const int64_t lo = static_cast<int64_t>(blk) * share;
  const int64_t hi = min(lo + share, n) & ~int64_t{15};
  const uint8_t *base = static_cast<const uint8_t *>(p);
  for (int64_t o = lo; o < hi; o += 32768) {
    const int64_t len = hi - o < 32768 ? hi - o : 32768;
    prefetch_l2_bulk(base + o, static_cast<uint32_t>(len));
  }
}

// prefetch_blocks > 0: before waiting for the previous kernel, thread 0 of
// each of the first prefetch_blocks blocks (those resident earliest, one per
// SM) prefetches its share of both inputs into L2, so that their DRAM reads
// overlap the end of the previous kernel (which, in the grouped gated MLP,
// lets this grid launch only as it starts its last tiles).  When the previous
// kernel has already finished, the prefetch merely runs beside the loads.
template <bool WIDE>
__global__ void __launch_bounds__(kEwThreads)
    quant_static_pair_kernel(const QuantSeg a, const QuantSeg b, int split,
                             int *__restrict__ zero_words, int n_zero, int prefetch_blocks) {
  pdl_launch_dependents();
  if (threadIdx.x == 0 && prefetch_blocks > 0) {
    prefetch_share_l2(a.x, a.numel * 2, blockIdx.x, prefetch_blocks);
    prefetch_share_l2(b.x, b.numel * 2, blockIdx.x, prefetch_blocks);
  }
  pdl_wait();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero_words[i] = 0;
  if (static_cast<int>(blockIdx.x) < split)
    quant_static_range<WIDE>(a.x, a.numel, a.s_in, a.xq, blockIdx.x, split);
  else
    quant_static_range<WIDE>(b.x, b.numel, b.s_in, b.xq, blockIdx.x - split, gridDim.x - split);
}

// ---------------------------------------------------- quantize, staged form
// The staged quantizer: one CTA per SM (fewer for short inputs).  The input
// runs (one or two activations, each with its own scale) are cut into chunks
// of kStagedChunk bytes of whole 8-value vectors, dealt to the CTAs round
// robin.  A producer thread streams its CTA's chunks into a ring of
// kStagedStages shared-memory slots with cp.async.bulk, each completing an
// mbarrier by its byte count; kStagedConsumerWarps warps convert each chunk
// and store the codes, then release the slot.  The bytes in flight per SM are
// set by the ring, not by registers, so reads keep streaming while the
// consumers work.  With two CTAs' worth of shared memory and threads free on
// each SM, the next launch's CTA can become resident and wait beside it.
constexpr int kStagedChunk = 16384;  // input bytes per chunk (8192 BF16 values)
constexpr int kStagedStages = 6;
constexpr int kStagedConsumerWarps = 16;
constexpr int kStagedConsumers = kStagedConsumerWarps * 32;
constexpr int kStagedThreads = kStagedConsumers + 32;  // + the producer warp
constexpr int kStagedSmem = kStagedStages * kStagedChunk + 2 * kStagedStages * 8 + 16;

__host__ __device__ __forceinline__ int64_t staged_chunks(int64_t numel) {
  return ((numel >> 3) * 16 + kStagedChunk - 1) / kStagedChunk;
}

// Chunk c of the two runs: its run, its byte offset in that run's input and
// its length in bytes (a multiple of 16).
__device__ __forceinline__ void staged_chunk(const QuantSeg &a, const QuantSeg &b, int64_t ca,
                                             int64_t c, bool &second, int64_t &off,
                                             uint32_t &bytes) {
  second = c >= ca;
  const QuantSeg &g = second ? b : a;
  off = (second ? c - ca : c) * kStagedChunk;
  const int64_t run = (g.numel >> 3) * 16;
  bytes = static_cast<uint32_t>(run - off < kStagedChunk ? run - off : kStagedChunk);
}

// a, b: the two runs (b.numel = 0 for one).  Block 0 also clears n_zero words
// at zero_words and quantizes the fewer than 8 values past each run's last
// whole vector.  prefetch: before waiting for the previous kernel, the
// producer prefetches its CTA's chunks into L2.  Waits give up after
// timeout_ns (device status word, wait sites 7 and 8).
__global__ void __launch_bounds__(kStagedThreads, 2)
    quant_staged_kernel(const QuantSeg a, const QuantSeg b, int *__restrict__ zero_words,
                        int n_zero, int prefetch, uint64_t timeout_ns) {
  extern __shared__ __align__(128) uint8_t staged_smem[];
  uint8_t *ring = staged_smem;
  uint64_t *full = reinterpret_cast<uint64_t *>(staged_smem + kStagedStages * kStagedChunk);
  uint64_t *empty = full + kStagedStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kStagedStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ca = staged_chunks(a.numel);
  const int64_t total = ca + staged_chunks(b.numel);
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStagedStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kStagedConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kStagedConsumerWarps && lane == 0 && prefetch) {
    for (int64_t c = blockIdx.x; c < total; c += gridDim.x) {
      bool second;
      int64_t off;
      uint32_t bytes;
      staged_chunk(a, b, ca, c, second, off, bytes);
      prefetch_l2_bulk(reinterpret_cast<const uint8_t *>(second ? b.x : a.x) + off, bytes);
    }
  }
  __syncthreads();
  pdl_wait();

  if (warp == kStagedConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    const uint64_t pol = l2_policy_evict_first();
    uint32_t issued = 0, parity = 0;
    bool ok = true;
    int j = 0;
    for (int64_t c = blockIdx.x; c < total; c += gridDim.x, ++j) {
      const int slot = j % kStagedStages;
      const uint32_t ph = (j / kStagedStages) & 1u;
      if (!mbar_wait_bounded(&empty[slot], ph ^ 1u, abort_flag, timeout_ns)) {
        record_timeout(kSiteStagedEmpty);
        *abort_flag = 1;
        ok = false;
        break;
      }
      bool second;
      int64_t off;
      uint32_t bytes;
      staged_chunk(a, b, ca, c, second, off, bytes);
      mbar_arrive_expect_tx(&full[slot], bytes);
      bulk_load_1d(ring + slot * kStagedChunk,
                   reinterpret_cast<const uint8_t *>(second ? b.x : a.x) + off, bytes,
                   &full[slot], pol);
      issued |= 1u << slot;
      parity = (parity & ~(1u << slot)) | (ph << slot);
    }
    if (!ok) {
      // let the copies this CTA started land before it can exit
      int zero = 0;
      for (int s = 0; s < kStagedStages; ++s)
        if (issued & (1u << s)) mbar_wait_bounded(&full[s], (parity >> s) & 1u, &zero, timeout_ns);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int t = threadIdx.x;
  const QuantBracket qa = quant_bracket(a.numel > 0 ? __ldg(a.s_in) : 1.0f);
  const QuantBracket qb = quant_bracket(b.numel > 0 ? __ldg(b.s_in) : 1.0f);
  if (blockIdx.x == 0) {
    for (int i = t; i < n_zero; i += kStagedConsumers) zero_words[i] = 0;
    // the values past the last whole vector of each run (fewer than 8 each)
    const int ra = static_cast<int>(a.numel & 7), rb = static_cast<int>(b.numel & 7);
    if (t < ra) {
      const int64_t i = a.numel - ra + t;
      a.xq[i] = static_cast<uint8_t>(
          quant1(__uint_as_float(static_cast<uint32_t>(a.x[i]) << 16), qa.s, quant_recip(qa.s)));
    } else if (t >= 8 && t - 8 < rb) {
      const int64_t i = b.numel - rb + (t - 8);
      b.xq[i] = static_cast<uint8_t>(
          quant1(__uint_as_float(static_cast<uint32_t>(b.x[i]) << 16), qb.s, quant_recip(qb.s)));
    }
  }
  int j = 0;
  for (int64_t c = blockIdx.x; c < total; c += gridDim.x, ++j) {
    const int slot = j % kStagedStages;
    const uint32_t ph = (j / kStagedStages) & 1u;
    if (!mbar_wait_bounded_warp(&full[slot], ph, abort_flag, timeout_ns)) {
      if (lane == 0) {
        record_timeout(kSiteStagedFull);
        *abort_flag = 1;
      }
      break;
    }
    bool second;
    int64_t off;
    uint32_t bytes;
    staged_chunk(a, b, ca, c, second, off, bytes);
    const QuantBracket &q = second ? qb : qa;
    const uint4 *sv = reinterpret_cast<const uint4 *>(ring + slot * kStagedChunk);
    uint2 *ov = reinterpret_cast<uint2 *>((second ? b.xq : a.xq) + (off >> 1));
    const int nv = static_cast<int>(bytes >> 4);
    if (nv == kStagedChunk / 16) {
      static_assert(kStagedChunk / 16 == 2 * kStagedConsumers, "two vectors per thread");
      const uint4 v0 = sv[t], v1 = sv[t + kStagedConsumers];
      st_stream(ov + t, quant8_bracket(v0, q));
      st_stream(ov + t + kStagedConsumers, quant8_bracket(v1, q));
    } else {
      for (int i = t; i < nv; i += kStagedConsumers) st_stream(ov + i, quant8_bracket(sv[i], q));
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
}

// ------------------------------------------------------ SwiGLU -> FP8
// SiLU(g) u (1/s) in fp32, with e^-g written as 2^(-g log2 e) (the ex2.approx
// instruction) and the sigmoid as rcp.approx(1 + e^-g):
//   e = 2^(g * -log2 e);  r = 1 / (1 + e);  h = ((g * u) * (1/s)) * r
// every product and sum rounded to nearest.  The element-wise kernels and
// the fused GEMM epilogue run exactly these operations, so their codes agree
// bit for bit.
constexpr float kNegLog2e = -1.44269504088896341f;

// 1 / (1 + e^-x)
__device__ __forceinline__ float sigmoid_f(float x) {
  return rcp_approx(__fadd_rn(1.0f, ex2_approx(__fmul_rn(x, kNegLog2e))));
}

// SiLU(g) * u * inv_s
__device__ __forceinline__ float silu_mul_scaled(float g, float u, float inv_s) {
  return __fmul_rn(__fmul_rn(__fmul_rn(g, u), inv_s), sigmoid_f(g));
}

// SiLU(g) * u, unscaled (calibration maxima and the per-row scales)
__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fmul_rn(__fmul_rn(g, u), sigmoid_f(g));
}

// SwiGLU variant: g' sigmoid(alpha g') (u' + beta) * inv_s, with the clamp
// g' <= limit, |u'| <= limit when has_limit, and the offset only when beta !=
// 0.  With alpha = 1, beta = 0 and no limit this performs exactly
// silu_mul_scaled's operations (alpha * g == g), so the codes are identical.
struct SwigluParams {
  float alpha, beta, limit;
  int has_limit;
};

__device__ __forceinline__ float swiglu_mul_scaled(float g, float u, float inv_s,
                                                   const SwigluParams &p) {
  if (p.has_limit) {
    g = fminf(g, p.limit);
    u = fminf(fmaxf(u, -p.limit), p.limit);
  }
  const float up = p.beta != 0.0f ? __fadd_rn(u, p.beta) : u;
  return __fmul_rn(__fmul_rn(__fmul_rn(g, up), inv_s), sigmoid_f(__fmul_rn(p.alpha, g)));
}

__device__ __forceinline__ uint32_t swiglu_quant2(uint32_t g, uint32_t u, float inv_s,
                                                  const SwigluParams &p) {
  return cvt_e4m3x2(swiglu_mul_scaled(bf16_lo(g), bf16_lo(u), inv_s, p),
                    swiglu_mul_scaled(bf16_hi(g), bf16_hi(u), inv_s, p));
}

__device__ __forceinline__ uint2 swiglu_quant8(uint4 g, uint4 u, float inv_s,
                                               const SwigluParams &p) {
  uint2 o;
  o.x = pack4(swiglu_quant2(g.x, u.x, inv_s, p), swiglu_quant2(g.y, u.y, inv_s, p));
  o.y = pack4(swiglu_quant2(g.z, u.z, inv_s, p), swiglu_quant2(g.w, u.w, inv_s, p));
  return o;
}

// Register caps (both two-input SwiGLU kernels): the 16-byte form at six blocks
// per SM (40 registers instead of 64; four blocks before): 26.5 against 27.2 us
// at 4096 x 8192, the same within 0.3% at 4096 x 12288, on one box.  The wide
// form keeps the compiler's choice (0: no minimum); six blocks cost it 1-2%.
template <bool WIDE>
__global__ void __launch_bounds__(kEwThreads, WIDE ? 0 : 6) swiglu_2in_kernel(
    const uint16_t *__restrict__ g, const uint16_t *__restrict__ u, int64_t numel,
    const float *__restrict__ s_down, SwigluParams p, uint8_t *__restrict__ h) {
  pdl_launch_dependents();
  pdl_wait();
  const float inv_s = __frcp_rn(__ldg(s_down));
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t done = stream2<WIDE>(g, u, numel, h, tid, nthreads, [inv_s, p](uint4 a, uint4 b) {
    return swiglu_quant8(a, b, inv_s, p);
  });
  const int64_t t = done + tid;
  if (t < numel) {
    float a = __uint_as_float(static_cast<uint32_t>(g[t]) << 16);
    float b = __uint_as_float(static_cast<uint32_t>(u[t]) << 16);
    h[t] = static_cast<uint8_t>(cvt_e4m3x2(swiglu_mul_scaled(a, b, inv_s, p), 0.0f) & 0xFFu);
  }
}

// one 32-bit word (two BF16 values) of G and of U -> two codes
__device__ __forceinline__ uint32_t silu_quant2(uint32_t g, uint32_t u, float inv_s) {
  return cvt_e4m3x2(silu_mul_scaled(bf16_lo(g), bf16_lo(u), inv_s),
                    silu_mul_scaled(bf16_hi(g), bf16_hi(u), inv_s));
}

__device__ __forceinline__ uint2 silu_mul_quant8(uint4 g, uint4 u, float inv_s) {
  const float is = inv_s;
  uint2 o;
  o.x = pack4(silu_quant2(g.x, u.x, is), silu_quant2(g.y, u.y, is));
  o.y = pack4(silu_quant2(g.z, u.z, is), silu_quant2(g.w, u.w, is));
  return o;
}

template <bool WIDE>
__global__ void __launch_bounds__(kEwThreads, WIDE ? 0 : 6) silu_mul_2in_kernel(
    const uint16_t *__restrict__ g, const uint16_t *__restrict__ u, int64_t numel,
    const float *__restrict__ s_down, uint8_t *__restrict__ h) {
  pdl_launch_dependents();
  pdl_wait();
  const float inv_s = __frcp_rn(__ldg(s_down));
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t done = stream2<WIDE>(g, u, numel, h, tid, nthreads, [inv_s](uint4 a, uint4 b) {
    return silu_mul_quant8(a, b, inv_s);
  });
  const int64_t t = done + tid;
  if (t < numel) {
    float a = __uint_as_float(static_cast<uint32_t>(g[t]) << 16);
    float b = __uint_as_float(static_cast<uint32_t>(u[t]) << 16);
    h[t] = static_cast<uint8_t>(cvt_e4m3x2(silu_mul_scaled(a, b, inv_s), 0.0f) & 0xFFu);
  }
}

// -------------------------------------------------------- calibration
__device__ __forceinline__ float block_max(float m) {
  __shared__ float red[kEwThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (kEwThreads / 32) ? red[threadIdx.x] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  }
  return m;
}

__device__ __forceinline__ float absmax8(uint4 v, float m) {
  m = fmaxf(m, fabsf(bf16_lo(v.x)));
  m = fmaxf(m, fabsf(bf16_hi(v.x)));
  m = fmaxf(m, fabsf(bf16_lo(v.y)));
  m = fmaxf(m, fabsf(bf16_hi(v.y)));
  m = fmaxf(m, fabsf(bf16_lo(v.z)));
  m = fmaxf(m, fabsf(bf16_hi(v.z)));
  m = fmaxf(m, fabsf(bf16_lo(v.w)));
  m = fmaxf(m, fabsf(bf16_hi(v.w)));
  return m;
}

// *amax_bits must be zero before the launch; non-negative floats order like
// their bit patterns, so an unsigned atomicMax on the bits is a float max.
__global__ void __launch_bounds__(kEwThreads) absmax_bf16_kernel(
    const uint16_t *__restrict__ x, int64_t numel, unsigned int *__restrict__ amax_bits) {
  const int64_t nvec = numel >> 3;
  const uint4 *xv = reinterpret_cast<const uint4 *>(x);
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  float m = 0.0f;
  for (int64_t i = tid; i < nvec; i += stride) m = absmax8(ld_stream(xv + i), m);
  const int64_t t = (nvec << 3) + tid;
  if (t < numel) m = fmaxf(m, fabsf(__uint_as_float(static_cast<uint32_t>(x[t]) << 16)));
  m = block_max(m);
  if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(m));
}

__global__ void __launch_bounds__(kEwThreads) silu_mul_absmax_kernel(
    const uint16_t *__restrict__ g, const uint16_t *__restrict__ u, int64_t numel,
    unsigned int *__restrict__ amax_bits) {
  const int64_t nvec = numel >> 3;
  const uint4 *gv = reinterpret_cast<const uint4 *>(g);
  const uint4 *uv = reinterpret_cast<const uint4 *>(u);
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  float m = 0.0f;
  for (int64_t i = tid; i < nvec; i += stride) {
    uint4 a = ld_stream(gv + i), b = ld_stream(uv + i);
    m = fmaxf(m, fabsf(silu_mul(bf16_lo(a.x), bf16_lo(b.x))));
    m = fmaxf(m, fabsf(silu_mul(bf16_hi(a.x), bf16_hi(b.x))));
    m = fmaxf(m, fabsf(silu_mul(bf16_lo(a.y), bf16_lo(b.y))));
    m = fmaxf(m, fabsf(silu_mul(bf16_hi(a.y), bf16_hi(b.y))));
    m = fmaxf(m, fabsf(silu_mul(bf16_lo(a.z), bf16_lo(b.z))));
    m = fmaxf(m, fabsf(silu_mul(bf16_hi(a.z), bf16_hi(b.z))));
    m = fmaxf(m, fabsf(silu_mul(bf16_lo(a.w), bf16_lo(b.w))));
    m = fmaxf(m, fabsf(silu_mul(bf16_hi(a.w), bf16_hi(b.w))));
  }
  const int64_t t = (nvec << 3) + tid;
  if (t < numel) {
    float a = __uint_as_float(static_cast<uint32_t>(g[t]) << 16);
    float b = __uint_as_float(static_cast<uint32_t>(u[t]) << 16);
    m = fmaxf(m, fabsf(silu_mul(a, b)));
  }
  m = block_max(m);
  if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(m));
}

// Moving average of per-batch maxima in fp64, written without fused
// multiply-adds so that every step rounds exactly as the definition reads:
// A_1 = a_1, A_b = A_{b-1} + c (a_b - A_{b-1}); scale = fp32(A / 448).
__global__ void observer_scale_kernel(const float *__restrict__ amaxes, int nbatch, double c,
                                      float *__restrict__ scale) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  double A = static_cast<double>(amaxes[0]);
  for (int b = 1; b < nbatch; ++b)
    A = __dadd_rn(A, __dmul_rn(c, __dsub_rn(static_cast<double>(amaxes[b]), A)));
  *scale = __double2float_rn(__ddiv_rn(A, 448.0));
}

// RTN weight scale in place: s = amax / 448 (IEEE fp32 division).
__global__ void rtn_scale_kernel(float *__restrict__ s) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  *s = __fdiv_rn(*s, 448.0f);
}

}  // namespace fp8ws

// --------------------------------------------- per-token / per-channel rows
namespace fp8ws {

constexpr int kRowThreads = 256;       // threads per row of the per-token SwiGLU
constexpr int kQuantRowThreads = 128;  // threads per row of the per-token quantizer

template <int THREADS = kRowThreads>
__device__ __forceinline__ float block_max_rows(float m, float *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int w = 1; w < THREADS / 32; ++w) m = fmaxf(m, red[w]);
  return m;
}

// One block per row of a [rows, K] BF16 tensor (K % 8 == 0): s[r] = max|x| /
// 448 (1 for an all-zero row), codes q(x, s[r]) as the static quantizer.
// Per-token scales for activations, per-channel scales for weights.
// HELD: 8-element vectors per thread that a row may keep in registers (rows
// of up to kQuantRowThreads * HELD vectors take the single-read path).
template <int HELD>
__global__ void __launch_bounds__(kQuantRowThreads) quant_rows_kernel(
    const uint16_t *__restrict__ x, int K, float *__restrict__ s_out, uint8_t *__restrict__ q) {
  __shared__ float red[kQuantRowThreads / 32];
  pdl_launch_dependents();
  pdl_wait();
  const int64_t row = blockIdx.x;
  const uint4 *xv = reinterpret_cast<const uint4 *>(x + row * K);
  uint2 *qv = reinterpret_cast<uint2 *>(q + row * K);
  const int nvec = K >> 3;
  float m = 0.0f;
  if (nvec <= kQuantRowThreads * HELD) {
    // the whole row fits in the threads' registers: every load in flight at
    // once, and the quantization reuses the values instead of reading again
    uint4 v[HELD];
#pragma unroll
    for (int k = 0; k < HELD; ++k) {
      const int i = threadIdx.x + k * kQuantRowThreads;
      v[k] = i < nvec ? ld_stream(xv + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < HELD; ++k) m = absmax8(v[k], m);
    m = block_max_rows<kQuantRowThreads>(m, red);
    const float s = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
    const QuantBracket qb = quant_bracket(s);
    if (threadIdx.x == 0) s_out[row] = s;
#pragma unroll
    for (int k = 0; k < HELD; ++k) {
      const int i = threadIdx.x + k * kQuantRowThreads;
      if (i < nvec) st_stream(qv + i, quant8_bracket(v[k], qb));
    }
    return;
  }
  for (int i = threadIdx.x; i < nvec; i += kQuantRowThreads) m = absmax8(__ldg(xv + i), m);
  m = block_max_rows<kQuantRowThreads>(m, red);
  const float s = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
  const QuantBracket qb = quant_bracket(s);
  if (threadIdx.x == 0) s_out[row] = s;
  for (int i = threadIdx.x; i < nvec; i += kQuantRowThreads)
    qv[i] = quant8_bracket(__ldg(xv + i), qb);
}

// One block per row of G, U [rows, I] (I % 8 == 0, I <= kMaxRowI): v =
// SiLU(g) * u in fp32 kept in shared memory, s[r] = max|v| / 448 (1 for an
// all-zero row), h = E4M3(v * (1/s)).
constexpr int kMaxRowI = 16384;

// BATCH: vector pairs a thread loads before using the first.  The host takes
// BATCH = 6 for rows of 5 or 6 pairs per thread (8192 < I <= 12288), so that a
// row costs one memory round trip, and 4 otherwise (80 against 64 registers:
// three blocks per SM instead of four where one round trip is not reached
// anyway).  The batch of 4 is held to four blocks' registers (64; 26.9 against
// 27.5 us at 4096 x 8192 with the compiler's own 59); the batch of 6 to three
// blocks' (at 64 registers it spills: 56.7 against 41.0 us at 4096 x 12288).
template <int BATCH>
__global__ void __launch_bounds__(kRowThreads, BATCH == 4 ? 4 : 3) silu_mul_rows_kernel(
    const uint16_t *__restrict__ g, const uint16_t *__restrict__ u, int I,
    float *__restrict__ s_out, uint8_t *__restrict__ h) {
  extern __shared__ float vrow[];
  __shared__ float red[kRowThreads / 32];
  pdl_launch_dependents();
  pdl_wait();
  const int64_t row = blockIdx.x;
  const uint4 *gv = reinterpret_cast<const uint4 *>(g + row * I);
  const uint4 *uv = reinterpret_cast<const uint4 *>(u + row * I);
  const int nvec = I >> 3;
  float m = 0.0f;
  // BATCH vector pairs per thread are loaded before the first is used, so a
  // row costs one or two memory round trips instead of one per vector
  for (int base = threadIdx.x; base < nvec; base += kRowThreads * BATCH) {
    uint4 a[BATCH], b[BATCH];
#pragma unroll
    for (int k = 0; k < BATCH; ++k) {
      const int i = base + k * kRowThreads;
      if (i < nvec) {
        a[k] = ld_stream(gv + i);
        b[k] = ld_stream(uv + i);
      }
    }
#pragma unroll
    for (int k = 0; k < BATCH; ++k) {
      const int i = base + k * kRowThreads;
      if (i < nvec) {
        float v[8] = {silu_mul(bf16_lo(a[k].x), bf16_lo(b[k].x)),
                      silu_mul(bf16_hi(a[k].x), bf16_hi(b[k].x)),
                      silu_mul(bf16_lo(a[k].y), bf16_lo(b[k].y)),
                      silu_mul(bf16_hi(a[k].y), bf16_hi(b[k].y)),
                      silu_mul(bf16_lo(a[k].z), bf16_lo(b[k].z)),
                      silu_mul(bf16_hi(a[k].z), bf16_hi(b[k].z)),
                      silu_mul(bf16_lo(a[k].w), bf16_lo(b[k].w)),
                      silu_mul(bf16_hi(a[k].w), bf16_hi(b[k].w))};
        // v of vector i as two float4 planes (values 0-3 at i, 4-7 at nvec + i),
        // so that a warp's 16-byte shared-memory accesses are contiguous
        reinterpret_cast<float4 *>(vrow)[i] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4 *>(vrow)[nvec + i] = make_float4(v[4], v[5], v[6], v[7]);
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[e]));
      }
    }
  }
  m = block_max_rows(m, red);
  const float s = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
  const float inv = __frcp_rn(s);
  if (threadIdx.x == 0) s_out[row] = s;
  uint2 *hv = reinterpret_cast<uint2 *>(h + row * I);
  for (int i = threadIdx.x; i < nvec; i += kRowThreads) {
    const float4 lo = reinterpret_cast<const float4 *>(vrow)[i];
    const float4 hi = reinterpret_cast<const float4 *>(vrow)[nvec + i];
    uint2 o;
    o.x = pack4(cvt_e4m3x2(lo.x * inv, lo.y * inv), cvt_e4m3x2(lo.z * inv, lo.w * inv));
    o.y = pack4(cvt_e4m3x2(hi.x * inv, hi.y * inv), cvt_e4m3x2(hi.z * inv, hi.w * inv));
    st_stream(hv + i, o);
  }
}

}  // namespace fp8ws
