/*
 * fp8ws: static per-tensor FP8 E4M3 W8A8 Linear blocks for B200 (sm_100a).
 *
 * C ABI.  Plain pointers and sizes only; no CUDA or torch types appear in the
 * signatures.  `stream` is a cudaStream_t passed as void* (NULL = the legacy
 * default stream).
 *
 * Conventions for every entry point:
 *  - Return value: FP8WS_OK (0) or one of the FP8WS_ERR_* codes below.  No
 *    call aborts or throws.  Argument checks happen before any work is
 *    enqueued, so a call that returns an argument error has launched nothing.
 *  - Memory: the caller owns every buffer.  The hot-path calls allocate
 *    nothing, never synchronize the device and never read a scale on the host;
 *    they enqueue kernels on `stream` and return.
 *  - Tensors are dense and row-major ("contiguous").  BF16 data is passed as
 *    uint16_t bit patterns, FP8 E4M3 data as uint8_t codes, scales as pointers
 *    to one device fp32 value each.
 *  - Alignment: every tensor pointer must be 16-byte aligned
 *    (FP8WS_ERR_ALIGN otherwise).  A tensor with no elements (numel == 0,
 *    M == 0) may be passed as NULL; such a call succeeds and launches nothing.
 *    BF16 inputs that are 32-byte aligned let the quantizer and the SwiGLU
 *    kernels load 32 bytes at a time (faster on most lengths; the codes are
 *    the same either way).
 *  - FP8 E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; largest finite
 *    value 448; quantization divides by the scale, saturates to +-448 and
 *    rounds to nearest, ties to even.
 *  - Errors found inside a kernel (a bounded wait that ran out) are recorded
 *    in a device status word; fp8ws_device_status() reads and clears it.
 *  - The *_workspace functions return 0 for a negative size, and SIZE_MAX
 *    (which cannot be allocated) when the byte count does not fit in size_t:
 *    the count is formed without wrap-around, so no shape yields a small one.
 *
 * Sources of the operations (the pages this library implements):
 *  [MC] Hugging Face model card "Cosmos3-Nano-Policy-DROID, FP8 + RTN +
 *       moving-average activation observer (ModelOpt W8A8, per-tensor
 *       static)", Scheme table.
 *  [PR] TensorRT-LLM pull request "Load static FP8 Cosmos3 Nano/Super
 *       checkpoints without re-quantizing them", sections Description and
 *       What changed.
 *  [BLOG] "Running Cosmos 3 Robot Policies on a Single RTX 4090", section
 *       "Make it fit via quantization".
 */
#ifndef FP8WS_H
#define FP8WS_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FP8WS_API __attribute__((visibility("default")))
#else
#define FP8WS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  FP8WS_OK = 0,
  FP8WS_ERR_NULL = 1,           /* a required pointer is NULL */
  FP8WS_ERR_SHAPE = 2,          /* a size is negative, zero where not allowed, or unsupported */
  FP8WS_ERR_ALIGN = 3,          /* a pointer is not 16-byte aligned */
  FP8WS_ERR_SCALE_MISMATCH = 4, /* group members carry different input scales */
  FP8WS_ERR_BAD_SCALE = 5,      /* a scale is not finite or not > 0 */
  FP8WS_ERR_CUDA = 6,           /* a CUDA runtime call failed */
  FP8WS_ERR_DEVICE_TIMEOUT = 7, /* a bounded wait inside a kernel ran out */
  FP8WS_ERR_UNSUPPORTED = 8,    /* the current device is not sm_100 */
  FP8WS_ERR_WORKSPACE = 9       /* workspace NULL or misaligned */
};

/* ---------------------------------------------------------------- hot path */

/*
 * fp8_quant_static -- quantize an activation once with its static scale.
 * [MC] Scheme table (activations FP8 E4M3 with one static scale per tensor);
 * [PR] What changed (the shared activation is quantized once and handed to
 * every projection of the group).
 *
 *   xq[i] = E4M3_satRNE( fp32(x[i]) / s_in[0] )   (IEEE fp32 division)
 *
 * x: device, numel BF16 values, any rank, read as one flat run.
 * s_in: device, one fp32 value.
 * xq: device, numel FP8 codes (written).
 * numel >= 0 (0 launches nothing).
 * The codes are those of the IEEE quotient for every value of s_in, a zero or
 * subnormal scale included, whichever form of the kernel runs
 * (fp8ws_set_quant_form).
 */
FP8WS_API int fp8_quant_static(const uint16_t *x, int64_t numel, const float *s_in, uint8_t *xq,
                     void *stream);

/*
 * fp8_linear_static -- W8A8 Linear with the dequant in the GEMM epilogue.
 * [PR] What changed (each Linear applies its own scale in the GEMM epilogue;
 * split projections are contiguous Linear outputs); Description (static FP8
 * keeps one scale per projection).
 *
 *   y[m,n] = bf16_RN( (s_in[0]*s_w[0]) * sum_k deq(xq[m,k]) * deq(wq[n,k]) ),
 *   fp32 accumulation on the tensor cores.
 *
 * xq: device [M,K] FP8 codes, row-major.
 * wq: device [N,K] FP8 codes, row-major (the Linear's [out,in] weight).
 * s_in, s_w: device, one fp32 value each.
 * y: device [M,N] BF16, row-major, contiguous (row stride N).
 * Sizes: M >= 0 (0 launches nothing), N >= 8 with N % 8 == 0, K >= 16 with
 * K % 16 == 0; M, N, K < 2^31.
 * Tiling: 256 x 256 tiles on CTA pairs (one-CTA tiles where a cost model finds
 * them faster); when the tiles past the last full wave of pairs would fill
 * at most half a wave, each of them runs as two 256 x 128 halves over the
 * full K, which gives the same result per element.  fp8ws_split_plan reports
 * the plan for a shape.
 */
FP8WS_API int fp8_linear_static(const uint8_t *xq, const uint8_t *wq, int64_t M, int64_t N, int64_t K,
                      const float *s_in, const float *s_w, uint16_t *y, void *stream);

/*
 * fp8_linear_static_ws -- fp8_linear_static with a scratch workspace that lets
 * the tiles past the last full wave of CTA pairs be split over K (2..4 ranges,
 * chosen from the shape and the number of resident CTA pairs), so the GPU is
 * not left partly idle by a ragged last wave.  Tiles of fewer than 64 K steps
 * of 128 bytes (ceil(K / 128) < 64, i.e. K <= 8064 for the multiples of 16
 * allowed here) are never split: there the split's fixed cost exceeds the
 * time it saves.  Each split stores an fp32 partial in the workspace; the last
 * split of a tile to finish adds the partials in split order (deterministic:
 * the same inputs give the same bits on every call) and applies the epilogue.
 * The sum may differ from the unsplit kernel's in the last bits of fp32, well
 * inside the GEMM tolerance.  It pays only when few tiles remain past the last
 * full wave and K is long: on a single tower's down projection (48 or 192
 * tiles of 256 x 256 for 74 CTA pairs, K = 12288) the partial traffic and
 * reduction cost more than the idle tail they remove, so the single-tower
 * composite calls do not use it; the grouped down projection of both towers
 * (240 tiles, 18 past the third wave) does.  fp8ws_split_plan reports the
 * plan for a shape.
 * workspace: device, >= fp8_linear_static_ws_bytes() bytes, 256-byte aligned;
 * overwritten (the call clears its counters first).  Other arguments and
 * errors as fp8_linear_static; FP8WS_ERR_WORKSPACE for a missing, misaligned
 * or short workspace.
 */
FP8WS_API size_t fp8_linear_static_ws_bytes(void);
FP8WS_API int fp8_linear_static_ws(const uint8_t *xq, const uint8_t *wq, int64_t M, int64_t N,
                                   int64_t K, const float *s_in, const float *s_w, uint16_t *y,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * silu_mul_2in_fp8 -- two-input SwiGLU quantized straight to FP8 for the
 * down projection.  [PR] What changed (SiLU(G)*U from two separate tensors,
 * quantized directly for the FP8 down_proj; flat indexing over a 1-D grid, so
 * any rank works; strided inputs are refused, not copied).
 *
 *   h[i] = E4M3_satRNE( SiLU(g[i]) * u[i] / s_down[0] ),  SiLU(g) = g/(1+e^-g),
 *   computed in fp32 (fast exp and reciprocal; the result may differ from an
 *   exact evaluation by one E4M3 step on values within rounding noise of a
 *   code boundary).
 *
 * g, u: device, numel BF16 values each, contiguous.  s_down: device fp32.
 * h: device, numel FP8 codes.  numel >= 0.
 */
FP8WS_API int silu_mul_2in_fp8(const uint16_t *g, const uint16_t *u, int64_t numel, const float *s_down,
                     uint8_t *h, void *stream);

/*
 * SwiGLU variants.  [PR] commit notes on the two-input SwiGLU: the activation
 * may carry swiglu_alpha (a gain inside the sigmoid), swiglu_beta (an offset
 * on up) and swiglu_limit; omitting all of them is plain SwiGLU.  The limit is
 * read as the clamp of the "swigluoai" shape: gate <= limit and
 * -limit <= up <= limit.
 *
 *   h = E4M3_satRNE( g' * sigmoid(alpha * g') * (u' + beta) / s_down )
 *
 * A NULL descriptor, or alpha = 1, beta = 0, has_limit = 0, gives exactly the
 * results of silu_mul_2in_fp8.  alpha and beta must be finite and limit > 0
 * when has_limit (FP8WS_ERR_BAD_SCALE otherwise).
 */
typedef struct {
  float alpha;
  float beta;
  float limit;
  int32_t has_limit;
} fp8ws_swiglu;

/* swiglu_2in_fp8 -- silu_mul_2in_fp8 with an optional variant descriptor. */
FP8WS_API int swiglu_2in_fp8(const uint16_t *g, const uint16_t *u, int64_t numel,
                             const float *s_down, const fp8ws_swiglu *act, uint8_t *h,
                             void *stream);

/*
 * gated_mlp_static_fp8 -- the split gated MLP on the static FP8 path.
 * [PR] What changed (GatedMLP with split gate/up: quantize the shared
 * activation once, hand the FP8 tensor to both projections, two-input SwiGLU
 * to FP8, FP8 down projection).
 *
 *   Xq = fp8_quant_static(x, s_in)
 *   G  = fp8_linear_static(Xq, Wg, s_in, s_wg)      [M,I] BF16
 *   U  = fp8_linear_static(Xq, Wu, s_in, s_wu)      [M,I] BF16
 *   H  = silu_mul_2in_fp8(G, U, s_down)             [M,I] FP8
 *   y  = fp8_linear_static(H, Wd, s_down, s_wd)     [M,d] BF16
 *
 * Gate and up share s_in; fp8_check_shared_input_scale proves at load time
 * that their calibrated input scales are equal.
 * x: device [M,d] BF16.  Wg, Wu: device [I,d] FP8.  Wd: device [d,I] FP8.
 * workspace: device, at least gated_mlp_static_fp8_workspace(M,d,I) bytes,
 * 256-byte aligned; holds Xq, G, U and H (in that order, each region 256-byte
 * aligned) and is overwritten.  y: device [M,d] BF16.
 * Sizes: as fp8_linear_static for (M, I, d) and (M, d, I).
 */
FP8WS_API size_t gated_mlp_static_fp8_workspace(int64_t M, int64_t d, int64_t I);
FP8WS_API int gated_mlp_static_fp8(const uint16_t *x, int64_t M, int64_t d, int64_t I, const float *s_in,
                         const uint8_t *Wg, const float *s_wg, const uint8_t *Wu,
                         const float *s_wu, const float *s_down, const uint8_t *Wd,
                         const float *s_wd, void *workspace, uint16_t *y, void *stream);

/*
 * fp8_gate_up_swiglu_static -- gate and up projections and the two-input
 * SwiGLU-quant in one kernel (the fusion of fp8_linear_static x 2 and
 * silu_mul_2in_fp8 on the MLP path; [PR] What changed describes the three
 * steps, this call runs them without writing G and U to memory).
 *
 *   G = bf16((s_in*s_wg) . Xq Wg^T),  U = bf16((s_in*s_wu) . Xq Wu^T)   (kept on chip)
 *   h = E4M3_satRNE( SiLU(G) * U / s_down )   in fp32 as silu_mul_2in_fp8
 *
 * Bit-identical to fp8_linear_static (gate), fp8_linear_static (up) and
 * silu_mul_2in_fp8 run one after the other on the same inputs.
 * xq: device [M,K] FP8.  Wg, Wu: device [I,K] FP8.  Scales: device fp32.
 * act: SwiGLU variant (NULL = plain), as swiglu_2in_fp8.
 * h: device [M,I] FP8.  Sizes: as fp8_linear_static with N = I, and I % 16 == 0.
 */
FP8WS_API int fp8_gate_up_swiglu_static(const uint8_t *xq, const uint8_t *Wg, const uint8_t *Wu,
                                        int64_t M, int64_t I, int64_t K, const float *s_in,
                                        const float *s_wg, const float *s_wu,
                                        const float *s_down, const fp8ws_swiglu *act,
                                        uint8_t *h, void *stream);

/*
 * gated_mlp_static_fp8_fused -- gated_mlp_static_fp8 with the gate/up GEMMs
 * and the SwiGLU-quant fused (fp8_gate_up_swiglu_static): three launches
 * (quantize X, fused gate/up/SwiGLU, down GEMM) instead of five, and no G or U
 * round trip through memory.  Same result, bit for bit.
 * workspace: device, gated_mlp_static_fp8_fused_workspace(M,d,I) bytes,
 * 256-byte aligned; holds Xq [M,d] then H [M,I] (each region 256-byte
 * aligned).  act: SwiGLU variant (NULL = plain).  Other arguments as
 * gated_mlp_static_fp8.
 */
FP8WS_API size_t gated_mlp_static_fp8_fused_workspace(int64_t M, int64_t d, int64_t I);
FP8WS_API int gated_mlp_static_fp8_fused(const uint16_t *x, int64_t M, int64_t d, int64_t I,
                                         const float *s_in, const uint8_t *Wg, const float *s_wg,
                                         const uint8_t *Wu, const float *s_wu,
                                         const float *s_down, const fp8ws_swiglu *act,
                                         const uint8_t *Wd, const float *s_wd, void *workspace,
                                         uint16_t *y, void *stream);

/* ------------------------------------------------- grouped (two-tower) calls
 *
 * A Mixture-of-Transformers decoder layer has two towers, an understanding and
 * a generation branch, with the same Linear shapes but their own token counts,
 * weights and calibrated scales ([BLOG] Make it fit via quantization: the two
 * branches are quantized separately; [MC] Scheme table: one static scale per
 * tensor).  A grouped call runs the same step for up to FP8WS_MAX_GROUP such
 * problems in ONE kernel launch: their tiles form one sequence dealt to the
 * persistent CTAs, so the smaller tower fills the last, partly idle wave of
 * the larger one.  Each problem's result is the one the single-problem call
 * gives, bit for bit (the split-K variant excepted, as fp8_linear_static_ws).
 * Problems with no rows (M == 0, numel == 0) are skipped and may carry NULL
 * tensor pointers.  count: 1..FP8WS_MAX_GROUP (FP8WS_ERR_SHAPE otherwise).
 * The problem arrays live in host memory and are read during the call only.
 */
#define FP8WS_MAX_GROUP 2

typedef struct {
  const uint16_t *x; /* device, numel BF16 values */
  int64_t numel;     /* >= 0 */
  const float *s_in; /* device fp32 scale of this tensor */
  uint8_t *xq;       /* device, numel FP8 codes (written) */
} fp8ws_quant_problem;

typedef struct {
  const uint8_t *xq; /* device [M,K] FP8 */
  const uint8_t *wq; /* device [N,K] FP8 */
  int64_t M;         /* >= 0 */
  const float *s_in; /* device fp32 */
  const float *s_w;  /* device fp32 */
  uint16_t *y;       /* device [M,N] BF16 (written) */
} fp8ws_linear_problem;

typedef struct {
  const uint8_t *xq;   /* device [M,K] FP8 */
  const uint8_t *Wg;   /* device [I,K] FP8 */
  const uint8_t *Wu;   /* device [I,K] FP8 */
  int64_t M;           /* >= 0 */
  const float *s_in;   /* device fp32, shared by gate and up */
  const float *s_wg;   /* device fp32 */
  const float *s_wu;   /* device fp32 */
  const float *s_down; /* device fp32, down_proj's input scale */
  uint8_t *h;          /* device [M,I] FP8 (written) */
} fp8ws_gate_up_problem;

typedef struct {
  const uint16_t *x;   /* device [M,d] BF16 */
  int64_t M;           /* >= 0 */
  const float *s_in;   /* device fp32, gate/up input scale */
  const uint8_t *Wg;   /* device [I,d] FP8 */
  const float *s_wg;
  const uint8_t *Wu;   /* device [I,d] FP8 */
  const float *s_wu;
  const float *s_down; /* device fp32, down_proj's input scale */
  const uint8_t *Wd;   /* device [d,I] FP8 */
  const float *s_wd;
  uint16_t *y;         /* device [M,d] BF16 (written) */
} fp8ws_mlp_tower;

/*
 * fp8_quant_static_group -- fp8_quant_static for count activations, each
 * with its own scale, in one launch.  Errors as fp8_quant_static.
 */
FP8WS_API int fp8_quant_static_group(const fp8ws_quant_problem *problems, int count,
                                     void *stream);

/*
 * fp8_linear_static_group -- fp8_linear_static for count problems sharing N
 * and K, in one CTA-pair launch when the tile cost model picks CTA pairs for
 * the group's combined tiles, else one launch per problem.
 * workspace: NULL (no split), or >= fp8_linear_static_ws_bytes() bytes,
 * 256-byte aligned, for splitting the tiles of the group's last partial wave
 * over K as fp8_linear_static_ws does (deterministic; the call clears its
 * counters first).  Sizes and errors as fp8_linear_static, per problem;
 * FP8WS_ERR_WORKSPACE for a misaligned or short workspace.
 */
FP8WS_API int fp8_linear_static_group(const fp8ws_linear_problem *problems, int count,
                                      int64_t N, int64_t K, void *workspace,
                                      size_t workspace_bytes, void *stream);

/*
 * fp8_gate_up_swiglu_static_group -- fp8_gate_up_swiglu_static for count
 * problems sharing I and K (each with its own rows, weights and scales) in
 * one launch; act (NULL = plain SwiGLU) applies to all.  Bit-identical per
 * problem to fp8_gate_up_swiglu_static.  Sizes and errors as that call.
 */
FP8WS_API int fp8_gate_up_swiglu_static_group(const fp8ws_gate_up_problem *problems, int count,
                                              int64_t I, int64_t K, const fp8ws_swiglu *act,
                                              void *stream);

/*
 * gated_mlp_static_fp8_group -- gated_mlp_static_fp8_fused for the towers of
 * one decoder layer (shared d and I) in three launches in all:
 * fp8_quant_static_group, fp8_gate_up_swiglu_static_group and
 * fp8_linear_static_group (down projections; split-K scratch in the
 * workspace).  Each tower's y equals gated_mlp_static_fp8_fused's for that
 * tower within the GEMM tolerance; with no tile of the down group split over
 * K (the plan splits only a ragged last wave) the two are identical bit for
 * bit.
 * workspace: device, gated_mlp_static_fp8_group_workspace(M, count, d, I)
 * bytes, 256-byte aligned; holds Xq and H of each tower and the split-K
 * scratch, and is overwritten.  M: host array of the towers' row counts.
 * Sizes: as gated_mlp_static_fp8_fused per tower.
 */
FP8WS_API size_t gated_mlp_static_fp8_group_workspace(const int64_t *M, int count, int64_t d,
                                                      int64_t I);
FP8WS_API int gated_mlp_static_fp8_group(const fp8ws_mlp_tower *towers, int count, int64_t d,
                                         int64_t I, const fp8ws_swiglu *act, void *workspace,
                                         size_t workspace_bytes, void *stream);

/*
 * qkv_shared_quant -- Q/K/V projections from one shared quantization.
 * [PR] What changed (Attention with shared Q/K/V input quantization: the
 * activation is quantized once for all three projections; each projection
 * writes its own contiguous output).
 *
 * x: device [M,d] BF16.  Wq [Nq,d], Wk [Nk,d], Wv [Nv,d]: device FP8.
 * workspace: device, at least qkv_shared_quant_workspace(M,d) bytes, 256-byte
 * aligned: Xq [M,d], then scratch for splitting the ragged last wave of the
 * projection GEMMs over K (as fp8_linear_static_ws).  q [M,Nq], k [M,Nk],
 * v [M,Nv]: device BF16, contiguous.  The three projections run as one
 * grouped GEMM launch (their tiles dealt as one sequence, each projection
 * with its own weight, scale and output).  Cross-attention, where K/V come
 * from another tensor, must not use this call.
 */
FP8WS_API size_t qkv_shared_quant_workspace(int64_t M, int64_t d);
FP8WS_API int qkv_shared_quant(const uint16_t *x, int64_t M, int64_t d, const float *s_in,
                     const uint8_t *Wq, int64_t Nq, const float *s_wq, const uint8_t *Wk,
                     int64_t Nk, const float *s_wk, const uint8_t *Wv, int64_t Nv,
                     const float *s_wv, void *workspace, uint16_t *q, uint16_t *k, uint16_t *v,
                     void *stream);

/*
 * gated_mlp_static_fp8_noalloc -- the same gated MLP as gated_mlp_static_fp8,
 * for callers that cannot allocate device memory when they call it.  The pages
 * have no counterpart to this entry point; it exists for the caller, not the
 * method.
 *
 * Who needs it: code whose device memory is fixed before it runs, so that a
 * workspace cannot be obtained per call -- a plugin inside an inference engine
 * whose enqueue step may not allocate, or a process that hands all device
 * memory to its own pool at start-up (a robot's policy server, say), where a
 * cudaMalloc would fail or stall the control loop.
 *
 * Instead of a caller-supplied workspace, the call uses one scratch area that
 * the library reserves as a static device array of
 * FP8WS_NOALLOC_SCRATCH_BYTES (64 MiB) on every GPU that loads the library,
 * held until the process exits.  The call itself allocates nothing: no
 * cudaMalloc, no cudaFree, no allocating library routine.
 *
 * Limits and behaviour:
 *  - The rule is gated_mlp_static_fp8_workspace(M, d, I) <=
 *    FP8WS_NOALLOC_SCRATCH_BYTES; larger shapes are refused with
 *    FP8WS_ERR_SHAPE before any launch.  That workspace is
 *    M * (d + 5 I) bytes, each of its four regions rounded up to 256 bytes,
 *    so for d = 3072, I = 12288 it allows up to M = 1040 rows (1040 * 64512 =
 *    67,092,480 bytes).  Shapes gated_mlp_static_fp8 refuses (d or I not a
 *    positive multiple of 16, a size of 2^31 or more) are refused here with
 *    FP8WS_ERR_SHAPE too, before the size is formed, so no shape can wrap the
 *    byte count into the limit.
 *  - The first call on each device looks up the scratch area's device
 *    address on that device (cudaGetSymbolAddress, with the device current);
 *    make that first call before any stream capture.
 *  - When the array is reserved: under CUDA's lazy module loading (the
 *    default), the library's module -- its kernels and this 64 MiB array --
 *    is loaded onto a device at the library's first use of that device, and
 *    that may be this entry point's first call.  A caller that hands all
 *    device memory to its own pool at start-up must therefore make one call
 *    on each device before it builds the pool (a call with M = 0 and the
 *    weight and scale pointers of the later calls does the set-up and
 *    launches nothing), or run with CUDA_MODULE_LOADING=EAGER so that the
 *    array is reserved when the library is loaded; otherwise that first call
 *    can fail with FP8WS_ERR_CUDA (out of memory).
 *  - Every call on a device shares the one scratch area, which keeps the
 *    previous call's contents.  Each call overwrites every byte it reads, so
 *    nothing needs clearing, but calls that overlap on the GPU (different
 *    streams without ordering, or different host threads) race on the scratch
 *    and give wrong results.  Order them on one stream.
 * Arguments are those of gated_mlp_static_fp8 without the workspace.
 */
#define FP8WS_NOALLOC_SCRATCH_BYTES (64ull * 1024 * 1024)
FP8WS_API int gated_mlp_static_fp8_noalloc(const uint16_t *x, int64_t M, int64_t d, int64_t I,
                                           const float *s_in, const uint8_t *Wg,
                                           const float *s_wg, const uint8_t *Wu,
                                           const float *s_wu, const float *s_down,
                                           const uint8_t *Wd, const float *s_wd, uint16_t *y,
                                           void *stream);

/*
 * fp8_shared_quant_linears -- quantize one activation once and run n Linears
 * on that single FP8 copy (the general form of qkv_shared_quant; with n = 1 it
 * is a standalone projection such as o_proj).  [PR] What changed: members of
 * a formerly fused group consume one quantized activation, which is only
 * sound while their calibrated input scales agree (checked at load with
 * fp8_check_shared_input_scale).
 *
 * x: device [M,d] BF16.  n: 1..FP8WS_MAX_PROJECTIONS.  W, N, s_w, y: host
 * arrays of n entries: device [N[i],d] FP8 weights, output widths, device fp32
 * weight scales and device [M,N[i]] BF16 outputs (each contiguous).
 * workspace: device, fp8_shared_quant_linears_workspace(M,d) bytes, 256-byte
 * aligned: Xq [M,d], then the split-K scratch of the projection GEMMs.  The
 * projections run in grouped GEMM launches of up to three.
 */
#define FP8WS_MAX_PROJECTIONS 16
FP8WS_API size_t fp8_shared_quant_linears_workspace(int64_t M, int64_t d);
FP8WS_API int fp8_shared_quant_linears(const uint16_t *x, int64_t M, int64_t d, const float *s_in,
                                       int n, const uint8_t *const *W, const int64_t *N,
                                       const float *const *s_w, uint16_t *const *y,
                                       void *workspace, void *stream);

/*
 * fp8_linears_static -- n Linears over one activation that the caller has
 * already quantized at s_in (with fp8_quant_static, or with a kernel of its
 * own that writes the same codes): fp8_shared_quant_linears without its
 * quantize launch.  [PR] What changed: the members of a formerly fused group
 * consume one quantized activation; their calibrated input scales must agree
 * (fp8_check_shared_input_scale).  The projections run in grouped GEMM
 * launches of up to three (Q, K and V in one launch).
 * xq: device [M,K] FP8.  s_in: device fp32.  W, N, s_w, y: host arrays of n
 * (1..FP8WS_MAX_PROJECTIONS): W[i] device [N[i],K] FP8, s_w[i] device fp32,
 * y[i] device [M,N[i]] BF16, contiguous.
 * workspace: NULL (no split over K), or device, >= fp8_linear_static_ws_bytes()
 * bytes, 256-byte aligned, which lets the tiles past the last full wave of a
 * long-K launch split over K as in fp8_linear_static_ws (the call clears its
 * counters first).
 * Errors: those of fp8_linear_static for each projection, FP8WS_ERR_SHAPE for
 * n out of range, FP8WS_ERR_NULL for a NULL host array, FP8WS_ERR_WORKSPACE
 * for a misaligned or short workspace; all found before anything is enqueued.
 */
FP8WS_API int fp8_linears_static(const uint8_t *xq, int64_t M, int64_t K, const float *s_in,
                                 int n, const uint8_t *const *W, const int64_t *N,
                                 const float *const *s_w, uint16_t *const *y, void *workspace,
                                 size_t workspace_bytes, void *stream);

/*
 * cross_attention_qkv_static_fp8 -- projections of a cross-attention: Q from
 * the query-side activation x, K and V from a different tensor ctx.  [PR] Test
 * Coverage: where K/V come from another tensor, sharing must not engage
 * between Q and K/V.  So x is quantized with its own s_q for Q, and ctx is
 * quantized once with s_kv and shared by K and V (whose calibrated input
 * scales must agree).
 * x: device [Mq,d] BF16; ctx: device [Mkv,d] BF16; Wq [Nq,d], Wk [Nk,d],
 * Wv [Nv,d] FP8; q [Mq,Nq], k [Mkv,Nk], v [Mkv,Nv] BF16, contiguous.
 * workspace: cross_attention_qkv_static_fp8_workspace(Mq,Mkv,d) bytes,
 * 256-byte aligned: Xq [Mq,d], the quantized context [Mkv,d], then the
 * split-K scratch.  Two launches: one quantize for both inputs, one grouped
 * GEMM for Q, K and V.
 */
FP8WS_API size_t cross_attention_qkv_static_fp8_workspace(int64_t Mq, int64_t Mkv, int64_t d);
FP8WS_API int cross_attention_qkv_static_fp8(const uint16_t *x, int64_t Mq, const uint16_t *ctx,
                                             int64_t Mkv, int64_t d, const float *s_q,
                                             const uint8_t *Wq, int64_t Nq, const float *s_wq,
                                             const float *s_kv, const uint8_t *Wk, int64_t Nk,
                                             const float *s_wk, const uint8_t *Wv, int64_t Nv,
                                             const float *s_wv, void *workspace, uint16_t *q,
                                             uint16_t *k, uint16_t *v, void *stream);

/* ----------------------------------- per-channel / per-token scales (rows) */

/*
 * The finer-grained FP8 scheme of the exploratory builds ([MC] comparison
 * report, table 3.2: per-channel weight, per-token activation scales).
 *
 * fp8_quant_per_token -- one scale per row of x [rows,K] BF16 (K % 8 == 0),
 *   computed at run time: s[r] = max_k |x[r,k]| / 448 (IEEE fp32; 1 for an
 *   all-zero row), xq[r,k] = E4M3_satRNE(x[r,k] / s[r]).  For activations the
 *   rows are tokens; for weights [N,K] the rows are output channels (per-channel
 *   RTN).  s: device, rows fp32 (written).  xq: device [rows,K] FP8.
 * fp8_linear_scaled -- fp8_linear_static with vector scales:
 *   y[m,n] = bf16( sx * sw * sum_k deq(xq[m,k]) deq(wq[n,k]) ), where sx is
 *   s_x[m] if x_per_row else s_x[0], and sw is s_w[n] if w_per_col else s_w[0].
 * silu_mul_2in_fp8_per_token -- SiLU(G) * U quantized with one scale per row,
 *   computed at run time: v = SiLU(g) * u in fp32, s[r] = max |v| / 448 (1 for
 *   an all-zero row), h = E4M3_satRNE(v / s[r]).  G, U: device [rows,I] BF16,
 *   I % 8 == 0, I <= 16384.  s: device, rows fp32 (written).  h: [rows,I] FP8.
 * gated_mlp_per_token_fp8 -- the gated MLP on this scheme: per-token X
 *   quantization, gate and up GEMMs with (per-token x per-channel) scales in
 *   one grouped launch, per-token SwiGLU quantization, down GEMM likewise:
 *   four launches.  s_wg, s_wu: device [I]
 *   fp32, s_wd: device [d] fp32 (per-channel).  workspace:
 *   gated_mlp_per_token_fp8_workspace(M,d,I) bytes, 256-byte aligned:
 *   Xq [M,d] | s_x [M] | G [M,I] | U [M,I] | H [M,I] | s_h [M], each region
 *   256-byte aligned.
 */
FP8WS_API int fp8_quant_per_token(const uint16_t *x, int64_t rows, int64_t K, float *s,
                                  uint8_t *xq, void *stream);
FP8WS_API int fp8_linear_scaled(const uint8_t *xq, const uint8_t *wq, int64_t M, int64_t N,
                                int64_t K, const float *s_x, int x_per_row, const float *s_w,
                                int w_per_col, uint16_t *y, void *stream);
FP8WS_API int silu_mul_2in_fp8_per_token(const uint16_t *g, const uint16_t *u, int64_t rows,
                                         int64_t I, float *s, uint8_t *h, void *stream);
FP8WS_API size_t gated_mlp_per_token_fp8_workspace(int64_t M, int64_t d, int64_t I);
FP8WS_API int gated_mlp_per_token_fp8(const uint16_t *x, int64_t M, int64_t d, int64_t I,
                                      const uint8_t *Wg, const float *s_wg, const uint8_t *Wu,
                                      const float *s_wu, const uint8_t *Wd, const float *s_wd,
                                      void *workspace, uint16_t *y, void *stream);

/* ------------------------------------------------------------- load time */

/*
 * fp8_check_shared_input_scale -- the invariant that shared quantization rests
 * on: every member of a group carries the same calibrated input scale.
 * [PR] What changed (post_load_weights validates it at load, never in forward,
 * because reading a scale on the host synchronizes the device).
 *
 * d_scales: host array of n device pointers, each to one fp32 input scale.
 * n >= 1.  Copies the n values to the host (synchronizes `stream`) and returns
 * FP8WS_OK if all are finite, > 0 and bitwise equal; FP8WS_ERR_BAD_SCALE if
 * one is not finite or not > 0; FP8WS_ERR_SCALE_MISMATCH if two differ.
 */
FP8WS_API int fp8_check_shared_input_scale(const float *const *d_scales, int n, void *stream);

/*
 * Calibration helpers (load time; asynchronous on `stream`).
 * [MC] Scheme table: RTN weights with one scale per tensor; activation scales
 * from the MOVING_AVERAGE_MINMAX observer with averaging constant 0.01.
 *
 * fp8_absmax_bf16: amax[0] = max |x[i]| over numel BF16 values (exact; NaN
 *   values are ignored; 0 for numel == 0).  amax: device fp32, overwritten.
 * fp8_silu_mul_absmax: amax[0] = max |SiLU(g[i]) * u[i]| in fp32.
 * fp8_observer_scale: A_1 = amaxes[0], A_b = A_{b-1} + c (amaxes[b-1] -
 *   A_{b-1}) in fp64 (no fused multiply-add), then scale[0] = fp32(A / 448).
 *   amaxes: device, nbatch fp32 values; nbatch >= 1.
 * fp8_rtn_quantize_weight: s_w[0] = fp32(max|w|) / 448 (fp32 division), then
 *   wq = fp8_quant_static(w, s_w).  w: device numel BF16; wq: numel FP8.
 */
FP8WS_API int fp8_absmax_bf16(const uint16_t *x, int64_t numel, float *amax, void *stream);
FP8WS_API int fp8_silu_mul_absmax(const uint16_t *g, const uint16_t *u, int64_t numel, float *amax,
                        void *stream);
FP8WS_API int fp8_observer_scale(const float *amaxes, int nbatch, double c, float *scale, void *stream);
FP8WS_API int fp8_rtn_quantize_weight(const uint16_t *w, int64_t numel, float *s_w, uint8_t *wq,
                            void *stream);

/* ------------------------------------------------------------ diagnostics */

/* Human-readable name of a status code (static string). */
FP8WS_API const char *fp8ws_status_string(int status);

/* FP8WS_OK if the current device is sm_100 (B200), FP8WS_ERR_UNSUPPORTED
 * otherwise, FP8WS_ERR_CUDA if no device can be queried. */
FP8WS_API int fp8ws_device_check(void);

/* Read and clear the device status word of the current device (synchronizes
 * the device).  *status receives FP8WS_OK or FP8WS_ERR_DEVICE_TIMEOUT;
 * *where receives a code naming the wait that ran out (0 if none): in the
 * GEMMs 1 (producer, free stage), 2 (MMA, loaded stage), 3 (MMA, free
 * accumulator), 4 (epilogue, finished accumulator), 5 (teardown, last MMAs);
 * 6 the self-test below; in the staged quantizer 7 (consumers, loaded chunk),
 * 8 (producer, free slot). */
FP8WS_API int fp8ws_device_status(int *status, int *where);

/* Self-test of the bounded waits every GEMM kernel uses (failure detection
 * without a GPU fault): one small kernel waits on an mbarrier that nothing
 * arrives at.  mode 0: the wait runs out after limit_ns, the kernel records
 * wait site 6 in the device status word (read it with fp8ws_device_status)
 * and returns.  mode 1: a second warp raises the kernel's abort flag after
 * limit_ns / 4; the wait returns then and records nothing.  Synchronizes
 * `stream`; *elapsed_ns (host) receives how long the wait took, measured on
 * the device.  limit_ns: 1 .. 4e9 (FP8WS_ERR_SHAPE otherwise). */
FP8WS_API int fp8ws_selftest_bounded_wait(int64_t limit_ns, int mode, int64_t *elapsed_ns,
                                          void *stream);

/* Tile configuration of fp8_linear_static and of the down projection of the
 * gated MLPs, for tuning and tests: 0 = chosen per shape by the cost model
 * (default), 1 = CTA-pair 256x256 tiles, 2/3/4 = one CTA with 128x256,
 * 128x128 or 128x64 tiles.  Applies to later calls from every thread;
 * FP8WS_ERR_SHAPE for other values. */
FP8WS_API int fp8ws_set_gemm_config(int config);

/* Form of the static quantizer (fp8_quant_static and the quantization step
 * of every composite call), for tests and timing; the codes are the same in
 * every form.  0 = by size (default): the streaming kernels for BF16 inputs
 * smaller than 1.5 times L2, the staged kernel from there up.  1 = staged: one CTA per SM,
 * input chunks streamed into a shared-memory ring by the bulk copy engine.
 * 2 = streaming: each thread loads its own vectors (32 bytes at a time for
 * 32-byte-aligned inputs).  FP8WS_QUANT=staged or =stream in the environment
 * sets the starting value.  Applies to later calls from every thread;
 * FP8WS_ERR_SHAPE for other values. */
FP8WS_API int fp8ws_set_quant_form(int form);

/* The tile configuration the GEMM cost model picks, for tests and tuning;
 * host only, touches no device, ignores a configuration forced by
 * fp8ws_set_gemm_config.  Problems: M[p] x N[p] outputs for p < count (1..3,
 * the most one launch groups: the projections of one shared quantization), on
 * a GPU with `sms` SMs holding `pairs` CTA pairs at once.  *config receives
 * fp8ws_set_gemm_config's numbering: 1 CTA-pair 256x256 tiles, 2/3/4 one CTA
 * with 128x256, 128x128 or 128x64 tiles.  FP8WS_ERR_NULL for a NULL pointer,
 * FP8WS_ERR_SHAPE for sms < 1, pairs < 1, count outside 1..3, M < 0 or N < 1. */
FP8WS_API int fp8ws_gemm_plan(int sms, int pairs, const int64_t *M, const int64_t *N, int count,
                              int *config);

/* The plan of the CTA-pair GEMM for the tiles past its last full wave, for
 * tests and tuning; host only, touches no device.  For `tiles` 256x256 tiles
 * on `pairs` resident CTA pairs with `num_kb` 128-byte K steps per tile, with
 * split-K scratch (has_scratch != 0: fp8_linear_static_ws and the composite
 * calls that carry scratch) or without: the first *dp_tiles tiles run whole,
 * and each of the last *split_tiles is either cut into *splits K ranges of
 * *kb_per_split steps (needs scratch; tiles of fewer than 64 K steps are
 * never split), or, when *halves == 2, run as two 256x128 halves over the
 * full K (chosen when no K split is made and the remainder fills at most half
 * a wave).  *splits == 1 and *halves == 1: every tile runs whole.
 * FP8WS_ERR_NULL for a NULL output, FP8WS_ERR_SHAPE for tiles < 0, pairs < 1
 * or num_kb < 1. */
FP8WS_API int fp8ws_split_plan(int tiles, int pairs, int num_kb, int has_scratch, int *dp_tiles,
                               int *split_tiles, int *splits, int *kb_per_split, int *halves);

/* Launch log.  Every kernel the library enqueues is counted and recorded in a
 * small ring (the most recent FP8WS_LOG_CAPACITY records).  kind: 1 quant,
 * 2 GEMM, 3 SwiGLU-quant, 4 calibration, 5 fused gate/up SwiGLU-quant.
 * in0/in1 are the primary input pointers (for a GEMM: activation and weight),
 * out the output pointer.  A grouped launch writes one record per problem,
 * member 0, 1, ... in group order, and counts as one launch. */
#define FP8WS_LOG_CAPACITY 64
typedef struct {
  int32_t kind;
  int32_t member;
  const void *in0;
  const void *in1;
  const void *out;
} fp8ws_launch_record;

/* Total kernels launched by this library since load (all devices). */
FP8WS_API int64_t fp8ws_launch_count(void);
/* Copy up to max most recent records, oldest first; returns how many. */
FP8WS_API int fp8ws_launch_log(fp8ws_launch_record *out, int max);
/* Empty the ring (the total count keeps running). */
FP8WS_API void fp8ws_launch_log_clear(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8WS_H */
