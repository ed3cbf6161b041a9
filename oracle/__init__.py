"""Oracle for static per-tensor FP8 E4M3 W8A8 Linear blocks.

TEST INFRASTRUCTURE ONLY.  The plain, slow CPU definition of what the CUDA
path computes.  Only the tests, the smoke check and the CPU-baseline leg of
the benchmark may import this package.  It shares no code with the CUDA path
and never loads it.

The arithmetic lives in ``fp8_oracle.c`` (plain C, fp64 unless a step says
fp32, compiled without fast-math or FMA contraction).  This wrapper marshals
numpy arrays and composes the C primitives in the order the pages give:

* Hugging Face model card "Cosmos3-Nano-Policy-DROID, FP8 + RTN +
  moving-average activation observer (ModelOpt W8A8, per-tensor static)",
  Scheme table (RTN weights, one scale per tensor, static activation scales
  from a moving average with constant 0.01) and the experiment-setup table
  (the fake-quant path: dequantized FP8 weights times a quantize-dequantized
  input).
* TensorRT-LLM pull request "Load static FP8 Cosmos3 Nano/Super checkpoints
  without re-quantizing them", Description (the fused-group re-quantization)
  and What changed (two-input SiLU(G)*U quantized for the FP8 down_proj;
  gate/up and Q/K/V sharing one quantized activation; the equal-input-scale
  check at load).

BF16 tensors cross this interface as ``numpy.uint16`` bit patterns, FP8
tensors as ``numpy.uint8`` codes.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fp8_oracle.c")
BUILD_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(BUILD_DIR, "liboracle.so")

OBSERVER_CONSTANT = 0.01
E4M3_MAX = 448.0


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, -O2, no fast-math, no FMA contraction)."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", SRC, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        dp = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        f32 = ctypes.c_float
        f64 = ctypes.c_double
        sig = {
            "oracle_e4m3_codebook": (None, [dp]),
            "oracle_e4m3_decode": (f64, [ctypes.c_uint8]),
            "oracle_round_bf16": (ctypes.c_uint16, [f64]),
            "oracle_round_bf16_array": (None, [dp, i64, u16p]),
            "oracle_quant_f32": (ctypes.c_uint8, [f32, f32]),
            "oracle_quant_f64": (ctypes.c_uint8, [f64, f64]),
            "oracle_quantize_bf16": (None, [u16p, i64, f32, u8p]),
            "oracle_absmax_bf16": (f64, [u16p, i64]),
            "oracle_moving_average": (f64, [dp, ctypes.c_int, f64]),
            "oracle_scale_from_amax_f64": (f32, [f64]),
            "oracle_rtn_weight": (f32, [u16p, i64, u8p]),
            "oracle_linear": (None, [u8p, u8p, i64, i64, i64, f32, f32, u16p]),
            "oracle_silu_mul_2in": (None, [u16p, u16p, i64, f32, u8p]),
            "oracle_silu_and_mul_fused": (None, [u16p, i64, i64, f32, u8p]),
            "oracle_silu_mul_f64": (None, [dp, dp, i64, dp]),
            "oracle_quantize_rows": (None, [u16p, i64, i64, ctypes.POINTER(ctypes.c_float), u8p]),
            "oracle_linear_scaled": (None, [u8p, u8p, i64, i64, i64, ctypes.POINTER(ctypes.c_float),
                                            ctypes.c_int, ctypes.POINTER(ctypes.c_float),
                                            ctypes.c_int, u16p]),
            "oracle_silu_mul_2in_rows": (None, [u16p, u16p, i64, i64, ctypes.POINTER(ctypes.c_float),
                                                u8p]),
            "oracle_swiglu_2in": (None, [u16p, u16p, i64, f32, f32, f32, ctypes.c_int, f32, u8p]),
            "oracle_swiglu_fused": (None, [u16p, i64, i64, f32, f32, f32, ctypes.c_int, f32, u8p]),
            "oracle_requant_group_member": (None, [u8p, i64, f32, f32, u8p]),
            "oracle_dequant": (None, [u8p, i64, dp]),
            "oracle_num_threads": (ctypes.c_int, []),
            "oracle_set_num_threads": (None, [ctypes.c_int]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray, ct):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("BF16 data must be passed as uint16 bit patterns")
    return a


def _u8(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint8:
        raise TypeError("FP8 data must be passed as uint8 codes")
    return a


def f32(v) -> float:
    """Round a Python float to the nearest fp32 value."""
    return float(np.float32(v))


# ------------------------------------------------------------------ format


def codebook() -> np.ndarray:
    """All 256 E4M3 values (NaN for 0x7F and 0xFF)."""
    out = np.empty(256, dtype=np.float64)
    lib().oracle_e4m3_codebook(_p(out, ctypes.c_double))
    return out


def dequant(q) -> np.ndarray:
    q = _u8(q)
    out = np.empty(q.shape, dtype=np.float64)
    lib().oracle_dequant(_p(q, ctypes.c_uint8), q.size, _p(out, ctypes.c_double))
    return out


def round_bf16(x) -> np.ndarray:
    """fp64 values -> BF16 bit patterns, nearest, ties to even."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().oracle_round_bf16_array(_p(x, ctypes.c_double), x.size, _p(out, ctypes.c_uint16))
    return out


def bf16_to_f64(b) -> np.ndarray:
    """BF16 bit patterns -> exact fp64 values."""
    b = _u16(b)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def quant_f32(v: float, s: float) -> int:
    return lib().oracle_quant_f32(v, s)


def quant_f64(v: float, s: float) -> int:
    return lib().oracle_quant_f64(v, s)


# ------------------------------------------------------------------ kernels


def quantize(x_bf16, s: float) -> np.ndarray:
    """fp8_quant_static: q = nearest-code(fp32(x) / fp32(s)), saturating."""
    x = _u16(x_bf16)
    q = np.empty(x.shape, dtype=np.uint8)
    lib().oracle_quantize_bf16(_p(x, ctypes.c_uint16), x.size, s, _p(q, ctypes.c_uint8))
    return q


def linear(xq, wq, s_in: float, s_w: float) -> np.ndarray:
    """fp8_linear_static: Y[M,N] = bf16((s_in*s_w) * deq(Xq) @ deq(Wq)^T), exact fp64 sum."""
    xq = _u8(xq)
    wq = _u8(wq)
    M, K = xq.shape
    N, K2 = wq.shape
    if K != K2:
        raise ValueError("inner sizes differ")
    y = np.empty((M, N), dtype=np.uint16)
    lib().oracle_linear(_p(xq, ctypes.c_uint8), _p(wq, ctypes.c_uint8), M, N, K, s_in, s_w,
                        _p(y, ctypes.c_uint16))
    return y


def silu_mul_2in(g_bf16, u_bf16, s_down: float) -> np.ndarray:
    """silu_mul_2in_fp8: h = q64(SiLU(g) * u, s_down) in fp64."""
    g = _u16(g_bf16)
    u = _u16(u_bf16)
    if g.shape != u.shape:
        raise ValueError("G and U shapes differ")
    h = np.empty(g.shape, dtype=np.uint8)
    lib().oracle_silu_mul_2in(_p(g, ctypes.c_uint16), _p(u, ctypes.c_uint16), g.size, s_down,
                              _p(h, ctypes.c_uint8))
    return h


def silu_and_mul_fused(gu_bf16, s_down: float) -> np.ndarray:
    """The fused form on one [..., 2I] tensor: gate = first half, up = second half."""
    gu = _u16(gu_bf16)
    I2 = gu.shape[-1]
    if I2 % 2:
        raise ValueError("last dim must be even")
    rows = gu.size // I2
    h = np.empty(gu.shape[:-1] + (I2 // 2,), dtype=np.uint8)
    lib().oracle_silu_and_mul_fused(_p(gu, ctypes.c_uint16), rows, I2 // 2, s_down,
                                    _p(h, ctypes.c_uint8))
    return h


def swiglu_2in(g_bf16, u_bf16, s_down: float, alpha: float = 1.0, beta: float = 0.0,
               limit=None) -> np.ndarray:
    """Two-input SwiGLU variant quantized to FP8: g' sigmoid(alpha g') (u' + beta),
    with the optional clamp g' = min(g, limit), u' = clamp(u, -limit, limit)."""
    g = _u16(g_bf16)
    u = _u16(u_bf16)
    if g.shape != u.shape:
        raise ValueError("G and U shapes differ")
    h = np.empty(g.shape, dtype=np.uint8)
    lib().oracle_swiglu_2in(_p(g, ctypes.c_uint16), _p(u, ctypes.c_uint16), g.size, s_down,
                            alpha, beta, int(limit is not None),
                            0.0 if limit is None else limit, _p(h, ctypes.c_uint8))
    return h


def swiglu_fused(gu_bf16, s_down: float, alpha: float = 1.0, beta: float = 0.0,
                 limit=None) -> np.ndarray:
    """The variant on one [..., 2I] tensor (gate = first half, up = second half)."""
    gu = _u16(gu_bf16)
    I2 = gu.shape[-1]
    rows = gu.size // I2
    h = np.empty(gu.shape[:-1] + (I2 // 2,), dtype=np.uint8)
    lib().oracle_swiglu_fused(_p(gu, ctypes.c_uint16), rows, I2 // 2, s_down, alpha, beta,
                              int(limit is not None), 0.0 if limit is None else limit,
                              _p(h, ctypes.c_uint8))
    return h


def quantize_rows(x_bf16):
    """Per-row (per-token / per-channel) quantization of a [rows, K] tensor:
    returns (codes, fp32 scales[rows])."""
    x = _u16(x_bf16)
    rows, K = x.shape
    q = np.empty(x.shape, dtype=np.uint8)
    s = np.empty(rows, dtype=np.float32)
    lib().oracle_quantize_rows(_p(x, ctypes.c_uint16), rows, K, _p(s, ctypes.c_float),
                               _p(q, ctypes.c_uint8))
    return q, s


def linear_scaled(xq, wq, sx, sw) -> np.ndarray:
    """Linear with vector scales: sx per token (length M) or one value, sw per
    output channel (length N) or one value."""
    xq = _u8(xq)
    wq = _u8(wq)
    M, K = xq.shape
    N = wq.shape[0]
    sx = np.ascontiguousarray(np.atleast_1d(np.asarray(sx, dtype=np.float32)))
    sw = np.ascontiguousarray(np.atleast_1d(np.asarray(sw, dtype=np.float32)))
    y = np.empty((M, N), dtype=np.uint16)
    lib().oracle_linear_scaled(_p(xq, ctypes.c_uint8), _p(wq, ctypes.c_uint8), M, N, K,
                               _p(sx, ctypes.c_float), int(sx.size > 1), _p(sw, ctypes.c_float),
                               int(sw.size > 1), _p(y, ctypes.c_uint16))
    return y


def silu_mul_2in_rows(g_bf16, u_bf16):
    """Two-input SwiGLU with per-token FP8 output: (codes, fp32 scales[rows])."""
    g = _u16(g_bf16)
    u = _u16(u_bf16)
    rows, I = g.shape
    h = np.empty(g.shape, dtype=np.uint8)
    s = np.empty(rows, dtype=np.float32)
    lib().oracle_silu_mul_2in_rows(_p(g, ctypes.c_uint16), _p(u, ctypes.c_uint16), rows, I,
                                   _p(s, ctypes.c_float), _p(h, ctypes.c_uint8))
    return h, s


def gated_mlp_per_token(x_bf16, wgq, s_wg, wuq, s_wu, wdq, s_wd):
    """Gated MLP with per-channel weight scales (vectors) and per-token
    activation scales computed at run time for X and for H."""
    xq, sx = quantize_rows(x_bf16)
    g = linear_scaled(xq, wgq, sx, s_wg)
    u = linear_scaled(xq, wuq, sx, s_wu)
    h, sh = silu_mul_2in_rows(g, u)
    return linear_scaled(h, wdq, sh, s_wd)


def requant_group_member(qw, s_i: float, s_max: float) -> np.ndarray:
    """The fused loader's second rounding: q64(s_i * deq(qW) / s_max)."""
    qw = _u8(qw)
    out = np.empty(qw.shape, dtype=np.uint8)
    lib().oracle_requant_group_member(_p(qw, ctypes.c_uint8), qw.size, s_i, s_max,
                                      _p(out, ctypes.c_uint8))
    return out


# -------------------------------------------------------------- calibration


def absmax(x_bf16) -> float:
    x = _u16(x_bf16)
    return lib().oracle_absmax_bf16(_p(x, ctypes.c_uint16), x.size)


def moving_average(amaxes, c: float = OBSERVER_CONSTANT) -> float:
    a = np.ascontiguousarray(amaxes, dtype=np.float64)
    return lib().oracle_moving_average(_p(a, ctypes.c_double), a.size, c)


def scale_from_amax(A: float) -> float:
    """s = fp32(A / 448), A in fp64."""
    return lib().oracle_scale_from_amax_f64(A)


def observer_scale(batches_bf16, c: float = OBSERVER_CONSTANT) -> float:
    """Static input scale from a moving-average observer over calibration batches."""
    return scale_from_amax(moving_average([absmax(b) for b in batches_bf16], c))


def rtn_weight(w_bf16):
    """RTN weight quantization: s_w = fp32(max|W|)/448 in fp32; codes q(W, s_w)."""
    w = _u16(w_bf16)
    wq = np.empty(w.shape, dtype=np.uint8)
    sw = lib().oracle_rtn_weight(_p(w, ctypes.c_uint16), w.size, _p(wq, ctypes.c_uint8))
    return wq, sw


def silu_mul_f64(g, u) -> np.ndarray:
    g = np.ascontiguousarray(g, dtype=np.float64)
    u = np.ascontiguousarray(u, dtype=np.float64)
    out = np.empty(g.shape, dtype=np.float64)
    lib().oracle_silu_mul_f64(_p(g, ctypes.c_double), _p(u, ctypes.c_double), g.size,
                              _p(out, ctypes.c_double))
    return out


def down_scale(batches_bf16, wg_bf16, wu_bf16, c: float = OBSERVER_CONSTANT) -> float:
    """Static input scale of down_proj: the observer over the unquantized
    SiLU(X Wg^T) * (X Wu^T) of each calibration batch, in fp64 (the fp64
    matmul is a library primitive; BF16 inputs widen exactly)."""
    wg = bf16_to_f64(wg_bf16)
    wu = bf16_to_f64(wu_bf16)
    am = []
    for b in batches_bf16:
        x = bf16_to_f64(b)
        h = silu_mul_f64(x @ wg.T, x @ wu.T)
        am.append(float(np.max(np.abs(h))))
    return scale_from_amax(moving_average(am, c))


def swiglu_down_scale(pairs_bf16, c: float = OBSERVER_CONSTANT) -> float:
    """Observer over SiLU(G)*U for standalone (G, U) calibration pairs."""
    am = []
    for g, u in pairs_bf16:
        h = silu_mul_f64(bf16_to_f64(g), bf16_to_f64(u))
        am.append(float(np.max(np.abs(h))))
    return scale_from_amax(moving_average(am, c))


def shared_scales_equal(scales) -> bool:
    """The load-time invariant of a shared-quant group: every member's
    input_scale is the same finite, positive fp32 value, bit for bit."""
    bits = [np.float32(s).view(np.uint32) for s in scales]
    ok = all(np.isfinite(np.float32(s)) and np.float32(s) > 0 for s in scales)
    return ok and all(b == bits[0] for b in bits)


# ------------------------------------------------------------- compositions


def gated_mlp(x_bf16, s_in, wgq, s_wg, wuq, s_wu, s_down, wdq, s_wd):
    """Split gated MLP on the static FP8 path: quantize X once, gate and up
    Linears (BF16 out), two-input SiLU(G)*U to FP8 at s_down, down Linear."""
    xq = quantize(x_bf16, s_in)
    g = linear(xq, wgq, s_in, s_wg)
    u = linear(xq, wuq, s_in, s_wu)
    h = silu_mul_2in(g, u, s_down)
    return linear(h, wdq, s_down, s_wd)


def gated_mlp_intermediates(x_bf16, s_in, wgq, s_wg, wuq, s_wu, s_down, wdq, s_wd):
    xq = quantize(x_bf16, s_in)
    g = linear(xq, wgq, s_in, s_wg)
    u = linear(xq, wuq, s_in, s_wu)
    h = silu_mul_2in(g, u, s_down)
    y = linear(h, wdq, s_down, s_wd)
    return dict(xq=xq, g=g, u=u, h=h, y=y)


def qkv_shared_quant(x_bf16, s_in, projections):
    """Quantize X once, then one Linear per (Wq, s_w) in projections."""
    xq = quantize(x_bf16, s_in)
    return [linear(xq, wq, s_in, sw) for wq, sw in projections]


def cross_attention_qkv(x_bf16, ctx_bf16, s_q, q_proj, s_kv, k_proj, v_proj):
    """Cross-attention projections: Q from x at its own scale s_q; K and V
    from ctx through one shared quantization at s_kv (sharing between Q and
    K/V must not engage, since they read different tensors)."""
    (q,) = qkv_shared_quant(x_bf16, s_q, [q_proj])
    k, v = qkv_shared_quant(ctx_bf16, s_kv, [k_proj, v_proj])
    return q, k, v


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(n)
