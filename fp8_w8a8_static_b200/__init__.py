"""Static per-tensor FP8 E4M3 W8A8 Linear blocks on B200 (sm_100a).

A thin ctypes binding over the C ABI in ``include/fp8ws.h``.  The functions
keep the C names; they check the torch tensors they are given (device, dtype,
contiguity, alignment), pass raw pointers and the current CUDA stream, and
raise :class:`FP8WSError` on a nonzero status.  Every step of the path runs in
the library's own sm_100a kernels; there is no fallback.  If the compiled
library is missing, the first call raises with the command that builds it.

Pages the operations follow: the TensorRT-LLM pull request "Load static FP8
Cosmos3 Nano/Super checkpoints without re-quantizing them" (What changed) and
the Hugging Face model card "Cosmos3-Nano-Policy-DROID, FP8 + RTN +
moving-average activation observer (ModelOpt W8A8, per-tensor static)"
(Scheme table).
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "FP8WSError", "library_path", "load",
    "fp8_quant_static", "fp8_linear_static", "fp8_linear_static_ws", "silu_mul_2in_fp8",
    "gated_mlp_static_fp8", "gated_mlp_static_fp8_workspace",
    "fp8_gate_up_swiglu_static", "gated_mlp_static_fp8_fused", "swiglu_2in_fp8", "swiglu",
    "gated_mlp_static_fp8_fused_workspace",
    "MAX_GROUP", "QuantProblem", "LinearProblem", "GateUpProblem", "MlpTower",
    "fp8_quant_static_group", "fp8_linear_static_group", "fp8_gate_up_swiglu_static_group",
    "gated_mlp_static_fp8_group", "gated_mlp_static_fp8_group_workspace", "group_workspace_views",
    "qkv_shared_quant", "qkv_shared_quant_workspace", "fp8_shared_quant_linears",
    "fp8_linears_static",
    "cross_attention_qkv_static_fp8", "fp8_quant_per_token", "fp8_linear_scaled",
    "silu_mul_2in_fp8_per_token", "gated_mlp_per_token_fp8",
    "fp8_check_shared_input_scale", "fp8_absmax_bf16", "fp8_silu_mul_absmax",
    "fp8_observer_scale", "fp8_rtn_quantize_weight",
    "device_check", "device_status", "launch_count", "launch_log", "launch_log_clear",
    "split_plan", "gemm_plan",
    "selftest_bounded_wait", "SITE_SELFTEST",
    "FP8", "OBSERVER_CONSTANT", "EXPORTED_SYMBOLS",
]

FP8 = torch.float8_e4m3fn
OBSERVER_CONSTANT = 0.01

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "_lib", "libfp8ws.so")

STATUS = {
    0: "ok", 1: "null pointer", 2: "unsupported size", 3: "pointer not 16-byte aligned",
    4: "group input scales differ", 5: "scale not finite or not positive",
    6: "CUDA runtime error", 7: "bounded wait in a kernel ran out",
    8: "device is not sm_100", 9: "workspace NULL or not 256-byte aligned",
}
OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_SCALE_MISMATCH, ERR_BAD_SCALE, ERR_CUDA, \
    ERR_DEVICE_TIMEOUT, ERR_UNSUPPORTED, ERR_WORKSPACE = range(10)

KIND_QUANT, KIND_GEMM, KIND_SWIGLU, KIND_CALIB, KIND_DUAL = 1, 2, 3, 4, 5
SITE_SELFTEST = 6  # wait site recorded by the bounded-wait self-test


class FP8WSError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call}: status {status} ({STATUS.get(status, 'unknown')})")


class Swiglu(ctypes.Structure):
    """SwiGLU variant descriptor: g' sigmoid(alpha g') (u' + beta), with the
    clamp g' <= limit, |u'| <= limit when has_limit."""
    _fields_ = [("alpha", ctypes.c_float), ("beta", ctypes.c_float), ("limit", ctypes.c_float),
                ("has_limit", ctypes.c_int32)]


def swiglu(alpha: float = 1.0, beta: float = 0.0, limit=None) -> "Swiglu":
    return Swiglu(alpha, beta, 0.0 if limit is None else limit, int(limit is not None))


def _act(act):
    return None if act is None else ctypes.byref(act)


class LaunchRecord(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("member", ctypes.c_int32), ("in0", ctypes.c_void_p),
                ("in1", ctypes.c_void_p), ("out", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64

MAX_GROUP = 2  # problems per grouped call (the towers of a decoder layer)


class QuantProblem(ctypes.Structure):
    _fields_ = [("x", _P), ("numel", _I64), ("s_in", _P), ("xq", _P)]


class LinearProblem(ctypes.Structure):
    _fields_ = [("xq", _P), ("wq", _P), ("M", _I64), ("s_in", _P), ("s_w", _P), ("y", _P)]


class GateUpProblem(ctypes.Structure):
    _fields_ = [("xq", _P), ("Wg", _P), ("Wu", _P), ("M", _I64), ("s_in", _P), ("s_wg", _P),
                ("s_wu", _P), ("s_down", _P), ("h", _P)]


class MlpTower(ctypes.Structure):
    _fields_ = [("x", _P), ("M", _I64), ("s_in", _P), ("Wg", _P), ("s_wg", _P), ("Wu", _P),
                ("s_wu", _P), ("s_down", _P), ("Wd", _P), ("s_wd", _P), ("y", _P)]

_SIGS = {
    "fp8_quant_static": (ctypes.c_int, [_P, _I64, _P, _P, _P]),
    "fp8_linear_static": (ctypes.c_int, [_P, _P, _I64, _I64, _I64, _P, _P, _P, _P]),
    "silu_mul_2in_fp8": (ctypes.c_int, [_P, _P, _I64, _P, _P, _P]),
    "fp8_linear_static_ws_bytes": (ctypes.c_size_t, []),
    "fp8_linear_static_ws": (ctypes.c_int, [_P, _P, _I64, _I64, _I64, _P, _P, _P, _P,
                                            ctypes.c_size_t, _P]),
    "gated_mlp_static_fp8_workspace": (ctypes.c_size_t, [_I64, _I64, _I64]),
    "gated_mlp_static_fp8": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _P,
                                            _P, _P, _P]),
    "swiglu_2in_fp8": (ctypes.c_int, [_P, _P, _I64, _P, _P, _P, _P]),
    "fp8_gate_up_swiglu_static": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P,
                                                 _P, _P, _P]),
    "gated_mlp_static_fp8_fused_workspace": (ctypes.c_size_t, [_I64, _I64, _I64]),
    "gated_mlp_static_fp8_fused": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P,
                                                  _P, _P, _P, _P, _P, _P]),
    "fp8_quant_static_group": (ctypes.c_int, [_P, ctypes.c_int, _P]),
    "fp8_linear_static_group": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I64, _P, ctypes.c_size_t,
                                               _P]),
    "fp8_gate_up_swiglu_static_group": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I64, _P, _P]),
    "gated_mlp_static_fp8_group_workspace": (ctypes.c_size_t, [_P, ctypes.c_int, _I64, _I64]),
    "gated_mlp_static_fp8_group": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I64, _P, _P,
                                                  ctypes.c_size_t, _P]),
    "gated_mlp_static_fp8_noalloc": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P,
                                                    _P, _P, _P, _P]),
    "qkv_shared_quant_workspace": (ctypes.c_size_t, [_I64, _I64]),
    "fp8_shared_quant_linears_workspace": (ctypes.c_size_t, [_I64, _I64]),
    "fp8_shared_quant_linears": (ctypes.c_int, [_P, _I64, _I64, _P, ctypes.c_int,
                                                ctypes.POINTER(ctypes.c_void_p),
                                                ctypes.POINTER(ctypes.c_int64),
                                                ctypes.POINTER(ctypes.c_void_p),
                                                ctypes.POINTER(ctypes.c_void_p), _P, _P]),
    "fp8_linears_static": (ctypes.c_int, [_P, _I64, _I64, _P, ctypes.c_int,
                                          ctypes.POINTER(ctypes.c_void_p),
                                          ctypes.POINTER(ctypes.c_int64),
                                          ctypes.POINTER(ctypes.c_void_p),
                                          ctypes.POINTER(ctypes.c_void_p), _P, ctypes.c_size_t,
                                          _P]),
    "cross_attention_qkv_static_fp8_workspace": (ctypes.c_size_t, [_I64, _I64, _I64]),
    "cross_attention_qkv_static_fp8": (ctypes.c_int, [_P, _I64, _P, _I64, _I64, _P, _P, _I64, _P,
                                                      _P, _P, _I64, _P, _P, _I64, _P, _P, _P, _P,
                                                      _P, _P]),
    "qkv_shared_quant": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _I64, _P, _P, _I64, _P, _P, _I64,
                                        _P, _P, _P, _P, _P, _P]),
    "fp8_quant_per_token": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P]),
    "fp8_linear_scaled": (ctypes.c_int, [_P, _P, _I64, _I64, _I64, _P, ctypes.c_int, _P,
                                         ctypes.c_int, _P, _P]),
    "silu_mul_2in_fp8_per_token": (ctypes.c_int, [_P, _P, _I64, _I64, _P, _P, _P]),
    "gated_mlp_per_token_fp8_workspace": (ctypes.c_size_t, [_I64, _I64, _I64]),
    "gated_mlp_per_token_fp8": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P,
                                               _P, _P]),
    "fp8_check_shared_input_scale": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int,
                                                    _P]),
    "fp8_absmax_bf16": (ctypes.c_int, [_P, _I64, _P, _P]),
    "fp8_silu_mul_absmax": (ctypes.c_int, [_P, _P, _I64, _P, _P]),
    "fp8_observer_scale": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_double, _P, _P]),
    "fp8_rtn_quantize_weight": (ctypes.c_int, [_P, _I64, _P, _P, _P]),
    "fp8ws_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "fp8ws_device_check": (ctypes.c_int, []),
    "fp8ws_device_status": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int),
                                           ctypes.POINTER(ctypes.c_int)]),
    "fp8ws_set_gemm_config": (ctypes.c_int, [ctypes.c_int]),
    "fp8ws_set_quant_form": (ctypes.c_int, [ctypes.c_int]),
    "fp8ws_selftest_bounded_wait": (ctypes.c_int, [_I64, ctypes.c_int,
                                                   ctypes.POINTER(ctypes.c_int64), _P]),
    "fp8ws_gemm_plan": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int64),
                                       ctypes.POINTER(ctypes.c_int64), ctypes.c_int,
                                       ctypes.POINTER(ctypes.c_int)]),
    "fp8ws_split_plan": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
                         + [ctypes.POINTER(ctypes.c_int)] * 5),
    "fp8ws_launch_count": (ctypes.c_int64, []),
    "fp8ws_launch_log": (ctypes.c_int, [ctypes.POINTER(LaunchRecord), ctypes.c_int]),
    "fp8ws_launch_log_clear": (None, []),
}
EXPORTED_SYMBOLS = tuple(_SIGS)

_lib = None


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load the compiled library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with `python -m fp8_w8a8_static_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


# ------------------------------------------------------------------ helpers


def _check(status: int, call: str) -> None:
    if status != OK:
        raise FP8WSError(status, call)


def _dev_ptr(t: torch.Tensor, name: str, dtypes) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} is not contiguous; strided tensors are refused, not copied")
    return t.data_ptr()


def _bf16(t, name):
    return _dev_ptr(t, name, (torch.bfloat16,))


def _fp8(t, name):
    return _dev_ptr(t, name, (FP8, torch.uint8))


def _f32(t, name):
    p = _dev_ptr(t, name, (torch.float32,))
    if t.numel() < 1:
        raise ValueError(f"{name} must hold at least one fp32 value")
    return p


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _device_of(t: torch.Tensor):
    return torch.cuda.device(t.device)


# ---------------------------------------------------------------- hot path


def fp8_quant_static(x: torch.Tensor, s_in: torch.Tensor, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """Xq = E4M3_satRNE(x / s_in), any shape, BF16 in, FP8 out."""
    lib = load()
    if out is None:
        out = torch.empty(x.shape, dtype=FP8, device=x.device)
    if out.numel() != x.numel():
        raise ValueError("out size differs from x")
    with _device_of(x):
        _check(lib.fp8_quant_static(_bf16(x, "x"), x.numel(), _f32(s_in, "s_in"),
                                    _fp8(out, "out"), _stream(stream)), "fp8_quant_static")
    return out


def fp8_linear_static(xq: torch.Tensor, wq: torch.Tensor, s_in: torch.Tensor, s_w: torch.Tensor,
                      out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Y[M,N] = bf16((s_in*s_w) * Xq[M,K] . Wq[N,K]^T)."""
    lib = load()
    if xq.dim() != 2 or wq.dim() != 2 or xq.shape[1] != wq.shape[1]:
        raise ValueError(f"shapes {tuple(xq.shape)} x {tuple(wq.shape)}^T do not match")
    M, K = xq.shape
    N = wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    if tuple(out.shape) != (M, N):
        raise ValueError("out must be [M, N]")
    with _device_of(xq):
        _check(lib.fp8_linear_static(_fp8(xq, "xq"), _fp8(wq, "wq"), M, N, K, _f32(s_in, "s_in"),
                                     _f32(s_w, "s_w"), _bf16(out, "out"), _stream(stream)),
               "fp8_linear_static")
    return out


def fp8_linear_static_ws(xq, wq, s_in, s_w, workspace=None, out=None, stream=None):
    """fp8_linear_static with split-K of the ragged last wave (workspace scratch)."""
    lib = load()
    M, K = xq.shape
    N = wq.shape[0]
    need = lib.fp8_linear_static_ws_bytes()
    if workspace is None:
        workspace = _workspace(need, xq.device)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    with _device_of(xq):
        _check(lib.fp8_linear_static_ws(_fp8(xq, "xq"), _fp8(wq, "wq"), M, N, K, _f32(s_in, "s_in"),
                                        _f32(s_w, "s_w"), _bf16(out, "out"),
                                        _dev_ptr(workspace, "workspace", (torch.uint8,)),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)), "fp8_linear_static_ws")
    return out


def silu_mul_2in_fp8(g: torch.Tensor, u: torch.Tensor, s_down: torch.Tensor,
                     out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """H = E4M3_satRNE(SiLU(G) * U / s_down) from two separate BF16 tensors (any rank)."""
    lib = load()
    if g.shape != u.shape:
        raise ValueError("G and U shapes differ")
    if out is None:
        out = torch.empty(g.shape, dtype=FP8, device=g.device)
    if out.numel() != g.numel():
        raise ValueError("out size differs from G")
    with _device_of(g):
        _check(lib.silu_mul_2in_fp8(_bf16(g, "g"), _bf16(u, "u"), g.numel(),
                                    _f32(s_down, "s_down"), _fp8(out, "out"), _stream(stream)),
               "silu_mul_2in_fp8")
    return out


def gated_mlp_static_fp8_workspace(M: int, d: int, I: int) -> int:
    return load().gated_mlp_static_fp8_workspace(M, d, I)


def _workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator hands out 512-byte aligned blocks
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def gated_mlp_static_fp8(x, s_in, wg, s_wg, wu, s_wu, s_down, wd, s_wd, workspace=None, out=None,
                         stream=None) -> torch.Tensor:
    """Split gated MLP: quantize X once, gate and up FP8 GEMMs, two-input
    SwiGLU to FP8, FP8 down GEMM.  x [M,d] BF16; wg, wu [I,d], wd [d,I] FP8."""
    lib = load()
    if x.dim() != 2:
        raise ValueError("x must be [M, d]")
    M, d = x.shape
    I = wg.shape[0]
    if tuple(wg.shape) != (I, d) or tuple(wu.shape) != (I, d) or tuple(wd.shape) != (d, I):
        raise ValueError("weight shapes must be Wg, Wu [I,d] and Wd [d,I]")
    need = lib.gated_mlp_static_fp8_workspace(M, d, I)
    if workspace is None:
        workspace = _workspace(need, x.device)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes")
    if out is None:
        out = torch.empty((M, d), dtype=torch.bfloat16, device=x.device)
    with _device_of(x):
        _check(lib.gated_mlp_static_fp8(
            _bf16(x, "x"), M, d, I, _f32(s_in, "s_in"), _fp8(wg, "wg"), _f32(s_wg, "s_wg"),
            _fp8(wu, "wu"), _f32(s_wu, "s_wu"), _f32(s_down, "s_down"), _fp8(wd, "wd"),
            _f32(s_wd, "s_wd"), _dev_ptr(workspace, "workspace", (torch.uint8,)),
            _bf16(out, "out"), _stream(stream)), "gated_mlp_static_fp8")
    return out


def gated_mlp_workspace_views(workspace: torch.Tensor, M: int, d: int, I: int):
    """Views of the regions gated_mlp_static_fp8 writes: Xq [M,d], G [M,I],
    U [M,I] (BF16) and H [M,I] (FP8)."""
    def r256(v):
        return (v + 255) // 256 * 256
    o_g = r256(M * d)
    o_u = o_g + r256(M * I * 2)
    o_h = o_u + r256(M * I * 2)
    ws = workspace.view(torch.uint8)
    xq = ws[:M * d].view(FP8).view(M, d)
    g = ws[o_g:o_g + M * I * 2].view(torch.bfloat16).view(M, I)
    u = ws[o_u:o_u + M * I * 2].view(torch.bfloat16).view(M, I)
    h = ws[o_h:o_h + M * I].view(FP8).view(M, I)
    return dict(xq=xq, g=g, u=u, h=h)


def swiglu_2in_fp8(g: torch.Tensor, u: torch.Tensor, s_down: torch.Tensor, act=None,
                   out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """silu_mul_2in_fp8 with an optional variant descriptor (see swiglu())."""
    lib = load()
    if g.shape != u.shape:
        raise ValueError("G and U shapes differ")
    if out is None:
        out = torch.empty(g.shape, dtype=FP8, device=g.device)
    with _device_of(g):
        _check(lib.swiglu_2in_fp8(_bf16(g, "g"), _bf16(u, "u"), g.numel(), _f32(s_down, "s_down"),
                                  _act(act), _fp8(out, "out"), _stream(stream)), "swiglu_2in_fp8")
    return out


def fp8_gate_up_swiglu_static(xq, wg, wu, s_in, s_wg, s_wu, s_down, act=None, out=None,
                              stream=None) -> torch.Tensor:
    """H = E4M3(SiLU(bf16(G)) * bf16(U) / s_down) with G, U the gate and up
    projections of xq [M,K] (Wg, Wu [I,K]), computed in one kernel."""
    lib = load()
    M, K = xq.shape
    I = wg.shape[0]
    if tuple(wg.shape) != (I, K) or tuple(wu.shape) != (I, K):
        raise ValueError("Wg and Wu must both be [I, K]")
    if out is None:
        out = torch.empty((M, I), dtype=FP8, device=xq.device)
    with _device_of(xq):
        _check(lib.fp8_gate_up_swiglu_static(
            _fp8(xq, "xq"), _fp8(wg, "wg"), _fp8(wu, "wu"), M, I, K, _f32(s_in, "s_in"),
            _f32(s_wg, "s_wg"), _f32(s_wu, "s_wu"), _f32(s_down, "s_down"), _act(act),
            _fp8(out, "out"), _stream(stream)), "fp8_gate_up_swiglu_static")
    return out


def gated_mlp_static_fp8_fused_workspace(M: int, d: int, I: int) -> int:
    return load().gated_mlp_static_fp8_fused_workspace(M, d, I)


def gated_mlp_static_fp8_fused(x, s_in, wg, s_wg, wu, s_wu, s_down, wd, s_wd, workspace=None,
                               out=None, stream=None, act=None) -> torch.Tensor:
    """The gated MLP with gate/up and the SwiGLU-quant fused: quantize X, one
    fused gate/up/SwiGLU kernel, the down GEMM.  Same result as
    gated_mlp_static_fp8, bit for bit."""
    lib = load()
    if x.dim() != 2:
        raise ValueError("x must be [M, d]")
    M, d = x.shape
    I = wg.shape[0]
    if tuple(wg.shape) != (I, d) or tuple(wu.shape) != (I, d) or tuple(wd.shape) != (d, I):
        raise ValueError("weight shapes must be Wg, Wu [I,d] and Wd [d,I]")
    need = lib.gated_mlp_static_fp8_fused_workspace(M, d, I)
    if workspace is None:
        workspace = _workspace(need, x.device)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes")
    if out is None:
        out = torch.empty((M, d), dtype=torch.bfloat16, device=x.device)
    with _device_of(x):
        _check(lib.gated_mlp_static_fp8_fused(
            _bf16(x, "x"), M, d, I, _f32(s_in, "s_in"), _fp8(wg, "wg"), _f32(s_wg, "s_wg"),
            _fp8(wu, "wu"), _f32(s_wu, "s_wu"), _f32(s_down, "s_down"), _act(act),
            _fp8(wd, "wd"), _f32(s_wd, "s_wd"), _dev_ptr(workspace, "workspace", (torch.uint8,)),
            _bf16(out, "out"), _stream(stream)), "gated_mlp_static_fp8_fused")
    return out


def fused_workspace_views(workspace: torch.Tensor, M: int, d: int, I: int):
    """Views of the regions gated_mlp_static_fp8_fused writes: Xq [M,d], H [M,I]."""
    o_h = (M * d + 255) // 256 * 256
    ws = workspace.view(torch.uint8)
    return dict(xq=ws[:M * d].view(FP8).view(M, d), h=ws[o_h:o_h + M * I].view(FP8).view(M, I))


# ------------------------------------------------------ grouped (two towers)


def _group_array(cls, items):
    if not 1 <= len(items) <= MAX_GROUP:
        raise ValueError(f"a group holds 1..{MAX_GROUP} problems, got {len(items)}")
    return (cls * len(items))(*items)


def fp8_quant_static_group(xs, scales, outs=None, stream=None):
    """[E4M3_satRNE(x_p / s_p)] for up to two activations, in one launch."""
    lib = load()
    if len(xs) != len(scales):
        raise ValueError("one scale per activation")
    if outs is None:
        outs = [torch.empty(x.shape, dtype=FP8, device=x.device) for x in xs]
    for x, o in zip(xs, outs):
        if o.numel() != x.numel():
            raise ValueError("out size differs from x")
    arr = _group_array(QuantProblem, [
        QuantProblem(_bf16(x, "x"), x.numel(), _f32(s, "s_in"), _fp8(o, "out"))
        for x, s, o in zip(xs, scales, outs)])
    with _device_of(xs[0]):
        _check(lib.fp8_quant_static_group(ctypes.byref(arr), len(arr), _stream(stream)),
               "fp8_quant_static_group")
    return outs


def fp8_linear_static_group(problems, outs=None, split_k=False, workspace=None, stream=None):
    """fp8_linear_static for up to two problems (xq [M_p,K], wq [N,K], s_in,
    s_w) sharing N and K, in one launch; split_k lets the tiles of the last
    partial wave be split over K (workspace scratch)."""
    lib = load()
    N, K = problems[0][1].shape
    if outs is None:
        outs = [torch.empty((xq.shape[0], N), dtype=torch.bfloat16, device=xq.device)
                for xq, *_ in problems]
    items = []
    for (xq, wq, s_in, s_w), y in zip(problems, outs):
        if xq.dim() != 2 or tuple(wq.shape) != (N, K) or xq.shape[1] != K:
            raise ValueError("every problem must be xq [M,K] x wq [N,K]^T with shared N, K")
        if tuple(y.shape) != (xq.shape[0], N):
            raise ValueError("out must be [M, N]")
        items.append(LinearProblem(_fp8(xq, "xq"), _fp8(wq, "wq"), xq.shape[0],
                                   _f32(s_in, "s_in"), _f32(s_w, "s_w"), _bf16(y, "out")))
    arr = _group_array(LinearProblem, items)
    ws_ptr, ws_bytes = None, 0
    if split_k:
        if workspace is None:
            workspace = _workspace(lib.fp8_linear_static_ws_bytes(), problems[0][0].device)
        ws_ptr = _dev_ptr(workspace, "workspace", (torch.uint8,))
        ws_bytes = workspace.numel() * workspace.element_size()
    with _device_of(problems[0][0]):
        _check(lib.fp8_linear_static_group(ctypes.byref(arr), len(arr), N, K, ws_ptr, ws_bytes,
                                           _stream(stream)), "fp8_linear_static_group")
    return outs


def fp8_gate_up_swiglu_static_group(problems, act=None, outs=None, stream=None):
    """fp8_gate_up_swiglu_static for up to two problems (xq [M_p,K], wg, wu
    [I,K], s_in, s_wg, s_wu, s_down) sharing I and K, in one launch."""
    lib = load()
    I, K = problems[0][1].shape
    if outs is None:
        outs = [torch.empty((p[0].shape[0], I), dtype=FP8, device=p[0].device) for p in problems]
    items = []
    for (xq, wg, wu, s_in, s_wg, s_wu, s_down), h in zip(problems, outs):
        if tuple(wg.shape) != (I, K) or tuple(wu.shape) != (I, K) or xq.shape[1] != K:
            raise ValueError("Wg and Wu must be [I, K], shared by the group")
        if tuple(h.shape) != (xq.shape[0], I):
            raise ValueError("out must be [M, I]")
        items.append(GateUpProblem(_fp8(xq, "xq"), _fp8(wg, "wg"), _fp8(wu, "wu"), xq.shape[0],
                                   _f32(s_in, "s_in"), _f32(s_wg, "s_wg"), _f32(s_wu, "s_wu"),
                                   _f32(s_down, "s_down"), _fp8(h, "out")))
    arr = _group_array(GateUpProblem, items)
    with _device_of(problems[0][0]):
        _check(lib.fp8_gate_up_swiglu_static_group(ctypes.byref(arr), len(arr), I, K, _act(act),
                                                   _stream(stream)),
               "fp8_gate_up_swiglu_static_group")
    return outs


def gated_mlp_static_fp8_group_workspace(Ms, d: int, I: int) -> int:
    rows = (ctypes.c_int64 * len(Ms))(*Ms)
    return load().gated_mlp_static_fp8_group_workspace(ctypes.byref(rows), len(Ms), d, I)


_TOWER_KEYS = ("x", "s_in", "wg", "s_wg", "wu", "s_wu", "s_down", "wd", "s_wd")


def gated_mlp_static_fp8_group(towers, act=None, workspace=None, outs=None, stream=None):
    """The fused gated MLP of up to two towers sharing d and I (dicts with
    keys x, s_in, wg, s_wg, wu, s_wu, s_down, wd, s_wd) in three launches:
    grouped quantize, grouped gate/up/SwiGLU, grouped down GEMM."""
    lib = load()
    for t in towers:
        missing = [k for k in _TOWER_KEYS if k not in t]
        if missing:
            raise ValueError(f"tower lacks {missing}")
    d = towers[0]["x"].shape[1]
    I = towers[0]["wg"].shape[0]
    Ms = [t["x"].shape[0] for t in towers]
    for t in towers:
        if t["x"].dim() != 2 or t["x"].shape[1] != d:
            raise ValueError("every x must be [M, d] with the shared d")
        if (tuple(t["wg"].shape) != (I, d) or tuple(t["wu"].shape) != (I, d)
                or tuple(t["wd"].shape) != (d, I)):
            raise ValueError("weight shapes must be Wg, Wu [I,d] and Wd [d,I], shared d and I")
    need = gated_mlp_static_fp8_group_workspace(Ms, d, I)
    if workspace is None:
        workspace = _workspace(need, towers[0]["x"].device)
    if outs is None:
        outs = [torch.empty((M, d), dtype=torch.bfloat16, device=t["x"].device)
                for M, t in zip(Ms, towers)]
    items = []
    for t, y in zip(towers, outs):
        if tuple(y.shape) != (t["x"].shape[0], d):
            raise ValueError("out must be [M, d]")
        items.append(MlpTower(_bf16(t["x"], "x"), t["x"].shape[0], _f32(t["s_in"], "s_in"),
                              _fp8(t["wg"], "wg"), _f32(t["s_wg"], "s_wg"), _fp8(t["wu"], "wu"),
                              _f32(t["s_wu"], "s_wu"), _f32(t["s_down"], "s_down"),
                              _fp8(t["wd"], "wd"), _f32(t["s_wd"], "s_wd"), _bf16(y, "out")))
    arr = _group_array(MlpTower, items)
    with _device_of(towers[0]["x"]):
        _check(lib.gated_mlp_static_fp8_group(
            ctypes.byref(arr), len(arr), d, I, _act(act),
            _dev_ptr(workspace, "workspace", (torch.uint8,)),
            workspace.numel() * workspace.element_size(), _stream(stream)),
            "gated_mlp_static_fp8_group")
    return outs


def group_workspace_views(workspace: torch.Tensor, Ms, d: int, I: int):
    """Per tower, views of the regions gated_mlp_static_fp8_group writes:
    Xq [M,d] and H [M,I] (FP8)."""
    views, off = [], 0
    ws = workspace.view(torch.uint8)
    for M in Ms:
        size = gated_mlp_static_fp8_fused_workspace(M, d, I)
        views.append(fused_workspace_views(ws[off:off + size], M, d, I))
        off += size
    return views


def qkv_shared_quant_workspace(M: int, d: int) -> int:
    return load().qkv_shared_quant_workspace(M, d)


def qkv_shared_quant(x, s_in, wq, s_wq, wk, s_wk, wv, s_wv, workspace=None, out=None, stream=None):
    """Q, K, V = three FP8 GEMMs over one shared quantization of x [M,d]."""
    lib = load()
    M, d = x.shape
    Nq, Nk, Nv = wq.shape[0], wk.shape[0], wv.shape[0]
    for w, n in ((wq, "wq"), (wk, "wk"), (wv, "wv")):
        if w.dim() != 2 or w.shape[1] != d:
            raise ValueError(f"{n} must be [N, {d}]")
    need = lib.qkv_shared_quant_workspace(M, d)
    if workspace is None:
        workspace = _workspace(need, x.device)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes")
    if out is None:
        out = tuple(torch.empty((M, n), dtype=torch.bfloat16, device=x.device) for n in (Nq, Nk, Nv))
    q, k, v = out
    with _device_of(x):
        _check(lib.qkv_shared_quant(
            _bf16(x, "x"), M, d, _f32(s_in, "s_in"), _fp8(wq, "wq"), Nq, _f32(s_wq, "s_wq"),
            _fp8(wk, "wk"), Nk, _f32(s_wk, "s_wk"), _fp8(wv, "wv"), Nv, _f32(s_wv, "s_wv"),
            _dev_ptr(workspace, "workspace", (torch.uint8,)), _bf16(q, "q"), _bf16(k, "k"),
            _bf16(v, "v"), _stream(stream)), "qkv_shared_quant")
    return q, k, v


def fp8_shared_quant_linears(x, s_in, projections, workspace=None, out=None, stream=None):
    """Quantize x [M,d] once, then one Linear per (W [N,d] FP8, s_w) in
    projections; returns the BF16 outputs [M,N] (n = 1 is e.g. o_proj)."""
    lib = load()
    M, d = x.shape
    n = len(projections)
    for i, (w, _) in enumerate(projections):
        if w.dim() != 2 or w.shape[1] != d:
            raise ValueError(f"projection {i} must be [N, {d}]")
    if out is None:
        out = [torch.empty((M, w.shape[0]), dtype=torch.bfloat16, device=x.device)
               for w, _ in projections]
    need = lib.fp8_shared_quant_linears_workspace(M, d)
    if workspace is None:
        workspace = _workspace(need, x.device)
    W = (ctypes.c_void_p * n)(*[_fp8(w, f"W[{i}]") for i, (w, _) in enumerate(projections)])
    N = (ctypes.c_int64 * n)(*[w.shape[0] for w, _ in projections])
    S = (ctypes.c_void_p * n)(*[_f32(sw, f"s_w[{i}]") for i, (_, sw) in enumerate(projections)])
    Y = (ctypes.c_void_p * n)(*[_bf16(y, f"y[{i}]") for i, y in enumerate(out)])
    with _device_of(x):
        _check(lib.fp8_shared_quant_linears(_bf16(x, "x"), M, d, _f32(s_in, "s_in"), n, W, N, S, Y,
                                            _dev_ptr(workspace, "workspace", (torch.uint8,)),
                                            _stream(stream)), "fp8_shared_quant_linears")
    return out


def fp8_linears_static(xq, s_in, projections, out=None, workspace=None, stream=None):
    """One Linear per (W [N,K] FP8, s_w) in projections over an activation
    xq [M,K] already quantized at s_in; grouped launches of up to three.
    workspace (optional, fp8_linear_static_ws_bytes()) lets long-K tails split."""
    lib = load()
    M, K = xq.shape
    n = len(projections)
    for i, (w, _) in enumerate(projections):
        if w.dim() != 2 or w.shape[1] != K:
            raise ValueError(f"projection {i} must be [N, {K}]")
    if out is None:
        out = [torch.empty((M, w.shape[0]), dtype=torch.bfloat16, device=xq.device)
               for w, _ in projections]
    W = (ctypes.c_void_p * n)(*[_fp8(w, f"W[{i}]") for i, (w, _) in enumerate(projections)])
    N = (ctypes.c_int64 * n)(*[w.shape[0] for w, _ in projections])
    S = (ctypes.c_void_p * n)(*[_f32(sw, f"s_w[{i}]") for i, (_, sw) in enumerate(projections)])
    Y = (ctypes.c_void_p * n)(*[_bf16(y, f"y[{i}]") for i, y in enumerate(out)])
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev_ptr(workspace, "workspace", (torch.uint8,))
        ws_bytes = workspace.numel()
    with _device_of(xq):
        _check(lib.fp8_linears_static(_fp8(xq, "xq"), M, K, _f32(s_in, "s_in"), n, W, N, S, Y,
                                      ws_ptr, ws_bytes, _stream(stream)), "fp8_linears_static")
    return out


def cross_attention_qkv_static_fp8(x, ctx, s_q, wq, s_wq, s_kv, wk, s_wk, wv, s_wv,
                                   workspace=None, out=None, stream=None):
    """Q from x (own quantization at s_q); K and V from ctx (one shared
    quantization at s_kv).  Returns contiguous BF16 q, k, v."""
    lib = load()
    Mq, d = x.shape
    Mkv = ctx.shape[0]
    if out is None:
        out = (torch.empty((Mq, wq.shape[0]), dtype=torch.bfloat16, device=x.device),
               torch.empty((Mkv, wk.shape[0]), dtype=torch.bfloat16, device=x.device),
               torch.empty((Mkv, wv.shape[0]), dtype=torch.bfloat16, device=x.device))
    q, k, v = out
    need = lib.cross_attention_qkv_static_fp8_workspace(Mq, Mkv, d)
    if workspace is None:
        workspace = _workspace(need, x.device)
    with _device_of(x):
        _check(lib.cross_attention_qkv_static_fp8(
            _bf16(x, "x"), Mq, _bf16(ctx, "ctx"), Mkv, d, _f32(s_q, "s_q"), _fp8(wq, "wq"),
            wq.shape[0], _f32(s_wq, "s_wq"), _f32(s_kv, "s_kv"), _fp8(wk, "wk"), wk.shape[0],
            _f32(s_wk, "s_wk"), _fp8(wv, "wv"), wv.shape[0], _f32(s_wv, "s_wv"),
            _dev_ptr(workspace, "workspace", (torch.uint8,)), _bf16(q, "q"), _bf16(k, "k"),
            _bf16(v, "v"), _stream(stream)), "cross_attention_qkv_static_fp8")
    return q, k, v


# -------------------------------------------- per-channel / per-token scales


def fp8_quant_per_token(x: torch.Tensor, out=None, scales=None, stream=None):
    """(xq, s): one scale per row of x [rows, K], computed at run time
    (per-token for activations, per-channel RTN for weights [N, K])."""
    lib = load()
    rows, K = x.shape
    if out is None:
        out = torch.empty((rows, K), dtype=FP8, device=x.device)
    if scales is None:
        scales = torch.empty(rows, dtype=torch.float32, device=x.device)
    with _device_of(x):
        _check(lib.fp8_quant_per_token(_bf16(x, "x"), rows, K, _dev_ptr(scales, "s", (torch.float32,)),
                                       _fp8(out, "out"), _stream(stream)), "fp8_quant_per_token")
    return out, scales


def fp8_linear_scaled(xq, wq, s_x, s_w, out=None, stream=None) -> torch.Tensor:
    """Linear with vector scales: s_x of M values (per token) or 1, s_w of N
    values (per output channel) or 1."""
    lib = load()
    M, K = xq.shape
    N = wq.shape[0]
    if s_x.numel() not in (1, M) or s_w.numel() not in (1, N):
        raise ValueError("s_x must hold 1 or M values, s_w 1 or N values")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    with _device_of(xq):
        _check(lib.fp8_linear_scaled(_fp8(xq, "xq"), _fp8(wq, "wq"), M, N, K, _f32(s_x, "s_x"),
                                     int(s_x.numel() == M and M > 1), _f32(s_w, "s_w"),
                                     int(s_w.numel() == N and N > 1), _bf16(out, "out"),
                                     _stream(stream)), "fp8_linear_scaled")
    return out


def silu_mul_2in_fp8_per_token(g, u, out=None, scales=None, stream=None):
    """(h, s): SiLU(G) * U quantized with one scale per row, computed at run time."""
    lib = load()
    rows, I = g.shape
    if out is None:
        out = torch.empty((rows, I), dtype=FP8, device=g.device)
    if scales is None:
        scales = torch.empty(rows, dtype=torch.float32, device=g.device)
    with _device_of(g):
        _check(lib.silu_mul_2in_fp8_per_token(_bf16(g, "g"), _bf16(u, "u"), rows, I,
                                              _dev_ptr(scales, "s", (torch.float32,)),
                                              _fp8(out, "out"), _stream(stream)),
               "silu_mul_2in_fp8_per_token")
    return out, scales


def gated_mlp_per_token_fp8(x, wg, s_wg, wu, s_wu, wd, s_wd, workspace=None, out=None,
                            stream=None) -> torch.Tensor:
    """Gated MLP with per-channel weight scales and per-token activation scales."""
    lib = load()
    M, d = x.shape
    I = wg.shape[0]
    need = lib.gated_mlp_per_token_fp8_workspace(M, d, I)
    if workspace is None:
        workspace = _workspace(need, x.device)
    if out is None:
        out = torch.empty((M, d), dtype=torch.bfloat16, device=x.device)
    with _device_of(x):
        _check(lib.gated_mlp_per_token_fp8(
            _bf16(x, "x"), M, d, I, _fp8(wg, "wg"), _f32(s_wg, "s_wg"), _fp8(wu, "wu"),
            _f32(s_wu, "s_wu"), _fp8(wd, "wd"), _f32(s_wd, "s_wd"),
            _dev_ptr(workspace, "workspace", (torch.uint8,)), _bf16(out, "out"), _stream(stream)),
            "gated_mlp_per_token_fp8")
    return out


# ---------------------------------------------------------------- load time


def fp8_check_shared_input_scale(scales: Sequence[torch.Tensor], stream=None) -> int:
    """Status of the equal-input-scale invariant of a group (0 = holds).  Syncs."""
    lib = load()
    ptrs = (ctypes.c_void_p * len(scales))(*[_f32(s, f"scales[{i}]") for i, s in enumerate(scales)])
    with _device_of(scales[0]):
        return lib.fp8_check_shared_input_scale(ptrs, len(scales), _stream(stream))


def fp8_absmax_bf16(x, out=None, stream=None) -> torch.Tensor:
    lib = load()
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    with _device_of(x):
        _check(lib.fp8_absmax_bf16(_bf16(x, "x"), x.numel(), _f32(out, "out"), _stream(stream)),
               "fp8_absmax_bf16")
    return out


def fp8_silu_mul_absmax(g, u, out=None, stream=None) -> torch.Tensor:
    lib = load()
    if g.shape != u.shape:
        raise ValueError("G and U shapes differ")
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=g.device)
    with _device_of(g):
        _check(lib.fp8_silu_mul_absmax(_bf16(g, "g"), _bf16(u, "u"), g.numel(), _f32(out, "out"),
                                       _stream(stream)), "fp8_silu_mul_absmax")
    return out


def fp8_observer_scale(amaxes: torch.Tensor, c: float = OBSERVER_CONSTANT, out=None,
                       stream=None) -> torch.Tensor:
    lib = load()
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=amaxes.device)
    with _device_of(amaxes):
        _check(lib.fp8_observer_scale(_f32(amaxes, "amaxes"), amaxes.numel(), float(c),
                                      _f32(out, "out"), _stream(stream)), "fp8_observer_scale")
    return out


def fp8_rtn_quantize_weight(w: torch.Tensor, wq=None, s_w=None, stream=None):
    """(Wq, s_w): RTN per-tensor weight quantization with s_w = max|W| / 448."""
    lib = load()
    if wq is None:
        wq = torch.empty(w.shape, dtype=FP8, device=w.device)
    if s_w is None:
        s_w = torch.empty(1, dtype=torch.float32, device=w.device)
    with _device_of(w):
        _check(lib.fp8_rtn_quantize_weight(_bf16(w, "w"), w.numel(), _f32(s_w, "s_w"),
                                           _fp8(wq, "wq"), _stream(stream)),
               "fp8_rtn_quantize_weight")
    return wq, s_w


# ------------------------------------------------------------- diagnostics


def device_check() -> int:
    return load().fp8ws_device_check()


def device_status():
    """(status, where): reads and clears the device status word (syncs)."""
    st, wh = ctypes.c_int(0), ctypes.c_int(0)
    _check(load().fp8ws_device_status(ctypes.byref(st), ctypes.byref(wh)), "fp8ws_device_status")
    return st.value, wh.value


GEMM_CONFIGS = {"auto": 0, "pair256": 1, "cta256": 2, "cta128": 3, "cta64": 4}


def selftest_bounded_wait(limit_ns: int, mode: int = 0, stream=None) -> int:
    """Run the bounded-wait self-test kernel (mode 0: the wait runs out and
    records site 6; mode 1: the abort flag ends it early).  Returns the wait's
    duration in ns, measured on the device."""
    out = ctypes.c_int64(0)
    _check(load().fp8ws_selftest_bounded_wait(limit_ns, mode, ctypes.byref(out), _stream(stream)),
           "fp8ws_selftest_bounded_wait")
    return out.value


def set_gemm_config(name: str = "auto") -> None:
    """Force a GEMM tile configuration (see GEMM_CONFIGS); "auto" = cost model."""
    _check(load().fp8ws_set_gemm_config(GEMM_CONFIGS[name]), "fp8ws_set_gemm_config")


QUANT_FORMS = {"auto": 0, "staged": 1, "stream": 2}


def set_quant_form(name: str = "auto") -> None:
    """Force the static quantizer's form (see QUANT_FORMS); "auto" chooses by
    input size.  The codes are the same in every form."""
    _check(load().fp8ws_set_quant_form(QUANT_FORMS[name]), "fp8ws_set_quant_form")


def gemm_plan(shapes, sms: int = 148, pairs: int = 74) -> str:
    """The tile configuration the cost model picks for [(M, N), ...] (host
    only): one of the GEMM_CONFIGS names other than "auto"."""
    n = len(shapes)
    M = (ctypes.c_int64 * n)(*[m for m, _ in shapes])
    N = (ctypes.c_int64 * n)(*[c for _, c in shapes])
    cfg = ctypes.c_int()
    _check(load().fp8ws_gemm_plan(sms, pairs, M, N, n, ctypes.byref(cfg)), "fp8ws_gemm_plan")
    return {v: k for k, v in GEMM_CONFIGS.items()}[cfg.value]


def split_plan(tiles: int, pairs: int, num_kb: int, scratch: bool = True) -> dict:
    """The CTA-pair GEMM's plan past its last full wave (host only): dp_tiles
    whole tiles, then split_tiles tiles each cut into `splits` K ranges of
    kb_per_split steps (needs scratch), or run as two 256x128 halves when
    halves == 2."""
    out = [ctypes.c_int() for _ in range(5)]
    _check(load().fp8ws_split_plan(tiles, pairs, num_kb, int(scratch),
                                   *[ctypes.byref(o) for o in out]), "fp8ws_split_plan")
    return dict(zip(("dp_tiles", "split_tiles", "splits", "kb_per_split", "halves"),
                    (o.value for o in out)))


def launch_count() -> int:
    return load().fp8ws_launch_count()


def launch_log(max_records: int = 64):
    """The most recent launch records as (kind, in0, in1, out, member) tuples;
    a grouped launch has one record per problem (member 0, 1, ...)."""
    buf = (LaunchRecord * max_records)()
    n = load().fp8ws_launch_log(buf, max_records)
    return [(r.kind, r.in0 or 0, r.in1 or 0, r.out or 0, r.member) for r in buf[:n]]


def launch_log_clear() -> None:
    load().fp8ws_launch_log_clear()
