"""The fused gate/up GEMM + two-input SwiGLU-quant (fp8_gate_up_swiglu_static)
and the fused gated MLP built on it.

Bars: H from the fused kernel equals, bit for bit, H from the unfused GPU path
(two fp8_linear_static calls and silu_mul_2in_fp8) on the same inputs, since
the fused epilogue performs the same roundings and fp32 operations; against
the oracle, H meets the SwiGLU bar (one E4M3 step on at most 1e-4 of
elements) and Y the GEMM bar (relative Frobenius error <= 1e-2)."""

import numpy as np
import pytest
import torch

import fp8_w8a8_static_b200 as fw
import oracle
import synth
from _util import (GEMM_REL_FRO, SWIGLU_MAX_FRAC, bits, code_step_diff, codes, rel_fro,
                   scalar, stratified_rows)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(M, K, I, seed):
    x = synth.activation_with_outliers(M, K, 8, seed, 0, DEV)
    s_in = fw.fp8_observer_scale(fw.fp8_absmax_bf16(x))
    xq = fw.fp8_quant_static(x, s_in)
    wg, s_wg = fw.fp8_rtn_quantize_weight(synth.normal((I, K), 0.02, seed * 3 + 1, DEV))
    wu, s_wu = fw.fp8_rtn_quantize_weight(synth.normal((I, K), 0.02, seed * 3 + 2, DEV))
    return x, s_in, xq, wg, s_wg, wu, s_wu


def _unfused_h(xq, wg, s_wg, wu, s_wu, s_in, s_down):
    g = fw.fp8_linear_static(xq, wg, s_in, s_wg)
    u = fw.fp8_linear_static(xq, wu, s_in, s_wu)
    return fw.silu_mul_2in_fp8(g, u, s_down), g, u


@pytest.mark.parametrize("M,K,I", [
    (64, 256, 704),        # tiny MLP (I tail: 704 = 5.5 x 128)
    (1, 32, 16),           # smallest legal problem
    (129, 272, 400),       # ragged M, K and I
    (300, 3072, 1024),
    (1024, 3072, 12288),   # understanding tower of the two-tower pass
    (4096, 3072, 12288),   # generation tower
])
def test_fused_equals_unfused_bitwise(M, K, I):
    x, s_in, xq, wg, s_wg, wu, s_wu = _inputs(M, K, I, M + I)
    s_down = scalar(0.003, DEV)
    h_ref, g, u = _unfused_h(xq, wg, s_wg, wu, s_wu, s_in, s_down)
    h = fw.fp8_gate_up_swiglu_static(xq, wg, wu, s_in, s_wg, s_wu, s_down)
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.uint8), h_ref.view(torch.uint8))
    assert fw.device_status()[0] == fw.OK


def test_fused_against_oracle_sampled_rows():
    M, K, I = 4096, 3072, 12288
    x, s_in, xq, wg, s_wg, wu, s_wu = _inputs(M, K, I, 5)
    s_down = scalar(0.0031, DEV)
    h = fw.fp8_gate_up_swiglu_static(xq, wg, wu, s_in, s_wg, s_wu, s_down)
    rows = stratified_rows(M, 2)
    xr = np.ascontiguousarray(codes(xq)[rows])
    g = oracle.linear(xr, codes(wg), s_in.item(), s_wg.item())
    u = oracle.linear(xr, codes(wu), s_in.item(), s_wu.item())
    ref = oracle.silu_mul_2in(g, u, s_down.item())
    diff = code_step_diff(codes(h[rows]), ref)
    assert diff.max() <= 1 and (diff > 0).mean() <= SWIGLU_MAX_FRAC


@pytest.mark.parametrize("M,d,I", [(64, 256, 704), (1024, 3072, 12288), (4096, 3072, 12288)])
def test_fused_mlp_equals_unfused_mlp(M, d, I):
    x, s_in, xq, wg, s_wg, wu, s_wu = _inputs(M, d, I, 11 + M)
    wd, s_wd = fw.fp8_rtn_quantize_weight(synth.normal((d, I), 0.02, 99 + M, DEV))
    s_down = scalar(0.0029, DEV)
    ws_ref = torch.empty(fw.gated_mlp_static_fp8_workspace(M, d, I), dtype=torch.uint8,
                         device=DEV)
    y_ref = fw.gated_mlp_static_fp8(x, s_in, wg, s_wg, wu, s_wu, s_down, wd, s_wd,
                                    workspace=ws_ref)
    ws = torch.empty(fw.gated_mlp_static_fp8_fused_workspace(M, d, I), dtype=torch.uint8,
                     device=DEV)
    fw.launch_log_clear()
    y = fw.gated_mlp_static_fp8_fused(x, s_in, wg, s_wg, wu, s_wu, s_down, wd, s_wd,
                                      workspace=ws)
    log = fw.launch_log()
    torch.cuda.synchronize()
    h = fw.fused_workspace_views(ws, M, d, I)["h"]
    h_ref = fw.gated_mlp_workspace_views(ws_ref, M, d, I)["h"]
    assert torch.equal(h.view(torch.uint8), h_ref.view(torch.uint8))
    assert torch.equal(y, y_ref)
    assert [r[0] for r in log] == [fw.KIND_QUANT, fw.KIND_DUAL, fw.KIND_GEMM]
    assert log[0][3] == ws.data_ptr() and log[1][1] == ws.data_ptr()   # one shared Xq
    assert log[2][1] == log[1][3]                                       # down reads H


def test_fused_mlp_c0_against_oracle():
    d = synth.c0_mlp(device=DEV)
    w = {n: fw.fp8_rtn_quantize_weight(d[n]) for n in ("wg", "wu", "wd")}
    calib = [bits(b) for b in d["calib"]]
    s_in = oracle.observer_scale(calib)
    s_down = oracle.down_scale(calib, bits(d["wg"]), bits(d["wu"]))
    y = fw.gated_mlp_static_fp8_fused(d["x"], scalar(s_in, DEV), *w["wg"], *w["wu"],
                                      scalar(s_down, DEV), *w["wd"])
    ref = oracle.gated_mlp(bits(d["x"]), s_in, codes(w["wg"][0]), w["wg"][1].item(),
                           codes(w["wu"][0]), w["wu"][1].item(), s_down, codes(w["wd"][0]),
                           w["wd"][1].item())
    assert rel_fro(bits(y), ref) <= GEMM_REL_FRO


@pytest.mark.parametrize("alpha,beta,limit", [(1.702, 1.0, 7.0), (1.0, 1.0, None)])
def test_fused_variant_equals_unfused_variant(alpha, beta, limit):
    M, K, I = 1024, 3072, 1024
    x, s_in, xq, wg, s_wg, wu, s_wu = _inputs(M, K, I, 77)
    s_down = scalar(0.004, DEV)
    act = fw.swiglu(alpha, beta, limit)
    g = fw.fp8_linear_static(xq, wg, s_in, s_wg)
    u = fw.fp8_linear_static(xq, wu, s_in, s_wu)
    h_ref = fw.swiglu_2in_fp8(g, u, s_down, act)
    h = fw.fp8_gate_up_swiglu_static(xq, wg, wu, s_in, s_wg, s_wu, s_down, act)
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.uint8), h_ref.view(torch.uint8))
    # and differs from plain SwiGLU, so the descriptor reached the kernel
    h_plain = fw.fp8_gate_up_swiglu_static(xq, wg, wu, s_in, s_wg, s_wu, s_down)
    assert not torch.equal(h.view(torch.uint8), h_plain.view(torch.uint8))
