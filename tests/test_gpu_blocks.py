"""The composed blocks on the GPU against the oracle: the split gated MLP,
shared-quant Q/K/V, the calibration helpers, single quantization by storage
identity, and the load-time equal-scale check."""

import numpy as np
import pytest
import torch

import fp8_w8a8_static_b200 as fw
import oracle
import synth
from _util import (GEMM_REL_FRO, SWIGLU_MAX_FRAC, bits, code_step_diff, codes, rel_fro, scalar,
                   stratified_rows)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gpu_rtn(w):
    wq, sw = fw.fp8_rtn_quantize_weight(w)
    return wq, sw


def _check_rtn(w, wq, sw):
    oq, osw = oracle.rtn_weight(bits(w))
    assert np.array_equal(codes(wq), oq)
    assert sw.item() == osw


# ------------------------------------------------------------ calibration


def test_absmax_exact():
    x = synth.activation_with_outliers(333, 264, 9, 0, 0, DEV)
    assert fw.fp8_absmax_bf16(x).item() == oracle.absmax(bits(x))
    assert fw.fp8_absmax_bf16(x[:0]).item() == 0.0


def test_observer_scale_bitexact():
    d = synth.c1_linear(256, 2048, device=DEV, calib_rows=128)
    amax = torch.cat([fw.fp8_absmax_bf16(b) for b in d["calib"]])
    s = fw.fp8_observer_scale(amax).item()
    assert s == oracle.observer_scale([bits(b) for b in d["calib"]])


def test_rtn_weights_bitexact():
    for shape, std, seed in (((704, 256), 0.02, 1), ((1000, 136), 0.5, 2), ((3, 16), 1e-3, 3)):
        w = synth.normal(shape, std, seed, DEV)
        _check_rtn(w, *_gpu_rtn(w))


def test_silu_mul_absmax_close():
    g = synth.normal((128, 704), 2.0, 4, DEV)
    u = synth.normal((128, 704), 1.0, 5, DEV)
    got = fw.fp8_silu_mul_absmax(g, u).item()
    want = np.abs(oracle.silu_mul_f64(oracle.bf16_to_f64(bits(g)), oracle.bf16_to_f64(bits(u)))).max()
    assert abs(got - want) <= 1e-5 * want


# -------------------------------------------------------------- gated MLP


def _c0():
    d = synth.c0_mlp(device=DEV)
    w = {n: _gpu_rtn(d[n]) for n in ("wg", "wu", "wd")}
    for n in w:
        _check_rtn(d[n], *w[n])
    calib = [bits(b) for b in d["calib"]]
    s_in = oracle.observer_scale(calib)
    s_down = oracle.down_scale(calib, bits(d["wg"]), bits(d["wu"]))
    return d, w, s_in, s_down


def test_gated_mlp_c0_and_intermediates():
    d, w, s_in, s_down = _c0()
    M, dm, I = 64, 256, 704
    ws = torch.empty(fw.gated_mlp_static_fp8_workspace(M, dm, I), dtype=torch.uint8, device=DEV)
    y = fw.gated_mlp_static_fp8(d["x"], scalar(s_in, DEV), *w["wg"], *w["wu"],
                                scalar(s_down, DEV), *w["wd"], workspace=ws)
    v = fw.gated_mlp_workspace_views(ws, M, dm, I)
    ref = oracle.gated_mlp_intermediates(bits(d["x"]), s_in, codes(w["wg"][0]), w["wg"][1].item(),
                                         codes(w["wu"][0]), w["wu"][1].item(), s_down,
                                         codes(w["wd"][0]), w["wd"][1].item())
    assert np.array_equal(codes(v["xq"]), ref["xq"])           # quant: bit-exact
    assert rel_fro(bits(v["g"]), ref["g"]) <= GEMM_REL_FRO     # gate GEMM
    assert rel_fro(bits(v["u"]), ref["u"]) <= GEMM_REL_FRO     # up GEMM
    # SwiGLU-quant on the GPU's own G, U against the oracle on the same G, U
    h_ref_same_in = oracle.silu_mul_2in(bits(v["g"]), bits(v["u"]), s_down)
    diff = code_step_diff(codes(v["h"]), h_ref_same_in)
    assert diff.max() <= 1 and (diff > 0).mean() <= SWIGLU_MAX_FRAC
    assert rel_fro(bits(y), ref["y"]) <= GEMM_REL_FRO          # whole block


def test_gated_mlp_single_quantization_by_storage_identity():
    """One quantize launch per call, and every GEMM of the gate/up pair reads
    that same buffer (checked by pointer, not by dtype)."""
    d, w, s_in, s_down = _c0()
    M, dm, I = 64, 256, 704
    ws = torch.empty(fw.gated_mlp_static_fp8_workspace(M, dm, I), dtype=torch.uint8, device=DEV)
    fw.launch_log_clear()
    n0 = fw.launch_count()
    fw.gated_mlp_static_fp8(d["x"], scalar(s_in, DEV), *w["wg"], *w["wu"], scalar(s_down, DEV),
                            *w["wd"], workspace=ws)
    log = fw.launch_log()
    assert fw.launch_count() - n0 == 5
    kinds = [r[0] for r in log]
    assert kinds == [fw.KIND_QUANT, fw.KIND_GEMM, fw.KIND_GEMM, fw.KIND_SWIGLU, fw.KIND_GEMM]
    xq_ptr = log[0][3]
    assert xq_ptr == ws.data_ptr()
    assert log[1][1] == xq_ptr and log[2][1] == xq_ptr          # gate and up read Xq
    assert log[1][2] == w["wg"][0].data_ptr() and log[2][2] == w["wu"][0].data_ptr()
    assert log[3][1] == log[1][3] and log[3][2] == log[2][3]    # SwiGLU reads G and U
    assert log[4][1] == log[3][3]                                # down reads H


@pytest.mark.parametrize("tower", ["und", "gen"])
def test_gated_mlp_two_tower_layer_sampled_rows(tower):
    """One layer of the two-tower pass at full size, in the launch
    configuration the benchmark times; the oracle checks sampled rows."""
    L = synth.c4_layer(3, tower, device=DEV, n_calib=4, calib_rows=4)
    w = {n: _gpu_rtn(L[n]) for n in ("wg", "wu", "wd")}
    for n in w:
        _check_rtn(L[n], *w[n])
    calib = [bits(b) for b in L["calib"]]
    s_in = oracle.observer_scale(calib)
    s_down = oracle.down_scale(calib, bits(L["wg"]), bits(L["wu"]))
    y = fw.gated_mlp_static_fp8(L["x"], scalar(s_in, DEV), *w["wg"], *w["wu"],
                                scalar(s_down, DEV), *w["wd"])
    rows = stratified_rows(L["M"], 7)
    ref = oracle.gated_mlp(bits(L["x"][rows]), s_in, codes(w["wg"][0]), w["wg"][1].item(),
                           codes(w["wu"][0]), w["wu"][1].item(), s_down, codes(w["wd"][0]),
                           w["wd"][1].item())
    assert rel_fro(bits(y[rows]), ref) <= GEMM_REL_FRO
    st, where = fw.device_status()
    assert st == 0, where


# ---------------------------------------------------------------- QKV


def test_qkv_shared_quant_c3_sampled_rows():
    d = synth.c3_qkv(device=DEV, n_calib=4, calib_rows=16)
    s_in = oracle.observer_scale([bits(b) for b in d["calib"]])
    w = {n: _gpu_rtn(d[n]) for n in ("wq", "wk", "wv")}
    ws = torch.empty(fw.qkv_shared_quant_workspace(2048, 3072), dtype=torch.uint8, device=DEV)
    fw.launch_log_clear()
    q, k, v = fw.qkv_shared_quant(d["x"], scalar(s_in, DEV), *w["wq"], *w["wk"], *w["wv"],
                                  workspace=ws)
    log = fw.launch_log()
    assert [r[0] for r in log] == [fw.KIND_QUANT] + [fw.KIND_GEMM] * 3
    assert all(r[1] == ws.data_ptr() for r in log[1:])
    for t, n in ((q, 3072), (k, 1024), (v, 1024)):
        assert t.shape == (2048, n) and t.is_contiguous()
    rows = stratified_rows(2048, 1)
    refs = oracle.qkv_shared_quant(bits(d["x"][rows]), s_in,
                                   [(codes(w[n][0]), w[n][1].item()) for n in ("wq", "wk", "wv")])
    for t, r in zip((q, k, v), refs):
        assert rel_fro(bits(t[rows]), r) <= GEMM_REL_FRO
    # and the shared quantization equals three separate quantizations
    xq = codes(fw.fp8_quant_static(d["x"], scalar(s_in, DEV)))
    assert np.array_equal(codes(ws[:2048 * 3072].view(fw.FP8)).reshape(2048, 3072), xq)


# ------------------------------------------------------- load-time check


def test_shared_input_scale_check():
    s = scalar(0.0123, DEV)
    assert fw.fp8_check_shared_input_scale([s, s.clone(), s.clone()]) == fw.OK
    nxt = torch.tensor([np.nextafter(np.float32(0.0123), np.float32(1))], device=DEV)
    assert fw.fp8_check_shared_input_scale([s, nxt]) == fw.ERR_SCALE_MISMATCH
    assert fw.fp8_check_shared_input_scale([scalar(0.0, DEV)] * 2) == fw.ERR_BAD_SCALE
    assert fw.fp8_check_shared_input_scale([scalar(float("inf"), DEV)] * 2) == fw.ERR_BAD_SCALE
    assert fw.fp8_check_shared_input_scale([scalar(-1.0, DEV)] * 2) == fw.ERR_BAD_SCALE


def test_argument_errors_launch_nothing():
    x = torch.zeros(64, 256, dtype=torch.bfloat16, device=DEV)
    lib = fw.load()
    n0 = fw.launch_count()
    s = scalar(1.0, DEV)
    xq = torch.empty(64 * 256 + 16, dtype=torch.uint8, device=DEV)
    # misaligned output pointer
    assert lib.fp8_quant_static(x.data_ptr(), x.numel(), s.data_ptr(), xq.data_ptr() + 1,
                                None) == fw.ERR_ALIGN
    # K not a multiple of 16
    assert lib.fp8_linear_static(xq.data_ptr(), xq.data_ptr(), 4, 16, 24, s.data_ptr(),
                                 s.data_ptr(), x.data_ptr(), None) == fw.ERR_SHAPE
    assert fw.launch_count() == n0
    assert fw.device_status()[0] == 0
