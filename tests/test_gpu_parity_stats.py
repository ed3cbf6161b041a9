"""Parity statistics on every workload configuration: each test asserts the
bars (quantized codes bit-exact, SwiGLU codes within one E4M3 step on at most
1e-4 of elements, GEMM outputs within relative Frobenius error 1e-2) and
prints the measured figures as one `PARITY {...}` line (visible with -s).

Configurations: c0 tiny gated MLP, c1 Linear sweep, c2 SwiGLU sweep, c3
shared-quant Q/K/V, c4 one layer of the two-tower pass (grouped call)."""

import json

import numpy as np
import pytest
import torch

import fp8_w8a8_static_b200 as fw
import oracle
import synth
from _util import (GEMM_REL_FRO, SWIGLU_MAX_FRAC, SWIGLU_MAX_STEP, bits, code_step_diff, codes,
                   rel_fro, scalar, stratified_rows)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _report(**kw):
    print("PARITY " + json.dumps(kw, default=float))


def _rtn(w):
    return fw.fp8_rtn_quantize_weight(w)


def test_c0_tiny_mlp():
    d = synth.c0_mlp(device=DEV)
    w = {n: _rtn(d[n]) for n in ("wg", "wu", "wd")}
    calib = [bits(b) for b in d["calib"]]
    s_in = oracle.observer_scale(calib)
    s_down = oracle.down_scale(calib, bits(d["wg"]), bits(d["wu"]))
    M, dm, I = 64, 256, 704
    ws = torch.empty(fw.gated_mlp_static_fp8_workspace(M, dm, I), dtype=torch.uint8, device=DEV)
    y = fw.gated_mlp_static_fp8(d["x"], scalar(s_in, DEV), *w["wg"], *w["wu"],
                                scalar(s_down, DEV), *w["wd"], workspace=ws)
    v = fw.gated_mlp_workspace_views(ws, M, dm, I)
    args = (s_in, codes(w["wg"][0]), w["wg"][1].item(), codes(w["wu"][0]), w["wu"][1].item(),
            s_down, codes(w["wd"][0]), w["wd"][1].item())
    ref = oracle.gated_mlp_intermediates(bits(d["x"]), *args)
    xq_mismatch = int((codes(v["xq"]) != ref["xq"]).sum())
    diff = code_step_diff(codes(v["h"]), oracle.silu_mul_2in(bits(v["g"]), bits(v["u"]), s_down))
    stats = dict(config="c0", xq_mismatch=xq_mismatch, g_rel_fro=rel_fro(bits(v["g"]), ref["g"]),
                 u_rel_fro=rel_fro(bits(v["u"]), ref["u"]), h_max_step=int(diff.max()),
                 h_off_frac=float((diff > 0).mean()), y_rel_fro=rel_fro(bits(y), ref["y"]))
    yf = fw.gated_mlp_static_fp8_fused(d["x"], scalar(s_in, DEV), *w["wg"], *w["wu"],
                                       scalar(s_down, DEV), *w["wd"])
    stats["y_fused_rel_fro"] = rel_fro(bits(yf), ref["y"])
    _report(**stats)
    assert xq_mismatch == 0 and stats["h_max_step"] <= SWIGLU_MAX_STEP
    assert stats["h_off_frac"] <= SWIGLU_MAX_FRAC
    assert max(stats["g_rel_fro"], stats["u_rel_fro"], stats["y_rel_fro"],
               stats["y_fused_rel_fro"]) <= GEMM_REL_FRO


@pytest.mark.parametrize("M", synth.C1_M)
@pytest.mark.parametrize("N", synth.C1_N)
def test_c1_linear(M, N):
    d = synth.c1_linear(M, N, device=DEV, calib_rows=256)
    s_in = oracle.observer_scale([bits(b) for b in d["calib"]])
    wq, s_w = _rtn(d["w"])
    xq = fw.fp8_quant_static(d["x"], scalar(s_in, DEV))
    ref_q = oracle.quantize(bits(d["x"]), s_in)
    mismatch = int((codes(xq) != ref_q).sum())
    saturated = int(((ref_q & 0x7F) == 0x7E).sum())
    y = fw.fp8_linear_static(xq, wq, scalar(s_in, DEV), s_w)
    rows = stratified_rows(M, M + N)
    ref_y = oracle.linear(np.ascontiguousarray(ref_q[rows]), codes(wq), s_in, s_w.item())
    rf = rel_fro(bits(y)[rows], ref_y)
    _report(config="c1", M=M, N=N, K=synth.C1_K, xq_mismatch=mismatch,
            xq_elements=int(ref_q.size), saturated_codes=saturated, y_rows=len(rows), y_rel_fro=rf)
    # saturation itself is exercised bit-exactly by the quantizer tests (every
    # BF16 pattern at six scales); here it is reported, as the calibration
    # decides whether the sweep's own inputs reach 448 * s_in
    assert mismatch == 0 and rf <= GEMM_REL_FRO


@pytest.mark.parametrize("M", synth.C2_M)
@pytest.mark.parametrize("I", synth.C2_I)
def test_c2_swiglu(M, I):
    d = synth.c2_swiglu(M, I, device=DEV, n_calib=4, calib_rows=8)
    s = oracle.swiglu_down_scale([(bits(a), bits(b)) for a, b in d["calib"]])
    h = fw.silu_mul_2in_fp8(d["g"], d["u"], scalar(s, DEV))
    rows = stratified_rows(M, M * 3 + I)
    diff = code_step_diff(codes(h[rows]),
                          oracle.silu_mul_2in(bits(d["g"][rows]), bits(d["u"][rows]), s))
    _report(config="c2", M=M, I=I, rows=len(rows), elements=int(diff.size),
            max_step=int(diff.max()), off_by_one=int((diff > 0).sum()),
            off_frac=float((diff > 0).mean()))
    assert diff.max() <= SWIGLU_MAX_STEP and (diff > 0).mean() <= SWIGLU_MAX_FRAC
    del d, h
    torch.cuda.empty_cache()


def test_c3_qkv():
    d = synth.c3_qkv(device=DEV, n_calib=4, calib_rows=16)
    s_in = oracle.observer_scale([bits(b) for b in d["calib"]])
    w = {n: _rtn(d[n]) for n in ("wq", "wk", "wv")}
    q, k, v = fw.qkv_shared_quant(d["x"], scalar(s_in, DEV), *w["wq"], *w["wk"], *w["wv"])
    rows = stratified_rows(2048, 1)
    refs = oracle.qkv_shared_quant(bits(d["x"][rows]), s_in,
                                   [(codes(w[n][0]), w[n][1].item()) for n in ("wq", "wk", "wv")])
    rf = [rel_fro(bits(t[rows]), r) for t, r in zip((q, k, v), refs)]
    _report(config="c3", rows=len(rows), q_rel_fro=rf[0], k_rel_fro=rf[1], v_rel_fro=rf[2])
    assert max(rf) <= GEMM_REL_FRO


def test_c4_two_tower_layer_grouped():
    towers, refs_args = [], []
    for tower in ("gen", "und"):
        L = synth.c4_layer(0, tower, device=DEV, n_calib=4, calib_rows=8)
        w = {n: _rtn(L[n]) for n in ("wg", "wu", "wd")}
        calib = [bits(b) for b in L["calib"]]
        s_in = oracle.observer_scale(calib)
        s_down = oracle.down_scale(calib, bits(L["wg"]), bits(L["wu"]))
        towers.append(dict(x=L["x"], s_in=scalar(s_in, DEV), wg=w["wg"][0], s_wg=w["wg"][1],
                           wu=w["wu"][0], s_wu=w["wu"][1], s_down=scalar(s_down, DEV),
                           wd=w["wd"][0], s_wd=w["wd"][1]))
        refs_args.append((s_in, codes(w["wg"][0]), w["wg"][1].item(), codes(w["wu"][0]),
                          w["wu"][1].item(), s_down, codes(w["wd"][0]), w["wd"][1].item()))
    ys = fw.gated_mlp_static_fp8_group(towers)
    stats = dict(config="c4", layer=0)
    for (name, t, y, args) in zip(("gen", "und"), towers, ys, refs_args):
        rows = stratified_rows(t["x"].shape[0], len(name))
        ref = oracle.gated_mlp(bits(t["x"][rows]), *args)
        stats[f"{name}_rows"] = len(rows)
        stats[f"{name}_y_rel_fro"] = rel_fro(bits(y[rows]), ref)
    _report(**stats)
    assert max(stats["gen_y_rel_fro"], stats["und_y_rel_fro"]) <= GEMM_REL_FRO
    assert fw.device_status()[0] == fw.OK
