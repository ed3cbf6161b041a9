"""Attention projections on the static FP8 path: o_proj (one Linear over its
own quantization), the general shared-quant projection call, and
cross-attention Q/K/V, where Q reads the query-side activation and K/V a
different tensor, so Q does not share their quantization."""

import pytest
import torch

import fp8_w8a8_static_b200 as fw
import oracle
import synth
from _util import GEMM_REL_FRO, bits, codes, rel_fro, scalar, stratified_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _proj(N, d, seed):
    return fw.fp8_rtn_quantize_weight(synth.normal((N, d), 0.02, seed, DEV))


def _ref(p):
    return codes(p[0]), p[1].item()


def test_o_proj_single_linear():
    M, d = 2048, 3072
    x = synth.activation_with_outliers(M, d, 5, 3, 0, DEV)
    s = oracle.f32(0.03)
    wo = _proj(d, d, 501)
    (y,) = fw.fp8_shared_quant_linears(x, scalar(s, DEV), [wo])
    rows = stratified_rows(M, 5)
    ref = oracle.qkv_shared_quant(bits(x[rows]), s, [_ref(wo)])[0]
    assert rel_fro(bits(y[rows]), ref) <= GEMM_REL_FRO


def test_general_call_matches_qkv_shared_quant_bitwise():
    M, d = 512, 3072
    x = synth.activation_with_outliers(M, d, 5, 4, 0, DEV)
    s = scalar(0.03, DEV)
    wq, wk, wv = _proj(3072, d, 511), _proj(1024, d, 512), _proj(1024, d, 513)
    a = fw.fp8_shared_quant_linears(x, s, [wq, wk, wv])
    b = fw.qkv_shared_quant(x, s, *wq, *wk, *wv)
    for t, r in zip(a, b):
        assert torch.equal(t, r)


def test_cross_attention_projections():
    Mq, Mkv, d = 4096, 1024, 3072   # generation-tower queries over understanding-tower context
    x = synth.activation_with_outliers(Mq, d, 5, 5, 0, DEV)
    ctx = synth.activation_with_outliers(Mkv, d, 5, 6, 0, DEV)
    s_q, s_kv = oracle.f32(0.031), oracle.f32(0.027)
    wq, wk, wv = _proj(3072, d, 521), _proj(1024, d, 522), _proj(1024, d, 523)
    ws = torch.empty(fw.load().cross_attention_qkv_static_fp8_workspace(Mq, Mkv, d),
                     dtype=torch.uint8, device=DEV)
    fw.launch_log_clear()
    q, k, v = fw.cross_attention_qkv_static_fp8(x, ctx, scalar(s_q, DEV), *wq, scalar(s_kv, DEV),
                                                *wk, *wv, workspace=ws)
    log = fw.launch_log()
    # one quantize launch for both inputs, one grouped GEMM launch for Q, K, V
    assert [(r[0], r[4]) for r in log] == [(fw.KIND_QUANT, 0), (fw.KIND_QUANT, 1),
                                           (fw.KIND_GEMM, 0), (fw.KIND_GEMM, 1), (fw.KIND_GEMM, 2)]
    xq_ptr, ctxq_ptr = log[0][3], log[1][3]
    assert log[0][1] == x.data_ptr() and log[1][1] == ctx.data_ptr()
    assert xq_ptr != ctxq_ptr                        # Q does not share K/V's quantization
    assert log[2][1] == xq_ptr and log[2][3] == q.data_ptr()
    assert log[3][1] == ctxq_ptr and log[4][1] == ctxq_ptr   # K and V share one
    assert log[3][3] == k.data_ptr() and log[4][3] == v.data_ptr()
    rq = stratified_rows(Mq, 6)
    rk = stratified_rows(Mkv, 7)
    ref_q = oracle.qkv_shared_quant(bits(x[rq]), s_q, [_ref(wq)])[0]
    ref_k, ref_v = oracle.qkv_shared_quant(bits(ctx[rk]), s_kv, [_ref(wk), _ref(wv)])
    assert rel_fro(bits(q[rq]), ref_q) <= GEMM_REL_FRO
    assert rel_fro(bits(k[rk]), ref_k) <= GEMM_REL_FRO
    assert rel_fro(bits(v[rk]), ref_v) <= GEMM_REL_FRO
    for t in (q, k, v):
        assert t.is_contiguous()


def test_kv_input_scales_checked_at_load():
    s = scalar(0.027, DEV)
    assert fw.fp8_check_shared_input_scale([s, s.clone()]) == fw.OK
    other = scalar(0.031, DEV)
    assert fw.fp8_check_shared_input_scale([s, other]) == fw.ERR_SCALE_MISMATCH


def test_many_projections_in_groups_of_three():
    """Seven projections of one shared quantization (two full groups of three
    and a remainder, ragged widths) against the oracle; one launch per group."""
    M, d = 300, 512
    x = synth.activation_with_outliers(M, d, 5, 8, 0, DEV)
    s = oracle.f32(0.029)
    widths = (264, 1024, 8, 520, 256, 3072, 128)
    projs = [_proj(n, d, 530 + i) for i, n in enumerate(widths)]
    fw.launch_log_clear()
    ys = fw.fp8_shared_quant_linears(x, scalar(s, DEV), projs)
    log = fw.launch_log()
    assert [(r[0], r[4]) for r in log] == [(fw.KIND_QUANT, 0)] + [
        (fw.KIND_GEMM, m) for m in (0, 1, 2, 0, 1, 2, 0)]
    assert all(r[1] == log[0][3] for r in log[1:])          # every GEMM reads the one Xq
    refs = oracle.qkv_shared_quant(bits(x), s, [_ref(p) for p in projs])
    for y, r, n in zip(ys, refs, widths):
        assert y.shape == (M, n) and y.is_contiguous()
        assert rel_fro(bits(y), r) <= GEMM_REL_FRO
    assert fw.device_status()[0] == fw.OK


@pytest.mark.parametrize("Mq,Mkv", [(0, 256), (256, 0)])
def test_cross_attention_with_an_empty_side(Mq, Mkv):
    d = 512
    x = synth.activation_with_outliers(max(Mq, 1), d, 5, 9, 0, DEV)[:Mq]
    ctx = synth.activation_with_outliers(max(Mkv, 1), d, 5, 10, 0, DEV)[:Mkv]
    s_q, s_kv = oracle.f32(0.031), oracle.f32(0.027)
    wq, wk, wv = _proj(512, d, 541), _proj(256, d, 542), _proj(256, d, 543)
    q, k, v = fw.cross_attention_qkv_static_fp8(x, ctx, scalar(s_q, DEV), *wq, scalar(s_kv, DEV),
                                                *wk, *wv)
    assert q.shape == (Mq, 512) and k.shape == (Mkv, 256) and v.shape == (Mkv, 256)
    if Mq:
        ref_q = oracle.qkv_shared_quant(bits(x), s_q, [_ref(wq)])[0]
        assert rel_fro(bits(q), ref_q) <= GEMM_REL_FRO
    if Mkv:
        ref_k, ref_v = oracle.qkv_shared_quant(bits(ctx), s_kv, [_ref(wk), _ref(wv)])
        assert rel_fro(bits(k), ref_k) <= GEMM_REL_FRO and rel_fro(bits(v), ref_v) <= GEMM_REL_FRO
    assert fw.device_status()[0] == fw.OK


@pytest.mark.parametrize("M,Ns", [(2048, (3072, 1024, 1024)),          # the c3 projections
                                  (300, (512, 256, 768, 128, 1024, 64, 320))])
def test_linears_over_a_prequantized_activation(M, Ns):
    """fp8_linears_static on the caller's own Xq gives the outputs of the
    shared-quant call (which quantizes first) bit for bit, and the oracle's
    on sampled rows."""
    d = 3072 if M == 2048 else 272
    x = synth.activation_with_outliers(M, d, 5, 8, 0, DEV)
    s = oracle.f32(0.029)
    ws = [_proj(n, d, 600 + i) for i, n in enumerate(Ns)]
    ref = fw.fp8_shared_quant_linears(x, scalar(s, DEV), ws)
    xq = fw.fp8_quant_static(x, scalar(s, DEV))
    fw.launch_log_clear()
    got = fw.fp8_linears_static(xq, scalar(s, DEV), ws)
    log = fw.launch_log()
    assert all(r[0] == fw.KIND_GEMM and r[1] == xq.data_ptr() for r in log)
    assert len(log) == len(Ns)
    for g, r in zip(got, ref):
        assert torch.equal(g.view(torch.int16), r.view(torch.int16))
    rows = stratified_rows(M, 9)
    refs = oracle.qkv_shared_quant(bits(x[rows]), s, [_ref(w) for w in ws])
    for g, r in zip(got, refs):
        assert rel_fro(bits(g[rows]), r) <= GEMM_REL_FRO
    assert fw.device_status()[0] == fw.OK
