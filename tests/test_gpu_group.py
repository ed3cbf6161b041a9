"""Grouped (two-tower) calls: one launch covers the same step of both towers
of a Mixture-of-Transformers layer.

Bars: each problem's result equals, bit for bit, the single-problem call on
the same inputs (quantize; GEMM with the same CTA-pair kernel; fused
gate/up/SwiGLU; the gated MLP's H).  Against the oracle: quantized codes
exactly, GEMM outputs within the GEMM bar (relative Frobenius error <= 1e-2
plus the element-wise bound), H within the SwiGLU bar.  The split-K variant
meets the GEMM bar and is deterministic."""

import numpy as np
import pytest
import torch

import fp8_w8a8_static_b200 as fw
import oracle
import synth
from _util import (GEMM_REL_FRO, SWIGLU_MAX_FRAC, bits, code_step_diff, codes, from_codes,
                   gemm_elementwise_bound_ok, rel_fro, scalar, stratified_rows)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture
def pair_config():
    fw.set_gemm_config("pair256")
    yield
    fw.set_gemm_config("auto")


def _random_codes(rng, shape, spread=1.0):
    v = (rng.standard_normal(shape) * spread).astype(np.float32)
    b = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return oracle.quantize(b, 1.0 / 64)


def _check_gemm(y, xq, wq, s_in, s_w, rows=None):
    yb = bits(y)
    if rows is not None:
        xq, yb = np.ascontiguousarray(xq[rows]), np.ascontiguousarray(yb[rows])
    ref = oracle.linear(xq, wq, s_in, s_w)
    absref = oracle.linear(xq & 0x7F, wq & 0x7F, s_in, s_w)
    assert rel_fro(yb, ref) <= GEMM_REL_FRO
    assert gemm_elementwise_bound_ok(yb, ref, absref, xq.shape[1]).all()


# ------------------------------------------------------------------ quantize


@pytest.mark.parametrize("form", ["stream", "staged"])
@pytest.mark.parametrize("n0,n1", [(4096 * 3072, 1024 * 3072), (7, 100_003), (1, 1),
                                   (0, 4097), (4097, 0), (64 * 256, 64 * 256), (8195, 13),
                                   (131_079, 8_189)])
def test_quant_group_against_oracle(n0, n1, form):
    """Both forms of the quantizer; ragged runs leave fewer than 8 values past
    the last whole vector of either run, or of both at once."""
    xs = [synth.normal((max(n0, 1),), 3.0, 1, DEV)[:n0], synth.normal((max(n1, 1),), 0.5, 2, DEV)[:n1]]
    s = [oracle.f32(0.0213), oracle.f32(0.00317)]
    fw.set_quant_form(form)
    try:
        outs = fw.fp8_quant_static_group(xs, [scalar(v, DEV) for v in s])
    finally:
        fw.set_quant_form("auto")
    for x, o, sv in zip(xs, outs, s):
        ref = oracle.quantize(bits(x), sv) if x.numel() else np.zeros(0, np.uint8)
        assert np.array_equal(codes(o), ref)


def test_quant_group_single_member():
    x = synth.normal((1000,), 2.0, 3, DEV)
    (q,) = fw.fp8_quant_static_group([x], [scalar(0.01, DEV)])
    assert torch.equal(q.view(torch.uint8),
                       fw.fp8_quant_static(x, scalar(0.01, DEV)).view(torch.uint8))


# ---------------------------------------------------------------------- GEMM


@pytest.mark.parametrize("M0,M1,N,K", [
    (4096, 1024, 3072, 12288),  # down projections of the two towers
    (1024, 4096, 1024, 3072),   # smaller problem first
    (300, 129, 520, 272),       # ragged everything
    (1, 255, 8, 16),            # smallest legal problems
    (64, 0, 256, 704),          # an empty member
])
def test_linear_group_equals_single(M0, M1, N, K, pair_config):
    rng = np.random.default_rng(M0 + 3 * M1 + N + K)
    xq = [_random_codes(rng, (M, K)) for M in (M0, M1)]
    wq = [_random_codes(rng, (N, K), 0.5) for _ in range(2)]
    s_in = [oracle.f32(0.013), oracle.f32(0.021)]
    s_w = [oracle.f32(0.0021), oracle.f32(0.0017)]
    probs = [(from_codes(xq[p], DEV), from_codes(wq[p], DEV), scalar(s_in[p], DEV),
              scalar(s_w[p], DEV)) for p in range(2)]
    ys = fw.fp8_linear_static_group(probs)
    for p in range(2):
        if xq[p].shape[0] == 0:
            assert ys[p].numel() == 0
            continue
        single = fw.fp8_linear_static(*probs[p])
        assert torch.equal(ys[p], single)
        rows = None
        if xq[p].shape[0] > 64:
            rows = stratified_rows(xq[p].shape[0], p)
        _check_gemm(ys[p], xq[p], wq[p], s_in[p], s_w[p], rows)
    assert fw.device_status()[0] == fw.OK


def test_linear_group_auto_config():
    """The cost model's choice for the group (whatever it is) meets the bar."""
    rng = np.random.default_rng(5)
    K, N = 512, 264
    xq = [_random_codes(rng, (M, K)) for M in (40, 90)]
    wq = [_random_codes(rng, (N, K)) for _ in range(2)]
    probs = [(from_codes(xq[p], DEV), from_codes(wq[p], DEV), scalar(0.01, DEV),
              scalar(0.002, DEV)) for p in range(2)]
    ys = fw.fp8_linear_static_group(probs)
    for p in range(2):
        _check_gemm(ys[p], xq[p], wq[p], oracle.f32(0.01), oracle.f32(0.002))


@pytest.mark.parametrize("M0,M1,N,K", [(4096, 1024, 3072, 12288), (300, 520, 264, 8208),
                                       (300, 520, 264, 1040)])
def test_linear_group_split_k(M0, M1, N, K):
    rng = np.random.default_rng(M0 + M1)
    xq = [_random_codes(rng, (M, K)) for M in (M0, M1)]
    wq = [_random_codes(rng, (N, K), 0.5) for _ in range(2)]
    probs = [(from_codes(xq[p], DEV), from_codes(wq[p], DEV), scalar(0.013, DEV),
              scalar(0.0021, DEV)) for p in range(2)]
    ws = torch.empty(fw.load().fp8_linear_static_ws_bytes(), dtype=torch.uint8, device=DEV)
    ys = fw.fp8_linear_static_group(probs, split_k=True, workspace=ws)
    ys2 = fw.fp8_linear_static_group(probs, split_k=True, workspace=ws)
    for p in range(2):
        assert torch.equal(ys[p], ys2[p])
        rows = stratified_rows(xq[p].shape[0], p + 7)
        _check_gemm(ys[p], xq[p], wq[p], oracle.f32(0.013), oracle.f32(0.0021), rows)
    assert fw.device_status()[0] == fw.OK


# ------------------------------------------------------- fused gate/up/SwiGLU


def _gate_up_inputs(M, K, I, seed):
    x = synth.activation_with_outliers(M, K, 8, seed, 0, DEV) if M else \
        torch.empty((0, K), dtype=torch.bfloat16, device=DEV)
    s_in = fw.fp8_observer_scale(fw.fp8_absmax_bf16(x)) if M else scalar(0.01, DEV)
    xq = fw.fp8_quant_static(x, s_in)
    wg, s_wg = fw.fp8_rtn_quantize_weight(synth.normal((I, K), 0.02, seed * 3 + 1, DEV))
    wu, s_wu = fw.fp8_rtn_quantize_weight(synth.normal((I, K), 0.02, seed * 3 + 2, DEV))
    return xq, wg, wu, s_in, s_wg, s_wu


@pytest.mark.parametrize("M0,M1,K,I", [
    (4096, 1024, 3072, 12288),  # the two towers
    (129, 300, 272, 400),       # ragged
    (1, 64, 32, 16),
    (0, 200, 256, 704),         # an empty member
])
def test_gate_up_group_equals_single(M0, M1, K, I):
    probs = []
    for p, (M, sd) in enumerate(((M0, 0.003), (M1, 0.0041))):
        probs.append(_gate_up_inputs(M, K, I, 31 + p) + (scalar(sd, DEV),))
    hs = fw.fp8_gate_up_swiglu_static_group(probs)
    for p in range(2):
        if probs[p][0].shape[0] == 0:
            continue
        single = fw.fp8_gate_up_swiglu_static(*probs[p])
        assert torch.equal(hs[p].view(torch.uint8), single.view(torch.uint8))
    assert fw.device_status()[0] == fw.OK


def test_gate_up_group_against_oracle_sampled_rows():
    M0, M1, K, I = 4096, 1024, 3072, 12288
    probs = [_gate_up_inputs(M, K, I, 50 + p) + (scalar(sd, DEV),)
             for p, (M, sd) in enumerate(((M0, 0.0031), (M1, 0.0027)))]
    hs = fw.fp8_gate_up_swiglu_static_group(probs)
    for p, (xq, wg, wu, s_in, s_wg, s_wu, s_down) in enumerate(probs):
        rows = stratified_rows(xq.shape[0], p)
        xr = np.ascontiguousarray(codes(xq)[rows])
        g = oracle.linear(xr, codes(wg), s_in.item(), s_wg.item())
        u = oracle.linear(xr, codes(wu), s_in.item(), s_wu.item())
        ref = oracle.silu_mul_2in(g, u, s_down.item())
        diff = code_step_diff(codes(hs[p][rows]), ref)
        assert diff.max() <= 1 and (diff > 0).mean() <= SWIGLU_MAX_FRAC


def test_gate_up_group_variant():
    K, I = 1024, 1024
    act = fw.swiglu(1.702, 1.0, 7.0)
    probs = [_gate_up_inputs(M, K, I, 70 + M) + (scalar(0.004, DEV),) for M in (512, 256)]
    hs = fw.fp8_gate_up_swiglu_static_group(probs, act)
    for p in range(2):
        single = fw.fp8_gate_up_swiglu_static(*probs[p], act)
        assert torch.equal(hs[p].view(torch.uint8), single.view(torch.uint8))


# ----------------------------------------------------------------- gated MLP


def _tower(M, d, I, seed, s_down):
    x = synth.activation_with_outliers(M, d, 9, seed, 0, DEV)
    s_in = fw.fp8_observer_scale(fw.fp8_absmax_bf16(x))
    t = dict(x=x, s_in=s_in, s_down=scalar(s_down, DEV))
    for name, shape, k in (("wg", (I, d), 1), ("wu", (I, d), 2), ("wd", (d, I), 3)):
        t[name], t["s_" + name] = fw.fp8_rtn_quantize_weight(
            synth.normal(shape, 0.02, seed * 5 + k, DEV))
    return t


def _single(t):
    M, d = t["x"].shape
    I = t["wg"].shape[0]
    ws = torch.empty(fw.gated_mlp_static_fp8_fused_workspace(M, d, I), dtype=torch.uint8,
                     device=DEV)
    y = fw.gated_mlp_static_fp8_fused(t["x"], t["s_in"], t["wg"], t["s_wg"], t["wu"], t["s_wu"],
                                      t["s_down"], t["wd"], t["s_wd"], workspace=ws)
    return y, fw.fused_workspace_views(ws, M, d, I)


@pytest.mark.parametrize("M0,M1,d,I", [(4096, 1024, 3072, 12288), (64, 200, 256, 704),
                                       (129, 1, 272, 400)])
def test_mlp_group_matches_single_towers(M0, M1, d, I):
    towers = [_tower(M0, d, I, 1, 0.0029), _tower(M1, d, I, 2, 0.0035)]
    ws = torch.empty(fw.gated_mlp_static_fp8_group_workspace([M0, M1], d, I), dtype=torch.uint8,
                     device=DEV)
    fw.launch_log_clear()
    ys = fw.gated_mlp_static_fp8_group(towers, workspace=ws)
    log = fw.launch_log()
    torch.cuda.synchronize()
    # three launches, each with one record per tower
    assert [(r[0], r[4]) for r in log] == [(fw.KIND_QUANT, 0), (fw.KIND_QUANT, 1),
                                           (fw.KIND_DUAL, 0), (fw.KIND_DUAL, 1),
                                           (fw.KIND_GEMM, 0), (fw.KIND_GEMM, 1)]
    xq0, xq1 = log[0][3], log[1][3]
    assert log[2][1] == xq0 and log[3][1] == xq1     # gate/up read each tower's Xq
    assert log[4][1] == log[2][3] and log[5][1] == log[3][3]   # down reads each H
    views = fw.group_workspace_views(ws, [M0, M1], d, I)
    for p, t in enumerate(towers):
        y1, v1 = _single(t)
        assert torch.equal(views[p]["xq"].view(torch.uint8), v1["xq"].view(torch.uint8))
        assert torch.equal(views[p]["h"].view(torch.uint8), v1["h"].view(torch.uint8))
        # the grouped down GEMM may split its last partial wave over K, which
        # changes the fp32 summation order of those tiles only
        assert rel_fro(bits(ys[p]), bits(y1)) <= 1e-3
    assert fw.device_status()[0] == fw.OK


def test_mlp_group_against_oracle():
    d, I = 256, 704
    towers = [_tower(64, d, I, 11, 0.003), _tower(200, d, I, 12, 0.0027)]
    ys = fw.gated_mlp_static_fp8_group(towers)
    for t, y in zip(towers, ys):
        ref = oracle.gated_mlp(bits(t["x"]), t["s_in"].item(), codes(t["wg"]), t["s_wg"].item(),
                               codes(t["wu"]), t["s_wu"].item(), t["s_down"].item(),
                               codes(t["wd"]), t["s_wd"].item())
        assert rel_fro(bits(y), ref) <= GEMM_REL_FRO


def test_mlp_group_full_size_sampled_rows_against_oracle():
    """The two-tower layer at full size; rows sampled from each tower."""
    d, I = 3072, 12288
    towers = [_tower(4096, d, I, 21, 0.0031), _tower(1024, d, I, 22, 0.0033)]
    ys = fw.gated_mlp_static_fp8_group(towers)
    for p, (t, y) in enumerate(zip(towers, ys)):
        rows = stratified_rows(t["x"].shape[0], p + 40)
        xr = np.ascontiguousarray(bits(t["x"])[rows])
        ref = oracle.gated_mlp(xr, t["s_in"].item(), codes(t["wg"]), t["s_wg"].item(),
                               codes(t["wu"]), t["s_wu"].item(), t["s_down"].item(),
                               codes(t["wd"]), t["s_wd"].item())
        assert rel_fro(bits(y)[rows], ref) <= GEMM_REL_FRO


def test_mlp_group_one_tower_empty():
    d, I = 256, 704
    t0 = _tower(96, d, I, 31, 0.003)
    t1 = dict(t0, x=torch.empty((0, d), dtype=torch.bfloat16, device=DEV))
    ys = fw.gated_mlp_static_fp8_group([t0, t1])
    y1, _ = _single(t0)
    assert ys[1].shape == (0, d)
    assert rel_fro(bits(ys[0]), bits(y1)) <= 1e-3


def test_mlp_group_large_sizes_sampled_rows():
    """Beyond the benchmark's shapes: towers of 16384 and 8192 tokens, d=4096,
    I=16384 (6,144 gate/up tiles and 384 down tiles per launch, K up to
    16384); the oracle checks sampled rows of each tower."""
    d, I = 4096, 16384
    towers = [_tower(16384, d, I, 61, 0.0025), _tower(8192, d, I, 62, 0.0027)]
    ys = fw.gated_mlp_static_fp8_group(towers)
    for p, (t, y) in enumerate(zip(towers, ys)):
        rows = stratified_rows(t["x"].shape[0], p + 90)
        ref = oracle.gated_mlp(np.ascontiguousarray(bits(t["x"])[rows]), t["s_in"].item(),
                               codes(t["wg"]), t["s_wg"].item(), codes(t["wu"]), t["s_wu"].item(),
                               t["s_down"].item(), codes(t["wd"]), t["s_wd"].item())
        assert rel_fro(bits(y)[rows], ref) <= GEMM_REL_FRO
    assert fw.device_status()[0] == fw.OK
    del towers, ys
    torch.cuda.empty_cache()
