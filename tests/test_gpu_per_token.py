"""Per-channel weight and per-token activation scales on the GPU against the
oracle: row-wise quantization bit-exact (codes and scales), Linear with vector
scales and the gated MLP on this scheme within the GEMM bar, per-token
SwiGLU-quant within the SwiGLU bar."""

import numpy as np
import pytest
import torch

import fp8_w8a8_static_b200 as fw
import oracle
import synth
from _util import (GEMM_REL_FRO, SWIGLU_MAX_FRAC, bits, code_step_diff, codes, rel_fro,
                   stratified_rows)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("rows,K", [(1, 8), (7, 264), (300, 3072), (4096, 3072),
                                    (9, 1032), (17, 3080), (33, 4096), (5, 4104), (3, 8200),
                                    (2, 16384)])
def test_quant_rows_bitexact(rows, K):
    """One block per row: rows of up to 3072 values held in registers as 3
    vectors per thread, up to 4096 as 4, up to 8192 as 8, longer ones read
    twice; codes and scales bit-exact in each regime and at its edges."""
    x = synth.activation_with_outliers(rows, K, 6, rows, 0, DEV)
    if rows > 3:
        x[2] = 0  # an all-zero row
    q, s = fw.fp8_quant_per_token(x)
    sample = np.arange(rows) if rows <= 300 else stratified_rows(rows, 1)
    rq, rs = oracle.quantize_rows(bits(x[sample]))
    assert np.array_equal(s.cpu().numpy()[sample], rs)
    assert np.array_equal(codes(q[sample]), rq)


def test_quant_rows_of_tiny_magnitude():
    """Rows whose max |x| is below 448 * 2^-128, so that the row's scale is a
    subnormal fp32 number and 1/s overflows: codes still the oracle's (the
    zeros of the row give 0, not a NaN), scales equal."""
    K = 3072
    x = synth.activation_with_outliers(4, K, 6, 9, 0, DEV).float()
    x = x / x.abs().amax(dim=1, keepdim=True)
    x[0] *= 1e-37
    x[1] *= 3e-39
    x[2] *= 1e-36
    x[3] *= 1e-30          # an ordinary small row beside them
    x = x.to(torch.bfloat16)
    x[:, ::7] = 0
    q, s = fw.fp8_quant_per_token(x)
    rq, rs = oracle.quantize_rows(bits(x))
    assert (rs[:3] < 2.0 ** -126).all()
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(codes(q), rq)


def test_per_channel_weights_bitexact():
    w = synth.normal((1024, 3072), 0.02, 71, DEV)
    q, s = fw.fp8_quant_per_token(w)
    rq, rs = oracle.quantize_rows(bits(w))
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(codes(q), rq)


@pytest.mark.parametrize("x_vec,w_vec", [(True, True), (True, False), (False, True), (False, False)])
def test_linear_scaled(x_vec, w_vec):
    M, N, K = 520, 776, 1024
    x = synth.activation_with_outliers(M, K, 6, 9, 0, DEV)
    w = synth.normal((N, K), 0.02, 72, DEV)
    if x_vec:
        xq, sx = fw.fp8_quant_per_token(x)
    else:
        sx = fw.fp8_observer_scale(fw.fp8_absmax_bf16(x))
        xq = fw.fp8_quant_static(x, sx)
    if w_vec:
        wq, sw = fw.fp8_quant_per_token(w)
    else:
        wq, sw = fw.fp8_rtn_quantize_weight(w)
    y = fw.fp8_linear_scaled(xq, wq, sx, sw)
    ref = oracle.linear_scaled(codes(xq), codes(wq), sx.cpu().numpy(), sw.cpu().numpy())
    assert rel_fro(bits(y), ref) <= GEMM_REL_FRO
    if not x_vec and not w_vec:
        assert torch.equal(y, fw.fp8_linear_static(xq, wq, sx, sw))


@pytest.mark.parametrize("rows,I", [(256, 12288), (64, 8192), (64, 8200), (64, 12296),
                                    (32, 16384), (300, 264)])
def test_silu_mul_per_token(rows, I):
    """Rows of 4 to 8 vector pairs per thread: 5 or 6 (8192 < I <= 12288) load
    in one batch of 6, the others in batches of 4; within the SwiGLU bar of
    the oracle either way, scales within fp32 rounding of its fp64 ones."""
    g = synth.normal((rows, I), 2.0, 73, DEV)
    u = synth.normal((rows, I), 1.0, 74, DEV)
    g[5] = 0
    h, s = fw.silu_mul_2in_fp8_per_token(g, u)
    rh, rs = oracle.silu_mul_2in_rows(bits(g), bits(u))
    assert np.allclose(s.cpu().numpy(), rs, rtol=1e-6, atol=0)
    diff = code_step_diff(codes(h), rh)
    assert diff.max() <= 1 and (diff > 0).mean() <= SWIGLU_MAX_FRAC


@pytest.mark.parametrize("M", [64, 1024])
def test_gated_mlp_per_token(M):
    d, I = 3072, 12288
    x = synth.activation_with_outliers(M, d, 6, 10 + M, 0, DEV)
    wg, s_wg = fw.fp8_quant_per_token(synth.normal((I, d), 0.02, 75, DEV))
    wu, s_wu = fw.fp8_quant_per_token(synth.normal((I, d), 0.02, 76, DEV))
    wd, s_wd = fw.fp8_quant_per_token(synth.normal((d, I), 0.02, 77, DEV))
    y = fw.gated_mlp_per_token_fp8(x, wg, s_wg, wu, s_wu, wd, s_wd)
    rows = np.arange(M) if M <= 64 else stratified_rows(M, 3)
    ref = oracle.gated_mlp_per_token(bits(x[rows]), codes(wg), s_wg.cpu().numpy(), codes(wu),
                                     s_wu.cpu().numpy(), codes(wd), s_wd.cpu().numpy())
    assert rel_fro(bits(y[rows]), ref) <= GEMM_REL_FRO
    assert fw.device_status()[0] == fw.OK
