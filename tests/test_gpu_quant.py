"""fp8_quant_static on the GPU against the oracle: FP8 codes bit-exact."""

import numpy as np
import pytest
import torch

import fp8_w8a8_static_b200 as fw
import oracle
import synth
from _util import bits, codes, from_bits, is_nan_code, scalar, stratified_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(params=["staged", "stream", "auto"])
def quant_form(request):
    fw.set_quant_form(request.param)
    yield request.param
    fw.set_quant_form("auto")


def _check(x_bits, s):
    x = from_bits(x_bits, DEV)
    q = codes(fw.fp8_quant_static(x, scalar(s, DEV)))
    ref = oracle.quantize(x_bits, s)
    nan = is_nan_code(ref)
    assert np.array_equal(is_nan_code(q), nan)
    assert np.array_equal(q[~nan], ref[~nan])


@pytest.mark.parametrize("s", [1.0, 2.0 ** -10, 0.0123, 3.7, 1e-6, 1e4,
                               1e-39,        # subnormal: 1/s overflows to inf
                               2.0 ** -126,  # smallest normal: 1/s = 2^126
                               2.0 ** 127,   # 1/s subnormal
                               3e38,
                               0.0, -0.0123, float("inf"), float("nan")])  # outside any calibration
def test_every_bf16_pattern(s, quant_form):
    """All 65536 BF16 bit patterns (zeros, subnormals, NaN, inf, everything in
    between) against the oracle at several scales, in both forms of the
    quantizer.  From 1e-39 on, the reciprocal-based tests of the kernels
    cannot be trusted and every value goes to IEEE division; an input of 0
    must still give the code 0 at a subnormal scale (0 * inf would be a NaN),
    and zero, negative, infinite and NaN scales give the IEEE quotient's codes
    too."""
    _check(np.arange(65536, dtype=np.uint32).astype(np.uint16), oracle.f32(s))


def test_c0_input():
    d = synth.c0_mlp(device=DEV)
    s = oracle.observer_scale([bits(b) for b in d["calib"]])
    _check(bits(d["x"]), s)


@pytest.mark.parametrize("M", synth.C1_M)
def test_c1_inputs_with_saturation(M):
    d = synth.c1_linear(M, 2048, device=DEV, calib_rows=64)
    s = oracle.observer_scale([bits(b) for b in d["calib"]])
    xb = bits(d["x"])
    ref = oracle.quantize(xb, s)
    assert ((ref & 0x7F) == 0x7E).any(), "the workload must saturate somewhere"
    _check(xb, s)


def test_c3_input():
    d = synth.c3_qkv(device=DEV, calib_rows=64)
    s = oracle.observer_scale([bits(b) for b in d["calib"]])
    _check(bits(d["x"]), s)


@pytest.mark.parametrize("n", [1, 7, 8, 9, 15, 17, 4095, 8191, 8192, 8199, 1_000_003,
                               148 * 8192 + 13])
def test_ragged_lengths(n, quant_form):
    """Lengths around the staged form's 8192-value chunks and one CTA per SM,
    and tails of fewer than 8 values."""
    rng = np.random.default_rng(n)
    x = torch.from_numpy((rng.standard_t(3, size=n) * 40).astype(np.float32)).to(torch.bfloat16)
    _check(bits(x), oracle.f32(0.071))


def test_empty():
    x = torch.empty(0, dtype=torch.bfloat16, device=DEV)
    q = fw.fp8_quant_static(x, scalar(1.0, DEV))
    assert q.numel() == 0


def test_rank3_input_flat():
    """Any rank is read as one flat run."""
    x = synth.normal((3, 5, 40), 3.0, 11, DEV)
    q = fw.fp8_quant_static(x, scalar(0.05, DEV))
    assert q.shape == x.shape
    assert np.array_equal(codes(q).ravel(), oracle.quantize(bits(x).ravel(), oracle.f32(0.05)))


def test_forms_agree_on_two_tower_group():
    """The pass's grouped quantization (4096 + 1024 rows x 3072): the staged
    and the streaming forms write the same codes, byte for byte."""
    xs = [synth.activation_with_outliers(M, 3072, 4, 2, t, DEV) for t, M in enumerate((4096, 1024))]
    ss = [scalar(0.0417, DEV), scalar(0.0213, DEV)]
    out = {}
    try:
        for form in ("staged", "stream"):
            fw.set_quant_form(form)
            out[form] = [codes(q) for q in fw.fp8_quant_static_group(xs, ss)]
    finally:
        fw.set_quant_form("auto")
    for a, b in zip(out["staged"], out["stream"]):
        assert np.array_equal(a, b)
    assert fw.device_status()[0] == fw.OK


def test_default_form_above_l2():
    """12288 x 8192 (201 MB of BF16, past 1.5 x L2, where the default form is
    the staged kernel): the same codes as the streaming form, byte for byte,
    and the oracle's on stratified rows."""
    M, K = 12288, 8192
    x = synth.activation_with_outliers(M, K, 4, 3, 0, DEV)
    s = oracle.f32(0.0389)
    q_auto = fw.fp8_quant_static(x, scalar(s, DEV))
    fw.set_quant_form("stream")
    try:
        q_stream = fw.fp8_quant_static(x, scalar(s, DEV))
    finally:
        fw.set_quant_form("auto")
    assert torch.equal(q_auto.view(torch.uint8), q_stream.view(torch.uint8))
    rows = stratified_rows(M, 4)
    xb = bits(x[rows])
    assert np.array_equal(codes(q_auto[rows]), oracle.quantize(xb, s))
    assert fw.device_status()[0] == fw.OK


def test_large_bench_size():
    """Full size of the largest activation the two-tower pass quantizes."""
    x = synth.activation_with_outliers(4096, 3072, 4, 1, 0, DEV)
    s = oracle.f32(0.0417)
    q = codes(fw.fp8_quant_static(x, scalar(s, DEV)))
    xb = bits(x)
    rows = stratified_rows(4096, 0)
    for r in rows:
        assert np.array_equal(q[r], oracle.quantize(np.ascontiguousarray(xb[r]), s))
