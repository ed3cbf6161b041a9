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


def _check(x_bits, s):
    x = from_bits(x_bits, DEV)
    q = codes(fw.fp8_quant_static(x, scalar(s, DEV)))
    ref = oracle.quantize(x_bits, s)
    nan = is_nan_code(ref)
    assert np.array_equal(is_nan_code(q), nan)
    assert np.array_equal(q[~nan], ref[~nan])


@pytest.mark.parametrize("s", [1.0, 2.0 ** -10, 0.0123, 3.7, 1e-6, 1e4])
def test_every_bf16_pattern(s):
    """All 65536 BF16 bit patterns (zeros, subnormals, NaN, inf, everything in
    between) against the oracle at several scales."""
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


@pytest.mark.parametrize("n", [1, 7, 8, 9, 15, 17, 4095, 1_000_003])
def test_ragged_lengths(n):
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


def test_large_bench_size():
    """Full size of the largest activation the two-tower pass quantizes."""
    x = synth.activation_with_outliers(4096, 3072, 4, 1, 0, DEV)
    s = oracle.f32(0.0417)
    q = codes(fw.fp8_quant_static(x, scalar(s, DEV)))
    xb = bits(x)
    rows = stratified_rows(4096, 0)
    for r in rows:
        assert np.array_equal(q[r], oracle.quantize(np.ascontiguousarray(xb[r]), s))
