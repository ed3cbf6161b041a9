"""silu_mul_2in_fp8 on the GPU against the oracle (fp64 SiLU, exact
quantization of the fp64 value).

Bar (stated requirement): codes within one E4M3 step on at most 1e-4 of the
elements, identical elsewhere."""

import numpy as np
import pytest
import torch

import fp8_w8a8_static_b200 as fw
import oracle
import synth
from _util import (SWIGLU_MAX_FRAC, SWIGLU_MAX_STEP, bits, code_step_diff, codes, scalar,
                   stratified_rows)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _compare(h_gpu, ref):
    diff = code_step_diff(h_gpu, ref)
    assert diff.max(initial=0) <= SWIGLU_MAX_STEP
    assert (diff > 0).mean() <= SWIGLU_MAX_FRAC if diff.size else True


def test_c0_shape():
    rng = np.random.default_rng(0)
    g = synth.normal((64, 704), 2.0, 5, DEV)
    u = synth.normal((64, 704), 1.0, 6, DEV)
    s = oracle.f32(0.0213)
    h = codes(fw.silu_mul_2in_fp8(g, u, scalar(s, DEV)))
    _compare(h, oracle.silu_mul_2in(bits(g), bits(u), s))


def test_equals_fused_split_form():
    """The two-input result equals the oracle's fused [M,2I] form on the
    concatenation (the fused kernel's reference the pages compare against)."""
    d = synth.c2_swiglu(1024, 8192, device=DEV, n_calib=4, calib_rows=16)
    s = oracle.swiglu_down_scale([(bits(a), bits(b)) for a, b in d["calib"]])
    h = codes(fw.silu_mul_2in_fp8(d["g"], d["u"], scalar(s, DEV)))
    gu = np.concatenate([bits(d["g"]), bits(d["u"])], axis=1)
    _compare(h, oracle.silu_and_mul_fused(gu, s))


@pytest.mark.parametrize("M", synth.C2_M)
@pytest.mark.parametrize("I", synth.C2_I)
def test_sweep_full_size(M, I):
    """Full-size sweep shapes; the oracle checks a seeded sample of rows."""
    d = synth.c2_swiglu(M, I, device=DEV, n_calib=4, calib_rows=8)
    s = oracle.swiglu_down_scale([(bits(a), bits(b)) for a, b in d["calib"]])
    h = fw.silu_mul_2in_fp8(d["g"], d["u"], scalar(s, DEV))
    rows = stratified_rows(M, M * I)
    hc = codes(h[rows])
    ref = oracle.silu_mul_2in(bits(d["g"][rows]), bits(d["u"][rows]), s)
    _compare(hc, ref)
    del d, h
    torch.cuda.empty_cache()


@pytest.mark.parametrize("n", [1, 7, 9, 4097, 100_003])
def test_ragged_and_rank3(n):
    g = synth.normal((n,), 2.0, n, DEV)
    u = synth.normal((n,), 1.0, n + 1, DEV)
    s = oracle.f32(0.0117)
    h = codes(fw.silu_mul_2in_fp8(g.view(1, 1, n), u.view(1, 1, n), scalar(s, DEV))).ravel()
    _compare(h, oracle.silu_mul_2in(bits(g), bits(u), s))


def test_special_values():
    g = torch.tensor([0.0, -0.0, 100.0, -100.0, 30.0, -30.0, 1.0, -1.0] * 4,
                     dtype=torch.bfloat16, device=DEV)
    u = torch.tensor([1.0, 2.0, 3.0, -3.0, 50.0, 50.0, -0.5, 0.5] * 4, dtype=torch.bfloat16,
                     device=DEV)
    s = 0.125
    h = codes(fw.silu_mul_2in_fp8(g, u, scalar(s, DEV)))
    ref = oracle.silu_mul_2in(bits(g), bits(u), s)
    assert np.array_equal(code_step_diff(h, ref), np.zeros_like(h, dtype=np.int32))


def test_noncontiguous_refused():
    g = synth.normal((64, 128), 2.0, 1, DEV)
    u = synth.normal((64, 128), 1.0, 2, DEV)
    with pytest.raises(ValueError):
        fw.silu_mul_2in_fp8(g[:, ::2], u[:, ::2], scalar(1.0, DEV))


def test_empty():
    g = torch.empty(0, dtype=torch.bfloat16, device=DEV)
    assert fw.silu_mul_2in_fp8(g, g, scalar(1.0, DEV)).numel() == 0


# ------------------------------------------------------------------ variants

VARIANTS = [(1.702, 1.0, 7.0), (1.702, 0.0, None), (1.0, 1.0, None), (1.0, 0.0, 2.0)]


def test_variant_defaults_bitwise_equal_plain():
    g = synth.normal((256, 704), 2.0, 21, DEV)
    u = synth.normal((256, 704), 1.0, 22, DEV)
    s = scalar(0.0213, DEV)
    plain = fw.silu_mul_2in_fp8(g, u, s)
    assert torch.equal(fw.swiglu_2in_fp8(g, u, s).view(torch.uint8), plain.view(torch.uint8))
    assert torch.equal(fw.swiglu_2in_fp8(g, u, s, fw.swiglu()).view(torch.uint8),
                       plain.view(torch.uint8))


@pytest.mark.parametrize("alpha,beta,limit", VARIANTS)
def test_variant_against_oracle(alpha, beta, limit):
    g = synth.normal((512, 1000), 4.0, 23, DEV)
    u = synth.normal((512, 1000), 3.0, 24, DEV)
    s = oracle.f32(0.05)
    h = codes(fw.swiglu_2in_fp8(g, u, scalar(s, DEV), fw.swiglu(alpha, beta, limit)))
    ref = oracle.swiglu_2in(bits(g), bits(u), s, alpha, beta, limit)
    _compare(h, ref)
    # the fused [M, 2I] form of the oracle agrees too
    gu = np.concatenate([bits(g), bits(u)], axis=1)
    _compare(h, oracle.swiglu_fused(gu, s, alpha, beta, limit))


def test_variant_bad_descriptor_refused():
    g = synth.normal((8, 16), 1.0, 25, DEV)
    with pytest.raises(fw.FP8WSError):
        fw.swiglu_2in_fp8(g, g, scalar(1.0, DEV), fw.swiglu(1.0, 0.0, -1.0))
    with pytest.raises(fw.FP8WSError):
        fw.swiglu_2in_fp8(g, g, scalar(1.0, DEV), fw.swiglu(float("nan"), 0.0, None))
