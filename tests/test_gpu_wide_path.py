"""The streaming kernels (quantizer, two-input SwiGLU) have two forms: 32-byte
loads, which need 32-byte-aligned BF16 inputs, and 16-byte loads, which need
only the 16-byte alignment the C ABI asks for.  The host takes the wide form
for aligned inputs (for SwiGLU: of up to 2^24 elements or at least the L2
size), so the lengths here (all short) run the wide form when aligned and the
16-byte form when shifted.  Both forms give the oracle's codes and the same codes as each
other, byte for byte, on lengths that exercise every tail (fewer than 16
leftover elements).  The long lengths of the workloads' sweeps run in the
parity tests of each kernel.  The quantizer also has a staged form (input
chunks moved by the bulk copy engine; 16-byte alignment is all it needs),
which it takes by default only for inputs of 1.5 times L2 and more, so the quantizer
tests here select the streaming form explicitly."""

import numpy as np
import pytest
import torch

import fp8_w8a8_static_b200 as fw
import oracle
import synth
from _util import (SWIGLU_MAX_FRAC, SWIGLU_MAX_STEP, bits, code_step_diff, codes, is_nan_code,
                   scalar)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _shifted(t):
    """A contiguous copy of t starting 16 bytes past a 32-byte boundary."""
    buf = torch.empty(t.numel() + 16, dtype=t.dtype, device=t.device)
    base = (-buf.data_ptr() % 32) // t.element_size()  # elements to the next 32-byte boundary
    v = buf[base + 16 // t.element_size():][: t.numel()].view(t.shape)
    v.copy_(t)
    assert v.data_ptr() % 32 == 16
    return v


def _aligned(t):
    assert t.data_ptr() % 32 == 0
    return t


LENGTHS = [1, 8, 9, 15, 16, 17, 31, 33, 4095, 65_543, 1_000_003]


@pytest.fixture
def stream_form():
    fw.set_quant_form("stream")
    yield
    fw.set_quant_form("auto")


def _heavy(n, seed, scale=40.0):
    rng = np.random.default_rng(seed)
    x = (rng.standard_t(3, size=n) * scale).astype(np.float32)
    return torch.from_numpy(x).to(torch.bfloat16).to(DEV)


@pytest.mark.parametrize("n", LENGTHS)
def test_quant_forms_agree_with_oracle(n, stream_form):
    x = _aligned(_heavy(n, n))
    s = oracle.f32(0.071)
    q_wide = codes(fw.fp8_quant_static(x, scalar(s, DEV)))
    q_narrow = codes(fw.fp8_quant_static(_shifted(x), scalar(s, DEV)))
    assert np.array_equal(q_wide, q_narrow)
    ref = oracle.quantize(bits(x), s)
    nan = is_nan_code(ref)
    assert np.array_equal(is_nan_code(q_wide), nan)
    assert np.array_equal(q_wide[~nan], ref[~nan])


def test_quant_every_bf16_pattern_narrow_form(stream_form):
    """All 65536 BF16 patterns through the 16-byte form."""
    x = torch.from_numpy(np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.int16))
    x = x.view(torch.bfloat16).to(DEV)
    s = oracle.f32(0.0123)
    q = codes(fw.fp8_quant_static(_shifted(x), scalar(s, DEV)))
    ref = oracle.quantize(bits(x), s)
    nan = is_nan_code(ref)
    assert np.array_equal(is_nan_code(q), nan)
    assert np.array_equal(q[~nan], ref[~nan])


@pytest.mark.parametrize("n", LENGTHS)
def test_staged_quant_on_shifted_input(n):
    """The staged form on an input 16 bytes past a 32-byte boundary gives the
    codes it gives on the aligned copy, and the oracle's."""
    fw.set_quant_form("staged")
    try:
        _staged_shifted_check(n)
    finally:
        fw.set_quant_form("auto")


def _staged_shifted_check(n):
    x = _aligned(_heavy(n, n + 1))
    s = oracle.f32(0.071)
    q_aligned = codes(fw.fp8_quant_static(x, scalar(s, DEV)))
    q_shifted = codes(fw.fp8_quant_static(_shifted(x), scalar(s, DEV)))
    assert np.array_equal(q_aligned, q_shifted)
    ref = oracle.quantize(bits(x), s)
    nan = is_nan_code(ref)
    assert np.array_equal(is_nan_code(q_aligned), nan)
    assert np.array_equal(q_aligned[~nan], ref[~nan])


def _swiglu_check(h, g, u, s):
    diff = code_step_diff(h, oracle.silu_mul_2in(bits(g), bits(u), s))
    assert diff.max(initial=0) <= SWIGLU_MAX_STEP
    if diff.size:
        assert (diff > 0).mean() <= SWIGLU_MAX_FRAC


@pytest.mark.parametrize("n", LENGTHS)
def test_silu_forms_agree(n):
    g = _aligned(_heavy(n, 2 * n, 2.0))
    u = _aligned(_heavy(n, 2 * n + 1, 1.0))
    s = oracle.f32(0.37)
    h_wide = codes(fw.silu_mul_2in_fp8(g, u, scalar(s, DEV)))
    # either input off the 32-byte grid selects the 16-byte form
    h_g = codes(fw.silu_mul_2in_fp8(_shifted(g), u, scalar(s, DEV)))
    h_u = codes(fw.silu_mul_2in_fp8(g, _shifted(u), scalar(s, DEV)))
    assert np.array_equal(h_wide, h_g) and np.array_equal(h_wide, h_u)
    _swiglu_check(h_wide, g, u, s)


@pytest.mark.parametrize("n", [17, 4095, 1_000_003])
def test_swiglu_variant_forms_agree(n):
    g = _aligned(_heavy(n, 3 * n, 2.0))
    u = _aligned(_heavy(n, 3 * n + 1, 1.0))
    act = fw.swiglu(1.702, 1.0, 7.0)
    s = scalar(0.05, DEV)
    h_wide = codes(fw.swiglu_2in_fp8(g, u, s, act))
    h_narrow = codes(fw.swiglu_2in_fp8(_shifted(g), _shifted(u), s, act))
    assert np.array_equal(h_wide, h_narrow)
    plain = codes(fw.swiglu_2in_fp8(g, u, s, fw.swiglu()))
    assert np.array_equal(plain, codes(fw.silu_mul_2in_fp8(_shifted(g), u, s)))


@pytest.mark.parametrize("M0,M1,K", [(129, 33, 3072), (5, 1, 24), (1000, 64, 272)])
def test_group_quant_forms(M0, M1, K, stream_form):
    """The grouped quantizer takes the wide form only when both activations are
    32-byte aligned; one shifted activation moves both to the 16-byte form."""
    xs = [synth.normal((M, K), 1.0, M + K, DEV) for M in (M0, M1)]
    s = [oracle.f32(0.013), oracle.f32(0.02)]
    ss = [scalar(v, DEV) for v in s]
    wide = [codes(q) for q in fw.fp8_quant_static_group(xs, ss)]
    narrow = [codes(q) for q in fw.fp8_quant_static_group([xs[0], _shifted(xs[1])], ss)]
    for a, b, x, sv in zip(wide, narrow, xs, s):
        assert np.array_equal(a, b)
        assert np.array_equal(a, oracle.quantize(bits(x), sv))
    assert fw.device_status()[0] == fw.OK
