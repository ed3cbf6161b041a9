"""Pins of the oracle against things other than itself: hand-derived values
(tests/golden), closed forms, invariants, library routines run as a
cross-check (torch's float8_e4m3fn and bfloat16 casts, numpy's fp64 matmul),
and brute force on tiny inputs.  Each pin is chosen so that a plausible slip in
the oracle (a dropped term, a wrong sign or index, a transposed operand, a
wrong tie rule) fails at least one of them.  CPU only."""

import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_hand.txt")


def _golden(kind):
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith(kind + " "):
                rows.append(line.split()[1:])
    assert rows
    return rows


def bits_of(t: torch.Tensor) -> np.ndarray:
    """BF16 torch tensor -> uint16 numpy bit patterns."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def torch_e4m3(values_f32: np.ndarray) -> np.ndarray:
    """Library cross-check: clamp to +-448 ourselves, then let torch cast."""
    t = torch.from_numpy(np.clip(values_f32, -448.0, 448.0).astype(np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def bitfield_decode(c: int) -> float:
    """Independent decode of one code from its bit fields with ldexp."""
    s = -1.0 if c & 0x80 else 1.0
    e = (c >> 3) & 0xF
    m = c & 7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return s * math.ldexp(m, -9)
    return s * math.ldexp(8 + m, e - 10)


# ------------------------------------------------------------------ codebook


def test_codebook_closed_form():
    cb = oracle.codebook()
    assert cb.shape == (256,)
    assert np.isnan(cb).sum() == 2 and np.isnan(cb[0x7F]) and np.isnan(cb[0xFF])
    assert np.isfinite(cb).sum() == 254
    assert cb[0x7E] == 448.0 and cb[0xFE] == -448.0
    assert np.nanmax(cb) == 448.0
    assert cb[0x08] == 2.0 ** -6 and cb[0x01] == 2.0 ** -9
    # magnitude strictly increasing in the low 7 bits
    pos = cb[0:0x7F]
    assert np.all(np.diff(pos) > 0)
    # the negative half mirrors the positive half
    assert np.array_equal(cb[0x80:0xFF], -cb[0:0x7F])


def test_codebook_bitfield_decode():
    cb = oracle.codebook()
    for c in range(256):
        v = bitfield_decode(c)
        if math.isnan(v):
            assert np.isnan(cb[c])
        else:
            assert cb[c] == v, hex(c)


def test_codebook_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    tv = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    cb = oracle.codebook()
    same = (tv == cb) | (np.isnan(tv) & np.isnan(cb))
    assert same.all()


def test_golden_decode():
    cb = oracle.codebook()
    for code, val in _golden("decode"):
        assert cb[int(code, 16)] == float(val), code


# ------------------------------------------------------------------ quantize


def test_golden_quant():
    for v, s, code in _golden("quant"):
        assert oracle.quant_f32(float(v), float(s)) == int(code, 16), (v, s)


@pytest.mark.parametrize("s", [1.0, 2.0 ** -5, 8.0])
def test_roundtrip_every_finite_code(s):
    cb = oracle.codebook()
    for c in range(256):
        if np.isnan(cb[c]):
            continue
        v = np.float32(cb[c] * s)
        assert oracle.quant_f32(float(v), s) == c, hex(c)


def test_idempotence_and_saturation():
    rng = np.random.default_rng(0)
    x = (rng.standard_t(3, size=20000) * 50).astype(np.float32)
    xb = bits_of(torch.from_numpy(x).to(torch.bfloat16))
    s = oracle.f32(0.37)
    q = oracle.quantize(xb, s)
    deq = oracle.dequant(q)
    # q(deq(q(x)) * s) == q(x)
    re = np.array([oracle.quant_f32(float(np.float32(d * s)), s) for d in deq])
    # (the fp32 product d*s is off by at most 2^-24 relative, far from any
    # rounding midpoint, which sits at least 1/16 of a value away)
    assert np.array_equal(re, q)
    xv = oracle.bf16_to_f64(xb)
    big = np.abs(xv) >= 448.0 * s * (1 + 1e-6)
    assert big.any()
    assert np.all(q[big & (xv > 0)] == 0x7E)
    assert np.all(q[big & (xv < 0)] == 0xFE)


def test_ties_go_to_even_codes():
    cb = oracle.codebook()
    for c in range(0, 0x7E):
        mid = (cb[c] + cb[c + 1]) / 2.0  # exact in fp32 for E4M3 neighbours
        assert np.float32(mid) == mid
        want = c if c % 2 == 0 else c + 1
        assert oracle.quant_f32(mid, 1.0) == want, hex(c)
        assert oracle.quant_f32(-mid, 1.0) == (0x80 | want)


def test_quantize_matches_torch_cast_after_clamp():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(50000) * 3,
        rng.standard_t(4, size=50000) * 100,
        rng.standard_normal(5000) * 1e-3,
    ]).astype(np.float32)
    xb = bits_of(torch.from_numpy(x).to(torch.bfloat16))
    for s in (1.0, oracle.f32(0.0123), oracle.f32(1.7)):
        q = oracle.quantize(xb, s)
        xf = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).float()
        t = (xf / torch.tensor(s, dtype=torch.float32)).numpy()  # IEEE fp32 divide
        assert np.array_equal(q, torch_e4m3(t)), s


def test_zero_sign_and_nan():
    assert oracle.quant_f32(0.0, 1.0) == 0x00
    assert oracle.quant_f32(-0.0, 1.0) == 0x80
    assert oracle.quant_f32(-1e-12, 1.0) == 0x80
    assert oracle.quant_f32(float("nan"), 1.0) & 0x7F == 0x7F


def test_fp32_divide_not_reciprocal():
    """The scale is a divisor: find a case where x * (1/s) and x / s round to
    different fp32 values and check the oracle follows the divide."""
    rng = np.random.default_rng(2)
    s = np.float32(0.3)
    xs = rng.standard_normal(200000).astype(np.float32) * 100
    div = xs / s
    mul = xs * (np.float32(1.0) / s)
    idx = np.nonzero(div != mul)[0]
    assert idx.size > 0
    got = np.array([oracle.quant_f32(float(xs[i]), float(s)) for i in idx[:200]])
    want = torch_e4m3(div[idx[:200]])
    assert np.array_equal(got, want)


# --------------------------------------------------------------- bf16 round


def test_round_bf16_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(3)
    f = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * 1e3,
        (rng.standard_normal(20000) * 1e-38).astype(np.float32),  # subnormals
        np.array([3.3e38, -3.3e38, 3.39e38, 1.0, 1.00390625, 1.01171875], dtype=np.float32),
    ])
    got = oracle.round_bf16(f.astype(np.float64))
    want = bits_of(torch.from_numpy(f).to(torch.bfloat16))
    assert np.array_equal(got, want)


def test_round_bf16_single_rounding():
    # 1 + 2^-8 + 2^-40 is just above the midpoint of 1 and 1+2^-7: must go up,
    # while rounding through fp32 first would land on the tie and go to even (1.0).
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert oracle.round_bf16(np.array([x]))[0] == 0x3F81
    assert oracle.round_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80


# ---------------------------------------------------------------- observer


def test_golden_observer():
    for maxima, want in _golden("observer"):
        a = [float(v) for v in maxima.split(",")]
        assert abs(oracle.moving_average(a) - float(want)) < 1e-12


def test_observer_closed_forms():
    assert oracle.moving_average([5.0] * 16) == 5.0
    a1, a2 = 3.0, 7.5
    assert abs(oracle.moving_average([a1, a2]) - (0.99 * a1 + 0.01 * a2)) < 1e-15
    # geometric closed form: a_1 = 0 then constant a gives A_B = a (1 - 0.99^(B-1))
    B, a = 16, 2.0
    got = oracle.moving_average([0.0] + [a] * (B - 1))
    assert abs(got - a * (1 - 0.99 ** (B - 1))) < 1e-12
    assert oracle.scale_from_amax(448.0) == 1.0
    assert oracle.scale_from_amax(4.04) == np.float32(4.04 / 448.0)


def test_observer_clips_heavy_tails():
    """With heavy-tailed batches the moving average sits below the largest
    batch maximum, so the rarest activations saturate."""
    data = synth.c1_linear(256, 2048, n_calib=16, calib_rows=64)
    s = oracle.observer_scale([bits_of(b) for b in data["calib"]])
    maxima = [oracle.absmax(bits_of(b)) for b in data["calib"]]
    assert s * 448.0 < max(maxima)
    q = oracle.quantize(bits_of(data["x"]), s)
    assert ((q & 0x7F) == 0x7E).any()


def test_rtn_weight():
    w = synth.normal((64, 96), 0.02, 123)
    wb = bits_of(w)
    wq, sw = oracle.rtn_weight(wb)
    amax = np.abs(oracle.bf16_to_f64(wb)).max()
    assert sw == np.float32(np.float32(amax) / np.float32(448.0))
    # the largest weight maps to the largest code
    i = np.argmax(np.abs(oracle.bf16_to_f64(wb)))
    assert wq.ravel()[i] & 0x7F == 0x7E
    # dequantized error within half a step of the grid around each value
    err = np.abs(oracle.dequant(wq) * sw - oracle.bf16_to_f64(wb))
    assert np.all(err <= np.abs(oracle.bf16_to_f64(wb)) * 2.0 ** -4 + 2.0 ** -10 * sw)


# ------------------------------------------------------------------- linear


def test_linear_integer_exact():
    """Integer-valued codes with unit scales: exact integer arithmetic."""
    rng = np.random.default_rng(4)
    ints = {int(c): v for c, v in enumerate(oracle.codebook()) if np.isfinite(v) and v == int(v) and abs(v) <= 4}
    codes = np.array(list(ints.keys()), dtype=np.uint8)
    M, N, K = 5, 7, 15
    xq = rng.choice(codes, size=(M, K)).astype(np.uint8)
    wq = rng.choice(codes, size=(N, K)).astype(np.uint8)
    y = oracle.linear(xq, wq, 1.0, 1.0)
    xi = np.vectorize(ints.get)(xq).astype(np.int64)
    wi = np.vectorize(ints.get)(wq).astype(np.int64)
    ref = xi @ wi.T
    assert np.all(np.abs(ref) < 256)  # exact in bf16 (8 significant bits)
    assert np.array_equal(oracle.bf16_to_f64(y), ref.astype(np.float64))


def test_linear_matches_numpy_fp64_matmul():
    rng = np.random.default_rng(5)
    M, N, K = 9, 13, 160
    xq = rng.integers(0, 256, size=(M, K), dtype=np.uint8)
    wq = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    xq[(xq & 0x7F) == 0x7F] = 0x3A
    wq[(wq & 0x7F) == 0x7F] = 0xB1
    s_in, s_w = oracle.f32(0.0137), oracle.f32(0.00021)
    y = oracle.linear(xq, wq, s_in, s_w)
    cb = oracle.codebook()
    acc = cb[xq] @ cb[wq].T  # exact: every partial sum fits in fp64
    ref = oracle.round_bf16((float(s_in) * float(s_w)) * acc)
    assert np.array_equal(y, ref)
    # and the orientation matters: Y[m, n] uses row n of W
    assert not np.array_equal(y[:, :M], oracle.round_bf16((float(s_in) * float(s_w)) * (cb[xq] @ cb[wq][:M].T).T[:M]))


def test_linear_torch_cross_check():
    """Library cross-check through torch: fp64 matmul then torch's bf16 cast
    (which may round twice, so allow one BF16 ulp on a tiny fraction)."""
    rng = np.random.default_rng(6)
    M, N, K = 16, 24, 256
    xq = rng.integers(0, 0x7E, size=(M, K), dtype=np.uint8) | (rng.integers(0, 2, size=(M, K), dtype=np.uint8) << 7)
    wq = rng.integers(0, 0x7E, size=(N, K), dtype=np.uint8) | (rng.integers(0, 2, size=(N, K), dtype=np.uint8) << 7)
    y = oracle.linear(xq, wq, 0.5, 0.25)
    xt = torch.from_numpy(xq).view(torch.float8_e4m3fn).double()
    wt = torch.from_numpy(wq).view(torch.float8_e4m3fn).double()
    ref = bits_of(((xt @ wt.T) * 0.125).to(torch.bfloat16))
    diff = np.abs(y.astype(np.int32) - ref.astype(np.int32))
    assert diff.max() <= 1 and (diff > 0).mean() < 1e-2


# ------------------------------------------------------------------- swiglu


def test_swiglu_2in_equals_fused_split_form():
    d = synth.c2_swiglu(1024, 8192, device="cpu", n_calib=0)
    g = bits_of(d["g"][:32, :704].contiguous())
    u = bits_of(d["u"][:32, :704].contiguous())
    s = oracle.f32(0.031)
    h2 = oracle.silu_mul_2in(g, u, s)
    gu = np.concatenate([g, u], axis=1)
    hf = oracle.silu_and_mul_fused(gu, s)
    assert np.array_equal(h2, hf)
    # swapping gate and up is a different function: the pin can tell them apart
    assert not np.array_equal(h2, oracle.silu_mul_2in(u, g, s))


def test_swiglu_special_cases():
    s = 1.0
    zero = bits_of(torch.zeros(8, dtype=torch.bfloat16))
    u = bits_of(torch.linspace(-4, 4, 8).to(torch.bfloat16))
    h = oracle.silu_mul_2in(zero, u, s)
    assert np.all((h & 0x7F) == 0)  # SiLU(0) = 0
    # large positive g: SiLU(g) * u -> g * u; large negative g: -> 0
    g = bits_of(torch.full((8,), 40.0).to(torch.bfloat16))
    u = bits_of(torch.tensor([0.5, 1, 2, 3, -1, -2, 0.25, 5]).to(torch.bfloat16))
    h = oracle.silu_mul_2in(g, u, s)
    want = [oracle.quant_f64(40.0 * float(v), 1.0) for v in oracle.bf16_to_f64(u)]
    assert list(h) == want
    gneg = bits_of(torch.full((8,), -60.0).to(torch.bfloat16))
    assert np.all((oracle.silu_mul_2in(gneg, u, s) & 0x7F) == 0)


def test_swiglu_independent_sigmoid_form():
    """SiLU written another way: g * (1 + tanh(g/2)) / 2.  Codes agree except
    where the fp64 value lies within rounding noise of a code boundary."""
    d = synth.c2_swiglu(1024, 8192, device="cpu", n_calib=0)
    g = bits_of(d["g"][:16, :1024].contiguous())
    u = bits_of(d["u"][:16, :1024].contiguous())
    s = oracle.f32(0.02)
    h = oracle.silu_mul_2in(g, u, s)
    gv, uv = oracle.bf16_to_f64(g), oracle.bf16_to_f64(u)
    v = gv * (1.0 + np.tanh(gv / 2.0)) / 2.0 * uv / float(s)
    want = torch_e4m3(np.clip(v, -448, 448).astype(np.float32))
    # fp32 rounding of v may move a value across a tie; allow 1e-4 of elements
    assert (h != want).mean() < 1e-4


def test_swiglu_quantize_saturates():
    g = bits_of(torch.full((4,), 8.0).to(torch.bfloat16))
    u = bits_of(torch.tensor([100.0, -100.0, 1.0, -1.0]).to(torch.bfloat16))
    h = oracle.silu_mul_2in(g, u, 0.5)
    assert list(h[:2]) == [0x7E, 0xFE]


# ---------------------------------------------------- shared quant and groups


def test_shared_quant_equals_three_separate_quantizations():
    d = synth.c3_qkv(n_calib=0)
    x = bits_of(d["x"][:48].contiguous())
    s = oracle.f32(0.05)
    wqs = []
    for name in ("wq", "wk", "wv"):
        wq, sw = oracle.rtn_weight(bits_of(d[name][:40].contiguous()))
        wqs.append((wq, sw))
    shared = oracle.qkv_shared_quant(x, s, wqs)
    separate = [oracle.linear(oracle.quantize(x, s), wq, s, sw) for wq, sw in wqs]
    for a, b in zip(shared, separate):
        assert np.array_equal(a, b)


def test_shared_scale_invariant():
    s = np.float32(0.0123)
    assert oracle.shared_scales_equal([s, s, s])
    one_ulp = np.nextafter(s, np.float32(1))
    assert not oracle.shared_scales_equal([s, s, one_ulp])
    assert not oracle.shared_scales_equal([0.0, 0.0])
    assert not oracle.shared_scales_equal([np.inf, np.inf])
    assert not oracle.shared_scales_equal([-s, -s])


def test_golden_requant():
    """Hand-derived values of the fused loader's re-quantization
    qW' = q(s_i * deq(qW) / s_max) (pull request "Load static FP8 Cosmos3
    Nano/Super checkpoints without re-quantizing them", Description).  Each
    case's inverted ratio s_max * deq / s_i gives another code, so a swapped
    operand fails here."""
    for code, s_i, s_max, want in _golden("requant"):
        q = np.array([int(code, 16)], np.uint8)
        got = oracle.requant_group_member(q, float(s_i), float(s_max))
        assert int(got[0]) == int(want, 16), (code, s_i, s_max)


def test_fused_group_requant_changes_codes_split_keeps_them():
    """Group with genuinely different weight scales (asserted first): the
    fused loader's second rounding changes codes; the split path keeps the
    calibrated codes exactly."""
    wg = bits_of(synth.normal((64, 128), 0.02, 7))
    wu = bits_of(synth.normal((64, 128), 0.05, 8))
    qg, sg = oracle.rtn_weight(wg)
    qu, su = oracle.rtn_weight(wu)
    assert sg != su
    smax = max(sg, su)
    smin_q = qg if sg < su else qu
    s_small = min(sg, su)
    re = oracle.requant_group_member(smin_q, s_small, smax)
    assert (re != smin_q).any()
    # re-quantizing onto its own scale is the identity (the split path)
    assert np.array_equal(oracle.requant_group_member(smin_q, s_small, s_small), smin_q)


# --------------------------------------------------------------- gated MLP


def _c0_weights():
    d = synth.c0_mlp()
    wgq, swg = oracle.rtn_weight(bits_of(d["wg"]))
    wuq, swu = oracle.rtn_weight(bits_of(d["wu"]))
    wdq, swd = oracle.rtn_weight(bits_of(d["wd"]))
    calib = [bits_of(b) for b in d["calib"]]
    s_in = oracle.observer_scale(calib)
    s_down = oracle.down_scale(calib, bits_of(d["wg"]), bits_of(d["wu"]))
    return d, (s_in, wgq, swg, wuq, swu, s_down, wdq, swd)


def test_gated_mlp_row_independence():
    d, args = _c0_weights()
    x = bits_of(d["x"])
    y = oracle.gated_mlp(x, *args)
    rows = [0, 5, 17, 63]
    y_rows = oracle.gated_mlp(np.ascontiguousarray(x[rows]), *args)
    assert np.array_equal(y[rows], y_rows)


def test_gated_mlp_brute_force_tiny():
    """Independent composition from library routines on a tiny slice: torch
    casts for the quantizers, numpy fp64 matmuls, tanh-form SiLU.  Equal up to
    rare one-step differences of H near code boundaries."""
    d, (s_in, wgq, swg, wuq, swu, s_down, wdq, swd) = _c0_weights()
    x = bits_of(d["x"][:8].contiguous())
    y = oracle.gated_mlp(x, s_in, wgq, swg, wuq, swu, s_down, wdq, swd)
    cb = oracle.codebook()
    xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).float()
    xq = torch_e4m3((xf / torch.tensor(s_in)).numpy())
    g = ((cb[xq] @ cb[wgq].T) * (float(s_in) * float(swg)))
    u = ((cb[xq] @ cb[wuq].T) * (float(s_in) * float(swu)))
    g = torch.from_numpy(g).to(torch.bfloat16).double().numpy()
    u = torch.from_numpy(u).to(torch.bfloat16).double().numpy()
    hv = g * (1 + np.tanh(g / 2)) / 2 * u / float(s_down)
    hq = torch_e4m3(np.clip(hv, -448, 448).astype(np.float32))
    ref = torch.from_numpy((cb[hq] @ cb[wdq].T) * (float(s_down) * float(swd))).to(torch.bfloat16)
    ref = ref.double().numpy()
    yv = oracle.bf16_to_f64(y)
    rel = np.linalg.norm(yv - ref) / np.linalg.norm(ref)
    assert rel < 1e-2
    assert np.isfinite(yv).all() and np.abs(yv).max() > 0


# ---------------------------------------------------------- SwiGLU variants


def _gu(seed, rows=16, cols=512, gstd=3.0):
    g = bits_of(synth.normal((rows, cols), gstd, seed))
    u = bits_of(synth.normal((rows, cols), 2.0, seed + 1))
    return g, u


def test_swiglu_variant_defaults_equal_plain():
    """alpha = 1, beta = 0 and no limit is plain SwiGLU, bit for bit."""
    g, u = _gu(40)
    s = oracle.f32(0.017)
    assert np.array_equal(oracle.swiglu_2in(g, u, s), oracle.silu_mul_2in(g, u, s))


@pytest.mark.parametrize("alpha,beta,limit", [(1.702, 1.0, 7.0), (1.702, 0.0, None),
                                              (1.0, 1.0, None), (1.0, 0.0, 2.0)])
def test_swiglu_variant_two_input_equals_fused(alpha, beta, limit):
    g, u = _gu(41)
    s = oracle.f32(0.031)
    h2 = oracle.swiglu_2in(g, u, s, alpha, beta, limit)
    hf = oracle.swiglu_fused(np.concatenate([g, u], axis=1), s, alpha, beta, limit)
    assert np.array_equal(h2, hf)


def test_swiglu_variant_independent_form():
    """Same variant written another way (tanh-form sigmoid, numpy clamps)."""
    g, u = _gu(42)
    alpha, beta, limit, s = 1.702, 1.0, 7.0, oracle.f32(0.05)
    h = oracle.swiglu_2in(g, u, s, alpha, beta, limit)
    gv = np.minimum(oracle.bf16_to_f64(g), limit)
    uv = np.clip(oracle.bf16_to_f64(u), -limit, limit)
    v = gv * (1.0 + np.tanh(alpha * gv / 2.0)) / 2.0 * (uv + beta) / float(s)
    want = torch_e4m3(np.clip(v, -448, 448).astype(np.float32))
    assert (h != want).mean() < 1e-3
    # and each term matters: dropping the offset, the gain or the clamp changes codes
    assert not np.array_equal(h, oracle.swiglu_2in(g, u, s, alpha, 0.0, limit))
    assert not np.array_equal(h, oracle.swiglu_2in(g, u, s, 1.0, beta, limit))
    assert not np.array_equal(h, oracle.swiglu_2in(g, u, s, alpha, beta, None))


def test_swiglu_variant_closed_forms():
    s = 1.0
    big = bits_of(torch.full((4,), 20.0).to(torch.bfloat16))
    one = bits_of(torch.full((4,), 1.0).to(torch.bfloat16))
    # the clamp: gate 20 limited to 7, up 1: 7 sigmoid(7 alpha) (1 + beta)
    h = oracle.swiglu_2in(big, one, s, 1.702, 1.0, 7.0)
    want = oracle.quant_f64(7.0 / (1.0 + np.exp(-7.0 * np.float32(1.702).item())) * 2.0, 1.0)
    assert np.all(h == want)
    # up equal to -beta gives zero
    neg = bits_of(torch.full((4,), -1.0).to(torch.bfloat16))
    assert np.all((oracle.swiglu_2in(one, neg, s, 1.0, 1.0, None) & 0x7F) == 0)


# ------------------------------------------------------ attention projections


def test_cross_attention_reduces_to_self_attention():
    """With ctx = x and equal scales the cross-attention projections are the
    shared-quant Q/K/V; with a different context K and V change, Q does not."""
    d = synth.c3_qkv(n_calib=0)
    x = bits_of(d["x"][:24].contiguous())
    ctx = bits_of(d["x"][100:124].contiguous())
    s = oracle.f32(0.04)
    proj = [oracle.rtn_weight(bits_of(d[n][:32].contiguous())) for n in ("wq", "wk", "wv")]
    self_q, self_k, self_v = oracle.qkv_shared_quant(x, s, proj)
    q, k, v = oracle.cross_attention_qkv(x, x, s, proj[0], s, proj[1], proj[2])
    assert np.array_equal(q, self_q) and np.array_equal(k, self_k) and np.array_equal(v, self_v)
    q2, k2, v2 = oracle.cross_attention_qkv(x, ctx, s, proj[0], oracle.f32(0.05), proj[1], proj[2])
    assert np.array_equal(q2, self_q)
    assert not np.array_equal(k2, self_k) and not np.array_equal(v2, self_v)
    # K from ctx equals a plain quantize-then-Linear of ctx at s_kv
    assert np.array_equal(k2, oracle.linear(oracle.quantize(ctx, oracle.f32(0.05)), *proj[1][:1],
                                            oracle.f32(0.05), proj[1][1]))


# ------------------------------------------- per-channel / per-token scales


def test_quantize_rows_is_per_row_rtn():
    """Each row is its own RTN tensor: same codes and scale as rtn_weight on
    that row alone; an all-zero row gets scale 1 and zero codes."""
    w = bits_of(synth.normal((12, 200), 0.3, 61))
    w[5] = 0
    q, s = oracle.quantize_rows(w)
    for r in range(12):
        if r == 5:
            assert s[r] == 1.0 and np.all(q[r] == 0)
            continue
        qr, sr = oracle.rtn_weight(np.ascontiguousarray(w[r]))
        assert sr == s[r] and np.array_equal(qr, q[r])
        assert (q[r] & 0x7F).max() == 0x7E   # each row reaches the largest code


def test_linear_scaled_reduces_to_per_tensor():
    rng = np.random.default_rng(62)
    xq = rng.integers(0, 0x7E, size=(7, 64), dtype=np.uint8)
    wq = rng.integers(0, 0x7E, size=(9, 64), dtype=np.uint8) | 0x80
    a, b = oracle.f32(0.3), oracle.f32(0.002)
    ref = oracle.linear(xq, wq, a, b)
    assert np.array_equal(oracle.linear_scaled(xq, wq, a, b), ref)
    assert np.array_equal(oracle.linear_scaled(xq, wq, np.full(7, a, np.float32),
                                               np.full(9, b, np.float32)), ref)
    # a per-row scale multiplies that row only; a per-column scale that column only
    sx = np.full(7, a, np.float32)
    sx[3] *= 2
    y = oracle.linear_scaled(xq, wq, sx, b)
    assert np.array_equal(y[:3], ref[:3]) and np.array_equal(y[4:], ref[4:])
    assert np.array_equal(oracle.bf16_to_f64(y[3]), 2 * oracle.bf16_to_f64(ref[3]))
    sw = np.full(9, b, np.float32)
    sw[6] *= 4
    y = oracle.linear_scaled(xq, wq, a, sw)
    assert np.array_equal(oracle.bf16_to_f64(y[:, 6]), 4 * oracle.bf16_to_f64(ref[:, 6]))
    assert np.array_equal(np.delete(y, 6, axis=1), np.delete(ref, 6, axis=1))


def test_silu_mul_rows_uses_each_rows_maximum():
    g, u = _gu(63, rows=6, cols=300)
    h, s = oracle.silu_mul_2in_rows(g, u)
    v = oracle.silu_mul_f64(oracle.bf16_to_f64(g), oracle.bf16_to_f64(u))
    for r in range(6):
        assert s[r] == np.float32(np.abs(v[r]).max() / 448.0)
        assert np.array_equal(h[r], oracle.silu_mul_2in(np.ascontiguousarray(g[r]),
                                                        np.ascontiguousarray(u[r]), float(s[r])))
        assert (h[r] & 0x7F).max() == 0x7E


def test_gated_mlp_per_token_rows_and_weight_channels():
    """Per-token scales make every output row depend on its own input row only
    (a row keeps its result when computed alone or beside other rows), and a
    weight channel's scale multiplies that channel's output exactly: doubling
    the down projection's scale of one output channel doubles that column and
    leaves the others."""
    d = synth.c0_mlp()
    wg, swg = oracle.quantize_rows(bits_of(d["wg"]))
    wu, swu = oracle.quantize_rows(bits_of(d["wu"]))
    wd, swd = oracle.quantize_rows(bits_of(d["wd"]))
    x = bits_of(d["x"])
    y = oracle.gated_mlp_per_token(x, wg, swg, wu, swu, wd, swd)
    rows = [2, 9, 40]
    y_rows = oracle.gated_mlp_per_token(np.ascontiguousarray(x[rows]), wg, swg, wu, swu, wd, swd)
    assert np.array_equal(y[rows], y_rows)
    swd2 = swd.copy()
    swd2[7] *= 2
    y2 = oracle.gated_mlp_per_token(x, wg, swg, wu, swu, wd, swd2)
    assert np.array_equal(oracle.bf16_to_f64(y2[:, 7]), 2 * oracle.bf16_to_f64(y[:, 7]))
    assert np.array_equal(np.delete(y2, 7, axis=1), np.delete(y, 7, axis=1))


def test_down_scales_match_an_independent_composition():
    """With one calibration batch the moving average is that batch's maximum,
    so the down_proj scale is fp32(max|SiLU(X Wg^T) * (X Wu^T)| / 448): checked
    against torch's fp64 matmul and the x * sigmoid(x) form of SiLU.  Swapping
    gate and up changes it (SiLU belongs to the gate)."""
    d = synth.c0_mlp()
    x, wg, wu = d["calib"][0], d["wg"], d["wu"]
    s = oracle.down_scale([bits_of(x)], bits_of(wg), bits_of(wu))
    g = x.double() @ wg.double().T
    u = x.double() @ wu.double().T
    want = float((g * torch.sigmoid(g) * u).abs().max()) / 448.0
    assert abs(s - want) <= 2.0 ** -22 * want          # one fp32 rounding of the same value
    swapped = oracle.down_scale([bits_of(x)], bits_of(wu), bits_of(wg))
    assert swapped != s
    gg = synth.normal((64, 300), 2.0, 71)
    uu = synth.normal((64, 300), 1.0, 72)
    s2 = oracle.swiglu_down_scale([(bits_of(gg), bits_of(uu))])
    want2 = float((gg.double() * torch.sigmoid(gg.double()) * uu.double()).abs().max()) / 448.0
    assert abs(s2 - want2) <= 2.0 ** -22 * want2


def test_silu_mul_f64_identities():
    """The fp64 SiLU(g)*u the per-row SwiGLU scales come from, pinned by two
    identities of the function: SiLU(x) - SiLU(-x) = x (as sigmoid(x) +
    sigmoid(-x) = 1), over the full range, and SiLU(x) = (x/2)(1 + tanh(x/2)),
    evaluated with numpy's tanh rather than the oracle's exp, where that form
    does not cancel; u scales the product."""
    rng = np.random.default_rng(71)
    x = np.concatenate([rng.normal(0.0, 3.0, 500), [0.0, 1e-300, -1e-300, 30.0, -30.0, 700.0]])
    one = np.ones_like(x)
    pos = oracle.silu_mul_f64(x, one)
    neg = oracle.silu_mul_f64(-x, one)
    assert np.allclose(pos - neg, x, rtol=1e-13, atol=1e-300)
    # the tanh form cancels for large negative x (1 + tanh(x/2) -> 0): compared where |x| <= 8
    m = np.abs(x) <= 8.0
    assert np.allclose(pos[m], 0.5 * x[m] * (1.0 + np.tanh(0.5 * x[m])), rtol=1e-12, atol=1e-300)
    u = rng.normal(0.0, 1.0, x.size)
    assert np.allclose(oracle.silu_mul_f64(x, u), pos * u, rtol=1e-15, atol=0.0)
    assert oracle.silu_mul_f64(np.array([0.0]), np.array([5.0]))[0] == 0.0
