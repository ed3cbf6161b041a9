"""fp8_linear_static on the GPU against the oracle's exact fp64 sum.

Bar: relative Frobenius error <= 1e-2 (the stated requirement), and every
element within one BF16 step plus a worst-case fp32 accumulation error."""

import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import fp8_w8a8_static_b200 as fw
import oracle
import synth
from _util import (GEMM_REL_FRO, bits, from_codes, gemm_elementwise_bound_ok, rel_fro, scalar,
                   stratified_rows)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _random_codes(rng, shape, spread=1.0):
    """Codes of N(0, spread) values quantized at unit scale: realistic mix."""
    v = (rng.standard_normal(shape) * spread).astype(np.float32)
    b = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return oracle.quantize(b, 1.0 / 64)


def _run(xq, wq, s_in, s_w, rows=None):
    y = fw.fp8_linear_static(from_codes(xq, DEV), from_codes(wq, DEV), scalar(s_in, DEV),
                             scalar(s_w, DEV))
    yb = bits(y)
    if rows is not None:
        xq = np.ascontiguousarray(xq[rows])
        yb = np.ascontiguousarray(yb[rows])
    ref = oracle.linear(xq, wq, s_in, s_w)
    absref = oracle.linear(xq & 0x7F, wq & 0x7F, s_in, s_w)
    K = xq.shape[1]
    assert rel_fro(yb, ref) <= GEMM_REL_FRO
    ok = gemm_elementwise_bound_ok(yb, ref, absref, K)
    assert ok.all(), f"{(~ok).sum()} elements outside the bound"
    return yb, ref


@pytest.fixture(params=["auto", "pair256", "cta256", "cta128", "cta64"])
def gemm_config(request):
    fw.set_gemm_config(request.param)
    yield request.param
    fw.set_gemm_config("auto")


@pytest.mark.parametrize("M,N,K", [
    (1, 8, 16),          # smallest legal problem
    (64, 704, 256),      # tiny-MLP gate/up
    (64, 256, 704),      # tiny-MLP down (K tail: 704 = 5.5 x 128)
    (127, 264, 144),     # ragged everything
    (129, 512, 128),     # one row past a tile
    (256, 2048, 2048),   # one full K sweep, narrow-tile dispatch
    (300, 1000, 272),
    (1024, 4096, 512),   # widest-tile dispatch
])
def test_shapes(M, N, K, gemm_config):
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    xq = _random_codes(rng, (M, K))
    wq = _random_codes(rng, (N, K), 0.5)
    _run(xq, wq, oracle.f32(0.013), oracle.f32(0.0021))


def test_zero_rows():
    xq = torch.empty((0, 64), dtype=fw.FP8, device=DEV)
    wq = torch.zeros((16, 64), dtype=fw.FP8, device=DEV)
    y = fw.fp8_linear_static(xq, wq, scalar(1.0, DEV), scalar(1.0, DEV))
    assert y.shape == (0, 16)


def test_extreme_codes_no_overflow(gemm_config):
    """Largest codes everywhere: 448*448*K stays finite in fp32."""
    M, N, K = 128, 256, 512
    xq = np.full((M, K), 0x7E, np.uint8)
    wq = np.full((N, K), 0xFE, np.uint8)
    yb, ref = _run(xq, wq, oracle.f32(1e-6), oracle.f32(1e-3))
    assert np.array_equal(yb, ref)


def test_integer_exact():
    """Integer codes with unit scales: every output is an exact small integer."""
    rng = np.random.default_rng(3)
    ints = [c for c, v in enumerate(oracle.codebook()) if np.isfinite(v) and v == int(v) and abs(v) <= 2]
    xq = rng.choice(np.array(ints, np.uint8), size=(200, 32))
    wq = rng.choice(np.array(ints, np.uint8), size=(136, 32))
    yb, ref = _run(xq, wq, 1.0, 1.0)
    assert np.array_equal(yb, ref)


@pytest.mark.parametrize("M", synth.C1_M)
@pytest.mark.parametrize("N", synth.C1_N)
def test_linear_sweep_full_size(M, N):
    """The single-Linear sweep at full size, checked on sampled rows (rows are
    independent, so a row of Y depends only on its row of Xq)."""
    d = synth.c1_linear(M, N, device=DEV, calib_rows=64)
    s_in = oracle.observer_scale([bits(b) for b in d["calib"]])
    wq, s_w = oracle.rtn_weight(bits(d["w"]))
    xq = oracle.quantize(bits(d["x"]), s_in)
    rows = stratified_rows(M, M + N)
    _run(xq, wq, s_in, s_w, rows=rows)



# ------------------------------------------------------------------ split-K


@pytest.mark.parametrize("M,N,K", [
    (1024, 3072, 12288),   # understanding-tower down projection: 48 tiles, all split
    (4096, 3072, 12288),   # generation-tower down projection: 2 full waves + 44 split tiles
    (300, 520, 8208),      # ragged M, N and K (65 K steps, the last partial): split 4 ways
    (2048, 1024, 3072),    # K/V projection shape: 24 K steps, too few to split
    (300, 520, 1040),      # ragged, 9 K steps: not split
    (64, 256, 704),
])
def test_split_k_against_oracle(M, N, K):
    rng = np.random.default_rng(M + N + K)
    xq = _random_codes(rng, (M, K))
    wq = _random_codes(rng, (N, K), 0.5)
    s_in, s_w = oracle.f32(0.013), oracle.f32(0.0021)
    y = fw.fp8_linear_static_ws(from_codes(xq, DEV), from_codes(wq, DEV), scalar(s_in, DEV),
                                scalar(s_w, DEV))
    rows = stratified_rows(M, 1)
    yb = bits(y)[rows]
    ref = oracle.linear(np.ascontiguousarray(xq[rows]), wq, s_in, s_w)
    absref = oracle.linear(np.ascontiguousarray(xq[rows]) & 0x7F, wq & 0x7F, s_in, s_w)
    assert rel_fro(yb, ref) <= GEMM_REL_FRO
    assert gemm_elementwise_bound_ok(yb, ref, absref, K).all()
    # deterministic: the same bits on a second call, with counters reused
    y2 = fw.fp8_linear_static_ws(from_codes(xq, DEV), from_codes(wq, DEV), scalar(s_in, DEV),
                                 scalar(s_w, DEV))
    assert torch.equal(y, y2)
    assert fw.device_status()[0] == fw.OK


@pytest.mark.parametrize("split", [False, True])
def test_long_k(split):
    """K = 65536, 512 K steps per tile: the K coordinates and, with the
    workspace, a 4-way split at the far end of the allowed range.  The oracle's
    fp64 sum stays exact (448^2 * 2^16 < 2^35 at a granularity of 2^-18)."""
    M, N, K = 300, 264, 65536
    rng = np.random.default_rng(K)
    xq = _random_codes(rng, (M, K))
    wq = _random_codes(rng, (N, K), 0.5)
    s_in, s_w = oracle.f32(0.013), oracle.f32(0.0021)
    args = (from_codes(xq, DEV), from_codes(wq, DEV), scalar(s_in, DEV), scalar(s_w, DEV))
    y = fw.fp8_linear_static_ws(*args) if split else fw.fp8_linear_static(*args)
    rows = stratified_rows(M, 5)
    yb = bits(y)[rows]
    xr = np.ascontiguousarray(xq[rows])
    ref = oracle.linear(xr, wq, s_in, s_w)
    absref = oracle.linear(xr & 0x7F, wq & 0x7F, s_in, s_w)
    assert rel_fro(yb, ref) <= GEMM_REL_FRO
    assert gemm_elementwise_bound_ok(yb, ref, absref, K).all()
    assert fw.device_status()[0] == fw.OK


def test_split_k_short_workspace_refused():
    xq = torch.zeros((256, 256), dtype=fw.FP8, device=DEV)
    ws = torch.empty(1024, dtype=torch.uint8, device=DEV)
    with pytest.raises(fw.FP8WSError):
        fw.fp8_linear_static_ws(xq, xq, scalar(1.0, DEV), scalar(1.0, DEV), workspace=ws)


# ----------------------------------------------------- ragged last wave: halves


@pytest.mark.parametrize("M,N,K", [
    (256, 19008, 256),   # 75 tiles: the 75th (64 columns) runs as halves, its second one empty
    (512, 19200, 512),   # 150 tiles: the last 2 run as halves, both halves full
    (2048, 3072, 3072),  # 96 tiles: 22 past the first wave, 44 halves (the c3 Q projection)
    (300, 520, 1040),    # 6 tiles, one partial wave: 12 units; the 8-column block's second half empty
    (96, 4104, 512),     # ragged M and N: 17 tiles, the last one 8 columns wide
])
def test_tail_halves_against_oracle(M, N, K):
    """Shapes whose tiles past the last full wave run as 256x128 halves (the
    plan is checked on the host first), against the oracle on every row or
    on stratified rows, under the per-element bound."""
    fw.set_gemm_config("pair256")
    try:
        tiles = -(-M // 256) * -(-N // 256)
        assert fw.split_plan(tiles, 74, -(-K // 128), scratch=False)["halves"] == 2
        rng = np.random.default_rng(M + N + K)
        xq = _random_codes(rng, (M, K))
        wq = _random_codes(rng, (N, K), 0.5)
        rows = stratified_rows(M, 3) if M * N * K > 2 ** 31 else None
        _run(xq, wq, oracle.f32(0.011), oracle.f32(0.0023), rows=rows)
    finally:
        fw.set_gemm_config("auto")
    assert fw.device_status()[0] == fw.OK


_HALVES_CHILD = textwrap.dedent("""
    import hashlib, sys
    import numpy as np, torch
    sys.path.insert(0, {root!r})
    sys.path.insert(0, {tests!r})
    import fp8_w8a8_static_b200 as fw
    from _util import from_codes, scalar
    fw.set_gemm_config("pair256")
    out = []
    for M, N, K in {shapes!r}:
        rng = np.random.default_rng(M * 31 + N * 7 + K)
        xq = rng.integers(0, 0x7F, (M, K), dtype=np.uint8) | (rng.integers(0, 2, (M, K), dtype=np.uint8) << 7)
        wq = rng.integers(0, 0x7F, (N, K), dtype=np.uint8) | (rng.integers(0, 2, (N, K), dtype=np.uint8) << 7)
        xq[(xq & 0x7F) == 0x7F] = 0x00   # no NaN codes
        wq[(wq & 0x7F) == 0x7F] = 0x00
        y = fw.fp8_linear_static(from_codes(xq, "cuda"), from_codes(wq, "cuda"), scalar(0.011, "cuda"),
                                 scalar(0.0023, "cuda"))
        out.append(hashlib.sha256(y.cpu().view(torch.int16).numpy().tobytes()).hexdigest())
    print(" ".join(out))
""")


def test_tail_halves_bit_identical_to_whole_tiles():
    """A 256 x 128 half (an N = 128 MMA over 64-row boxes of B) gives every
    element the bits the whole 256 x 256 tile gives: the same seeded GEMMs,
    run in a child process with the halves switched off (FP8WS_TAIL_HALVES=0,
    read once per process), hash to the same bytes."""
    shapes = [(300, 520, 1040), (2048, 3072, 3072), (256, 19008, 256)]
    for M, N, K in shapes:
        assert fw.split_plan(-(-M // 256) * -(-N // 256), 74, -(-K // 128), scratch=False)["halves"] == 2
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = _HALVES_CHILD.format(root=root, tests=os.path.join(root, "tests"), shapes=shapes)
    hashes = {}
    for halves in ("1", "0"):
        env = dict(os.environ, FP8WS_TAIL_HALVES=halves)
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600,
                           env=env)
        assert r.returncode == 0, r.stdout + r.stderr
        hashes[halves] = r.stdout.split()
    assert len(hashes["1"]) == len(shapes) and hashes["1"] == hashes["0"]


@pytest.mark.parametrize("x_rows,w_cols", [(False, False), (True, False), (False, True),
                                           (True, True)])
def test_tail_halves_vector_scales(x_rows, w_cols):
    """The four scale modes of the epilogue on half units: 300 x 520 (6 tiles,
    one partial wave, all run as halves), per-row and per-column scales
    checked against the oracle's fp64 sum on every element."""
    M, N, K = 300, 520, 272
    rng = np.random.default_rng(17 + 2 * x_rows + w_cols)
    xq = _random_codes(rng, (M, K))
    wq = _random_codes(rng, (N, K), 0.5)
    sx = (rng.uniform(0.5, 2.0, M if x_rows else 1) * 0.01).astype(np.float32)
    sw = (rng.uniform(0.5, 2.0, N if w_cols else 1) * 0.002).astype(np.float32)
    y = fw.fp8_linear_scaled(from_codes(xq, DEV), from_codes(wq, DEV),
                             torch.from_numpy(sx).to(DEV), torch.from_numpy(sw).to(DEV))
    ref = oracle.linear_scaled(xq, wq, sx, sw)
    assert rel_fro(bits(y), ref) <= GEMM_REL_FRO
    assert fw.device_status()[0] == fw.OK
