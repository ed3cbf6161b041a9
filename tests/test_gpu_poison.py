"""Every output element is written: outputs are filled with a NaN pattern
(0xFF bytes: a NaN BF16 and the NaN E4M3 code) before each call, on ragged
and tile-boundary shapes.  The inputs are finite, so a valid output is never
NaN (the FP8 conversion saturates), and a NaN left behind is an element the
kernels did not write."""

import pytest
import torch

import fp8_w8a8_static_b200 as fw
import synth
from _util import scalar

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _poisoned(shape, dtype):
    t = torch.empty(shape, dtype=dtype, device=DEV)
    t.view(torch.uint8).fill_(0xFF)
    return t


def _assert_written(*outs):
    torch.cuda.synchronize()
    for t in outs:
        if t.dtype == fw.FP8:
            assert not bool(((t.view(torch.uint8) & 0x7F) == 0x7F).any()), "unwritten FP8 codes"
        else:
            assert not bool(torch.isnan(t.float()).any()), "unwritten BF16 elements"
    assert fw.device_status()[0] == fw.OK


def _w(n, k, seed):
    return fw.fp8_rtn_quantize_weight(synth.normal((n, k), 0.02, seed, DEV))


SHAPES = [(1, 16, 32), (129, 264, 144), (255, 520, 272), (257, 1024, 512), (1000, 3072, 128)]


@pytest.fixture(params=["auto", "pair256", "cta256", "cta128", "cta64"])
def gemm_config(request):
    fw.set_gemm_config(request.param)
    yield request.param
    fw.set_gemm_config("auto")


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_quant_and_linear(M, N, K, gemm_config):
    x = synth.normal((M, K), 1.0, M + K, DEV)
    xq = fw.fp8_quant_static(x, scalar(0.01, DEV), out=_poisoned((M, K), fw.FP8))
    wq, s_w = _w(N, K, N)
    y = fw.fp8_linear_static(xq, wq, scalar(0.01, DEV), s_w, out=_poisoned((M, N), torch.bfloat16))
    _assert_written(xq, y)


@pytest.mark.parametrize("M,N,K", SHAPES + [(300, 520, 8208)])  # the last: long enough to split
def test_linear_split_k_and_group(M, N, K):
    x = synth.normal((M, K), 1.0, M + 2 * K, DEV)
    xq = fw.fp8_quant_static(x, scalar(0.01, DEV))
    wq, s_w = _w(N, K, N + 1)
    y = fw.fp8_linear_static_ws(xq, wq, scalar(0.01, DEV), s_w,
                                out=_poisoned((M, N), torch.bfloat16))
    probs = [(xq, wq, scalar(0.01, DEV), s_w), (xq[: max(M // 3, 1)], wq, scalar(0.02, DEV), s_w)]
    outs = [_poisoned((p[0].shape[0], N), torch.bfloat16) for p in probs]
    fw.fp8_linear_static_group(probs, outs=outs, split_k=True)
    _assert_written(y, *outs)


@pytest.mark.parametrize("M,I,K", [(1, 16, 32), (129, 400, 272), (300, 1024, 512),
                                   (513, 12288, 256)])
def test_swiglu_and_gate_up(M, I, K):
    g = synth.normal((M, I), 2.0, 1, DEV)
    u = synth.normal((M, I), 1.0, 2, DEV)
    h1 = fw.silu_mul_2in_fp8(g, u, scalar(0.01, DEV), out=_poisoned((M, I), fw.FP8))
    h2 = fw.swiglu_2in_fp8(g, u, scalar(0.01, DEV), fw.swiglu(1.702, 1.0, 7.0),
                           out=_poisoned((M, I), fw.FP8))
    xq = fw.fp8_quant_static(synth.normal((M, K), 1.0, 3, DEV), scalar(0.01, DEV))
    wg, s_wg = _w(I, K, 4)
    wu, s_wu = _w(I, K, 5)
    h3 = fw.fp8_gate_up_swiglu_static(xq, wg, wu, scalar(0.01, DEV), s_wg, s_wu, scalar(0.003, DEV),
                                      out=_poisoned((M, I), fw.FP8))
    probs = [(xq, wg, wu, scalar(0.01, DEV), s_wg, s_wu, scalar(0.003, DEV)),
             (xq[: max(M // 2, 1)], wg, wu, scalar(0.02, DEV), s_wg, s_wu, scalar(0.004, DEV))]
    hs = fw.fp8_gate_up_swiglu_static_group(
        probs, outs=[_poisoned((p[0].shape[0], I), fw.FP8) for p in probs])
    _assert_written(h1, h2, h3, *hs)


@pytest.mark.parametrize("M0,M1,d,I", [(129, 1, 272, 400), (300, 64, 256, 704)])
def test_composite_blocks(M0, M1, d, I):
    towers = []
    for j, M in enumerate((M0, M1)):
        t = dict(x=synth.normal((M, d), 1.0, 10 + j, DEV), s_in=scalar(0.01, DEV),
                 s_down=scalar(0.004, DEV))
        for name, shape, k in (("wg", (I, d), 1), ("wu", (I, d), 2), ("wd", (d, I), 3)):
            t[name], t["s_" + name] = _w(*shape, 20 * j + k)
        towers.append(t)
    ys = fw.gated_mlp_static_fp8_group(towers, outs=[_poisoned((M, d), torch.bfloat16)
                                                    for M in (M0, M1)])
    t = towers[0]
    args = (t["x"], t["s_in"], t["wg"], t["s_wg"], t["wu"], t["s_wu"], t["s_down"], t["wd"], t["s_wd"])
    y1 = fw.gated_mlp_static_fp8(*args, out=_poisoned((M0, d), torch.bfloat16))
    y2 = fw.gated_mlp_static_fp8_fused(*args, out=_poisoned((M0, d), torch.bfloat16))
    wq, s_wq = _w(264, d, 31)
    wk, s_wk = _w(128, d, 32)
    wv, s_wv = _w(128, d, 33)
    qkv = fw.qkv_shared_quant(t["x"], t["s_in"], wq, s_wq, wk, s_wk, wv, s_wv,
                              out=tuple(_poisoned((M0, n), torch.bfloat16) for n in (264, 128, 128)))
    ctx = towers[1]["x"]
    xa = fw.cross_attention_qkv_static_fp8(
        t["x"], ctx, t["s_in"], wq, s_wq, scalar(0.02, DEV), wk, s_wk, wv, s_wv,
        out=(_poisoned((M0, 264), torch.bfloat16), _poisoned((M1, 128), torch.bfloat16),
             _poisoned((M1, 128), torch.bfloat16)))
    _assert_written(*ys, y1, y2, *qkv, *xa)


@pytest.mark.parametrize("M,N,K", [(129, 264, 144), (300, 1024, 512)])
def test_per_token_path(M, N, K):
    x = synth.normal((M, K), 1.0, 40, DEV)
    xq, sx = fw.fp8_quant_per_token(x, out=_poisoned((M, K), fw.FP8))
    wq, sw = fw.fp8_quant_per_token(synth.normal((N, K), 0.02, 41, DEV))
    y = fw.fp8_linear_scaled(xq, wq, sx, sw, out=_poisoned((M, N), torch.bfloat16))
    g = synth.normal((M, N), 2.0, 42, DEV)
    u = synth.normal((M, N), 1.0, 43, DEV)
    h, sh = fw.silu_mul_2in_fp8_per_token(g, u, out=_poisoned((M, N), fw.FP8))
    _assert_written(xq, y, h)
