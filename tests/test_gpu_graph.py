"""The hot-path calls are asynchronous on the caller's stream and can be
captured into a CUDA graph: a captured call replays to the same bits as the
eager call (the kernels' programmatic-launch edges survive capture)."""

import pytest
import torch

import fp8_w8a8_static_b200 as fw
import synth
from _util import scalar

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _tower(M, d, I, seed, s_down):
    x = synth.activation_with_outliers(M, d, 9, seed, 0, DEV)
    t = dict(x=x, s_in=fw.fp8_observer_scale(fw.fp8_absmax_bf16(x)), s_down=scalar(s_down, DEV))
    for name, shape, k in (("wg", (I, d), 1), ("wu", (I, d), 2), ("wd", (d, I), 3)):
        t[name], t["s_" + name] = fw.fp8_rtn_quantize_weight(
            synth.normal(shape, 0.02, seed * 7 + k, DEV))
    return t


@pytest.mark.parametrize("M0,M1,d,I", [(4096, 1024, 3072, 12288), (200, 64, 256, 704)])
def test_group_mlp_graph_replay_equals_eager(M0, M1, d, I):
    towers = [_tower(M0, d, I, 1, 0.003), _tower(M1, d, I, 2, 0.0035)]
    ws = torch.empty(fw.gated_mlp_static_fp8_group_workspace([M0, M1], d, I), dtype=torch.uint8,
                     device=DEV)
    eager = [y.clone() for y in fw.gated_mlp_static_fp8_group(towers, workspace=ws)]
    outs = [torch.empty_like(y) for y in eager]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # one call outside capture: per-device set-up happens here
        fw.gated_mlp_static_fp8_group(towers, workspace=ws, outs=outs, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for o in outs:
        o.zero_()
    g = torch.cuda.CUDAGraph()
    n0 = fw.launch_count()
    with torch.cuda.graph(g):
        fw.gated_mlp_static_fp8_group(towers, workspace=ws, outs=outs)
    assert fw.launch_count() - n0 == 3  # quantize, gate/up + SwiGLU, down: captured, not run
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for o, e in zip(outs, eager):
        assert torch.equal(o, e)
    assert fw.device_status()[0] == fw.OK


def test_fused_mlp_and_qkv_graph_replay():
    d, I, M = 256, 704, 64
    t = _tower(M, d, I, 5, 0.004)
    ws = torch.empty(fw.gated_mlp_static_fp8_fused_workspace(M, d, I), dtype=torch.uint8,
                     device=DEV)
    eager = fw.gated_mlp_static_fp8_fused(t["x"], t["s_in"], t["wg"], t["s_wg"], t["wu"],
                                          t["s_wu"], t["s_down"], t["wd"], t["s_wd"], workspace=ws)
    wq, s_wq = fw.fp8_rtn_quantize_weight(synth.normal((d, d), 0.02, 9, DEV))
    q_eager = fw.qkv_shared_quant(t["x"], t["s_in"], wq, s_wq, wq, s_wq, wq, s_wq)
    torch.cuda.synchronize()
    y = torch.empty_like(eager)
    qws = torch.empty(fw.qkv_shared_quant_workspace(M, d), dtype=torch.uint8, device=DEV)
    qo = [torch.empty_like(v) for v in q_eager]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fw.gated_mlp_static_fp8_fused(t["x"], t["s_in"], t["wg"], t["s_wg"], t["wu"], t["s_wu"],
                                      t["s_down"], t["wd"], t["s_wd"], workspace=ws, out=y)
        fw.qkv_shared_quant(t["x"], t["s_in"], wq, s_wq, wq, s_wq, wq, s_wq, workspace=qws,
                            out=qo)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, eager)
    for a, b in zip(qo, q_eager):
        assert torch.equal(a, b)
