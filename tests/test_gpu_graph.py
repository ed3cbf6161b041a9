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


@pytest.mark.parametrize("form", ["staged", "stream"])
def test_quantizer_forms_graph_replay(form):
    """Both forms of the quantizer, captured in a graph as the first step of
    the grouped gated MLP and on their own, replay to the eager codes; the
    staged form's mbarrier ring and bulk copies are set up anew in every
    replayed launch."""
    fw.set_quant_form(form)
    try:
        M0, M1, d, I = 300, 96, 512, 1040
        towers = [_tower(M0, d, I, 11, 0.003), _tower(M1, d, I, 12, 0.0035)]
        # 6,408,693 values: 783 chunks of 16 KB in the staged form, the last partial, and a
        # 5-value tail past the last whole vector
        x = synth.activation_with_outliers(1031, 6216, 4, 13, 0, DEV).flatten()[:-3]
        s = scalar(0.021, DEV)
        ws = torch.empty(fw.gated_mlp_static_fp8_group_workspace([M0, M1], d, I),
                         dtype=torch.uint8, device=DEV)
        eager = [y.clone() for y in fw.gated_mlp_static_fp8_group(towers, workspace=ws)]
        q_eager = fw.fp8_quant_static(x, s).clone()
        torch.cuda.synchronize()
        outs = [torch.empty_like(y) for y in eager]
        q = torch.empty_like(q_eager)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fw.gated_mlp_static_fp8_group(towers, workspace=ws, outs=outs)
            fw.fp8_quant_static(x, s, out=q)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        for o, e in zip(outs, eager):
            assert torch.equal(o, e)
        assert torch.equal(q.view(torch.uint8), q_eager.view(torch.uint8))
        assert fw.device_status()[0] == fw.OK
    finally:
        fw.set_quant_form("auto")
