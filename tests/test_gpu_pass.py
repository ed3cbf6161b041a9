"""The benchmark's own pass against the oracle.

The 36-layer two-tower decoder-MLP pass is built exactly as bench.py builds
it: its synthetic checkpoint (RTN FP8 weights and moving-average input scales
made by the library's load-time calls), one grouped composite call per layer
with the towers in the benchmark's order, and the step captured as a CUDA
graph and replayed.  Every output is poisoned with NaN before the replay, so
what is checked was written by the replay.  Stratified rows of the first, a
middle and the last layer of both towers are compared with the oracle, which
is handed the inputs, codes and scales the device holds (the RTN codes and
scales themselves are checked against the oracle in test_gpu_blocks)."""

import numpy as np
import pytest
import torch

import bench
import fp8_w8a8_static_b200 as fw
import oracle
from _util import GEMM_REL_FRO, bits, codes, rel_fro, stratified_rows

pytestmark = pytest.mark.gpu
CHECKED_LAYERS = (0, 17, 35)


def test_benchmark_pass_against_oracle():
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    fw.load()
    layers = bench.prepare(fw, device, bench.LAYERS, lambda m: None)
    ws, _ = bench.make_buffers(fw, layers, device, fused=True, grouped=True)
    stream = torch.cuda.current_stream(device)
    value_plan, keep = bench.build_group_value_plan(fw, layers, ws, stream.cuda_stream)
    assert len(value_plan) == bench.LAYERS   # one grouped call per layer

    def run_current():
        h = torch.cuda.current_stream().cuda_stream
        for _, fn, a, _, _ in value_plan:
            assert fn(*(a[:-1] + (h,))) == fw.OK

    graph = bench.capture_graph(run_current)
    for L in layers:
        L.y.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert fw.device_status()[0] == fw.OK
    checked = 0
    for L in layers:
        assert torch.isfinite(L.y.float()).all(), (L.index, L.tower)
        if L.index not in CHECKED_LAYERS:
            continue
        rows = stratified_rows(L.M, 100 * L.index + L.M)
        ref = oracle.gated_mlp(np.ascontiguousarray(bits(L.x)[rows]), L.s_in.item(),
                               codes(L.wg), L.s_wg.item(), codes(L.wu), L.s_wu.item(),
                               L.s_down.item(), codes(L.wd), L.s_wd.item())
        rf = rel_fro(bits(L.y)[rows], ref)
        assert rf <= GEMM_REL_FRO, (L.index, L.tower, rf)
        checked += 1
    assert checked == 2 * len(CHECKED_LAYERS)
    del graph, keep
    torch.cuda.empty_cache()
