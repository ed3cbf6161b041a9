"""gated_mlp_static_fp8_noalloc: the gated MLP for callers that cannot
allocate device memory when they call it (an inference-engine plugin whose
enqueue step may not allocate, a process that gave all device memory to its
own pool at start-up).  It runs out of a fixed scratch area the library
reserves on each GPU instead of a caller-supplied workspace.

Called through the C ABI and checked against the regular entry point (which
takes a workspace) within the tolerance the other tests use, on two calls in
a row, so that the second call cannot lean on what the first one left behind
in the shared scratch area.  This file sorts last so that a run that stops at
the first failure has already run every other test."""

import numpy as np
import pytest
import torch

import fp8_w8a8_static_b200 as fw
import synth
from _util import GEMM_REL_FRO, bits, rel_fro, scalar

pytestmark = pytest.mark.gpu
DEV = "cuda"
MAX_BYTES = 64 * 1024 * 1024


def _weights(d, I, seed):
    wg = fw.fp8_rtn_quantize_weight(synth.normal((I, d), 0.02, seed, DEV))
    wu = fw.fp8_rtn_quantize_weight(synth.normal((I, d), 0.02, seed + 1, DEV))
    wd = fw.fp8_rtn_quantize_weight(synth.normal((d, I), 0.02, seed + 2, DEV))
    return wg, wu, wd


def _noalloc(x, s_in, wg, wu, s_down, wd):
    lib = fw.load()
    M, d = x.shape
    I = wg[0].shape[0]
    y = torch.empty((M, d), dtype=torch.bfloat16, device=DEV)
    rc = lib.gated_mlp_static_fp8_noalloc(
        x.data_ptr(), M, d, I, s_in.data_ptr(), wg[0].data_ptr(), wg[1].data_ptr(),
        wu[0].data_ptr(), wu[1].data_ptr(), s_down.data_ptr(), wd[0].data_ptr(),
        wd[1].data_ptr(), y.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == fw.OK, fw.STATUS.get(rc)
    return y


def _with_workspace(x, s_in, wg, wu, s_down, wd):
    return fw.gated_mlp_static_fp8(x, s_in, *wg, *wu, s_down, *wd)


@pytest.mark.parametrize("M,d,I", [(64, 256, 704), (1024, 3072, 12288)])
def test_matches_workspace_entry_point_twice(M, d, I):
    assert fw.gated_mlp_static_fp8_workspace(M, d, I) <= MAX_BYTES
    wg, wu, wd = _weights(d, I, 40 + M)
    s_in, s_down = scalar(0.02, DEV), scalar(0.004, DEV)
    outs = []
    for call in range(2):
        # a different input each call: the second result must not depend on
        # what the first call left in the shared scratch area
        x = synth.activation_with_outliers(M, d, 7, call, 0, DEV)
        y_noalloc = _noalloc(x, s_in, wg, wu, s_down, wd)
        y_ref = _with_workspace(x, s_in, wg, wu, s_down, wd)
        torch.cuda.synchronize()
        assert rel_fro(bits(y_noalloc), bits(y_ref)) <= GEMM_REL_FRO
        assert torch.isfinite(y_noalloc.float()).all()
        outs.append(bits(y_noalloc))
    assert not np.array_equal(outs[0], outs[1])
    assert fw.device_status()[0] == fw.OK


def test_refuses_sizes_beyond_the_scratch_area():
    lib = fw.load()
    M, d, I = 2048, 3072, 12288  # needs about 132 MB of scratch
    assert fw.gated_mlp_static_fp8_workspace(M, d, I) > MAX_BYTES
    n0 = fw.launch_count()
    a = 1 << 20  # never dereferenced: the size check comes first
    rc = lib.gated_mlp_static_fp8_noalloc(a, M, d, I, a, a, a, a, a, a, a, a, a, None)
    assert rc == fw.ERR_SHAPE
    assert fw.launch_count() == n0
