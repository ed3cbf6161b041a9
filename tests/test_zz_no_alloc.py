"""gated_mlp_static_fp8_noalloc: the gated MLP for callers that cannot
allocate device memory when they call it (an inference-engine plugin whose
enqueue step may not allocate, a process that gave all device memory to its
own pool at start-up).  It runs out of a fixed scratch area the library
reserves on each GPU instead of a caller-supplied workspace.

Called through the C ABI.  It runs the same kernels as the regular entry
point (which takes a workspace) on the same inputs, so the two outputs must be
identical bit for bit -- stricter than the GEMM tolerance the other tests use
-- on two calls in a row with different inputs, so that the second call
cannot lean on what the first one left behind in the shared scratch area.
Sampled rows are also checked against the oracle, the largest shape that fits
the scratch area runs, the first one that does not is refused before any
launch, and a fresh process whose first library call is this entry point
gets the same result.  This file sorts last so that a run that stops at the
first failure has already run every other test."""

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
from _util import GEMM_REL_FRO, bits, codes, rel_fro, scalar, stratified_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"
MAX_BYTES = 64 * 1024 * 1024
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


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


@pytest.mark.parametrize("M,d,I", [(64, 256, 704), (1024, 3072, 12288),
                                   (1040, 3072, 12288)])  # 1040: the largest M that fits
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
        assert torch.equal(y_noalloc.view(torch.int16), y_ref.view(torch.int16))
        assert torch.isfinite(y_noalloc.float()).all()
        outs.append(bits(y_noalloc))
    assert not np.array_equal(outs[0], outs[1])
    assert fw.device_status()[0] == fw.OK


def test_against_oracle_sampled_rows():
    """M = 1024, d = 3072, I = 12288 (the understanding tower's size): one
    sampled row in every 128-row slab, checked against the oracle."""
    M, d, I = 1024, 3072, 12288
    wg, wu, wd = _weights(d, I, 77)
    x = synth.activation_with_outliers(M, d, 7, 5, 0, DEV)
    s_in = fw.fp8_observer_scale(fw.fp8_absmax_bf16(x))
    s_down = scalar(0.0031, DEV)
    y = _noalloc(x, s_in, wg, wu, s_down, wd)
    torch.cuda.synchronize()
    rows = stratified_rows(M, 11)
    ref = oracle.gated_mlp(np.ascontiguousarray(bits(x)[rows]), s_in.item(), codes(wg[0]),
                           wg[1].item(), codes(wu[0]), wu[1].item(), s_down.item(),
                           codes(wd[0]), wd[1].item())
    assert rel_fro(bits(y)[rows], ref) <= GEMM_REL_FRO


@pytest.mark.parametrize("M", [1041, 2048])
def test_refuses_sizes_beyond_the_scratch_area(M):
    """M = 1041 is the first row count whose workspace (1041 * 64512 bytes at
    d = 3072, I = 12288) exceeds the 64 MiB area: refused before any launch."""
    lib = fw.load()
    d, I = 3072, 12288
    assert fw.gated_mlp_static_fp8_workspace(M, d, I) > MAX_BYTES
    n0 = fw.launch_count()
    a = 1 << 20  # never dereferenced: the size check comes first
    rc = lib.gated_mlp_static_fp8_noalloc(a, M, d, I, a, a, a, a, a, a, a, a, a, None)
    assert rc == fw.ERR_SHAPE
    assert fw.launch_count() == n0


_FRESH = textwrap.dedent("""
    import sys, torch
    sys.path.insert(0, {root!r})
    import fp8_w8a8_static_b200 as fw
    dev = "cuda"
    M, d, I = 256, 512, 1024
    g = torch.Generator(device=dev).manual_seed(5)
    def codes(r, c):
        # finite E4M3 codes of magnitude <= 1 (exponent field <= 7), random signs
        v = torch.randint(0, 0x39, (r, c), device=dev, generator=g, dtype=torch.int32)
        s = torch.randint(0, 2, (r, c), device=dev, generator=g, dtype=torch.int32) << 7
        return (v | s).to(torch.uint8).view(torch.float8_e4m3fn)
    x = torch.randn((M, d), device=dev, generator=g).to(torch.bfloat16)
    wg, wu, wd = codes(I, d), codes(I, d), codes(d, I)
    sc = lambda v: torch.tensor([v], dtype=torch.float32, device=dev)
    s_in, s_wg, s_wu, s_down, s_wd = sc(0.02), sc(0.003), sc(0.0035), sc(0.004), sc(0.0025)
    lib = fw.load()
    y = torch.empty((M, d), dtype=torch.bfloat16, device=dev)
    # the first library call of this process
    rc = lib.gated_mlp_static_fp8_noalloc(
        x.data_ptr(), M, d, I, s_in.data_ptr(), wg.data_ptr(), s_wg.data_ptr(), wu.data_ptr(),
        s_wu.data_ptr(), s_down.data_ptr(), wd.data_ptr(), s_wd.data_ptr(), y.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert rc == fw.OK, fw.STATUS.get(rc)
    ref = fw.gated_mlp_static_fp8(x, s_in, wg, s_wg, wu, s_wu, s_down, wd, s_wd)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    assert y.float().abs().sum().item() > 0
    print("fresh-process first call ok")
""")


def test_first_call_in_a_fresh_process():
    """The entry point as the first library call of a process: its set-up
    (the scratch area's address, which under lazy module loading also loads
    the library's module onto the GPU) happens inside that call."""
    out = subprocess.run([sys.executable, "-c", _FRESH.format(root=ROOT)], capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "fresh-process first call ok" in out.stdout
