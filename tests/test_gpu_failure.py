"""Failure detection on the GPU without a GPU fault: the bounded wait that
every GEMM kernel uses runs out on a barrier nothing arrives at, the kernel
records where and returns, the host reads the status, and the context stays
usable.  The abort path (another role gave up) ends a wait early."""

import numpy as np
import pytest
import torch

import fp8_w8a8_static_b200 as fw
import oracle
from _util import GEMM_REL_FRO, bits, from_codes, rel_fro, scalar

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_is_reported():
    fw.device_status()  # start from a clear status word
    limit = 2_000_000  # 2 ms
    elapsed = fw.selftest_bounded_wait(limit, mode=0)
    assert limit <= elapsed < 1_000_000_000
    assert fw.device_status() == (fw.ERR_DEVICE_TIMEOUT, fw.SITE_SELFTEST)
    assert fw.device_status() == (fw.OK, 0)  # reading clears it


def test_abort_flag_ends_the_wait_early():
    fw.device_status()
    limit = 400_000_000  # the other warp raises the flag after 100 ms
    elapsed = fw.selftest_bounded_wait(limit, mode=1)
    assert 100_000_000 <= elapsed < 300_000_000
    assert fw.device_status() == (fw.OK, 0)  # an aborted wait records nothing


def test_context_usable_after_a_timeout():
    fw.selftest_bounded_wait(1_000_000, mode=0)
    assert fw.device_status()[0] == fw.ERR_DEVICE_TIMEOUT
    rng = np.random.default_rng(0)
    v = rng.standard_normal((256, 512)).astype(np.float32) / 8
    b = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    xq = oracle.quantize(b, 1.0 / 64)
    wq = oracle.quantize(b[:264], 1.0 / 64)
    y = fw.fp8_linear_static(from_codes(xq, "cuda"), from_codes(wq, "cuda"), scalar(0.5, "cuda"),
                             scalar(0.25, "cuda"))
    assert rel_fro(bits(y), oracle.linear(xq, wq, 0.5, 0.25)) <= GEMM_REL_FRO
    assert fw.device_status() == (fw.OK, 0)
