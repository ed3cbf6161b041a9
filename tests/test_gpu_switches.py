"""The library's timing switches (environment variables read once per
process) select other launch shapes, pipelines or kernel forms for
measurements; none may change a result.  The same seeded calls run in child
processes under several settings and must write the same bytes as under the
defaults: the grouped two-tower gated MLP (pair quantizer, grouped dual
gate/up + SwiGLU-quant kernel, grouped down GEMM split over K), a Linear
whose ragged last wave runs as halves, a Linear split over K, and a large
flat quantization."""

import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_CHILD = textwrap.dedent("""
    import hashlib, sys
    import torch
    sys.path.insert(0, {root!r})
    sys.path.insert(0, {tests!r})
    import fp8_w8a8_static_b200 as fw
    import synth
    from _util import scalar
    dev = "cuda"

    def digest(t):
        return hashlib.sha256(t.contiguous().cpu().view(torch.uint8).numpy().tobytes()).hexdigest()[:20]

    out = []
    # both towers through the grouped calls; the down GEMM's 12 tiles (K = 8192,
    # 64 K steps) for 74 pairs are split over K
    d, I = 1024, 8192
    towers = []
    for k, M in enumerate((512, 256)):
        wg = fw.fp8_rtn_quantize_weight(synth.normal((I, d), 0.02, 60 + k, dev))
        wu = fw.fp8_rtn_quantize_weight(synth.normal((I, d), 0.02, 70 + k, dev))
        wd = fw.fp8_rtn_quantize_weight(synth.normal((d, I), 0.02, 80 + k, dev))
        towers.append(dict(x=synth.activation_with_outliers(M, d, 4, 50 + k, 0, dev),
                           s_in=scalar(0.03, dev), wg=wg[0], s_wg=wg[1], wu=wu[0], s_wu=wu[1],
                           s_down=scalar(0.002, dev), wd=wd[0], s_wd=wd[1]))
    out += [digest(y) for y in fw.gated_mlp_static_fp8_group(towers)]
    # a Linear whose ragged last wave runs as halves, and one split over K
    for M, N, K, ws in ((300, 520, 1040, False), (300, 520, 8208, True), (2048, 3072, 3072, False)):
        x = synth.activation_with_outliers(M, K, 4, M + K, 0, dev)
        s_in = scalar(0.031, dev)
        xq = fw.fp8_quant_static(x, s_in)
        wq, s_w = fw.fp8_rtn_quantize_weight(synth.normal((N, K), 0.02, N + K, dev))
        y = fw.fp8_linear_static_ws(xq, wq, s_in, s_w) if ws else fw.fp8_linear_static(xq, wq, s_in, s_w)
        out += [digest(xq), digest(y)]
    # a flat quantization of 12288 x 8192 values (past 1.5 x L2)
    x = synth.activation_with_outliers(12288, 8192, 4, 7, 0, dev)
    out.append(digest(fw.fp8_quant_static(x, scalar(0.0389, dev))))
    torch.cuda.synchronize()
    assert fw.device_status()[0] == fw.OK
    print(" ".join(out))
""")

_KEYS = ("FP8WS_PDL", "FP8WS_EPILOGUE", "FP8WS_PAIR_STAGES", "FP8WS_TAIL_HALVES",
         "FP8WS_L2_HINTS", "FP8WS_PREFETCH", "FP8WS_LATE_TRIGGER", "FP8WS_QUANT")


def _run(settings):
    env = {k: v for k, v in os.environ.items() if k not in _KEYS}
    env.update(settings)
    code = _CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600,
                       env=env)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    return r.stdout.split()


def test_timing_switches_change_no_result():
    base = _run({})
    assert len(base) == 9
    for settings in (
            # every switch that turns an optimisation off, at once
            {"FP8WS_PDL": "0", "FP8WS_TAIL_HALVES": "0", "FP8WS_L2_HINTS": "0",
             "FP8WS_PREFETCH": "0", "FP8WS_LATE_TRIGGER": "0", "FP8WS_QUANT": "staged"},
            # register-store epilogues (seven stages), the streaming quantizer everywhere
            {"FP8WS_EPILOGUE": "direct", "FP8WS_QUANT": "stream"},
            # the five-stage pair GEMM
            {"FP8WS_PAIR_STAGES": "5"}):
        assert _run(settings) == base, settings
