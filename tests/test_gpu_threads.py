"""Concurrent first use from several host threads: in a fresh process, four
threads make their first library calls at the same time, each on its own
stream with its own workspace (the per-device set-up runs once, under a lock),
and every result equals the one a single thread computes afterwards."""

import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = textwrap.dedent("""
    import sys, threading
    sys.path.insert(0, ROOT)
    import torch
    import fp8_w8a8_static_b200 as fw
    import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    d, I = 256, 704

    def tower(M, seed):
        x = synth.activation_with_outliers(M, d, 9, seed, 0, dev)
        t = dict(x=x, s_in=torch.tensor([0.02], device=dev), s_down=torch.tensor([0.004], device=dev))
        for name, shape, k in (("wg", (I, d), 1), ("wu", (I, d), 2), ("wd", (d, I), 3)):
            w = synth.normal(shape, 0.02, seed * 7 + k, dev)
            amax = w.abs().max().float().reshape(1)
            s = amax / 448
            t[name] = (w.float() / s).to(fw.FP8)
            t["s_" + name] = s
        return t

    jobs = [[tower(64 + 32 * j, 10 * j + 1), tower(48, 10 * j + 2)] for j in range(4)]
    torch.cuda.synchronize()
    out = [None] * 4
    errors = []
    start = threading.Barrier(4)

    def work(j):
        try:
            s = torch.cuda.Stream(dev)
            with torch.cuda.stream(s):
                start.wait()
                ys = fw.gated_mlp_static_fp8_group(jobs[j], stream=s)
                t = jobs[j][0]
                lin = fw.fp8_linear_static(fw.fp8_quant_static(t["x"], t["s_in"], stream=s),
                                           t["wg"], t["s_in"], t["s_wg"], stream=s)
            s.synchronize()
            out[j] = [y.clone() for y in ys] + [lin.clone()]
        except Exception as e:  # reported below
            errors.append(repr(e))

    threads = [threading.Thread(target=work, args=(j,)) for j in range(4)]
    for th in threads:
        th.start()
    for th in threads:
        th.join(timeout=120)
    assert not errors, errors
    assert all(not th.is_alive() for th in threads)
    for j in range(4):
        ys = fw.gated_mlp_static_fp8_group(jobs[j])
        t = jobs[j][0]
        lin = fw.fp8_linear_static(fw.fp8_quant_static(t["x"], t["s_in"]), t["wg"], t["s_in"],
                                   t["s_wg"])
        for a, b in zip(out[j], list(ys) + [lin]):
            assert torch.equal(a, b)
    assert fw.device_status() == (fw.OK, 0)
    print("threads ok")
""")


def test_concurrent_first_use_from_threads():
    code = "ROOT = %r\n" % ROOT + SCRIPT
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "threads ok" in r.stdout
