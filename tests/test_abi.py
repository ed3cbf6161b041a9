"""The C ABI without a GPU: the library builds and loads, exports every
symbol the header declares, and rejects bad arguments before it touches CUDA.
Also checks that the product path never reaches the oracle."""

import ast
import os
import re

import pytest

import fp8_w8a8_static_b200 as fw
from fp8_w8a8_static_b200 import build as fw_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8ws.h")


@pytest.fixture(scope="module")
def lib():
    fw_build.build()
    return fw.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^FP8WS_API\s+[\w\s\*]*?\b(\w+)\s*\(", text, re.M)))


def test_header_declares_the_path():
    names = declared_symbols()
    for want in ("fp8_quant_static", "fp8_linear_static", "silu_mul_2in_fp8",
                 "gated_mlp_static_fp8", "qkv_shared_quant", "fp8_check_shared_input_scale"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(declared_symbols()) == set(fw.EXPORTED_SYMBOLS)


def test_no_internal_symbols_leak(lib):
    out = os.popen(f"nm -D --defined-only {fw.library_path()}").read()
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert exported == set(declared_symbols())


def test_status_strings(lib):
    for code in range(10):
        assert lib.fp8ws_status_string(code).decode() == fw.STATUS[code]


def test_workspace_sizes(lib):
    def r256(v):
        return (v + 255) // 256 * 256
    assert lib.gated_mlp_static_fp8_workspace(64, 256, 704) == r256(64 * 256) + 2 * r256(64 * 704 * 2) + r256(64 * 704)
    assert lib.qkv_shared_quant_workspace(2048, 3072) == 2048 * 3072
    assert lib.gated_mlp_static_fp8_workspace(-1, 1, 1) == 0


def test_argument_checks_before_cuda(lib):
    """Null pointers, bad sizes and misaligned pointers are refused before any
    CUDA call, so these run without a GPU."""
    a = 1 << 20  # a 16-byte aligned fake address, never dereferenced
    n0 = fw.launch_count()
    assert lib.fp8_quant_static(None, 8, a, a, None) == fw.ERR_NULL
    assert lib.fp8_quant_static(a, -1, a, a, None) == fw.ERR_SHAPE
    assert lib.fp8_quant_static(a + 2, 8, a, a, None) == fw.ERR_ALIGN
    assert lib.silu_mul_2in_fp8(a, None, 8, a, a, None) == fw.ERR_NULL
    assert lib.silu_mul_2in_fp8(a, a, 8, a, a + 8, None) == fw.ERR_ALIGN
    assert lib.fp8_linear_static(a, a, 4, 12, 32, a, a, a, None) == fw.ERR_SHAPE   # N % 8
    assert lib.fp8_linear_static(a, a, 4, 16, 40, a, a, a, None) == fw.ERR_SHAPE   # K % 16
    assert lib.fp8_linear_static(a, a, -1, 16, 32, a, a, a, None) == fw.ERR_SHAPE
    assert lib.fp8_linear_static(a, a, 4, 16, 32, None, a, a, None) == fw.ERR_NULL
    assert lib.fp8_linear_static(a + 16, a + 4, 4, 16, 32, a, a, a, None) == fw.ERR_ALIGN
    args = [a, 64, 256, 704, a, a, a, a, a, a, a, a]
    assert lib.gated_mlp_static_fp8(*args, None, a, None) == fw.ERR_WORKSPACE
    assert lib.gated_mlp_static_fp8(*args, a + 16, a, None) == fw.ERR_WORKSPACE
    assert lib.gated_mlp_static_fp8(a, 64, 256, 700, *[a] * 8, a, a, None) == fw.ERR_SHAPE
    assert lib.qkv_shared_quant(a, 8, 3072, a, a, 12, a, a, 1024, a, a, 1024, a, a, a, a, a,
                                None) == fw.ERR_SHAPE
    assert lib.fp8_observer_scale(a, 0, 0.01, a, None) == fw.ERR_SHAPE
    assert lib.fp8_rtn_quantize_weight(a, 0, a, a, None) == fw.ERR_SHAPE
    assert lib.fp8_check_shared_input_scale(None, 2, None) == fw.ERR_NULL
    # empty tensors carry NULL data pointers: nothing to do, nothing launched
    assert lib.fp8_quant_static(None, 0, None, None, None) == fw.OK
    assert lib.silu_mul_2in_fp8(None, None, 0, None, None, None) == fw.OK
    assert fw.launch_count() == n0


def test_product_never_imports_the_oracle():
    """The package and the benchmark's GPU legs do not import oracle/."""
    pkg = os.path.join(ROOT, "fp8_w8a8_static_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py"):
                tree = ast.parse(open(os.path.join(dirpath, f)).read())
                for node in ast.walk(tree):
                    if isinstance(node, ast.Import):
                        assert all(not a.name.startswith("oracle") for a in node.names), f
                    if isinstance(node, ast.ImportFrom):
                        assert not (node.module or "").startswith("oracle"), f
    for dirpath, _, files in os.walk(os.path.join(pkg, "csrc")):
        for f in files:
            assert "oracle" not in open(os.path.join(dirpath, f)).read().lower(), f


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(fw, "_lib", None)
    monkeypatch.setattr(fw, "_LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="missing"):
        fw.load()
