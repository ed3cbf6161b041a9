"""The C ABI without a GPU: the library builds and loads, exports every
symbol the header declares, and rejects bad arguments before it touches CUDA.
Also checks that the product path never reaches the oracle."""

import ast
import ctypes
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
    # Xq, then the split-K scratch of the grouped projection GEMMs
    assert lib.qkv_shared_quant_workspace(2048, 3072) == 2048 * 3072 + lib.fp8_linear_static_ws_bytes()
    assert lib.gated_mlp_static_fp8_workspace(-1, 1, 1) == 0


def test_workspace_sizes_saturate(lib):
    """Byte counts that do not fit in 64 bits give SIZE_MAX, never a wrapped
    small number: M = 2147391056, d = 2147483616, I = 1288564272 (each below
    2^31) would sum to 2^64 + 65,143,040 bytes for the gated MLP."""
    size_max = 2 ** 64 - 1
    M, d, I = 2147391056, 2147483616, 1288564272
    assert lib.gated_mlp_static_fp8_workspace(M, d, I) == size_max
    big = 2 ** 62
    assert lib.gated_mlp_static_fp8_fused_workspace(big, big, big) == size_max
    assert lib.gated_mlp_per_token_fp8_workspace(big, big, big) == size_max
    assert lib.fp8_shared_quant_linears_workspace(big, big) == size_max
    assert lib.cross_attention_qkv_static_fp8_workspace(big, big, big) == size_max
    rows = (ctypes.c_int64 * 2)(big, big)
    assert lib.gated_mlp_static_fp8_group_workspace(rows, 2, big, big) == size_max
    # ordinary sizes are unchanged
    assert lib.gated_mlp_static_fp8_workspace(1040, 3072, 12288) == 1040 * 64512


@pytest.mark.parametrize("M,d,I", [
    (2147391056, 2147483616, 1288564272),  # wrapped to 65 MB under a 64-bit sum
    (1041, 3072, 12288),                    # the first M past the 64 MiB area
    (1, 100, 704),                          # d not a multiple of 16
    (1, 256, 8),                            # I below 16
    (2 ** 31, 256, 704),                    # M of 2^31
    (-1, 256, 704),
])
def test_noalloc_refuses_before_cuda(lib, M, d, I):
    """The no-alloc gated MLP validates the shape and the scratch size before
    any CUDA call (here, with no GPU, any CUDA call would fail differently)."""
    n0 = lib.fp8ws_launch_count()
    a = 1 << 20  # never dereferenced
    assert lib.gated_mlp_static_fp8_noalloc(a, M, d, I, a, a, a, a, a, a, a, a, a, None) == \
        fw.ERR_SHAPE
    assert lib.fp8ws_launch_count() == n0


def test_linears_static_argument_checks(lib):
    """fp8_linears_static refuses bad arguments before any CUDA call."""
    import ctypes as C
    a = 1 << 20
    W = (C.c_void_p * 2)(a, a)
    N = (C.c_int64 * 2)(256, 256)
    S = (C.c_void_p * 2)(a, a)
    Y = (C.c_void_p * 2)(a, a)
    assert lib.fp8_linears_static(a, 64, 256, a, 0, W, N, S, Y, None, 0, None) == fw.ERR_SHAPE
    assert lib.fp8_linears_static(a, 64, 256, a, 17, W, N, S, Y, None, 0, None) == fw.ERR_SHAPE
    assert lib.fp8_linears_static(a, 64, 256, a, 2, None, N, S, Y, None, 0, None) == fw.ERR_NULL
    bad_n = (C.c_int64 * 2)(256, 100)  # N % 8 != 0
    assert lib.fp8_linears_static(a, 64, 256, a, 2, W, bad_n, S, Y, None, 0, None) == fw.ERR_SHAPE
    assert lib.fp8_linears_static(a + 8, 64, 256, a, 2, W, N, S, Y, None, 0, None) == fw.ERR_ALIGN
    assert lib.fp8_linears_static(a, 64, 256, a, 2, W, N, S, Y, a + 16, 1 << 30, None) == \
        fw.ERR_WORKSPACE


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


def _header_struct_fields(name):
    """Field names of `typedef struct { ... } name;` in the header, in order."""
    text = open(HEADER).read()
    body = re.search(r"typedef struct \{([^{}]*)\}\s*" + name + r"\s*;", text).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = []
    for decl in body.split(";"):
        decl = decl.strip()
        if decl:
            fields += [part.strip().lstrip("*").split()[-1].lstrip("*")
                       for part in decl.split(",")]
    return fields


@pytest.mark.parametrize("cname,pyname", [
    ("fp8ws_quant_problem", "QuantProblem"), ("fp8ws_linear_problem", "LinearProblem"),
    ("fp8ws_gate_up_problem", "GateUpProblem"), ("fp8ws_mlp_tower", "MlpTower"),
    ("fp8ws_swiglu", "Swiglu"), ("fp8ws_launch_record", "LaunchRecord")])
def test_group_structs_match_header(cname, pyname):
    """The ctypes layouts follow the header's fields in order.  The group
    structs hold only pointers and 64-bit integers, and the SwiGLU descriptor
    only 4-byte fields, so matching names in order fixes the layout."""
    cls = getattr(fw, pyname)
    assert [f for f, _ in cls._fields_] == _header_struct_fields(cname)


def test_group_argument_checks_before_cuda(lib):
    import ctypes
    a = 1 << 20
    n0 = fw.launch_count()
    q = (fw.QuantProblem * 2)(fw.QuantProblem(a, 64, a, a), fw.QuantProblem(a + 2, 64, a, a))
    assert lib.fp8_quant_static_group(ctypes.byref(q), 2, None) == fw.ERR_ALIGN
    assert lib.fp8_quant_static_group(ctypes.byref(q), 3, None) == fw.ERR_SHAPE
    assert lib.fp8_quant_static_group(ctypes.byref(q), 0, None) == fw.ERR_SHAPE
    assert lib.fp8_quant_static_group(None, 1, None) == fw.ERR_NULL
    lp = (fw.LinearProblem * 2)(fw.LinearProblem(a, a, 64, a, a, a),
                                fw.LinearProblem(a, a, 64, None, a, a))
    assert lib.fp8_linear_static_group(ctypes.byref(lp), 2, 256, 512, None, 0, None) == fw.ERR_NULL
    assert lib.fp8_linear_static_group(ctypes.byref(lp), 1, 260, 512, None, 0, None) == fw.ERR_SHAPE
    assert lib.fp8_linear_static_group(ctypes.byref(lp), 1, 256, 512, a + 16, 1 << 30,
                                       None) == fw.ERR_WORKSPACE
    assert lib.fp8_linear_static_group(ctypes.byref(lp), 1, 256, 512, a, 1024,
                                       None) == fw.ERR_WORKSPACE
    gp = (fw.GateUpProblem * 1)(fw.GateUpProblem(a, a, a, 64, a, a, a, a, a))
    assert lib.fp8_gate_up_swiglu_static_group(ctypes.byref(gp), 1, 264, 512, None,
                                               None) == fw.ERR_SHAPE   # I % 16
    bad = fw.swiglu(1.0, 0.0, -1.0)
    assert lib.fp8_gate_up_swiglu_static_group(ctypes.byref(gp), 1, 256, 512, ctypes.byref(bad),
                                               None) == fw.ERR_BAD_SCALE
    t = fw.MlpTower(a, 64, a, a, a, a, a, a, a, a, a)
    tw = (fw.MlpTower * 2)(t, t)
    rows = (ctypes.c_int64 * 2)(64, 64)
    need = lib.gated_mlp_static_fp8_group_workspace(ctypes.byref(rows), 2, 256, 704)
    assert need == 2 * lib.gated_mlp_static_fp8_fused_workspace(64, 256, 704) + \
        lib.fp8_linear_static_ws_bytes()
    assert lib.gated_mlp_static_fp8_group(ctypes.byref(tw), 2, 256, 704, None, a, need - 256,
                                          None) == fw.ERR_WORKSPACE
    assert lib.gated_mlp_static_fp8_group(ctypes.byref(tw), 2, 256, 700, None, a, 1 << 40,
                                          None) == fw.ERR_SHAPE
    assert lib.gated_mlp_static_fp8_group_workspace(None, 2, 256, 704) == 0
    # towers with no rows: nothing to do, nothing launched
    e = fw.MlpTower(None, 0, a, a, a, a, a, a, a, a, None)
    te = (fw.MlpTower * 2)(e, e)
    assert lib.gated_mlp_static_fp8_group(ctypes.byref(te), 2, 256, 704, None, a, 1 << 30,
                                          None) == fw.OK
    assert fw.launch_count() == n0
    eq = (fw.QuantProblem * 2)(fw.QuantProblem(None, 0, None, None),
                               fw.QuantProblem(None, 0, None, None))
    assert lib.fp8_quant_static_group(ctypes.byref(eq), 2, None) == fw.OK
    el = (fw.LinearProblem * 1)(fw.LinearProblem(None, a, 0, a, a, None))
    assert lib.fp8_linear_static_group(ctypes.byref(el), 1, 256, 512, None, 0, None) == fw.OK
    eg = (fw.GateUpProblem * 1)(fw.GateUpProblem(None, a, a, 0, a, a, a, a, None))
    assert lib.fp8_gate_up_swiglu_static_group(ctypes.byref(eg), 1, 256, 512, None,
                                               None) == fw.OK
    assert fw.launch_count() == n0


def test_selftest_argument_checks(lib):
    import ctypes
    out = ctypes.c_int64(0)
    assert lib.fp8ws_selftest_bounded_wait(1000, 0, None, None) == fw.ERR_NULL
    assert lib.fp8ws_selftest_bounded_wait(0, 0, ctypes.byref(out), None) == fw.ERR_SHAPE
    assert lib.fp8ws_selftest_bounded_wait(5_000_000_000, 0, ctypes.byref(out), None) == fw.ERR_SHAPE
    assert lib.fp8ws_selftest_bounded_wait(1000, 2, ctypes.byref(out), None) == fw.ERR_SHAPE


def test_quant_form_switch(lib):
    """fp8ws_set_quant_form takes 0 (by size), 1 (staged) or 2 (streaming),
    nothing else; host only."""
    for bad in (-1, 3, 7):
        assert lib.fp8ws_set_quant_form(bad) == fw.ERR_SHAPE
    for good in (2, 1, 0):
        assert lib.fp8ws_set_quant_form(good) == fw.OK
