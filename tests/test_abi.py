"""The C-ABI library: it loads, exports every symbol the headers under include/ declare,
and rejects bad arguments on the host before touching a device.  No compute
calls here (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import weight_only_int4_linear_b200 as w4
from weight_only_int4_linear_b200 import build as w4build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a16.h")


@pytest.fixture(scope="module")
def lib():
    w4build.build()
    return w4.load()


HEADERS = [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include")))
           if h.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        names |= set(re.findall(r"W4A16_API\s+[\w\s\*]+?\b(w[48]a16_\w+)\s*\(", open(h).read()))
    return sorted(names)


def test_header_declares_entry_points():
    names = declared_functions()
    for required in ["w4a16_linear", "w4a16_quantize_pack", "w4a16_workspace_bytes", "w4a16_unpack",
                     "w4a16_dequant", "w4a16_status_string"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", w4.LIB_PATH]).decode()
    exported = set(re.findall(r"\bT (w[48]a16_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for n in declared_functions():
        assert hasattr(lib, n)
    # binding signatures cover exactly the declared entry points
    assert sorted(w4.SIGNATURES) == declared_functions()


def test_header_compiles_as_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "w4a16.h"\n#include "w8a16.h"\nint main(void){return W4A16_OK + W4A16_PATH_AUTO;}\n')
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-c",
                           str(src), "-o", str(tmp_path / "t.o")])


def test_status_strings(lib):
    assert w4.version() >= 100
    for s in range(0, 9):
        assert len(w4.status_string(s)) > 0
    assert w4.status_string(0) == "ok"
    assert w4.status_string(999) == "unknown status"


def test_host_validation_without_device(lib):
    """Bad arguments are rejected before any CUDA call (fake, never-dereferenced pointers)."""
    P = ctypes.c_void_p(0x10000)        # aligned fake device pointer
    U = ctypes.c_void_p(0x10008)        # misaligned
    lin = lib.w4a16_linear_path
    assert lin(None, 1, 128, P, P, P, 16, P, None, 0, 0, None) == w4.ERR_ARG
    assert lin(P, 0, 128, P, P, P, 16, P, None, 0, 0, None) == w4.ERR_ARG
    assert lin(P, 1, 100, P, P, P, 16, P, None, 0, 0, None) == w4.ERR_SHAPE
    assert lin(P, 1, 128, P, P, P, -1, P, None, 0, 0, None) == w4.ERR_ARG
    assert lin(P, 1, 128, P, P, P, 16, P, None, 0, 7, None) == w4.ERR_ARG
    assert lin(P, 1, 128, U, P, P, 16, P, None, 0, 0, None) == w4.ERR_ALIGN
    assert lin(P, 1, 1 << 31, P, P, P, 16, P, None, 0, 0, None) == w4.ERR_SHAPE
    assert lib.w4a16_quantize_pack(P, 4, 96, P, P, P, P, None) == w4.ERR_SHAPE
    assert lib.w4a16_quantize_pack(P, 4, 128, P, P, P, None, None) == w4.ERR_ARG
    assert lib.w4a16_unpack(P, 4, 128, U, None) == w4.ERR_ALIGN
    assert lib.w4a16_dequant(P, P, None, 4, 128, P, None) == w4.ERR_ARG
    assert lib.w4a16_renorm_rows(P, 0, 8, P, None) == w4.ERR_ARG
    assert lib.w8a16_linear(None, 1, 128, P, P, 16, P, P, 1 << 20, None) == w4.ERR_ARG
    assert lib.w8a16_linear(P, 1, 100, P, P, 16, P, P, 1 << 20, None) == w4.ERR_SHAPE
    assert lib.w8a16_linear(P, 1, 128, U, P, 16, P, P, 1 << 20, None) == w4.ERR_ALIGN
    assert lib.w8a16_quantize(P, 0, 128, P, P, P, None) == w4.ERR_ARG
    assert lib.w8a16_quantize(P, 4, 128, P, P, None, None) == w4.ERR_ARG
    assert lib.w8a16_dequant(P, U, 4, 128, P, None) == w4.ERR_ALIGN
    assert lib.w8a16_workspace_bytes(1, 16, 100) == 0
    # symmetric packing, the AWQ entries and the group-size entries validate the same way
    assert lib.w4a16_quantize_pack_sym(P, 4, 96, P, P, P, P, None) == w4.ERR_SHAPE
    assert lib.w4a16_quantize_pack_awq(P, None, 4, 128, P, P, P, P, None) == w4.ERR_ARG
    assert lib.w4a16_quantize_pack_awq(P, U, 4, 128, P, P, P, P, None) == w4.ERR_ALIGN
    assert lib.w4a16_linear_awq(P, None, 1, 128, P, P, P, 16, P, None, 0, 0, None) == w4.ERR_ARG
    assert lib.w4a16_linear_awq(P, U, 1, 128, P, P, P, 16, P, None, 0, 0, None) == w4.ERR_ALIGN
    assert lib.w4a16_quantize_pack_g(P, 4, 128, 48, 0, P, P, P, P, None) == w4.ERR_ARG
    assert lib.w4a16_quantize_pack_g(P, 4, 96, 64, 0, P, P, P, P, None) == w4.ERR_SHAPE
    assert lib.w4a16_linear_g(P, 1, 512, 48, P, P, P, 16, P, P, 1 << 20, None) == w4.ERR_ARG
    assert lib.w4a16_linear_g(P, 1, 384, 64, P, P, P, 16, P, P, 1 << 20, None) == w4.ERR_SHAPE
    assert lib.w4a16_linear_g(P, 1, 512, 32, U, P, P, 16, P, P, 1 << 20, None) == w4.ERR_ALIGN
    assert lib.w4a16_workspace_bytes_g(1, 16, 384, 64) == 0
    assert lib.w4a16_workspace_bytes_g(1, 16, 512, 48) == 0
    # the failure-path self-test checks its limit before touching a device
    assert lib.w4a16_selftest_wait(0, None) == w4.ERR_ARG
    assert lib.w4a16_selftest_wait(2_000_000_001, None) == w4.ERR_ARG
    if not torch.cuda.is_available():
        assert lib.w4a16_selftest_wait(1000, None) == w4.ERR_DEVICE
        # well-formed arguments reach the device check, which fails without a GPU
        assert lin(P, 1, 128, P, P, P, 16, P, None, 0, 0, None) == w4.ERR_DEVICE
        assert lib.w4a16_workspace_init(P, 64, None) == w4.ERR_DEVICE


def test_selftest_constants_match_the_header():
    text = open(HEADER).read()
    assert re.search(r"#define W4A16_SELFTEST_SITE (\d+)", text).group(1) == str(w4.SELFTEST_SITE)
    assert int(re.search(r"#define W4A16_SELFTEST_MAX_CYCLES (\d+)LL", text).group(1)) == 2_000_000_000


def test_workspace_bytes(lib):
    assert lib.w4a16_workspace_bytes(1, 16, 100) == 0           # invalid shape -> 0
    for (M, N, K) in [(1, 4096, 4096), (1, 5120, 25600), (32, 8192, 28672), (4096, 8192, 8192)]:
        b = w4.workspace_bytes(M, N, K)
        assert b % 256 == 0


def test_binding_refuses_host_tensors(lib):
    X = torch.zeros((1, 128), dtype=torch.bfloat16)
    qw = torch.zeros((16, 16), dtype=torch.int32)
    sc = torch.zeros((16, 1), dtype=torch.bfloat16)
    z = torch.zeros((16, 1), dtype=torch.int32)
    Y = torch.zeros((1, 16), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        w4.linear(X, qw, sc, z, Y)


def test_product_does_not_reference_oracle():
    """The product package never imports or links the oracle."""
    pkg = os.path.join(ROOT, "weight_only_int4_linear_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "liboracle" not in text and "orc_" not in text, f
