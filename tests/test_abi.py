"""The C-ABI library loads and exports every entry point include/w4a16.h declares.

No GPU is needed: only symbol lookup and argument checks that fail before
any CUDA call are exercised here.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(w4\w*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("w4_quantize_pack", "w4a16_gemm", "w4a16_gemv", "w4_workspace_bytes",
                     "w4_quantize_workspace_bytes", "w4_status_string", "w4_device_error"):
        assert required in names


def test_library_exports_every_declared_symbol():
    import gemv_w4a16_groupwise_b200 as w4
    lib = ctypes.CDLL(w4._build.build())
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_host_validation():
    import gemv_w4a16_groupwise_b200 as w4
    lib = w4.library()
    for code in range(7):
        assert lib.w4_status_string(code)
    assert b"unknown" in lib.w4_status_string(99)
    fake = 1 << 20   # never dereferenced: validation fails before any CUDA call
    args = lambda M, N, K, mode, g: (fake, M, N, K, fake, fake, fake, mode, g, None, 0, fake, None, 0,
                                     None)
    assert lib.w4a16_gemm(*args(0, 64, 256, 2, 64)) == 1
    assert lib.w4a16_gemm(*args(4, 64, 252, 2, 64)) == 1
    assert lib.w4a16_gemm(*args(4, 64, 256, 2, 48)) == 1
    assert lib.w4a16_gemm(*args(4, 64, 256, 9, 64)) == 1
    assert lib.w4a16_gemm(*args(4, 64, 256, 2 | 0x40, 64)) == 1      # unknown format flag
    assert lib.w4_gather_columns(fake, 0, 8, fake, 8, fake, None) == 1
    assert lib.w4_scatter_columns(fake, 4, 8, None, 8, fake, None) == 1
    assert lib.w4a16_gemv(*args(4, 64, 256, 2, 64)[:0] + (None, 4, 64, 256, fake, fake, fake, 2, 64,
                                                           None, 0, fake, None, 0, None)) == 1
    assert lib.w4_quantize_pack(fake, 64, 250, 1, 0, fake, fake, fake, None, 0, None) == 1
    assert lib.w4_quantize_workspace_bytes(64, 256, 0) > 0
    assert lib.w4_quantize_workspace_bytes(64, 256, 2) == 0


def test_product_path_has_no_oracle_dependency():
    """The library package must not import, link or execute the oracle."""
    pkg = os.path.join(ROOT, "gemv_w4a16_groupwise_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "liboracle" not in text and "w4a16_oracle" not in text, fn
