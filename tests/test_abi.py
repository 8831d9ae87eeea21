"""The C ABI library loads and exports every symbol include/moemx.h declares (CPU only: no
compute calls), and its host-side size queries and argument checks behave as documented."""
import ctypes
import os
import re

import pytest

import mxfp8_quantize_b200 as moe
from mxfp8_quantize_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moe.load_library()


def test_header_declarations_are_exported(lib):
    header = open(os.path.join(ROOT, "include", "moemx.h")).read()
    names = set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(\w+)\s*\(", header, flags=re.M))
    names = {n for n in names if n.startswith(("moe_", "mxfp8_", "fp8_"))}
    assert names == set(moe.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_capacity_and_sizes(lib):
    assert moe.capacity_rows(8192, 2, 8) == 16384 + 1024
    assert moe.capacity_rows(1, 1, 1) == 128
    s = moe.sizes(8192, 4096, 14336, 8, 2, "mxfp8", True)
    cap = 17408
    # saved holds at least the bf16 h and the transposed MXFP8 weights
    assert s["saved"] >= cap * 2 * 14336 * 2 + 8 * 3 * 4096 * 14336
    assert s["fwd_ws"] >= 8 * 3 * 4096 * 14336
    # unsupported shapes give 0
    assert lib.moe_saved_size(8192, 2, 8, 4000, 14336, 1) == 0
    assert lib.moe_fwd_workspace_size(8192, 2, 300, 4096, 14336, 1, 1) == 0


def test_null_context_is_rejected(lib):
    assert lib.mxfp8_quantize(None, None, 1, 32, 32, 1, None, None, None, None, None) == 1
    assert lib.moe_get_status(None, None) == 1
    assert lib.moe_ctx_destroy(None) == 1
    assert lib.moe_status_string(6) == b"bounded in-kernel wait expired"


def test_buffer_address_is_consistent(lib):
    base = 1 << 40
    p1 = lib.moe_buffer_address(4096, 2, 8, 1024, 2048, 1, 1, 0, base, b"h")
    p2 = lib.moe_buffer_address(4096, 2, 8, 1024, 2048, 1, 1, 0, base, b"aT_q")
    assert p1 and p2 and p1 > p2 and (p1 - base) % 1024 == 0
    assert lib.moe_buffer_address(4096, 2, 8, 1024, 2048, 1, 1, 0, base, b"nope") is None
    assert p1 - base + 4096 * 2 * 0 < lib.moe_saved_size(4096, 2, 8, 1024, 2048, 1)


def test_product_path_has_no_cpu_fallback():
    """The binding never imports the oracle and refuses to run without the library."""
    src = open(os.path.join(ROOT, "mxfp8_quantize_b200", "__init__.py")).read()
    assert "oracle" not in src.replace("oracle_", "")
    for f in os.listdir(os.path.join(ROOT, "mxfp8_quantize_b200", "csrc")):
        assert "oracle" not in open(os.path.join(ROOT, "mxfp8_quantize_b200", "csrc", f)).read()
