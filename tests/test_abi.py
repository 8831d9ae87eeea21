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


def test_fp8_sizes_and_layout(lib):
    """Per-tensor FP8 (precision 2): codes without scale bytes, so its buffers are smaller than
    MXFP8's; it saves h in bf16 only; the maxima have names in the saved buffer, the inference
    workspace and the backward workspace, and every named part lies inside its buffer."""
    T, d, f, E, k = 4096, 1024, 2048, 8, 2
    mx, f8 = moe.sizes(T, d, f, E, k, "mxfp8", True), moe.sizes(T, d, f, E, k, "fp8", True)
    assert 0 < f8["saved"] < mx["saved"]
    assert f8["fwd_ws"] > 0 and f8["bwd_ws"] > 0
    assert moe.sizes(T, d, f, E, k, "fp8", True, "mxfp8")["saved"] == 0
    assert moe.sizes(T, d, f, E, k, "fp8", True, "recompute")["saved"] == 0
    base = 1 << 40
    for which, training, name, limit in ((0, 1, b"pt_amax", f8["saved"]),
                                         (1, 0, b"pt_amax", moe.sizes(T, d, f, E, k, "fp8", False)["fwd_ws"]),
                                         (2, 1, b"pt_amax", f8["bwd_ws"]),
                                         (1, 1, b"a", f8["fwd_ws"]), (2, 1, b"dh", f8["bwd_ws"])):
        p = lib.moe_buffer_address_ex(T, k, E, d, f, 2, training, 0, which, base, name)
        assert p and (p - base) % 1024 == 0 and p - base < limit, (which, name)
    # MXFP8-only parts do not exist in the FP8 layout
    assert lib.moe_buffer_address_ex(T, k, E, d, f, 2, 1, 0, 1, base, b"w1_s") is None
    assert lib.moe_buffer_address_ex(T, k, E, d, f, 2, 1, 0, 0, base, b"xT_s") is None


def test_fp8_quantize_argument_checks(lib):
    """Refused on the host before anything is enqueued: no context, no row-wise flag, an unknown
    flag, rows or cols not multiples of 128."""
    assert lib.fp8_quantize(None, None, 1, 128, 128, 1, None, None, None, None) == 1
    assert lib.moe_tensor_peak_flops(None, 2, 10) == 0.0
