"""The C-ABI library loads and exports every entry point its header declares
(no GPU needed: nothing is called that touches a device)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:moe_status|float|const char\*)\s+(moe_\w+)\(", text, re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("moe_create", "moe_load_expert_weights", "moe_route", "moe_forward", "moe_destroy"):
        assert required in names


def test_library_exports_every_declared_symbol():
    from bit_quantized_mixture_b200 import moe
    if not os.path.exists(moe.LIB_PATH):
        pytest.fail("libmoe_b200.so is not built (python -m bit_quantized_mixture_b200.build)")
    L = ctypes.CDLL(moe.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_host_only_entry_points():
    from bit_quantized_mixture_b200 import moe
    L = moe.lib()
    assert L.moe_status_str(0) == b"ok"
    assert L.moe_status_str(3) == b"invalid state"
    # amax / (6 * 448) in fp32
    assert moe.nvfp4_global_scale(2688.0) == 1.0
    # null configuration is rejected before any device work
    assert L.moe_create(None, None) == moe.MOE_ERR_INVALID_ARG
    assert b"null" in L.moe_last_error(None)
