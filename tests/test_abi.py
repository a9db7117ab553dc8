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


def _create(**kw):
    from bit_quantized_mixture_b200 import moe
    cfg = dict(hidden=2048, inter=512, num_experts=512, top_k=10, quant=0, has_shared=1, max_tokens=8, device=0)
    cfg.update(kw)
    c = moe.Config(*(cfg[n] for n, _ in moe.Config._fields_))
    h = ctypes.c_void_p()
    st = moe.lib().moe_create(ctypes.byref(c), ctypes.byref(h))
    return st, moe.lib().moe_last_error(None).decode(), h


@pytest.mark.parametrize("kw,status,text", [
    ({"hidden": 0}, 1, "positive"),
    ({"max_tokens": -1}, 1, "positive"),
    ({"hidden": 2000}, 2, "multiples of 128"),
    ({"inter": 100}, 2, "multiples of 128"),
    ({"num_experts": 2048}, 2, "E <= 1024"),
    ({"top_k": 33}, 2, "k <= min"),
    ({"num_experts": 8, "top_k": 9}, 2, "k <= min"),
    ({"quant": 3}, 2, "routed quant"),
    ({"quant": 99}, 2, "routed quant"),
])
def test_create_rejects_unsupported_configurations_before_device_work(kw, status, text):
    """Shape, limit and format errors come back from moe_create before it
    touches a device, with no handle and a message naming the rule."""
    st, msg, h = _create(**kw)
    assert st == status and text in msg
    assert not h.value


def test_create_without_a_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    st, msg, h = _create()
    assert st == 1 and "no CUDA device" in msg and not h.value


def test_format_kernels_reject_null_arguments():
    from bit_quantized_mixture_b200 import moe
    L = moe.lib()
    for q in (0, 1, 2, 4, 5, 6):
        assert L.moe_quantize(q, None, 128, 128, ctypes.c_float(1.0), None, None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_absmax(None, 16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_sync_status(None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_forward(None, None, 1, None, None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_route_forward(None, None, 1, None, None, None, None) == moe.MOE_ERR_INVALID_ARG


def test_peak_loop_arguments_are_checked_on_the_host():
    from bit_quantized_mixture_b200 import moe
    L = moe.lib()
    flops = ctypes.c_double(0.0)
    dummy = ctypes.c_void_p(16)      # never dereferenced: the checks come first
    for kind, iss, iters in ((2, 1, 10), (0, 3, 10), (1, 4, 10), (1, 0, 10), (0, 1, 0)):
        assert L.moe_mma_peak_loop(kind, iss, iters, dummy, ctypes.byref(flops), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_mma_peak_loop(0, 1, 10, None, ctypes.byref(flops), None) == moe.MOE_ERR_INVALID_ARG
