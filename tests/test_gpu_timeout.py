"""The bounded device-side waits give up and report, without a fault: one CTA
of the fused decode kernel withholds its arrival at a grid barrier (the
library's test hook), every CTA's wait runs out after a short limit, the
kernel stops, moe_sync_status reports MOE_ERR_TIMEOUT and resets the barrier,
and the next call on the same handle is correct."""
import pytest
import torch

from bit_quantized_mixture_b200 import moe, synth
from bit_quantized_mixture_b200.layer import build_layer
from tests.gpu_util import bf16_tensor

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
SHORT = 2_000_000          # SM cycles: about a millisecond


@pytest.mark.parametrize("which_cta", ["first", "last"])
def test_withheld_arrival_times_out_and_the_handle_recovers(which_cta):
    wl = synth.custom("tiny-int4", H=384, I=256, E=16, k=4, shared=True, T=3)
    layer, _ = build_layer(wl, 0, max_tokens=8)
    layer.set_decode_path("fused")
    x = bf16_tensor(synth.activations_bf16(wl, steps=1)[:wl.T], DEV)
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device=DEV)
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device=DEV)
    y_ref = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=DEV)
    layer.route_forward(x, ids, w, y_ref)
    layer.sync_status()

    cta = 0 if which_cta == "first" else torch.cuda.get_device_properties(DEV).multi_processor_count - 1
    layer.debug_set_wait_test(cta, SHORT)
    y = torch.zeros_like(y_ref)
    layer.route_forward(x, ids, w, y)
    with pytest.raises(moe.MoeError) as ei:
        layer.sync_status()
    assert ei.value.status == moe.MOE_ERR_TIMEOUT
    assert "timed out" in str(ei.value) or "bounded wait" in str(ei.value)

    # the hook was one-shot and the barrier was reset: the next calls are correct
    for _ in range(2):
        y2 = torch.zeros_like(y_ref)
        layer.route_forward(x, ids, w, y2)
        layer.sync_status()
        assert torch.equal(y2, y_ref)
    layer.close()


def test_wait_test_hook_rejects_a_negative_limit():
    wl = synth.custom("tiny-int4", H=384, I=256, E=16, k=4, shared=True, T=3)
    layer = moe.MoeLayer(wl.H, wl.I, wl.E, wl.k, "int4", True, 8, 0)
    with pytest.raises(moe.MoeError) as ei:
        layer.debug_set_wait_test(0, -1)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    layer.debug_set_wait_test(-1, 0)        # clearing is always accepted
    layer.close()
