"""The tensor-core throughput loops that measure the peaks the grouped GEMMs'
tensor-pipe fractions are reported against: they run on every SM, their
bounded waits complete, and the throughput they report lies between a floor
far below any B200 figure and the nominal dense peak of the instruction kind
(bf16 2.25 PFLOP/s, e2m1 9 PFLOP/s) plus 10 %."""
import pytest
import torch

from bit_quantized_mixture_b200 import moe

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


@pytest.mark.parametrize("kind,issuers,nominal", [(0, 1, 2250.0), (0, 2, 2250.0), (1, 1, 9000.0), (1, 3, 9000.0)])
def test_peak_loop_runs_and_reports_a_plausible_rate(kind, issuers, nominal):
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    st = torch.cuda.current_stream()
    moe.mma_peak_loop(kind, issuers, 2000, err, st)          # warm-up
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    flops = moe.mma_peak_loop(kind, issuers, 20000, err, st)
    e1.record(st)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    sms = torch.cuda.get_device_properties(DEV).multi_processor_count
    n, k = (256, 16) if kind == 0 else (128, 64)
    assert flops == 2.0 * 128 * n * k * 20000 * issuers * sms
    tflops = flops / (e0.elapsed_time(e1) * 1e-3) / 1e12
    assert 50.0 < tflops < 1.1 * nominal, tflops
