"""The algorithmic work bench.py divides by kernel time: packed bytes of one
expert per format, grouped-GEMM FLOPs and the choice of the binding bound,
against figures derived independently from the formats' definitions."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bit_quantized_mixture_b200 import synth  # noqa: E402

PEAKS = {"hbm_gbs": 6538.6, "bf16_tflops": 1663.3}


@pytest.mark.parametrize("quant,total", [
    # per expert, all three matrices of 512 x 2048 weights:
    ("int4", 3 * (512 * 2048 // 2 + 512 * 16 * 2)),              # codes + fp16 scale per 128 = 1,622,016
    ("int2", 3 * (512 * 2048 // 4 + 512 * 16 * 2 + 512 * 16 // 4)),  # + 2-bit zero per 128 = 841,728
    ("nvfp4", 3 * (512 * 2048 // 2 + 512 * 2048 // 16)),          # e2m1 + e4m3 per 16 = 1,769,472
    ("int4g32", 3 * (512 * 2048 // 2 + 512 * 64 * 2)),
    ("fp8", 3 * (512 * 2048 + 4 * 16 * 4)),                       # E4M3 + fp32 per 128 x 128 block
    ("fp6", 3 * (512 * 2048 * 6 // 8 + 512 * 64 * 2)),            # 6 bits + fp16 scale per 32
])
def test_expert_bytes(quant, total):
    wl = synth.custom("decode-b1-int4", quant=quant)
    gu, dn = bench.expert_bytes(wl)
    assert gu + dn == total
    assert gu == 2 * dn                        # gate and up are each the size of down here (H x I)


def test_expert_bytes_match_the_stated_per_expert_sizes():
    sizes = {"int4": 1_622_016, "int2": 841_728, "nvfp4": 1_769_484}
    for quant, size in sizes.items():
        gu, dn = bench.expert_bytes(synth.custom("decode-b1-int4", quant=quant))
        # NVFP4's figure also counts three fp32 global scales (12 bytes)
        assert size - 12 <= gu + dn <= size


def test_prefill_flops():
    wl = synth.workload("prefill-int4-zipf")
    gu, dn = bench.prefill_flops(wl, wl.T * wl.k)
    assert gu + dn == pytest.approx(2 * 4096 * 10 * 3 * 2048 * 512)      # 257.7 GFLOP, no shared expert
    wl4 = synth.workload("prefill-nvfp4")
    gu4, dn4 = bench.prefill_flops(wl4, wl4.T * wl4.k)
    assert gu4 + dn4 == pytest.approx(2 * (8192 * 10 + 8192) * 3 * 2048 * 512)   # + the shared rows


def test_gateup_bound_follows_arithmetic_intensity():
    wl = synth.workload("prefill-int4-zipf")
    r = bench.gateup_roofline(wl, wl.T * wl.k, wl.E, 0.335, PEAKS, "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["arithmetic_intensity"] == pytest.approx(280.5, abs=0.1)        # > ridge 254
    assert r["ridge_flop_per_byte"] == pytest.approx(1663.3e3 / 6538.6)
    assert r["achieved"] == pytest.approx(2 * 40960 * 2048 * 1024 / 0.335e-3 / 1e12)
    wl4 = synth.workload("prefill-nvfp4")
    r4 = bench.gateup_roofline(wl4, wl4.T * wl4.k, wl4.E, 0.254, PEAKS, "measured")
    assert r4["bound"] == "hbm" and r4["unit"] == "GB/s"
    assert r4["tensor_peak_tflops"] == pytest.approx(4 * 1663.3)
    assert r4["arithmetic_intensity"] < r4["ridge_flop_per_byte"]


def test_nvfp4_roofline_takes_the_measured_e2m1_peak():
    wl4 = synth.workload("prefill-nvfp4")
    tp = {"e2m1_block16_tflops": 7000.0, "bf16_tflops": 2000.0}
    r = bench.gateup_roofline(wl4, wl4.T * wl4.k, wl4.E, 0.254, PEAKS, "measured", tp)
    assert r["tensor_peak_tflops"] == 7000.0
    assert r["frac_of_tensor_peak"] == pytest.approx(r["achieved_tflops"] / 7000.0)
    assert r["frac_of_tensor_peak_nominal_ratio"] == pytest.approx(r["achieved_tflops"] / (4 * 1663.3))
    assert "measured in this run" in r["peak_source"]
    # the bf16 formats keep the measured bf16 burst
    wl = synth.workload("prefill-int4-zipf")
    assert bench.gateup_roofline(wl, wl.T * wl.k, wl.E, 0.335, PEAKS, "measured", tp)["tensor_peak_tflops"] == 1663.3


def test_prefill_layer_fractions():
    wl = synth.workload("prefill-nvfp4")
    f = bench.prefill_layer_fractions(wl, 512, 0.5, PEAKS, 7000.0)
    gu, dn = bench.prefill_flops(wl, wl.T * wl.k)
    assert f["flops_per_step"] == pytest.approx(gu + dn + 2 * 8192 * 512 * 2048)
    g, d = bench.expert_bytes(wl)
    assert f["bytes_per_step"] == 512 * (g + d) + 512 * 2048 * 2 + 3 * 2048 * 512 * 2 + 2 * 8192 * 2048 * 2
    assert f["frac_of_hbm"] == pytest.approx(f["bytes_per_step"] / 0.5e-3 / 1e9 / 6538.6)


def test_default_line_is_the_largest_workload():
    args = bench.parse_args([])
    assert args.workload == "prefill-nvfp4"
    extra = args.extra_workloads.split(",")
    assert set(extra) == {"decode-b1-int4", "decode-b4-int2", "prefill-int4-zipf", "m-sweep"}
    line = {"value": 1.0, "unit": "tokens/s", "ms_per_step": 2.0, "config": {}, "roofline": {}, "metric": "m",
            "n_gpus": 1, "e2e": {}, "clocks": {}, "kernels_ms": {}, "layer": {}}
    e = bench.workload_entry(line)
    assert "metric" not in e and "n_gpus" not in e and e["roofline"] == {} and e["layer"] == {}


def test_traffic_is_reported_only_for_the_source_it_was_measured_on(tmp_path, monkeypatch):
    """The ncu DRAM bytes of a kernel key the sha256 of its source file: the
    bench reports them while that file is unchanged and null after an edit."""
    import hashlib
    import json

    src_dir = tmp_path / "bit_quantized_mixture_b200" / "csrc"
    src_dir.mkdir(parents=True)
    src = src_dir / "kernel.cu"
    src.write_text("// one kernel\n")
    (tmp_path / "profiles").mkdir()
    table = {"work-a:k_one": {"source": "kernel.cu", "sha256": hashlib.sha256(src.read_bytes()).hexdigest(),
                              "dram_bytes_per_launch": 123456, "from": "profiles/k_one.md"}}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(table))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_traffic("k_one", "work-a") == 123456
    assert bench.load_traffic("k_one", "work-b") is None          # another workload
    assert bench.load_traffic("k_two", "work-a") is None          # another kernel
    src.write_text("// one kernel, edited\n")
    assert bench.load_traffic("k_one", "work-a") is None
