"""Host logic of bench.py with several ranks (replicas, one process per GPU),
run as two gloo processes on the CPU: the rank environment, the barrier, the
maximum of the ranks' device times and the whole-job value of the JSON line."""
import os
import socket
import sys
import types

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bit_quantized_mixture_b200 import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world)})
    r_env, lr_env, w_env = bench.dist_env()
    assert (r_env, lr_env, w_env) == (rank, rank, world)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cpu = torch.device("cpu")
        # each replica measured its own device time; rank 1 was slower
        total = 10.0 + 5.0 * rank
        e2e = 20.0 + 1.0 * rank
        bench.barrier(world)
        tmax = bench.allreduce_max(total, cpu, world)
        emax = bench.allreduce_max(e2e, cpu, world)
        wl = synth.workload("decode-b1-int4")
        args = types.SimpleNamespace(steps=100, warmup=3, flush_mb=512, expert_table=False)
        r = {"steps_tokens": 100 * wl.T, "total_ms": tmax, "e2e_ms": emax, "roofline": {}, "kernels_ms": {},
             "h2d": 4096, "d2h": 4096, "launches_per_step": 3, "clocks": {}, "warm_ms_per_step": 0.03}
        line = bench.bench_line(args, wl, r, world, prefill=False)
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write("|".join(str(v) for v in (tmax, emax, line["value"], line["n_gpus"],
                                              line["config"]["parallelism"], line["scaling"], line["ms_per_step"])))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_replicas_max_time_and_whole_job_value(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    rows = [open(tmp_path / f"rank{r}.txt").read().split("|") for r in range(world)]
    for row in rows:
        tmax, emax, value, n, par, scaling, ms = row
        assert float(tmax) == 15.0 and float(emax) == 21.0          # max over ranks, on every rank
        # all ranks' tokens (2 x 100) over the slowest rank's time
        assert float(value) == pytest.approx(2 * 100 / 15.0e-3)
        assert int(n) == 2 and par == "replicas x2"
        assert scaling == "weak"
        assert float(ms) == pytest.approx(15.0 / 100)


@pytest.mark.parametrize("name,prefill", [("decode-b1-int4", False), ("prefill-int4-zipf", True)])
def test_bench_line_carries_the_contract_keys(name, prefill):
    """One JSON line with every key the measurement contract names, the
    roofline object's fields and the end-to-end object with its byte counts."""
    wl = synth.workload(name)
    args = types.SimpleNamespace(steps=20, warmup=3, flush_mb=512, expert_table=False)
    roof = {"bound": "hbm", "achieved": 1000.0, "peak": 6538.6, "unit": "GB/s", "frac": 1000.0 / 6538.6,
            "traffic": None}
    r = {"steps_tokens": 20 * wl.T, "total_ms": 2.0, "e2e_ms": 3.0, "roofline": roof, "kernels_ms": {"k": 0.1},
         "h2d": wl.T * wl.H * 2, "d2h": wl.T * wl.H * 2, "launches_per_step": 3,
         "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}, "e2e_method": "m"}
    line = bench.bench_line(args, wl, r, 1, prefill=prefill)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in line, key
    assert line["config"]["workload"] == name
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in line["roofline"], key
    e2e = line["e2e"]
    assert e2e["unit"] == line["unit"] and e2e["value"] == pytest.approx(20 * wl.T / 3.0e-3)
    assert e2e["h2d_bytes_per_step"] == wl.T * wl.H * 2 and e2e["d2h_bytes_per_step"] == wl.T * wl.H * 2
    assert line["value"] == pytest.approx(20 * wl.T / 2.0e-3)
    assert line["gpu_launches"] == 3 * 20
    assert line["higher_is_better"] is True and line["data"] == "synthetic"
