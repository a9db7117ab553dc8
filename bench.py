#!/usr/bin/env python
"""Throughput of the routed-expert MoE layer on B200 (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the CPU oracle arm

A step is one pass of the whole layer (router, top-k, expert GEMVs/GEMMs,
combine) over one batch of seeded synthetic tokens of the workload.  Default
workload: the largest configuration, a prefill chunk of T=8192 tokens with
NVFP4 W4A4 routed experts (H=2048, I=512, E=512, top-10, uniform routing,
one bf16 shared expert).  The same run also measures the other workloads of
the metric (decode batch 1 INT4, decode batch 4 INT2, prefill INT4 with Zipf
routing) and reports each under "workloads", and it measures the tensor-core
peaks it reports fractions against with its own tcgen05 throughput loops.
Multi-GPU: one process per GPU (torchrun); every rank runs an independent
replica on its own tokens (the layer is per-token, so there is no exchange),
and the slowest rank's device time defines the whole-job throughput.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "prefill-nvfp4"
EXTRA_WORKLOADS = "decode-b1-int4,decode-b4-int2,prefill-int4-zipf,m-sweep"
METRIC = "MoE-layer tokens/s; decode HBM GB/s and prefill TFLOPS as % of B200 roofline"
UNIT = "tokens/s"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--extra-workloads", default=EXTRA_WORKLOADS,
                    help="comma-separated workloads measured after the main one ('none': only the main one)")
    ap.add_argument("--no-peak-loop", action="store_true", help="skip the tensor-core peak loops")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="bounded oracle sample length")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--flush-mb", type=int, default=512)
    ap.add_argument("--expert-table", action="store_true",
                    help="read the routed experts through the per-expert address table from a shuffled pool")
    return ap.parse_args(argv)


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ----------------------------------------------------------- clock sampling
class _NoClock:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        # samples go to a file named by BENCH_CLOCKS_DIR when set (to keep
        # the raw record), else to a temporary file
        out_dir = os.environ.get("BENCH_CLOCKS_DIR") or None
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv", dir=out_dir)
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        time.sleep(0.25)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) < 9 or parts[0] != str(self.idx):
                        continue
                    try:
                        sm.append(float(parts[1]))
                        smax.append(float(parts[2]))
                    except ValueError:
                        continue
                    for n, v in zip(names, parts[5:9]):
                        if v.lower() == "active":
                            reasons.add(n)
        except OSError:
            pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# -------------------------------------------------------------- oracle arm
NVFP4_INTER_AMAX = 8.0   # calibration bound of the W4A4 intermediate (see prefill_act_scales)


class OracleSampler:
    """Times the CPU oracle (as it stands) on bounded samples of a workload.

    Decode workloads: whole decode steps (router, top-k, expert SwiGLU from
    the packed weights, combine).  Prefill workloads: chunks of 4 consecutive
    tokens of the batch (top-k of the workload's routing logits, expert
    SwiGLU, combine).  Prefill samples cycle over the first `prefill_chunks`
    chunks of the batch, so the set of experts to quantize stays bounded.
    Quantization of the weights is set-up, as on the GPU: it is not timed,
    runs in a thread pool, is kept across samples, and stops a sample early
    once it has taken `setup_cap_s` in total."""

    def __init__(self, wl, setup_cap_s=90.0, prefill_chunks=4):
        from bit_quantized_mixture_b200 import synth
        from oracle import moe_oracle as O
        self.O, self.synth, self.wl = O, synth, wl
        self.setup_cap_s = setup_cap_s
        self.xs = synth.activations_bf16(wl)
        self.prefill = wl.routing != "router"
        self.wr = None if self.prefill else synth.router_bf16(wl)
        self.logits = synth.routing_logits(wl) if self.prefill else None
        self.shared = tuple(O.bf16_bits_to_f64(m) for m in synth.shared_bf16(wl)) if wl.shared else None
        self.act = None
        if wl.quant == "nvfp4":
            g_x = O.nvfp4_global_scale(np.abs(O.bf16_bits_to_f32(self.xs)).max())
            self.act = (g_x, O.nvfp4_global_scale(NVFP4_INTER_AMAX))
        self.q = {}
        self.setup = 0.0
        self.chunk = 4 if self.prefill else wl.T
        self.n_chunks = min(wl.T // self.chunk, prefill_chunks) if self.prefill else wl.steps

    def quantized(self, e):
        O, wl = self.O, self.wl
        if e not in self.q:
            t0 = time.perf_counter()
            g, u, d = self.synth.expert_fp32(wl, e)
            ew = {}
            if wl.quant == "nvfp4":
                g_gu = O.nvfp4_global_scale(max(np.abs(g).max(), np.abs(u).max()))
                g_d = O.nvfp4_global_scale(np.abs(d).max())
            for name, m in zip(("gate", "up", "down"), (g, u, d)):
                if wl.quant in ("int4", "int4g32"):
                    c, sc = O.quantize_int4(m, group=32 if wl.quant == "int4g32" else 128)
                    ew[name] = {"codes": c, "scales": sc}
                elif wl.quant == "fp8":
                    c, sc = O.quantize_fp8_block(m)
                    ew[name] = {"codes": c, "scales": sc}
                elif wl.quant == "fp6":
                    c, sc = O.quantize_fp6(m)
                    ew[name] = {"codes": c, "scales": sc}
                elif wl.quant == "int2":
                    c, sc, z = O.quantize_int2(m)
                    ew[name] = {"codes": c, "scales": sc, "zeros": z}
                else:
                    gg = g_d if name == "down" else g_gu
                    c, sc = O.quantize_nvfp4(m, gg)
                    ew[name] = {"codes": c, "scales": sc, "g": gg}
            self.q[e] = ew
            self.setup += time.perf_counter() - t0
        return self.q[e]

    def _route(self, i, x):
        lg = self.logits[i * self.chunk:(i + 1) * self.chunk] if self.prefill else self.O.router_logits(x, self.wr)
        return self.O.route_topk(lg, self.wl.k)

    def sample(self, seconds, offset=0):
        """(tokens/s, info) over chunks starting at chunk `offset`."""
        from threadpoolctl import threadpool_info
        O, wl = self.O, self.wl
        spent, tokens, done = 0.0, 0, 0
        while spent < seconds and done < self.n_chunks and (done == 0 or self.setup < self.setup_cap_s):
            i = (offset + done) % self.n_chunks
            x = self.xs[i * self.chunk:(i + 1) * self.chunk]
            ids_probe, _ = self._route(i, x)
            new = [int(e) for e in np.unique(ids_probe) if int(e) not in self.q]
            if new:
                from concurrent.futures import ThreadPoolExecutor
                with ThreadPoolExecutor(max(1, min(len(new), os.cpu_count() or 4))) as ex:
                    list(ex.map(self.quantized, new))
            t0 = time.perf_counter()
            ids, w = self._route(i, x)
            O.moe_forward(x, ids, w, wl.quant, lambda e: O.dequantize_expert(wl.quant, self.quantized(e)),
                          shared=self.shared, act_scales=self.act)
            spent += time.perf_counter() - t0
            tokens += self.chunk
            done += 1
        threads = max([d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"] or [1])
        what = f"{done} chunks x {self.chunk} tokens" if self.prefill else f"{done} steps x {wl.T} tokens"
        return tokens / spent, {"cores": int(threads), "sample": f"{what} of {wl.name}", "seconds": spent}


def oracle_tokens_per_s(wl, seconds, rank_offset=0):
    return OracleSampler(wl).sample(seconds, rank_offset)


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    from bit_quantized_mixture_b200 import synth
    wl = synth.workload(args.workload)
    per_step = max(0.5, args.cpu_seconds / max(1, args.steps))
    sampler = OracleSampler(wl)
    vals = []
    for _ in range(args.warmup):
        sampler.sample(per_step / 4)
    info = None
    for s in range(args.steps):
        v, info = sampler.sample(per_step, offset=s)
        vals.append(v)
    value = float(np.mean(vals))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * wl.T / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "k": wl.k,
                       "quant": wl.quant, "shared": wl.shared},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": info["cores"], "kind": "oracle",
                             "sample": info["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm
def expert_bytes(wl):
    """Packed bytes of one routed expert's gate+up and down matrices."""
    H, I = wl.H, wl.I
    if wl.quant in ("int4", "int4g32"):
        gs = 32 if wl.quant == "int4g32" else 128
        gu = 2 * (I * H // 2 + I * (H // gs) * 2)
        dn = H * I // 2 + H * (I // gs) * 2
    elif wl.quant == "fp8":
        gu = 2 * (I * H + (I // 128) * (H // 128) * 4)
        dn = H * I + (H // 128) * (I // 128) * 4
    elif wl.quant == "fp6":
        gu = 2 * (I * H * 3 // 4 + I * (H // 32) * 2)
        dn = H * I * 3 // 4 + H * (I // 32) * 2
    elif wl.quant == "int2":      # 2-bit zeros, four per byte (the algorithmic minimum)
        gu = 2 * (I * H // 4 + I * (H // 128) * 2 + (I // 4) * (H // 128))
        dn = H * I // 4 + H * (I // 128) * 2 + (H // 4) * (I // 128)
    else:
        gu = 2 * (I * H // 2 + I * (H // 16))
        dn = H * I // 2 + H * (I // 16)
    return gu, dn


def expert_pool(layer, wl, dev):
    """Move the routed experts' blocks into a separate device pool in a
    seeded shuffled order and point the layer's address table at them (the
    kernels then read every expert through the table)."""
    import torch
    bb = layer.expert_block_bytes()
    pool = torch.empty(wl.E * bb + 256, dtype=torch.uint8, device=dev)
    base = (pool.data_ptr() + 255) // 256 * 256
    slot = np.random.default_rng(1234).permutation(wl.E)
    for e in range(wl.E):
        off = base - pool.data_ptr() + int(slot[e]) * bb
        layer.export_expert(e, pool[off:off + bb])
    torch.cuda.synchronize(dev)
    layer.set_expert_table([base + int(slot[e]) * bb for e in range(wl.E)])
    return pool


class _DeviceView:
    """A device address range seen by torch as a CUDA array (no copy)."""

    def __init__(self, ptr, nbytes):
        self.__cuda_array_interface__ = {"shape": (nbytes // 2,), "typestr": "<i2", "data": (ptr, False),
                                         "version": 3}


def _mapped_host_pair(cudart, nbytes, dev):
    """Two mapped pinned host buffers of nbytes and torch views of their
    device addresses, or None where the device cannot map host memory."""
    import torch
    err, can_map = cudart.cudaDeviceGetAttribute(cudart.cudaDeviceAttr.cudaDevAttrCanMapHostMemory, dev.index)
    if err != cudart.cudaError_t.cudaSuccess or not can_map:
        return None
    out = []
    for _ in range(2):
        err, h = cudart.cudaHostAlloc(nbytes, cudart.cudaHostAllocMapped)
        if err != cudart.cudaError_t.cudaSuccess:
            return None
        err, d = cudart.cudaHostGetDevicePointer(h, 0)
        if err != cudart.cudaError_t.cudaSuccess:
            cudart.cudaFreeHost(h)
            return None
        out.append((h, d))
    (hx, dx), (hy, dy) = out
    return hx, hy, torch.as_tensor(_DeviceView(dx, nbytes), device=dev), torch.as_tensor(_DeviceView(dy, nbytes), device=dev)


def measure_tensor_peaks(dev):
    """Burst throughput of the library's tcgen05 loops on this GPU (every SM;
    operands resident in shared memory): bf16 kind::f16 (M128 N256 K16) and
    the block-scaled e2m1 kind::mxf4nvf4 (M128 N128 K64), best of several
    launches and issuing-warp counts, each launch a few milliseconds."""
    import torch

    from bit_quantized_mixture_b200 import moe
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    out = {}
    for kind, name, issuers, iters in ((0, "bf16_tflops", (1, 2), 20000), (1, "e2m1_block16_tflops", (1, 2, 3), 40000)):
        best, best_iss = 0.0, 0
        for iss in issuers:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(6)]
            flops = 0.0
            with torch.cuda.stream(stream):
                for e0, e1 in evs:
                    e0.record(stream)
                    flops = moe.mma_peak_loop(kind, iss, iters, err, stream)
                    e1.record(stream)
            stream.synchronize()
            t = min(a.elapsed_time(b) for a, b in evs[1:])
            tf = flops / (t * 1e-3) / 1e12
            if tf > best:
                best, best_iss = tf, iss
        out[name] = best
        out[name.replace("_tflops", "_issuers")] = best_iss
    if int(err.item()) != 0:
        raise RuntimeError(f"tensor peak loop: a bounded wait gave up (code {int(err.item())})")
    out["method"] = ("tcgen05 throughput loops of the library (moe_mma_peak_loop): one CTA per SM, operands "
                     "resident in shared memory, fp32 accumulators in TMEM; best of 5 timed launches (CUDA events) "
                     "over 1..3 issuing warps")
    return out


def run_decode(args, wl, dev, rank, world):
    import torch

    from bit_quantized_mixture_b200 import synth
    from bit_quantized_mixture_b200.layer import build_layer

    layer, _ = build_layer(wl, dev.index, max_tokens=wl.T)
    pool = expert_pool(layer, wl, dev) if args.expert_table else None
    # the path moe_route_forward takes inside a CUDA graph (router kernel and
    # the two GEMV kernels), also for the eager per-kernel breakdown below
    layer.set_decode_path("kernels")
    xs_host = synth.activations_bf16(wl)
    xs = torch.from_numpy(xs_host.view(np.int16)).to(dev).view(torch.bfloat16)
    T, k = wl.T, wl.k
    nsteps = wl.steps
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    y = torch.empty((T, wl.H), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(args.flush_mb * (1 << 20) // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    off = rank * 37  # replicas work on different tokens

    # one CUDA graph per seeded token batch: route + forward
    graphs = []
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for i in range(nsteps):       # eager pass first (also a warm-up of every path)
            xi = xs[i * T:(i + 1) * T]
            layer.route_forward(xi, ids, w, y)
    stream.synchronize()
    for i in range(nsteps):
        g = torch.cuda.CUDAGraph()
        xi = xs[i * T:(i + 1) * T]
        with torch.cuda.graph(g, stream=stream):
            layer.route_forward(xi, ids, w, y)
        graphs.append(g)
    torch.cuda.synchronize(dev)

    def step_index(s):
        return (off + s) % nsteps

    with torch.cuda.stream(stream):
        for s in range(args.warmup):
            flush.zero_()
            graphs[step_index(s)].replay()
    stream.synchronize()

    # ---- timed region: device time of K steps, L2 flushed between steps
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev.index)
    with clocks:
        with torch.cuda.stream(stream):
            for s in range(args.steps):
                flush.zero_()
                ev0[s].record(stream)
                graphs[step_index(s)].replay()
                ev1[s].record(stream)
        stream.synchronize()
        torch.cuda.synchronize(dev)
        barrier(world)
    step_ms = [a.elapsed_time(b) for a, b in zip(ev0, ev1)]
    total_ms = float(sum(step_ms))
    total_ms_max = allreduce_max(total_ms, dev, world)

    # ---- the same steps back to back with warm caches (no flush): the
    # router and shared expert stay L2-resident, and experts that repeat
    w0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    w1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with torch.cuda.stream(stream):
        for s in range(args.steps):
            w0[s].record(stream)
            graphs[step_index(s)].replay()
            w1[s].record(stream)
    stream.synchronize()
    warm_ms = allreduce_max(float(sum(a.elapsed_time(b) for a, b in zip(w0, w1))), dev, world)

    # ---- per-kernel breakdown (events between the library's kernels)
    # Kernel time: eager launches with the library's profiling events around
    # its one kernel (events inside graphs cannot be timed).  The 512 MB flush
    # before each step keeps the host ahead of the GPU.
    pev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    with torch.cuda.stream(stream):
        for evs in pev:            # torch creates the CUDA event on first record
            for ev in evs:
                ev.record(stream)
    stream.synchronize()
    with torch.cuda.stream(stream):
        for s in range(args.steps):
            i = step_index(s)
            # several flushes: the GPU then takes longer than the host needs to
            # queue the three kernels, so the events time the kernels, not
            # the host's launch calls
            for _ in range(4):
                flush.zero_()
            layer.set_profile_events(pev[s])
            layer.route_forward(xs[i * T:(i + 1) * T], ids, w, y)
    layer.set_profile_events(None)
    stream.synchronize()
    k_router = [p[0].elapsed_time(p[1]) for p in pev]
    k_gateup = [p[2].elapsed_time(p[3]) for p in pev]
    k_down = [p[3].elapsed_time(p[4]) for p in pev]
    uniq_per_step = []
    with torch.cuda.stream(stream):
        for s in range(args.steps):
            i = step_index(s)
            layer.route(xs[i * T:(i + 1) * T], ids, w)
            uniq_per_step.append(torch.unique(ids).numel())
    stream.synchronize()

    # ---- end to end through the public API with host buffers: one CUDA graph
    # per seeded token (the steps stay serial, as a decode loop's are).  x and
    # y live in mapped pinned host memory: a small copy kernel reads the
    # step's x from it into a device buffer, and the layer writes y into it
    # directly (4 KB each way; a copy-engine transfer costs several times a
    # kernel's latency at this size).  Where mapped memory cannot be had, the
    # graph copies with cudaMemcpyAsync instead.
    from cuda.bindings import runtime as cudart
    row_bytes = T * wl.H * 2
    x_stage = torch.empty((T, wl.H), dtype=torch.bfloat16, device=dev)
    mapped = _mapped_host_pair(cudart, nsteps * row_bytes, dev)
    if mapped is not None:
        hx, hy, x_map, y_map = mapped
        np.copyto(np.ctypeslib.as_array((ctypes.c_int16 * (nsteps * T * wl.H)).from_address(hx)),
                  xs_host.view(np.int16).reshape(-1))
        x_map = x_map.view(torch.bfloat16).view(nsteps, T, wl.H)
        y_map = y_map.view(torch.bfloat16).view(nsteps, T, wl.H)
        e2e_method = "mapped"
    else:
        x_pin = torch.from_numpy(xs_host.view(np.int16)).view(torch.bfloat16).pin_memory()
        y_pin = torch.empty((nsteps, T, wl.H), dtype=torch.bfloat16).pin_memory()
        e2e_method = "memcpy"

    def memcpy(dst, src, kind):
        err, = cudart.cudaMemcpyAsync(dst, src, row_bytes, kind, stream.cuda_stream)
        if err != cudart.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaMemcpyAsync: {err}")

    g_e2e = []
    for i in range(nsteps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            if e2e_method == "mapped":
                torch.mul(x_map[i], 1, out=x_stage)
                layer.route_forward(x_stage, ids, w, y_map[i])
            else:
                memcpy(x_stage.data_ptr(), x_pin[i * T:(i + 1) * T].data_ptr(),
                       cudart.cudaMemcpyKind.cudaMemcpyHostToDevice)
                layer.route_forward(x_stage, ids, w, y)
                memcpy(y_pin[i].data_ptr(), y.data_ptr(), cudart.cudaMemcpyKind.cudaMemcpyDeviceToHost)
        g_e2e.append(g)
    with torch.cuda.stream(stream):
        for g in g_e2e:                 # first replays upload the graphs
            g.replay()
    stream.synchronize()
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for s in range(args.steps):
            i = step_index(s)
            flush.zero_()
            e0[s].record(stream)
            g_e2e[i].replay()
            e1[s].record(stream)
    stream.synchronize()
    # the host's copy of the last step's y against the device path's result
    last = step_index(args.steps - 1)
    with torch.cuda.stream(stream):
        layer.route_forward(xs[last * T:(last + 1) * T], ids, w, y)
    stream.synchronize()
    y_host = y_map[last].cpu() if e2e_method == "mapped" else y_pin[last]
    if not torch.equal(y_host, y.cpu()):
        raise RuntimeError("end-to-end decode: the host copy of y differs from the device result")
    del g_e2e
    if e2e_method == "mapped":
        del x_map, y_map
        torch.cuda.synchronize(dev)
        cudart.cudaFreeHost(hx)
        cudart.cudaFreeHost(hy)
    e2e_ms = float(sum(a.elapsed_time(b) for a, b in zip(e0, e1)))
    e2e_ms_max = allreduce_max(e2e_ms, dev, world)

    # ---- roofline of the dominant decode kernel: its algorithmic bytes over
    # its event-measured duration.  router: Wr, x, logits; gate/up: the
    # distinct experts' gate and up weights, the shared gate/up, x and the fp32
    # intermediates; down: the distinct experts' down weights, the shared down,
    # the intermediates, the fp32 partials (written and read) and y.
    gu_b, dn_b = expert_bytes(wl)
    H, I = wl.H, wl.I
    mean_uniq = float(np.mean(uniq_per_step))
    rows = T * k + T
    by = {
        "k_router_small": wl.E * H * 2 + T * H * 2 + T * wl.E * 4,
        "k_dec_gateup": mean_uniq * gu_b + (2 * I * H * 2 if wl.shared else 0) + T * H * 2 + rows * I * 4,
        "k_dec_down": mean_uniq * dn_b + (I * H * 2 if wl.shared else 0) + rows * I * 4 + rows * H * 4 * 2
                      + T * H * 2,
    }
    step_bytes = float(sum(by.values()))
    kern = {"k_router_small": float(np.mean(k_router)), "k_dec_gateup": float(np.mean(k_gateup)),
            "k_dec_down": float(np.mean(k_down))}
    dom = max(kern, key=kern.get)
    peaks, peak_kind = measured_peaks()
    achieved = by[dom] / (kern[dom] * 1e-3) / 1e9
    traffic = load_traffic(dom, wl.name)
    layer.close()
    return {
        "total_ms": total_ms_max, "steps_tokens": args.steps * T, "e2e_ms": e2e_ms_max,
        "clocks": clocks.summary(), "kernels_ms": kern, "dominant": dom,
        "e2e_method": ("one CUDA graph per step, steps serial: " +
                       ("a copy kernel reads x from mapped pinned host memory, the layer writes y into mapped "
                        "pinned host memory" if e2e_method == "mapped" else
                        "cudaMemcpyAsync of x from and of y to pinned host memory around the layer call")),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "algorithmic_bytes_per_launch": by[dom], "peak_source": peak_kind,
                     "decode_path": "router kernel + two GEMV kernels (CUDA graph)"},
        "layer_gbs": step_bytes / (total_ms / args.steps * 1e-3) / 1e9,
        "layer": {"bytes_per_step": step_bytes, "hbm_gbs": step_bytes / (total_ms / args.steps * 1e-3) / 1e9,
                  "frac_of_hbm": step_bytes / (total_ms / args.steps * 1e-3) / 1e9 / peaks["hbm_gbs"],
                  "ms_per_step": total_ms / args.steps,
                  "note": "whole step (graph-timed, kernels overlapping through programmatic launch) against "
                          "HBM; the roofline object is the dominant kernel timed alone with events"},
        "warm_ms_per_step": warm_ms / args.steps,
        "launches_per_step": 3, "h2d": T * H * 2, "d2h": T * H * 2, "mean_distinct_experts": mean_uniq,
    }


def run_m_sweep(args, dev, rank, world):
    """Tokens per call M = 1, 2, 4, 8, 16 on the decode-b1 INT4 layer (H=2048,
    I=512, E=512, top-10, bf16 shared expert): one CUDA graph of
    moe_route_forward per seeded token batch on the GEMV path and on the
    grouped-GEMM path, L2 flushed before every step; mean device time per
    step and the smallest M at which the grouped GEMM is the faster."""
    import torch

    from bit_quantized_mixture_b200 import synth
    from bit_quantized_mixture_b200.layer import build_layer
    wl = synth.workload("decode-b1-int4")
    layer, _ = build_layer(wl, dev.index, max_tokens=16)
    xs = torch.from_numpy(synth.activations_bf16(wl).view(np.int16)).to(dev).view(torch.bfloat16)
    flush = torch.empty(args.flush_mb * (1 << 20) // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    nb = 6                       # distinct token batches per M (cycled)
    table = {}
    for M in (1, 2, 4, 8, 16):
        row = {}
        ids = torch.empty((M, wl.k), dtype=torch.int32, device=dev)
        w = torch.empty((M, wl.k), dtype=torch.float32, device=dev)
        y = torch.empty((M, wl.H), dtype=torch.bfloat16, device=dev)
        for path in ("kernels", "gemm"):
            layer.set_decode_path(path)
            graphs = []
            for b in range(nb):
                xb = xs[(b * M) % (wl.steps - M + 1):][:M]
                with torch.cuda.stream(stream):
                    layer.route_forward(xb, ids, w, y)           # warm-up, uploads nothing new
                stream.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    layer.route_forward(xb, ids, w, y)
                graphs.append(g)
            steps = max(args.steps, 2 * nb)
            e0 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
            e1 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
            with torch.cuda.stream(stream):
                for s in range(nb):
                    flush.zero_()
                    graphs[s].replay()
                for s in range(steps):
                    flush.zero_()
                    e0[s].record(stream)
                    graphs[s % nb].replay()
                    e1[s].record(stream)
            stream.synchronize()
            layer.sync_status(stream)
            ms = allreduce_max(float(np.mean([a.elapsed_time(b) for a, b in zip(e0, e1)])), dev, world)
            row["gemv_us" if path == "kernels" else "gemm_us"] = ms * 1e3
            del graphs
        row["tokens_per_s_gemv"] = M / (row["gemv_us"] * 1e-6)
        table[str(M)] = row
    layer.set_decode_path("auto")
    layer.close()
    cross = next((int(m) for m, r in table.items() if r["gemm_us"] < r["gemv_us"]), None)
    return {"workload": "decode-b1-int4 layer, M tokens per call", "l2": "flushed between steps",
            "us_per_step": table, "gemm_faster_from_M": cross,
            "method": "one CUDA graph of moe_route_forward per token batch; decode path 'kernels' (GEMV) vs 'gemm'"}


def prefill_flops(wl, slots):
    """Algorithmic FLOPs of the grouped GEMMs of one prefill step: gate/up
    2*m*H*2I and down 2*m*I*H over the routed slots and the shared rows."""
    m = slots + (wl.T if wl.shared else 0)
    return 2.0 * m * wl.H * 2 * wl.I, 2.0 * m * wl.I * wl.H


def gateup_roofline(wl, slots, experts_touched, t_ms, peaks, peak_kind, tensor_peaks=None):
    """Roofline of the routed gate/up grouped GEMM (one launch).  Algorithmic
    work: FLOPs 2 * slots * H * 2I; bytes = the touched experts' packed gate
    and up weights (codes + scales [+ zeros]) once, the token activations once
    (bf16 x for INT4/INT2, e2m1 codes + e4m3 scales for NVFP4) and the
    intermediate written once (bf16, or e2m1 + e4m3 for NVFP4).  The binding
    bound is the larger of FLOPs / tensor peak and bytes / HBM bandwidth; the
    tensor peak is the measured bf16 burst (fp16 operands run at the same
    rate); for the block-scaled e2m1 MMA it is the e2m1 peak measured by this
    run's tcgen05 loop when given (else 4 x the bf16 burst, the nominal
    9 : 2.25 ratio, which is also reported)."""
    H, I, T = wl.H, wl.I, wl.T
    n = 2 * I                                     # gate + up rows per expert
    if wl.quant in ("int4", "int4g32"):
        w_bytes = n * H // 2 + n * (H // (32 if wl.quant == "int4g32" else 128)) * 2
        act, out = T * H * 2, slots * I * 2
    elif wl.quant == "fp8":
        w_bytes = n * H + (n // 128) * (H // 128) * 4
        act, out = T * H * 2, slots * I * 2
    elif wl.quant == "fp6":
        w_bytes = n * H * 3 // 4 + n * (H // 32) * 2
        act, out = T * H * 2, slots * I * 2
    elif wl.quant == "int2":
        w_bytes = n * H // 4 + n * (H // 128) * 2 + (n // 4) * (H // 128)
        act, out = T * H * 2, slots * I * 2
    else:
        w_bytes = n * H // 2 + n * (H // 16)
        act, out = T * (H // 2 + H // 16), slots * (I // 2 + I // 16)
    flops = 2.0 * slots * H * n
    nbytes = float(experts_touched * w_bytes + act + out)
    t = t_ms * 1e-3
    fp4 = wl.quant == "nvfp4"
    nominal_fp4 = peaks["bf16_tflops"] * 4.0
    fp4_measured = bool(fp4 and tensor_peaks and tensor_peaks.get("e2m1_block16_tflops"))
    tensor_peak = (tensor_peaks["e2m1_block16_tflops"] if fp4_measured else nominal_fp4) if fp4 else peaks["bf16_tflops"]
    hbm = peaks["hbm_gbs"]
    t_tensor, t_hbm = flops / (tensor_peak * 1e12), nbytes / (hbm * 1e9)
    tfl, gbs = flops / t / 1e12, nbytes / t / 1e9
    kname = "k_fp4_gemm<0> (routed gate/up)" if wl.quant == "nvfp4" else "k_grouped_gemm<0,false> (routed gate/up)"
    common = {"kernel": kname, "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": nbytes,
              "arithmetic_intensity": flops / nbytes, "ridge_flop_per_byte": tensor_peak * 1e3 / hbm,
              "achieved_tflops": tfl, "tensor_peak_tflops": tensor_peak, "frac_of_tensor_peak": tfl / tensor_peak,
              "achieved_gbs": gbs, "frac_of_hbm": gbs / hbm, "ms_per_launch": t_ms,
              "peak_source": ((("e2m1 block-scaled peak measured in this run by the library's tcgen05 loop"
                                if fp4_measured else f"{peak_kind} dense bf16 burst x 4 (nominal e2m1 : bf16 ratio)")
                               if fp4 else f"{peak_kind} dense bf16 burst") + f"; {peak_kind} HBM copy bandwidth")}
    if fp4:
        common["frac_of_tensor_peak_nominal_ratio"] = tfl / nominal_fp4
    if t_hbm >= t_tensor:
        return dict({"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm}, **common)
    return dict({"bound": "tensor", "achieved": tfl, "peak": tensor_peak, "unit": "TFLOP/s", "frac": tfl / tensor_peak},
                **common)


def run_prefill(args, wl, dev, rank, world, tensor_peaks=None):
    """A prefill step: router GEMM on x (logits only), softmax/top-k of the
    workload's synthetic routing logits (the skewed / uniform routing the
    workload prescribes, standing in for the router's own), permutation,
    gate/up and down grouped GEMMs, combine: the layer's work once.  Eager
    launches; per-kernel events in a separate pass."""
    import torch

    from bit_quantized_mixture_b200 import moe, synth
    from bit_quantized_mixture_b200.layer import build_layer

    layer, _ = build_layer(wl, dev.index, max_tokens=wl.T)
    pool = expert_pool(layer, wl, dev) if args.expert_table else None
    T, k, H, E = wl.T, wl.k, wl.H, wl.E
    x_host = synth.activations_bf16(wl)
    lg_host = synth.routing_logits(wl).astype(np.float32)
    x = torch.from_numpy(x_host.view(np.int16)).to(dev).view(torch.bfloat16)
    lg = torch.from_numpy(lg_host).to(dev)
    if wl.quant == "nvfp4":
        # static W4A4 activation scales (set-up, not timed): g_x from the
        # batch's |x| max, g_a from a fixed calibration bound (values of the
        # intermediate above it saturate to the largest code)
        amax = torch.zeros(1, dtype=torch.float32, device=dev)
        moe.absmax(x.float(), amax)
        layer.set_act_global_scales(moe.nvfp4_global_scale(float(amax.item())),
                                    moe.nvfp4_global_scale(NVFP4_INTER_AMAX))
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(args.flush_mb * (1 << 20) // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(xin, lgin, yout=y):
        layer.route(xin, None, None, logits=logits)   # router GEMM (logits only)
        layer.route_from_logits(lgin, ids, w)         # the workload's routing
        layer.forward(xin, ids, w, yout)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            step(x, lg)
    layer.sync_status(stream)

    # the step as one CUDA graph (the layer's launches replayed without host
    # launch gaps); the eager step is timed too and reported beside it
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step(x, lg)
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            graph.replay()
    layer.sync_status(stream)

    def timed(run, clock=None):
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        barrier(world)
        torch.cuda.synchronize(dev)
        with (clock if clock is not None else _NoClock()):
            with torch.cuda.stream(stream):
                for s in range(args.steps):
                    flush.zero_()
                    e0[s].record(stream)
                    run()
                    e1[s].record(stream)
            stream.synchronize()
            torch.cuda.synchronize(dev)
            barrier(world)
        layer.sync_status(stream)
        return allreduce_max(float(sum(a.elapsed_time(b) for a, b in zip(e0, e1))), dev, world)

    clocks = ClockSampler(dev.index)
    total_ms_max = timed(graph.replay, clocks)
    eager_ms_max = timed(lambda: step(x, lg))
    del graph

    # ---- per-kernel breakdown: the library's profiling events
    pev = [[torch.cuda.Event(enable_timing=True) for _ in range(10)] for _ in range(args.steps)]
    with torch.cuda.stream(stream):
        for evs in pev:
            for ev in evs:
                ev.record(stream)
    stream.synchronize()
    with torch.cuda.stream(stream):
        for s in range(args.steps):
            flush.zero_()
            layer.set_profile_events(pev[s])
            step(x, lg)
    layer.set_profile_events(None)
    stream.synchronize()

    def mean_ms(i, j):
        return float(np.mean([p[i].elapsed_time(p[j]) for p in pev]))

    kern = {"route_router_gemm": mean_ms(0, 1), "forward": mean_ms(2, 4), "grouped_gemm_gate_up": mean_ms(5, 3),
            "grouped_gemm_gate_up_routed": mean_ms(5, 8), "grouped_gemm_down": mean_ms(6, 7),
            "grouped_gemm_down_routed": mean_ms(6, 9), "combine": mean_ms(7, 4)}
    experts_touched = int(np.count_nonzero(np.bincount(ids.cpu().numpy().ravel(), minlength=E)))

    # ---- end to end through the public API: x and the routing logits from
    # pinned host memory, y back to pinned host memory.  Prefill chunks are
    # independent, so the next chunk's inputs are copied in and the previous
    # chunk's output copied out (two copy streams, two staging buffers) while
    # a chunk computes; the layer's own work stays on one stream (its
    # workspace is shared).  Timed from the first input copy to the last
    # output copy.  The working set (every expert's weights) exceeds L2, so
    # no flush is interleaved.
    x_pin = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).pin_memory()
    lg_pin = torch.from_numpy(lg_host).pin_memory()
    y_pin = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_st = [torch.empty_like(x) for _ in range(2)]
    lg_st = [torch.empty_like(lg) for _ in range(2)]
    y_st = [torch.empty_like(y) for _ in range(2)]
    h2d = torch.cuda.Stream(device=dev)
    d2h = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(args.steps)]
    ev_done = [torch.cuda.Event() for _ in range(args.steps)]
    ev_out = [torch.cuda.Event() for _ in range(args.steps)]
    t_first = torch.cuda.Event(enable_timing=True)
    t_last = torch.cuda.Event(enable_timing=True)

    def copy_in(s):
        b = s % 2
        with torch.cuda.stream(h2d):
            if s >= 2:
                h2d.wait_event(ev_done[s - 2])           # chunk s-2 has finished reading buffer b
            x_st[b].copy_(x_pin, non_blocking=True)
            lg_st[b].copy_(lg_pin, non_blocking=True)
            ev_in[s].record(h2d)

    # one CUDA graph of the layer per staging buffer
    g_st = []
    for b in range(2):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(x_st[b], lg_st[b], y_st[b])
        g_st.append(g)
    torch.cuda.synchronize(dev)
    t_first.record(h2d)
    copy_in(0)
    for s in range(args.steps):
        b = s % 2
        if s + 1 < args.steps:
            copy_in(s + 1)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[s])
            if s >= 2:
                stream.wait_event(ev_out[s - 2])         # y_st[b] has been copied out
            g_st[b].replay()
            ev_done[s].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(ev_done[s])
            y_pin[b].copy_(y_st[b], non_blocking=True)
            ev_out[s].record(d2h)
    t_last.record(d2h)
    torch.cuda.synchronize(dev)
    layer.sync_status(stream)
    if not torch.equal(y_pin[(args.steps - 1) % 2], y_st[(args.steps - 1) % 2].cpu()):
        raise RuntimeError("end-to-end prefill: the host copy of y differs from the device result")
    e2e_ms = float(t_first.elapsed_time(t_last))
    e2e_ms_max = allreduce_max(e2e_ms, dev, world)
    del g_st

    fl_gu, fl_dn = prefill_flops(wl, T * k)
    peaks, peak_kind = measured_peaks()
    layer.close()
    roof = gateup_roofline(wl, T * k, experts_touched, kern["grouped_gemm_gate_up_routed"], peaks, peak_kind,
                           tensor_peaks)
    roof["traffic"] = load_traffic("k_fp4_gemm<0>" if wl.quant == "nvfp4" else "k_grouped_gemm<0,false>", wl.name)
    roof["down_routed_tflops"] = 2.0 * T * k * wl.I * H / (kern["grouped_gemm_down_routed"] * 1e-3) / 1e12
    return {
        "total_ms": total_ms_max, "steps_tokens": args.steps * T, "e2e_ms": e2e_ms_max,
        "eager_ms_per_step": eager_ms_max / args.steps,
        "clocks": clocks.summary(), "kernels_ms": kern, "roofline": roof,
        "e2e_method": ("chunks pipelined: inputs copied in and outputs copied out on two copy streams while the "
                       "previous chunk computes (the layer as one CUDA graph per staging buffer); first input copy "
                       "to last output copy"),
        # router GEMM, top-k, 3 permutation, 1 activation pass, 1 launch for
        # both tile lists, 2 routed GEMMs (+2 shared), combine
        "launches_per_step": 10 + (2 if wl.shared else 0), "h2d": T * H * 2 + T * E * 4, "d2h": T * H * 2,
        "layer_tflops": (fl_gu + fl_dn) / (total_ms_max / args.steps * 1e-3) / 1e12,
        "layer": prefill_layer_fractions(wl, experts_touched, total_ms_max / args.steps, peaks,
                                         roof["tensor_peak_tflops"]),
        "dtype": "e2m1" if wl.quant == "nvfp4" else "f16",
    }


def prefill_layer_fractions(wl, experts_touched, ms_per_step, peaks, tensor_peak):
    """The whole step against the roofline (beside the dominant kernel's
    figure): FLOPs of the router GEMM and of the routed and shared expert
    GEMMs over the step time, and the step's algorithmic bytes (the touched
    experts' packed weights, the bf16 router and shared expert, x in and y
    out) over the step time."""
    T, H, I, E, k = wl.T, wl.H, wl.I, wl.E, wl.k
    fl_gu, fl_dn = prefill_flops(wl, T * k)
    flops = fl_gu + fl_dn + 2.0 * T * E * H
    gu_b, dn_b = expert_bytes(wl)
    nbytes = experts_touched * (gu_b + dn_b) + E * H * 2 + (3 * H * I * 2 if wl.shared else 0) + 2 * T * H * 2
    t = ms_per_step * 1e-3
    return {"flops_per_step": flops, "bytes_per_step": float(nbytes), "tflops": flops / t / 1e12,
            "frac_of_tensor_peak": flops / t / 1e12 / tensor_peak, "hbm_gbs": nbytes / t / 1e9,
            "frac_of_hbm": nbytes / t / 1e9 / peaks["hbm_gbs"], "ms_per_step": ms_per_step}


def load_traffic(kernel, workload):
    """Per-launch DRAM bytes of `kernel` from a committed ncu summary, only if
    the kernel source has not changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    import hashlib
    with open(p) as f:
        d = json.load(f)
    ent = d.get(f"{workload}:{kernel}")
    if not ent:
        return None
    src = os.path.join(ROOT, "bit_quantized_mixture_b200", "csrc", ent["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != ent["sha256"]:
        return None
    return ent["dram_bytes_per_launch"]


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def allreduce_max(v, dev, world):
    if world <= 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def bench_line(args, wl, r, world, prefill):
    """The JSON line of a run from the per-rank results r, whose times are
    already the maximum over the ranks: value = all ranks' tokens over that
    time (replicas, weak scaling)."""
    tokens_all = r["steps_tokens"] * world
    value = tokens_all / (r["total_ms"] * 1e-3)
    e2e = tokens_all / (r["e2e_ms"] * 1e-3)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": r["total_ms"] / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": r.get("dtype", "bf16"), "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "k": wl.k, "quant": wl.quant,
                   "shared": wl.shared, "routing": wl.routing, "parallelism": f"replicas x{world}",
                   "l2": f"flushed ({args.flush_mb} MB write) between timed steps",
                   "cuda_graph": True,
                   "experts": "address table, shuffled pool" if args.expert_table else "arena"},
        "roofline": r["roofline"],
        "kernels_ms": r["kernels_ms"],
        "e2e": {"value": e2e, "unit": UNIT, "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "method": r.get("e2e_method", "")},
        "gpu_launches": r["launches_per_step"] * args.steps,
        "clocks": r["clocks"],
    }
    if "layer_gbs" in r:
        line["layer_hbm_gbs"] = r["layer_gbs"]
    if "warm_ms_per_step" in r:      # decode without the L2 flush (a reported variant, not the value)
        line["warm_ms_per_step"] = r["warm_ms_per_step"]
    if "eager_ms_per_step" in r:     # prefill launched eagerly (a reported variant, not the value)
        line["eager_ms_per_step"] = r["eager_ms_per_step"]
    if "layer_tflops" in r:
        line["layer_tflops"] = r["layer_tflops"]
    if "layer" in r:
        line["layer"] = r["layer"]
    return line


def workload_entry(line):
    """A workload measured after the main one: its own value, step time,
    roofline, per-kernel times, end-to-end figure and clocks."""
    keep = ("value", "unit", "ms_per_step", "dtype", "config", "roofline", "layer", "kernels_ms", "e2e",
            "gpu_launches", "clocks", "layer_hbm_gbs", "layer_tflops", "warm_ms_per_step", "eager_ms_per_step")
    return {k: line[k] for k in keep if k in line}


def run_ours(args):
    import torch

    from bit_quantized_mixture_b200 import synth
    rank, local_rank, world = dist_env()
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    tensor_peaks = None if args.no_peak_loop else measure_tensor_peaks(dev)

    def run_workload(name):
        wl = synth.workload(name)
        prefill = wl.routing != "router"
        r = run_prefill(args, wl, dev, rank, world, tensor_peaks) if prefill else run_decode(args, wl, dev, rank, world)
        torch.cuda.empty_cache()
        return wl, bench_line(args, wl, r, world, prefill)

    wl, line = run_workload(args.workload)
    if tensor_peaks:
        line["tensor_peaks_measured"] = tensor_peaks
    extras = [n for n in (args.extra_workloads or "").split(",") if n and n != "none" and n != wl.name]
    if extras:
        line["workloads"] = {n: (run_m_sweep(args, dev, rank, world) if n == "m-sweep" else
                                 workload_entry(run_workload(n)[1])) for n in extras}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, info = oracle_tokens_per_s(wl, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": info["cores"], "kind": "oracle",
                                "sample": info["sample"]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
