"""Seeded synthetic inputs for the MoE-layer workloads.

This module only draws numbers: fp32 expert weights N(0, 0.02), bf16
activations N(0, 1), a bf16 router matrix N(0, 0.02) and, for the prefill
workloads, fp32 routing logits with a prescribed skew.  It holds none of the
layer's arithmetic (no quantization, routing or expert math), so both the
CPU oracle's tests and the CUDA path take their inputs from here.

Every tensor has its own numpy PCG64 stream keyed by
(seed, workload index, tensor tag, expert), so any expert can be regenerated
on its own and experts can be drawn in parallel threads.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace

import numpy as np
import torch

# tensor tags of the seeded streams
TAG_X, TAG_ROUTER, TAG_GATE, TAG_UP, TAG_DOWN, TAG_LOGITS, TAG_PERM = 1, 2, 3, 4, 5, 6, 7
SHARED = -1          # expert index of the always-on shared expert


@dataclass(frozen=True)
class Workload:
    index: int          # position in the list below (part of the seed)
    name: str
    T: int              # tokens per step
    H: int              # hidden size
    I: int              # expert intermediate size
    E: int              # routed experts
    k: int              # experts per token
    quant: str          # 'int4' | 'int2' | 'nvfp4'
    shared: bool        # one always-on bf16 shared expert (I columns)
    routing: str        # 'router' (x Wr^T) | 'zipf' | 'uniform' (synthetic logits)
    steps: int = 1      # distinct seeded token batches (decode: one per step)
    seed: int = 0

    @property
    def slots(self) -> int:
        return self.T * self.k


WORKLOADS = [
    Workload(0, "tiny-int4", T=4, H=256, I=128, E=8, k=2, quant="int4", shared=False, routing="router"),
    Workload(1, "decode-b1-int4", T=1, H=2048, I=512, E=512, k=10, quant="int4", shared=True,
             routing="router", steps=100),
    Workload(2, "decode-b4-int2", T=4, H=2048, I=512, E=512, k=10, quant="int2", shared=True,
             routing="router", steps=100),
    Workload(3, "prefill-int4-zipf", T=4096, H=2048, I=512, E=512, k=10, quant="int4", shared=False,
             routing="zipf"),
    Workload(4, "prefill-nvfp4", T=8192, H=2048, I=512, E=512, k=10, quant="nvfp4", shared=True,
             routing="uniform"),
    # the INT4 group-32 format of the MTP-draft experts on the decode-b1 and
    # prefill-Zipf shapes
    Workload(5, "decode-b1-int4g32", T=1, H=2048, I=512, E=512, k=10, quant="int4g32", shared=True,
             routing="router", steps=100),
    Workload(6, "prefill-int4g32-zipf", T=4096, H=2048, I=512, E=512, k=10, quant="int4g32", shared=False,
             routing="zipf"),
    # FP8 experts with 128x128 block scales (the MTP-draft format of the NVFP4
    # card) on the same shapes
    Workload(7, "decode-b1-fp8", T=1, H=2048, I=512, E=512, k=10, quant="fp8", shared=True,
             routing="router", steps=100),
    Workload(8, "prefill-fp8-zipf", T=4096, H=2048, I=512, E=512, k=10, quant="fp8", shared=False,
             routing="zipf"),
    # FP6 e2m3 experts with fp16 scales per 32 inputs (the FP6 card) on the
    # same shapes
    Workload(9, "decode-b1-fp6", T=1, H=2048, I=512, E=512, k=10, quant="fp6", shared=True,
             routing="router", steps=100),
    Workload(10, "prefill-fp6-zipf", T=4096, H=2048, I=512, E=512, k=10, quant="fp6", shared=False,
             routing="zipf"),
]
ZIPF_S = 1.1


def workload(key) -> Workload:
    if isinstance(key, Workload):
        return key
    if isinstance(key, int):
        return WORKLOADS[key]
    for w in WORKLOADS:
        if w.name == key:
            return w
    raise KeyError(key)


def custom(base, **kw) -> Workload:
    """A workload with changed shapes (parity cases at reduced sizes)."""
    return replace(workload(base), **kw)


def _rng(wl: Workload, tag: int, idx: int = 0) -> np.random.Generator:
    seq = np.random.SeedSequence([wl.seed, wl.index, tag, idx + 1])
    return np.random.Generator(np.random.PCG64(seq))


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round fp32 draws to bf16 (round-to-nearest-even) -> uint16 bits."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def expert_fp32(wl: Workload, e: int):
    """fp32 weights of routed expert e: gate [I,H], up [I,H], down [H,I]."""
    wl = workload(wl)
    out = []
    for tag, shape in ((TAG_GATE, (wl.I, wl.H)), (TAG_UP, (wl.I, wl.H)), (TAG_DOWN, (wl.H, wl.I))):
        g = _rng(wl, tag, e)
        out.append(g.standard_normal(shape, dtype=np.float32) * np.float32(0.02))
    return tuple(out)


def experts_fp32_iter(wl: Workload, experts, threads: int = 8):
    """Yield (e, gate, up, down) for the given experts, drawn in threads."""
    wl = workload(wl)
    experts = list(experts)
    with ThreadPoolExecutor(max(1, threads)) as ex:
        for e, ws in zip(experts, ex.map(lambda e: expert_fp32(wl, e), experts)):
            yield (e,) + ws


def shared_bf16(wl: Workload):
    """bf16 bit patterns of the shared expert: gate [I,H], up [I,H], down [H,I]."""
    return tuple(f32_to_bf16_bits(m) for m in expert_fp32(wl, SHARED))


def router_bf16(wl: Workload) -> np.ndarray:
    """bf16 bit patterns of the router matrix [E, H], N(0, 0.02)."""
    wl = workload(wl)
    g = _rng(wl, TAG_ROUTER)
    return f32_to_bf16_bits(g.standard_normal((wl.E, wl.H), dtype=np.float32) * np.float32(0.02))


def activations_bf16(wl: Workload, steps: int | None = None) -> np.ndarray:
    """bf16 bit patterns of x, [steps*T, H], N(0, 1); step i uses rows
    [i*T, (i+1)*T)."""
    wl = workload(wl)
    n = (wl.steps if steps is None else steps) * wl.T
    g = _rng(wl, TAG_X)
    return f32_to_bf16_bits(g.standard_normal((n, wl.H), dtype=np.float32))


def routing_logits(wl: Workload) -> np.ndarray | None:
    """Synthetic fp32 routing logits [T, E] for the prefill workloads.

    'zipf'   : log p_e + Gumbel noise, p over a seeded permutation of the
               experts proportional to rank^-1.1; the top-k of these logits
               is a draw of k experts without replacement with probabilities
               p, so per-expert token counts follow the Zipf law.
    'uniform': i.i.d. N(0, 1), i.e. uniformly random expert sets.
    'router' : None (logits come from the router matrix)."""
    wl = workload(wl)
    if wl.routing == "router":
        return None
    g = _rng(wl, TAG_LOGITS)
    if wl.routing == "uniform":
        return g.standard_normal((wl.T, wl.E), dtype=np.float32)
    perm = _rng(wl, TAG_PERM).permutation(wl.E)
    pmf = np.arange(1, wl.E + 1, dtype=np.float64) ** -ZIPF_S
    p = np.empty(wl.E)
    p[perm] = pmf / pmf.sum()
    u = g.random((wl.T, wl.E))
    gumbel = -np.log(-np.log(np.clip(u, 1e-300, 1.0 - 1e-16)))
    return (np.log(p)[None, :] + gumbel).astype(np.float32)
