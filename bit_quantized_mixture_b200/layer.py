"""Set-up helpers: build a MoeLayer on the GPU from a synthetic workload.

The fp32 weights come from the seeded input generator; quantization, the
NVFP4 global scales and the re-layout all run in the CUDA library.
"""
from __future__ import annotations

import numpy as np
import torch

from . import moe, synth


def quantize_expert_gpu(quant, gate, up, down, device):
    """fp32 host (numpy) matrices -> interchange tensors on the device."""
    out = {}
    mats = {"gate": gate, "up": up, "down": down}
    dev = {k: torch.from_numpy(np.ascontiguousarray(v)).to(device, non_blocking=False) for k, v in mats.items()}
    if quant == "nvfp4":
        amax = torch.zeros(2, dtype=torch.float32, device=device)
        moe.absmax(dev["gate"], amax[0:1])
        moe.absmax(dev["up"], amax[0:1])
        moe.absmax(dev["down"], amax[1:2])
        a = amax.cpu().numpy()
        g_gu, g_d = moe.nvfp4_global_scale(a[0]), moe.nvfp4_global_scale(a[1])
    for name, w in dev.items():
        g = 0.0
        if quant == "nvfp4":
            g = g_d if name == "down" else g_gu
        codes, scales, zeros = moe.quantize(quant, w, g)
        out[name] = {"codes": codes, "scales": scales, "zeros": zeros, "g": g}
    return out


def build_layer(wl, device=0, max_tokens=None, threads=8, keep_interchange=False):
    """Create and fully load the layer of workload `wl` on `device`.

    Returns (layer, extras) where extras may hold the interchange tensors of
    every expert when keep_interchange is set (for parity checks)."""
    wl = synth.workload(wl)
    dev = torch.device("cuda", device)
    layer = moe.MoeLayer(wl.H, wl.I, wl.E, wl.k, wl.quant, wl.shared, max_tokens or wl.T, device)
    layer.load_router(torch.from_numpy(synth.router_bf16(wl).view(np.int16)).to(dev))
    kept = {}
    for e, g, u, d in synth.experts_fp32_iter(wl, range(wl.E), threads=threads):
        q = quantize_expert_gpu(wl.quant, g, u, d, dev)
        layer.load_expert(e, q)
        if keep_interchange:
            kept[e] = q
    if wl.shared:
        sh = synth.shared_bf16(wl)
        shd = {n: {"codes": torch.from_numpy(m.view(np.int16)).to(dev)} for n, m in zip(("gate", "up", "down"), sh)}
        layer.load_expert(moe.SHARED, shd)
    torch.cuda.synchronize(dev)
    return layer, kept
