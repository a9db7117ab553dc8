"""Shared helpers of the GPU parity tests: oracle-side quantization of a
synthetic workload, comparison metrics and the tolerance of the layer output."""
import numpy as np
import torch

from bit_quantized_mixture_b200 import synth
from oracle import moe_oracle as O

# Output tolerance of the bf16 layer output against the fp64 oracle:
# relative RMS error <= 1e-2 and max-abs error <= 3e-2 * RMS(oracle).
REL_RMS_TOL = 1e-2
MAX_ABS_TOL = 3e-2


def oracle_quantize_expert(quant, gate, up, down):
    ew = {}
    if quant == "nvfp4":
        g_gu = O.nvfp4_global_scale(max(np.abs(gate).max(), np.abs(up).max()))
        g_d = O.nvfp4_global_scale(np.abs(down).max())
    for name, m in (("gate", gate), ("up", up), ("down", down)):
        if quant == "int4":
            c, s = O.quantize_int4(m)
            ew[name] = {"codes": c, "scales": s}
        elif quant == "fp6":
            c, s = O.quantize_fp6(m)
            ew[name] = {"codes": c, "scales": s}
        elif quant == "fp8":
            c, s = O.quantize_fp8_block(m)
            ew[name] = {"codes": c, "scales": s}
        elif quant == "int4g32":
            c, s = O.quantize_int4(m, group=O.GROUP_INT4_G32)
            ew[name] = {"codes": c, "scales": s}
        elif quant == "int2":
            c, s, z = O.quantize_int2(m)
            ew[name] = {"codes": c, "scales": s, "zeros": z}
        else:
            g = g_d if name == "down" else g_gu
            c, s = O.quantize_nvfp4(m, g)
            ew[name] = {"codes": c, "scales": s, "g": g}
    return ew


class OracleExperts:
    """Lazily quantizes (oracle) and dequantizes the experts of a workload."""

    def __init__(self, wl):
        self.wl = synth.workload(wl)
        self.q = {}
        self.deq = {}

    def quantized(self, e):
        if e not in self.q:
            self.q[e] = oracle_quantize_expert(self.wl.quant, *synth.expert_fp32(self.wl, e))
        return self.q[e]

    def __call__(self, e):
        if e not in self.deq:
            self.deq[e] = O.dequantize_expert(self.wl.quant, self.quantized(e))
        return self.deq[e]

    def shared(self):
        if not self.wl.shared:
            return None
        return tuple(O.bf16_bits_to_f64(m) for m in synth.shared_bf16(self.wl))


def bf16_tensor(bits, device):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def to_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def assert_close_output(y_gpu_bits, y_ref):
    y = O.bf16_bits_to_f64(y_gpu_bits)
    rms = np.sqrt(np.mean(y_ref ** 2))
    rel = np.sqrt(np.mean((y - y_ref) ** 2)) / rms
    mx = np.abs(y - y_ref).max() / rms
    assert np.all(np.isfinite(y))
    assert rel <= REL_RMS_TOL and mx <= MAX_ABS_TOL, f"rel-RMS {rel:.3e}, max-abs/RMS {mx:.3e}"
    return rel, mx
