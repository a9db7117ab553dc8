"""Shared helpers of the GPU parity tests: oracle-side quantization of a
synthetic workload, comparison metrics and the tolerance of the layer output."""
import numpy as np
import torch

from bit_quantized_mixture_b200 import synth
from oracle import moe_oracle as O

# Output tolerance of the bf16 layer output against the fp64 oracle:
# relative RMS error <= 1e-2 and max-abs error <= 3e-2 * RMS(oracle).  The
# max-abs bound applies to the error beyond the bf16 output's own rounding:
# half a bf16 ulp is 2^-8 of an output's binade, i.e. up to 3.5 % of the RMS
# for an output of 9 x RMS, so even the exact result rounded to bf16 can miss
# a raw 3e-2 x RMS bound (it does on the INT4 group-32 Zipf workload: 3.03e-2
# at an output of 8.43 x RMS).  The rel-RMS bound applies to the raw error.
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


def bf16_rounding_error(y_ref):
    """|bf16(y) - y| of the exact values: the error the bf16 output format
    forces on any implementation (round to nearest even, one rounding)."""
    yb = torch.from_numpy(np.ascontiguousarray(y_ref, dtype=np.float64)).to(torch.bfloat16).double().numpy()
    return np.abs(yb - y_ref)


def assert_close_output(y_gpu_bits, y_ref):
    y = O.bf16_bits_to_f64(y_gpu_bits)
    rms = np.sqrt(np.mean(y_ref ** 2))
    err = np.abs(y - y_ref)
    rel = np.sqrt(np.mean(err ** 2)) / rms
    mx = np.maximum(err - bf16_rounding_error(y_ref), 0.0).max() / rms
    assert np.all(np.isfinite(y))
    assert rel <= REL_RMS_TOL and mx <= MAX_ABS_TOL, \
        f"rel-RMS {rel:.3e}, max-abs beyond the bf16 rounding / RMS {mx:.3e} (raw {err.max() / rms:.3e})"
    return rel, mx


class StreamingExperts:
    """Oracle experts for whole-layer checks at full size: experts are
    quantized (oracle) and dequantized by a thread pool a bounded number of
    experts ahead of the order in which the oracle asks for them (ascending
    expert id, as moe_forward and intermediate_amax walk np.unique), and a
    dequantized expert is dropped once handed out, so memory stays bounded.
    With keep_quantized the compact quantized experts are kept for a second
    pass (the NVFP4 calibration pass, then the forward)."""

    def __init__(self, wl, threads=None, ahead=24, keep_quantized=False):
        import os
        from concurrent.futures import ThreadPoolExecutor
        self.wl = synth.workload(wl)
        self.pool = ThreadPoolExecutor(max(2, threads or (os.cpu_count() or 4)))
        self.ahead = ahead
        self.keep = keep_quantized
        self.q = {}
        self.pending = {}
        self.order = []
        self.pos = 0

    def _job(self, e):
        ew = self.q.get(e)
        if ew is None:
            ew = oracle_quantize_expert(self.wl.quant, *synth.expert_fp32(self.wl, e))
            if self.keep:
                self.q[e] = ew
        return O.dequantize_expert(self.wl.quant, ew)

    def start(self, experts):
        """The experts of the next pass, in the order they will be asked for."""
        self.order = [int(e) for e in experts]
        self.pos = 0
        self.pending = {}
        self._fill()

    def _fill(self):
        while len(self.pending) < self.ahead and self.pos < len(self.order):
            e = self.order[self.pos]
            self.pending[e] = self.pool.submit(self._job, e)
            self.pos += 1

    def __call__(self, e):
        fut = self.pending.pop(int(e), None)
        res = fut.result() if fut is not None else self._job(int(e))
        self._fill()
        return res

    def shared(self):
        if not self.wl.shared:
            return None
        return tuple(O.bf16_bits_to_f64(m) for m in synth.shared_bf16(self.wl))

    def close(self):
        self.pool.shutdown(wait=True)


def valid_experts(ids, E):
    u = np.unique(np.asarray(ids))
    return u[(u >= 0) & (u < E)]
