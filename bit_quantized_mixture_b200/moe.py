"""Python binding of libmoe_b200.so (argument marshalling only).

Every name mirrors an entry point of include/moe_b200.h.  Tensors are torch
CUDA tensors (device memory and streams come from PyTorch); host-side inputs
of the load calls may also be numpy arrays.  There is no fallback: if the
library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_STATE, MOE_ERR_OOM, MOE_ERR_CUDA, MOE_ERR_TIMEOUT = range(7)
QUANT = {"int4": 0, "int2": 1, "nvfp4": 2, "bf16": 3, "int4g32": 4, "fp8": 5, "fp6": 6}
SHARED = -1


class MoeError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"[{status}] {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("hidden", "inter", "num_experts", "top_k", "quant", "has_shared", "max_tokens", "device")]


class QMatrix(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p),
                ("global_scale", ctypes.c_float)]


class ExpertWeights(ctypes.Structure):
    _fields_ = [("gate", QMatrix), ("up", QMatrix), ("down", QMatrix)]


_lib = None


def lib():
    """Load the CUDA library once; raise if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m bit_quantized_mixture_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
        sig = {
            "moe_create": [ctypes.POINTER(Config), ctypes.POINTER(vp)],
            "moe_destroy": [vp],
            "moe_load_router": [vp, vp, vp],
            "moe_load_expert_weights": [vp, i32, ctypes.POINTER(ExpertWeights), vp],
            "moe_set_act_global_scales": [vp, f32, f32],
            "moe_route": [vp, vp, i32, vp, vp, vp, vp],
            "moe_route_from_logits": [vp, vp, i32, vp, vp, vp],
            "moe_forward": [vp, vp, i32, vp, vp, vp, vp],
            "moe_route_forward": [vp, vp, i32, vp, vp, vp, vp],
            "moe_quantize": [i32, vp, i32, i32, f32, vp, vp, vp, vp],
            "moe_absmax": [vp, i64, vp, vp],
            "moe_quantize_act_nvfp4": [vp, i32, i32, f32, vp, vp, vp],
            "moe_permute": [vp, i32, i32, i32, vp, vp, vp, vp, vp],
            "moe_debug_unpack_matrix": [vp, i32, i32, vp, vp, vp, vp, vp],
            "moe_set_profile_events": [vp, ctypes.POINTER(vp), i32],
            "moe_sync_status": [vp, vp],
            "moe_permute_noalloc": [vp, i32, i32, i32, vp, vp, vp, vp, vp],
            "moe_expert_block_bytes": [vp, ctypes.POINTER(ctypes.c_size_t)],
            "moe_set_decode_path": [vp, i32],
            "moe_export_expert": [vp, i32, vp, vp],
            "moe_set_expert_table": [vp, ctypes.POINTER(vp), vp],
            "moe_debug_get_permutation": [vp, vp, vp, vp, vp, vp],
            "moe_debug_get_act_nvfp4": [vp, vp, vp, vp],
            "moe_debug_set_wait_test": [vp, i32, i64],
            "moe_mma_peak_loop": [i32, i32, i64, vp, ctypes.POINTER(ctypes.c_double), vp],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.moe_status_str.argtypes = [ctypes.c_int]
        L.moe_status_str.restype = ctypes.c_char_p
        L.moe_last_error.argtypes = [vp]
        L.moe_last_error.restype = ctypes.c_char_p
        L.moe_nvfp4_global_scale.argtypes = [f32]
        L.moe_nvfp4_global_scale.restype = f32
        _lib = L
    return _lib


def _check(status, handle=None):
    if status != MOE_OK:
        raise MoeError(status, lib().moe_last_error(handle).decode())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    if isinstance(t, np.ndarray):
        assert t.flags["C_CONTIGUOUS"]
        return t.ctypes.data
    raise TypeError(type(t))


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def nvfp4_global_scale(amax: float) -> float:
    return float(lib().moe_nvfp4_global_scale(float(amax)))


class MoeLayer:
    """One MoE layer: owns the weight arena and workspace on one device."""

    def __init__(self, hidden, inter, num_experts, top_k, quant, has_shared, max_tokens, device=0):
        self.cfg = Config(hidden, inter, num_experts, top_k, QUANT[quant], int(bool(has_shared)), max_tokens, device)
        self.quant = quant
        h = ctypes.c_void_p()
        _check(lib().moe_create(ctypes.byref(self.cfg), ctypes.byref(h)))
        self.h = h
        self._keep = []            # host arrays that must outlive asynchronous copies

    def close(self):
        if getattr(self, "h", None):
            lib().moe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def load_router(self, w_bf16, stream=None):
        _check(lib().moe_load_router(self.h, _ptr(w_bf16), _stream(stream)), self.h)

    def load_expert(self, expert, mats, stream=None):
        """mats: {'gate'|'up'|'down': {'codes', 'scales', 'zeros', 'g'}} arrays in
        interchange layout (torch tensors or numpy arrays)."""
        ew = ExpertWeights()
        for name in ("gate", "up", "down"):
            m = mats[name]
            q = getattr(ew, name)
            q.codes = _ptr(m["codes"])
            q.scales = _ptr(m.get("scales"))
            q.zeros = _ptr(m.get("zeros"))
            q.global_scale = float(m.get("g", 0.0))
        _check(lib().moe_load_expert_weights(self.h, int(expert), ctypes.byref(ew), _stream(stream)), self.h)

    def set_act_global_scales(self, g_x, g_a):
        _check(lib().moe_set_act_global_scales(self.h, float(g_x), float(g_a)), self.h)

    def route(self, x, ids, w, logits=None, stream=None):
        _check(lib().moe_route(self.h, _ptr(x), x.shape[0], _ptr(ids), _ptr(w), _ptr(logits), _stream(stream)), self.h)

    def route_from_logits(self, logits, ids, w, stream=None):
        _check(lib().moe_route_from_logits(self.h, _ptr(logits), logits.shape[0], _ptr(ids), _ptr(w),
                                           _stream(stream)), self.h)

    def forward(self, x, ids, w, y, stream=None):
        _check(lib().moe_forward(self.h, _ptr(x), x.shape[0], _ptr(ids), _ptr(w), _ptr(y), _stream(stream)), self.h)

    def sync_status(self, stream=None):
        """Synchronize the stream; raise on a device-side timeout or CUDA error."""
        _check(lib().moe_sync_status(self.h, _stream(stream)), self.h)

    def route_forward(self, x, ids, w, y, stream=None):
        """The whole layer (route + forward) in one call."""
        _check(lib().moe_route_forward(self.h, _ptr(x), x.shape[0], _ptr(ids), _ptr(w), _ptr(y), _stream(stream)),
               self.h)

    def set_profile_events(self, events):
        """events: 5 to 10 torch.cuda.Event(enable_timing=True) (recorded once
        beforehand) or None; slot meanings as in moe_set_profile_events."""
        if events is None:
            _check(lib().moe_set_profile_events(self.h, None, 0), self.h)
            return
        arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
        _check(lib().moe_set_profile_events(self.h, arr, len(events)), self.h)

    def set_decode_path(self, path):
        """'auto' (fused kernel eagerly, three kernels inside a CUDA graph),
        'fused', 'kernels' or 'gemm' (the grouped-GEMM path for every T)."""
        _check(lib().moe_set_decode_path(self.h, {"auto": 0, "fused": 1, "kernels": 2, "gemm": 3}[path]), self.h)

    def expert_block_bytes(self):
        n = ctypes.c_size_t(0)
        _check(lib().moe_expert_block_bytes(self.h, ctypes.byref(n)), self.h)
        return int(n.value)

    def export_expert(self, expert, dst, stream=None):
        """Copy expert `expert`'s block (device layout) to the CUDA buffer dst."""
        _check(lib().moe_export_expert(self.h, int(expert), _ptr(dst), _stream(stream)), self.h)

    def set_expert_table(self, addresses, stream=None):
        """addresses: E device addresses (ints) of expert blocks, or None for the arena."""
        if addresses is None:
            _check(lib().moe_set_expert_table(self.h, None, _stream(stream)), self.h)
            return
        arr = (ctypes.c_void_p * len(addresses))(*[int(a) for a in addresses])
        _check(lib().moe_set_expert_table(self.h, arr, _stream(stream)), self.h)

    def debug_permutation(self, T, stream=None):
        """(counts, offsets, perm, inv) of the last grouped-GEMM forward of T tokens."""
        E, k = self.cfg.num_experts, self.cfg.top_k
        dev = torch.device("cuda", self.cfg.device)
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(T * k, dtype=torch.int32, device=dev)
        inv = torch.empty(T * k, dtype=torch.int32, device=dev)
        _check(lib().moe_debug_get_permutation(self.h, _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv),
                                               _stream(stream)), self.h)
        return counts, offsets, perm, inv

    def debug_act_nvfp4(self, T, stream=None):
        """(codes [T*k, H/2], scales [T*k, H/16]) of the W4A4 operand of the last
        block-scaled NVFP4 grouped-GEMM forward of T tokens, permuted order."""
        slots, H = T * self.cfg.top_k, self.cfg.hidden
        dev = torch.device("cuda", self.cfg.device)
        codes = torch.empty((slots, H // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((slots, H // 16), dtype=torch.uint8, device=dev)
        _check(lib().moe_debug_get_act_nvfp4(self.h, _ptr(codes), _ptr(scales), _stream(stream)), self.h)
        return codes, scales

    def debug_set_wait_test(self, withhold_cta, wait_limit_cycles=0):
        """One-shot test hook: the next fused decode launch has CTA
        withhold_cta skip a grid-barrier arrival, and its waits give up after
        wait_limit_cycles (0: the default limit)."""
        _check(lib().moe_debug_set_wait_test(self.h, int(withhold_cta), int(wait_limit_cycles)), self.h)

    def debug_unpack(self, expert, which, codes, scales=None, zeros=None, global_scale=None, stream=None):
        _check(lib().moe_debug_unpack_matrix(self.h, int(expert), int(which), _ptr(codes), _ptr(scales),
                                             _ptr(zeros), _ptr(global_scale), _stream(stream)), self.h)


def quantize(quant, w, global_scale=0.0, stream=None):
    """w: CUDA fp32 [N, K] -> (codes, scales, zeros) CUDA uint8/fp16 tensors."""
    N, K = w.shape
    dev = w.device
    q = QUANT[quant]
    zeros = None
    if quant in ("int4", "int4g32"):
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((N, K // (32 if quant == "int4g32" else 128)), dtype=torch.float16, device=dev)
    elif quant == "fp6":
        codes = torch.empty((N, K), dtype=torch.uint8, device=dev)
        scales = torch.empty((N, K // 32), dtype=torch.float16, device=dev)
    elif quant == "fp8":
        codes = torch.empty((N, K), dtype=torch.uint8, device=dev)
        scales = torch.empty((N // 128, K // 128), dtype=torch.float32, device=dev)
    elif quant == "int2":
        codes = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
        scales = torch.empty((N, K // 128), dtype=torch.float16, device=dev)
        zeros = torch.empty((N // 4, K // 128), dtype=torch.uint8, device=dev)
    else:
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((N, K // 16), dtype=torch.uint8, device=dev)
    _check(lib().moe_quantize(q, _ptr(w), N, K, float(global_scale), _ptr(codes), _ptr(scales), _ptr(zeros),
                              _stream(stream)))
    return codes, scales, zeros


def absmax(x, out, stream=None):
    _check(lib().moe_absmax(_ptr(x), x.numel(), _ptr(out), _stream(stream)))


def quantize_act_nvfp4(x, g, stream=None):
    T, K = x.shape
    codes = torch.empty((T, K // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((T, K // 16), dtype=torch.uint8, device=x.device)
    _check(lib().moe_quantize_act_nvfp4(_ptr(x), T, K, float(g), _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def permute(ids, num_experts, stream=None):
    T, k = ids.shape
    dev = ids.device
    counts = torch.empty(num_experts, dtype=torch.int32, device=dev)
    offsets = torch.empty(num_experts + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T * k, dtype=torch.int32, device=dev)
    _check(lib().moe_permute(_ptr(ids), T, k, num_experts, _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv),
                             _stream(stream)))
    return counts, offsets, perm, inv


def permute_noalloc(ids, num_experts, stream=None):
    """moe_permute without device allocation (scratch in a static device array)."""
    T, k = ids.shape
    dev = ids.device
    counts = torch.empty(num_experts, dtype=torch.int32, device=dev)
    offsets = torch.empty(num_experts + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T * k, dtype=torch.int32, device=dev)
    _check(lib().moe_permute_noalloc(_ptr(ids), T, k, num_experts, _ptr(counts), _ptr(offsets), _ptr(perm),
                                     _ptr(inv), _stream(stream)))
    return counts, offsets, perm, inv


def mma_peak_loop(kind, issuers, iters, err, stream=None):
    """Launch the tensor-core throughput loop (kind 0: bf16 kind::f16, 1: e2m1
    block-scaled) on every SM; returns the FLOPs of the launch.  err: a
    zeroed int32 CUDA tensor that receives a code if a wait gave up."""
    flops = ctypes.c_double(0.0)
    _check(lib().moe_mma_peak_loop(int(kind), int(issuers), int(iters), _ptr(err), ctypes.byref(flops),
                                   _stream(stream)))
    return flops.value
