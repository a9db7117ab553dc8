"""The W4A4 activation operand of the block-scaled NVFP4 prefill path, read
back from the layer's workspace after a forward: the permutation and every
permuted row's E2M1 codes and E4M3 scales equal the oracle's NVFP4 quantizer
("meshapplied/Qwen3.8-Flash-Next-NVFP4-Latest", section "Format") byte for
byte, at the full prefill size, with dropped slots, and on blocks whose scale
decodes to zero (all-zero, negative-zero and underflowing rows)."""
import numpy as np
import pytest
import torch

from bit_quantized_mixture_b200 import moe, synth
from bit_quantized_mixture_b200.layer import build_layer
from oracle import moe_oracle as O
from tests.gpu_util import bf16_tensor

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _check_operand(layer, x_bits, ids, w, g_x, E, k):
    T, H = x_bits.shape
    y = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)
    layer.forward(bf16_tensor(x_bits, DEV), torch.from_numpy(ids).to(DEV),
                  torch.from_numpy(w.astype(np.float32)).to(DEV), y)
    layer.sync_status()
    counts, offsets, perm, inv = (t.cpu().numpy() for t in layer.debug_permutation(T))
    rc, ro, rp, ri = O.permute(ids, E)
    n = int(ro[-1])
    assert np.array_equal(counts, rc) and np.array_equal(offsets, ro)
    assert np.array_equal(perm[:n], rp[:n]) and np.array_equal(inv, ri)
    codes, scales = (t.cpu().numpy() for t in layer.debug_act_nvfp4(T))
    ref_codes, ref_scales = O.quantize_nvfp4(O.bf16_bits_to_f32(x_bits), g_x)
    tok = rp[:n] // k
    bad = np.nonzero(np.any(codes[:n] != ref_codes[tok], axis=1) | np.any(scales[:n] != ref_scales[tok], axis=1))[0]
    assert bad.size == 0, f"{bad.size} of {n} permuted rows differ, first at position {bad[:5]}"
    return n


def test_nvfp4_operand_full_size_bit_exact():
    """prefill-nvfp4 (T = 8192, H = 2048, E = 512, k = 10, uniform routing):
    all 81,920 permuted rows."""
    wl = synth.workload("prefill-nvfp4")
    layer, _ = build_layer(wl, 0, max_tokens=wl.T)
    x = synth.activations_bf16(wl)
    ids, w = O.route_topk(synth.routing_logits(wl), wl.k)
    g_x = O.nvfp4_global_scale(np.abs(O.bf16_bits_to_f32(x)).max())
    layer.set_act_global_scales(g_x, O.nvfp4_global_scale(8.0))
    assert _check_operand(layer, x, ids, w, g_x, wl.E, wl.k) == wl.T * wl.k
    layer.close()


def test_nvfp4_operand_dropped_slots_and_zero_scales():
    """Slots with ids outside [0, E) take no position; rows of +0, of -0 and
    of values so small that their block scale rounds to zero give scale 0
    and signed-zero codes, as the oracle's quantizer does."""
    wl = synth.custom("tiny-int4", quant="nvfp4", H=512, I=256, E=24, k=6, shared=True, T=300)
    layer, _ = build_layer(wl, 0, max_tokens=wl.T)
    x = synth.activations_bf16(wl, steps=1)[:wl.T].copy()
    x[0] = 0x0000                                            # +0
    x[1] = 0x8000                                            # -0
    x[2] = O_bits(-1e-30)                                     # underflows the block scale
    x[3, :16] = O_bits(3e-29)                                 # one tiny block, the rest normal
    rng = np.random.default_rng(5)
    ids = np.stack([rng.choice(wl.E, wl.k, replace=False) for _ in range(wl.T)]).astype(np.int32)
    flat = ids.reshape(-1)
    drop = rng.choice(flat.size, 40, replace=False)
    flat[drop[:20]] = -1
    flat[drop[20:]] = wl.E + 3
    w = np.full(ids.shape, 1.0 / wl.k)
    g_x = O.nvfp4_global_scale(np.abs(O.bf16_bits_to_f32(x)).max())
    layer.set_act_global_scales(g_x, O.nvfp4_global_scale(8.0))
    n = _check_operand(layer, x, ids, w, g_x, wl.E, wl.k)
    assert n == wl.T * wl.k - 40
    layer.close()


def O_bits(v):
    """bf16 bit pattern of the fp32 value v (round to nearest even)."""
    return synth.f32_to_bf16_bits(np.array([v], np.float32))[0]


def test_nvfp4_quantizer_zero_global_scale():
    """g = 0 (standalone activation quantizer; the layer requires g > 0):
    scale codes and element codes are all zero, as in the oracle."""
    wl = synth.custom("tiny-int4", quant="nvfp4", H=512, T=64)
    x = synth.activations_bf16(wl, steps=1)[:64]
    codes, scales = moe.quantize_act_nvfp4(bf16_tensor(x, DEV), 0.0)
    torch.cuda.synchronize()
    rc, rs = O.quantize_nvfp4(O.bf16_bits_to_f32(x), 0.0)
    assert np.array_equal(codes.cpu().numpy(), rc) and np.array_equal(scales.cpu().numpy(), rs)
    assert not rc.any() and not rs.any()
