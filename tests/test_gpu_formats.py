"""GPU quantization, activation quantization and weight re-layout against the
oracle: every code, scale and zero byte must be identical."""
import numpy as np
import pytest
import torch

from bit_quantized_mixture_b200 import moe, synth
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _weights(N, K, seed):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[0, :128] = 0.0                                         # all-zero group
    w[1, :128] = np.linspace(0.001, 0.3, 128)                # one-sided groups
    w[2, :128] = -np.linspace(0.001, 0.3, 128)
    w[3, 0:9] = [0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 7.0, -7.0, 3.5]   # exact ties (s = 1)
    w[3, 9:128] = 0.0
    w[4, :16] = [6.0, 0.25, 0.75, -1.25, 1.75, 2.5, 3.5, 5.0, -6.0, 0.1, -0.1, 4.5, 0, 0, 0, 0]
    w[5, 200:220] = 1e-30                                    # tiny values
    return w


@pytest.mark.parametrize("quant", ["int4", "int4g32", "int2", "nvfp4", "fp8", "fp6"])
@pytest.mark.parametrize("shape", [(128, 256), (512, 2048), (2048, 512), (132, 384)])
def test_quantize_bit_exact(quant, shape):
    N, K = shape
    if quant == "fp8" and N % 128:
        pytest.skip("FP8 blocks are 128 x 128")
    w = _weights(N, K, seed=N + K)
    g = O.nvfp4_global_scale(np.abs(w).max()) if quant == "nvfp4" else 0.0
    wd = torch.from_numpy(w).to(DEV)
    if quant == "nvfp4":
        amax = torch.zeros(1, dtype=torch.float32, device=DEV)
        moe.absmax(wd, amax)
        assert amax.item() == np.float32(np.abs(w).max())
        assert moe.nvfp4_global_scale(amax.item()) == g
    codes, scales, zeros = moe.quantize(quant, wd, g)
    torch.cuda.synchronize()
    if quant in ("int4", "int4g32"):
        rc, rs = O.quantize_int4(w, group=32 if quant == "int4g32" else 128)
        assert np.array_equal(codes.cpu().numpy(), rc)
        assert np.array_equal(scales.cpu().numpy().view(np.uint16), rs.view(np.uint16))
    elif quant == "int2":
        rc, rs, rz = O.quantize_int2(w)
        assert np.array_equal(codes.cpu().numpy(), rc)
        assert np.array_equal(scales.cpu().numpy().view(np.uint16), rs.view(np.uint16))
        assert np.array_equal(zeros.cpu().numpy(), rz)
    elif quant == "fp6":
        rc, rs = O.quantize_fp6(w)
        assert np.array_equal(codes.cpu().numpy(), rc)
        assert np.array_equal(scales.cpu().numpy().view(np.uint16), rs.view(np.uint16))
    elif quant == "fp8":
        rc, rs = O.quantize_fp8_block(w)
        assert np.array_equal(codes.cpu().numpy(), rc)
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    else:
        rc, rs = O.quantize_nvfp4(w, g)
        assert np.array_equal(scales.cpu().numpy(), rs)
        assert np.array_equal(codes.cpu().numpy(), rc)


def test_quantize_act_nvfp4_bit_exact():
    wl = synth.custom("tiny-int4", T=37, H=512)
    x = synth.activations_bf16(wl)
    xf = O.bf16_bits_to_f32(x)
    g = O.nvfp4_global_scale(np.abs(xf).max())
    xd = torch.from_numpy(x.view(np.int16)).to(DEV)
    codes, scales = moe.quantize_act_nvfp4(xd, g)
    rc, rs = O.quantize_nvfp4(xf, g)
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_e2m1_conversion_around_every_midpoint():
    # a grid of fp32 values around each E2M1 midpoint, both signs, through
    # the activation quantizer with g chosen so that s_b = 1 and r = 1
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    vals = []
    for m in mids:
        for d in (-2, -1, 0, 1, 2):
            vals.append(np.nextafter(m, np.float32(np.inf if d > 0 else -np.inf), dtype=np.float32) if d else m)
            if abs(d) == 2:
                vals[-1] = np.float32(m + d * 1e-3)
    vals = np.array(vals, np.float32)
    n = (len(vals) + 14) // 15 * 15
    pad = np.zeros(n, np.float32)
    pad[:len(vals)] = vals
    blocks = pad.reshape(-1, 15)
    x = np.concatenate([np.full((blocks.shape[0], 1), 6.0, np.float32), blocks], axis=1)   # amax 6 -> s_b = 1
    x = np.concatenate([x, -x], axis=0)
    x = np.pad(x, ((0, 0), (0, 16)))                        # K = 32
    bits = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    xf = bits.float().numpy()
    g = np.float32(1.0)                                      # amax 6 -> s_b = e4m3(1) = 1, r = 1
    codes, scales = moe.quantize_act_nvfp4(bits.view(torch.int16).to(DEV).view(torch.bfloat16), g)
    rc, rs = O.quantize_nvfp4(xf, g)
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)


@pytest.mark.parametrize("quant", ["int4", "int4g32", "int2", "nvfp4", "fp8", "fp6"])
def test_relayout_round_trip(quant):
    from bit_quantized_mixture_b200.layer import quantize_expert_gpu
    wl = synth.custom("tiny-int4", quant=quant, H=384, I=256, E=3, k=2, shared=True)
    layer = moe.MoeLayer(wl.H, wl.I, wl.E, wl.k, quant, True, 4, 0)
    qs = {}
    for e in range(wl.E):
        qs[e] = quantize_expert_gpu(quant, *synth.expert_fp32(wl, e), DEV)
        layer.load_expert(e, qs[e])
    sh = [torch.from_numpy(m.view(np.int16)).to(DEV) for m in synth.shared_bf16(wl)]
    layer.load_expert(moe.SHARED, {n: {"codes": t} for n, t in zip(("gate", "up", "down"), sh)})
    for e in range(wl.E):
        for which, name in enumerate(("gate", "up", "down")):
            ref = qs[e][name]
            codes = torch.empty_like(ref["codes"])
            scales = torch.empty_like(ref["scales"])
            zeros = torch.empty_like(ref["zeros"]) if ref["zeros"] is not None else None
            gs = torch.zeros(1, dtype=torch.float32, device=DEV)
            layer.debug_unpack(e, which, codes, scales, zeros, gs)
            torch.cuda.synchronize()
            assert torch.equal(codes, ref["codes"])
            assert torch.equal(scales.view(torch.uint8), ref["scales"].view(torch.uint8))
            if zeros is not None:
                assert torch.equal(zeros, ref["zeros"])
            if quant == "nvfp4":
                assert gs.item() == np.float32(ref["g"])
    for which in range(3):
        out = torch.empty_like(sh[which])
        layer.debug_unpack(moe.SHARED, which, out)
        torch.cuda.synchronize()
        assert torch.equal(out, sh[which])
    layer.close()
