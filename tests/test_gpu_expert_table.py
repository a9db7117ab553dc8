"""Per-expert address table: with the experts' blocks in a separate pool, in
shuffled order, the layer reads them there.  The arena is then overwritten
with other experts' weights, so an output that still matches proves that the
table, not the arena, was read."""
import numpy as np
import pytest
import torch

from bit_quantized_mixture_b200 import moe, synth
from bit_quantized_mixture_b200.layer import build_layer
from oracle import moe_oracle as O

from gpu_util import OracleExperts, assert_close_output, bf16_tensor, to_bits

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)

WL = {
    "int4": synth.custom("tiny-int4", H=512, I=256, E=24, k=6, shared=True),
    "int2": synth.custom("tiny-int4", quant="int2", H=512, I=256, E=24, k=6, shared=True),
    "nvfp4": synth.custom("tiny-int4", quant="nvfp4", H=512, I=256, E=24, k=6, shared=True),
}


def _inputs(wl, T, ox):
    x = synth.activations_bf16(wl, steps=max(1, (T + wl.T - 1) // wl.T))[:T]
    ids, w = O.route_topk(O.router_logits(x, synth.router_bf16(wl)), wl.k)
    act = None
    if wl.quant == "nvfp4":
        g_x = O.nvfp4_global_scale(np.abs(O.bf16_bits_to_f32(x)).max())
        g_a = O.nvfp4_global_scale(O.intermediate_amax(x, ids, "nvfp4", ox, g_x))
        act = (g_x, g_a)
    return x, ids, w, act


def _forward(layer, x, ids, w, H):
    y = torch.empty((x.shape[0], H), dtype=torch.bfloat16, device=DEV)
    layer.forward(bf16_tensor(x, DEV), torch.from_numpy(ids).to(DEV), torch.from_numpy(w.astype(np.float32)).to(DEV), y)
    layer.sync_status()
    return to_bits(y)


@pytest.mark.parametrize("quant,T", [("int4", 1), ("int4", 4), ("int2", 4), ("int4", 37), ("int2", 300),
                                     ("nvfp4", 2), ("nvfp4", 37)])
def test_layer_reads_experts_through_the_table(quant, T):
    wl = WL[quant]
    ox = OracleExperts(wl)
    layer, kept = build_layer(wl, 0, max_tokens=max(T, 4), keep_interchange=True)
    x, ids, w, act = _inputs(wl, T, ox)
    if act:
        layer.set_act_global_scales(*act)
    y_arena = _forward(layer, x, ids, w, wl.H)

    # a pool of expert blocks in shuffled order, 256-byte aligned
    bb = layer.expert_block_bytes()
    assert bb % 256 == 0
    pool = torch.zeros(wl.E * bb + 256, dtype=torch.uint8, device=DEV)
    base = (pool.data_ptr() + 255) // 256 * 256
    slot = np.random.default_rng(5).permutation(wl.E)
    for e in range(wl.E):
        off = base - pool.data_ptr() + int(slot[e]) * bb
        layer.export_expert(e, pool[off:off + bb])
    torch.cuda.synchronize()
    layer.set_expert_table([base + int(slot[e]) * bb for e in range(wl.E)])
    # the arena now holds other experts' weights (expert e <- expert e+1)
    for e in range(wl.E):
        layer.load_expert(e, kept[(e + 1) % wl.E])
    torch.cuda.synchronize()

    y_table = _forward(layer, x, ids, w, wl.H)
    if quant == "nvfp4" and T > 8:
        # prefill with a table takes the exact bf16 dequantization path
        y_ref = O.moe_forward(x, ids, w, quant, ox, shared=ox.shared(), act_scales=act)
        assert_close_output(y_table, y_ref)
        assert_close_output(y_arena, y_ref)
    else:
        assert np.array_equal(y_table, y_arena)

    # back on the arena, which now holds the rotated experts: a different layer
    layer.set_expert_table(None)
    y_rot = _forward(layer, x, ids, w, wl.H)
    assert not np.array_equal(y_rot, y_arena)
    layer.close()


def test_table_entries_are_validated():
    wl = WL["int4"]
    layer, _ = build_layer(wl, 0, max_tokens=4)
    bb = layer.expert_block_bytes()
    buf = torch.zeros(wl.E * bb + 512, dtype=torch.uint8, device=DEV)
    base = (buf.data_ptr() + 255) // 256 * 256
    with pytest.raises(moe.MoeError):
        layer.set_expert_table([base + 16] + [base] * (wl.E - 1))      # misaligned
    with pytest.raises(moe.MoeError):
        layer.set_expert_table([0] * wl.E)                              # null
    with pytest.raises(moe.MoeError):
        layer.export_expert(wl.E, buf)                                  # out of range
    layer.close()
