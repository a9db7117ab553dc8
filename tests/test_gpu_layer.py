"""GPU routing, permutation and layer output against the oracle, through the
C ABI: ids / permutation bit-exact, weights and outputs within tolerance."""
import numpy as np
import pytest
import torch

from bit_quantized_mixture_b200 import moe, synth
from bit_quantized_mixture_b200.layer import build_layer
from oracle import moe_oracle as O
from tests.gpu_util import OracleExperts, StreamingExperts, assert_close_output, bf16_tensor, to_bits, valid_experts

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)

_layers = {}


def get_layer(wl, max_tokens):
    key = (wl, max_tokens)
    if key not in _layers:
        _layers[key] = build_layer(wl, 0, max_tokens=max_tokens)[0]
    return _layers[key]


def _route_gpu(layer, x_bits, wl):
    T = x_bits.shape[0]
    ids = torch.empty((T, wl.k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, wl.k), dtype=torch.float32, device=DEV)
    logits = torch.empty((T, wl.E), dtype=torch.float32, device=DEV)
    layer.route(bf16_tensor(x_bits, DEV), ids, w, logits)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy(), logits.cpu().numpy()


# ------------------------------------------------------------------ route
@pytest.mark.parametrize("T", [1, 3, 4, 16, 17, 100, 300, 4096, 8192])
def test_route_matches_oracle(T):
    wl = synth.custom("decode-b1-int4", T=T, E=512, k=10)
    layer = moe.MoeLayer(wl.H, wl.I, wl.E, wl.k, "int4", False, max(T, 1), 0)
    wr = synth.router_bf16(wl)
    layer.load_router(bf16_tensor(wr, DEV))
    x = synth.activations_bf16(wl, steps=1)
    ids, w, logits = _route_gpu(layer, x, wl)
    ref_logits = O.router_logits(x, wr)
    # (ii) logits agree up to fp32 summation order
    assert np.abs(logits - ref_logits).max() <= 1e-4
    # (i) the oracle's top-k rule applied to the GPU's own logits: bit-exact ids
    rid, rw = O.route_topk(logits, wl.k)
    assert np.array_equal(ids, rid)
    assert np.allclose(w, rw, rtol=2e-6, atol=1e-7)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-5)
    # (iii) against the oracle's own logits, ids may differ only at near-ties
    oid, _ = O.route_topk(ref_logits, wl.k)
    srt = -np.sort(-ref_logits, axis=1)
    gap = srt[:, wl.k - 1] - srt[:, wl.k]
    differ = np.any(oid != ids, axis=1)
    assert np.all(gap[differ] < 1e-4)
    layer.close()


@pytest.mark.parametrize("T", [3, 300])
def test_route_logits_only(T):
    """moe_route with no ids / weights computes the same logits and nothing else."""
    wl = synth.custom("decode-b1-int4", T=T, E=512, k=10)
    layer = moe.MoeLayer(wl.H, wl.I, wl.E, wl.k, "int4", False, T, 0)
    layer.load_router(bf16_tensor(synth.router_bf16(wl), DEV))
    x = synth.activations_bf16(wl, steps=1)
    ids, w, logits = _route_gpu(layer, x, wl)
    xd = bf16_tensor(x, DEV)
    lg2 = torch.full((T, wl.E), float("nan"), dtype=torch.float32, device=DEV)
    layer.route(xd, None, None, logits=lg2)
    layer.sync_status()
    assert np.array_equal(lg2.cpu().numpy().view(np.uint32), logits.view(np.uint32))
    layer.close()


def test_route_from_logits_ties_and_order():
    wl = synth.custom("tiny-int4", T=64, E=40, k=7)
    layer = moe.MoeLayer(wl.H, wl.I, wl.E, wl.k, "int4", False, wl.T, 0)
    rng = np.random.default_rng(11)
    L = rng.integers(-4, 5, size=(wl.T, wl.E)).astype(np.float32)     # many exact ties
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device=DEV)
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device=DEV)
    layer.route_from_logits(torch.from_numpy(L).to(DEV), ids, w)
    torch.cuda.synchronize()
    rid, rw = O.route_topk(L, wl.k)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert np.allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=1e-7)
    layer.close()


# the threshold selection (candidates ranked in a shared list) and its
# fallback to selection rounds (more than 32 candidates): continuous logits,
# coarse grids with ties at the threshold, all logits equal, the smallest and
# largest E and k, and E = 1024 (32 logits per lane)
@pytest.mark.parametrize("E,k,kind", [(512, 10, "normal"), (512, 10, "grid"), (512, 10, "fine"), (512, 10, "equal"),
                                      (512, 1, "normal"),
                                      (1024, 10, "normal"), (1024, 32, "grid"), (32, 32, "normal"), (7, 3, "grid"),
                                      (600, 10, "normal")])
def test_route_from_logits_selection_paths(E, k, kind):
    T = 333
    wl = synth.custom("tiny-int4", T=T, E=E, k=k)
    layer = moe.MoeLayer(wl.H, wl.I, wl.E, wl.k, "int4", False, T, 0)
    rng = np.random.default_rng(E * 37 + k)
    if kind == "normal":
        L = rng.standard_normal((T, E)).astype(np.float32)
    elif kind == "grid":
        L = rng.integers(-6, 7, size=(T, E)).astype(np.float32) * np.float32(0.25)
    elif kind == "fine":
        L = rng.integers(-100, 101, size=(T, E)).astype(np.float32) * np.float32(0.03125)
    else:
        L = np.full((T, E), 0.5, dtype=np.float32)
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    layer.route_from_logits(torch.from_numpy(L).to(DEV), ids, w)
    torch.cuda.synchronize()
    rid, rw = O.route_topk(L, k)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert np.allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=1e-7)
    layer.close()


@pytest.mark.parametrize("wl_name", ["prefill-int4-zipf", "prefill-nvfp4"])
def test_route_from_logits_full_size(wl_name):
    wl = synth.workload(wl_name)
    layer = moe.MoeLayer(wl.H, wl.I, wl.E, wl.k, wl.quant, False, wl.T, 0)
    L = synth.routing_logits(wl)
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device=DEV)
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device=DEV)
    layer.route_from_logits(torch.from_numpy(L).to(DEV), ids, w)
    torch.cuda.synchronize()
    rid, rw = O.route_topk(L, wl.k)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert np.allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=1e-7)
    layer.close()


# ---------------------------------------------------------------- permute
@pytest.mark.parametrize("T,k,E", [(1, 10, 512), (4, 10, 512), (37, 4, 16), (4096, 10, 512), (8192, 10, 512)])
def test_permute_bit_exact(T, k, E):
    rng = np.random.default_rng(T + E)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = moe.permute(torch.from_numpy(ids).to(DEV), E)
    torch.cuda.synchronize()
    rc, ro, rp, ri = O.permute(ids, E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy(), rp)
    assert np.array_equal(inv.cpu().numpy(), ri)


# chunks of 2048 slots (more than 128 x 1024 slots), the largest E, an E
# that is not a multiple of 32, every token on the same k experts (one
# segment spans all warps and chunks), and ids outside [0, E) (dropped)
@pytest.mark.parametrize("case", ["chunk2048", "e1024", "e7", "same_experts", "invalid_ids"])
def test_permute_bit_exact_edge_cases(case):
    rng = np.random.default_rng(7)
    if case == "chunk2048":
        T, k, E = 20000, 10, 512
    elif case == "e1024":
        T, k, E = 3000, 8, 1024
    elif case == "e7":
        T, k, E = 1000, 3, 7
    else:
        T, k, E = 5000, 10, 512
    if case == "same_experts":
        ids = np.tile(np.arange(k, dtype=np.int32)[::-1], (T, 1))
    else:
        ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    if case == "invalid_ids":
        mask = rng.random(ids.shape) < 0.05
        ids[mask] = rng.choice(np.array([-1, E, E + 100, -(1 << 30)], dtype=np.int32), int(mask.sum()))
    counts, offsets, perm, inv = moe.permute(torch.from_numpy(ids).to(DEV), E)
    torch.cuda.synchronize()
    rc, ro, rp, ri = O.permute(ids, E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    n = int(ro[-1])
    assert np.array_equal(perm.cpu().numpy()[:n], rp[:n])
    assert np.array_equal(inv.cpu().numpy(), ri)


# ---------------------------------------------------------------- forward
def _forward_case(wl, T, seed_tokens=None):
    ox = OracleExperts(wl)
    layer = get_layer(wl, max(T, 4))
    x = synth.activations_bf16(wl, steps=max(1, (T + wl.T - 1) // wl.T))[:T]
    wr = synth.router_bf16(wl)
    logits = O.router_logits(x, wr)
    ids, w = O.route_topk(logits, wl.k)
    act = None
    if wl.quant == "nvfp4":
        xf = O.bf16_bits_to_f32(x)
        g_x = O.nvfp4_global_scale(np.abs(xf).max())
        g_a = O.nvfp4_global_scale(O.intermediate_amax(x, ids, "nvfp4", ox, g_x))
        act = (g_x, g_a)
        layer.set_act_global_scales(g_x, g_a)
    y_ref = O.moe_forward(x, ids, w, wl.quant, ox, shared=ox.shared(), act_scales=act)
    y = torch.empty((T, wl.H), dtype=torch.bfloat16, device=DEV)
    layer.forward(bf16_tensor(x, DEV), torch.from_numpy(ids).to(DEV),
                  torch.from_numpy(w.astype(np.float32)).to(DEV), y)
    torch.cuda.synchronize()
    return to_bits(y), y_ref, layer, (x, ids, w)


SMALL = {
    "int4": synth.custom("tiny-int4", H=384, I=256, E=16, k=4, shared=True),
    "int4g32": synth.custom("tiny-int4", quant="int4g32", H=384, I=256, E=16, k=4, shared=True),
    "fp8": synth.custom("tiny-int4", quant="fp8", H=384, I=256, E=16, k=4, shared=True),
    "fp6": synth.custom("tiny-int4", quant="fp6", H=384, I=256, E=16, k=4, shared=True),
    "int2": synth.custom("tiny-int4", quant="int2", H=384, I=256, E=16, k=4, shared=True),
    "nvfp4": synth.custom("tiny-int4", quant="nvfp4", H=384, I=256, E=16, k=4, shared=True),
}


def test_forward_tiny_workload():
    wl = synth.workload("tiny-int4")
    y, y_ref, _, _ = _forward_case(wl, wl.T)
    assert_close_output(y, y_ref)


@pytest.mark.parametrize("quant", ["int4", "int4g32", "int2", "nvfp4", "fp8", "fp6"])
@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 9])
def test_forward_small_layers(quant, T):
    y, y_ref, _, _ = _forward_case(SMALL[quant], T)
    assert_close_output(y, y_ref)


def test_forward_is_deterministic_and_token_independent():
    wl = SMALL["int4"]
    y1, y_ref, layer, (x, ids, w) = _forward_case(wl, 4)
    y2, _, _, _ = _forward_case(wl, 4)
    assert np.array_equal(y1, y2)
    # one token alone gives the same row as in the batch (up to accumulation
    # order, which is identical here: per-token sums do not depend on T)
    y_single, _, _, _ = _forward_case(wl, 1)
    assert np.array_equal(y_single[0], y1[0])


def _decode_all_steps(wl_name):
    """Every step of a decode workload (oracle routing of each step's tokens,
    one moe_forward per step) against one batched oracle pass: the layer is
    per token, so the batch's rows are the steps' outputs."""
    wl = synth.workload(wl_name)
    layer, _ = build_layer(wl, 0, max_tokens=wl.T)
    xs = synth.activations_bf16(wl)
    ids, w = O.route_topk(O.router_logits(xs, synth.router_bf16(wl)), wl.k)
    y = torch.empty((wl.steps * wl.T, wl.H), dtype=torch.bfloat16, device=DEV)
    xd = bf16_tensor(xs, DEV)
    idd = torch.from_numpy(ids).to(DEV)
    wd = torch.from_numpy(w.astype(np.float32)).to(DEV)
    for i in range(wl.steps):
        r = slice(i * wl.T, (i + 1) * wl.T)
        layer.forward(xd[r], idd[r], wd[r], y[r])
    layer.sync_status()
    layer.close()
    sx = StreamingExperts(wl)
    sx.start(valid_experts(ids, wl.E))
    y_ref = O.moe_forward(xs, ids, w, wl.quant, sx, shared=sx.shared())
    sx.close()
    yb = to_bits(y)
    for i in range(wl.steps):
        r = slice(i * wl.T, (i + 1) * wl.T)
        assert_close_output(yb[r], y_ref[r])


def test_decode_b1_workload_all_tokens():
    _decode_all_steps("decode-b1-int4")


def test_decode_b4_int2_workload_all_steps():
    _decode_all_steps("decode-b4-int2")


# ------------------------------------------- 9 to 16 tokens on the GEMV path
@pytest.mark.parametrize("quant", ["int4", "int4g32", "int2", "nvfp4", "fp8", "fp6"])
@pytest.mark.parametrize("T", [9, 12, 16])
def test_decode_gemv_up_to_16_tokens(quant, T):
    """9 to 16 tokens on the GEMV kernels (forced; two 8-column MMA groups)
    and on the grouped-GEMM path, the default for these sizes."""
    wl = SMALL[quant]
    layer = get_layer(wl, max(T, 4))
    layer.set_decode_path("kernels")
    y, y_ref, layer, (x, ids, w) = _forward_case(wl, T)
    assert_close_output(y, y_ref)
    layer.set_decode_path("gemm")
    y2 = torch.empty((T, wl.H), dtype=torch.bfloat16, device=DEV)
    layer.forward(bf16_tensor(x, DEV), torch.from_numpy(ids).to(DEV), torch.from_numpy(w.astype(np.float32)).to(DEV), y2)
    layer.sync_status()
    layer.set_decode_path("auto")
    assert_close_output(to_bits(y2), y_ref)


def test_decode_b1_int4_16_tokens_full_size():
    """The decode-b1 INT4 layer at full size with 16 tokens per call (a
    speculative verify step), GEMV path and grouped-GEMM path."""
    wl = synth.workload("decode-b1-int4")
    layer, _ = build_layer(wl, 0, max_tokens=16)
    xs = synth.activations_bf16(wl)[:16]
    ids, w = O.route_topk(O.router_logits(xs, synth.router_bf16(wl)), wl.k)
    ys = {}
    for path in ("kernels", "gemm"):
        layer.set_decode_path(path)
        y = torch.empty((16, wl.H), dtype=torch.bfloat16, device=DEV)
        layer.forward(bf16_tensor(xs, DEV), torch.from_numpy(ids).to(DEV), torch.from_numpy(w.astype(np.float32)).to(DEV), y)
        layer.sync_status()
        ys[path] = to_bits(y)
    layer.close()
    sx = StreamingExperts(wl)
    sx.start(valid_experts(ids, wl.E))
    y_ref = O.moe_forward(xs, ids, w, wl.quant, sx, shared=sx.shared())
    sx.close()
    for yb in ys.values():
        assert_close_output(yb, y_ref)


# ------------------------------------------------- slots without an expert
@pytest.mark.parametrize("quant", ["int4", "int2", "nvfp4"])
@pytest.mark.parametrize("T", [5, 300])
def test_forward_out_of_range_ids_contribute_zero(quant, T):
    """A slot whose id lies outside [0, E) (here -1, E and a large id, at most
    one per token) selects no expert: the layer matches the oracle that skips
    it, on the decode path (T = 5) and the grouped-GEMM path (T = 300), with
    stale values left in the workspace by an earlier call."""
    wl = MID[quant] if T > 8 else SMALL[quant]
    ox = OracleExperts(wl)
    layer = get_layer(wl, max(T, 4))
    x = synth.activations_bf16(wl, steps=max(1, (T + wl.T - 1) // wl.T))[:T]
    ids, w = O.route_topk(O.router_logits(x, synth.router_bf16(wl)), wl.k)
    act = None
    if quant == "nvfp4":
        g_x = O.nvfp4_global_scale(np.abs(O.bf16_bits_to_f32(x)).max())
        g_a = O.nvfp4_global_scale(O.intermediate_amax(x, ids, "nvfp4", ox, g_x))
        act = (g_x, g_a)
        layer.set_act_global_scales(g_x, g_a)
    y = torch.empty((T, wl.H), dtype=torch.bfloat16, device=DEV)
    xd = bf16_tensor(x, DEV)
    wd = torch.from_numpy(w.astype(np.float32)).to(DEV)
    layer.forward(xd, torch.from_numpy(ids).to(DEV), wd, y)       # leaves every slot's output in the workspace
    rng = np.random.default_rng(T)
    bad = ids.copy()
    rows = rng.choice(T, max(1, T // 3), replace=False)
    cols = rng.integers(0, wl.k, rows.size)
    bad[rows, cols] = rng.choice(np.array([-1, wl.E, 1 << 20], np.int32), rows.size)
    layer.forward(xd, torch.from_numpy(bad).to(DEV), wd, y)
    layer.sync_status()
    y_ref = O.moe_forward(x, bad, w, quant, ox, shared=ox.shared(), act_scales=act, num_experts=wl.E)
    assert_close_output(to_bits(y), y_ref)


# ------------------------------------------------------------ error paths
def test_errors_are_reported_without_device_work():
    wl = SMALL["int4"]
    layer = moe.MoeLayer(wl.H, wl.I, wl.E, wl.k, "int4", True, 4, 0)
    x = torch.zeros((4, wl.H), dtype=torch.bfloat16, device=DEV)
    ids = torch.zeros((4, wl.k), dtype=torch.int32, device=DEV)
    w = torch.zeros((4, wl.k), dtype=torch.float32, device=DEV)
    y = torch.zeros((4, wl.H), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(moe.MoeError) as ei:
        layer.forward(x, ids, w, y)                  # nothing loaded yet
    assert ei.value.status == moe.MOE_ERR_STATE
    with pytest.raises(moe.MoeError) as ei:
        layer.route(x, ids, w)                       # router not loaded
    assert ei.value.status == moe.MOE_ERR_STATE
    big = torch.zeros((5, wl.H), dtype=torch.bfloat16, device=DEV)
    layer.load_router(torch.zeros((wl.E, wl.H), dtype=torch.bfloat16, device=DEV))
    with pytest.raises(moe.MoeError) as ei:
        layer.route(big, ids, w)                     # T > max_tokens
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoeError) as ei:
        layer.load_expert(wl.E, {n: {"codes": x, "scales": x} for n in ("gate", "up", "down")})
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoeError) as ei:
        moe.MoeLayer(100, 256, 8, 2, "int4", False, 4, 0)   # H not a multiple of 128
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
    with pytest.raises(moe.MoeError) as ei:
        layer.set_act_global_scales(1.0, 1.0)        # not an NVFP4 layer
    assert ei.value.status == moe.MOE_ERR_STATE
    layer.close()


# ------------------------------------------------ grouped GEMM (prefill) path
MID = {
    "int4": synth.custom("tiny-int4", H=512, I=384, E=24, k=6, shared=True),
    "int4g32": synth.custom("tiny-int4", quant="int4g32", H=512, I=384, E=24, k=6, shared=True),
    "fp8": synth.custom("tiny-int4", quant="fp8", H=512, I=384, E=24, k=6, shared=True),
    "fp6": synth.custom("tiny-int4", quant="fp6", H=512, I=384, E=24, k=6, shared=True),
    "int2": synth.custom("tiny-int4", quant="int2", H=512, I=384, E=24, k=6, shared=True),
    "nvfp4": synth.custom("tiny-int4", quant="nvfp4", H=512, I=384, E=24, k=6, shared=True),
}


@pytest.mark.parametrize("quant", ["int4", "int4g32", "int2", "nvfp4", "fp8", "fp6"])
@pytest.mark.parametrize("T", [5, 37, 300])
def test_prefill_matches_oracle(quant, T):
    """T > 4 runs the permutation + tcgen05 grouped GEMMs: several 128-row
    weight blocks, several 64-column K blocks, token tiles with ragged tails
    and the shared expert's tiles."""
    y, y_ref, layer, _ = _forward_case(MID[quant], T)
    layer.sync_status()
    assert_close_output(y, y_ref)


# H and I multiples of 256: NVFP4 runs the block-scaled (e2m1 x e2m1, e4m3
# scales in TMEM) tensor-core GEMMs instead of the bf16 dequantization path
NATIVE_FP4 = synth.custom("tiny-int4", quant="nvfp4", H=512, I=256, E=24, k=6, shared=True)


# T = 700 and 1500: experts with 129..176 tokens (one wide gate/up tile) and
# with more (several tiles, the last a ragged one)
@pytest.mark.parametrize("T", [5, 37, 300, 700, 1500])
def test_prefill_nvfp4_block_scaled_matches_oracle(T):
    y, y_ref, layer, _ = _forward_case(NATIVE_FP4, T)
    layer.sync_status()
    assert_close_output(y, y_ref)


def test_prefill_nvfp4_block_scaled_one_expert_takes_many_tokens():
    """Every token on the same six experts: gate/up tiles of 176 tokens and a
    ragged last tile, down tiles of 128."""
    wl = NATIVE_FP4
    T = 700
    ox = OracleExperts(wl)
    layer = get_layer(wl, T)
    x = synth.activations_bf16(wl, steps=T // wl.T + 1)[:T]
    ids = np.tile(np.array([3, 7, 0, 23, 11, 5], np.int32), (T, 1))
    w = np.tile(np.array([0.3, 0.2, 0.15, 0.15, 0.1, 0.1]), (T, 1))
    g_x = O.nvfp4_global_scale(np.abs(O.bf16_bits_to_f32(x)).max())
    g_a = O.nvfp4_global_scale(O.intermediate_amax(x, ids, "nvfp4", ox, g_x))
    layer.set_act_global_scales(g_x, g_a)
    y = torch.empty((T, wl.H), dtype=torch.bfloat16, device=DEV)
    layer.forward(bf16_tensor(x, DEV), torch.from_numpy(ids).to(DEV), torch.from_numpy(w.astype(np.float32)).to(DEV), y)
    layer.sync_status()
    y_ref = O.moe_forward(x, ids, w, "nvfp4", ox, shared=ox.shared(), act_scales=(g_x, g_a))
    assert_close_output(to_bits(y), y_ref)


def test_prefill_one_expert_takes_many_tokens():
    """All tokens on the same experts: segments of several 128-token tiles."""
    wl = MID["int4"]
    T = 700
    ox = OracleExperts(wl)
    layer = get_layer(wl, T)
    x = synth.activations_bf16(wl, steps=T // wl.T + 1)[:T]
    ids = np.tile(np.array([3, 7, 0, 23, 11, 5], np.int32), (T, 1))
    w = np.tile(np.array([0.3, 0.2, 0.15, 0.15, 0.1, 0.1]), (T, 1))
    y = torch.empty((T, wl.H), dtype=torch.bfloat16, device=DEV)
    layer.forward(bf16_tensor(x, DEV), torch.from_numpy(ids).to(DEV), torch.from_numpy(w.astype(np.float32)).to(DEV), y)
    layer.sync_status()
    y_ref = O.moe_forward(x, ids, w, "int4", ox, shared=ox.shared())
    assert_close_output(to_bits(y), y_ref)


def test_prefill_is_deterministic():
    wl = MID["int2"]
    y1, _, _, _ = _forward_case(wl, 300)
    y2, _, _, _ = _forward_case(wl, 300)
    assert np.array_equal(y1, y2)


def _full_size_all_rows(wl_name):
    """A full-size prefill workload, every token compared with the oracle.
    Routing is the oracle's top-k of the workload's routing logits; the
    oracle streams the experts (bounded memory); the NVFP4 intermediate's
    static global scale is calibrated on every routed slot."""
    wl = synth.workload(wl_name)
    layer, _ = build_layer(wl, 0, max_tokens=wl.T)
    x = synth.activations_bf16(wl)
    ids, w = O.route_topk(synth.routing_logits(wl), wl.k)
    nvfp4 = wl.quant == "nvfp4"
    sx = StreamingExperts(wl, keep_quantized=nvfp4)
    experts = valid_experts(ids, wl.E)
    act = None
    if nvfp4:
        g_x = O.nvfp4_global_scale(np.abs(O.bf16_bits_to_f32(x)).max())
        sx.start(experts)
        g_a = O.nvfp4_global_scale(O.intermediate_amax(x, ids, "nvfp4", sx, g_x))
        act = (g_x, g_a)
        layer.set_act_global_scales(g_x, g_a)
    y = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=DEV)
    layer.forward(bf16_tensor(x, DEV), torch.from_numpy(ids).to(DEV), torch.from_numpy(w.astype(np.float32)).to(DEV), y)
    layer.sync_status()
    layer.close()
    sx.start(experts)
    y_ref = O.moe_forward(x, ids, w, wl.quant, sx, shared=sx.shared(), act_scales=act)
    sx.close()
    yb = to_bits(y)
    assert_close_output(yb, y_ref)
    # and row by row: a wrong tile (a ragged tail, an expert with few tokens)
    # cannot hide in the layer-wide figure
    yf = O.bf16_bits_to_f64(yb)
    rms = np.sqrt(np.mean(y_ref ** 2))
    row_rel = np.sqrt(np.mean((yf - y_ref) ** 2, axis=1)) / rms
    worst = int(np.argmax(row_rel))
    assert row_rel.max() <= 3e-2, f"token {worst}: row rel-RMS {row_rel[worst]:.3e}"


def test_prefill_zipf_int4_full_size_all_tokens():
    _full_size_all_rows("prefill-int4-zipf")


def test_prefill_nvfp4_full_size_all_tokens():
    _full_size_all_rows("prefill-nvfp4")


def test_prefill_zipf_int4g32_full_size_all_tokens():
    _full_size_all_rows("prefill-int4g32-zipf")


def test_prefill_zipf_fp8_full_size_all_tokens():
    _full_size_all_rows("prefill-fp8-zipf")


def test_prefill_zipf_fp6_full_size_all_tokens():
    _full_size_all_rows("prefill-fp6-zipf")


# --------------------------------------------- whole layer in one call (fused)
@pytest.mark.parametrize("quant", ["int4", "int4g32", "int2", "nvfp4", "fp8", "fp6"])
@pytest.mark.parametrize("T", [1, 3, 8])
def test_route_forward_matches_route_then_oracle(quant, T):
    """moe_route_forward (one cooperative kernel for T <= 8): ids/weights equal
    moe_route's, output matches the oracle on those ids/weights."""
    wl = SMALL[quant]
    layer = get_layer(wl, 8)
    ox = OracleExperts(wl)
    x = synth.activations_bf16(wl, steps=2)[:T]
    xd = bf16_tensor(x, DEV)
    act = None
    if quant == "nvfp4":
        xf = O.bf16_bits_to_f32(x)
        g_x = O.nvfp4_global_scale(np.abs(xf).max())
        rid, _ = O.route_topk(O.router_logits(x, synth.router_bf16(wl)), wl.k)
        g_a = O.nvfp4_global_scale(O.intermediate_amax(x, rid, "nvfp4", ox, g_x))
        act = (g_x, g_a)
        layer.set_act_global_scales(g_x, g_a)
    ids_r = torch.empty((T, wl.k), dtype=torch.int32, device=DEV)
    w_r = torch.empty((T, wl.k), dtype=torch.float32, device=DEV)
    layer.route(xd, ids_r, w_r)
    ids = torch.full((T, wl.k), -1, dtype=torch.int32, device=DEV)
    w = torch.zeros((T, wl.k), dtype=torch.float32, device=DEV)
    y = torch.empty((T, wl.H), dtype=torch.bfloat16, device=DEV)
    layer.route_forward(xd, ids, w, y)
    layer.sync_status()
    assert torch.equal(ids, ids_r)
    assert torch.allclose(w, w_r, rtol=2e-6, atol=1e-7)
    ids_h, w_h = ids.cpu().numpy(), w.cpu().numpy().astype(np.float64)
    y_ref = O.moe_forward(x, ids_h, w_h, quant, ox, shared=ox.shared(), act_scales=act)
    assert_close_output(to_bits(y), y_ref)
    # twice in a row: tickets and the grid barrier are reusable, results identical
    y2 = torch.empty_like(y)
    layer.route_forward(xd, ids, w, y2)
    layer.sync_status()
    assert torch.equal(y, y2)


@pytest.mark.parametrize("quant", ["int4", "int2"])
def test_route_forward_paths(quant):
    """The fused kernel (eager default), the router + GEMV kernels (forced, and
    chosen by default under stream capture) compute the same layer; the
    captured graph equals moe_route followed by moe_forward bit for bit."""
    wl = SMALL[quant]
    T = 3
    layer = get_layer(wl, 8)
    ox = OracleExperts(wl)
    x = synth.activations_bf16(wl, steps=2)[:T]
    xd = bf16_tensor(x, DEV)
    ids = torch.empty((T, wl.k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, wl.k), dtype=torch.float32, device=DEV)
    ys = {}
    for path in ("fused", "kernels"):
        layer.set_decode_path(path)
        y = torch.empty((T, wl.H), dtype=torch.bfloat16, device=DEV)
        layer.route_forward(xd, ids, w, y)
        layer.sync_status()
        ys[path] = y
        ids_h, w_h = ids.cpu().numpy(), w.cpu().numpy().astype(np.float64)
        assert_close_output(to_bits(y), O.moe_forward(x, ids_h, w_h, quant, ox, shared=ox.shared()))
    layer.set_decode_path("auto")
    st = torch.cuda.Stream(device=DEV)
    yg = torch.empty((T, wl.H), dtype=torch.bfloat16, device=DEV)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        layer.route_forward(xd, ids, w, yg)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(yg, ys["kernels"])
    del g
    layer.set_decode_path("auto")


@pytest.mark.parametrize("wl_name", ["decode-b1-int4", "decode-b1-int4g32", "decode-b1-fp8", "decode-b1-fp6"])
def test_route_forward_decode_b1_full_size(wl_name):
    """All 100 tokens of the decode workload through moe_route_forward, on
    the fused kernel (eager) and on the router + GEMV kernels: ids equal the
    oracle's routing (up to near-ties of the logits), outputs match the
    oracle on the oracle's routing."""
    wl = synth.workload(wl_name)
    layer, _ = build_layer(wl, 0, max_tokens=4)
    xs = synth.activations_bf16(wl)
    logits = O.router_logits(xs, synth.router_bf16(wl))
    rid, rw = O.route_topk(logits, wl.k)
    xd = bf16_tensor(xs, DEV)
    out = {}
    for path in ("fused", "kernels"):
        layer.set_decode_path(path)
        ids = torch.empty((wl.steps, wl.k), dtype=torch.int32, device=DEV)
        w = torch.empty((wl.steps, wl.k), dtype=torch.float32, device=DEV)
        y = torch.empty((wl.steps, wl.H), dtype=torch.bfloat16, device=DEV)
        for i in range(wl.steps):
            layer.route_forward(xd[i:i + 1], ids[i:i + 1], w[i:i + 1], y[i:i + 1])
        layer.sync_status()
        out[path] = (ids.cpu().numpy(), w.cpu().numpy(), to_bits(y))
    layer.close()
    sx = StreamingExperts(wl)
    sx.start(valid_experts(rid, wl.E))
    y_ref = O.moe_forward(xs, rid, rw, wl.quant, sx, shared=sx.shared())
    sx.close()
    srt = -np.sort(-logits, axis=1)
    gap = srt[:, wl.k - 1] - srt[:, wl.k]
    for path, (ids_h, w_h, yb) in out.items():
        same = np.all(ids_h == rid, axis=1)
        assert np.all(gap[~same] < 1e-4), path
        assert np.allclose(w_h[same], rw[same], rtol=1e-5, atol=1e-7)
        for i in np.nonzero(same)[0]:
            assert_close_output(yb[i:i + 1], y_ref[i:i + 1])
