"""Pins of the oracle's routing, permutation and layer forward against brute
force on tiny inputs, textbook special cases (a plain SwiGLU MLP, a dense
softmax mixture), an unquantised torch layer and the layer's invariants."""
import math

import numpy as np
import pytest
import torch

from bit_quantized_mixture_b200 import synth
from oracle import moe_oracle as O

TINY = synth.workload("tiny-int4")


def _quantized_experts(wl, quant):
    ews = {}
    for e in range(wl.E):
        mats = synth.expert_fp32(wl, e)
        ew = {}
        if quant == "nvfp4":
            g_gu = O.nvfp4_global_scale(max(np.abs(mats[0]).max(), np.abs(mats[1]).max()))
            g_d = O.nvfp4_global_scale(np.abs(mats[2]).max())
        for name, m in zip(("gate", "up", "down"), mats):
            if quant == "int4":
                c, s = O.quantize_int4(m)
                ew[name] = {"codes": c, "scales": s}
            elif quant == "int2":
                c, s, z = O.quantize_int2(m)
                ew[name] = {"codes": c, "scales": s, "zeros": z}
            else:
                g = g_d if name == "down" else g_gu
                c, s = O.quantize_nvfp4(m, g)
                ew[name] = {"codes": c, "scales": s, "g": g}
        ews[e] = ew
    return ews


def _expert_fn(ews, quant):
    cache = {}

    def fn(e):
        if e not in cache:
            cache[e] = O.dequantize_expert(quant, ews[e])
        return cache[e]
    return fn


# ------------------------------------------------------------ routing ----

def test_topk_matches_sorted_with_ties():
    rng = np.random.default_rng(5)
    L = rng.integers(-3, 4, size=(50, 16)).astype(np.float32)     # many exact ties
    ids, w = O.route_topk(L, 5)
    for t in range(50):
        ref = sorted(range(16), key=lambda e: (-float(L[t, e]), e))[:5]
        assert list(ids[t]) == ref
        ex = [math.exp(float(L[t, e]) - float(L[t, ref[0]])) for e in ref]
        assert np.allclose(w[t], [v / sum(ex) for v in ex], rtol=0, atol=1e-15)


def test_topk_weights_are_renormalised_softmax():
    rng = np.random.default_rng(6)
    L = rng.standard_normal((40, 64)).astype(np.float32)
    ids, w = O.route_topk(L, 10)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-12)
    assert np.all(np.diff(w, axis=1) <= 0)
    p = torch.softmax(torch.from_numpy(L).double(), dim=1).numpy()
    sel = np.take_along_axis(p, ids.astype(np.int64), axis=1)
    assert np.allclose(w, sel / sel.sum(axis=1, keepdims=True), rtol=1e-12, atol=0)
    assert all(len(set(r)) == 10 for r in ids)


def test_permutation_matches_sorted():
    rng = np.random.default_rng(7)
    ids = np.stack([rng.choice(32, 6, replace=False) for _ in range(77)]).astype(np.int32)
    counts, offsets, perm, inv = O.permute(ids, 32)
    flat = ids.reshape(-1)
    ref = sorted(range(flat.size), key=lambda s: (flat[s], s))
    assert list(perm) == ref
    assert list(counts) == [int((flat == e).sum()) for e in range(32)]
    assert offsets[0] == 0 and offsets[-1] == flat.size
    assert np.array_equal(perm[inv], np.arange(flat.size))


def test_permutation_drops_out_of_range_ids():
    """Slots whose id lies outside [0, E) take no position: brute force over
    the valid slots, sorted by (expert, slot)."""
    rng = np.random.default_rng(8)
    E = 12
    ids = np.stack([rng.choice(E, 4, replace=False) for _ in range(40)]).astype(np.int32)
    flat = ids.reshape(-1).copy()
    bad = rng.choice(flat.size, 23, replace=False)
    flat[bad[:8]] = -1
    flat[bad[8:16]] = E
    flat[bad[16:]] = 1000
    ids = flat.reshape(ids.shape)
    counts, offsets, perm, inv = O.permute(ids, E)
    good = [s for s in range(flat.size) if 0 <= flat[s] < E]
    ref = sorted(good, key=lambda s: (flat[s], s))
    n = len(ref)
    assert n == flat.size - 23
    assert list(perm[:n]) == ref and np.all(perm[n:] == -1)
    assert offsets[-1] == n and list(counts) == [int((flat == e).sum()) for e in range(E)]
    for s in range(flat.size):
        assert inv[s] == (ref.index(s) if s in ref else -1)


# ---------------------------------------------------- brute force tiny ----

def _brute_unpack_int4(codes, scales):
    N, Kh = codes.shape
    W = [[0.0] * (2 * Kh) for _ in range(N)]
    for n in range(N):
        for j in range(Kh):
            b = int(codes[n, j])
            for nib, k in ((b & 15, 2 * j), (b >> 4, 2 * j + 1)):
                W[n][k] = (nib - 8) * float(scales[n, k // 128])
    return W


def _brute_bf16(bits):
    return [[float(np.array([int(b) << 16], np.uint32).view(np.float32)[0]) for b in row] for row in bits]


def _dot(a, b):
    s = 0.0
    for u, v in zip(a, b):
        s += u * v
    return s


def test_tiny_layer_brute_force():
    """Workload 'tiny-int4' computed with Python loops and floats only."""
    wl = TINY
    ews = _quantized_experts(wl, "int4")
    x_bits = synth.activations_bf16(wl)
    wr_bits = synth.router_bf16(wl)
    X = _brute_bf16(x_bits)
    Wr = _brute_bf16(wr_bits)
    Wb = {e: [_brute_unpack_int4(ews[e][m]["codes"], ews[e][m]["scales"]) for m in ("gate", "up", "down")]
          for e in range(wl.E)}
    y_ref = []
    for t in range(wl.T):
        logits = [_dot(X[t], Wr[e]) for e in range(wl.E)]
        sel = sorted(range(wl.E), key=lambda e: (-logits[e], e))[:wl.k]
        ex = [math.exp(logits[e] - logits[sel[0]]) for e in sel]
        wts = [v / sum(ex) for v in ex]
        y = [0.0] * wl.H
        for e, wt in zip(sel, wts):
            Wg, Wu, Wd = Wb[e]
            a = []
            for n in range(wl.I):
                g = _dot(X[t], Wg[n])
                a.append(g / (1.0 + math.exp(-g)) * _dot(X[t], Wu[n]))
            for h in range(wl.H):
                y[h] += wt * _dot(a, Wd[h])
        y_ref.append(y)
    y_ref = np.array(y_ref)

    logits = O.router_logits(x_bits, wr_bits)
    ids, w = O.route_topk(logits, wl.k)
    y = O.moe_forward(x_bits, ids, w, "int4", _expert_fn(ews, "int4"))
    rel = np.sqrt(np.mean((y - y_ref) ** 2) / np.mean(y_ref ** 2))
    assert rel < 1e-12


_E2M1_GRID = [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def _brute_nvfp4(codes, sb, g):
    """Python decode of packed E2M1 codes (low nibble first) with E4M3 scales
    per 16 values and the fp32 global scale g, as lists of floats."""
    N, Kh = codes.shape
    out = []
    for n in range(N):
        row = []
        for j in range(Kh):
            for nib in (int(codes[n, j]) & 15, int(codes[n, j]) >> 4):
                row.append(_E2M1_GRID[nib & 7] * (-1 if nib & 8 else 1))
        sc = [((1 + (s & 7) / 8) * 2.0 ** (((s >> 3) & 15) - 7)) if (s >> 3) & 15 else (s & 7) / 8 * 2.0 ** -6
              for s in (int(v) for v in sb[n])]
        out.append([row[k] * sc[k // 16] * float(g) for k in range(len(row))])
    return out


def test_tiny_nvfp4_layer_brute_force():
    wl = synth.custom(TINY, quant="nvfp4", E=4, k=2, T=3)
    ews = _quantized_experts(wl, "nvfp4")
    x_bits = synth.activations_bf16(wl)
    Xf = O.bf16_bits_to_f32(x_bits)
    g_x = O.nvfp4_global_scale(np.abs(Xf).max())
    ids, w = O.route_topk(O.router_logits(x_bits, synth.router_bf16(wl)), wl.k)
    fn = _expert_fn(ews, "nvfp4")
    g_a = O.nvfp4_global_scale(O.intermediate_amax(x_bits, ids, "nvfp4", fn, g_x))
    dq = _brute_nvfp4

    xc, xs = O.quantize_nvfp4(Xf, g_x)
    Xq = dq(xc, xs, g_x)
    y_ref = np.zeros((wl.T, wl.H))
    for t in range(wl.T):
        for j in range(wl.k):
            e = int(ids[t, j])
            Wg, Wu, Wd = (dq(ews[e][m]["codes"], ews[e][m]["scales"], ews[e][m]["g"]) for m in ("gate", "up", "down"))
            a = []
            for n in range(wl.I):
                g = _dot(Xq[t], Wg[n])
                a.append(g / (1.0 + math.exp(-g)) * _dot(Xq[t], Wu[n]))
            ac, as_ = O.quantize_nvfp4(np.array([a], np.float32), g_a)
            aq = dq(ac, as_, g_a)[0]
            for h in range(wl.H):
                y_ref[t, h] += w[t, j] * _dot(aq, Wd[h])
    y = O.moe_forward(x_bits, ids, w, "nvfp4", fn, act_scales=(g_x, g_a))
    assert np.sqrt(np.mean((y - y_ref) ** 2) / np.mean(y_ref ** 2)) < 1e-9


@pytest.mark.parametrize("quant", ["int4", "nvfp4"])
def test_intermediate_amax_brute_force(quant):
    """The calibration amax of the SwiGLU intermediate is the largest |a| over
    every routed slot, here with experts repeated across tokens; a computed by
    Python loops over the decoded weights (and, for NVFP4, the decoded
    quantized activations)."""
    wl = synth.custom(TINY, quant=quant, E=4, k=2, T=4)
    ews = _quantized_experts(wl, quant)
    x_bits = synth.activations_bf16(wl)
    ids = np.array([[0, 1], [1, 2], [3, 0], [1, 3]], dtype=np.int32)
    g_x = None
    if quant == "nvfp4":
        Xf = O.bf16_bits_to_f32(x_bits)
        g_x = O.nvfp4_global_scale(np.abs(Xf).max())
        xc, xs = O.quantize_nvfp4(Xf, g_x)
        X = _brute_nvfp4(xc, xs, g_x)
        W = {e: [_brute_nvfp4(ews[e][m]["codes"], ews[e][m]["scales"], ews[e][m]["g"]) for m in ("gate", "up")]
             for e in range(wl.E)}
    else:
        X = _brute_bf16(x_bits)
        W = {e: [_brute_unpack_int4(ews[e][m]["codes"], ews[e][m]["scales"]) for m in ("gate", "up")]
             for e in range(wl.E)}
    amax = 0.0
    for t in range(wl.T):
        for j in range(wl.k):
            Wg, Wu = W[int(ids[t, j])]
            for n in range(wl.I):
                g = _dot(X[t], Wg[n])
                amax = max(amax, abs(g / (1.0 + math.exp(-g)) * _dot(X[t], Wu[n])))
    got = O.intermediate_amax(x_bits, ids, quant, _expert_fn(ews, quant), g_x)
    assert got == pytest.approx(amax, rel=1e-12)
    # fewer tokens cannot raise it (up to the summation order of a different batch)
    got_sub = O.intermediate_amax(x_bits[:2], ids[:2], quant, _expert_fn(ews, quant), g_x)
    assert got_sub <= got * (1 + 1e-12)


# --------------------------------------------------- special cases ----

def _torch_mlp(X, Wg, Wu, Wd):
    return (torch.nn.functional.silu(X @ Wg.T) * (X @ Wu.T)) @ Wd.T


def test_single_expert_is_plain_swiglu_mlp():
    wl = synth.custom(TINY, E=1, k=1, T=6)
    ews = _quantized_experts(wl, "int4")
    fn = _expert_fn(ews, "int4")
    x_bits = synth.activations_bf16(wl)
    ids, w = O.route_topk(O.router_logits(x_bits, synth.router_bf16(wl)), 1)
    assert np.all(ids == 0) and np.all(w == 1.0)
    y = O.moe_forward(x_bits, ids, w, "int4", fn)
    X = torch.from_numpy(O.bf16_bits_to_f64(x_bits))
    ref = _torch_mlp(X, *(torch.from_numpy(m) for m in fn(0))).numpy()
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_k_equals_E_is_dense_softmax_mixture():
    wl = synth.custom(TINY, k=8, T=5)
    ews = _quantized_experts(wl, "int4")
    fn = _expert_fn(ews, "int4")
    x_bits = synth.activations_bf16(wl)
    logits = O.router_logits(x_bits, synth.router_bf16(wl))
    ids, w = O.route_topk(logits, wl.E)
    y = O.moe_forward(x_bits, ids, w, "int4", fn)
    X = torch.from_numpy(O.bf16_bits_to_f64(x_bits))
    p = torch.softmax(torch.from_numpy(logits), dim=1)
    ref = sum(p[:, e:e + 1] * _torch_mlp(X, *(torch.from_numpy(m) for m in fn(e))) for e in range(wl.E))
    assert np.allclose(y, ref.numpy(), rtol=1e-10, atol=1e-13)


def test_matches_unquantised_fp32_torch_layer():
    wl = synth.custom(TINY, T=16)
    ews = _quantized_experts(wl, "int4")
    fn = _expert_fn(ews, "int4")
    x_bits = synth.activations_bf16(wl)
    logits = O.router_logits(x_bits, synth.router_bf16(wl))
    ids, w = O.route_topk(logits, wl.k)
    y = O.moe_forward(x_bits, ids, w, "int4", fn)
    X = torch.from_numpy(O.bf16_bits_to_f32(x_bits))
    ref = torch.zeros(wl.T, wl.H)
    for t in range(wl.T):
        for j in range(wl.k):
            Wg, Wu, Wd = (torch.from_numpy(m.astype(np.float32)) for m in fn(int(ids[t, j])))
            ref[t] += float(w[t, j]) * _torch_mlp(X[t:t + 1], Wg, Wu, Wd)[0]
    rel = np.sqrt(np.mean((y - ref.double().numpy()) ** 2) / np.mean(y ** 2))
    assert rel < 1e-5


# --------------------------------------------------------- invariants ----

def test_linear_in_down_projection_and_token_independence():
    wl = synth.custom(TINY, T=12)
    ews = _quantized_experts(wl, "int4")
    x_bits = synth.activations_bf16(wl)
    ids, w = O.route_topk(O.router_logits(x_bits, synth.router_bf16(wl)), wl.k)
    y = O.moe_forward(x_bits, ids, w, "int4", _expert_fn(ews, "int4"))
    e = int(ids[0, 0])
    doubled = {k: v for k, v in ews.items()}
    doubled[e] = dict(ews[e], down={"codes": ews[e]["down"]["codes"],
                                    "scales": (ews[e]["down"]["scales"].astype(np.float32) * 2).astype(np.float16)})
    zeroed = dict(ews)
    zeroed[e] = dict(ews[e], down={"codes": ews[e]["down"]["codes"],
                                   "scales": np.zeros_like(ews[e]["down"]["scales"])})
    y2 = O.moe_forward(x_bits, ids, w, "int4", _expert_fn(doubled, "int4"))
    y0 = O.moe_forward(x_bits, ids, w, "int4", _expert_fn(zeroed, "int4"))
    assert np.allclose(y2 + y0, 2 * y, rtol=0, atol=1e-12)
    assert not np.allclose(y2, y)
    # tokens not routed to e are untouched
    untouched = ~np.any(ids == e, axis=1)
    assert np.array_equal(y0[untouched], y[untouched])
    # each token alone gives the same row; token order does not matter
    fn = _expert_fn(ews, "int4")
    for t in (0, 5, 11):
        yt = O.moe_forward(x_bits[t:t + 1], ids[t:t + 1], w[t:t + 1], "int4", fn)
        assert np.allclose(yt[0], y[t], rtol=1e-13, atol=1e-15)
    p = np.random.default_rng(8).permutation(wl.T)
    yp = O.moe_forward(x_bits[p], ids[p], w[p], "int4", fn)
    assert np.allclose(yp, y[p], rtol=1e-13, atol=1e-15)


def test_shared_expert_is_added_with_weight_one():
    wl = synth.custom(TINY, T=3, shared=True)
    ews = _quantized_experts(wl, "int4")
    fn = _expert_fn(ews, "int4")
    x_bits = synth.activations_bf16(wl)
    ids, w = O.route_topk(O.router_logits(x_bits, synth.router_bf16(wl)), wl.k)
    sh = tuple(O.bf16_bits_to_f64(m) for m in synth.shared_bf16(wl))
    y = O.moe_forward(x_bits, ids, w, "int4", fn)
    ys = O.moe_forward(x_bits, ids, w, "int4", fn, shared=sh)
    X = torch.from_numpy(O.bf16_bits_to_f64(x_bits))
    ref = _torch_mlp(X, *(torch.from_numpy(m) for m in sh)).numpy()
    assert np.allclose(ys - y, ref, rtol=1e-10, atol=1e-13)


def test_out_of_range_ids_contribute_zero():
    """With num_experts given, a slot whose id lies outside [0, E) adds
    nothing: the result equals the same routing with that slot's weight set
    to zero (the slot then pointing at a valid expert), computed by the plain
    Python-loop reference."""
    wl = synth.custom(TINY, T=7)
    ews = _quantized_experts(wl, "int4")
    fn = _expert_fn(ews, "int4")
    x_bits = synth.activations_bf16(wl)
    ids, w = O.route_topk(O.router_logits(x_bits, synth.router_bf16(wl)), wl.k)
    bad = ids.copy()
    bad[0, 1], bad[3, 0], bad[6, 1] = -1, wl.E, 10 ** 6
    y = O.moe_forward(x_bits, bad, w, "int4", fn, num_experts=wl.E)
    w0 = w.copy()
    w0[0, 1] = w0[3, 0] = w0[6, 1] = 0.0
    X = O.bf16_bits_to_f64(x_bits)
    ref = np.zeros_like(y)
    for t in range(wl.T):
        for j in range(wl.k):
            Wg, Wu, Wd = fn(int(ids[t, j]))
            ref[t] += w0[t, j] * (O.silu(X[t] @ Wg.T) * (X[t] @ Wu.T)) @ Wd.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-15)
    assert not np.allclose(y[0], O.moe_forward(x_bits, ids, w, "int4", fn)[0])
