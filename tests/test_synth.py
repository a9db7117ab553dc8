"""The seeded synthetic inputs: reproducible draw by draw, each tensor from
its own stream, the stated distributions, bf16 round-to-nearest-even, and the
realized routing histograms of the two prefill workloads (seed 0)."""
import numpy as np
import pytest

from bit_quantized_mixture_b200 import synth
from oracle import moe_oracle as O

TINY = synth.workload("tiny-int4")


def test_draws_are_reproducible_and_per_expert():
    a = synth.expert_fp32(TINY, 3)
    b = synth.expert_fp32(TINY, 3)
    for m, n in zip(a, b):
        assert np.array_equal(m, n)
    c = synth.expert_fp32(TINY, 4)
    assert not np.array_equal(a[0], c[0])
    # one expert regenerated alone equals the same expert drawn among others
    it = {e: ws for e, *ws in synth.experts_fp32_iter(TINY, range(TINY.E), threads=3)}
    for m, n in zip(it[3], a):
        assert np.array_equal(m, n)
    assert np.array_equal(synth.activations_bf16(TINY), synth.activations_bf16(TINY))
    assert np.array_equal(synth.router_bf16(TINY), synth.router_bf16(TINY))


def test_stated_distributions():
    wl = synth.workload("decode-b1-int4")
    g, u, d = synth.expert_fp32(wl, 7)
    assert g.shape == (wl.I, wl.H) and u.shape == (wl.I, wl.H) and d.shape == (wl.H, wl.I)
    for m in (g, u, d):
        assert abs(float(m.std()) - 0.02) < 0.0005 and abs(float(m.mean())) < 0.0005
    x = O.bf16_bits_to_f32(synth.activations_bf16(wl))
    assert x.shape == (wl.steps * wl.T, wl.H)
    assert abs(float(x.std()) - 1.0) < 0.01 and abs(float(x.mean())) < 0.01
    wr = O.bf16_bits_to_f32(synth.router_bf16(wl))
    assert wr.shape == (wl.E, wl.H) and abs(float(wr.std()) - 0.02) < 0.0005


def test_bf16_rounding_is_nearest_even():
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 1 + 2 ** -8 + 2 ** -20,
                                  3.0e38, 1e-40, 0.0, -0.0], dtype=np.float32)])
    bits = v.view(np.uint32).astype(np.uint64)
    # round-to-nearest-even on the upper 16 bits, written out on the integers
    ref = ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16).astype(np.uint16)
    assert np.array_equal(synth.f32_to_bf16_bits(v), ref)
    # the ties 1 + 2^-8 round down to 1.0 (even), 1 + 3 * 2^-8 up to 1 + 2^-6
    out = synth.f32_to_bf16_bits(v[-8:-4])
    assert list(out[:3]) == [0x3F80, 0x3F82, 0xBF80]


@pytest.mark.parametrize("name,stats", [
    ("prefill-int4-zipf", {"max": 3720, "ge128": 52, "lt64": 416, "lt16": 158, "min": 6}),
    ("prefill-nvfp4", {"max": 202, "ge128": 511, "lt64": 0, "lt16": 0, "min": 126}),
])
def test_realized_routing_histogram(name, stats):
    wl = synth.workload(name)
    ids, _ = O.route_topk(synth.routing_logits(wl), wl.k)
    c = np.bincount(ids.ravel(), minlength=wl.E)
    assert c.sum() == wl.T * wl.k
    got = {"max": int(c.max()), "ge128": int((c >= 128).sum()), "lt64": int((c < 64).sum()),
           "lt16": int((c < 16).sum()), "min": int(c.min())}
    assert got == stats
