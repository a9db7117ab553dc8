"""Pins of the oracle's number formats and quantizers against hand-worked
examples, exhaustive code tables, an independent library (torch's
float8_e4m3fn cast) and the error bounds the formats guarantee."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O


def _group(values, K=128):
    w = np.zeros((1, K), np.float32)
    for k, v in values.items():
        w[0, int(k)] = v
    return w


# ---------------------------------------------------------------- INT4 ----

def test_int4_worked_example(golden):
    g = golden["int4"]
    w = _group(g["group_values"])
    codes, s = O.quantize_int4(w)
    assert float(s[0, 0]) == g["scale"]["value_num"] * 2.0 ** g["scale"]["value_exp"]
    u = O.unpack_int4(codes)[0]
    for k, c in g["codes"].items():
        assert u[int(k)] == c
    assert np.all(np.delete(u, [int(k) for k in g["codes"]]) == 8)
    deq = O.dequantize_int4(codes, s)[0]
    for k, v in g["dequant"].items():
        assert deq[int(k)] == v


def test_int4_ties_round_half_even(golden):
    t = golden["int4"]["ties"]
    w = np.zeros((1, 128), np.float32)
    w[0, :len(t["w"])] = t["w"]
    codes, s = O.quantize_int4(w)
    assert float(s[0, 0]) == t["scale"]
    q = O.unpack_int4(codes)[0, :len(t["w"])].astype(int) - 8
    assert list(q) == t["q"]


def test_int4_nibble_packing_and_table():
    # every nibble value in every position parity, decoded as (u - 8) * s
    u = np.tile(np.arange(16, dtype=np.uint8), 8)[None, :]            # [1,128]
    codes = (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)
    assert codes[0, 0] == 0x10 and codes[0, 7] == 0xFE
    s = np.array([[0.25]], np.float16)
    deq = O.dequantize_int4(codes, s)[0]
    assert np.array_equal(deq, (np.arange(128) % 16 - 8) * 0.25)


def test_int4_zero_group_and_error_bound():
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((64, 512)) * 0.02).astype(np.float32)
    w[3, 128:256] = 0.0
    codes, s = O.quantize_int4(w)
    assert s[3, 1] == 0 and np.all(O.unpack_int4(codes)[3, 128:256] == 8)
    deq = O.dequantize_int4(codes, s)
    sf = np.repeat(s.astype(np.float64), 128, axis=1)
    # |w - deq| <= s/2, up to the fp16 rounding of the scale at the clamp
    assert np.all(np.abs(w - deq) <= sf * 0.5 * (1 + 2.0 ** -8) + 1e-30)
    q = O.unpack_int4(codes).astype(int) - 8
    assert q.min() >= -8 and q.max() <= 7


def test_int4_group32_worked_example(golden):
    g = golden["int4_g32"]
    w = _group(g["row_values"], K=g["K"])
    codes, s = O.quantize_int4(w, group=O.GROUP_INT4_G32)
    assert s.shape == (1, 2)
    for j, sc in enumerate(g["scales"]):
        assert float(s[0, j]) == sc["value_num"] * 2.0 ** sc["value_exp"]
    u = O.unpack_int4(codes)[0]
    for k, c in g["codes"].items():
        assert u[int(k)] == c
    assert np.all(np.delete(u, [int(k) for k in g["codes"]]) == 8)
    deq = O.dequantize_int4(codes, s)[0]
    for k, v in g["dequant"].items():
        assert deq[int(k)] == v
    # the same row in one 64-column group quantizes column 0 differently
    c2, s2 = O.quantize_int4(w, group=64)
    h = g["group128_contrast"]
    assert float(s2[0, 0]) == h["scale_value_num"] * 2.0 ** h["scale_value_exp"]
    assert O.unpack_int4(c2)[0, 0] == h["code_0"]


def test_int4_group32_dequant_by_element_loop():
    """dequantize_int4 with 32-column groups against a plain per-element loop."""
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((5, 96)) * 0.03).astype(np.float32)
    codes, s = O.quantize_int4(w, group=32)
    assert s.shape == (5, 3)
    deq = O.dequantize_int4(codes, s)
    for n in range(5):
        for k in range(96):
            byte = int(codes[n, k // 2])
            u = (byte >> 4) if k % 2 else (byte & 0xF)
            assert deq[n, k] == (u - 8) * float(s[n, k // 32])


def test_int4_group32_error_bound_and_finer_than_group128():
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((64, 512)) * 0.02).astype(np.float32)
    w[:, ::37] *= 8.0                                   # outliers that widen a group's range
    c32, s32 = O.quantize_int4(w, group=32)
    deq32 = O.dequantize_int4(c32, s32)
    sf = np.repeat(s32.astype(np.float64), 32, axis=1)
    assert np.all(np.abs(w - deq32) <= sf * 0.5 * (1 + 2.0 ** -8) + 1e-30)
    c128, s128 = O.quantize_int4(w)
    err32 = np.sqrt(np.mean((w - deq32) ** 2))
    err128 = np.sqrt(np.mean((w - O.dequantize_int4(c128, s128)) ** 2))
    assert err32 < err128


# ---------------------------------------------------------- FP6 e2m3 ----

def test_e2m3_table_all_codes(golden):
    g = golden["fp6_e2m3"]
    codes = np.arange(64, dtype=np.uint8)
    vals = O.e2m3_decode(codes)
    mags = np.array(g["magnitudes"])
    assert np.array_equal(vals[:32], mags)
    assert np.array_equal(vals[32:], -mags)
    # every value encodes back to its own code (signed zeros included)
    assert np.array_equal(O.e2m3_rne_satfinite(vals.astype(np.float32)), codes[:32].tolist() + [32 + i for i in range(32)])


def test_e2m3_midpoints_round_half_even(golden):
    for v, c in golden["fp6_e2m3"]["midpoints"].items():
        assert int(O.e2m3_rne_satfinite(np.float32(float(v)))) == c, v
    # every midpoint between neighbours goes to the even mantissa
    mags = np.array(golden["fp6_e2m3"]["magnitudes"])
    mids = (mags[1:] + mags[:-1]) / 2
    got = O.e2m3_rne_satfinite(mids.astype(np.float32)).astype(int)
    assert np.all(got % 2 == 0)


def test_fp6_worked_group(golden):
    g = golden["fp6_e2m3"]
    w = _group(g["group_values"], K=32)
    codes, s = O.quantize_fp6(w)
    assert float(s[0, 0]) == g["scale"]["value_num"] * 2.0 ** g["scale"]["value_exp"]
    for k, c in g["codes"].items():
        assert codes[0, int(k)] == c
    deq = O.dequantize_fp6(codes, s)[0]
    for k, c in g["codes"].items():
        assert deq[int(k)] == O.e2m3_decode(c) * float(s[0, 0])


def test_fp6_error_bound_and_groups_of_32():
    rng = np.random.default_rng(12)
    w = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    w[:, 32:64] *= 20.0                                         # one wide group per row
    codes, s = O.quantize_fp6(w)
    assert s.shape == (16, 8)
    deq = O.dequantize_fp6(codes, s)
    sf = np.repeat(s.astype(np.float64), 32, axis=1)
    r = np.abs(w) / np.where(sf == 0, 1, sf)
    half_q = np.where(r < 2, 0.0625, np.where(r < 4, 0.125, 0.25)) * sf
    assert np.all(np.abs(w - deq) <= half_q * (1 + 2.0 ** -8) + 1e-30)
    # a group's codes depend only on its own 32 values
    c2, s2 = O.quantize_fp6(w[:, 32:64])
    assert np.array_equal(c2, codes[:, 32:64]) and np.array_equal(s2[:, 0], s[:, 1])


# ----------------------------------------------------- FP8 128x128 blocks ----

def test_fp8_block_worked_example(golden):
    g = golden["fp8_block128"]
    w = np.zeros((128, 128), np.float32)
    for key, v in g["block_values"].items():
        n, k = map(int, key.split(","))
        w[n, k] = v
    codes, s = O.quantize_fp8_block(w)
    assert s.shape == (1, 1) and s.dtype == np.float32
    assert float(s[0, 0]) == g["scale"]["value_num"] * 2.0 ** g["scale"]["value_exp"]
    deq = O.dequantize_fp8_block(codes, s)
    for key, c in g["codes"].items():
        n, k = map(int, key.split(","))
        assert codes[n, k] == c
        assert deq[n, k] == g["dequant_e4m3"][key] * float(s[0, 0])
    mask = np.ones_like(codes, bool)
    for key in g["codes"]:
        n, k = map(int, key.split(","))
        mask[n, k] = False
    assert np.all(codes[mask] == 0)


def test_fp8_blocks_are_128_by_128():
    """Each 128x128 block has its own scale: a block's codes depend only on
    its own values."""
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((256, 384)) * 0.02).astype(np.float32)
    w[128:, 256:] *= 50.0                                     # one block much larger
    codes, s = O.quantize_fp8_block(w)
    assert s.shape == (2, 3)
    for bn in range(2):
        for bk in range(3):
            blk = w[bn * 128:(bn + 1) * 128, bk * 128:(bk + 1) * 128]
            c1, s1 = O.quantize_fp8_block(blk)
            assert s1[0, 0] == s[bn, bk]
            assert np.array_equal(c1, codes[bn * 128:(bn + 1) * 128, bk * 128:(bk + 1) * 128])
    assert s[1, 2] > 20 * s[0, 0]


def test_fp8_block_error_bound_and_zero_block():
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((128, 256)) * 0.02).astype(np.float32)
    w[:, 128:] = 0.0
    codes, s = O.quantize_fp8_block(w)
    assert s[0, 1] == 0 and np.all((codes[:, 128:] & 0x7F) == 0)
    deq = O.dequantize_fp8_block(codes, s)
    sc = float(s[0, 0])
    r = np.abs(w[:, :128]).astype(np.float64)
    err = np.abs(w[:, :128] - deq[:, :128])
    # half a quantum: 2^-4 relative in the normal range (|w/s| >= 2^-6), 2^-10 s below
    bound = np.where(r / sc >= 2.0 ** -6, r * 2.0 ** -4, sc * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound)
    assert np.abs(codes[:, :128].astype(np.int64) & 0x7F).max() <= 0x7E   # finite, at most 448


# ---------------------------------------------------------------- INT2 ----

def test_int2_worked_example(golden):
    g = golden["int2"]
    w = _group(g["group_values"], K=128)
    w = np.repeat(w, 4, axis=0)                     # N must be a multiple of 4
    codes, s, zeros = O.quantize_int2(w)
    assert float(s[0, 0]) == g["scale"]["value_num"] * 2.0 ** g["scale"]["value_exp"]
    z = O.unpack_int2_zeros(zeros)
    assert np.all(z[:, 0] == g["zero"])
    u = O.unpack_int2(codes)[0]
    for k, c in g["codes"].items():
        assert u[int(k)] == c
    assert np.all(u[4:] == 1)                       # zeros quantize to the zero point
    deq = O.dequantize_int2(codes, s, zeros)[0]
    for k, v in g["dequant"].items():
        assert deq[int(k)] == v


def test_int2_symmetric_special_case(golden):
    sc = golden["int2"]["symmetric_case"]
    w = np.zeros((4, 128), np.float32)
    w[:, 0], w[:, 1] = sc["min"], sc["max"]
    codes, s, zeros = O.quantize_int2(w)
    assert float(s[0, 0]) == sc["scale"]
    assert np.all(O.unpack_int2_zeros(zeros) == sc["zero"])


def test_int2_one_sided_groups():
    w = np.zeros((4, 256), np.float32)
    w[:, :128] = np.linspace(0.01, 0.3, 128)        # all positive: min forced to 0
    w[:, 128:] = -np.linspace(0.01, 0.3, 128)       # all negative: max forced to 0
    codes, s, zeros = O.quantize_int2(w)
    z = O.unpack_int2_zeros(zeros)
    assert np.all(z[:, 0] == 0) and np.all(z[:, 1] == 3)


def test_int2_crumb_and_zero_tables():
    # all 4 codes x all 4 zeros, codes in every position of the byte
    u = np.tile(np.arange(4, dtype=np.uint8), 32)[None, :].repeat(4, axis=0)   # [4,128]
    codes = (u[:, 0::4] | (u[:, 1::4] << 2) | (u[:, 2::4] << 4) | (u[:, 3::4] << 6)).astype(np.uint8)
    assert codes[0, 0] == 0b11100100
    zrow = np.arange(4, dtype=np.uint8)                                       # row n has zero n
    zeros = (zrow[0::4] | (zrow[1::4] << 2) | (zrow[2::4] << 4) | (zrow[3::4] << 6)).astype(np.uint8)[:, None]
    s = np.full((4, 1), 0.5, np.float16)
    deq = O.dequantize_int2(codes, s, zeros)
    for n in range(4):
        assert np.array_equal(deq[n], (np.arange(128) % 4 - n) * 0.5)


def test_int2_error_bound():
    rng = np.random.default_rng(2)
    w = (rng.standard_normal((64, 384)) * 0.02).astype(np.float32)
    codes, s, zeros = O.quantize_int2(w)
    deq = O.dequantize_int2(codes, s, zeros)
    sf = np.repeat(s.astype(np.float64), 128, axis=1)
    g = w.reshape(64, 3, 128)
    lo = np.repeat(np.minimum(g.min(axis=2), 0), 128, axis=1)
    hi = np.repeat(np.maximum(g.max(axis=2), 0), 128, axis=1)
    inside = (w >= lo) & (w <= hi)
    err = np.abs(w - deq)
    # inside the representable range [(0-z)s, (3-z)s] the error is <= s/2; the
    # range itself can miss [min,max] by the rounding of z and of the scale
    zf = np.repeat(O.unpack_int2_zeros(zeros).astype(np.float64), 128, axis=1)
    rep = (w >= -zf * sf) & (w <= (3 - zf) * sf)
    assert np.all(err[inside & rep] <= sf[inside & rep] * 0.5 * (1 + 2.0 ** -8))
    assert np.all(err[inside] <= sf[inside] * 1.0 + 1e-12)


# ------------------------------------------------------------ FP8 / FP4 ----

def test_e4m3_decode_matches_torch_all_bytes():
    b = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = O.e4m3_decode(np.arange(256, dtype=np.uint8))
    assert np.array_equal(np.isnan(ref), np.isnan(mine))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], mine[ok])
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9 and mine[0x38] == 1.0


def test_e4m3_rounding_matches_torch():
    rng = np.random.default_rng(3)
    finite = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))          # 0 .. 448 ascending
    mids = ((finite[1:] + finite[:-1]) / 2).astype(np.float32)       # exact ties
    rnd = np.exp2(rng.uniform(-12, 9.5, 20000)).astype(np.float32)
    v = np.concatenate([finite.astype(np.float32), mids, rnd, np.float32([0.0, 1e-30, 500.0, 1e6])])
    v = np.concatenate([v, -v])
    mine = O.e4m3_rne_satfinite(v)
    clamped = torch.from_numpy(np.clip(v, -448, 448))
    ref = clamped.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    nz = O.e4m3_decode(ref) != 0                                      # torch may drop -0 sign
    assert np.array_equal(mine[nz], ref[nz])
    assert np.all(O.e4m3_decode(mine[~nz]) == 0)


def test_e2m1_grid_and_midpoints():
    vals = O.e2m1_decode(np.arange(16, dtype=np.uint8))
    assert list(vals[:8]) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    assert list(vals[8:]) == [-0.0, -0.5, -1, -1.5, -2, -3, -4, -6]
    mid = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6, 6.0: 7, 7.0: 7, 100.0: 7}
    for v, c in mid.items():
        assert O.e2m1_rne_satfinite(np.float32(v)) == c, v
        assert O.e2m1_rne_satfinite(np.float32(-v)) == c | 8, -v
    # every grid value round-trips
    assert np.array_equal(O.e2m1_rne_satfinite(vals.astype(np.float32)), np.arange(16))


def test_nvfp4_worked_blocks(golden):
    g = golden["nvfp4"]
    w = np.zeros((3, 32), np.float32)
    w[0, :16] = g["blocks"][0]["values"]
    w[1, :16] = g["blocks"][1]["values"]
    w[2, 20] = g["matrix_amax"]
    gs = O.nvfp4_global_scale(np.abs(w).max())
    assert gs == np.float32(g["global_scale"])
    codes, sb = O.quantize_nvfp4(w, gs)
    q = O.unpack_nvfp4(codes)
    for r in range(2):
        blk = g["blocks"][r]
        assert sb[r, 0] == blk["block_scale_byte"]
        assert O.e4m3_decode(sb[r, 0]) == blk["block_scale"]
        assert list(q[r, :16]) == blk["codes"]
    deq = O.dequantize_nvfp4(codes, sb, gs)
    assert deq[2, 20] == 2688.0


def test_nvfp4_error_bound_random():
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((32, 256)) * 0.02).astype(np.float32)
    gs = O.nvfp4_global_scale(np.abs(w).max())
    codes, sb = O.quantize_nvfp4(w, gs)
    deq = O.dequantize_nvfp4(codes, sb, gs)
    unit = np.repeat(O.e4m3_decode(sb) * float(gs), 16, axis=1)
    # worst grid spacing is 2 (in [4, 6]) -> error <= 1 unit, plus scale rounding
    assert np.all(np.abs(w - deq) <= unit * 1.0 + 1e-12)
    amax_b = np.abs(w.reshape(32, 16, 16)).max(axis=2)
    # the block scale maps the block amax near the top of the E2M1 range
    ratio = amax_b / (O.e4m3_decode(sb) * float(gs))
    assert np.all((ratio > 6 / 1.07) & (ratio < 6 * 1.07))


def test_output_tolerance_discounts_only_the_bf16_rounding():
    """The comparison helper of the GPU tests: the exact result rounded to
    bf16 always passes, whatever its magnitude; one bf16 ulp more than that
    at an output of 9 x RMS fails."""
    import torch
    from tests.gpu_util import assert_close_output, bf16_rounding_error
    rng = np.random.default_rng(3)
    y = rng.standard_normal((64, 256))
    y[5, 7] = 9.0 * np.sqrt(np.mean(y ** 2)) * 1.0009765625        # a large output just above a bf16 binade start
    bits = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert_close_output(bits, y)
    assert bf16_rounding_error(y).max() > 0
    bad = bits.copy()
    bad[5, 7] += 4                                   # four ulps off at 9 x RMS: about 7 % of the RMS
    with pytest.raises(AssertionError):
        assert_close_output(bad, y)
