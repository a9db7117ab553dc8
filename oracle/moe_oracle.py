"""Plain CPU oracle for the routed-expert MoE layer with low-bit expert weights.

TEST INFRASTRUCTURE ONLY.  This module is the slow, obviously correct
reference that the CUDA path is checked against.  Only the test suite, the
smoke check of ``__graft_entry__`` and the ``cpu_baseline`` / reference leg
of ``bench.py`` may import it.  It shares no code with the CUDA library and
imports nothing from it.

What it computes, and where each step comes from
-------------------------------------------------
The pages describe a sparse MoE LLM whose routed experts are stored with
low-bit group quantization and whose routers stay 16-bit:

* "Qwen3.8-Flash-Next on one 24 GB GPU", section "What the patch does":
  ten experts of 512 are selected per layer per token; experts are 2-bit with
  group size 128 (section "Hardware and software requirements").
* "Qwen3.8-Flash-Next on 2x RTX 3090", storage-format table, and
  "albucino/Qwen3.8-Flash-Next-W4A16-FP8PLE", section "Composition": routed
  experts are W4A16, symmetric INT4, group 128.
* "Qwen3.8-Flash-Next on 2x RTX 3090", storage-format table, and
  "albucino/Qwen3.8-Flash-Next-W4A16-FP8PLE", section "Composition": the
  routed experts of the MTP draft are symmetric INT4 with group 32 (the same
  recipe with one scale per 32 inputs).
* "Qwen3.8-Flash-Next-FP6-INT8", introduction and section "Quantization
  quality": routed experts in fp6 e2m3 with fp16 scales.  Readings: the OCP
  MX FP6 E2M3 element (1 sign, 2 exponent bits with bias 1, 3 mantissa bits;
  magnitudes m/8 below 1, 2^(e-1) (1 + m/8) above, at most 7.5), one fp16
  scale per 32 inputs (6.5 bits per weight, as the card's bit budget),
  s = fp16(amax / 7.5) and q = e2m3(w / s) rounded half-to-even, saturating.
* "meshapplied/Qwen3.8-Flash-Next-NVFP4-Latest", section "Format": the
  MTP-draft routed experts are FP8 with 128x128 block scales (E4M3FN codes,
  one fp32 scale per 128 rows x 128 inputs; reading: s = amax/448).
* "meshapplied/Qwen3.8-Flash-Next-NVFP4-Latest", section "Format": routed
  experts are NVFP4 W4A4 (E2M1 values, one scale per 16 elements); the
  shared experts stay BF16.
* "Qwen3.8-Flash-Next-FP6-INT8", section "Precision map": routers stay bf16
  (near-tie routing decisions), activations bf16, accumulation fp32.

Readings taken where the pages are silent (each is listed in the design
notes of the repository):

* INT4: s = fp16(amax/7); q = clamp(rne(w/s), -8, 7); stored u = q + 8.
* INT2: asymmetric with a 2-bit zero per group: s = fp16((max-min)/3) with
  min <= 0 <= max forced; z = clamp(rne(-min/s), 0, 3);
  u = clamp(rne(w/s) + z, 0, 3).
* NVFP4: one fp32 global scale g = amax/(6*448) per matrix (gate and up
  share one); per 16-block s_b = e4m3(amax_b/(6 g)); q = e2m1(w / (s_b g)).
  Activations use the same recipe per row with a static global scale.
* Every rounding is round-half-to-even; every decision that yields an
  integer code is taken in IEEE fp32, as the CUDA kernels take it.
* Top-k orders by (logit descending, expert index ascending); the k
  weights are the softmax over the selected logits (softmax over all
  experts followed by renormalisation over the selected ones is the same
  quantity in exact arithmetic).
* Expert MLP is SwiGLU: a = silu(x W_gate^T) * (x W_up^T); o = a W_down^T.
* y_t = sum_j w_tj o_tj + shared(x_t); the shared expert has no gate.

Precision: quantization decisions are fp32 (as above); dequantized weights,
matrix products, softmax and combine are fp64.  Arrays of bf16 values are
passed around as their uint16 bit patterns.
"""
from __future__ import annotations

import numpy as np

GROUP_INT = 128      # INT4 / INT2 group size along K
GROUP_INT4_G32 = 32  # INT4 group size of the MTP-draft experts
GROUP_FP4 = 16       # NVFP4 block size along K
BLOCK_FP8 = 128      # FP8 experts: one scale per 128 x 128 block
GROUP_FP6 = 32       # FP6 e2m3 experts: one fp16 scale per 32 inputs
E2M3_MAX = 7.5
E4M3_MAX = 448.0
E2M1_MAX = 6.0

# --------------------------------------------------------------------------
# Number formats
# --------------------------------------------------------------------------


def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def fp16_rne(v) -> np.ndarray:
    """IEEE binary16 round-to-nearest-even of fp32 values."""
    return np.asarray(v, dtype=np.float32).astype(np.float16)


def e4m3_decode(byte) -> np.ndarray:
    """FP8 E4M3FN byte -> float64: 1 sign, 4 exponent (bias 7), 3 mantissa
    bits; exponent 0 is subnormal (m/8 * 2^-6); 0x7F/0xFF are NaN; no inf."""
    b = np.asarray(byte, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    val = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def _rne_to_grid(a: np.ndarray, quantum: np.ndarray) -> np.ndarray:
    # a / quantum is exact (quantum is a power of two), rint is half-even
    return np.rint(a / quantum) * quantum


def e4m3_rne_satfinite(v) -> np.ndarray:
    """fp32 -> FP8 E4M3FN byte, round-half-to-even, saturating to +-448.

    A value is first clamped to the finite range, then rounded on the grid
    of its binade: quantum 2^(e-3) for |v| in [2^e, 2^(e+1)), e >= -6, and
    2^-9 below 2^-6 (subnormals).  Negative inputs keep their sign bit."""
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(v), E4M3_MAX)
    _, ex = np.frexp(a)                       # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)                # binade exponent, floored at -6
    q = _rne_to_grid(a, np.exp2(e - 3.0))
    q = np.minimum(q, E4M3_MAX)
    # encode the (exactly representable) magnitude q
    _, qx = np.frexp(q)
    qe = qx - 1                               # q in [2^qe, 2^(qe+1))
    normal = q >= 2.0 ** -6
    with np.errstate(divide="ignore", invalid="ignore"):
        m_norm = np.where(normal, (q / np.exp2(qe.astype(np.float64)) - 1.0) * 8.0, 0.0)
    mag = np.where(normal,
                   ((qe + 7).astype(np.int64) << 3) | m_norm.astype(np.int64),
                   (q / 2.0 ** -9).astype(np.int64))
    sign = np.signbit(v).astype(np.int64) << 7
    return (mag | sign).astype(np.uint8)


E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(code) -> np.ndarray:
    """FP4 E2M1 nibble -> float64: bit 3 sign, bits 0-2 index the magnitude
    grid {0, 0.5, 1, 1.5, 2, 3, 4, 6}."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    mag = E2M1_GRID[c & 7]
    return np.where(c & 8, -mag, mag)


def e2m1_rne_satfinite(v) -> np.ndarray:
    """fp32 -> E2M1 nibble, round-half-to-even, saturating to +-6.
    Grid spacing is 0.5 below 2, 1 in [2, 4) and 2 from 4 up."""
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(v), E2M1_MAX)
    quantum = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    q = np.minimum(_rne_to_grid(a, quantum), E2M1_MAX)
    idx = np.searchsorted(E2M1_GRID, q)       # q lies exactly on the grid
    sign = np.signbit(v).astype(np.int64) << 3
    return (idx | sign).astype(np.uint8)


# --------------------------------------------------------------------------
# Weight formats (interchange layout)
#   A matrix W is [N, K] (output rows, input columns); groups run along K.
#   INT4 : codes uint8 [N, K/2], element k=2j in the low nibble of byte j;
#          scales fp16 [N, K/128] (group 32: [N, K/32]).
#   INT2 : codes uint8 [N, K/4], element k=4j+i at bits 2i..2i+1;
#          scales fp16 [N, K/128]; zeros uint8 [N/4, K/128], the zero of
#          row n at bits 2(n%4) of byte (n//4, group).
#   NVFP4: codes uint8 [N, K/2] (low nibble = even k); block scales E4M3
#          bytes [N, K/16]; one fp32 global scale.
#   FP8  : codes E4M3FN bytes [N, K]; scales fp32 [N/128, K/128].
#   FP6  : codes e2m3 [N, K], one per byte (bits 0-5: sign at bit 5, exponent
#          bits 3-4, mantissa bits 0-2); scales fp16 [N, K/32].
# --------------------------------------------------------------------------


def quantize_int4(w, group=GROUP_INT):
    """Symmetric INT4, group 128 (W4A16 experts) or 32 (MTP-draft experts)."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % group == 0
    g = w.reshape(N, K // group, group)
    amax = np.abs(g).max(axis=2)
    s16 = fp16_rne(amax / np.float32(7.0))
    s = s16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint(g / s)
    q = np.where(s == 0, 0.0, np.clip(q, -8, 7))
    u = (q + 8).astype(np.uint8).reshape(N, K)
    codes = (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)
    return codes, s16


def unpack_int4(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    N, Kh = c.shape
    u = np.empty((N, 2 * Kh), dtype=np.uint8)
    u[:, 0::2] = c & 0xF
    u[:, 1::2] = c >> 4
    return u


def dequantize_int4(codes, scales) -> np.ndarray:
    """(u - 8) * s; the group size is K over the number of scales per row."""
    u = unpack_int4(codes).astype(np.float64)
    N, K = u.shape
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)
    group = K // s.shape[1]
    return ((u - 8.0).reshape(N, K // group, group) * s[..., None]).reshape(N, K)


def quantize_int2(w):
    """Asymmetric INT2, group 128, fp16 scale and 2-bit zero per group."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % GROUP_INT == 0 and N % 4 == 0
    g = w.reshape(N, K // GROUP_INT, GROUP_INT)
    mn = np.minimum(g.min(axis=2), np.float32(0))
    mx = np.maximum(g.max(axis=2), np.float32(0))
    s16 = fp16_rne((mx - mn) / np.float32(3.0))
    s = s16.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        z = np.where(s == 0, 0.0, np.clip(np.rint(-mn / s), 0, 3))
        u = np.where(s[..., None] == 0, 0.0,
                     np.clip(np.rint(g / s[..., None]) + z[..., None], 0, 3))
    u = u.astype(np.uint8).reshape(N, K)
    codes = (u[:, 0::4] | (u[:, 1::4] << 2) | (u[:, 2::4] << 4) | (u[:, 3::4] << 6)).astype(np.uint8)
    z = z.astype(np.uint8)
    zeros = (z[0::4] | (z[1::4] << 2) | (z[2::4] << 4) | (z[3::4] << 6)).astype(np.uint8)
    return codes, s16, zeros


def unpack_int2(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    N, Kq = c.shape
    u = np.empty((N, 4 * Kq), dtype=np.uint8)
    for i in range(4):
        u[:, i::4] = (c >> (2 * i)) & 3
    return u


def unpack_int2_zeros(zeros) -> np.ndarray:
    zb = np.asarray(zeros, dtype=np.uint8)
    Nq, G = zb.shape
    z = np.empty((4 * Nq, G), dtype=np.uint8)
    for i in range(4):
        z[i::4] = (zb >> (2 * i)) & 3
    return z


def dequantize_int2(codes, scales, zeros) -> np.ndarray:
    u = unpack_int2(codes).astype(np.float64)
    N, K = u.shape
    z = unpack_int2_zeros(zeros).astype(np.float64)
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)
    ug = u.reshape(N, K // GROUP_INT, GROUP_INT)
    return ((ug - z[..., None]) * s[..., None]).reshape(N, K)


def nvfp4_global_scale(amax) -> np.float32:
    """fp32 global scale that maps the largest magnitude onto 6 * 448."""
    return np.float32(np.float32(amax) / np.float32(E2M1_MAX * E4M3_MAX))


def quantize_nvfp4(w, g):
    """NVFP4 with a given fp32 global scale g: rows of [N, K] in blocks of 16."""
    w = np.asarray(w, dtype=np.float32)
    g = np.float32(g)
    N, K = w.shape
    assert K % GROUP_FP4 == 0
    b = w.reshape(N, K // GROUP_FP4, GROUP_FP4)
    if g == 0:
        return np.zeros((N, K // 2), np.uint8), np.zeros((N, K // GROUP_FP4), np.uint8)
    amax_b = np.abs(b).max(axis=2)
    sb = e4m3_rne_satfinite(amax_b / (np.float32(E2M1_MAX) * g))
    sbv = e4m3_decode(sb).astype(np.float32)
    with np.errstate(divide="ignore"):
        r = np.where(sbv == 0, np.float32(0), np.float32(1.0) / (sbv * g)).astype(np.float32)
    q = e2m1_rne_satfinite(b * r[..., None]).reshape(N, K)
    codes = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    return codes, sb


def e2m3_decode(code) -> np.ndarray:
    """FP6 E2M3 code (6 bits) -> float64: exponent 0 is m/8, else
    2^(e-1) * (1 + m/8)."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    e = (c >> 3) & 3
    m = c & 7
    mag = np.where(e == 0, m / 8.0, np.exp2(e - 1.0) * (1.0 + m / 8.0))
    return np.where(c & 0x20, -mag, mag)


def e2m3_rne_satfinite(v) -> np.ndarray:
    """fp32 -> FP6 E2M3 code, round-half-to-even, saturating to +-7.5.  The
    grid spacing is 1/8 below 2 (subnormals and exponent 1), 1/4 in [2, 4)
    and 1/2 in [4, 7.5].  Negative inputs keep their sign bit."""
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(v), E2M3_MAX)
    quantum = np.where(a < 2.0, 0.125, np.where(a < 4.0, 0.25, 0.5))
    q = np.minimum(_rne_to_grid(a, quantum), E2M3_MAX)
    # encode the exactly representable magnitude q
    e = np.where(q < 1.0, 0, np.where(q < 2.0, 1, np.where(q < 4.0, 2, 3)))
    m = np.where(e == 0, q * 8.0, (q / np.exp2(e - 1.0) - 1.0) * 8.0)
    code = (e << 3) | m.astype(np.int64)
    return (code | (np.signbit(v).astype(np.int64) << 5)).astype(np.uint8)


def quantize_fp6(w):
    """FP6 E2M3 with one fp16 scale per 32 inputs: s = fp16(amax/7.5) and
    q = e2m3(w / s) (IEEE fp32 division); an all-zero group has s = 0 and
    codes of +-0."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % GROUP_FP6 == 0
    g = w.reshape(N, K // GROUP_FP6, GROUP_FP6)
    amax = np.abs(g).max(axis=2)
    s16 = fp16_rne(amax / np.float32(E2M3_MAX))
    s = s16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s == 0, g * np.float32(0.0), g / s).astype(np.float32)
    return e2m3_rne_satfinite(v).reshape(N, K), s16


def dequantize_fp6(codes, scales) -> np.ndarray:
    q = e2m3_decode(codes)
    N, K = q.shape
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)
    return (q.reshape(N, K // GROUP_FP6, GROUP_FP6) * s[..., None]).reshape(N, K)


def quantize_fp8_block(w):
    """FP8 E4M3FN with one fp32 scale per 128 x 128 block (MTP-draft experts):
    s = amax_block / 448 and q = e4m3(w / s), both divisions IEEE fp32; an
    all-zero block has s = 0 and codes of +-0."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    B = BLOCK_FP8
    assert N % B == 0 and K % B == 0
    b = w.reshape(N // B, B, K // B, B)
    amax = np.abs(b).max(axis=(1, 3)).astype(np.float32)            # [N/B, K/B]
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    sb = s[:, None, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(sb == 0, b * np.float32(0.0), b / sb).astype(np.float32)
    codes = e4m3_rne_satfinite(v).reshape(N, K)
    return codes, s


def dequantize_fp8_block(codes, scales) -> np.ndarray:
    q = e4m3_decode(codes)
    N, K = q.shape
    B = BLOCK_FP8
    s = np.asarray(scales, dtype=np.float32).astype(np.float64)
    return (q.reshape(N // B, B, K // B, B) * s[:, None, :, None]).reshape(N, K)


def unpack_nvfp4(codes) -> np.ndarray:
    return unpack_int4(codes)            # same nibble order


def dequantize_nvfp4(codes, block_scales, g) -> np.ndarray:
    q = e2m1_decode(unpack_nvfp4(codes))
    N, K = q.shape
    sb = e4m3_decode(block_scales)
    return (q.reshape(N, K // GROUP_FP4, GROUP_FP4) * sb[..., None] * np.float64(np.float32(g))).reshape(N, K)


def quantize_nvfp4_rows(x_f32, g):
    """Activation quantization (W4A4): each row of x with the static global
    scale g; returns codes, block scales and the dequantized fp64 rows."""
    codes, sb = quantize_nvfp4(x_f32, g)
    return codes, sb, dequantize_nvfp4(codes, sb, g)


# --------------------------------------------------------------------------
# Routing
# --------------------------------------------------------------------------


def router_logits(x_bits, wr_bits) -> np.ndarray:
    """logits[t, e] = sum_k x[t,k] * Wr[e,k] with bf16 inputs, fp64 sums."""
    return bf16_bits_to_f64(x_bits) @ bf16_bits_to_f64(wr_bits).T


def route_topk(logits, k):
    """Top-k experts per token and their renormalised softmax weights.

    Order: logit descending, expert index ascending on equal logits.
    w_j = exp(l_j - l_max) / sum_{selected} exp(l - l_max)."""
    L = np.asarray(logits)
    T, E = L.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    idx = np.arange(E)
    for t in range(T):
        lt = L[t].astype(np.float64)
        order = np.lexsort((idx, -lt))[:k]     # primary key: -logit
        ids[t] = order
        ex = np.exp(lt[order] - lt[order[0]])
        w[t] = ex / ex.sum()
    return ids, w


def permute(ids, num_experts):
    """Expert-major order of the flat slots s = t*k + j, stable in s.

    Returns counts[E], offsets[E+1], perm[T*k] (slot id at each permuted
    position) and inv[T*k] (permuted position of each slot).  A slot whose
    id lies outside [0, E) selects no expert: it is left out of the order
    and its inv entry is -1; perm then has only offsets[E] meaningful
    entries (the rest are -1)."""
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    valid = (flat >= 0) & (flat < num_experts)
    counts = np.bincount(flat[valid], minlength=num_experts).astype(np.int32)
    offsets = np.zeros(num_experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    fill = offsets[:-1].astype(np.int64).copy()
    perm = np.full(flat.size, -1, dtype=np.int32)
    inv = np.full(flat.size, -1, dtype=np.int32)
    for s, e in enumerate(flat):
        if not valid[s]:
            continue
        perm[fill[e]] = s
        inv[s] = fill[e]
        fill[e] += 1
    return counts, offsets, perm, inv


# --------------------------------------------------------------------------
# Experts and the layer
# --------------------------------------------------------------------------


def silu(z):
    return z / (1.0 + np.exp(-z))


def swiglu_intermediate(X, Wg, Wu):
    return silu(X @ Wg.T) * (X @ Wu.T)


def dequantize_expert(quant, ew):
    """Expert weights in interchange form -> fp64 (W_gate, W_up, W_down).

    ``ew`` maps 'gate'/'up'/'down' to dicts with keys codes, scales and,
    for INT2, zeros, for NVFP4, g.  quant is 'int4', 'int4g32', 'int2', 'nvfp4', 'fp8', 'fp6' or
    'bf16' (codes are then bf16 bit patterns)."""
    out = []
    for name in ("gate", "up", "down"):
        m = ew[name]
        if quant in ("int4", "int4g32"):
            out.append(dequantize_int4(m["codes"], m["scales"]))
        elif quant == "int2":
            out.append(dequantize_int2(m["codes"], m["scales"], m["zeros"]))
        elif quant == "nvfp4":
            out.append(dequantize_nvfp4(m["codes"], m["scales"], m["g"]))
        elif quant == "fp8":
            out.append(dequantize_fp8_block(m["codes"], m["scales"]))
        elif quant == "fp6":
            out.append(dequantize_fp6(m["codes"], m["scales"]))
        elif quant == "bf16":
            out.append(bf16_bits_to_f64(m["codes"]))
        else:
            raise ValueError(quant)
    return tuple(out)


def moe_forward(x_bits, ids, w, quant, expert_fn, shared=None, act_scales=None, num_experts=None):
    """MoE layer output y [T, H] in fp64.

    x_bits     bf16 bit patterns [T, H]
    ids, w     routing [T, k] (expert ids, weights); with num_experts given,
               a slot whose id lies outside [0, num_experts) selects no
               expert and contributes zero
    expert_fn  e -> fp64 (W_gate [I,H], W_up [I,H], W_down [H,I])
    shared     None or fp64 (W_gate, W_up, W_down) of the always-on expert
    act_scales (g_x, g_a) static global scales for NVFP4 activations and
               intermediates (W4A4); ignored otherwise."""
    X = bf16_bits_to_f64(x_bits)
    T, H = X.shape
    ids = np.asarray(ids)
    w = np.asarray(w, dtype=np.float64)
    if quant == "nvfp4":
        g_x, g_a = act_scales
        _, _, Xq = quantize_nvfp4_rows(X.astype(np.float32), g_x)
    else:
        Xq = X
    y = np.zeros((T, H), dtype=np.float64)
    for e in np.unique(ids):
        if num_experts is not None and not 0 <= e < num_experts:
            continue
        tok, slot = np.nonzero(ids == e)
        Wg, Wu, Wd = expert_fn(int(e))
        A = swiglu_intermediate(Xq[tok], Wg, Wu)
        if quant == "nvfp4":
            _, _, A = quantize_nvfp4_rows(A.astype(np.float32), g_a)
        O = A @ Wd.T
        y[tok] += w[tok, slot][:, None] * O
    if shared is not None:
        Wg, Wu, Wd = shared
        y += swiglu_intermediate(X, Wg, Wu) @ Wd.T
    return y


def intermediate_amax(x_bits, ids, quant, expert_fn, act_scale_x=None):
    """Largest |a| over all routed slots (calibration of the NVFP4
    intermediate global scale); a is computed as in moe_forward."""
    X = bf16_bits_to_f64(x_bits)
    if quant == "nvfp4":
        _, _, X = quantize_nvfp4_rows(X.astype(np.float32), act_scale_x)
    amax = 0.0
    for e in np.unique(ids):
        tok, _ = np.nonzero(np.asarray(ids) == e)
        Wg, Wu, _ = expert_fn(int(e))
        amax = max(amax, float(np.abs(swiglu_intermediate(X[tok], Wg, Wu)).max()))
    return amax
