// Device helpers shared by the MoE kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define MOE_DEV __device__ __forceinline__

namespace moe {

constexpr int kWarp = 32;

// ---------------------------------------------------------------- reductions
MOE_DEV float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
MOE_DEV float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
MOE_DEV float warp_min(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// ---------------------------------------------------------------- bf16 bits
MOE_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
MOE_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
MOE_DEV float bf16_to_f(__nv_bfloat16 h) { return __bfloat162float(h); }

// Two fp32 -> packed bf16x2 (round to nearest even); lo goes to the low half.
MOE_DEV uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ------------------------------------------------------------- fp8 / fp4 cvt
// fp32 -> E4M3FN byte, round to nearest even, saturating to +-448.
MOE_DEV uint32_t f32_to_e4m3(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return r & 0xffu;
}
// E4M3FN byte -> fp32 (exact).
MOE_DEV float e4m3_to_f32(uint32_t b) {
    uint32_t h2;
    uint16_t in = (uint16_t)(b & 0xffu);
    asm("{ .reg .b16 t; mov.b16 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
}
// fp32 -> FP6 E2M3 code (sign bit 5), round half to even, saturating to
// +-7.5: rounded on the grid of its binade (1/8 below 2, 1/4 in [2, 4), 1/2
// above); the scalings by powers of two are exact.
MOE_DEV uint32_t f32_to_e2m3(float v) {
    const float a = fminf(fabsf(v), 7.5f);
    const float inv_q = a < 2.0f ? 8.0f : (a < 4.0f ? 4.0f : 2.0f);
    const float q = fminf(rintf(a * inv_q) / inv_q, 7.5f);
    uint32_t e, m;
    if (q < 1.0f) { e = 0; m = (uint32_t)(q * 8.0f); }
    else if (q < 2.0f) { e = 1; m = (uint32_t)((q - 1.0f) * 8.0f); }
    else if (q < 4.0f) { e = 2; m = (uint32_t)((q * 0.5f - 1.0f) * 8.0f); }
    else { e = 3; m = (uint32_t)((q * 0.25f - 1.0f) * 8.0f); }
    return (signbit(v) ? 0x20u : 0u) | (e << 3) | m;
}
// Two e2m3 codes given as their low nibbles (bits 0-3 of each 16-bit half)
// and high crumbs (bits 0-1 of each half) -> fp16x2 bits of e2m3 * 2^-14:
// the mantissa and exponent bits land in the fp16 fields unchanged, so
// exponent 0 becomes an fp16 subnormal with the same 2^-14 ratio (exact)
MOE_DEV uint32_t e2m3x2_to_f16x2_scaled(uint32_t nib, uint32_t cr) {
    return (nib << 7) | ((cr & 0x00010001u) << 11) | ((cr & 0x00020002u) << 14);
}
// Two E4M3FN bytes (the low one first) -> fp16x2 (exact)
MOE_DEV uint32_t e4m3x2_to_f16x2(uint32_t two) {
    uint32_t h2;
    const uint16_t in = (uint16_t)(two & 0xffffu);
    asm("{ .reg .b16 t; mov.b16 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h2) : "h"(in));
    return h2;
}
// Two fp32 -> two E2M1 nibbles (lo in bits 0-3), RNE, saturating to +-6.
MOE_DEV uint32_t f32x2_to_e2m1(float lo, float hi) {
    uint32_t r;
    asm("{ .reg .b8 b0, b1, b2, b3;\n"
        "  cvt.rn.satfinite.e2m1x2.f32 b0, %1, %2;\n"
        "  mov.b32 %0, {b0, b1, b2, b3}; }"
        : "=r"(r) : "f"(hi), "f"(lo));
    return r & 0xffu;
}
// E2M1 code (low nibble) -> fp32 value (exact).
MOE_DEV float e2m1_to_f32(uint32_t c) {
    // magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 scaled by 2 fit in a nibble each
    const uint32_t twice = 0xC8643210u;   // nibble i = 2 * magnitude(i)
    float m = 0.5f * (float)((twice >> (4 * (c & 7u))) & 0xfu);
    return (c & 8u) ? -m : m;
}

// ------------------------------------------------------ NVFP4 block of 16
// The one NVFP4 quantizer of the library ("meshapplied/Qwen3.8-Flash-Next-
// NVFP4-Latest", section "Format": E2M1 values with one E4M3 scale per 16):
// with the fp32 global scale g, the scale code is e4m3(amax / (6 g)) and the
// codes are e2m1(v * r) with r = 1 / (s_b g), every decision in fp32 with
// IEEE division.  A block whose scale decodes to zero has r = 0, so its codes
// are signed zeros (0x8 for negative inputs, as an IEEE conversion gives);
// g == 0 gives scale code 0 and all-zero codes.  Returns the scale code;
// w[0] holds elements 0..7 and w[1] elements 8..15, element 2i in the low
// nibble of byte i.  The weight quantizer, the activation quantizers of the
// prefill and decode paths and the W4A4 value staging all call this.
MOE_DEV uint32_t nvfp4_quant_block16(const float (&v)[16], float g, uint32_t (&w)[2]) {
    w[0] = w[1] = 0u;
    if (g == 0.0f) return 0u;
    float amax = 0.0f;
#pragma unroll
    for (int q = 0; q < 16; ++q) amax = fmaxf(amax, fabsf(v[q]));
    const uint32_t sbc = f32_to_e4m3(__fdiv_rn(amax, __fmul_rn(6.0f, g)));
    const float sbv = e4m3_to_f32(sbc);
    const float r = (sbv == 0.0f) ? 0.0f : __fdiv_rn(1.0f, __fmul_rn(sbv, g));
#pragma unroll
    for (int q = 0; q < 8; ++q)
        w[q >> 2] |= f32x2_to_e2m1(__fmul_rn(v[2 * q], r), __fmul_rn(v[2 * q + 1], r)) << (8 * (q & 3));
    return sbc;
}
// The values q * s_b of the block quantized as above (the global scale g is
// left to the caller), in place.
MOE_DEV void nvfp4_block16_values(float (&v)[16], float g) {
    uint32_t w[2];
    const float sbv = e4m3_to_f32(nvfp4_quant_block16(v, g, w));
#pragma unroll
    for (int q = 0; q < 16; ++q) v[q] = e2m1_to_f32((w[q >> 3] >> (4 * (q & 7))) & 0xFu) * sbv;
}

// ------------------------------------------------------------ memory access
MOE_DEV uint4 ldg_nc_v4(const void* p) {
    uint4 r;
    asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}
MOE_DEV uint4 ldg_stream_v4(const void* p) {   // read once: do not keep in L1
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

// Programmatic dependent launch: wait for the previous grid's results / let
// the next grid start its prologue.
MOE_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
MOE_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Ticket of a grid-wide "last one finishes" pattern, taken by one thread
// after a CTA barrier: the add releases this CTA's earlier writes (ordered
// before it by the barrier) and acquires those released by the tickets
// before it (visible to the CTA after the next barrier).  Returns the count
// before the add.
MOE_DEV unsigned ticket_acq_rel(unsigned* p) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
    return old;
}

// ------------------------------------------------ packed codes -> bf16x2
// Exact conversions of two codes of a packed word into a bf16 pair (low
// half = the first column), shared by the GEMV and the grouped GEMM.
MOE_DEV uint32_t hsub2_bits(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}
MOE_DEV uint32_t hmul2_bits(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}
MOE_DEV uint32_t bf16x2_splat(float v) {
    const uint32_t h = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
    return h | (h << 16);
}
// INT4 pair j of a word: bf16x2 (u - 8), exact
MOE_DEV uint32_t int4_pair(uint32_t w, int j) {
    return hsub2_bits(((w >> (4 * j)) & 0x000F000Fu) | 0x43004300u, 0x43084308u);   // (128+u) - 136
}
// INT2 pair j of a word: bf16x2 (u - z), exact; off = bf16x2(128 + z)
MOE_DEV uint32_t int2_pair(uint32_t w, int j, uint32_t off) {
    return hsub2_bits(((w >> (2 * j)) & 0x00030003u) | 0x43004300u, off);
}
// E2M1 pair j of a word times the block scale (bf16x2 splat), exact:
// the codes placed at bf16 bits [8:6] (magnitude) and 15 (sign) read as
// e2m1 * 2^-126; one multiply by 2^126 and one by the scale.
MOE_DEV uint32_t fp4_pair(uint32_t w, int j, uint32_t sb2) {
    const uint32_t t = w >> (4 * j);
    const uint32_t b = ((t & 0x00070007u) << 6) | ((t & 0x00080008u) << 12);
    return hmul2_bits(hmul2_bits(b, 0x7E807E80u), sb2);       // 0x7E80 = 2^126
}


}  // namespace moe
