// Weight and activation quantization, and the re-layout between the
// interchange format and the tiled device layout (see layout.cuh).
//
// Formats (every code decision in IEEE fp32, round-half-to-even):
//   INT4 symmetric group-128 ("albucino/Qwen3.8-Flash-Next-W4A16-FP8PLE",
//        "Composition"): s = fp16(amax/7), u = clamp(rne(w/s), -8, 7) + 8.
//   INT2 group-128 with fp16 scale and 2-bit zero ("Qwen3.8-Flash-Next on
//        one 24 GB GPU", "Hardware and software requirements"; asymmetric
//        reading): s = fp16((max-min)/3) with min <= 0 <= max,
//        z = clamp(rne(-min/s), 0, 3), u = clamp(rne(w/s) + z, 0, 3).
//   NVFP4 ("meshapplied/Qwen3.8-Flash-Next-NVFP4-Latest", "Format": E2M1,
//        group 16): s_b = e4m3(amax_b / (6 g)), q = e2m1(w / (s_b g)).
#include "common.cuh"
#include "kernels.h"
#include "layout.cuh"

namespace moe {

// ------------------------------------------------------------------ INT4
// One warp per 128 consecutive values of a row (four per lane); a group of
// `group` values (128 or 32) is held by group/4 consecutive lanes.
__global__ void k_quantize_int4(const float* __restrict__ w, int N, int K, int group,
                                uint8_t* __restrict__ codes, __half* __restrict__ scales) {
    const int C = K / 128, G = K / group, lpg = group / 4;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= N * C) return;
    const int n = warp / C, ch = warp % C;
    const int g = (ch * 128 + lane * 4) / group;
    const float4 v = *reinterpret_cast<const float4*>(w + (size_t)n * K + ch * 128 + lane * 4);
    float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
    for (int o = lpg >> 1; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const __half s = __float2half_rn(__fdiv_rn(amax, 7.0f));
    const float sf = __half2float(s);
    float e[4] = {v.x, v.y, v.z, v.w};
    uint32_t u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float q = (sf == 0.0f) ? 0.0f : fminf(fmaxf(rintf(__fdiv_rn(e[i], sf)), -8.0f), 7.0f);
        u[i] = (uint32_t)((int)q + 8);
    }
    const uint16_t packed = (uint16_t)(u[0] | (u[1] << 4) | (u[2] << 8) | (u[3] << 12));
    *reinterpret_cast<uint16_t*>(codes + (size_t)n * (K / 2) + ch * 64 + lane * 2) = packed;
    if (lane % lpg == 0) scales[(size_t)n * G + g] = s;
}

// ------------------------------------------------------------------- FP6
// One warp per 128 consecutive values of a row (four per lane), groups of 32
// held by 8 lanes: s = fp16(amax / 7.5), code = e2m3(w / s) (IEEE fp32
// division); an all-zero group has s = 0 and codes of +-0.  codes: one
// e2m3 code per byte [N, K]; scales fp16 [N, K/32].
__global__ void k_quantize_fp6(const float* __restrict__ w, int N, int K, uint8_t* __restrict__ codes,
                               __half* __restrict__ scales) {
    const int C = K / 128, G = K / 32;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= N * C) return;
    const int n = warp / C, ch = warp % C;
    const int g = (ch * 128 + lane * 4) / 32;
    const float4 v = *reinterpret_cast<const float4*>(w + (size_t)n * K + ch * 128 + lane * 4);
    float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const __half s = __float2half_rn(__fdiv_rn(amax, 7.5f));
    const float sf = __half2float(s);
    const float e[4] = {v.x, v.y, v.z, v.w};
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) packed |= f32_to_e2m3(sf == 0.0f ? e[i] * 0.0f : __fdiv_rn(e[i], sf)) << (8 * i);
    *reinterpret_cast<uint32_t*>(codes + (size_t)n * K + ch * 128 + lane * 4) = packed;
    if (lane % 8 == 0) scales[(size_t)n * G + g] = s;
}

// ------------------------------------------------------------------- FP8
// One CTA of 256 threads per 128x128 block: s = amax / 448 and the E4M3 code
// of w / s, both divisions IEEE fp32; an all-zero block has s = 0 and codes
// of +-0 (w * 0 keeps the sign).  codes [N, K], scales fp32 [N/128, K/128].
__global__ void __launch_bounds__(256) k_quantize_fp8(const float* __restrict__ w, int N, int K,
                                                      uint8_t* __restrict__ codes, float* __restrict__ scales) {
    __shared__ float red[8];
    const int KB = K / 128;
    const int bn = blockIdx.x / KB, bk = blockIdx.x % KB;
    const int c4 = threadIdx.x & 31, r0 = threadIdx.x >> 5;      // 4 columns, rows r0, r0 + 8, ...
    const float* src = w + (size_t)(bn * 128) * K + bk * 128 + c4 * 4;
    float amax = 0.0f;
    for (int r = r0; r < 128; r += 8) {
        const float4 v = *reinterpret_cast<const float4*>(src + (size_t)r * K);
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    float m = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
    const float s = __fdiv_rn(m, 448.0f);
    for (int r = r0; r < 128; r += 8) {
        const float4 v = *reinterpret_cast<const float4*>(src + (size_t)r * K);
        const float e[4] = {v.x, v.y, v.z, v.w};
        uint32_t packed = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float q = (s == 0.0f) ? e[i] * 0.0f : __fdiv_rn(e[i], s);
            packed |= f32_to_e4m3(q) << (8 * i);
        }
        *reinterpret_cast<uint32_t*>(codes + (size_t)(bn * 128 + r) * K + bk * 128 + c4 * 4) = packed;
    }
    if (threadIdx.x == 0) scales[blockIdx.x] = s;
}

// ------------------------------------------------------------------ INT2
// One warp per (4 rows, 1 group): lanes 8r..8r+7 hold row r, 16 values each.
__global__ void k_quantize_int2(const float* __restrict__ w, int N, int K, uint8_t* __restrict__ codes,
                                __half* __restrict__ scales, uint8_t* __restrict__ zeros) {
    const int G = K / kGroup;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= (N / 4) * G) return;
    const int n4 = warp / G, g = warp % G;
    const int r = lane >> 3, part = lane & 7;
    const int n = n4 * 4 + r;
    const float* src = w + (size_t)n * K + g * kGroup + part * 16;
    float e[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 v = reinterpret_cast<const float4*>(src)[i];
        e[4 * i] = v.x; e[4 * i + 1] = v.y; e[4 * i + 2] = v.z; e[4 * i + 3] = v.w;
    }
    float mn = e[0], mx = e[0];
#pragma unroll
    for (int i = 1; i < 16; ++i) { mn = fminf(mn, e[i]); mx = fmaxf(mx, e[i]); }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    mn = fminf(mn, 0.0f);
    mx = fmaxf(mx, 0.0f);
    const __half s = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), 3.0f));
    const float sf = __half2float(s);
    const float z = (sf == 0.0f) ? 0.0f : fminf(fmaxf(rintf(__fdiv_rn(-mn, sf)), 0.0f), 3.0f);
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float u = (sf == 0.0f) ? 0.0f : fminf(fmaxf(rintf(__fdiv_rn(e[i], sf)) + z, 0.0f), 3.0f);
        packed |= (uint32_t)u << (2 * i);
    }
    *reinterpret_cast<uint32_t*>(codes + (size_t)n * (K / 4) + g * 32 + part * 4) = packed;
    // zero byte of the 4 rows: row r's zero at bits 2r
    uint32_t zb = (part == 0) ? ((uint32_t)z << (2 * r)) : 0u;
    zb |= __shfl_xor_sync(0xffffffffu, zb, 8);
    zb |= __shfl_xor_sync(0xffffffffu, zb, 16);
    if (lane == 0) zeros[(size_t)n4 * G + g] = (uint8_t)zb;
    if (part == 0) scales[(size_t)n * G + g] = s;
}

// ----------------------------------------------------------------- NVFP4
// One thread per 16-element block.  SRC is float or bf16 (activations).
template <typename SRC>
MOE_DEV float load_elem(const SRC* p, int i);
template <>
MOE_DEV float load_elem<float>(const float* p, int i) { return p[i]; }
template <>
MOE_DEV float load_elem<__nv_bfloat16>(const __nv_bfloat16* p, int i) { return __bfloat162float(p[i]); }

template <typename SRC>
__global__ void k_quantize_nvfp4(const SRC* __restrict__ w, int N, int K, float g,
                                 uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
    const int nblk = K / kFp4Blk;
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (long long)N * nblk) return;
    const int n = (int)(t / nblk), b = (int)(t % nblk);
    const SRC* src = w + (size_t)n * K + b * kFp4Blk;
    float e[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) e[i] = load_elem<SRC>(src, i);
    uint32_t wc[2];
    const uint32_t sb = nvfp4_quant_block16(e, g, wc);
    *reinterpret_cast<uint2*>(codes + (size_t)n * (K / 2) + b * 8) = make_uint2(wc[0], wc[1]);
    scales[(size_t)n * nblk + b] = (uint8_t)sb;
}

// ------------------------------------------------------------------ amax
__global__ void k_absmax(const float* __restrict__ x, long long n, float* __restrict__ out) {
    float m = 0.0f;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x)
        m = fmaxf(m, fabsf(x[i]));
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<int*>(out), __float_as_int(m));
}

// ------------------------------------------------------------ re-layout
// Position of element (n, k) of a quantized matrix in the device layout:
// byte offset inside the matrix's codes and bit shift.
MOE_DEV void dev_code_pos(const MatGeom& gm, int n, int k, size_t& off, int& shift) {
    const int rb = n / kBlkN, r = n % kBlkN, kb = k / kBlkK, kl = k % kBlkK;
    const size_t base = block_offset(gm, rb, kb);
    if (gm.quant == Q_INT2) {
        const int w = kl / 16, ki = kl % 16;
        const int p = ki / 2 + (ki % 2) * 8;
        off = base + (size_t)r * 16 + w * 4 + p / 4;
        shift = (p % 4) * 2;
    } else if (gm.quant == Q_FP8) {  // one byte per code, 16-column chunks
        off = base + ((size_t)(kl / 16) * kBlkN + r) * 16 + kl % 16;
        shift = 0;
    } else {  // INT4 / NVFP4 nibbles
        const int c = kl / 32, kc = kl % 32, w = kc / 8, ki = kc % 8;
        const int p = ki / 2 + (ki % 2) * 4;
        off = base + ((size_t)c * kBlkN + r) * 16 + w * 4 + p / 2;
        shift = (p % 2) * 4;
    }
}

MOE_DEV uint32_t interchange_code(const MatGeom& gm, const uint8_t* src, int n, int k) {
    if (gm.quant == Q_FP8) return src[(size_t)n * gm.K + k];
    if (gm.quant == Q_FP6) return src[(size_t)n * gm.K + k] & 0xFu;      // low plane: bits 0-3
    if (gm.quant == Q_INT2) return (src[(size_t)n * (gm.K / 4) + k / 4] >> (2 * (k & 3))) & 3u;
    return (src[(size_t)n * (gm.K / 2) + k / 2] >> (4 * (k & 1))) & 15u;
}

// one thread per device code byte
__global__ void k_relayout_codes(MatGeom gm, const uint8_t* __restrict__ src, uint8_t* __restrict__ dst) {
    const size_t total = gm.codes_bytes();
    const size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= total) return;
    if (gm.quant == Q_BF16) {
        // 16-byte chunks: t indexes one chunk of the swizzled tile image
        if (t >= total / 16) return;
        const size_t blk = t / 1024;            // 1024 chunks per 16 KB block
        const int within = (int)(t % 1024);
        const int r = within / 8, c = within % 8;
        const int rb = (int)(blk / gm.kbs()), kb = (int)(blk % gm.kbs());
        const int n = rb * kBlkN + r;
        const uint4 v = *reinterpret_cast<const uint4*>(src + ((size_t)n * gm.K + kb * kBlkK + c * 8) * 2);
        uint8_t* d = dst + blk * 16384 + (r / 8) * 1024 + (r % 8) * 128 + ((c ^ (r % 8)) * 16);
        *reinterpret_cast<uint4*>(d) = v;
        return;
    }
    if (gm.quant == Q_FP8) {
        const size_t blk = t / gm.block_bytes();
        const int within = (int)(t % gm.block_bytes());
        const int q = within / (kBlkN * 16), r = (within / 16) % kBlkN;
        const int rb = (int)(blk / gm.kbs()), kb = (int)(blk % gm.kbs());
        dst[t] = src[(size_t)(rb * kBlkN + r) * gm.K + kb * kBlkK + q * 16 + within % 16];
        return;
    }
    if (gm.quant == Q_FP6 && (int)(t % gm.block_bytes()) >= 4096) {   // high plane: 4 crumbs per byte
        const size_t blk = t / gm.block_bytes();
        const int hb = (int)(t % gm.block_bytes()) - 4096;
        const int c = hb / (kBlkN * 8), r = (hb / 8) % kBlkN, w = (hb % 8) / 2, half = hb % 2;
        const int rb = (int)(blk / gm.kbs()), kb = (int)(blk % gm.kbs());
        const int n = rb * kBlkN + r;
        uint32_t out = 0;
        for (int q = 0; q < 4; ++q) {
            const int p = half * 4 + q;                       // crumb p pairs with nibble p of word w
            const int k = kb * kBlkK + c * 32 + w * 8 + (p % 4) * 2 + p / 4;
            out |= ((uint32_t)(src[(size_t)n * gm.K + k] >> 4) & 3u) << (2 * q);
        }
        dst[t] = (uint8_t)out;
        return;
    }
    // invert dev_code_pos for this byte: locate block and row, then scan the
    // elements of the 16-byte chunk word that owns the byte (FP6: low plane)
    const size_t bb = gm.block_bytes();
    const size_t blk = t / bb;
    const int within = (int)(t % bb);
    const int rb = (int)(blk / gm.kbs()), kb = (int)(blk % gm.kbs());
    int r, c, wbyte;
    if (gm.quant == Q_INT2) { c = 0; r = within / 16; wbyte = within % 16; }
    else { c = within / (kBlkN * 16); r = (within / 16) % kBlkN; wbyte = within % 16; }
    const int n = rb * kBlkN + r;
    const int w = wbyte / 4, byte_in_word = wbyte % 4;
    uint32_t out = 0;
    if (gm.quant == Q_INT2) {
        for (int q = 0; q < 4; ++q) {
            const int p = byte_in_word * 4 + q;
            const int ki = (p % 8) * 2 + p / 8;
            const int k = kb * kBlkK + w * 16 + ki;
            out |= interchange_code(gm, src, n, k) << (2 * q);
        }
    } else {
        for (int q = 0; q < 2; ++q) {
            const int p = byte_in_word * 2 + q;
            const int ki = (p % 4) * 2 + p / 4;
            const int k = kb * kBlkK + c * 32 + w * 8 + ki;
            out |= interchange_code(gm, src, n, k) << (4 * q);
        }
    }
    dst[t] = (uint8_t)out;
}

// scales / zeros: one thread per (row, group or 16-block)
__global__ void k_relayout_scales(MatGeom gm, const uint8_t* __restrict__ src_scales,
                                  const uint8_t* __restrict__ src_zeros, uint8_t* __restrict__ dst_scales,
                                  uint8_t* __restrict__ dst_zeros) {
    const size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gm.quant == Q_NVFP4) {
        const int nblk = gm.K / kFp4Blk;
        if (t >= (size_t)gm.N * nblk) return;
        const int n = (int)(t / nblk), b = (int)(t % nblk);
        const int rb = n / kBlkN, r = n % kBlkN, kb = b / 4, sub = b % 4;
        dst_scales[(((size_t)rb * gm.kbs() + kb) * kBlkN + r) * 4 + sub] = src_scales[t];
        return;
    }
    if (gm.quant == Q_FP8) {      // [N/128][K/128] -> rows padded to fp8_scale_stride
        const int KB = gm.K / 128;
        if (t >= (size_t)gm.nb() * KB) return;
        reinterpret_cast<float*>(dst_scales)[(t / KB) * gm.fp8_scale_stride() + t % KB] =
            reinterpret_cast<const float*>(src_scales)[t];
        return;
    }
    const int G = gm.groups();
    if (t >= (size_t)gm.N * G) return;
    const int n = (int)(t / G), g = (int)(t % G);
    const int rb = n / kBlkN, r = n % kBlkN;
    const size_t d = ((size_t)rb * G + g) * kBlkN + r;
    reinterpret_cast<__half*>(dst_scales)[d] = reinterpret_cast<const __half*>(src_scales)[t];
    if (gm.quant == Q_INT2)
        dst_zeros[d] = (src_zeros[(size_t)(n / 4) * G + g] >> (2 * (n % 4))) & 3u;
}

// device layout -> interchange (debug round trip); one thread per output byte
__global__ void k_unpack_codes(MatGeom gm, const uint8_t* __restrict__ dev, uint8_t* __restrict__ dst) {
    const size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gm.quant == Q_BF16) {
        const size_t chunks = (size_t)gm.N * gm.K / 8;
        if (t >= chunks) return;
        const int n = (int)(t / (gm.K / 8)), c8 = (int)(t % (gm.K / 8));
        const int rb = n / kBlkN, r = n % kBlkN, kb = c8 / 8, c = c8 % 8;
        const uint8_t* s = dev + block_offset(gm, rb, kb) + (r / 8) * 1024 + (r % 8) * 128 + ((c ^ (r % 8)) * 16);
        *reinterpret_cast<uint4*>(dst + t * 16) = *reinterpret_cast<const uint4*>(s);
        return;
    }
    if (gm.quant == Q_FP6) {       // one code per byte: nibble of the low plane | crumb of the high plane
        if (t >= (size_t)gm.N * gm.K) return;
        const int n = (int)(t / gm.K), k = (int)(t % gm.K);
        const int rb = n / kBlkN, r = n % kBlkN, kb = k / kBlkK, kl = k % kBlkK;
        const int c = kl / 32, kc = kl % 32, w = kc / 8, ki = kc % 8;
        const int p = ki / 2 + (ki % 2) * 4;
        const uint8_t* base = dev + block_offset(gm, rb, kb);
        const uint32_t lo = (base[((size_t)c * kBlkN + r) * 16 + w * 4 + p / 2] >> ((p % 2) * 4)) & 15u;
        const uint32_t hi = (base[4096 + ((size_t)c * kBlkN + r) * 8 + w * 2 + p / 4] >> ((p % 4) * 2)) & 3u;
        dst[t] = (uint8_t)(lo | (hi << 4));
        return;
    }
    const int per_byte = gm.quant == Q_INT2 ? 4 : (gm.quant == Q_FP8 ? 1 : 2);
    const int bpr = gm.K / per_byte;
    if (t >= (size_t)gm.N * bpr) return;
    const int n = (int)(t / bpr), j = (int)(t % bpr);
    uint32_t out = 0;
    for (int q = 0; q < per_byte; ++q) {
        const int k = j * per_byte + q;
        size_t off;
        int shift;
        dev_code_pos(gm, n, k, off, shift);
        const uint32_t v = (dev[off] >> shift) & (gm.quant == Q_INT2 ? 3u : (gm.quant == Q_FP8 ? 255u : 15u));
        out |= v << ((8 / per_byte) * q);
    }
    dst[t] = (uint8_t)out;
}

__global__ void k_unpack_scales(MatGeom gm, const uint8_t* __restrict__ dev_scales,
                                const uint8_t* __restrict__ dev_zeros, uint8_t* __restrict__ scales,
                                uint8_t* __restrict__ zeros) {
    const size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gm.quant == Q_NVFP4) {
        const int nblk = gm.K / kFp4Blk;
        if (t >= (size_t)gm.N * nblk) return;
        const int n = (int)(t / nblk), b = (int)(t % nblk);
        const int rb = n / kBlkN, r = n % kBlkN;
        scales[t] = dev_scales[(((size_t)rb * gm.kbs() + b / 4) * kBlkN + r) * 4 + b % 4];
        return;
    }
    if (gm.quant == Q_FP8) {
        const int KB = gm.K / 128;
        if (t >= (size_t)gm.nb() * KB) return;
        reinterpret_cast<float*>(scales)[t] =
            reinterpret_cast<const float*>(dev_scales)[(t / KB) * gm.fp8_scale_stride() + t % KB];
        return;
    }
    const int G = gm.groups();
    if (t >= (size_t)gm.N * G) return;
    const int n = (int)(t / G), g = (int)(t % G);
    const size_t d = ((size_t)(n / kBlkN) * G + g) * kBlkN + n % kBlkN;
    reinterpret_cast<__half*>(scales)[t] = reinterpret_cast<const __half*>(dev_scales)[d];
    if (gm.quant == Q_INT2 && n % 4 == 0) {
        uint32_t zb = 0;
        for (int i = 0; i < 4; ++i) {
            const size_t di = ((size_t)((n + i) / kBlkN) * G + g) * kBlkN + (n + i) % kBlkN;
            zb |= (uint32_t)(dev_zeros[di] & 3u) << (2 * i);
        }
        zeros[(size_t)(n / 4) * G + g] = (uint8_t)zb;
    }
}

// ---------------------------------------------------------------- launchers
static inline unsigned blocks_for(size_t n, int tpb) { return (unsigned)((n + tpb - 1) / tpb); }

cudaError_t launch_quantize(int quant, const float* w, int N, int K, float g, void* codes, void* scales,
                            void* zeros, cudaStream_t st) {
    if (is_int4(quant)) {
        const size_t warps = (size_t)N * (K / 128);
        k_quantize_int4<<<blocks_for(warps * 32, 256), 256, 0, st>>>(w, N, K, group_size(quant), (uint8_t*)codes,
                                                                     (__half*)scales);
    } else if (quant == Q_INT2) {
        const size_t warps = (size_t)(N / 4) * (K / kGroup);
        k_quantize_int2<<<blocks_for(warps * 32, 256), 256, 0, st>>>(w, N, K, (uint8_t*)codes, (__half*)scales,
                                                                     (uint8_t*)zeros);
    } else if (quant == Q_FP6) {
        const size_t warps = (size_t)N * (K / 128);
        k_quantize_fp6<<<blocks_for(warps * 32, 256), 256, 0, st>>>(w, N, K, (uint8_t*)codes, (__half*)scales);
    } else if (quant == Q_FP8) {
        k_quantize_fp8<<<(unsigned)((N / 128) * (K / 128)), 256, 0, st>>>(w, N, K, (uint8_t*)codes, (float*)scales);
    } else {
        const size_t blocks = (size_t)N * (K / kFp4Blk);
        k_quantize_nvfp4<float><<<blocks_for(blocks, 256), 256, 0, st>>>(w, N, K, g, (uint8_t*)codes,
                                                                         (uint8_t*)scales);
    }
    return cudaGetLastError();
}

cudaError_t launch_quantize_act_nvfp4(const void* x, int T, int K, float g, void* codes, void* scales,
                                      cudaStream_t st) {
    const size_t blocks = (size_t)T * (K / kFp4Blk);
    k_quantize_nvfp4<__nv_bfloat16><<<blocks_for(blocks, 256), 256, 0, st>>>(
        (const __nv_bfloat16*)x, T, K, g, (uint8_t*)codes, (uint8_t*)scales);
    return cudaGetLastError();
}

cudaError_t launch_absmax(const float* x, long long n, float* out, cudaStream_t st) {
    unsigned grid = blocks_for((size_t)n, 256);
    if (grid > 148 * 8) grid = 148 * 8;
    if (grid == 0) grid = 1;
    k_absmax<<<grid, 256, 0, st>>>(x, n, out);
    return cudaGetLastError();
}

cudaError_t launch_relayout(const MatGeom& gm, const uint8_t* src_codes, const uint8_t* src_scales,
                            const uint8_t* src_zeros, uint8_t* dst_codes, uint8_t* dst_scales,
                            uint8_t* dst_zeros, cudaStream_t st) {
    k_relayout_codes<<<blocks_for(gm.codes_bytes(), 256), 256, 0, st>>>(gm, src_codes, dst_codes);
    if (gm.quant != Q_BF16) {
        const size_t n = gm.quant == Q_NVFP4 ? (size_t)gm.N * (gm.K / kFp4Blk)
                         : gm.quant == Q_FP8 ? (size_t)gm.nb() * (gm.K / 128) : (size_t)gm.N * gm.groups();
        k_relayout_scales<<<blocks_for(n, 256), 256, 0, st>>>(gm, src_scales, src_zeros, dst_scales, dst_zeros);
    }
    return cudaGetLastError();
}

// Block-scaled GEMM weight image of one NVFP4 matrix of one expert (codes
// [N][K/2], scales [N][K/16] in the interchange layout): for each 128-row
// block rb and 256-value stage ks, one contiguous block of nmat x 16 KB of
// codes followed by nmat x 2 KB of scales, at dst + (rb * K/256 + ks) *
// nmat * 18 KB.  This matrix fills slot `slot` of each block (gate 0 and up 1
// share the blocks of the gate/up image; down has nmat = 1).  The codes tile
// (128 rows x 128 bytes) is stored in the 128-byte swizzled order the tensor
// core reads from shared memory (16-byte chunk c of row r at chunk c ^ (r % 8)
// of its row), so a stage's weights and scales arrive in one bulk copy.
__global__ void k_fp4_block_image(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, int N, int K,
                                  int slot, int nmat, uint8_t* __restrict__ dst) {
    const int NS = K / 256;
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;     // (row n, stage ks)
    if (i >= (long long)N * NS) return;
    const int n = (int)(i / NS), ks = (int)(i % NS);
    const int rb = n >> 7, r = n & 127;
    uint8_t* blk = dst + ((size_t)rb * NS + ks) * (size_t)nmat * (16384 + 2048);
    const uint4* src = reinterpret_cast<const uint4*>(codes + (size_t)n * (K / 2) + ks * 128);
    uint8_t* tile = blk + slot * 16384 + r * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(tile + ((c ^ (r & 7)) << 4)) = src[c];
    *reinterpret_cast<uint4*>(blk + nmat * 16384 + slot * 2048 + r * 16) =
        *reinterpret_cast<const uint4*>(scales + (size_t)n * (K / 16) + ks * 16);
}

cudaError_t launch_fp4_block_image(const uint8_t* codes, const uint8_t* scales, int N, int K, int slot, int nmat,
                                   uint8_t* dst, cudaStream_t st) {
    if (N % 128 || K % 256 || slot < 0 || slot >= nmat || nmat < 1 || nmat > 2) return cudaErrorInvalidValue;
    const size_t n = (size_t)N * (K / 256);
    k_fp4_block_image<<<blocks_for(n, 256), 256, 0, st>>>(codes, scales, N, K, slot, nmat, dst);
    return cudaGetLastError();
}

__global__ void k_gather_global_scales(const uint8_t* const* __restrict__ table, size_t off, int E,
                                       float* __restrict__ g) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const float* src = reinterpret_cast<const float*>(table[e] + off);
    g[e] = src[0];
    g[E + e] = src[1];
}

cudaError_t launch_gather_global_scales(const uint8_t* const* table, size_t off, int E, float* g, cudaStream_t st) {
    k_gather_global_scales<<<(E + 255) / 256, 256, 0, st>>>(table, off, E, g);
    return cudaGetLastError();
}

cudaError_t launch_unpack(const MatGeom& gm, const uint8_t* dev_codes, const uint8_t* dev_scales,
                          const uint8_t* dev_zeros, uint8_t* codes, uint8_t* scales, uint8_t* zeros,
                          cudaStream_t st) {
    const size_t nbytes = gm.quant == Q_BF16 ? (size_t)gm.N * gm.K / 8
                                             : (size_t)gm.N * gm.K / (gm.quant == Q_INT2 ? 4 : ((gm.quant == Q_FP8 || gm.quant == Q_FP6) ? 1 : 2));
    k_unpack_codes<<<blocks_for(nbytes, 256), 256, 0, st>>>(gm, dev_codes, codes);
    if (gm.quant != Q_BF16) {
        const size_t n = gm.quant == Q_NVFP4 ? (size_t)gm.N * (gm.K / kFp4Blk)
                         : gm.quant == Q_FP8 ? (size_t)gm.nb() * (gm.K / 128) : (size_t)gm.N * gm.groups();
        k_unpack_scales<<<blocks_for(n, 256), 256, 0, st>>>(gm, dev_scales, dev_zeros, scales, zeros);
    }
    return cudaGetLastError();
}

}  // namespace moe
