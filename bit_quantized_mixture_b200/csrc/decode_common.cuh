// Building blocks shared by the decode kernels (few tokens, tensor-core GEMV):
// the per-launch plan of distinct experts, exact dequantization into MMA
// fragments, the m16n8k16 row-block products and activation staging.
// See decode.cu for the design.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kDecMaxT = 8;           // tokens per launch = MMA N
constexpr int kDecMaxSlots = 256;
constexpr int kXPad = 32;             // bf16 row padding of staged activations (bank spread)

struct Plan {
    int n_unique;
    int ids[kDecMaxSlots];
    int first[kDecMaxSlots];
    unsigned char is_first[kDecMaxSlots];
};

MOE_DEV void build_plan(const int32_t* __restrict__ ids, int n, Plan& p) {
    for (int s = threadIdx.x; s < n; s += blockDim.x) p.ids[s] = __ldcg(ids + s);
    __syncthreads();
    for (int s = threadIdx.x; s < n; s += blockDim.x) {
        const int e = p.ids[s];
        bool f = true;
        for (int q = 0; q < s; ++q) f = f && (p.ids[q] != e);
        p.is_first[s] = f;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int base = 0;
        for (int s0 = 0; s0 < n; s0 += 32) {
            const int s = s0 + lane;
            const bool f = (s < n) && p.is_first[s];
            const unsigned m = __ballot_sync(0xffffffffu, f);
            if (f) p.first[base + __popc(m & ((1u << lane) - 1u))] = s;
            base += __popc(m);
        }
        if (lane == 0) p.n_unique = base;
    }
    __syncthreads();
}

// Tokens of the item whose first slot is s0, in slot order.  With valid
// input (distinct ids per token) there are at most T <= kDecMaxT; repeated
// ids within a token are invalid input and the extra slots are dropped, so
// no buffer is overrun.
MOE_DEV int item_tokens(const int* __restrict__ ids, int n, int k, int s0, int* tok, int* slot, int cap = kDecMaxT) {
    const int e0 = ids[s0];
    int c = 0;
    for (int s = s0; s < n && c < cap; ++s) {
        if (ids[s] == e0) {
            if (threadIdx.x == 0) { tok[c] = s / k; slot[c] = s; }
            ++c;
        }
    }
    return c;
}

// ------------------------------------------------------------ MMA helpers
MOE_DEV void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// ------------------------------------------------------------ format traits
// KPW: k-blocks whose loads a warp issues before it multiplies (loads in
// flight); 2 for the formats where that fits the register budget and
// measured faster at batch 1 (INT4 group 32: 36.9 -> 33.5 us per step,
// FP8: 33.4 -> 33.0 us), 1 elsewhere.
template <int Q> struct Fmt;
template <> struct Fmt<Q_INT4>  { static constexpr int KPW = 1; };
template <> struct Fmt<Q_INT4G32> { static constexpr int KPW = 2; };
template <> struct Fmt<Q_FP8>   { static constexpr int KPW = 2; };
template <> struct Fmt<Q_FP6>   { static constexpr int KPW = 1; };

// FP6: pair j (columns 2j, 2j+1 of INT4-style word w) -> bf16x2, exact:
// low nibbles from w, high crumbs j and j+4 of the high-plane word hw
MOE_DEV uint32_t fp6_pair(uint32_t w, uint32_t hw, int j) {
    const uint32_t nib = (w >> (4 * j)) & 0x000F000Fu;
    const uint32_t x = hw >> (2 * j);
    const uint32_t cr = (x & 0x3u) | ((x & 0x300u) << 8);
    const uint32_t h2 = e2m3x2_to_f16x2_scaled(nib, cr);
    const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&h2), __float2half2_rn(16384.0f));   // exact
    return pack_bf16x2(__low2float(v), __high2float(v));
}

// Two E4M3 codes (low byte first) -> bf16x2: exact, since every E4M3 value
// is an fp16 and a bf16 value
MOE_DEV uint32_t fp8_pair(uint32_t word, int half) {
    const uint32_t h2 = e4m3x2_to_f16x2(word >> (16 * half));
    const __half2 h = *reinterpret_cast<const __half2*>(&h2);
    return pack_bf16x2(__low2float(h), __high2float(h));
}
template <> struct Fmt<Q_NVFP4> { static constexpr int KPW = 1; };
template <> struct Fmt<Q_INT2>  { static constexpr int KPW = 1; };
template <> struct Fmt<Q_BF16>  { static constexpr int KPW = 1; };

struct MatPtr {
    const uint8_t* codes;
    const uint8_t* scales;
    const uint8_t* zeros;
};

// Operands of rows (rl, rl+8) of one 128x64 block for lane (g, c)
template <int Q>
struct Blk {
    uint32_t w[4][2];        // INT4 / NVFP4: [chunk][row g, g+8] (FP8: four chunks); INT2: w[0][row]
    uint4 v[2][2];           // bf16: [32-column half][row g, g+8]
    float s0, s1;            // INT4/INT2 scales of the two rows (INT4 group 32: of chunk 0)
    float s2, s3;            // INT4 group 32 / FP6: scales of the two rows for chunk 1
    uint32_t hw[2][2];       // FP6: high-plane 16-bit word of [chunk][row g, g+8]
    uint32_t z0, z1;         // INT2: bf16x2(128 + z) of the two rows
    uint32_t sb0, sb1;       // NVFP4: four E4M3 block scales of each row
};

template <int Q>
MOE_DEV void load_blk(Blk<Q>& o, const MatPtr& m, int nb, int kb, int KB, int G, int rl, int c) {
    if constexpr (Q == Q_BF16) {
        const uint8_t* blk = m.codes + ((size_t)nb * KB + kb) * 16384;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int r = rl + 8 * rr;
                const int c8 = 4 * h + c;
                o.v[h][rr] = ldg_stream_v4(blk + (r >> 3) * 1024 + (r & 7) * 128 + ((c8 ^ (r & 7)) << 4));
            }
    } else if constexpr (Q == Q_FP8) {
        // four 16-column chunks; lane c takes columns 4c .. 4c+3 of each; the
        // block scale of (row block, 128-column group) is G-strided (padded)
        const uint8_t* blk = m.codes + ((size_t)nb * KB + kb) * (kBlkN * 64);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            o.w[q][0] = __ldg(reinterpret_cast<const uint32_t*>(blk + (q * kBlkN + rl) * 16 + c * 4));
            o.w[q][1] = __ldg(reinterpret_cast<const uint32_t*>(blk + (q * kBlkN + rl + 8) * 16 + c * 4));
        }
        o.s0 = __ldg(reinterpret_cast<const float*>(m.scales) + (size_t)nb * G + kb / 2);
    } else if constexpr (Q == Q_FP6) {
        const uint8_t* blk = m.codes + ((size_t)nb * KB + kb) * (kBlkN * 48);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
            o.w[ch][0] = __ldg(reinterpret_cast<const uint32_t*>(blk + (ch * kBlkN + rl) * 16 + c * 4));
            o.w[ch][1] = __ldg(reinterpret_cast<const uint32_t*>(blk + (ch * kBlkN + rl + 8) * 16 + c * 4));
            o.hw[ch][0] = __ldg(reinterpret_cast<const unsigned short*>(blk + 4096 + (ch * kBlkN + rl) * 8 + c * 2));
            o.hw[ch][1] = __ldg(reinterpret_cast<const unsigned short*>(blk + 4096 + (ch * kBlkN + rl + 8) * 8 + c * 2));
        }
        const size_t gi = ((size_t)nb * G + 2 * kb) * kBlkN + rl;      // chunk ch = group 2 kb + ch
        const __half* sp = reinterpret_cast<const __half*>(m.scales);
        o.s0 = __half2float(__ldg(sp + gi));
        o.s1 = __half2float(__ldg(sp + gi + 8));
        o.s2 = __half2float(__ldg(sp + gi + kBlkN));
        o.s3 = __half2float(__ldg(sp + gi + kBlkN + 8));
    } else if constexpr (Q == Q_INT2) {
        const uint8_t* blk = m.codes + ((size_t)nb * KB + kb) * (kBlkN * 16);
        o.w[0][0] = __ldg(reinterpret_cast<const uint32_t*>(blk + rl * 16 + c * 4));
        o.w[0][1] = __ldg(reinterpret_cast<const uint32_t*>(blk + (rl + 8) * 16 + c * 4));
        const size_t gi = ((size_t)nb * G + kb / 2) * kBlkN + rl;
        o.s0 = __half2float(__ldg(reinterpret_cast<const __half*>(m.scales) + gi));
        o.s1 = __half2float(__ldg(reinterpret_cast<const __half*>(m.scales) + gi + 8));
        o.z0 = bf16x2_splat(128.0f + (float)__ldg(m.zeros + gi));
        o.z1 = bf16x2_splat(128.0f + (float)__ldg(m.zeros + gi + 8));
    } else {
        const uint8_t* blk = m.codes + ((size_t)nb * KB + kb) * (kBlkN * 32);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
            o.w[ch][0] = __ldg(reinterpret_cast<const uint32_t*>(blk + (ch * kBlkN + rl) * 16 + c * 4));
            o.w[ch][1] = __ldg(reinterpret_cast<const uint32_t*>(blk + (ch * kBlkN + rl + 8) * 16 + c * 4));
        }
        if constexpr (Q == Q_INT4) {
            const size_t gi = ((size_t)nb * G + kb / 2) * kBlkN + rl;
            o.s0 = __half2float(__ldg(reinterpret_cast<const __half*>(m.scales) + gi));
            o.s1 = __half2float(__ldg(reinterpret_cast<const __half*>(m.scales) + gi + 8));
        } else if constexpr (Q == Q_INT4G32) {      // chunk ch = group 2 kb + ch
            const size_t gi = ((size_t)nb * G + 2 * kb) * kBlkN + rl;
            const __half* sp = reinterpret_cast<const __half*>(m.scales);
            o.s0 = __half2float(__ldg(sp + gi));
            o.s1 = __half2float(__ldg(sp + gi + 8));
            o.s2 = __half2float(__ldg(sp + gi + kBlkN));
            o.s3 = __half2float(__ldg(sp + gi + kBlkN + 8));
        } else {
            const size_t si = (((size_t)nb * KB + kb) * kBlkN + rl) * 4;
            o.sb0 = __ldg(reinterpret_cast<const uint32_t*>(m.scales + si));
            o.sb1 = __ldg(reinterpret_cast<const uint32_t*>(m.scales + si + 32));
        }
    }
}

// acc[0..3] (rows g, g+8 x tokens 2c, 2c+1) += block . x; xrow points at
// the lane's token row g of the staged activations at the block's column 0.
template <int Q>
MOE_DEV void mma_blk(float (&acc)[4], const Blk<Q>& o, const __nv_bfloat16* xrow, int c) {
    float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if constexpr (Q == Q_FP8) {
        // K16 step q: the lane's B pairs are columns (16q + 4c, +1) and
        // (16q + 4c + 2, +3), so its A pairs are bytes 0-1 and 2-3 of word c
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint2 xv = *reinterpret_cast<const uint2*>(xrow + 16 * q + 4 * c);
            mma16816(d, fp8_pair(o.w[q][0], 0), fp8_pair(o.w[q][1], 0), fp8_pair(o.w[q][0], 1),
                     fp8_pair(o.w[q][1], 1), xv.x, xv.y);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] = fmaf(o.s0, d[i], acc[i]);
        return;
    } else if constexpr (Q == Q_INT2) {
        const uint4 x0 = *reinterpret_cast<const uint4*>(xrow + 16 * c);
        const uint4 x1 = *reinterpret_cast<const uint4*>(xrow + 16 * c + 8);
        const uint32_t xb[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int mi = 0; mi < 4; ++mi)
            mma16816(d, int2_pair(o.w[0][0], 2 * mi, o.z0), int2_pair(o.w[0][1], 2 * mi, o.z1),
                     int2_pair(o.w[0][0], 2 * mi + 1, o.z0), int2_pair(o.w[0][1], 2 * mi + 1, o.z1), xb[2 * mi],
                     xb[2 * mi + 1]);
    } else {
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
            const uint4 xv = *reinterpret_cast<const uint4*>(xrow + 32 * ch + 8 * c);
            if constexpr (Q == Q_BF16) {
                const uint4 r0 = o.v[ch][0], r1 = o.v[ch][1];
                mma16816(acc, r0.x, r1.x, r0.y, r1.y, xv.x, xv.y);
                mma16816(acc, r0.z, r1.z, r0.w, r1.w, xv.z, xv.w);
            } else if constexpr (Q == Q_INT4) {
                const uint32_t w0 = o.w[ch][0], w1 = o.w[ch][1];
                mma16816(d, int4_pair(w0, 0), int4_pair(w1, 0), int4_pair(w0, 1), int4_pair(w1, 1), xv.x, xv.y);
                mma16816(d, int4_pair(w0, 2), int4_pair(w1, 2), int4_pair(w0, 3), int4_pair(w1, 3), xv.z, xv.w);
            } else if constexpr (Q == Q_FP6) {       // group 32 = one chunk, as INT4 group 32
                const uint32_t w0 = o.w[ch][0], w1 = o.w[ch][1], h0 = o.hw[ch][0], h1 = o.hw[ch][1];
                float dc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                mma16816(dc, fp6_pair(w0, h0, 0), fp6_pair(w1, h1, 0), fp6_pair(w0, h0, 1), fp6_pair(w1, h1, 1), xv.x,
                         xv.y);
                mma16816(dc, fp6_pair(w0, h0, 2), fp6_pair(w1, h1, 2), fp6_pair(w0, h0, 3), fp6_pair(w1, h1, 3), xv.z,
                         xv.w);
                const float sa = ch ? o.s2 : o.s0, sb = ch ? o.s3 : o.s1;
                acc[0] = fmaf(sa, dc[0], acc[0]);
                acc[1] = fmaf(sa, dc[1], acc[1]);
                acc[2] = fmaf(sb, dc[2], acc[2]);
                acc[3] = fmaf(sb, dc[3], acc[3]);
            } else if constexpr (Q == Q_INT4G32) {   // one group per chunk: its own partial sum and scale
                const uint32_t w0 = o.w[ch][0], w1 = o.w[ch][1];
                float dc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                mma16816(dc, int4_pair(w0, 0), int4_pair(w1, 0), int4_pair(w0, 1), int4_pair(w1, 1), xv.x, xv.y);
                mma16816(dc, int4_pair(w0, 2), int4_pair(w1, 2), int4_pair(w0, 3), int4_pair(w1, 3), xv.z, xv.w);
                const float sa = ch ? o.s2 : o.s0, sb = ch ? o.s3 : o.s1;
                acc[0] = fmaf(sa, dc[0], acc[0]);
                acc[1] = fmaf(sa, dc[1], acc[1]);
                acc[2] = fmaf(sb, dc[2], acc[2]);
                acc[3] = fmaf(sb, dc[3], acc[3]);
            } else {  // NVFP4: word c of chunk ch lies in 16-column block 2ch + c/2
                const int b = 2 * ch + (c >> 1);
                const uint32_t s0 = bf16x2_splat(e4m3_to_f32((o.sb0 >> (8 * b)) & 0xffu));
                const uint32_t s1 = bf16x2_splat(e4m3_to_f32((o.sb1 >> (8 * b)) & 0xffu));
                const uint32_t w0 = o.w[ch][0], w1 = o.w[ch][1];
                mma16816(d, fp4_pair(w0, 0, s0), fp4_pair(w1, 0, s1), fp4_pair(w0, 1, s0), fp4_pair(w1, 1, s1), xv.x,
                         xv.y);
                mma16816(d, fp4_pair(w0, 2, s0), fp4_pair(w1, 2, s1), fp4_pair(w0, 3, s0), fp4_pair(w1, 3, s1), xv.z,
                         xv.w);
            }
        }
    }
    if constexpr (Q == Q_INT4 || Q == Q_INT2) {
        acc[0] = fmaf(o.s0, d[0], acc[0]);
        acc[1] = fmaf(o.s0, d[1], acc[1]);
        acc[2] = fmaf(o.s1, d[2], acc[2]);
        acc[3] = fmaf(o.s1, d[3], acc[3]);
    } else if constexpr (Q == Q_NVFP4) {
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += d[i];
    }
}

// One warp: 16 rows (rl, rl+8 per lane) of NM matrices over k-blocks
// warp, warp + nwarps, ... against NG groups of 8 token columns (xrows[q]:
// the lane's token row of group q); each k-block's weights are loaded once
// for all groups.
template <int Q, int NM, int NG = 1>
MOE_DEV void warp_rows(float (&acc)[NM][NG][4], const MatPtr (&mats)[NM], int nb, int rl, int KB, int G, int warp,
                       int nwarps, const __nv_bfloat16* const (&xrows)[NG], int c) {
    constexpr int KPW = NG == 1 ? Fmt<Q>::KPW : 1;
    for (int kb0 = warp; kb0 < KB; kb0 += nwarps * KPW) {
        Blk<Q> blk[NM][KPW];
#pragma unroll
        for (int i = 0; i < KPW; ++i) {
            const int kb = kb0 + i * nwarps;
            if (kb < KB) {
#pragma unroll
                for (int q = 0; q < NM; ++q) load_blk<Q>(blk[q][i], mats[q], nb, kb, KB, G, rl, c);
            }
        }
#pragma unroll
        for (int i = 0; i < KPW; ++i) {
            const int kb = kb0 + i * nwarps;
            if (kb < KB) {
#pragma unroll
                for (int q = 0; q < NM; ++q)
#pragma unroll
                    for (int gq = 0; gq < NG; ++gq) mma_blk<Q>(acc[q][gq], blk[q][i], xrows[gq] + kb * kBlkK, c);
            }
        }
    }
}

// W4A4: the value q * s_b of a 16-element block (the global scale g is left
// to the epilogue), from the library's one NVFP4 block quantizer.
MOE_DEV void fp4_block_values(float (&v)[16], float g) { nvfp4_block16_values(v, g); }

// Stage rows (row_of[t], t < m) of a bf16 matrix [*, K] into smem rows of
// ldx elements; rows m..7 are zero.  16-byte accesses, loads issued first.
MOE_DEV void stage_rows_bf16(__nv_bfloat16* dst, int ldx, const __nv_bfloat16* src, int K, const int* row_of, int m,
                             int tid, int nthreads, int nrows = kDecMaxT) {
    const int per_row = K / 8;
    const int total = nrows * per_row;
    for (int i0 = tid; i0 < total; i0 += 4 * nthreads) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * nthreads;
            const int t = i / per_row, c = i % per_row;
            v[u] = (i < total && t < m) ? *reinterpret_cast<const uint4*>(src + (size_t)row_of[t] * K + c * 8)
                                        : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * nthreads;
            if (i < total) *reinterpret_cast<uint4*>(dst + (i / per_row) * ldx + (i % per_row) * 8) = v[u];
        }
    }
}

// Stage rows of bf16 activations [*, K] as W4A4 values (q * s_b).
MOE_DEV void stage_rows_fp4_from_bf16(__nv_bfloat16* dst, int ldx, const __nv_bfloat16* src, int K,
                                      const int* row_of, int m, float g, int tid, int nthreads,
                                      int nrows = kDecMaxT) {
    const int per_row = K / 16;
    const int total = nrows * per_row;
    for (int i = tid; i < total; i += nthreads) {
        const int t = i / per_row, b = i % per_row;
        float v[16];
        if (t < m) {
            const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)row_of[t] * K + b * 16);
            const uint4 q0 = s[0], q1 = s[1];
            const uint32_t wv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int q = 0; q < 8; ++q) { v[2 * q] = bf16_lo(wv[q]); v[2 * q + 1] = bf16_hi(wv[q]); }
            fp4_block_values(v, g);
        } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) v[q] = 0.0f;
        }
        uint32_t p[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) p[q] = pack_bf16x2(v[2 * q], v[2 * q + 1]);
        uint4* d = reinterpret_cast<uint4*>(dst + t * ldx + b * 16);
        d[0] = make_uint4(p[0], p[1], p[2], p[3]);
        d[1] = make_uint4(p[4], p[5], p[6], p[7]);
    }
}

// Stage rows of fp32 intermediates [*, K] as bf16 (W4A4: as q * s_b).
MOE_DEV void stage_rows_f32(__nv_bfloat16* dst, int ldx, const float* src, int K, const int* row_of, int m, bool fp4,
                            float g, int tid, int nthreads, int nrows = kDecMaxT) {
    const int per_row = K / 16;
    const int total = nrows * per_row;
    for (int i = tid; i < total; i += nthreads) {
        const int t = i / per_row, b = i % per_row;
        float v[16];
        if (t < m) {
            const float4* s = reinterpret_cast<const float4*>(src + (size_t)row_of[t] * K + b * 16);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 f = __ldcg(s + q);
                v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
            }
            if (fp4) fp4_block_values(v, g);
        } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) v[q] = 0.0f;
        }
        uint32_t p[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) p[q] = pack_bf16x2(v[2 * q], v[2 * q + 1]);
        uint4* d = reinterpret_cast<uint4*>(dst + t * ldx + b * 16);
        d[0] = make_uint4(p[0], p[1], p[2], p[3]);
        d[1] = make_uint4(p[4], p[5], p[6], p[7]);
    }
}

MOE_DEV MatPtr expert_mat(const MatView& v, int e) {
    const ExpertMat m = expert_matrix(v, e);
    MatPtr p;
    p.codes = m.codes;
    p.scales = m.scales;
    p.zeros = m.zeros;
    return p;
}


}  // namespace moe
