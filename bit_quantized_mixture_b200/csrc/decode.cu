// Decode path of the expert computation (up to 8 tokens per launch):
// memory-bound GEMVs that stream each selected expert's packed weights once,
// dequantize in registers and multiply on the tensor cores.
//
// The pages' decode kernel reads each expert "in place" from an N-contiguous
// packed layout ("Qwen3.8-Flash-Next on one 24 GB GPU", "What the patch
// does"), and expert GEMV dominates the per-stream decode cost
// ("Qwen3.8-Flash-Next-FP6-INT8", "Step budget and hardware floors").
//
// One warp computes 16 weight rows x 8 token columns with mma.sync m16n8k16
// (bf16 operands, fp32 accumulation).  The 16 "k" slots of each MMA are
// mapped onto the packed layout of layout.cuh so that a lane's A fragment is
// exactly the codes of one 32-bit word of its rows:
//   INT4 / NVFP4: lane (g, c) takes word c of a 16-byte chunk of rows g and
//       g+8 (8 columns 8c..8c+7 of the chunk's 32); its pairs 0,1 feed one
//       MMA and pairs 2,3 the next; the B fragment is x[8c .. 8c+7];
//   INT2: word c of rows g, g+8 (16 columns 16c..16c+15) feeds four MMAs.
// Dequantization gives exact bf16 operands: (u - 8) and (u - z) are small
// integers, and e2m1 times its E4M3 block scale has at most 6 significant
// bits.  Group scales multiply the fp32 accumulators of each 64-column block
// (INT4 / INT2) and NVFP4's global scales the final sums, so the only
// roundings are the bf16 activations (as given) and fp32 accumulation.
//
// Two kernels per forward:
//   k_dec_gateup: item = (selected expert, 16 intermediate rows), 8 warps
//       split K; a = silu(x Wg^T) * (x Wu^T) in fp32;
//   k_dec_down:   item = (selected expert, 16 hidden rows), 4 warps split K;
//       o = a Wd^T scaled by the routing weight into a per-slot partial; the
//       last item of a row block to finish (ticket counter, no waiting) sums
//       y_t = sum_j part[t*k+j] + shared_t in fixed j order, one bf16 rounding.
// The shared bf16 expert is one more item with all T tokens.  Every CTA
// derives the same list of distinct selected experts (order of first
// appearance among the flat slots) from the ids.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kDecMaxT = 8;           // tokens per launch = MMA N
constexpr int kDecMaxSlots = 256;
constexpr int kGuThreads = 256;       // 8 warps split K
constexpr int kDnThreads = 128;       // 4 warps split K
constexpr int kXPad = 32;             // bf16 row padding of staged activations (bank spread)

bool decode_supported(int T, int k) { return T >= 1 && T <= kDecMaxT && T * k <= kDecMaxSlots; }

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
MOE_DEV int item_tokens(const int* __restrict__ ids, int n, int k, int s0, int* tok, int* slot) {
    const int e0 = ids[s0];
    int c = 0;
    for (int s = s0; s < n && c < kDecMaxT; ++s) {
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

// ------------------------------------------------------------ format traits
template <int Q> struct Fmt;
template <> struct Fmt<Q_INT4>  { static constexpr int KPW = 4; };
template <> struct Fmt<Q_NVFP4> { static constexpr int KPW = 4; };
template <> struct Fmt<Q_INT2>  { static constexpr int KPW = 4; };
template <> struct Fmt<Q_BF16>  { static constexpr int KPW = 2; };

struct MatPtr {
    const uint8_t* codes;
    const uint8_t* scales;
    const uint8_t* zeros;
};

// Operands of rows (rl, rl+8) of one 128x64 block for lane (g, c)
template <int Q>
struct Blk {
    uint32_t w[2][2];        // INT4 / NVFP4: [chunk][row g, g+8]; INT2: w[0][row]
    uint4 v[2][2];           // bf16: [32-column half][row g, g+8]
    float s0, s1;            // INT4/INT2 scales of the two rows
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
    if constexpr (Q == Q_INT2) {
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
// warp, warp + nwarps, ...
template <int Q, int NM>
MOE_DEV void warp_rows(float (&acc)[NM][4], const MatPtr (&mats)[NM], int nb, int rl, int KB, int G, int warp,
                       int nwarps, const __nv_bfloat16* xrow, int c) {
    constexpr int KPW = Fmt<Q>::KPW;
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
                for (int q = 0; q < NM; ++q) mma_blk<Q>(acc[q], blk[q][i], xrow + kb * kBlkK, c);
            }
        }
    }
}

// W4A4: the value q * s_b of a 16-element block (the global scale g is left
// to the epilogue), with the recipe of the activation quantization kernel.
MOE_DEV void fp4_block_values(float (&v)[16], float g) {
    float amax = 0.0f;
#pragma unroll
    for (int q = 0; q < 16; ++q) amax = fmaxf(amax, fabsf(v[q]));
    float sbv = 0.0f, r = 0.0f;
    if (g != 0.0f) {
        sbv = e4m3_to_f32(f32_to_e4m3(__fdiv_rn(amax, __fmul_rn(6.0f, g))));
        r = (sbv == 0.0f) ? 0.0f : __fdiv_rn(1.0f, __fmul_rn(sbv, g));
    }
#pragma unroll
    for (int q = 0; q < 16; q += 2) {
        const uint32_t cc = f32x2_to_e2m1(__fmul_rn(v[q], r), __fmul_rn(v[q + 1], r));
        v[q] = e2m1_to_f32(cc & 0xFu) * sbv;
        v[q + 1] = e2m1_to_f32(cc >> 4) * sbv;
    }
}

// Stage rows (row_of[t], t < m) of a bf16 matrix [*, K] into smem rows of
// ldx elements; rows m..7 are zero.  16-byte accesses, loads issued first.
MOE_DEV void stage_rows_bf16(__nv_bfloat16* dst, int ldx, const __nv_bfloat16* src, int K, const int* row_of, int m) {
    const int per_row = K / 8;
    const int total = kDecMaxT * per_row;
    for (int i0 = threadIdx.x; i0 < total; i0 += 4 * blockDim.x) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * blockDim.x;
            const int t = i / per_row, c = i % per_row;
            v[u] = (i < total && t < m) ? *reinterpret_cast<const uint4*>(src + (size_t)row_of[t] * K + c * 8)
                                        : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * blockDim.x;
            if (i < total) *reinterpret_cast<uint4*>(dst + (i / per_row) * ldx + (i % per_row) * 8) = v[u];
        }
    }
}

// Stage rows of bf16 activations [*, K] as W4A4 values (q * s_b).
MOE_DEV void stage_rows_fp4_from_bf16(__nv_bfloat16* dst, int ldx, const __nv_bfloat16* src, int K,
                                      const int* row_of, int m, float g) {
    const int per_row = K / 16;
    const int total = kDecMaxT * per_row;
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
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
                            float g) {
    const int per_row = K / 16;
    const int total = kDecMaxT * per_row;
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
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
    MatPtr p;
    p.codes = v.codes + (size_t)e * v.stride;
    p.scales = v.scales ? v.scales + (size_t)e * v.stride : nullptr;
    p.zeros = v.zeros ? v.zeros + (size_t)e * v.stride : nullptr;
    return p;
}

// ------------------------------------------------------------- gate / up
template <int Q>
__global__ void __launch_bounds__(kGuThreads, 3) k_dec_gateup(DecodeArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ Plan plan;
    __shared__ int tok[kDecMaxT];
    __shared__ int slot_of[kDecMaxT];
    const ExpertArgs& ex = a.ex;
    const int H = ex.H, I = ex.I, k = ex.k, T = a.T;
    const int n = T * k;
    const int rb_per_exp = I / 16;
    const int u = blockIdx.x / rb_per_exp;          // distinct expert, or the shared one when u == n
    const int rb16 = blockIdx.x % rb_per_exp;
    const bool is_shared = (u == n);

    // The activations do not depend on the routing: stage all T token rows
    // (row t = token t, rows T..8 zero) before waiting for the router.
    const int ldx = H + kXPad;
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem_raw);                   // [9][ldx]
    float* red = reinterpret_cast<float*>(smem_raw + (size_t)(kDecMaxT + 1) * ldx * 2);   // [8][2][16][8]
    if (threadIdx.x < kDecMaxT) tok[threadIdx.x] = threadIdx.x;
    __syncthreads();
    const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(a.x);
    if (Q == Q_NVFP4 && !is_shared) stage_rows_fp4_from_bf16(xs, ldx, x, H, tok, T, ex.g_x);
    else stage_rows_bf16(xs, ldx, x, H, tok, T);
    for (int i = threadIdx.x; i < ldx / 8; i += blockDim.x)
        reinterpret_cast<uint4*>(xs + kDecMaxT * ldx)[i] = make_uint4(0, 0, 0, 0);

    int m;
    if (is_shared) {
        // the shared expert needs nothing from the router
        m = T;
        if (threadIdx.x < T) slot_of[threadIdx.x] = threadIdx.x;
        pdl_launch_dependents();
    } else {
        pdl_wait();                                  // ids come from the router
        pdl_launch_dependents();
        build_plan(a.ids, n, plan);
        if (u >= plan.n_unique) return;
        m = item_tokens(plan.ids, n, k, plan.first[u], tok, slot_of);
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int KB = H / kBlkK, G = H / kGroup;
    const int r0 = rb16 * 16;
    const int nb = r0 / kBlkN, rl = r0 % kBlkN + g;
    const __nv_bfloat16* xrow = xs + (g < m ? tok[g] : kDecMaxT) * ldx;     // item column g = token tok[g]
    float acc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
    int e = 0;
    if (is_shared) {
        const MatPtr mats[2] = {{ex.sh_gate, nullptr, nullptr}, {ex.sh_up, nullptr, nullptr}};
        warp_rows<Q_BF16, 2>(acc, mats, nb, rl, KB, G, warp, kGuThreads / 32, xrow, c);
    } else {
        e = plan.ids[plan.first[u]];
        if (e >= 0 && e < ex.E) {        // an id outside [0, E) contributes zero
            const MatPtr mats[2] = {expert_mat(ex.gate, e), expert_mat(ex.up, e)};
            warp_rows<Q, 2>(acc, mats, nb, rl, KB, G, warp, kGuThreads / 32, xrow, c);
        } else {
            e = 0;
        }
    }
    // red[warp][mat][row 16][token 8]
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        float* r = red + ((warp * 2 + q) * 16) * 8;
        r[g * 8 + 2 * c] = acc[q][0];
        r[g * 8 + 2 * c + 1] = acc[q][1];
        r[(g + 8) * 8 + 2 * c] = acc[q][2];
        r[(g + 8) * 8 + 2 * c + 1] = acc[q][3];
    }
    __syncthreads();
    const float gscale = (Q == Q_NVFP4 && !is_shared) ? ex.g_gate[e] * ex.g_x : 1.0f;
    if (threadIdx.x < 16 * kDecMaxT) {
        const int row = threadIdx.x / kDecMaxT, t = threadIdx.x % kDecMaxT;
        if (t < m) {
            float gg = 0.0f, uu = 0.0f;
#pragma unroll
            for (int w = 0; w < kGuThreads / 32; ++w) {
                gg += red[((w * 2 + 0) * 16 + row) * 8 + t];
                uu += red[((w * 2 + 1) * 16 + row) * 8 + t];
            }
            gg *= gscale;
            uu *= gscale;
            const float act = gg / (1.0f + expf(-gg)) * uu;
            if (is_shared) a.a_sh[(size_t)t * I + r0 + row] = act;
            else a.a[(size_t)slot_of[t] * I + r0 + row] = act;
        }
    }
}

// ------------------------------------------------------- down + combine
template <int Q>
__global__ void __launch_bounds__(kDnThreads, 10) k_dec_down(DecodeArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ Plan plan;
    __shared__ int tok[kDecMaxT];
    __shared__ int slot_of[kDecMaxT];
    __shared__ int s_last;
    const ExpertArgs& ex = a.ex;
    const int H = ex.H, I = ex.I, k = ex.k, T = a.T;
    const int n = T * k;
    const int rbs = H / 16;
    const int u = blockIdx.x / rbs;
    const int hb = blockIdx.x % rbs;

    // ids/w were produced before the previous kernel started (it waited for
    // them), so they can be read before this kernel's own dependency wait.
    build_plan(a.ids, n, plan);
    const bool is_shared = (u == n);
    if (!is_shared && u >= plan.n_unique) return;
    const int items_per_rb = plan.n_unique + (ex.sh_down ? 1 : 0);
    int m;
    if (is_shared) {
        m = T;
        if (threadIdx.x < T) { tok[threadIdx.x] = threadIdx.x; slot_of[threadIdx.x] = threadIdx.x; }
    } else {
        m = item_tokens(plan.ids, n, k, plan.first[u], tok, slot_of);
    }
    const int ldx = I + kXPad;
    __nv_bfloat16* as = reinterpret_cast<__nv_bfloat16*>(smem_raw);                   // [8][ldx]
    float* red = reinterpret_cast<float*>(smem_raw + (size_t)kDecMaxT * ldx * 2);      // [4][16][8]
    __syncthreads();
    pdl_wait();                                      // a comes from k_dec_gateup
    pdl_launch_dependents();
    stage_rows_f32(as, ldx, is_shared ? a.a_sh : a.a, I, slot_of, m, Q == Q_NVFP4 && !is_shared, ex.g_a);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int KB = I / kBlkK, G = I / kGroup;
    const int h0 = hb * 16;
    const int nb = h0 / kBlkN, rl = h0 % kBlkN + g;
    const __nv_bfloat16* xrow = as + g * ldx;
    float acc[1][4] = {{0, 0, 0, 0}};
    int e = 0;
    if (is_shared) {
        const MatPtr mats[1] = {{ex.sh_down, nullptr, nullptr}};
        warp_rows<Q_BF16, 1>(acc, mats, nb, rl, KB, G, warp, kDnThreads / 32, xrow, c);
    } else {
        e = plan.ids[plan.first[u]];
        if (e >= 0 && e < ex.E) {        // an id outside [0, E) contributes zero
            const MatPtr mats[1] = {expert_mat(ex.down, e)};
            warp_rows<Q, 1>(acc, mats, nb, rl, KB, G, warp, kDnThreads / 32, xrow, c);
        } else {
            e = 0;
        }
    }
    {
        float* r = red + (warp * 16) * 8;
        r[g * 8 + 2 * c] = acc[0][0];
        r[g * 8 + 2 * c + 1] = acc[0][1];
        r[(g + 8) * 8 + 2 * c] = acc[0][2];
        r[(g + 8) * 8 + 2 * c + 1] = acc[0][3];
    }
    __syncthreads();
    const float dscale = (Q == Q_NVFP4 && !is_shared) ? ex.g_down[e] * ex.g_a : 1.0f;
    {
        const int row = threadIdx.x / kDecMaxT, t = threadIdx.x % kDecMaxT;   // 128 threads = 16 x 8
        if (t < m) {
            float o = 0.0f;
#pragma unroll
            for (int w = 0; w < kDnThreads / 32; ++w) o += red[(w * 16 + row) * 8 + t];
            o *= dscale;
            const int h = h0 + row;
            if (is_shared) a.part_sh[(size_t)t * H + h] = o;
            else a.part[(size_t)slot_of[t] * H + h] = __ldcg(a.w + slot_of[t]) * o;
        }
    }
    // the last item of this row block to finish combines
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();                      // this CTA's partials before its ticket
        s_last = (atomicAdd(a.counters + hb, 1u) == (unsigned)items_per_rb - 1u);
        if (s_last) __threadfence();
    }
    __syncthreads();
    if (!s_last) return;
    __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(a.y);
    for (int i = threadIdx.x; i < T * 16; i += blockDim.x) {
        const int t = i / 16, h = h0 + i % 16;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = (j < k) ? __ldcg(a.part + (size_t)(t * k + j) * H + h) : 0.0f;
        float s = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; ++j) s += v[j];          // fixed order j = 0 .. k-1
        if (ex.sh_down) s += __ldcg(a.part_sh + (size_t)t * H + h);
        y[(size_t)t * H + h] = __float2bfloat16_rn(s);
    }
    __syncthreads();
    if (threadIdx.x == 0) a.counters[hb] = 0u;
}

template <int Q>
static cudaError_t launch_decode_q(const DecodeArgs& a, cudaStream_t st) {
    const ExpertArgs& ex = a.ex;
    const int n = a.T * ex.k;
    const int items_gu = (n + (ex.sh_gate ? 1 : 0)) * (ex.I / 16);
    const int items_dn = (n + (ex.sh_down ? 1 : 0)) * (ex.H / 16);
    const size_t smem_gu = (size_t)(kDecMaxT + 1) * (ex.H + kXPad) * 2 + 8 * 2 * 16 * 8 * sizeof(float);
    const size_t smem_dn = (size_t)kDecMaxT * (ex.I + kXPad) * 2 + 4 * 16 * 8 * sizeof(float);
    cudaError_t err = cudaFuncSetAttribute(k_dec_gateup<Q>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_gu);
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(k_dec_down<Q>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dn);
    if (err != cudaSuccess) return err;

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(items_gu);
    cfg.blockDim = dim3(kGuThreads);
    cfg.dynamicSmemBytes = smem_gu;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, k_dec_gateup<Q>, a);
    if (err != cudaSuccess) return err;
    if (a.ev_mid) {
        err = cudaEventRecord(a.ev_mid, st);
        if (err != cudaSuccess) return err;
    }
    cfg.gridDim = dim3(items_dn);
    cfg.blockDim = dim3(kDnThreads);
    cfg.dynamicSmemBytes = smem_dn;
    err = cudaLaunchKernelEx(&cfg, k_dec_down<Q>, a);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
    switch (a.ex.quant) {
        case Q_INT4: return launch_decode_q<Q_INT4>(a, st);
        case Q_INT2: return launch_decode_q<Q_INT2>(a, st);
        case Q_NVFP4: return launch_decode_q<Q_NVFP4>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
