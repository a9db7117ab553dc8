// Decode path of the expert computation (few tokens): memory-bound GEMVs that
// stream each selected expert's packed weights once with coalesced 16-byte
// loads, dequantize in registers and accumulate in fp32.
//
// The pages' decode kernel reads each expert "in place" from an N-contiguous
// packed layout ("Qwen3.8-Flash-Next on one 24 GB GPU", "What the patch
// does"), and expert GEMV dominates the per-stream decode cost
// ("Qwen3.8-Flash-Next-FP6-INT8", "Step budget and hardware floors").  Here
// one lane owns one weight row, so a warp reads 32 rows x 16 bytes = 512
// contiguous bytes per load and needs no cross-lane reduction.
//
// Two kernels per forward:
//   k_dec_gateup: item = (selected expert, 32 intermediate rows); computes
//       a = silu(x Wg^T) * (x Wu^T) for the expert's tokens (fp32);
//   k_dec_down:   item = (selected expert, 32 hidden rows); o = a Wd^T scaled
//       by the routing weight into a per-slot partial; the last item of a row
//       block to finish sums y_t = sum_j part[t*k+j] + shared_t in fixed j
//       order and rounds once to bf16 (no waiting: a ticket counter).
// The shared bf16 expert rides along as one more item with all T tokens.
// Every CTA derives the same list of distinct selected experts (in order of
// first appearance in the flat slot list) from the ids, so no separate
// permutation pass is needed.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kDecMaxT = 4;
constexpr int kDecMaxSlots = 128;
constexpr int kGuThreads = 256;   // 8 warps split K
constexpr int kDnThreads = 128;   // 4 warps split K

bool decode_supported(int T, int k) { return T >= 1 && T <= kDecMaxT && T * k <= kDecMaxSlots; }

struct Plan {
    int n_unique;
    int ids[kDecMaxSlots];       // the launch's expert ids (flat slots)
    int first[kDecMaxSlots];     // first slot of each distinct expert
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

// Tokens of item u (slots whose id equals the id of first[u]), in slot order.
// With valid input (distinct ids per token) there are at most T <= kDecMaxT;
// repeated ids within a token are invalid input: the extra slots are dropped
// so that no buffer is overrun.
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

// ------------------------------------------------------------ format traits
template <int Q> struct Fmt;
template <> struct Fmt<Q_INT4>  { static constexpr int CH = 2, KPW = 4; };
template <> struct Fmt<Q_NVFP4> { static constexpr int CH = 2, KPW = 4; };
template <> struct Fmt<Q_INT2>  { static constexpr int CH = 1, KPW = 4; };
template <> struct Fmt<Q_BF16>  { static constexpr int CH = 8, KPW = 1; };

// Matrix of one expert in device layout
struct MatPtr {
    const uint8_t* codes;
    const uint8_t* scales;
    const uint8_t* zeros;
};

// Loaded operands of one row (one lane) for one 64-column block
template <int Q>
struct RowBlk {
    uint4 c[Fmt<Q>::CH];
    float s;        // INT4/INT2 scale
    float zb;       // INT2: 2^23 + zero
    uint32_t sb4;   // NVFP4: four E4M3 block scales
};

template <int Q>
MOE_DEV void load_row_blk(RowBlk<Q>& o, const MatPtr& m, int nb, int kb, int KB, int G, int r) {
    if constexpr (Q == Q_BF16) {
        const uint8_t* blk = m.codes + ((size_t)nb * KB + kb) * 16384 + (r / 8) * 1024 + (r % 8) * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) o.c[c] = ldg_stream_v4(blk + ((c ^ (r % 8)) * 16));
    } else {
        constexpr int RB = Q == Q_INT2 ? 16 : 32;
        const uint8_t* blk = m.codes + ((size_t)nb * KB + kb) * (kBlkN * RB);
#pragma unroll
        for (int c = 0; c < Fmt<Q>::CH; ++c) o.c[c] = ldg_stream_v4(blk + (size_t)(c * kBlkN + r) * 16);
        if constexpr (Q == Q_NVFP4) {
            o.sb4 = __ldg(reinterpret_cast<const uint32_t*>(m.scales + (((size_t)nb * KB + kb) * kBlkN + r) * 4));
        } else {
            const size_t gi = ((size_t)nb * G + kb / 2) * kBlkN + r;
            o.s = __half2float(__ldg(reinterpret_cast<const __half*>(m.scales) + gi));
            if constexpr (Q == Q_INT2) o.zb = 8388608.0f + (float)__ldg(m.zeros + gi);
        }
    }
}

template <int MT>
MOE_DEV void fma_pair(float (&p)[MT], float w0, float w1, const float* __restrict__ xs, int ld, int m, int col) {
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        if (t < m) {
            const float2 xv = *reinterpret_cast<const float2*>(xs + t * ld + col);
            p[t] = fmaf(w0, xv.x, p[t]);
            p[t] = fmaf(w1, xv.y, p[t]);
        }
    }
}

// acc[t] += dot(row block, xs[t][col .. col+64))
template <int Q, int MT>
MOE_DEV void dot_row_blk(float (&acc)[MT], const RowBlk<Q>& o, const float* xs, int ld, int m, int col) {
    if constexpr (Q == Q_BF16) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint32_t wv[4] = {o.c[c].x, o.c[c].y, o.c[c].z, o.c[c].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) fma_pair<MT>(acc, bf16_lo(wv[i]), bf16_hi(wv[i]), xs, ld, m, col + c * 8 + 2 * i);
        }
    } else if constexpr (Q == Q_INT4) {
        float p[MT];
#pragma unroll
        for (int t = 0; t < MT; ++t) p[t] = 0.0f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint32_t wv[4] = {o.c[c].x, o.c[c].y, o.c[c].z, o.c[c].w};
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t t = (wv[w] >> (4 * j)) & 0x000F000Fu;
                    const float w0 = __uint_as_float(0x4B000000u | (t & 0xFFFFu)) - 8388616.0f;   // u - 8
                    const float w1 = __uint_as_float(0x4B000000u | (t >> 16)) - 8388616.0f;
                    fma_pair<MT>(p, w0, w1, xs, ld, m, col + c * 32 + w * 8 + 2 * j);
                }
        }
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[t] = fmaf(o.s, p[t], acc[t]);
    } else if constexpr (Q == Q_INT2) {
        float p[MT];
#pragma unroll
        for (int t = 0; t < MT; ++t) p[t] = 0.0f;
        const uint32_t wv[4] = {o.c[0].x, o.c[0].y, o.c[0].z, o.c[0].w};
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t t = (wv[w] >> (2 * j)) & 0x00030003u;
                const float w0 = __uint_as_float(0x4B000000u | (t & 0xFFFFu)) - o.zb;              // u - z
                const float w1 = __uint_as_float(0x4B000000u | (t >> 16)) - o.zb;
                fma_pair<MT>(p, w0, w1, xs, ld, m, col + w * 16 + 2 * j);
            }
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[t] = fmaf(o.s, p[t], acc[t]);
    } else {  // NVFP4: 16-column scale blocks, two words each
        const uint32_t wv[8] = {o.c[0].x, o.c[0].y, o.c[0].z, o.c[0].w, o.c[1].x, o.c[1].y, o.c[1].z, o.c[1].w};
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            float p[MT];
#pragma unroll
            for (int t = 0; t < MT; ++t) p[t] = 0.0f;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t t = wv[2 * b + h] >> (4 * j);
                    fma_pair<MT>(p, e2m1_to_f32(t & 0xFu), e2m1_to_f32((t >> 16) & 0xFu), xs, ld, m,
                                 col + 16 * b + 8 * h + 2 * j);
                }
            const float s = e4m3_to_f32((o.sb4 >> (8 * b)) & 0xffu);
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[t] = fmaf(s, p[t], acc[t]);
        }
    }
}

// One warp: rows r of the given matrices, k-blocks warp, warp+W, ...
template <int Q, int MT, int NM>
MOE_DEV void warp_rows_dot(float (&acc)[NM][MT], const MatPtr (&mats)[NM], int nb, int r, int KB, int G,
                           int warp, int nwarps, const float* xs, int ld, int m) {
    constexpr int KPW = Fmt<Q>::KPW;
    for (int kb0 = warp; kb0 < KB; kb0 += nwarps * KPW) {
        RowBlk<Q> blk[NM][KPW];
#pragma unroll
        for (int i = 0; i < KPW; ++i) {
            const int kb = kb0 + i * nwarps;
            if (kb < KB) {
#pragma unroll
                for (int q = 0; q < NM; ++q) load_row_blk<Q>(blk[q][i], mats[q], nb, kb, KB, G, r);
            }
        }
#pragma unroll
        for (int i = 0; i < KPW; ++i) {
            const int kb = kb0 + i * nwarps;
            if (kb < KB) {
#pragma unroll
                for (int q = 0; q < NM; ++q) dot_row_blk<Q, MT>(acc[q], blk[q][i], xs, ld, m, kb * kBlkK);
            }
        }
    }
}

// NVFP4 activations: replace a row of fp32 values by its W4A4 dequantized
// value q * s_b * g (same recipe as the activation quantization kernel).
MOE_DEV void fp4_requant_row_inplace(float* row, int K, float g, int tid, int nthreads) {
    for (int b = tid; b < K / kFp4Blk; b += nthreads) {
        float* v = row + b * kFp4Blk;
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
        float sbv = 0.0f, r = 0.0f;
        if (g != 0.0f) {
            sbv = e4m3_to_f32(f32_to_e4m3(__fdiv_rn(amax, __fmul_rn(6.0f, g))));
            r = (sbv == 0.0f) ? 0.0f : __fdiv_rn(1.0f, __fmul_rn(sbv, g));
        }
        const float scale = sbv * g;
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            const uint32_t c = f32x2_to_e2m1(__fmul_rn(v[i], r), __fmul_rn(v[i + 1], r));
            v[i] = e2m1_to_f32(c & 0xFu) * scale;
            v[i + 1] = e2m1_to_f32(c >> 4) * scale;
        }
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
template <int Q, int MT>
__global__ void __launch_bounds__(kGuThreads) k_dec_gateup(DecodeArgs a) {
    extern __shared__ float smem[];
    __shared__ Plan plan;
    __shared__ int tok[kDecMaxT];
    __shared__ int slot_of[kDecMaxT];
    const ExpertArgs& ex = a.ex;
    const int H = ex.H, I = ex.I, k = ex.k, T = a.T;
    const int n = T * k;
    const int rb_per_exp = I / 32;
    const int u = blockIdx.x / rb_per_exp;          // distinct expert, or the shared one when u == n
    const int ib = blockIdx.x % rb_per_exp;

    pdl_wait();                                      // ids come from the router
    pdl_launch_dependents();
    build_plan(a.ids, n, plan);
    const bool is_shared = (u == n);
    if (!is_shared && u >= plan.n_unique) return;
    int m;
    if (is_shared) {
        m = T;
        if (threadIdx.x < T) { tok[threadIdx.x] = threadIdx.x; slot_of[threadIdx.x] = threadIdx.x; }
    } else {
        m = min(item_tokens(plan.ids, n, k, plan.first[u], tok, slot_of), MT);
    }
    float* xs = smem;                                // [m][H] fp32
    float* red = smem + MT * H;                      // [8][2][MT][32]
    __syncthreads();
    const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(a.x);
    for (int i = threadIdx.x; i < m * H; i += blockDim.x) {
        const int t = i / H, c = i % H;
        xs[i] = __bfloat162float(x[(size_t)tok[t] * H + c]);
    }
    __syncthreads();
    if (Q == Q_NVFP4 && !is_shared) {
        for (int t = 0; t < m; ++t) fp4_requant_row_inplace(xs + t * H, H, ex.g_x, threadIdx.x, blockDim.x);
        __syncthreads();
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = H / kBlkK, G = H / kGroup;
    const int nb = ib / 4, r = (ib % 4) * 32 + lane;
    float acc[2][MT];
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[q][t] = 0.0f;
    int e = 0;
    if (is_shared) {
        const MatPtr mats[2] = {{ex.sh_gate, nullptr, nullptr}, {ex.sh_up, nullptr, nullptr}};
        warp_rows_dot<Q_BF16, MT, 2>(acc, mats, nb, r, KB, G, warp, kGuThreads / 32, xs, H, m);
    } else {
        e = plan.ids[plan.first[u]];
        if (e >= 0 && e < ex.E) {        // an id outside [0, E) contributes zero
            const MatPtr mats[2] = {expert_mat(ex.gate, e), expert_mat(ex.up, e)};
            warp_rows_dot<Q, MT, 2>(acc, mats, nb, r, KB, G, warp, kGuThreads / 32, xs, H, m);
        } else {
            e = 0;
        }
    }
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        red[((warp * 2 + 0) * MT + t) * 32 + lane] = acc[0][t];
        red[((warp * 2 + 1) * MT + t) * 32 + lane] = acc[1][t];
    }
    __syncthreads();
    const float gscale = (Q == Q_NVFP4 && !is_shared) ? ex.g_gate[e] : 1.0f;
    for (int i = threadIdx.x; i < m * 32; i += blockDim.x) {
        const int t = i / 32, rr = i % 32;
        float g = 0.0f, uu = 0.0f;
#pragma unroll
        for (int w = 0; w < kGuThreads / 32; ++w) {
            g += red[((w * 2 + 0) * MT + t) * 32 + rr];
            uu += red[((w * 2 + 1) * MT + t) * 32 + rr];
        }
        g *= gscale;
        uu *= gscale;
        const float act = g / (1.0f + expf(-g)) * uu;
        const int row = ib * 32 + rr;
        if (is_shared) a.a_sh[(size_t)t * I + row] = act;
        else a.a[(size_t)slot_of[t] * I + row] = act;
    }
}

// ------------------------------------------------------- down + combine
template <int Q, int MT>
__global__ void __launch_bounds__(kDnThreads) k_dec_down(DecodeArgs a) {
    extern __shared__ float smem[];
    __shared__ Plan plan;
    __shared__ int tok[kDecMaxT];
    __shared__ int slot_of[kDecMaxT];
    __shared__ int s_last;
    const ExpertArgs& ex = a.ex;
    const int H = ex.H, I = ex.I, k = ex.k, T = a.T;
    const int n = T * k;
    const int rbs = H / 32;
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
        m = min(item_tokens(plan.ids, n, k, plan.first[u], tok, slot_of), MT);
    }
    float* as = smem;                                // [m][I]
    float* red = smem + MT * I;                      // [4][MT][32]
    __syncthreads();
    pdl_wait();                                      // a comes from k_dec_gateup
    pdl_launch_dependents();
    for (int i = threadIdx.x; i < m * I; i += blockDim.x) {
        const int t = i / I, c = i % I;
        as[i] = is_shared ? __ldcg(a.a_sh + (size_t)t * I + c) : __ldcg(a.a + (size_t)slot_of[t] * I + c);
    }
    __syncthreads();
    if (Q == Q_NVFP4 && !is_shared) {
        for (int t = 0; t < m; ++t) fp4_requant_row_inplace(as + t * I, I, ex.g_a, threadIdx.x, blockDim.x);
        __syncthreads();
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = I / kBlkK, G = I / kGroup;
    const int nb = hb / 4, r = (hb % 4) * 32 + lane;
    float acc[1][MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[0][t] = 0.0f;
    int e = 0;
    if (is_shared) {
        const MatPtr mats[1] = {{ex.sh_down, nullptr, nullptr}};
        warp_rows_dot<Q_BF16, MT, 1>(acc, mats, nb, r, KB, G, warp, kDnThreads / 32, as, I, m);
    } else {
        e = plan.ids[plan.first[u]];
        if (e >= 0 && e < ex.E) {        // an id outside [0, E) contributes zero
            const MatPtr mats[1] = {expert_mat(ex.down, e)};
            warp_rows_dot<Q, MT, 1>(acc, mats, nb, r, KB, G, warp, kDnThreads / 32, as, I, m);
        } else {
            e = 0;
        }
    }
#pragma unroll
    for (int t = 0; t < MT; ++t) red[(warp * MT + t) * 32 + lane] = acc[0][t];
    __syncthreads();
    const float dscale = (Q == Q_NVFP4 && !is_shared) ? ex.g_down[e] : 1.0f;
    for (int i = threadIdx.x; i < m * 32; i += blockDim.x) {
        const int t = i / 32, rr = i % 32;
        float o = 0.0f;
#pragma unroll
        for (int w = 0; w < kDnThreads / 32; ++w) o += red[(w * MT + t) * 32 + rr];
        o *= dscale;
        const int h = hb * 32 + rr;
        if (is_shared) a.part_sh[(size_t)t * H + h] = o;
        else a.part[(size_t)slot_of[t] * H + h] = __ldcg(a.w + slot_of[t]) * o;
    }
    // the last item of this row block to finish combines
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(a.counters + hb, 1u) == (unsigned)items_per_rb - 1u);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(a.y);
    for (int i = threadIdx.x; i < T * 32; i += blockDim.x) {
        const int t = i / 32, h = hb * 32 + i % 32;
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

template <int Q, int MT>
static cudaError_t launch_decode_qmt(const DecodeArgs& a, cudaStream_t st) {
    const ExpertArgs& ex = a.ex;
    const int n = a.T * ex.k;
    const int items_gu = (n + (ex.sh_gate ? 1 : 0)) * (ex.I / 32);
    const int items_dn = (n + (ex.sh_down ? 1 : 0)) * (ex.H / 32);
    const size_t smem_gu = (size_t)(MT * ex.H + 8 * 2 * MT * 32) * sizeof(float);
    const size_t smem_dn = (size_t)(MT * ex.I + 4 * MT * 32) * sizeof(float);
    cudaError_t err = cudaFuncSetAttribute(k_dec_gateup<Q, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem_gu);
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(k_dec_down<Q, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dn);
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
    err = cudaLaunchKernelEx(&cfg, k_dec_gateup<Q, MT>, a);
    if (err != cudaSuccess) return err;
    if (a.ev_mid) {
        err = cudaEventRecord(a.ev_mid, st);
        if (err != cudaSuccess) return err;
    }
    cfg.gridDim = dim3(items_dn);
    cfg.blockDim = dim3(kDnThreads);
    cfg.dynamicSmemBytes = smem_dn;
    err = cudaLaunchKernelEx(&cfg, k_dec_down<Q, MT>, a);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

template <int Q>
static cudaError_t launch_decode_q(const DecodeArgs& a, cudaStream_t st) {
    if (a.T <= 1) return launch_decode_qmt<Q, 1>(a, st);
    if (a.T <= 2) return launch_decode_qmt<Q, 2>(a, st);
    return launch_decode_qmt<Q, 4>(a, st);
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
