// Decode path of the expert computation (up to 16 tokens per launch):
// memory-bound GEMVs that stream each selected expert's packed weights once,
// dequantize in registers and multiply on the tensor cores.
//
// The pages' decode kernel reads each expert "in place" from an N-contiguous
// packed layout ("Qwen3.8-Flash-Next on one 24 GB GPU", "What the patch
// does"), and expert GEMV dominates the per-stream decode cost
// ("Qwen3.8-Flash-Next-FP6-INT8", "Step budget and hardware floors").
//
// One warp computes 16 weight rows x 8 token columns with mma.sync m16n8k16
// (bf16 operands, fp32 accumulation); 9 to 16 tokens take a second group of
// 8 columns from the same dequantized fragments (the multi-token verify
// shapes of speculative decoding: "meshapplied/Qwen3.8-Flash-Next-NVFP4-
// Latest", NEXTN results; "Qwen3.8-Flash-Next-FP6-INT8", "Quantization
// quality": GEMV up to M = 16, GEMM above).  The 16 "k" slots of each MMA are
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
#include "decode_common.cuh"

namespace moe {

constexpr int kGuThreads = 256;       // 8 warps split K
constexpr int kDnThreads = 128;       // 4 warps split K
constexpr int kDecMaxT2 = 16;         // tokens per launch: NG = 2 groups of 8 MMA columns

bool decode_supported(int T, int k) { return T >= 1 && T <= kDecMaxT2 && T * k <= kDecMaxSlots; }

// ------------------------------------------------------------- gate / up
// NG: groups of 8 token columns (T <= 8 NG)
template <int Q, int NG>
__global__ void __launch_bounds__(kGuThreads, NG == 1 ? 3 : 2) k_dec_gateup(DecodeArgs a) {
    constexpr int MT = 8 * NG;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ Plan plan;
    __shared__ int tok[MT];
    __shared__ int slot_of[MT];
    const ExpertArgs& ex = a.ex;
    const int H = ex.H, I = ex.I, k = ex.k, T = a.T;
    const int n = T * k;
    const int rb_per_exp = I / 16;
    const int u = blockIdx.x / rb_per_exp;          // distinct expert, or the shared one when u == n
    const int rb16 = blockIdx.x % rb_per_exp;
    const bool is_shared = (u == n);

    // Up to 8 tokens: the activations do not depend on the routing, so all T
    // token rows are staged (row t = token t, rows T..MT zero) before waiting
    // for the router.  More tokens: an item stages only its own tokens' rows
    // (row j = the item's j-th token), after the routing is known.
    const int ldx = H + kXPad;
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem_raw);                   // [MT+1][ldx]
    float* red = reinterpret_cast<float*>(smem_raw + (size_t)(MT + 1) * ldx * 2);     // [8][2][16][MT]
    if (threadIdx.x < MT) tok[threadIdx.x] = threadIdx.x;
    __syncthreads();
    const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(a.x);
    auto stage_x = [&](int m_rows) {
        if (Q == Q_NVFP4 && !is_shared)
            stage_rows_fp4_from_bf16(xs, ldx, x, H, tok, m_rows, ex.g_x, threadIdx.x, blockDim.x, MT);
        else
            stage_rows_bf16(xs, ldx, x, H, tok, m_rows, threadIdx.x, blockDim.x, MT);
    };
    if (NG == 1 || is_shared) stage_x(T);
    for (int i = threadIdx.x; i < ldx / 8; i += blockDim.x)
        reinterpret_cast<uint4*>(xs + MT * ldx)[i] = make_uint4(0, 0, 0, 0);

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
        m = item_tokens(plan.ids, n, k, plan.first[u], tok, slot_of, MT);
        if (NG > 1) {
            __syncthreads();
            stage_x(m);                          // row j = token tok[j]
        }
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int KB = H / kBlkK, G = scale_stride(Q, H);
    const int r0 = rb16 * 16;
    const int nb = r0 / kBlkN, rl = r0 % kBlkN + g;
    // item column 8 gq + g: token tok[8 gq + g], staged in row tok[...] (all
    // tokens staged) or in row 8 gq + g (the item's tokens staged)
    const bool item_rows = NG > 1 && !is_shared;
    const __nv_bfloat16* xrows[NG];
#pragma unroll
    for (int gq = 0; gq < NG; ++gq) {
        const int j = 8 * gq + g;
        xrows[gq] = xs + (j < m ? (item_rows ? j : tok[j]) : MT) * ldx;
    }
    float acc[2][NG][4] = {};
    int e = 0;
    if (is_shared) {
        const MatPtr mats[2] = {{ex.sh_gate, nullptr, nullptr}, {ex.sh_up, nullptr, nullptr}};
        warp_rows<Q_BF16, 2, NG>(acc, mats, nb, rl, KB, G, warp, kGuThreads / 32, xrows, c);
    } else {
        e = plan.ids[plan.first[u]];
        if (e >= 0 && e < ex.E) {        // an id outside [0, E) contributes zero
            const MatPtr mats[2] = {expert_mat(ex.gate, e), expert_mat(ex.up, e)};
            warp_rows<Q, 2, NG>(acc, mats, nb, rl, KB, G, warp, kGuThreads / 32, xrows, c);
        } else {
            e = 0;
        }
    }
    // red[warp][mat][row 16][token MT]
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int gq = 0; gq < NG; ++gq) {
            float* r = red + ((warp * 2 + q) * 16) * MT + 8 * gq;
            r[g * MT + 2 * c] = acc[q][gq][0];
            r[g * MT + 2 * c + 1] = acc[q][gq][1];
            r[(g + 8) * MT + 2 * c] = acc[q][gq][2];
            r[(g + 8) * MT + 2 * c + 1] = acc[q][gq][3];
        }
    __syncthreads();
    const float gscale = (Q == Q_NVFP4 && !is_shared) ? ex.g_gate[e] * ex.g_x : 1.0f;
    if (threadIdx.x < 16 * MT) {
        const int row = threadIdx.x / MT, t = threadIdx.x % MT;
        if (t < m) {
            float gg = 0.0f, uu = 0.0f;
#pragma unroll
            for (int w = 0; w < kGuThreads / 32; ++w) {
                gg += red[((w * 2 + 0) * 16 + row) * MT + t];
                uu += red[((w * 2 + 1) * 16 + row) * MT + t];
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
template <int Q, int NG>
__global__ void __launch_bounds__(kDnThreads, NG == 1 ? 10 : 8) k_dec_down(DecodeArgs a) {
    constexpr int MT = 8 * NG;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ Plan plan;
    __shared__ int tok[MT];
    __shared__ int slot_of[MT];
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
        m = item_tokens(plan.ids, n, k, plan.first[u], tok, slot_of, MT);
    }
    const int ldx = I + kXPad;
    __nv_bfloat16* as = reinterpret_cast<__nv_bfloat16*>(smem_raw);                   // [MT][ldx]
    float* red = reinterpret_cast<float*>(smem_raw + (size_t)MT * ldx * 2);           // [4][16][MT]
    __syncthreads();
    pdl_wait();                                      // a comes from k_dec_gateup
    pdl_launch_dependents();
    stage_rows_f32(as, ldx, is_shared ? a.a_sh : a.a, I, slot_of, m, Q == Q_NVFP4 && !is_shared, ex.g_a,
                   threadIdx.x, blockDim.x, MT);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int KB = I / kBlkK, G = scale_stride(Q, I);
    const int h0 = hb * 16;
    const int nb = h0 / kBlkN, rl = h0 % kBlkN + g;
    const __nv_bfloat16* xrows[NG];
#pragma unroll
    for (int gq = 0; gq < NG; ++gq) xrows[gq] = as + (8 * gq + g) * ldx;
    float acc[1][NG][4] = {};
    int e = 0;
    if (is_shared) {
        const MatPtr mats[1] = {{ex.sh_down, nullptr, nullptr}};
        warp_rows<Q_BF16, 1, NG>(acc, mats, nb, rl, KB, G, warp, kDnThreads / 32, xrows, c);
    } else {
        e = plan.ids[plan.first[u]];
        if (e >= 0 && e < ex.E) {        // an id outside [0, E) contributes zero
            const MatPtr mats[1] = {expert_mat(ex.down, e)};
            warp_rows<Q, 1, NG>(acc, mats, nb, rl, KB, G, warp, kDnThreads / 32, xrows, c);
        } else {
            e = 0;
        }
    }
#pragma unroll
    for (int gq = 0; gq < NG; ++gq) {
        float* r = red + (warp * 16) * MT + 8 * gq;
        r[g * MT + 2 * c] = acc[0][gq][0];
        r[g * MT + 2 * c + 1] = acc[0][gq][1];
        r[(g + 8) * MT + 2 * c] = acc[0][gq][2];
        r[(g + 8) * MT + 2 * c + 1] = acc[0][gq][3];
    }
    __syncthreads();
    const float dscale = (Q == Q_NVFP4 && !is_shared) ? ex.g_down[e] * ex.g_a : 1.0f;
    for (int i = threadIdx.x; i < 16 * MT; i += kDnThreads) {   // 16 rows x MT tokens
        const int row = i / MT, t = i % MT;
        if (t < m) {
            float o = 0.0f;
#pragma unroll
            for (int w = 0; w < kDnThreads / 32; ++w) o += red[(w * 16 + row) * MT + t];
            o *= dscale;
            const int h = h0 + row;
            if (is_shared) a.part_sh[(size_t)t * H + h] = o;
            else a.part[(size_t)slot_of[t] * H + h] = __ldcg(a.w + slot_of[t]) * o;
        }
    }
    // the last item of this row block to finish combines
    __syncthreads();
    if (threadIdx.x == 0) s_last = (ticket_acq_rel(a.counters + hb) == (unsigned)items_per_rb - 1u);
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

template <int Q, int NG>
static cudaError_t launch_decode_qg(const DecodeArgs& a, cudaStream_t st) {
    constexpr int MT = 8 * NG;
    const ExpertArgs& ex = a.ex;
    const int n = a.T * ex.k;
    const int items_gu = (n + (ex.sh_gate ? 1 : 0)) * (ex.I / 16);
    const int items_dn = (n + (ex.sh_down ? 1 : 0)) * (ex.H / 16);
    const size_t smem_gu = (size_t)(MT + 1) * (ex.H + kXPad) * 2 + 8 * 2 * 16 * MT * sizeof(float);
    const size_t smem_dn = (size_t)MT * (ex.I + kXPad) * 2 + 4 * 16 * MT * sizeof(float);
    cudaError_t err =
        cudaFuncSetAttribute(k_dec_gateup<Q, NG>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_gu);
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(k_dec_down<Q, NG>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dn);
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
    err = cudaLaunchKernelEx(&cfg, k_dec_gateup<Q, NG>, a);
    if (err != cudaSuccess) return err;
    if (a.ev_mid) {
        err = cudaEventRecord(a.ev_mid, st);
        if (err != cudaSuccess) return err;
    }
    cfg.gridDim = dim3(items_dn);
    cfg.blockDim = dim3(kDnThreads);
    cfg.dynamicSmemBytes = smem_dn;
    err = cudaLaunchKernelEx(&cfg, k_dec_down<Q, NG>, a);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

// 1 to 8 tokens: one group of 8 MMA columns; 9 to 16: two
template <int Q>
static cudaError_t launch_decode_q(const DecodeArgs& a, cudaStream_t st) {
    return a.T <= 8 ? launch_decode_qg<Q, 1>(a, st) : launch_decode_qg<Q, 2>(a, st);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
    switch (a.ex.quant) {
        case Q_INT4: return launch_decode_q<Q_INT4>(a, st);
        case Q_INT4G32: return launch_decode_q<Q_INT4G32>(a, st);
        case Q_FP8: return launch_decode_q<Q_FP8>(a, st);
        case Q_FP6: return launch_decode_q<Q_FP6>(a, st);
        case Q_INT2: return launch_decode_q<Q_INT2>(a, st);
        case Q_NVFP4: return launch_decode_q<Q_NVFP4>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
