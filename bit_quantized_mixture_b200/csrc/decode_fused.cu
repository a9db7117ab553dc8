// Whole decode step of the layer (up to 8 tokens) in one persistent kernel:
// router GEMV and top-k, every selected expert's gate/up and down GEMV, the
// shared expert and the combine.
//
// Separate kernels leave the GPU idle between launches and put a chain of
// dependent memory round trips (ids -> plan -> weights -> partials) at the
// start of each; at decode sizes those fixed costs, not bytes, set the step
// time.  Here one cooperative grid (one 16-warp CTA per SM) walks three
// phases separated by two grid-wide barriers:
//   phase 0: router rows (one per warp) and the shared expert's gate/up rows
//            (it needs nothing from the router);
//   phase 1: every CTA computes the top-k of all tokens from the logits
//            itself (so no third barrier is needed), builds the list of
//            distinct experts and runs its share of their gate/up rows;
//   phase 2: down rows of every selected expert and of the shared expert,
//            each 128-row unit adding its routing-weighted partials; the last
//            unit of a row block (ticket counter, no waiting) sums
//            y_t = sum_j part[t*k+j] + shared_t in fixed j order.
// The GEMV arithmetic is that of decode.cu (mma.sync m16n8k16 on exact
// dequantized operands, group scales on fp32 accumulators).  The barriers
// wait a bounded time; on timeout the kernel records an error code, skips
// the remaining phases and returns (moe_sync_status reports it).
#include "decode_common.cuh"

namespace moe {

constexpr int kFWarps = 16;
constexpr int kFThreads = kFWarps * 32;
constexpr long long kBarrierLimitCycles = 4000000000LL;   // about 2 s

// Grid-wide barrier on {arrivals, generation}: the last CTA to arrive resets
// the count and advances the generation; the others spin on it (bounded).
MOE_DEV bool grid_barrier(unsigned int* bar, int* err, volatile int* abort_s) {
    __syncthreads();
    if (threadIdx.x == 0) {
        volatile unsigned int* gen = bar + 1;
        const unsigned int g0 = *gen;
        __threadfence();
        if (atomicAdd(bar, 1u) == gridDim.x - 1) {
            atomicExch(bar, 0u);
            __threadfence();
            atomicAdd(bar + 1, 1u);
        } else {
            const long long t0 = clock64();
            while (*gen == g0) {
                if (clock64() - t0 > kBarrierLimitCycles) {
                    *abort_s = 1;
                    if (err) atomicCAS(err, 0, 20);
                    break;
                }
                __nanosleep(32);
            }
        }
        __threadfence();
    }
    __syncthreads();
    return *abort_s == 0;
}

// One warp: logits[t][e] = x_t . Wr[e] for t < T (x staged as bf16 rows).
MOE_DEV void router_row(const uint8_t* __restrict__ wr, int e, int H, int T, const __nv_bfloat16* xs, int ldx,
                        float* __restrict__ logits, int E) {
    const int lane = threadIdx.x & 31;
    const uint8_t* row = wr + (size_t)e * H * 2;
    float acc[kDecMaxT];
#pragma unroll
    for (int t = 0; t < kDecMaxT; ++t) acc[t] = 0.0f;
    for (int c0 = 0; c0 < H / 8; c0 += 32 * 8) {
        uint4 q[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = c0 + lane + 32 * u;
            q[u] = (c < H / 8) ? ldg_stream_v4(row + (size_t)c * 16) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = c0 + lane + 32 * u;
            if (c < H / 8) {
                const uint32_t wv[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
                for (int t = 0; t < kDecMaxT; ++t) {
                    if (t < T) {
                        const uint4 xq = *reinterpret_cast<const uint4*>(xs + t * ldx + c * 8);
                        const uint32_t xv[4] = {xq.x, xq.y, xq.z, xq.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            acc[t] = fmaf(bf16_lo(wv[i]), bf16_lo(xv[i]), acc[t]);
                            acc[t] = fmaf(bf16_hi(wv[i]), bf16_hi(xv[i]), acc[t]);
                        }
                    }
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < kDecMaxT; ++t) {
        if (t < T) {
            const float s = warp_sum(acc[t]);
            if (lane == 0) logits[(size_t)t * E + e] = s;
        }
    }
}

// Top-k of one token by one warp (same rule as route.cu), results in smem.
MOE_DEV uint32_t fkey(float v) {
    const uint32_t b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
MOE_DEV void warp_topk_smem(const float* __restrict__ row, int E, int k, int* ids, float* wts) {
    const int lane = threadIdx.x & 31;
    uint32_t key[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int e = lane + 32 * i;
        key[i] = (e < E) ? fkey(__ldcg(row + e)) : 0u;
    }
    uint32_t live = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) live |= ((lane + 32 * i) < E ? 1u : 0u) << i;
    float my_val = 0.0f, lmax = 0.0f;
    int my_idx = 0;
    for (int j = 0; j < k; ++j) {
        uint32_t best = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if ((live >> i) & 1u) best = max(best, key[i]);
        const uint32_t top = __reduce_max_sync(0xffffffffu, best);
        uint32_t mine = 0xffffffffu;
#pragma unroll
        for (int i = 31; i >= 0; --i)
            if (((live >> i) & 1u) && key[i] == top) mine = (uint32_t)(lane + 32 * i);
        const uint32_t e = __reduce_min_sync(0xffffffffu, mine);
        if ((int)(e & 31u) == lane) live &= ~(1u << (e >> 5));
        const float v = __uint_as_float((top & 0x80000000u) ? (top & 0x7fffffffu) : ~top);
        if (j == 0) lmax = v;
        if (lane == j) { my_val = v; my_idx = (int)e; }
    }
    const float ex = (lane < k) ? expf(my_val - lmax) : 0.0f;
    const float sum = warp_sum(ex);
    if (lane < k) {
        ids[lane] = my_idx;
        wts[lane] = __fdiv_rn(ex, sum);
    }
}

// Rows of one unit: RB row blocks of 16 rows starting at r0; the 16 warps are
// (row block rbi = warp % RB) x (K split ks = warp / RB of 16/RB); partials
// of each warp go to red[warp][NM][16][8].
template <int Q, int NM, int RB>
MOE_DEV void unit_gemv(const MatPtr (&mats)[NM], int r0, int K, const __nv_bfloat16* xrow, float* red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int rbi = warp % RB, ks = warp / RB;
    const int r = r0 + rbi * 16;
    const int nb = r / kBlkN, rl = r % kBlkN + g;
    float acc[NM][4];
#pragma unroll
    for (int q = 0; q < NM; ++q)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[q][i] = 0.0f;
    warp_rows<Q, NM>(acc, mats, nb, rl, K / kBlkK, K / kGroup, ks, kFWarps / RB, xrow, c);
#pragma unroll
    for (int q = 0; q < NM; ++q) {
        float* rr = red + ((warp * NM + q) * 16) * 8;
        rr[g * 8 + 2 * c] = acc[q][0];
        rr[g * 8 + 2 * c + 1] = acc[q][1];
        rr[(g + 8) * 8 + 2 * c] = acc[q][2];
        rr[(g + 8) * 8 + 2 * c + 1] = acc[q][3];
    }
}

template <int Q>
__global__ void __launch_bounds__(kFThreads, 1) k_decode_fused(FusedArgs f) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ Plan plan;
    __shared__ int ids_s[kDecMaxSlots];
    __shared__ float w_s[kDecMaxSlots];
    __shared__ int tok[kDecMaxT], slot_of[kDecMaxT], ident[kDecMaxT];
    __shared__ int s_last;
    __shared__ volatile int abort_s;
    const DecodeArgs& a = f.d;
    const ExpertArgs& ex = a.ex;
    const int H = ex.H, I = ex.I, k = ex.k, E = ex.E, T = a.T;
    const int n = T * k;
    const int ldx = H + kXPad, lda = I + kXPad;
    const bool fp4 = (Q == Q_NVFP4);
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem_raw);                          // [9][ldx] raw x
    __nv_bfloat16* xq = xs + (size_t)(kDecMaxT + 1) * ldx;                                   // [9][ldx] W4A4 x
    __nv_bfloat16* as = xq + (size_t)(kDecMaxT + 1) * ldx;                                   // [9][lda]
    float* red = reinterpret_cast<float*>(as + (size_t)(kDecMaxT + 1) * lda);                 // [16][2][16][8]
    if (threadIdx.x == 0) abort_s = 0;
    if (threadIdx.x < kDecMaxT) ident[threadIdx.x] = threadIdx.x;
    __syncthreads();

    // ---- stage activations (rows t < T, rows T..8 zero)
    const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(a.x);
    stage_rows_bf16(xs, ldx, x, H, ident, T, threadIdx.x, blockDim.x);
    if (fp4) stage_rows_fp4_from_bf16(xq, ldx, x, H, ident, T, ex.g_x, threadIdx.x, blockDim.x);
    for (int i = threadIdx.x; i < ldx / 8; i += blockDim.x) {
        reinterpret_cast<uint4*>(xs + kDecMaxT * ldx)[i] = make_uint4(0, 0, 0, 0);
        reinterpret_cast<uint4*>(xq + kDecMaxT * ldx)[i] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2;

    // ---- phase 0: router rows + shared gate/up rows
    {
        const int router_units = f.wr ? (E + kFWarps - 1) / kFWarps : 0;
        const int shared_units = ex.sh_gate ? I / 16 : 0;
        for (int u = blockIdx.x; u < router_units + shared_units; u += gridDim.x) {
            if (u < router_units) {
                const int e = u * kFWarps + warp;
                if (e < E) router_row(reinterpret_cast<const uint8_t*>(f.wr), e, H, T, xs, ldx, f.logits, E);
            } else {
                const int r0 = (u - router_units) * 16;
                const MatPtr mats[2] = {{ex.sh_gate, nullptr, nullptr}, {ex.sh_up, nullptr, nullptr}};
                const __nv_bfloat16* xrow = xs + (g < T ? g : kDecMaxT) * ldx;
                unit_gemv<Q_BF16, 2, 1>(mats, r0, H, xrow, red);
                __syncthreads();
                if (threadIdx.x < 16 * kDecMaxT) {
                    const int row = threadIdx.x / kDecMaxT, t = threadIdx.x % kDecMaxT;
                    if (t < T) {
                        float gg = 0.0f, uu = 0.0f;
                        for (int w = 0; w < kFWarps; ++w) {
                            gg += red[((w * 2 + 0) * 16 + row) * 8 + t];
                            uu += red[((w * 2 + 1) * 16 + row) * 8 + t];
                        }
                        a.a_sh[(size_t)t * I + r0 + row] = gg / (1.0f + expf(-gg)) * uu;
                    }
                }
                __syncthreads();
            }
        }
    }
    if (f.wr && !grid_barrier(f.bar, f.err, &abort_s)) return;

    // ---- phase 1: top-k (every CTA), plan, routed gate/up rows
    if (f.wr) {
        for (int t = warp; t < T; t += kFWarps)
            warp_topk_smem(f.logits + (size_t)t * E, E, k, ids_s + t * k, w_s + t * k);
        __syncthreads();
        if (blockIdx.x == 0)
            for (int s = threadIdx.x; s < n; s += blockDim.x) { f.ids_out[s] = ids_s[s]; f.w_out[s] = w_s[s]; }
    } else {
        for (int s = threadIdx.x; s < n; s += blockDim.x) { ids_s[s] = __ldcg(a.ids + s); w_s[s] = __ldcg(a.w + s); }
    }
    __syncthreads();
    for (int s = threadIdx.x; s < n; s += blockDim.x) plan.ids[s] = ids_s[s];
    __syncthreads();
    for (int s = threadIdx.x; s < n; s += blockDim.x) {
        const int e = plan.ids[s];
        bool fst = true;
        for (int q = 0; q < s; ++q) fst = fst && (plan.ids[q] != e);
        plan.is_first[s] = fst;
    }
    __syncthreads();
    if (warp == 0) {
        int base = 0;
        for (int s0 = 0; s0 < n; s0 += 32) {
            const int s = s0 + lane;
            const bool fst = (s < n) && plan.is_first[s];
            const unsigned m = __ballot_sync(0xffffffffu, fst);
            if (fst) plan.first[base + __popc(m & ((1u << lane) - 1u))] = s;
            base += __popc(m);
        }
        if (lane == 0) plan.n_unique = base;
    }
    __syncthreads();
    const int nu = plan.n_unique;
    {
        const int units = nu * (I / 16);
        for (int u = blockIdx.x; u < units; u += gridDim.x) {
            const int ui = u / (I / 16), r0 = (u % (I / 16)) * 16;
            const int m = item_tokens(plan.ids, n, k, plan.first[ui], tok, slot_of);
            __syncthreads();
            const int e = plan.ids[plan.first[ui]];
            const bool valid = e >= 0 && e < E;
            const __nv_bfloat16* xb = fp4 ? xq : xs;
            const __nv_bfloat16* xrow = xb + (g < m ? tok[g] : kDecMaxT) * ldx;
            if (valid) {
                const MatPtr mats[2] = {expert_mat(ex.gate, e), expert_mat(ex.up, e)};
                unit_gemv<Q, 2, 1>(mats, r0, H, xrow, red);
            }
            __syncthreads();
            if (threadIdx.x < 16 * kDecMaxT) {
                const int row = threadIdx.x / kDecMaxT, t = threadIdx.x % kDecMaxT;
                if (t < m) {
                    float gg = 0.0f, uu = 0.0f;
                    if (valid)
                        for (int w = 0; w < kFWarps; ++w) {
                            gg += red[((w * 2 + 0) * 16 + row) * 8 + t];
                            uu += red[((w * 2 + 1) * 16 + row) * 8 + t];
                        }
                    const float sc = (fp4 && valid) ? ex.g_gate[e] * ex.g_x : 1.0f;
                    gg *= sc;
                    uu *= sc;
                    a.a[(size_t)slot_of[t] * I + r0 + row] = gg / (1.0f + expf(-gg)) * uu;
                }
            }
            __syncthreads();
        }
    }
    if (!grid_barrier(f.bar, f.err, &abort_s)) return;

    // ---- phase 2: down rows (128 per unit: 8 row blocks x 2 K halves) + combine
    {
        constexpr int RB = 8;
        const int rb128 = H / 128;
        const int items_per_rb = nu + (ex.sh_down ? 1 : 0);
        const int units = items_per_rb * rb128;
        for (int u = blockIdx.x; u < units; u += gridDim.x) {
            const int ui = u / rb128, hb = u % rb128, h0 = hb * 128;
            const bool is_shared = (ui == nu);
            int m, e = 0;
            if (is_shared) {
                m = T;
                if (threadIdx.x < kDecMaxT) { tok[threadIdx.x] = threadIdx.x; slot_of[threadIdx.x] = threadIdx.x; }
            } else {
                m = item_tokens(plan.ids, n, k, plan.first[ui], tok, slot_of);
                e = plan.ids[plan.first[ui]];
            }
            __syncthreads();
            const bool valid = is_shared || (e >= 0 && e < E);
            stage_rows_f32(as, lda, is_shared ? a.a_sh : a.a, I, slot_of, m, fp4 && !is_shared, ex.g_a, threadIdx.x,
                           blockDim.x);
            __syncthreads();
            const __nv_bfloat16* xrow = as + (g < m ? g : kDecMaxT) * lda;
            if (is_shared) {
                const MatPtr mats[1] = {{ex.sh_down, nullptr, nullptr}};
                unit_gemv<Q_BF16, 1, RB>(mats, h0, I, xrow, red);
            } else if (valid) {
                const MatPtr mats[1] = {expert_mat(ex.down, e)};
                unit_gemv<Q, 1, RB>(mats, h0, I, xrow, red);
            }
            __syncthreads();
            const float dscale = (fp4 && !is_shared && valid) ? ex.g_down[e] * ex.g_a : 1.0f;
            for (int i = threadIdx.x; i < 128 * kDecMaxT; i += blockDim.x) {
                const int row = i / kDecMaxT, t = i % kDecMaxT;
                if (t < m) {
                    const int rbi = row / 16, rr = row % 16;
                    float o = 0.0f;
                    if (valid)
                        for (int ks = 0; ks < kFWarps / RB; ++ks) o += red[((ks * RB + rbi) * 16 + rr) * 8 + t];
                    o *= dscale;
                    const int h = h0 + row;
                    if (is_shared) a.part_sh[(size_t)t * H + h] = o;
                    else a.part[(size_t)slot_of[t] * H + h] = w_s[slot_of[t]] * o;
                }
            }
            // the last unit of this 128-row block to finish sums the slots
            __syncthreads();
            if (threadIdx.x == 0) {
                __threadfence();
                s_last = (atomicAdd(a.counters + hb, 1u) == (unsigned)items_per_rb - 1u);
                if (s_last) __threadfence();
            }
            __syncthreads();
            if (s_last) {
                __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(a.y);
                for (int i = threadIdx.x; i < T * 128; i += blockDim.x) {
                    const int t = i / 128, hh = h0 + i % 128;
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = (j < k) ? __ldcg(a.part + (size_t)(t * k + j) * H + hh) : 0.0f;
                    float sum = 0.0f;
#pragma unroll
                    for (int j = 0; j < 32; ++j) sum += v[j];          // fixed order j = 0 .. k-1
                    if (ex.sh_down) sum += __ldcg(a.part_sh + (size_t)t * H + hh);
                    y[(size_t)t * H + hh] = __float2bfloat16_rn(sum);
                }
                __syncthreads();
                if (threadIdx.x == 0) a.counters[hb] = 0u;
            }
            __syncthreads();
        }
    }
}

size_t fused_smem_bytes(int H, int I) {
    const size_t xbuf = (size_t)(kDecMaxT + 1) * (H + kXPad) * 2;
    const size_t abuf = (size_t)(kDecMaxT + 1) * (I + kXPad) * 2;
    return 2 * xbuf + abuf + (size_t)kFWarps * 2 * 16 * 8 * sizeof(float);
}

template <int Q>
static cudaError_t launch_fused_q(const FusedArgs& f, cudaStream_t st, int grid) {
    const size_t smem = fused_smem_bytes(f.d.ex.H, f.d.ex.I);
    cudaError_t err = cudaFuncSetAttribute(k_decode_fused<Q>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, k_decode_fused<Q>, f);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

cudaError_t launch_decode_fused(const FusedArgs& f, cudaStream_t st) {
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
    switch (f.d.ex.quant) {
        case Q_INT4: return launch_fused_q<Q_INT4>(f, st, sms);
        case Q_INT2: return launch_fused_q<Q_INT2>(f, st, sms);
        case Q_NVFP4: return launch_fused_q<Q_NVFP4>(f, st, sms);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
