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

// Grid-wide barrier on one monotonically increasing 64-bit arrival count:
// arrival i belongs to barrier episode i / gridDim.x, and a CTA leaves once
// the count reaches the end of its episode.  One atomic per CTA, no reset;
// release on arrival and acquire on the polls order the writes before the
// barrier against the reads after it.  Bounded: on timeout the CTA records
// an error code and stops.
MOE_DEV unsigned long long ld_acquire64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
MOE_DEV unsigned long long atom_add_release64(unsigned long long* p, unsigned long long v) {
    unsigned long long old;
    asm volatile("atom.add.release.gpu.global.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
    return old;
}
MOE_DEV bool grid_barrier(unsigned long long* bar, int* err, volatile int* abort_s) {
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned long long n = gridDim.x;
        const unsigned long long ticket = atom_add_release64(bar, 1ull);
        const unsigned long long target = (ticket / n + 1) * n;
        const long long t0 = clock64();
        while (ld_acquire64(bar) < target) {
            if (clock64() - t0 > kBarrierLimitCycles) {
                *abort_s = 1;
                if (err) atomicCAS(err, 0, 20);
                break;
            }
        }
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

// Top-k of one token by one warp (rule of route.cu: logit descending, expert
// index ascending; weights = softmax over the selected).  Lane l holds the
// experts l, l+32, ...; each lane caches its best remaining (key, expert), so
// a round is two warp reductions plus a rescan by the winning lane only.
MOE_DEV uint32_t fkey(float v) {
    const uint32_t b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
MOE_DEV float fkey_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}
MOE_DEV void warp_topk_smem(const float* __restrict__ row, int E, int k, int* ids, float* wts) {
    const int lane = threadIdx.x & 31;
    uint32_t key[32];
    uint32_t live = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int e = lane + 32 * i;
        key[i] = (e < E) ? fkey(__ldcg(row + e)) : 0u;
        live |= (e < E ? 1u : 0u) << i;
    }
    uint32_t bk = 0, bi = 0xffffffffu;
#pragma unroll
    for (int i = 0; i < 32; ++i)
        if (((live >> i) & 1u) && key[i] > bk) { bk = key[i]; bi = (uint32_t)(lane + 32 * i); }
    float my_val = 0.0f, lmax = 0.0f;
    int my_idx = 0;
    for (int j = 0; j < k; ++j) {
        const uint32_t top = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t e = __reduce_min_sync(0xffffffffu, (bk == top) ? bi : 0xffffffffu);
        const float v = fkey_value(top);
        if (j == 0) lmax = v;
        if (lane == j) { my_val = v; my_idx = (int)e; }
        if (bi == e) {                                   // the owner drops it and rescans
            live &= ~(1u << (e >> 5));
            bk = 0; bi = 0xffffffffu;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (((live >> i) & 1u) && key[i] > bk) { bk = key[i]; bi = (uint32_t)(lane + 32 * i); }
        }
    }
    const float ex = (lane < k) ? expf(my_val - lmax) : 0.0f;
    const float sum = warp_sum(ex);
    if (lane < k) {
        ids[lane] = my_idx;
        wts[lane] = __fdiv_rn(ex, sum);
    }
}

// Named barrier of one 4-warp group (ids 1..4; 0 is __syncthreads).
MOE_DEV void group_sync(int group) { asm volatile("bar.sync %0, 128;" ::"r"(group + 1) : "memory"); }

// Tokens of the item whose first slot is s0 (slot order), written by the
// group's first thread; see item_tokens.
MOE_DEV int group_item_tokens(const int* __restrict__ ids, int n, int k, int s0, int* tok, int* slot, bool writer) {
    const int e0 = ids[s0];
    int c = 0;
    for (int s = s0; s < n && c < kDecMaxT; ++s) {
        if (ids[s] == e0) {
            if (writer) { tok[c] = s / k; slot[c] = s; }
            ++c;
        }
    }
    return c;
}

constexpr int kGroups = kFWarps / 4;

template <int Q>
__global__ void __launch_bounds__(kFThreads, 1) k_decode_fused(FusedArgs f) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ Plan plan;
    __shared__ int ids_s[kDecMaxSlots];
    __shared__ float w_s[kDecMaxSlots];
    __shared__ int ident[kDecMaxT];
    __shared__ int g_tok[kGroups][kDecMaxT], g_slot[kGroups][kDecMaxT];
    __shared__ int g_last[kGroups];
    __shared__ volatile int abort_s;
    const DecodeArgs& a = f.d;
    const ExpertArgs& ex = a.ex;
    const int H = ex.H, I = ex.I, k = ex.k, E = ex.E, T = a.T;
    const int n = T * k;
    const int ldx = H + kXPad, lda = I + kXPad;
    const bool fp4 = (Q == Q_NVFP4);
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem_raw);                 // [9][ldx] raw x
    __nv_bfloat16* xq = xs + (size_t)(kDecMaxT + 1) * ldx;                          // [9][ldx] W4A4 x
    __nv_bfloat16* as0 = xq + (size_t)(kDecMaxT + 1) * ldx;                         // [4][9][lda]
    float* red0 = reinterpret_cast<float*>(as0 + (size_t)kGroups * (kDecMaxT + 1) * lda);   // [4][4][2][16][8]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int group = warp >> 2, wg = warp & 3;                  // 4-warp group, warp within it
    const int gtid = threadIdx.x & 127;
    __nv_bfloat16* as = as0 + (size_t)group * (kDecMaxT + 1) * lda;
    float* red = red0 + (size_t)group * 4 * 2 * 16 * 8;
    int* tok = g_tok[group];
    int* slot_of = g_slot[group];
    if (threadIdx.x == 0) abort_s = 0;
    if (threadIdx.x < kDecMaxT) ident[threadIdx.x] = threadIdx.x;
    __syncthreads();

    // ---- stage activations (rows t < T; rows T..8 zero)
    const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(a.x);
    stage_rows_bf16(xs, ldx, x, H, ident, T, threadIdx.x, blockDim.x);
    if (fp4) stage_rows_fp4_from_bf16(xq, ldx, x, H, ident, T, ex.g_x, threadIdx.x, blockDim.x);
    for (int i = threadIdx.x; i < ldx / 8; i += blockDim.x) {
        reinterpret_cast<uint4*>(xs + kDecMaxT * ldx)[i] = make_uint4(0, 0, 0, 0);
        reinterpret_cast<uint4*>(xq + kDecMaxT * ldx)[i] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();

    // ---- phase 0: router rows, one per warp, spread over all SMs
    if (f.wr) {
        for (int e = warp * gridDim.x + blockIdx.x; e < E; e += kFWarps * gridDim.x)
            router_row(reinterpret_cast<const uint8_t*>(f.wr), e, H, T, xs, ldx, f.logits, E);
        if (!grid_barrier(f.bar, f.err, &abort_s)) return;
    }

    // ---- phase 1: top-k (every CTA), plan, gate/up of the selected experts
    //      and of the shared expert; a unit = (expert, 16 rows) on one 4-warp
    //      group whose warps split K
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
    const int nslots = kGroups * gridDim.x;                      // concurrent units in the grid
    const int my_slot = group * gridDim.x + blockIdx.x;          // spread groups over SMs
    {
        const int per = I / 16;
        const int units = (nu + (ex.sh_gate ? 1 : 0)) * per;
        for (int u = my_slot; u < units; u += nslots) {
            const int ui = u / per, r0 = (u % per) * 16;
            const bool is_shared = (ui == nu);
            int m, e = 0;
            if (is_shared) {
                m = T;
                if (gtid < kDecMaxT) { tok[gtid] = gtid; slot_of[gtid] = gtid; }
            } else {
                m = group_item_tokens(plan.ids, n, k, plan.first[ui], tok, slot_of, gtid == 0);
                e = plan.ids[plan.first[ui]];
            }
            group_sync(group);
            const bool valid = is_shared || (e >= 0 && e < E);
            const __nv_bfloat16* xb = (fp4 && !is_shared) ? xq : xs;
            const __nv_bfloat16* xrow = xb + (g < m ? tok[g] : kDecMaxT) * ldx;
            const int nb = r0 / kBlkN, rl = r0 % kBlkN + g;
            float acc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
            if (is_shared) {
                const MatPtr mats[2] = {{ex.sh_gate, nullptr, nullptr}, {ex.sh_up, nullptr, nullptr}};
                warp_rows<Q_BF16, 2>(acc, mats, nb, rl, H / kBlkK, H / kGroup, wg, 4, xrow, c);
            } else if (valid) {
                const MatPtr mats[2] = {expert_mat(ex.gate, e), expert_mat(ex.up, e)};
                warp_rows<Q, 2>(acc, mats, nb, rl, H / kBlkK, H / kGroup, wg, 4, xrow, c);
            }
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float* rr = red + ((wg * 2 + q) * 16) * 8;
                rr[g * 8 + 2 * c] = acc[q][0];
                rr[g * 8 + 2 * c + 1] = acc[q][1];
                rr[(g + 8) * 8 + 2 * c] = acc[q][2];
                rr[(g + 8) * 8 + 2 * c + 1] = acc[q][3];
            }
            group_sync(group);
            {
                const int row = gtid / kDecMaxT, t = gtid % kDecMaxT;   // 128 = 16 rows x 8 tokens
                if (t < m) {
                    float gg = 0.0f, uu = 0.0f;
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        gg += red[((w * 2 + 0) * 16 + row) * 8 + t];
                        uu += red[((w * 2 + 1) * 16 + row) * 8 + t];
                    }
                    const float sc = (fp4 && !is_shared && valid) ? ex.g_gate[e] * ex.g_x : 1.0f;
                    gg *= sc;
                    uu *= sc;
                    const float act = valid ? gg / (1.0f + expf(-gg)) * uu : 0.0f;
                    if (is_shared) a.a_sh[(size_t)t * I + r0 + row] = act;
                    else a.a[(size_t)slot_of[t] * I + r0 + row] = act;
                }
            }
            group_sync(group);
        }
    }
    if (!grid_barrier(f.bar, f.err, &abort_s)) return;

    // ---- phase 2: down; a unit = (expert, 64 rows) on one group, each warp
    //      16 rows over the whole K; the last unit of a 64-row block combines
    {
        const int per = H / 64;
        const int items_per_rb = nu + (ex.sh_down ? 1 : 0);
        const int units = items_per_rb * per;
        for (int u = my_slot; u < units; u += nslots) {
            const int ui = u / per, hb = u % per, h0 = hb * 64;
            const bool is_shared = (ui == nu);
            int m, e = 0;
            if (is_shared) {
                m = T;
                if (gtid < kDecMaxT) { tok[gtid] = gtid; slot_of[gtid] = gtid; }
            } else {
                m = group_item_tokens(plan.ids, n, k, plan.first[ui], tok, slot_of, gtid == 0);
                e = plan.ids[plan.first[ui]];
            }
            group_sync(group);
            const bool valid = is_shared || (e >= 0 && e < E);
            stage_rows_f32(as, lda, is_shared ? a.a_sh : a.a, I, slot_of, m, fp4 && !is_shared, ex.g_a, gtid, 128);
            group_sync(group);
            const __nv_bfloat16* xrow = as + (g < m ? g : kDecMaxT) * lda;
            const int r = h0 + wg * 16;
            const int nb = r / kBlkN, rl = r % kBlkN + g;
            float acc[1][4] = {{0, 0, 0, 0}};
            if (is_shared) {
                const MatPtr mats[1] = {{ex.sh_down, nullptr, nullptr}};
                warp_rows<Q_BF16, 1>(acc, mats, nb, rl, I / kBlkK, I / kGroup, 0, 1, xrow, c);
            } else if (valid) {
                const MatPtr mats[1] = {expert_mat(ex.down, e)};
                warp_rows<Q, 1>(acc, mats, nb, rl, I / kBlkK, I / kGroup, 0, 1, xrow, c);
            }
            // this warp owns rows r..r+15 completely: write the partials
            const float dscale = (fp4 && !is_shared && valid) ? ex.g_down[e] * ex.g_a : 1.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = r + g + (i >= 2 ? 8 : 0), t = 2 * c + (i & 1);
                if (t < m) {
                    const float o = valid ? acc[0][i] * dscale : 0.0f;
                    if (is_shared) a.part_sh[(size_t)t * H + row] = o;
                    else a.part[(size_t)slot_of[t] * H + row] = w_s[slot_of[t]] * o;
                }
            }
            group_sync(group);
            if (gtid == 0) {
                __threadfence();
                g_last[group] = (atomicAdd(a.counters + hb, 1u) == (unsigned)items_per_rb - 1u);
                if (g_last[group]) __threadfence();
            }
            group_sync(group);
            if (g_last[group]) {
                __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(a.y);
                for (int i = gtid; i < T * 64; i += 128) {
                    const int t = i / 64, hh = h0 + i % 64;
                    float sum = 0.0f;
                    for (int j0 = 0; j0 < k; j0 += 8) {                // fixed order j = 0 .. k-1
                        float v[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            v[j] = (j0 + j < k) ? __ldcg(a.part + (size_t)(t * k + j0 + j) * H + hh) : 0.0f;
#pragma unroll
                        for (int j = 0; j < 8; ++j) sum += v[j];
                    }
                    if (ex.sh_down) sum += __ldcg(a.part_sh + (size_t)t * H + hh);
                    y[(size_t)t * H + hh] = __float2bfloat16_rn(sum);
                }
                group_sync(group);
                if (gtid == 0) a.counters[hb] = 0u;
            }
            group_sync(group);
        }
    }
}

size_t fused_smem_bytes(int H, int I) {
    const size_t xbuf = (size_t)(kDecMaxT + 1) * (H + kXPad) * 2;
    const size_t abuf = (size_t)(kDecMaxT + 1) * (I + kXPad) * 2;
    return 2 * xbuf + kGroups * abuf + (size_t)kFWarps * 2 * 16 * 8 * sizeof(float);
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
