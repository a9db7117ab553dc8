// Router: logits = x Wr^T (bf16 inputs, fp32 accumulation), softmax and
// top-k with renormalised weights.
//
// Ten of 512 experts are selected per token ("Qwen3.8-Flash-Next on one 24 GB
// GPU", "What the patch does"); the router stays bf16 because a small logit
// perturbation changes routing on near-ties ("Qwen3.8-Flash-Next-FP6-INT8",
// "Precision map").  Order: logit descending, expert index ascending on
// equal logits.  Weights: w_j = exp(l_j - l_max) / sum_selected exp(l - l_max),
// which equals the full softmax renormalised over the selected experts.
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kRouteMaxTSmall = 8;    // decode router: tokens staged in smem
constexpr size_t kRouteMaxSmem = 160 * 1024;

// Order-preserving key of an fp32 value (larger value -> larger key).
MOE_DEV uint32_t order_key(float v) {
    const uint32_t b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Inverse of order_key.
MOE_DEV float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

constexpr int kTopkWarps = 8;        // warps of a CTA with shared candidate lists

// One warp selects the top-k of one token's logits (E <= 1024 values read
// through L2, expert e held by lane e % 32) and writes ids / weights, in the
// order key descending, expert ascending on equal keys.
//
// Threshold selection: the k-th largest of the 32 lanes' own maxima, t, is
// reached by at least k logits, so every selected expert is among the
// logits >= t (about 12 of 512 for continuous logits).  Those candidates are
// gathered into the warp's shared list and each is ranked exactly by
// counting the candidates ahead of it.  With more than 32 candidates (many
// equal logits), or without a shared list, selection rounds run instead:
// each lane keeps the best of its own live keys, a round takes the warp
// maximum with one max-reduction and, among lanes holding it, the smallest
// expert with one min-reduction; only the lane that lost its key rescans.
// sk / se: 64 entries of this warp's shared memory each, or null.
template <int SLOTS>
MOE_DEV void warp_topk_n(const float* __restrict__ row, int E, int k, int32_t* __restrict__ ids,
                         float* __restrict__ wout, uint32_t* sk, int* se) {
    const int lane = threadIdx.x & 31;
    uint32_t key[SLOTS];
#pragma unroll
    for (int i = 0; i < SLOTS; ++i) {
        const int e = lane + 32 * i;
        key[i] = (e < E) ? order_key(__ldcg(row + e)) : 0u;
    }
    uint32_t live = 0;
#pragma unroll
    for (int i = 0; i < SLOTS; ++i) live |= ((lane + 32 * i) < E ? 1u : 0u) << i;
    float my_val = 0.0f, lmax = 0.0f;
    int my_idx = 0;
    bool done = false;
    if (sk != nullptr) {
        uint32_t m = 0;                      // the lane's largest key
#pragma unroll
        for (int i = 0; i < SLOTS; ++i)
            if ((live >> i) & 1u) m = max(m, key[i]);
        // t: the k-th largest lane maximum (each round retires the lowest
        // lane holding the current maximum)
        bool alive = live != 0;
        uint32_t t = 0;
        for (int r = 0; r < k; ++r) {
            t = __reduce_max_sync(0xffffffffu, alive ? m : 0u);
            const unsigned hold = __ballot_sync(0xffffffffu, alive && m == t);
            if (lane == __ffs(hold) - 1) alive = false;
        }
        unsigned cm = 0;                     // the lane's candidates
#pragma unroll
        for (int i = 0; i < SLOTS; ++i) cm |= (((live >> i) & 1u) && key[i] >= t) ? (1u << i) : 0u;
        const int cl = __popc(cm);
        int incl = cl;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        const int C = __shfl_sync(0xffffffffu, incl, 31);
        if (C <= 32) {
            int p = incl - cl;
#pragma unroll
            for (int i = 0; i < SLOTS; ++i)
                if ((cm >> i) & 1u) {
                    sk[p] = key[i];
                    se[p] = lane + 32 * i;
                    ++p;
                }
            __syncwarp();
            const uint32_t mk = lane < C ? sk[lane] : 0u;
            const int me = lane < C ? se[lane] : 0x7fffffff;
            int rank = 0;                    // candidates ahead of this lane's
            for (int j = 0; j < C; ++j) {
                const uint32_t kj = sk[j];
                const int ej = se[j];
                rank += (kj > mk || (kj == mk && ej < me)) ? 1 : 0;
            }
            if (lane < C && rank < k) {
                sk[32 + rank] = mk;
                se[32 + rank] = me;
            }
            __syncwarp();
            if (lane < k) {
                my_val = key_value(sk[32 + lane]);
                my_idx = se[32 + lane];
            }
            lmax = key_value(sk[32]);
            __syncwarp();                    // the list is free for the warp's next token
            done = true;
        }
    }
    if (!done) {
        // best live key of this lane and its slot (first slot on equal keys)
        auto rescan = [&](uint32_t& best, int& slot) {
            best = 0;
            slot = -1;
#pragma unroll
            for (int i = 0; i < SLOTS; ++i)
                if (((live >> i) & 1u) && (slot < 0 || key[i] > best)) {
                    best = key[i];
                    slot = i;
                }
        };
        uint32_t best;
        int slot;
        rescan(best, slot);
        for (int j = 0; j < k; ++j) {
            const uint32_t top = __reduce_max_sync(0xffffffffu, slot >= 0 ? best : 0u);
            const uint32_t mine = (slot >= 0 && best == top) ? (uint32_t)(lane + 32 * slot) : 0xffffffffu;
            const uint32_t e = __reduce_min_sync(0xffffffffu, mine);
            if ((int)(e & 31u) == lane) {
                live &= ~(1u << (e >> 5));
                rescan(best, slot);
            }
            const float v = key_value(top);
            if (j == 0) lmax = v;
            if (lane == j) { my_val = v; my_idx = (int)e; }
        }
    }
    const float ex = (lane < k) ? expf(my_val - lmax) : 0.0f;
    const float sum = warp_sum(ex);
    if (lane < k) {
        ids[lane] = my_idx;
        wout[lane] = __fdiv_rn(ex, sum);
    }
}

// E <= 512: 16 slots per lane; E <= 1024: 32.  Warps beyond kTopkWarps of
// their CTA take the selection rounds.
MOE_DEV void warp_topk(const float* __restrict__ row, int E, int k, int32_t* __restrict__ ids,
                       float* __restrict__ wout) {
    __shared__ uint32_t s_key[kTopkWarps][64];
    __shared__ int s_exp[kTopkWarps][64];
    const int w = threadIdx.x >> 5;
    uint32_t* sk = w < kTopkWarps ? s_key[w] : nullptr;
    int* se = w < kTopkWarps ? s_exp[w] : nullptr;
    if (E <= 512) warp_topk_n<16>(row, E, k, ids, wout, sk, se);
    else warp_topk_n<32>(row, E, k, ids, wout, sk, se);
}

// Decode router (T <= 8): one warp per expert row, a grid-wide ticket lets
// the last CTA to finish run the top-k of every token (no waiting).  Asked
// for logits only, the CTAs end after their logits.
__global__ void __launch_bounds__(128) k_router_small(RouteArgs a) {
    extern __shared__ float xs[];          // [T][H] fp32
    __shared__ int s_last;
    const int H = a.H, T = a.T;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 4 + warp;
    pdl_launch_dependents();                 // let the expert kernel get resident
    const uint8_t* row = reinterpret_cast<const uint8_t*>(a.wr) + (size_t)(e < a.E ? e : 0) * H * 2;
    // first batch of router-row loads goes out before the activations are staged
    uint4 q0[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int c = lane + 32 * u;
        q0[u] = (e < a.E && c < H / 8) ? ldg_stream_v4(row + (size_t)c * 16) : make_uint4(0, 0, 0, 0);
    }
    {   // stage x as fp32: 16-byte loads, four in flight per thread
        const uint4* xv = reinterpret_cast<const uint4*>(a.x);
        const int nchunks = T * H / 8;
        for (int i0 = threadIdx.x; i0 < nchunks; i0 += 4 * blockDim.x) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * blockDim.x;
                v[u] = (i < nchunks) ? xv[i] : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * blockDim.x;
                if (i < nchunks) {
                    float4* d = reinterpret_cast<float4*>(xs + (size_t)i * 8);
                    d[0] = make_float4(bf16_lo(v[u].x), bf16_hi(v[u].x), bf16_lo(v[u].y), bf16_hi(v[u].y));
                    d[1] = make_float4(bf16_lo(v[u].z), bf16_hi(v[u].z), bf16_lo(v[u].w), bf16_hi(v[u].w));
                }
            }
        }
    }
    __syncthreads();
    if (e < a.E) {
        float acc[kRouteMaxTSmall];
#pragma unroll
        for (int t = 0; t < kRouteMaxTSmall; ++t) acc[t] = 0.0f;
        for (int c0 = 0; c0 < H / 8; c0 += 32 * 8) {
            uint4 q[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {          // 8 loads in flight per lane
                const int c = c0 + lane + 32 * u;
                q[u] = (c0 == 0) ? q0[u] : ((c < H / 8) ? ldg_stream_v4(row + (size_t)c * 16) : make_uint4(0, 0, 0, 0));
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int c = c0 + lane + 32 * u;
                if (c < H / 8) {
                    const uint32_t wv[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
                    for (int t = 0; t < kRouteMaxTSmall; ++t) {
                        if (t < T) {
                            const float* xr = xs + t * H + c * 8;
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                acc[t] = fmaf(bf16_lo(wv[i]), xr[2 * i], acc[t]);
                                acc[t] = fmaf(bf16_hi(wv[i]), xr[2 * i + 1], acc[t]);
                            }
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < kRouteMaxTSmall; ++t) {
            if (t < T) {
                const float s = warp_sum(acc[t]);
                if (lane == 0) a.logits[(size_t)t * a.E + e] = s;
            }
        }
    }
    if (!a.ids) return;
    __syncthreads();
    if (threadIdx.x == 0) s_last = (ticket_acq_rel(a.counter) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    for (int t = warp; t < T; t += 4)
        warp_topk(a.logits + (size_t)t * a.E, a.E, a.k, a.ids + (size_t)t * a.k, a.w + (size_t)t * a.k);
    __syncthreads();
    if (threadIdx.x == 0) *a.counter = 0u;      // ready for the next launch
}

__global__ void __launch_bounds__(256) k_topk(RouteArgs a) {
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= a.T) return;
    const float* row = (a.logits_in ? a.logits_in : a.logits) + (size_t)t * a.E;
    warp_topk(row, a.E, a.k, a.ids + (size_t)t * a.k, a.w + (size_t)t * a.k);
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
    if (a.logits_in == nullptr) {
        const size_t smem = (size_t)a.T * a.H * sizeof(float);
        if (a.T <= kRouteMaxTSmall && smem <= kRouteMaxSmem) {
            cudaError_t e = cudaFuncSetAttribute(k_router_small, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)kRouteMaxSmem);
            if (e != cudaSuccess) return e;
            k_router_small<<<(a.E + 3) / 4, 128, smem, st>>>(a);
            return cudaGetLastError();
        }
        cudaError_t e = launch_router_tc(a.x, a.wr, a.T, a.H, a.E, a.logits, a.err, st);
        if (e != cudaSuccess) return e;
    }
    if (a.ids) k_topk<<<(a.T + 7) / 8, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
