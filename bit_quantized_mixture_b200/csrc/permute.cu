// Token permutation: the flat slots s = t*k + j (token t's j-th expert) are
// put in expert-major order, stable in s, so each expert's tokens form one
// contiguous segment [offsets[e], offsets[e+1]) of perm.  The pages gather
// "the ten selected experts" per token ("Qwen3.8-Flash-Next on one 24 GB
// GPU", "What the patch does"); the order inside a segment is our reading
// (ascending slot id).  Three passes, all deterministic:
//   1. per chunk of kChunk slots, a histogram of expert ids;
//   2. one CTA turns the histograms into per-chunk bases and offsets;
//   3. per chunk, one warp ranks its slots (match_any per 32 slots) and
//      scatters them.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kChunk = 1024;
constexpr int kMaxE = 1024;

size_t permute_scratch_ints(int slots, int E) {
    const int chunks = (slots + kChunk - 1) / kChunk;
    return (size_t)chunks * E;
}

__global__ void k_perm_hist(const int32_t* __restrict__ ids, int n, int E, int32_t* __restrict__ chunk_cnt) {
    __shared__ int cnt[kMaxE];
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const int base = blockIdx.x * kChunk;
    for (int i = threadIdx.x; i < kChunk && base + i < n; i += blockDim.x) {
        const int e = ids[base + i];
        if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);      // invalid ids are dropped
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_cnt[(size_t)blockIdx.x * E + e] = cnt[e];
}

// single CTA of kMaxE threads: thread e walks the chunks of expert e
__global__ void __launch_bounds__(kMaxE) k_perm_scan(int chunks, int E, int32_t* __restrict__ chunk_cnt,
                                                     int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
    __shared__ int s[kMaxE];
    const int e = threadIdx.x;
    int total = 0;
    if (e < E) {
        // sixteen independent loads in flight per step
        for (int c0 = 0; c0 < chunks; c0 += 16) {
            int v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = (c0 + u < chunks) ? chunk_cnt[(size_t)(c0 + u) * E + e] : 0;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                if (c0 + u < chunks) chunk_cnt[(size_t)(c0 + u) * E + e] = total;   // exclusive base within the expert
                total += v[u];
            }
        }
        counts[e] = total;
    }
    s[e] = (e < E) ? total : 0;
    __syncthreads();
    // inclusive Hillis-Steele scan over experts
    for (int o = 1; o < kMaxE; o <<= 1) {
        const int v = (e >= o) ? s[e - o] : 0;
        __syncthreads();
        s[e] += v;
        __syncthreads();
    }
    const int excl = s[e] - ((e < E) ? total : 0);
    if (e < E) {
        offsets[e] = excl;
        for (int c0 = 0; c0 < chunks; c0 += 16) {
            int v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = (c0 + u < chunks) ? chunk_cnt[(size_t)(c0 + u) * E + e] : 0;
#pragma unroll
            for (int u = 0; u < 16; ++u)
                if (c0 + u < chunks) chunk_cnt[(size_t)(c0 + u) * E + e] = v[u] + excl;
        }
    }
    if (e == E - 1) offsets[E] = s[e];
}

__global__ void __launch_bounds__(32) k_perm_scatter(const int32_t* __restrict__ ids, int n, int E,
                                                     const int32_t* __restrict__ chunk_base,
                                                     int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
    __shared__ int cur[kMaxE];
    const int lane = threadIdx.x;
    for (int e = lane; e < E; e += 32) cur[e] = chunk_base[(size_t)blockIdx.x * E + e];
    __syncwarp();
    const int base = blockIdx.x * kChunk;
    int ev[kChunk / 32];                      // the chunk's expert ids, all loads in flight at once
#pragma unroll
    for (int step = 0; step < kChunk / 32; ++step) {
        const int s = base + step * 32 + lane;
        ev[step] = (s < n) ? __ldg(ids + s) : -1;
    }
#pragma unroll
    for (int step = 0; step < kChunk / 32; ++step) {
        const int s = base + step * 32 + lane;
        const int e_s = ev[step];
        const bool valid = (s < n) && e_s >= 0 && e_s < E;
        const unsigned active = __ballot_sync(0xffffffffu, valid);
        if (s < n && !valid) inv[s] = -1;          // dropped slot: no position
        if (valid) {
            const int e = e_s;
            const unsigned peers = __match_any_sync(active, e);
            const int rank = __popc(peers & ((1u << lane) - 1u));
            const int pos = cur[e] + rank;
            perm[pos] = s;
            inv[s] = pos;
            __syncwarp(active);
            if ((peers & ((1u << lane) - 1u)) == 0) cur[e] += __popc(peers);
        }
        __syncwarp();
    }
}

cudaError_t launch_permute(const int32_t* ids, int T, int k, int E, int32_t* counts, int32_t* offsets,
                           int32_t* perm, int32_t* inv, int32_t* chunk_scratch, cudaStream_t st) {
    const int n = T * k;
    const int chunks = (n + kChunk - 1) / kChunk;
    k_perm_hist<<<chunks, 256, 0, st>>>(ids, n, E, chunk_scratch);
    k_perm_scan<<<1, kMaxE, 0, st>>>(chunks, E, chunk_scratch, counts, offsets);
    k_perm_scatter<<<chunks, 32, 0, st>>>(ids, n, E, chunk_scratch, perm, inv);
    return cudaGetLastError();
}

}  // namespace moe
