// Token permutation: the flat slots s = t*k + j (token t's j-th expert) are
// put in expert-major order, stable in s, so each expert's tokens form one
// contiguous segment [offsets[e], offsets[e+1]) of perm.  The pages gather
// "the ten selected experts" per token ("Qwen3.8-Flash-Next on one 24 GB
// GPU", "What the patch does"); the order inside a segment is our reading
// (ascending slot id).  Two launches, both deterministic:
//   1. per chunk of slots, a histogram of expert ids;
//   2. per chunk, one CTA of 1024 threads: thread e sums expert e's counts
//      over all chunks (its total) and over the chunks before this one, one
//      CTA-wide scan of the totals gives the segment offsets, and the 32
//      warps rank and scatter the chunk's slots (per-warp counts, a scan
//      over the warps, then match_any ranks within each 32 slots).  When
//      asked, the same CTAs also write the grouped GEMMs' tile lists (each
//      CTA knows every expert's count and offset; the entries are spread
//      over the CTAs).
// Slots whose id lies outside [0, E) get no position (inv = -1).
#include "common.cuh"
#include "kernels.h"
#include "tiles.cuh"

namespace moe {

constexpr int kChunkMin = 1024;      // slots per chunk, at least
constexpr int kMaxChunks = 128;      // chunks grow beyond kChunkMin to keep at most this many
constexpr int kMaxE = 1024;
constexpr int kPlaceThreads = 1024;  // one expert per thread, 32 warps

// slots per chunk: a multiple of kChunkMin (so every warp takes a multiple of 32)
static int perm_chunk(long long n) {
    const long long per = (n + (long long)kChunkMin * kMaxChunks - 1) / ((long long)kChunkMin * kMaxChunks);
    return kChunkMin * (int)(per > 0 ? per : 1);
}
static int perm_chunks(long long n) {
    const int c = perm_chunk(n);
    return (int)((n + c - 1) / c);
}

size_t permute_scratch_ints(int slots, int E) { return (size_t)perm_chunks(slots) * E; }

__global__ void k_perm_hist(const int32_t* __restrict__ ids, int n, int E, int chunk, int32_t* __restrict__ chunk_cnt) {
    __shared__ int cnt[kMaxE];
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const long long base = (long long)blockIdx.x * chunk;
    for (int i = threadIdx.x; i < chunk && base + i < n; i += blockDim.x) {
        const int e = ids[base + i];
        if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);      // invalid ids are dropped
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_cnt[(size_t)blockIdx.x * E + e] = cnt[e];
}

__global__ void __launch_bounds__(kPlaceThreads, 1)
k_perm_place(const int32_t* __restrict__ ids, int n, int E, int chunk, int chunks,
             const int32_t* __restrict__ chunk_cnt, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
             int32_t* __restrict__ perm, int32_t* __restrict__ inv, TileListArgs tl) {
    extern __shared__ int wpos[];            // [32][E]: per-warp counts, then per-warp next positions
    __shared__ int s_cnt[kMaxE], s_off[kMaxE], wsum[32];
    __shared__ int s_sc[2][kMaxE], s_sg[2][kMaxE];
    const int e = threadIdx.x, lane = e & 31, w = e >> 5;
    const int c = blockIdx.x;                // the chunk

    // expert e's total over all chunks and its count in the chunks before c
    int tot = 0, pre = 0;
    if (e < E) {
        for (int c0 = 0; c0 < chunks; c0 += 16) {
            int v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = (c0 + u < chunks) ? __ldcg(chunk_cnt + (size_t)(c0 + u) * E + e) : 0;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                tot += v[u];
                pre += (c0 + u < c) ? v[u] : 0;
            }
        }
    }
    const int incl = block_incl_scan_1024(tot, wsum);
    const int off = incl - tot;              // segment offset of expert e
    s_cnt[e] = tot;
    s_off[e] = off;
    if (c == 0) {
        if (e < E) {
            counts[e] = tot;
            offsets[e] = off;
        }
        if (e == kPlaceThreads - 1) offsets[E] = incl;    // all placed slots
    }
    if (tl.tiles) {                          // both tile lists, entries spread over all CTAs
        tile_list_prefix(s_cnt, tl.RB0, tl.tok0, s_sc[0], s_sg[0], wsum);
        tile_list_prefix(s_cnt, tl.RB1, tl.tok1, s_sc[1], s_sg[1], wsum);
        __syncthreads();
        const long long first = (long long)c * kPlaceThreads + e, stride = (long long)gridDim.x * kPlaceThreads;
        for (int list = 0; list < 2; ++list)
            emit_tile_list(s_cnt, s_off, s_sc[list], s_sg[list], tl.T, list ? tl.RB1 : tl.RB0,
                           list ? tl.tok1 : tl.tok0, tl.tok_sh, tl.has_shared,
                           tl.grid, first, stride, tl.tiles + (size_t)list * tl.cap,
                           tl.groups + (size_t)list * tl.cap, tl.num_tiles + 4 * list, c == 0);
    }

    // warp w takes slots [s0, s0 + W) of the chunk, 32 at a time
    const int W = chunk / 32;
    const long long s0 = (long long)c * chunk + (long long)w * W;
    int* my = wpos + w * E;
    const unsigned lt = (1u << lane) - 1u;
    for (int i = lane; i < E; i += 32) my[i] = 0;
    __syncwarp();
    for (int st = 0; st < W; st += 32) {
        const long long s = s0 + st + lane;
        const int ev = (s < n) ? __ldg(ids + s) : -1;
        const bool valid = s < n && ev >= 0 && ev < E;
        const unsigned act = __ballot_sync(0xffffffffu, valid);
        if (valid) {
            const unsigned peers = __match_any_sync(act, ev);
            if ((peers & lt) == 0) my[ev] += __popc(peers);
        }
        __syncwarp();
    }
    __syncthreads();
    // expert e: the chunk's first position, then each warp's
    if (e < E) {
        int run = off + pre;
        for (int ww = 0; ww < 32; ++ww) {
            const int t = wpos[ww * E + e];
            wpos[ww * E + e] = run;
            run += t;
        }
    }
    __syncthreads();
    for (int st = 0; st < W; st += 32) {
        const long long s = s0 + st + lane;
        const int ev = (s < n) ? __ldg(ids + s) : -1;
        const bool valid = s < n && ev >= 0 && ev < E;
        const unsigned act = __ballot_sync(0xffffffffu, valid);
        if (s < n && !valid) inv[s] = -1;          // dropped slot: no position
        if (valid) {
            const unsigned peers = __match_any_sync(act, ev);
            const int pos = my[ev] + __popc(peers & lt);
            perm[pos] = (int32_t)s;
            inv[s] = pos;
            __syncwarp(act);
            if ((peers & lt) == 0) my[ev] += __popc(peers);
        }
        __syncwarp();
    }
}

cudaError_t launch_permute(const int32_t* ids, int T, int k, int E, int32_t* counts, int32_t* offsets,
                           int32_t* perm, int32_t* inv, int32_t* chunk_scratch, cudaStream_t st,
                           const TileListArgs* tl) {
    if (E < 1 || E > kMaxE) return cudaErrorInvalidValue;
    const long long n = (long long)T * k;
    const int chunk = perm_chunk(n), chunks = perm_chunks(n);
    k_perm_hist<<<chunks, 256, 0, st>>>(ids, (int)n, E, chunk, chunk_scratch);
    const int smem = 32 * E * (int)sizeof(int);
    cudaError_t e = cudaFuncSetAttribute(k_perm_place, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    TileListArgs none{};
    k_perm_place<<<chunks, kPlaceThreads, smem, st>>>(ids, (int)n, E, chunk, chunks, chunk_scratch,
                                                                     counts, offsets, perm, inv, tl ? *tl : none);
    return cudaGetLastError();
}

}  // namespace moe
