// Tile lists of the grouped GEMMs, built on the device from the expert
// counts and segment offsets of the token permutation.
//
// A routed tile is (expert e, 128-row block rb of the weight matrix, up to
// `tok` consecutive permuted positions of e's segment: kTileTokens, or more
// for a GEMM whose MMA takes wider tiles); the list holds
// every expert's tiles expert by expert, row block by row block, then (when
// the layer has a shared expert) the shared-expert tiles (expert -1, token
// rows instead of positions, tok_sh per tile).  A group is up to kGroupTiles consecutive token
// tiles of one (expert, row block), which read the same weight block.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kTileTokens = 128;     // tokens per tile (the MMA's N)
constexpr int kTileCache = 256;      // tiles a GEMM CTA keeps in shared memory
constexpr int kGroupTiles = 2;

// Inclusive scan of one int per thread over a CTA of exactly 1024 threads;
// wsum: 32 ints of shared memory.  Every thread must call it.
MOE_DEV int block_incl_scan_1024(int v, int* wsum) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    __syncthreads();                 // wsum may still be read by a previous call
    if (lane == 31) wsum[w] = v;
    __syncthreads();
    if (w == 0) {
        int t = wsum[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += u;
        }
        wsum[lane] = t;
    }
    __syncthreads();
    return v + (w ? wsum[w - 1] : 0);
}

// Inclusive prefixes over experts of one list's tile and group counts, into
// sc and sg (1024 ints of shared memory each; thread e takes expert e).
// s_cnt: 1024 expert counts, zero beyond E.  A CTA of 1024 threads; the
// caller synchronizes before reading sc / sg.
MOE_DEV void tile_list_prefix(const int* s_cnt, int RB, int tok, int* sc, int* sg, int* wsum) {
    const int e = threadIdx.x;
    const int nt = (s_cnt[e] + tok - 1) / tok;
    const int ci = block_incl_scan_1024(nt * RB, wsum);
    const int gi = block_incl_scan_1024(((nt + kGroupTiles - 1) / kGroupTiles) * RB, wsum);
    sc[e] = ci;
    sg[e] = gi;
}

// The expert of list entry i: the first whose inclusive prefix exceeds i.
MOE_DEV int tile_owner(const int* pre, int i) {
    int lo = 0, hi = 1023;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] > i) hi = mid;
        else lo = mid + 1;
    }
    return lo;
}

// Entries first, first + stride, ... of one tile list and its group list,
// from the expert counts / offsets and the prefixes of tile_list_prefix (so
// the CTAs of a launch can share the work).  The caller that passes
// write_counts sets num_tiles[0..3] = routed tiles, routed + shared tiles,
// routed groups, and 1 when every GEMM CTA's groups fit its shared-memory
// tile list (group order), else 0.
MOE_DEV void emit_tile_list(const int* s_cnt, const int* s_off, const int* sc, const int* sg, int T, int RB, int tok,
                            int tok_sh, int has_shared, int grid, long long first, long long stride, GemmTile* __restrict__ tiles,
                            int2* __restrict__ groups, int* __restrict__ num_tiles, bool write_counts) {
    const int total = sc[1023], ngroups = sg[1023];
    for (long long ii = first; ii < ngroups; ii += stride) {
        const int i = (int)ii;
        const int ex = tile_owner(sg, i);
        const int ntx = (s_cnt[ex] + tok - 1) / tok;
        const int gpr = (ntx + kGroupTiles - 1) / kGroupTiles;     // groups per row block
        const int j = i - (sg[ex] - gpr * RB);
        const int rb = j / gpr, q = j % gpr;
        groups[i] = make_int2(sc[ex] - ntx * RB + rb * ntx + q * kGroupTiles, min(kGroupTiles, ntx - q * kGroupTiles));
    }
    for (long long ii = first; ii < total; ii += stride) {
        const int i = (int)ii;
        const int ex = tile_owner(sc, i);
        const int c = s_cnt[ex];
        const int ntx = (c + tok - 1) / tok;
        const int j = i - (sc[ex] - ntx * RB);          // index within the expert's tiles
        const int rb = j / ntx, tt = j % ntx;
        GemmTile g;
        g.expert = ex;
        g.rb = rb;
        g.seg = s_off[ex] + tt * tok;
        g.count = min(tok, c - tt * tok);
        tiles[i] = g;
    }
    const int nts = has_shared ? (T + tok_sh - 1) / tok_sh : 0;
    for (long long ii = first; ii < (long long)nts * RB; ii += stride) {
        const int i = (int)ii;
        const int rb = i / nts, tt = i % nts;
        GemmTile g;
        g.expert = -1;
        g.rb = rb;
        g.seg = tt * tok_sh;
        g.count = min(tok_sh, T - tt * tok_sh);
        tiles[total + i] = g;
    }
    if (write_counts && threadIdx.x == 0) {
        num_tiles[0] = total;
        num_tiles[1] = total + nts * RB;
        num_tiles[2] = ngroups;
        num_tiles[3] = ((ngroups + grid - 1) / grid) * kGroupTiles <= kTileCache ? 1 : 0;
    }
}

}  // namespace moe
