// Whole decode step of the layer (up to 8 tokens) in one persistent kernel:
// router GEMV and top-k, every selected expert's gate/up and down GEMV, the
// shared expert and the combine.
//
// At decode sizes the step time is set by chains of dependent memory round
// trips (x -> logits -> ids -> weights -> intermediates -> partials), not by
// bytes.  One cooperative grid (one 16-warp CTA per SM, four 4-warp groups)
// therefore walks three phases separated by two grid-wide barriers and issues
// every weight load of a phase at once, as asynchronous copies into shared
// memory, before it computes anything:
//   start:   each group copies its router rows, its slices of the shared
//            expert's gate/up (16 rows x a part of K) and its shared down
//            slice (16 rows, kept until phase 2): none depends on routing;
//   phase 0: router logits and partial shared gate/up sums;
//   phase 1: every CTA computes the top-k of all tokens from the logits
//            itself (no third barrier), builds the same plan of distinct
//            experts, copies its gate/up units (expert x 16 rows) and, when
//            they fit, its down units (expert x 16 rows of H) at once, and
//            computes the gate/up units;
//   phase 2: the down units (weights already resident) and the shared down
//            slices add their routing-weighted partials; the last unit of a
//            16-row block (ticket counter, no waiting) sums
//            y_t = sum_j part[t*k+j] + shared_t in fixed j order.
// Units are spread over the 4 x #SM group slots with per-kind offsets so that
// no group holds more than its share of shared memory; units that do not fit
// are copied one at a time.  The GEMV arithmetic is that of decode.cu
// (mma.sync m16n8k16 on exact dequantized operands, group scales on fp32
// accumulators), read from shared memory.  Loops are kept small: every phase
// runs once per launch, so its code is fetched cold.  The barriers wait a
// bounded time; on timeout the kernel records an error code, skips the
// remaining phases and returns (moe_sync_status reports it).
#include "decode_common.cuh"

namespace moe {

constexpr int kFWarps = 16;
constexpr int kFThreads = kFWarps * 32;
constexpr int kGroups = kFWarps / 4;
constexpr long long kBarrierLimitCycles = 4000000000LL;   // about 2 s
constexpr int kFusedSmem = 232448 - 8192;                 // 227 KB per CTA less the static arrays

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
// `withhold` (a test hook of the bounded wait) makes this CTA skip its
// arrival, so the episode never completes and every CTA gives up after
// `limit` cycles.
MOE_DEV bool grid_barrier(unsigned long long* bar, int* err, volatile int* abort_s, bool withhold, long long limit) {
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned long long n = gridDim.x;
        const unsigned long long ticket = withhold ? ld_acquire64(bar) : atom_add_release64(bar, 1ull);
        const unsigned long long target = (ticket / n + 1) * n;
        const long long t0 = clock64();
        while (ld_acquire64(bar) < target) {
            if (clock64() - t0 > limit) {
                *abort_s = 1;
                if (err) atomicCAS(err, 0, 20);
                break;
            }
        }
    }
    __syncthreads();
    return *abort_s == 0;
}

// ------------------------------------------------------------ async copies
// 16-byte global -> shared copies (L2 only); completion per thread, in
// commit-group order.
MOE_DEV void cp16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src) : "memory");
}
MOE_DEV void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
MOE_DEV void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// named barrier of one 4-warp group (ids 1..4; 0 is __syncthreads)
MOE_DEV void group_sync(int group) { asm volatile("bar.sync %0, 128;" ::"r"(group + 1) : "memory"); }

// ------------------------------------------------- 16-row matrix slices
// A slice is rows r0 .. r0+15 (r0 % 16 == 0) of one quantized matrix [N, K]
// over all of K, copied in the order of the device layout: codes
// [kb][chunk][16 rows][16 B], then scales (INT4/INT2: [K/128][16] fp16;
// NVFP4: [K/64][16][4] e4m3), then INT2 zero points [K/128][16].
struct Slice {
    int KB, G, nch, blk_bytes, code_bytes, scale_bytes, zero_bytes, bytes;
};
__host__ __device__ inline Slice qslice(int quant, int K) {
    Slice s;
    s.KB = K / kBlkK;
    s.G = scale_stride(quant, K);
    s.nch = quant == Q_INT2 ? 1 : (quant == Q_FP8 ? 4 : 2);
    s.blk_bytes = kBlkN * 16 * s.nch;
    s.code_bytes = s.KB * s.nch * 256;
    // NVFP4: 4 e4m3 per row and k-block; FP8: the row block's fp32 scales
    // (G of them, a multiple of 4); else fp16 per row and group
    s.scale_bytes = quant == Q_NVFP4 ? s.KB * 64 : (quant == Q_FP8 ? s.G * 4 : s.G * 32);
    s.zero_bytes = quant == Q_INT2 ? s.G * 16 : 0;
    s.bytes = s.code_bytes + s.scale_bytes + s.zero_bytes;
    return s;
}

// Copies by one 4-warp group (gtid 0..127).  The kernel runs each phase's
// code once per launch, fetched cold, so the helpers called from several
// places are kept out of line.  With 128 threads and 16-byte chunks a
// thread's chunk inside each 256-byte code row is fixed, so its source and
// destination advance by constants.
template <int Q>
__device__ __noinline__ void load_qslice(uint8_t* dst, MatPtr m, Slice s, int r0, int gtid) {
    constexpr int NCH = Q == Q_INT2 ? 1 : (Q == Q_FP8 ? 4 : 2);
    const int nb = r0 / kBlkN, rl0 = r0 % kBlkN;
    {
        const int p0 = gtid >> 4, c16 = gtid & 15;          // piece p0 + 8 j, chunk c16 of its 16
        const int kb0 = p0 / NCH, ch = p0 % NCH;
        const uint8_t* src = m.codes + ((size_t)nb * s.KB + kb0) * s.blk_bytes + (ch * kBlkN + rl0) * 16 + c16 * 16;
        uint8_t* d = dst + gtid * 16;
        const size_t step = (size_t)(8 / NCH) * s.blk_bytes;
        const int npieces = s.KB * NCH;
#pragma unroll 1
        for (int p = p0; p < npieces; p += 8, src += step, d += 2048) cp16(d, src);
    }
    uint8_t* ds = dst + s.code_bytes;
    if constexpr (Q == Q_NVFP4) {
#pragma unroll 1
        for (int j = gtid; j < s.KB * 4; j += 128)
            cp16(ds + j * 16, m.scales + (((size_t)nb * s.KB + (j >> 2)) * kBlkN + rl0) * 4 + (j & 3) * 16);
    } else if constexpr (Q == Q_FP8) {
#pragma unroll 1
        for (int j = gtid; j < s.G / 4; j += 128) cp16(ds + j * 16, m.scales + ((size_t)nb * s.G + j * 4) * 4);
    } else {
#pragma unroll 1
        for (int j = gtid; j < s.G * 2; j += 128)
            cp16(ds + j * 16, m.scales + (((size_t)nb * s.G + (j >> 1)) * kBlkN + rl0) * 2 + (j & 1) * 16);
    }
    if constexpr (Q == Q_INT2) {
#pragma unroll 1
        for (int j = gtid; j < s.G; j += 128)
            cp16(ds + s.scale_bytes + j * 16, m.zeros + ((size_t)nb * s.G + j) * kBlkN + rl0);
    }
}
// bf16 slice of the shared expert's tile images: rows r0 .. r0+15 of k-blocks
// kb0 .. kb0+nkb-1, 2 KB per k-block (the two 8-row swizzle atoms); thread
// gtid copies chunk gtid of every k-block.
__device__ __noinline__ void load_bslice(uint8_t* dst, const uint8_t* img, int KB, int r0, int kb0, int nkb, int gtid) {
    const int nb = r0 / kBlkN, rl0 = r0 % kBlkN;
    const uint8_t* src = img + ((size_t)nb * KB + kb0) * 16384 + (rl0 >> 3) * 1024 + gtid * 16;
    uint8_t* d = dst + gtid * 16;
#pragma unroll 1
    for (int j = 0; j < nkb; ++j, src += 16384, d += 2048) cp16(d, src);
}

// Operands of local rows gl, gl+8 of k-block kb of a staged slice (for the
// bf16 slices kb counts from the first staged k-block).
template <int Q>
MOE_DEV void load_blk_s(Blk<Q>& o, const uint8_t* base, const Slice& s, int kb, int gl, int c) {
    if constexpr (Q == Q_BF16) {
        const uint8_t* blk = base + kb * 2048;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int r = gl + 8 * rr, c8 = 4 * h + c;
                o.v[h][rr] = *reinterpret_cast<const uint4*>(blk + (r >> 3) * 1024 + (r & 7) * 128 + ((c8 ^ (r & 7)) << 4));
            }
    } else {
        constexpr int NCH = Q == Q_INT2 ? 1 : (Q == Q_FP8 ? 4 : 2);
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
            const uint8_t* p = base + (kb * NCH + ch) * 256 + c * 4;
            o.w[ch][0] = *reinterpret_cast<const uint32_t*>(p + gl * 16);
            o.w[ch][1] = *reinterpret_cast<const uint32_t*>(p + (gl + 8) * 16);
        }
        const uint8_t* sc = base + s.code_bytes;
        if constexpr (Q == Q_FP8) {
            o.s0 = reinterpret_cast<const float*>(sc)[kb >> 1];
        } else if constexpr (Q == Q_NVFP4) {
            o.sb0 = *reinterpret_cast<const uint32_t*>(sc + kb * 64 + gl * 4);
            o.sb1 = *reinterpret_cast<const uint32_t*>(sc + kb * 64 + (gl + 8) * 4);
        } else if constexpr (Q == Q_INT4G32) {      // groups 2 kb, 2 kb + 1 (16 rows x fp16 each)
            const __half* sh = reinterpret_cast<const __half*>(sc + kb * 64);
            o.s0 = __half2float(sh[gl]);
            o.s1 = __half2float(sh[gl + 8]);
            o.s2 = __half2float(sh[16 + gl]);
            o.s3 = __half2float(sh[16 + gl + 8]);
        } else {
            const __half* sh = reinterpret_cast<const __half*>(sc + (kb >> 1) * 32);
            o.s0 = __half2float(sh[gl]);
            o.s1 = __half2float(sh[gl + 8]);
            if constexpr (Q == Q_INT2) {
                const uint8_t* z = sc + s.scale_bytes + (kb >> 1) * 16;
                o.z0 = bf16x2_splat(128.0f + (float)z[gl]);
                o.z1 = bf16x2_splat(128.0f + (float)z[gl + 8]);
            }
        }
    }
}

// One warp's share of staged slices: k-blocks kb0 + wg, kb0 + wg + 4, ...
// (< kb1) of NM matrices; xrow is the lane's token row at column 0.
template <int Q, int NM>
MOE_DEV void slice_mma(float (&acc)[NM][4], const uint8_t* const (&base)[NM], const Slice& s, int kb0, int kb1, int wg,
                       const __nv_bfloat16* xrow, int gl, int c) {
#pragma unroll 1
    for (int kb = kb0 + wg; kb < kb1; kb += 4) {
#pragma unroll
        for (int q = 0; q < NM; ++q) {
            Blk<Q> b;
            load_blk_s<Q>(b, base[q], s, Q == Q_BF16 ? kb - kb0 : kb, gl, c);
            mma_blk<Q>(acc[q], b, xrow + kb * kBlkK, c);
        }
    }
}

// Group reduction of the four warps' fragments: red[w][q][row][tok].
template <int NM>
MOE_DEV void frag_store(float* red, const float (&acc)[NM][4], int wg, int gl, int c) {
#pragma unroll
    for (int q = 0; q < NM; ++q) {
        float* r = red + ((wg * NM + q) * 16) * 8;
        r[gl * 8 + 2 * c] = acc[q][0];
        r[gl * 8 + 2 * c + 1] = acc[q][1];
        r[(gl + 8) * 8 + 2 * c] = acc[q][2];
        r[(gl + 8) * 8 + 2 * c + 1] = acc[q][3];
    }
}
MOE_DEV float frag_sum(const float* red, int NM, int q, int row, int t) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < 4; ++w) v += red[((w * NM + q) * 16 + row) * 8 + t];
    return v;
}

// Top-k of one token by one warp (rule of route.cu: logit descending, expert
// index ascending; weights = softmax over the selected).  Lane l owns the
// experts l, l+32, ... (keys staged in shared memory); each lane caches its
// best remaining (key, expert), so a round is two warp reductions plus a
// rescan by the winning lane only.
MOE_DEV uint32_t fkey(float v) {
    const uint32_t b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
MOE_DEV float fkey_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}
__device__ __noinline__ void warp_topk_smem(const float* __restrict__ row, int E, int k, uint32_t* keys, int* ids,
                                            float* wts) {
    // keys[l + 32 i] = order-preserving key of expert l + 32 i (0 = absent)
    const int lane = threadIdx.x & 31;
    const int per = (E + 31) / 32;
    uint32_t bk = 0, bi = 0xffffffffu;
#pragma unroll 1
    for (int i0 = 0; i0 < per; i0 += 8) {              // 8 loads in flight per lane
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = lane + 32 * (i0 + u);
            v[u] = (i0 + u < per && e < E) ? __ldcg(row + e) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = lane + 32 * (i0 + u);
            if (i0 + u < per) {
                const uint32_t kk = e < E ? fkey(v[u]) : 0u;
                keys[e] = kk;
                if (kk > bk) { bk = kk; bi = (uint32_t)e; }
            }
        }
    }
    __syncwarp();
    float my_val = 0.0f, lmax = 0.0f;
    int my_idx = 0;
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
        const uint32_t top = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t e = __reduce_min_sync(0xffffffffu, (bk == top) ? bi : 0xffffffffu);
        const float v = fkey_value(top);
        if (j == 0) lmax = v;
        if (lane == j) { my_val = v; my_idx = (int)e; }
        if (bi == e) {                                   // the owner drops it and rescans its entries
            keys[e] = 0u;
            bk = 0; bi = 0xffffffffu;
#pragma unroll 1
            for (int i = 0; i < per; ++i) {
                const uint32_t kk = keys[lane + 32 * i];
                if (kk > bk) { bk = kk; bi = (uint32_t)(lane + 32 * i); }
            }
        }
    }
    const float ex = (lane < k) ? expf(my_val - lmax) : 0.0f;
    const float sum = warp_sum(ex);
    if (lane < k) {
        ids[lane] = my_idx;
        wts[lane] = __fdiv_rn(ex, sum);
    }
}

// Parallel top-k for the plan: every warp sorts chunks of 32 logits
// (bitonic, descending on the composite (key, ~expert): larger logit first,
// then smaller expert index, the rule above) and keeps the best RL of each;
// then one warp per token merges the sorted runs, two warp reductions per
// selected expert.  cand holds T x ceil(E/32) runs of RL composites.
MOE_DEV unsigned long long topk_composite(float v, int e) {
    return ((unsigned long long)fkey(v) << 32) | (uint32_t)~(uint32_t)e;
}
MOE_DEV unsigned long long warp_sort_desc(unsigned long long v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, stride);
            const bool desc = (lane & size) == 0 || size == 32;
            const bool lower = (lane & stride) == 0;
            v = (desc == lower) ? (v > o ? v : o) : (v < o ? v : o);
        }
    return v;
}
__device__ __noinline__ void topk_sort_chunks(const float* __restrict__ logits, int T, int E, int RL,
                                              unsigned long long* cand) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int NC = (E + 31) / 32;
#pragma unroll 1
    for (int ch = warp; ch < T * NC; ch += nw) {
        const int t = ch / NC, e = (ch % NC) * 32 + lane;
        const unsigned long long v = warp_sort_desc(e < E ? topk_composite(__ldcg(logits + (size_t)t * E + e), e) : 0ull);
        if (lane < RL) cand[(size_t)ch * RL + lane] = v;
    }
}
__device__ __noinline__ void topk_merge(const unsigned long long* cand, int NC, int RL, int k, int* ids, float* wts) {
    const int lane = threadIdx.x & 31;
    int ptr = 0;
    unsigned long long head = lane < NC ? cand[(size_t)lane * RL] : 0ull;
    float my_val = 0.0f, lmax = 0.0f;
    int my_idx = 0;
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
        const uint32_t hi = (uint32_t)(head >> 32);
        const uint32_t mhi = __reduce_max_sync(0xffffffffu, hi);
        const uint32_t mlo = __reduce_max_sync(0xffffffffu, hi == mhi ? (uint32_t)head : 0u);
        const float v = fkey_value(mhi);
        if (j == 0) lmax = v;
        if (lane == j) { my_val = v; my_idx = (int)~mlo; }
        if (hi == mhi && (uint32_t)head == mlo) {       // the winning run advances
            ++ptr;
            head = ptr < RL ? cand[(size_t)lane * RL + ptr] : 0ull;
        }
    }
    const float ex = (lane < k) ? expf(my_val - lmax) : 0.0f;
    const float sum = warp_sum(ex);
    if (lane < k) {
        ids[lane] = my_idx;
        wts[lane] = __fdiv_rn(ex, sum);
    }
}

// Tokens of the item whose first slot is s0 (slot order); written by the
// group's first thread.
__device__ __noinline__ int group_item_tokens(const int* __restrict__ ids, int n, int k, int s0, int* tok, int* slot, bool writer) {
    const int e0 = ids[s0];
    int c = 0;
#pragma unroll 1
    for (int s = s0; s < n && c < kDecMaxT; ++s) {
        if (ids[s] == e0) {
            if (writer) { tok[c] = s / k; slot[c] = s; }
            ++c;
        }
    }
    return c;
}

// Staging of m rows (row_of[t], t < m) into rows 0..m-1 of dst (row stride ld
// elements) and zeros into row m, by threads tid0 .. tid0+nthr-1.
MOE_DEV void pack16(__nv_bfloat16* d, const float (&v)[16]) {
    uint4* p = reinterpret_cast<uint4*>(d);
    p[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
    p[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                      pack_bf16x2(v[14], v[15]));
}
__device__ __noinline__ void stage_bf16(__nv_bfloat16* dst, int ld, const __nv_bfloat16* src, int K, const int* row_of, int m,
                        int tid, int nthr) {
    const int per = K / 8;
#pragma unroll 1
    for (int i = tid; i < (m + 1) * per; i += nthr) {
        const int t = i / per, c = i % per;
        const uint4 v = t < m ? *reinterpret_cast<const uint4*>(src + (size_t)row_of[t] * K + c * 8) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(dst + (size_t)t * ld + c * 8) = v;
    }
}
// W4A4 activations: the NVFP4 values q * s_b of each 16-element block.
__device__ __noinline__ void stage_fp4(__nv_bfloat16* dst, int ld, const __nv_bfloat16* src, int K, const int* row_of, int m, float g,
                       int tid, int nthr) {
    const int per = K / 16;
#pragma unroll 1
    for (int i = tid; i < (m + 1) * per; i += nthr) {
        const int t = i / per, b = i % per;
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
        pack16(dst + (size_t)t * ld + b * 16, v);
    }
}
// fp32 rows read from L2, as bf16 or (fp4) as NVFP4 values with global scale g.
__device__ __noinline__ void stage_f32(__nv_bfloat16* dst, int ld, const float* src, int K, const int* row_of, int m, bool fp4, float g,
                       int tid, int nthr) {
    const int per = K / 16;
#pragma unroll 1
    for (int i = tid; i < (m + 1) * per; i += nthr) {
        const int t = i / per, b = i % per;
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
        pack16(dst + (size_t)t * ld + b * 16, v);
    }
}

// Shared-expert intermediate of all T tokens from the KP partial gate/up
// sums: a_sh[t][i] = silu(sum_p g) * sum_p u (fixed p order), as bf16 rows
// and a zero row, by all threads of the CTA.
__device__ __noinline__ void stage_shared_act(__nv_bfloat16* dst, int ld, const float* gu, int KP, int T, int I) {
#pragma unroll 1
    for (int i = threadIdx.x; i < (T + 1) * I; i += blockDim.x) {
        const int t = i / I, j = i % I;
        float act = 0.0f;
        if (t < T) {
            float g = 0.0f, u = 0.0f;
#pragma unroll 4
            for (int p = 0; p < KP; ++p) {
                g += __ldcg(gu + ((size_t)p * T + t) * 2 * I + j);
                u += __ldcg(gu + ((size_t)p * T + t) * 2 * I + I + j);
            }
            act = g / (1.0f + expf(-g)) * u;
        }
        dst[(size_t)t * ld + j] = __float2bfloat16_rn(act);
    }
}

// Units of one kind on group slot `slot` of `nslots`: unit u lives on slot
// (u + off) % nslots, so the slot holds first, first + nslots, ... < n.
__host__ __device__ inline int first_unit(int slot, int off, int nslots) {
    return ((slot - off) % nslots + nslots) % nslots;
}
__host__ __device__ inline int count_units(int first, int n, int nslots) {
    return first < n ? (n - 1 - first) / nslots + 1 : 0;
}
// K parts of the shared gate/up slices
__host__ __device__ inline int shared_kparts(int H) {
    const int KB = H / kBlkK;
    return (KB % 4 == 0) ? 4 : (KB % 2 == 0 ? 2 : 1);
}

// Shared-memory carve-up of one launch (byte offsets, 16-aligned): staged x
// (and W4A4 x), the group reduction buffers, the shared-expert activations,
// then four equal group regions.
struct FusedSmem {
    int xs, xq, red, act, grp, grp_bytes;
};
__host__ __device__ inline FusedSmem fused_layout(int T, int H, int I, bool fp4) {
    FusedSmem L;
    const int xrow = (H + kXPad) * 2, arow = (I + kXPad) * 2;
    L.xs = 0;
    L.xq = L.xs + (T + 1) * xrow;
    L.red = L.xq + (fp4 ? (T + 1) * xrow : 0);
    L.act = L.red + kGroups * 4 * 2 * 16 * 8 * 4;
    L.grp = L.act + (T + 1) * arow;
    L.grp_bytes = ((kFusedSmem - L.grp) / kGroups) & ~15;
    return L;
}
__host__ __device__ inline int stage_bytes(int I) { return (kDecMaxT + 1) * (I + kXPad) * 2; }

// Slots of the item whose first slot is s0 (slot order), by one thread.
__device__ __noinline__ int item_slots(const int* __restrict__ ids, int n, int s0, int* slot) {
    const int e0 = ids[s0];
    int c = 0;
#pragma unroll 1
    for (int s = s0; s < n && c < kDecMaxT; ++s)
        if (ids[s] == e0) slot[c++] = s;
    return c;
}

// Staging of the intermediate rows of several down units at once (one L2
// round trip): unit j owns staging rows row0[j] .. row0[j] + m[j], the last
// of them zero; rows of units with fp4_of[j] become NVFP4 values.
__device__ __noinline__ void stage_units(__nv_bfloat16* dst, int ld, const float* src, int I, const int* m,
                                         const int* row0, const int* slots, const unsigned char* fp4_of, int nu_,
                                         int rows, float g, int gtid) {
    const int per = I / 16;
#pragma unroll 1
    for (int i0 = gtid; i0 < rows * per; i0 += 2 * 128) {
        float v[2][16];
        int rr[2], bb[2], jj[2], tt[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int i = i0 + q * 128;
            rr[q] = i / per;
            bb[q] = i % per;
            int j = 0;
#pragma unroll 1
            while (j + 1 < nu_ && row0[j + 1] <= rr[q]) ++j;
            jj[q] = j;
            tt[q] = rr[q] - row0[j];
            const bool live = i < rows * per && tt[q] < m[j];
            const float4* s = reinterpret_cast<const float4*>(src + (size_t)(live ? slots[j * kDecMaxT + tt[q]] : 0) * I + bb[q] * 16);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float4 f = live ? __ldcg(s + w) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                v[q][4 * w] = f.x; v[q][4 * w + 1] = f.y; v[q][4 * w + 2] = f.z; v[q][4 * w + 3] = f.w;
            }
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            if (i0 + q * 128 < rows * per) {
                if (fp4_of[jj[q]]) fp4_block_values(v[q], g);
                pack16(dst + (size_t)rr[q] * ld + bb[q] * 16, v[q]);
            }
        }
    }
}

// y rows of block hb (16 columns of H, T tokens): sum of the k partials in
// fixed slot order plus the shared expert's, by one group.
__device__ __noinline__ void combine_block(const float* part, const float* part_sh, __nv_bfloat16* y, int H, int k,
                                           int T, int hb, int gtid) {
    if (gtid < 16 * T) {
        const int t = gtid >> 4, hh = hb * 16 + (gtid & 15);
        float sum = 0.0f;
#pragma unroll 1
        for (int j0 = 0; j0 < k; j0 += 8) {             // fixed order j = 0 .. k-1, 8 loads in flight
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = j0 + u < k ? __ldcg(part + (size_t)(t * k + j0 + u) * H + hh) : 0.0f;
#pragma unroll
            for (int u = 0; u < 8; ++u) sum += v[u];
        }
        if (part_sh) sum += __ldcg(part_sh + (size_t)t * H + hh);
        y[(size_t)t * H + hh] = __float2bfloat16_rn(sum);
    }
}

// Ticket of a 16-row block of H: the last of its `items` units sums the
// partials in fixed slot order, y_t = sum_j part[t*k+j] + shared_t, and
// clears the counter.  Called by all threads of one group.
__device__ __noinline__ void finish_block(unsigned int* counters, const float* part, const float* part_sh,
                                          __nv_bfloat16* y, int H, int k, int T, int items, int hb, int group, int gtid,
                                          volatile int* last) {
    group_sync(group);
    if (gtid == 0) *last = (ticket_acq_rel(counters + hb) == (unsigned)items - 1u);
    group_sync(group);
    if (*last) {
        if (gtid < 16 * T) {
            const int t = gtid >> 4, hh = hb * 16 + (gtid & 15);
            float sum = 0.0f;
#pragma unroll 1
            for (int j0 = 0; j0 < k; j0 += 8) {         // fixed order j = 0 .. k-1, 8 loads in flight
                float v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = j0 + u < k ? __ldcg(part + (size_t)(t * k + j0 + u) * H + hh) : 0.0f;
#pragma unroll
                for (int u = 0; u < 8; ++u) sum += v[u];
            }
            if (part_sh) sum += __ldcg(part_sh + (size_t)t * H + hh);
            y[(size_t)t * H + hh] = __float2bfloat16_rn(sum);
        }
        group_sync(group);
        if (gtid == 0) counters[hb] = 0u;
    }
}

template <int Q, int TM>
__global__ void __launch_bounds__(kFThreads, 1) k_decode_fused(FusedArgs f) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ Plan plan;
    __shared__ int ids_s[kDecMaxSlots];
    __shared__ float w_s[kDecMaxSlots];
    __shared__ int ident[kDecMaxT];
    __shared__ int g_tok[kGroups][kDecMaxT], g_slot[kGroups][kDecMaxT];
    __shared__ volatile int g_last[kGroups];
    __shared__ volatile int abort_s;
    constexpr int kMaxDn = 16;                   // down units per group handled as one batch
    __shared__ int u_m[kGroups][kMaxDn], u_row0[kGroups][kMaxDn], u_slot[kGroups][kMaxDn * kDecMaxT];
    __shared__ unsigned char u_fp4[kGroups][kMaxDn];
    __shared__ int u_rows[kGroups];
    __shared__ int u_last[kGroups][kMaxDn + 4];
    const DecodeArgs& a = f.d;
    const ExpertArgs& ex = a.ex;
    const int H = ex.H, I = ex.I, k = ex.k, E = ex.E, T = a.T;
    const int n = T * k;
    const bool fp4 = (Q == Q_NVFP4);
    const int ldx = H + kXPad, lda = I + kXPad;
    const FusedSmem L = fused_layout(T, H, I, fp4);
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem_raw + L.xs);
    __nv_bfloat16* xq = reinterpret_cast<__nv_bfloat16*>(smem_raw + L.xq);
    __nv_bfloat16* ash = reinterpret_cast<__nv_bfloat16*>(smem_raw + L.act);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gl = lane >> 2, c = lane & 3;
    const int group = warp >> 2, wg = warp & 3, gtid = threadIdx.x & 127;
    float* red = reinterpret_cast<float*>(smem_raw + L.red) + group * 4 * 2 * 16 * 8;
    uint8_t* gbase = smem_raw + L.grp + group * L.grp_bytes;
    const int GB = L.grp_bytes;
    int* tok = g_tok[group];
    int* slot_of = g_slot[group];
    const int nslots = kGroups * gridDim.x;
    const int my_slot = group * gridDim.x + blockIdx.x;      // groups spread over the SMs first
    const int KBH = H / kBlkK, KBI = I / kBlkK;
    const int KP = shared_kparts(H), KBP = KBH / KP;         // shared gate/up: K parts, k-blocks per part
    const Slice s_gu = qslice(Q, H), s_dn = qslice(Q, I);
    const bool has_sh = ex.sh_gate != nullptr;
    const int stg_bytes = stage_bytes(I);

    // ---- routing-independent units and their place in the group region:
    //      [shared down (kept until phase 2) | router rows | shared gate/up]
    const int U_R = f.wr ? E : 0, U_SGU = has_sh ? (I / 16) * KP : 0, U_SD = has_sh ? H / 16 : 0;
    const int r_first = first_unit(my_slot, 0, nslots);
    const int sgu_first = first_unit(my_slot, nslots / 2, nslots);
    const int sd_first = first_unit(my_slot, (3 * nslots) / 4, nslots);
    const int n_r = count_units(r_first, U_R, nslots);
    const int n_sgu = count_units(sgu_first, U_SGU, nslots);
    const int n_sd = count_units(sd_first, U_SD, nslots);
    const int sd_bytes = KBI * 2048, sgu_bytes = 2 * KBP * 2048, r_bytes = H * 2;
    const int gu_bytes = 2 * s_gu.bytes, dn_bytes = s_dn.bytes;
    const int one_unit = max(max(r_bytes + sgu_bytes, gu_bytes), stg_bytes + dn_bytes);
    const bool sd_pre = n_sd * sd_bytes + one_unit <= GB;
    const int sd_end = sd_pre ? n_sd * sd_bytes : 0;
    const int r_off = sd_end;
    const bool r_all = r_off + n_r * r_bytes + sgu_bytes <= GB;
    const int sgu_off = r_off + (r_all ? n_r * r_bytes : r_bytes);
    const bool sgu_all = sgu_off + n_sgu * sgu_bytes <= GB;

    if (threadIdx.x == 0) abort_s = 0;
    if (threadIdx.x < kDecMaxT) ident[threadIdx.x] = threadIdx.x;
    __syncthreads();

    // ---- copies that need nothing from the router, in commit order
    //      B: router rows, C: shared gate/up, A: shared down
    if (r_all)
#pragma unroll 1
        for (int j = 0; j < n_r; ++j) {
            const uint8_t* src = reinterpret_cast<const uint8_t*>(f.wr) + (size_t)(r_first + j * nslots) * r_bytes;
#pragma unroll 1
            for (int i = gtid; i < r_bytes / 16; i += 128) cp16(gbase + r_off + j * r_bytes + i * 16, src + i * 16);
        }
    cp_commit();
    if (sgu_all)
#pragma unroll 1
        for (int j = 0; j < n_sgu; ++j) {
            const int u = sgu_first + j * nslots, r0 = (u / KP) * 16, kp = u % KP;
            uint8_t* d = gbase + sgu_off + j * sgu_bytes;
            load_bslice(d, ex.sh_gate, KBH, r0, kp * KBP, KBP, gtid);
            load_bslice(d + KBP * 2048, ex.sh_up, KBH, r0, kp * KBP, KBP, gtid);
        }
    cp_commit();
    if (sd_pre)
#pragma unroll 1
        for (int j = 0; j < n_sd; ++j)
            load_bslice(gbase + j * sd_bytes, ex.sh_down, KBI, (sd_first + j * nslots) * 16, 0, KBI, gtid);
    cp_commit();

    // ---- stage activations (rows t < T, zero row T)
    const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(a.x);
    stage_bf16(xs, ldx, x, H, ident, T, threadIdx.x, blockDim.x);
    if (fp4) stage_fp4(xq, ldx, x, H, ident, T, ex.g_x, threadIdx.x, blockDim.x);
    __syncthreads();

    // ---- phase 0a: router rows, one warp per row
#pragma unroll 1
    for (int j0 = 0; j0 < n_r; j0 += (r_all ? n_r : 1)) {
        const int nj = r_all ? n_r : 1;
        if (r_all) {
            cp_wait<2>();                                      // B done
        } else {
#pragma unroll 1
            for (int i = gtid; i < r_bytes / 16; i += 128)
                cp16(gbase + r_off + i * 16,
                     reinterpret_cast<const uint8_t*>(f.wr) + (size_t)(r_first + j0 * nslots) * r_bytes + i * 16);
            cp_commit();
            cp_wait<0>();
        }
        group_sync(group);
#pragma unroll 1
        for (int j = wg; j < nj; j += 4) {
            const int e = r_first + (j0 + j) * nslots;
            const __nv_bfloat16* row = reinterpret_cast<const __nv_bfloat16*>(gbase + r_off + j * r_bytes);
            float acc[TM];
#pragma unroll
            for (int t = 0; t < TM; ++t) acc[t] = 0.0f;
#pragma unroll 1
            for (int c8 = lane; c8 < H / 8; c8 += 32) {
                const uint4 wq = *reinterpret_cast<const uint4*>(row + c8 * 8);
                const uint32_t wv[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
                for (int t = 0; t < TM; ++t) {
                    if (t < T) {
                        const uint4 xv4 = *reinterpret_cast<const uint4*>(xs + t * ldx + c8 * 8);
                        const uint32_t xv[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            acc[t] = fmaf(bf16_lo(wv[i]), bf16_lo(xv[i]), acc[t]);
                            acc[t] = fmaf(bf16_hi(wv[i]), bf16_hi(xv[i]), acc[t]);
                        }
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < TM; ++t) {
                if (t < T) {
                    const float sum = warp_sum(acc[t]);
                    if (lane == 0) f.logits[(size_t)t * E + e] = sum;
                }
            }
        }
        group_sync(group);
    }

    // ---- phase 0b: partial shared gate/up sums over the group's K parts
#pragma unroll 1
    for (int j0 = 0; j0 < n_sgu; j0 += (sgu_all ? n_sgu : 1)) {
        const int nj = sgu_all ? n_sgu : 1;
        if (sgu_all) {
            cp_wait<1>();                                      // B, C done
        } else {
            const int u = sgu_first + j0 * nslots, r0 = (u / KP) * 16, kp = u % KP;
            load_bslice(gbase + sgu_off, ex.sh_gate, KBH, r0, kp * KBP, KBP, gtid);
            load_bslice(gbase + sgu_off + KBP * 2048, ex.sh_up, KBH, r0, kp * KBP, KBP, gtid);
            cp_commit();
            cp_wait<0>();
        }
        group_sync(group);
#pragma unroll 1
        for (int j = 0; j < nj; ++j) {
            const int u = sgu_first + (j0 + j) * nslots, r0 = (u / KP) * 16, kp = u % KP;
            const uint8_t* d = gbase + sgu_off + j * sgu_bytes;
            const uint8_t* const mats[2] = {d, d + KBP * 2048};
            float acc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
            slice_mma<Q_BF16, 2>(acc, mats, s_gu, kp * KBP, (kp + 1) * KBP, wg, xs + (gl < T ? gl : T) * ldx, gl, c);
            frag_store<2>(red, acc, wg, gl, c);
            group_sync(group);
            {
                const int row = gtid >> 3, t = gtid & 7;
                if (t < T) {
                    float* dst = f.gu_sh + ((size_t)kp * T + t) * 2 * I + r0 + row;
                    dst[0] = frag_sum(red, 2, 0, row, t);
                    dst[I] = frag_sum(red, 2, 1, row, t);
                }
            }
            group_sync(group);
        }
    }

    const long long wait_limit = f.wait_limit > 0 ? f.wait_limit : kBarrierLimitCycles;
    bool withhold = f.withhold_cta == (int)blockIdx.x;
    if (f.wr && !grid_barrier(f.bar, f.err, &abort_s, withhold, wait_limit)) {
        cp_wait<0>();                    // no copy of this CTA outlives it
        return;
    }
    if (f.wr) withhold = false;          // the test hook withholds one arrival only

    // ---- phase 1: top-k (every CTA), plan, routed gate/up units
    if (f.wr) {
        const int NC = (E + 31) / 32, RL = k <= 16 ? 16 : 32;
        if (T * NC * RL * 8 <= kGroups * 4 * 2 * 16 * 8 * 4) {
            // sorted runs in the (idle) reduction buffers
            unsigned long long* cand = reinterpret_cast<unsigned long long*>(smem_raw + L.red);
            topk_sort_chunks(f.logits, T, E, RL, cand);
            __syncthreads();
            if (warp < T) topk_merge(cand + (size_t)warp * NC * RL, NC, RL, k, ids_s + warp * k, w_s + warp * k);
        } else {
            // keys in the group region past the kept shared down slices (free now)
#pragma unroll 1
            for (int t = warp; t < T; t += kFWarps)
                warp_topk_smem(f.logits + (size_t)t * E, E, k, reinterpret_cast<uint32_t*>(gbase + sd_end) + wg * 1024,
                               ids_s + t * k, w_s + t * k);
        }
        __syncthreads();
        if (blockIdx.x == 0)
#pragma unroll 1
            for (int s = threadIdx.x; s < n; s += blockDim.x) { f.ids_out[s] = ids_s[s]; f.w_out[s] = w_s[s]; }
    } else {
#pragma unroll 1
        for (int s = threadIdx.x; s < n; s += blockDim.x) { ids_s[s] = __ldcg(a.ids + s); w_s[s] = __ldcg(a.w + s); }
    }
    __syncthreads();
#pragma unroll 1
    for (int s = threadIdx.x; s < n; s += blockDim.x) plan.ids[s] = ids_s[s];
    __syncthreads();
#pragma unroll 1
    for (int s = threadIdx.x; s < n; s += blockDim.x) {
        const int e = plan.ids[s];
        bool fst = true;
#pragma unroll 1
        for (int q = 0; q < s; ++q) fst = fst && (plan.ids[q] != e);
        plan.is_first[s] = fst;
    }
    __syncthreads();
    if (warp == 0) {
        int base = 0;
#pragma unroll 1
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
    const int RBI = I / 16, RBH = H / 16;
    const int U_GU = nu * RBI, U_DN = nu * RBH;
    const int gu_first = first_unit(my_slot, 0, nslots);
    const int dn_first = first_unit(my_slot, U_GU % nslots, nslots);   // down units after the gate/up slots
    const int n_gu = count_units(gu_first, U_GU, nslots);
    const int n_dn = count_units(dn_first, U_DN, nslots);
    //      [shared down (kept) | gate/up units, then the a staging | down units]
    const bool gu_all = sd_end + n_gu * gu_bytes <= GB;
    const int gu_space = gu_all ? n_gu * gu_bytes : gu_bytes;
    const int dn_off = sd_end + max(gu_space, stg_bytes);
    const bool dn_pre = gu_all && dn_off + n_dn * dn_bytes <= GB;

    auto unit_expert = [&](int ui) { return plan.ids[plan.first[ui]]; };
    auto valid_expert = [&](int e) { return e >= 0 && e < E; };
    auto load_gu = [&](uint8_t* d, int u) {
        const int e = unit_expert(u / RBI), r0 = (u % RBI) * 16;
        if (valid_expert(e)) {
            load_qslice<Q>(d, expert_mat(ex.gate, e), s_gu, r0, gtid);
            load_qslice<Q>(d + s_gu.bytes, expert_mat(ex.up, e), s_gu, r0, gtid);
        }
    };
    auto load_dn = [&](uint8_t* d, int u) {
        const int e = unit_expert(u / RBH), r0 = (u % RBH) * 16;
        if (valid_expert(e)) load_qslice<Q>(d, expert_mat(ex.down, e), s_dn, r0, gtid);
    };
    if (gu_all)
#pragma unroll 1
        for (int j = 0; j < n_gu; ++j) load_gu(gbase + sd_end + j * gu_bytes, gu_first + j * nslots);
    cp_commit();                                                         // D: gate/up
    if (dn_pre)
#pragma unroll 1
        for (int j = 0; j < n_dn; ++j) load_dn(gbase + dn_off + j * dn_bytes, dn_first + j * nslots);
    cp_commit();                                                         // E: down

    const __nv_bfloat16* xg = fp4 ? xq : xs;
#pragma unroll 1
    for (int j0 = 0; j0 < n_gu; j0 += (gu_all ? n_gu : 1)) {
        const int nj = gu_all ? n_gu : 1;
        if (gu_all) {
            cp_wait<1>();                                                // D (and all before it) done
        } else {
            load_gu(gbase + sd_end, gu_first + j0 * nslots);
            cp_commit();
            cp_wait<0>();
        }
        group_sync(group);
#pragma unroll 1
        for (int j = 0; j < nj; ++j) {
            const int u = gu_first + (j0 + j) * nslots;
            const int ui = u / RBI, r0 = (u % RBI) * 16, e = unit_expert(ui);
            const int m = group_item_tokens(plan.ids, n, k, plan.first[ui], tok, slot_of, gtid == 0);
            group_sync(group);
            const bool valid = valid_expert(e);
            float acc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
            if (valid) {
                const uint8_t* d = gbase + sd_end + j * gu_bytes;
                const uint8_t* const mats[2] = {d, d + s_gu.bytes};
                slice_mma<Q, 2>(acc, mats, s_gu, 0, KBH, wg, xg + (gl < m ? tok[gl] : T) * ldx, gl, c);
            }
            frag_store<2>(red, acc, wg, gl, c);
            group_sync(group);
            {
                const int row = gtid >> 3, t = gtid & 7;
                if (t < m) {
                    const float sc = (fp4 && valid) ? ex.g_gate[e] * ex.g_x : 1.0f;
                    const float gg = frag_sum(red, 2, 0, row, t) * sc, uu = frag_sum(red, 2, 1, row, t) * sc;
                    a.a[(size_t)slot_of[t] * I + r0 + row] = valid ? gg / (1.0f + expf(-gg)) * uu : 0.0f;
                }
            }
            group_sync(group);
        }
    }
    if (!grid_barrier(f.bar, f.err, &abort_s, withhold, wait_limit)) {
        cp_wait<0>();
        return;
    }

    // ---- phase 2: down units and the shared down slices; tickets, combine
    cp_wait<0>();                                                        // every prefetch landed
    if (has_sh) stage_shared_act(ash, lda, f.gu_sh, KP, T, I);
    __syncthreads();
    __nv_bfloat16* as = reinterpret_cast<__nv_bfloat16*>(gbase + sd_end);
    const int items = nu + (has_sh ? 1 : 0);
    __nv_bfloat16* const y = reinterpret_cast<__nv_bfloat16*>(a.y);
    // batched path: every down unit's rows staged at once, all units and the
    // shared slices computed, then all tickets taken together
    bool batch = dn_pre && n_dn <= kMaxDn && n_sd <= 4 && sd_pre;
    if (batch) {
        if (gtid < n_dn) {
            const int u = dn_first + gtid * nslots, ui = u / RBH;
            u_m[group][gtid] = item_slots(plan.ids, n, plan.first[ui], &u_slot[group][gtid * kDecMaxT]);
            u_fp4[group][gtid] = fp4 && valid_expert(unit_expert(ui));
        }
        group_sync(group);
        if (gtid == 0) {
            int r = 0;
#pragma unroll 1
            for (int j = 0; j < n_dn; ++j) { u_row0[group][j] = r; r += u_m[group][j] + 1; }
            u_rows[group] = r;
        }
        group_sync(group);
        batch = u_rows[group] * lda * 2 <= dn_off - sd_end;
    }
    if (batch) {
        stage_units(as, lda, a.a, I, u_m[group], u_row0[group], u_slot[group], u_fp4[group], n_dn, u_rows[group], ex.g_a,
                    gtid);
        group_sync(group);
#pragma unroll 1
        for (int j = 0; j < n_dn; ++j) {
            const int u = dn_first + j * nslots;
            const int ui = u / RBH, r0 = (u % RBH) * 16, e = unit_expert(ui);
            const bool valid = valid_expert(e);
            const int m = u_m[group][j];
            float acc[1][4] = {{0, 0, 0, 0}};
            if (valid) {
                const uint8_t* const mats[1] = {gbase + dn_off + j * dn_bytes};
                slice_mma<Q, 1>(acc, mats, s_dn, 0, KBI, wg, as + (u_row0[group][j] + (gl < m ? gl : m)) * lda, gl, c);
            }
            frag_store<1>(red, acc, wg, gl, c);
            group_sync(group);
            {
                const int row = gtid >> 3, t = gtid & 7;
                if (t < m) {
                    const float dsc = (fp4 && valid) ? ex.g_down[e] * ex.g_a : 1.0f;
                    const int s = u_slot[group][j * kDecMaxT + t];
                    a.part[(size_t)s * H + r0 + row] = valid ? w_s[s] * frag_sum(red, 1, 0, row, t) * dsc : 0.0f;
                }
            }
            group_sync(group);
        }
#pragma unroll 1
        for (int j = 0; j < n_sd; ++j) {
            const int r0 = (sd_first + j * nslots) * 16;
            float acc[1][4] = {{0, 0, 0, 0}};
            const uint8_t* const mats[1] = {gbase + j * sd_bytes};
            slice_mma<Q_BF16, 1>(acc, mats, s_dn, 0, KBI, wg, ash + (gl < T ? gl : T) * lda, gl, c);
            frag_store<1>(red, acc, wg, gl, c);
            group_sync(group);
            {
                const int row = gtid >> 3, t = gtid & 7;
                if (t < T) a.part_sh[(size_t)t * H + r0 + row] = frag_sum(red, 1, 0, row, t);
            }
            group_sync(group);
        }
        // tickets: one per unit, all in flight together (each releases the
        // group's partials, ordered before it by the barrier)
        group_sync(group);
        if (gtid < n_dn + n_sd) {
            const int hb = gtid < n_dn ? (dn_first + gtid * nslots) % RBH : sd_first + (gtid - n_dn) * nslots;
            const bool last = ticket_acq_rel(a.counters + hb) == (unsigned)items - 1u;
            u_last[group][gtid] = last ? hb : -1;
        }
        group_sync(group);
#pragma unroll 1
        for (int j = 0; j < n_dn + n_sd; ++j) {
            const int hb = u_last[group][j];
            if (hb >= 0) {
                combine_block(a.part, has_sh ? a.part_sh : nullptr, y, H, k, T, hb, gtid);
                if (gtid == 0) a.counters[hb] = 0u;
            }
        }
        return;
    }
#pragma unroll 1
    for (int j = 0; j < n_dn; ++j) {
        const int u = dn_first + j * nslots;
        const int ui = u / RBH, r0 = (u % RBH) * 16, e = unit_expert(ui);
        const bool valid = valid_expert(e);
        const uint8_t* dsl = gbase + dn_off + j * dn_bytes;
        if (!dn_pre) {
            dsl = gbase + sd_end + stg_bytes;
            load_dn(gbase + sd_end + stg_bytes, u);
            cp_commit();
        }
        const int m = group_item_tokens(plan.ids, n, k, plan.first[ui], tok, slot_of, gtid == 0);
        group_sync(group);
        stage_f32(as, lda, a.a, I, slot_of, m, fp4 && valid, ex.g_a, gtid, 128);
        if (!dn_pre) cp_wait<0>();
        group_sync(group);
        float acc[1][4] = {{0, 0, 0, 0}};
        if (valid) {
            const uint8_t* const mats[1] = {dsl};
            slice_mma<Q, 1>(acc, mats, s_dn, 0, KBI, wg, as + (gl < m ? gl : m) * lda, gl, c);
        }
        frag_store<1>(red, acc, wg, gl, c);
        group_sync(group);
        {
            const int row = gtid >> 3, t = gtid & 7;
            if (t < m) {
                const float dsc = (fp4 && valid) ? ex.g_down[e] * ex.g_a : 1.0f;
                const int s = slot_of[t];
                a.part[(size_t)s * H + r0 + row] = valid ? w_s[s] * frag_sum(red, 1, 0, row, t) * dsc : 0.0f;
            }
        }
        finish_block(a.counters, a.part, has_sh ? a.part_sh : nullptr, reinterpret_cast<__nv_bfloat16*>(a.y), H, k, T, items,
                     r0 / 16, group, gtid, &g_last[group]);
    }
#pragma unroll 1
    for (int j = 0; j < n_sd; ++j) {
        const int r0 = (sd_first + j * nslots) * 16;
        const uint8_t* dsl = gbase + j * sd_bytes;
        if (!sd_pre) {
            dsl = gbase;
            load_bslice(gbase, ex.sh_down, KBI, r0, 0, KBI, gtid);
            cp_commit();
            cp_wait<0>();
            group_sync(group);
        }
        float acc[1][4] = {{0, 0, 0, 0}};
        const uint8_t* const mats[1] = {dsl};
        slice_mma<Q_BF16, 1>(acc, mats, s_dn, 0, KBI, wg, ash + (gl < T ? gl : T) * lda, gl, c);
        frag_store<1>(red, acc, wg, gl, c);
        group_sync(group);
        {
            const int row = gtid >> 3, t = gtid & 7;
            if (t < T) a.part_sh[(size_t)t * H + r0 + row] = frag_sum(red, 1, 0, row, t);
        }
        finish_block(a.counters, a.part, has_sh ? a.part_sh : nullptr, reinterpret_cast<__nv_bfloat16*>(a.y), H, k, T, items,
                     r0 / 16, group, gtid, &g_last[group]);
    }
}

size_t fused_smem_bytes(int H, int I) {
    (void)H;
    (void)I;
    return kFusedSmem;
}

// The fused kernel needs one unit of every kind to fit a group's region;
// otherwise the two-kernel decode path runs.
bool fused_supported(int T, int H, int I, int quant) {
    if (T < 1 || T > kDecMaxT) return false;
    if (quant == Q_FP6) return false;          // two-plane units: the two-kernel path
    const FusedSmem L = fused_layout(T, H, I, quant == Q_NVFP4);
    const Slice gu = qslice(quant, H), dn = qslice(quant, I);
    const int KBP = (H / kBlkK) / shared_kparts(H);
    const int need_a = H * 2 + 2 * KBP * 2048;                // a router row and a shared gate/up slice
    const int need_b = 2 * gu.bytes + dn.bytes;               // a gate/up unit (and room for one down unit)
    const int need_c = stage_bytes(I) + dn.bytes;             // the a staging and one down unit
    const int need_d = (I / kBlkK) * 2048;                    // a shared down slice
    return L.grp_bytes >= need_a && L.grp_bytes >= need_b && L.grp_bytes >= need_c && L.grp_bytes >= need_d;
}

template <int Q, int TM>
static cudaError_t launch_fused_qt(const FusedArgs& f, cudaStream_t st, int grid) {
    const size_t smem = fused_smem_bytes(f.d.ex.H, f.d.ex.I);
    cudaError_t err = cudaFuncSetAttribute(k_decode_fused<Q, TM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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
    err = cudaLaunchKernelEx(&cfg, k_decode_fused<Q, TM>, f);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}
// token-count specialisations: 1, 2, 4, 8
template <int Q>
static cudaError_t launch_fused_q(const FusedArgs& f, cudaStream_t st, int grid) {
    const int T = f.d.T;
    if (T <= 1) return launch_fused_qt<Q, 1>(f, st, grid);
    if (T <= 2) return launch_fused_qt<Q, 2>(f, st, grid);
    if (T <= 4) return launch_fused_qt<Q, 4>(f, st, grid);
    return launch_fused_qt<Q, 8>(f, st, grid);
}

cudaError_t launch_decode_fused(const FusedArgs& f, cudaStream_t st) {
    if (!fused_supported(f.d.T, f.d.ex.H, f.d.ex.I, f.d.ex.quant)) return cudaErrorNotSupported;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
    switch (f.d.ex.quant) {
        case Q_INT4: return launch_fused_q<Q_INT4>(f, st, sms);
        case Q_INT4G32: return launch_fused_q<Q_INT4G32>(f, st, sms);
        case Q_FP8: return launch_fused_q<Q_FP8>(f, st, sms);
        case Q_INT2: return launch_fused_q<Q_INT2>(f, st, sms);
        case Q_NVFP4: return launch_fused_q<Q_NVFP4>(f, st, sms);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
