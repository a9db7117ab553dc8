// Prefill path of the expert computation: grouped GEMMs over the expert
// segments of the permuted tokens on the 5th-generation tensor cores.
//
// The pages run the prefill expert math as a fused MoE GEMM over the tokens
// routed to each expert (the moe_wna16 Triton kernel with a 2-bit unpack,
// "Qwen3.8-Flash-Next on one 24 GB GPU", "What the patch does"; a CUTLASS FP4
// GEMM for NVFP4, "meshapplied/Qwen3.8-Flash-Next-NVFP4-Latest", serve
// command), and prefill is bounded by the expert GEMM once the interconnect
// is out of the way ("Qwen3.8-Flash-Next-FP6-INT8", "Step budget and hardware
// floors").
//
// Design (sm_100a):
//   * swap-AB: 128 weight rows are the MMA's M, up to 128 tokens its N, so an
//     expert with few tokens does not pad M; one tile = (expert, 128 weight
//     rows, up to 128 tokens), K walked in 64-column blocks;
//   * persistent CTAs (one per SM) walk a tile list built on the device from
//     the permutation, grouped by (expert, row block) so consecutive CTAs
//     reuse the same weight tile from L2;
//   * the token operand is stored in permuted (expert-major) order before the
//     GEMMs, so each k-block of a tile is one 2D TMA box of 128 rows;
//   * warp roles: a producer warp issues bulk copies of the packed weights
//     and the TMA loads of the token rows; four dequant warps turn
//     INT4 / INT2 / NVFP4 codes into bf16 A tiles in the 128-byte swizzle the
//     MMA reads; one thread issues tcgen05.mma (kind::f16, fp32 accumulators
//     in TMEM, double buffered); four epilogue warps read TMEM and apply
//     SwiGLU (gate/up) or the routing weight (down);
//   * every mbarrier wait is bounded: on timeout the CTA records an error
//     code, stops all roles, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace moe {

using namespace sm100;

constexpr int kBN = 128;            // tokens per tile (MMA N <= 128)
constexpr int kGemmThreads = 320;   // 10 warps
constexpr int kWarpProducer = 0, kWarpMma = 1, kWarpDeq0 = 2, kWarpEpi0 = 6;
constexpr uint32_t kTmemCols = 512;

template <int MODE> struct GemmCfg;
template <> struct GemmCfg<0> { static constexpr int NMAT = 2, STAGES = 3; };   // gate + up
template <> struct GemmCfg<1> { static constexpr int NMAT = 1, STAGES = 4; };   // down

constexpr int kATile = kBlkN * 128;          // 16 KB: 128 rows x 64 bf16
constexpr int kBTile = kBN * 128;            // 16 KB: 128 tokens x 64 bf16
constexpr int kStgMat = 4096 + 512 + 256;    // packed codes + scales + zeros of one matrix block

template <int MODE>
struct SmemLayout {
    static constexpr int NMAT = GemmCfg<MODE>::NMAT, S = GemmCfg<MODE>::STAGES;
    static constexpr int A = 0;                                  // [S][NMAT][16 KB]
    static constexpr int B = A + S * NMAT * kATile;              // [S][16 KB]
    static constexpr int STG = B + S * kBTile;                   // [S][NMAT][kStgMat]
    static constexpr int BYTES = STG + S * NMAT * kStgMat;
    static constexpr int ALLOC = BYTES + 1024;                   // slack for 1024-byte alignment
};

struct GemmArgs {
    int quant;                // routed weight format
    MatView w0, w1;           // gate/up (mode 0) or down (w0, mode 1)
    const uint8_t* sh0;       // shared expert bf16 images (gate/up or down)
    const uint8_t* sh1;
    const int32_t* perm;      // slot at each permuted position
    const GemmTile* tiles;
    const int* num_tiles;
    int K;                    // reduction length (H or I)
    int k_top;
    int out_ld;               // row length of the outputs (I or H)
    __nv_bfloat16* out;       // mode 0: A_perm [slots, I] (bf16)
    __nv_bfloat16* out_sh;    // mode 0: shared expert intermediate [T, I] (bf16)
    __half* o16;              // mode 1: O [slots, H] by slot id (fp16)
    __half* o16_sh;           // mode 1: shared expert output [T, H] (fp16)
    const float* topk_w;      // mode 1: routing weight of each slot
    const float* g_w;         // NVFP4 per-expert weight global scale, or null
    float g_act;              // NVFP4 activation global scale of the B operand
    float g_req;              // NVFP4: global scale of the requantized intermediate (mode 0)
    const float* tok_scale;   // mode 0, INT4/INT2: power of two of each token's fp16 activations
    int* err;
};

// ------------------------------------------------------------------ dequant
// Row r of one 128x64 block: codes at stg (device layout of layout.cuh),
// written as 64 bf16 into the swizzled A tile.
MOE_DEV void store_chunk(uint8_t* a_tile, int r, int c8, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
    uint8_t* p = a_tile + (r >> 3) * 1024 + (r & 7) * 128 + ((c8 ^ (r & 7)) << 4);
    *reinterpret_cast<uint4*>(p) = make_uint4(w0, w1, w2, w3);
}

MOE_DEV uint32_t bf16x2_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t*>(&v); }

MOE_DEV uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }
MOE_DEV __half f16_sat(float v) { return __float2half_rn(fminf(fmaxf(v, -65504.0f), 65504.0f)); }

// INT4 / INT2 codes -> fp16 (u - 8) * s or (u - z) * s: the integer is exact
// in fp16 and so is the fp16 scale, so each weight is rounded once (2^-12).
MOE_DEV void dequant_row_f16(int quant, const uint8_t* stg, uint8_t* a_tile, int r) {
    if (quant == Q_INT4) {
        const __half2 s2 = __half2half2(reinterpret_cast<const __half*>(stg + 4096)[r]);
        const __half2 off = __float2half2_rn(1032.0f);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint4 q = *reinterpret_cast<const uint4*>(stg + (c * kBlkN + r) * 16);
            const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint32_t o[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t t = ((wv[w] >> (4 * j)) & 0x000F000Fu) | 0x64006400u;   // 1024 + u
                    o[j] = h2_bits(__hmul2(__hsub2(*reinterpret_cast<const __half2*>(&t), off), s2));
                }
                store_chunk(a_tile, r, c * 4 + w, o[0], o[1], o[2], o[3]);
            }
        }
    } else {
        const __half2 s2 = __half2half2(reinterpret_cast<const __half*>(stg + 2048)[r]);
        const __half2 off = __float2half2_rn(1024.0f + (float)stg[2048 + 256 + r]);
        const uint4 q = *reinterpret_cast<const uint4*>(stg + r * 16);
        const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t t = ((wv[w] >> (2 * j)) & 0x00030003u) | 0x64006400u;   // 1024 + u
                o[j] = h2_bits(__hmul2(__hsub2(*reinterpret_cast<const __half2*>(&t), off), s2));
            }
            store_chunk(a_tile, r, 2 * w, o[0], o[1], o[2], o[3]);
            store_chunk(a_tile, r, 2 * w + 1, o[4], o[5], o[6], o[7]);
        }
    }
}

MOE_DEV void dequant_row(int quant, const uint8_t* stg, uint8_t* a_tile, int r) {
    if (quant == Q_INT4) {
        const __half s16 = reinterpret_cast<const __half*>(stg + 4096)[r];
        const __nv_bfloat162 s2 = __bfloat162bfloat162(__float2bfloat16_rn(__half2float(s16)));
        const __nv_bfloat162 off = __bfloat162bfloat162(__float2bfloat16_rn(136.0f));
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint4 q = *reinterpret_cast<const uint4*>(stg + (c * kBlkN + r) * 16);
            const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint32_t o[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t t = ((wv[w] >> (4 * j)) & 0x000F000Fu) | 0x43004300u;   // 128 + u
                    __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&t);
                    v = __hmul2(__hsub2(v, off), s2);                                   // (u - 8) * s
                    o[j] = bf16x2_bits(v);
                }
                store_chunk(a_tile, r, c * 4 + w, o[0], o[1], o[2], o[3]);
            }
        }
    } else if (quant == Q_INT2) {
        const __half s16 = reinterpret_cast<const __half*>(stg + 2048)[r];
        const __nv_bfloat162 s2 = __bfloat162bfloat162(__float2bfloat16_rn(__half2float(s16)));
        const float z = (float)stg[2048 + 256 + r];
        const __nv_bfloat162 off = __bfloat162bfloat162(__float2bfloat16_rn(128.0f + z));
        const uint4 q = *reinterpret_cast<const uint4*>(stg + r * 16);
        const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t t = ((wv[w] >> (2 * j)) & 0x00030003u) | 0x43004300u;   // 128 + u
                __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&t);
                v = __hmul2(__hsub2(v, off), s2);                                   // (u - z) * s
                o[j] = bf16x2_bits(v);
            }
            store_chunk(a_tile, r, 2 * w, o[0], o[1], o[2], o[3]);
            store_chunk(a_tile, r, 2 * w + 1, o[4], o[5], o[6], o[7]);
        }
    } else {  // NVFP4: e2m1 * e4m3 block scale is exact in bf16 (global scale in the epilogue)
        const uint32_t sb4 = *reinterpret_cast<const uint32_t*>(stg + 4096 + r * 4);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint4 q = *reinterpret_cast<const uint4*>(stg + (c * kBlkN + r) * 16);
            const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float sb = e4m3_to_f32((sb4 >> (8 * ((c * 4 + w) >> 1))) & 0xffu);
                uint32_t o[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t t = wv[w] >> (4 * j);
                    o[j] = pack_bf16x2(e2m1_to_f32(t & 0xFu) * sb, e2m1_to_f32((t >> 16) & 0xFu) * sb);
                }
                store_chunk(a_tile, r, c * 4 + w, o[0], o[1], o[2], o[3]);
            }
        }
    }
}

// bytes of one matrix block in the staging area
MOE_DEV void stage_bytes(int quant, int& codes, int& scales, int& zeros) {
    codes = quant == Q_INT2 ? 2048 : 4096;
    scales = quant == Q_NVFP4 ? 512 : 256;
    zeros = quant == Q_INT2 ? 128 : 0;
}

// named barrier of the four epilogue warps
MOE_DEV void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// ------------------------------------------------------------------ kernel
template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
k_grouped_gemm(const __grid_constant__ CUtensorMap map_routed, const __grid_constant__ CUtensorMap map_shared,
               GemmArgs a) {
    using L = SmemLayout<MODE>;
    constexpr int NMAT = GemmCfg<MODE>::NMAT, S = GemmCfg<MODE>::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t wfull[S], full[S], empty[S], acc_full[2], acc_empty[2];
    __shared__ uint32_t tmem_base_slot;
    __shared__ volatile int abort_flag;
    __shared__ float ep_scale[kBN];             // epilogue: per token column of the current tile
    __shared__ int ep_row[kBN];
    __shared__ int ep_stop;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&full[s], 1 + 128);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 128);
        }
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) tmem_alloc(&tmem_base_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_slot;
    const int num_tiles = __ldcg(a.num_tiles);
    const int KB = a.K / kBlkK;

    if (warp == kWarpProducer) {
        // ---------------------------------------------------------- producer
        int g = 0;
        for (int ti = blockIdx.x; ti < num_tiles && !abort_flag; ti += gridDim.x) {
            const GemmTile t = a.tiles[ti];
            const bool shared = t.expert < 0;
            for (int kb = 0; kb < KB; ++kb, ++g) {
                const int s = g % S;
                const uint32_t r = (uint32_t)(g / S);
                if (!mbar_wait(&empty[s], (r & 1u) ^ 1u, &abort_flag, a.err, 1)) break;
                if (lane == 0) {
                    uint8_t* A = smem + L::A + s * NMAT * kATile;
                    uint8_t* B = smem + L::B + s * kBTile;
                    uint8_t* stg = smem + L::STG + s * NMAT * kStgMat;
                    const uint32_t b_bytes = kBTile;   // a whole box; rows past the end read as zero
                    if (shared) {
                        mbar_arrive(&wfull[s]);                       // nothing to dequantize
                        mbar_arrive_expect_tx(&full[s], b_bytes + NMAT * kATile);
                        for (int m = 0; m < NMAT; ++m) {
                            const uint8_t* img = (m == 0 ? a.sh0 : a.sh1) + ((size_t)t.rb * KB + kb) * kATile;
                            bulk_g2s(A + m * kATile, img, kATile, &full[s]);
                        }
                    } else {
                        int cb, sbb, zb;
                        stage_bytes(a.quant, cb, sbb, zb);
                        mbar_arrive_expect_tx(&wfull[s], (uint32_t)(NMAT * (cb + sbb + zb)));
                        for (int m = 0; m < NMAT; ++m) {
                            const MatView& v = m == 0 ? a.w0 : a.w1;
                            const size_t eo = (size_t)t.expert * v.stride;
                            const size_t blk = ((size_t)t.rb * KB + kb) * (size_t)cb;
                            uint8_t* d = stg + m * kStgMat;
                            bulk_g2s(d, v.codes + eo + blk, cb, &wfull[s]);
                            if (a.quant == Q_NVFP4) {
                                bulk_g2s(d + cb, v.scales + eo + ((size_t)t.rb * KB + kb) * 512, sbb, &wfull[s]);
                            } else {
                                const int G = a.K / kGroup;
                                const size_t go = ((size_t)t.rb * G + kb / 2) * 256;
                                bulk_g2s(d + cb, v.scales + eo + go, sbb, &wfull[s]);
                                if (zb) bulk_g2s(d + cb + sbb, v.zeros + eo + go / 2, zb, &wfull[s]);
                            }
                        }
                        mbar_arrive_expect_tx(&full[s], b_bytes);
                    }
                    // token rows t.seg .. t.seg + 127 of the permuted operand
                    // (shared tiles: of x / the shared intermediate)
                    tma_load_2d(B, shared ? &map_shared : &map_routed, kb * kBlkK, t.seg, &full[s]);
                }
                __syncwarp();
            }
        }
    } else if (warp == kWarpMma) {
        // --------------------------------------------------------- MMA issue
        int g = 0, local = 0;
        for (int ti = blockIdx.x; ti < num_tiles && !abort_flag; ti += gridDim.x, ++local) {
            const GemmTile t = a.tiles[ti];
            const int n_mma = (t.count + 15) & ~15;
            const bool f16 = MODE == 0 && a.tok_scale != nullptr && t.expert >= 0;
            const uint32_t idesc = f16 ? idesc_f16_f32(128, n_mma) : idesc_bf16_f32(128, n_mma);
            const int ab = local & 1;
            if (!mbar_wait(&acc_empty[ab], ((uint32_t)(local >> 1) & 1u) ^ 1u, &abort_flag, a.err, 2)) break;
            tc_fence_after();
            bool ok = true;
            for (int kb = 0; kb < KB; ++kb, ++g) {
                const int s = g % S;
                const uint32_t r = (uint32_t)(g / S);
                if (!mbar_wait(&full[s], r & 1u, &abort_flag, a.err, 3)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t A = smem_u32(smem + L::A + s * NMAT * kATile);
                    const uint32_t B = smem_u32(smem + L::B + s * kBTile);
                    const uint64_t bdesc = desc_kmajor_sw128(B);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                        for (int m = 0; m < NMAT; ++m) {
                            const uint64_t adesc = desc_kmajor_sw128(A + m * kATile);
                            mma_bf16(tmem + ab * 256 + m * 128, adesc + 2 * kk, bdesc + 2 * kk, idesc,
                                     (kb | kk) != 0);
                        }
                    }
                    mma_commit(&empty[s]);
                    if (kb == KB - 1) mma_commit(&acc_full[ab]);
                }
                __syncwarp();
            }
            if (!ok) break;
        }
    } else if (warp >= kWarpDeq0 && warp < kWarpDeq0 + 4) {
        // ------------------------------------------------------------ dequant
        const int r = threadIdx.x - kWarpDeq0 * 32;          // weight row 0..127
        int g = 0;
        for (int ti = blockIdx.x; ti < num_tiles && !abort_flag; ti += gridDim.x) {
            const GemmTile t = a.tiles[ti];
            bool ok = true;
            for (int kb = 0; kb < KB; ++kb, ++g) {
                const int s = g % S;
                const uint32_t rr = (uint32_t)(g / S);
                if (!mbar_wait(&wfull[s], rr & 1u, &abort_flag, a.err, 4)) { ok = false; break; }
                if (t.expert >= 0) {
                    uint8_t* A = smem + L::A + s * NMAT * kATile;
                    const uint8_t* stg = smem + L::STG + s * NMAT * kStgMat;
                    const bool f16 = MODE == 0 && a.tok_scale != nullptr;
#pragma unroll
                    for (int m = 0; m < NMAT; ++m) {
                        if (f16) dequant_row_f16(a.quant, stg + m * kStgMat, A + m * kATile, r);
                        else dequant_row(a.quant, stg + m * kStgMat, A + m * kATile, r);
                    }
                    fence_proxy_async_smem();
                }
                mbar_arrive(&full[s]);
            }
            if (!ok) break;
        }
    } else if (warp >= kWarpEpi0) {
        // ----------------------------------------------------------- epilogue
        const int lane_base = (warp & 3) * 32;
        const int row = lane_base + lane;                    // weight row within the block
        const int ej = threadIdx.x - kWarpEpi0 * 32;         // 0..127: token column this thread looks up
        // The four warps leave the loop together (named barriers): the stop
        // decision is taken by one thread between two barriers.
        int local = 0;
        for (int ti = blockIdx.x; ti < num_tiles; ti += gridDim.x, ++local) {
            const GemmTile t = a.tiles[ti];
            const bool shared = t.expert < 0;
            const int ab = local & 1;
            float gsc = 1.0f;
            if (!shared && a.g_w) gsc = a.g_w[t.expert] * a.g_act;
            // token columns of the tile: scale (mode 0) or routing weight
            // (mode 1) and output row, looked up once per tile
            epi_sync();                                      // the previous tile's readers are done
            if (ej == 0) ep_stop = abort_flag;
            if (ej < t.count) {
                if (shared) {
                    ep_scale[ej] = gsc;
                    ep_row[ej] = t.seg + ej;
                } else {
                    const int slot = __ldg(a.perm + t.seg + ej);
                    if (MODE == 0) {
                        ep_scale[ej] = a.tok_scale ? __ldg(a.tok_scale + slot / a.k_top) : gsc;
                        ep_row[ej] = t.seg + ej;
                    } else {
                        ep_scale[ej] = gsc * __ldg(a.topk_w + slot);
                        ep_row[ej] = slot;
                    }
                }
            }
            epi_sync();
            if (ep_stop) break;
            // a failed wait sets abort_flag: this tile is skipped and all four
            // warps stop at the next tile's decision
            if (!mbar_wait(&acc_full[ab], (uint32_t)(local >> 1) & 1u, &abort_flag, a.err, 5)) continue;
            tc_fence_after();
            const int n_mma = (t.count + 15) & ~15;
            const int col_out = t.rb * kBlkN + row;
            for (int c0 = 0; c0 < n_mma; c0 += 16) {
                const uint32_t taddr = tmem + ((uint32_t)lane_base << 16) + ab * 256 + c0;
                float v0[16];
                tmem_ld16(taddr, v0);
                if (MODE == 0) {
                    float v1[16];
                    tmem_ld16(taddr + 128, v1);
                    __nv_bfloat16* dst = shared ? a.out_sh : a.out;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int col = c0 + i;
                        const float tsc = col < t.count ? ep_scale[col] : 0.0f;
                        const float gg = v0[i] * tsc, uu = v1[i] * tsc;
                        float act = gg / (1.0f + expf(-gg)) * uu;
                        if (!shared && a.quant == Q_NVFP4) {
                            // W4A4: requantize the intermediate per 16 consecutive rows
                            float amax = fabsf(act);
#pragma unroll
                            for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                            const float g = a.g_req;
                            float sbv = 0.0f, rcp = 0.0f;
                            if (g != 0.0f) {
                                sbv = e4m3_to_f32(f32_to_e4m3(__fdiv_rn(amax, __fmul_rn(6.0f, g))));
                                rcp = (sbv == 0.0f) ? 0.0f : __fdiv_rn(1.0f, __fmul_rn(sbv, g));
                            }
                            act = e2m1_to_f32(f32x2_to_e2m1(__fmul_rn(act, rcp), 0.0f) & 0xFu) * sbv;
                        }
                        if (col < t.count) dst[(size_t)ep_row[col] * a.out_ld + col_out] = __float2bfloat16_rn(act);
                    }
                } else {
                    // per-slot outputs are fp16 (saturating at +-65504): their
                    // rounding error stays well below the final bf16 one
                    __half* dst = shared ? a.o16_sh : a.o16;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int col = c0 + i;
                        if (col < t.count)
                            dst[(size_t)ep_row[col] * a.out_ld + col_out] = f16_sat(v0[i] * ep_scale[col]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[ab]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) tmem_dealloc(tmem, kTmemCols);
}

// --------------------------------------------------------------- tile list
// One CTA of 1024 threads: thread e emits the tiles of expert e, grouped by
// (expert, row block) so that the token tiles of one weight block are
// consecutive; the shared expert's tiles (all T tokens) come last.
__global__ void __launch_bounds__(1024) k_build_tiles(const int32_t* __restrict__ counts,
                                                      const int32_t* __restrict__ offsets, int E, int T, int RB,
                                                      int has_shared, GemmTile* __restrict__ tiles,
                                                      int* __restrict__ num_tiles) {
    __shared__ int sc[1024];
    const int e = threadIdx.x;
    const int cnt = (e < E) ? counts[e] : 0;
    const int nt = (cnt + kBN - 1) / kBN;
    const int mine = nt * RB;
    sc[e] = mine;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        const int v = (e >= o) ? sc[e - o] : 0;
        __syncthreads();
        sc[e] += v;
        __syncthreads();
    }
    const int base = sc[e] - mine;
    const int total = sc[1023];
    if (e < E) {
        for (int rb = 0; rb < RB; ++rb)
            for (int tt = 0; tt < nt; ++tt) {
                GemmTile g;
                g.expert = e;
                g.rb = rb;
                g.seg = offsets[e] + tt * kBN;
                g.count = min(kBN, cnt - tt * kBN);
                tiles[base + rb * nt + tt] = g;
            }
    }
    const int nts = has_shared ? (T + kBN - 1) / kBN : 0;
    for (int i = e; i < nts * RB; i += 1024) {
        const int rb = i / nts, tt = i % nts;
        GemmTile g;
        g.expert = -1;
        g.rb = rb;
        g.seg = tt * kBN;
        g.count = min(kBN, T - tt * kBN);
        tiles[total + i] = g;
    }
    if (e == 0) *num_tiles = total + nts * RB;
}

// --------------------------------------------------------------- combine
// y[t] = sum_{j<k} O[t*k + j] + S[t], fp32 sum in fixed j order, one bf16 rounding.
MOE_DEV float h_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu))); }
MOE_DEV float h_hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }

__global__ void k_combine(const __half* __restrict__ O, const __half* __restrict__ S, int T, int H, int k,
                          __nv_bfloat16* __restrict__ y) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // one thread per 8 columns
    const int per_row = H / 8;
    if (i >= (long long)T * per_row) return;
    const int t = (int)(i / per_row), c = (int)(i % per_row) * 8;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j = 0; j < k; ++j) {
        const uint4 q = *reinterpret_cast<const uint4*>(O + ((size_t)t * k + j) * H + c);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) { acc[2 * p] += h_lo(w[p]); acc[2 * p + 1] += h_hi(w[p]); }
    }
    if (S) {
        const uint4 q = *reinterpret_cast<const uint4*>(S + (size_t)t * H + c);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) { acc[2 * p] += h_lo(w[p]); acc[2 * p + 1] += h_hi(w[p]); }
    }
    uint4 out;
    out.x = pack_bf16x2(acc[0], acc[1]);
    out.y = pack_bf16x2(acc[2], acc[3]);
    out.z = pack_bf16x2(acc[4], acc[5]);
    out.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(y + (size_t)t * H + c) = out;
}

// INT4 / INT2 gate/up operand: each token row of x scaled by a power of two
// 2^-p (exact) so that its largest magnitude lies in [2^14, 2^15), stored as
// fp16 (exact: bf16 has 8 significant bits); scale[t] = 2^p undoes it in the
// GEMM epilogue.  One warp per token row.
__global__ void k_x_to_f16(const __nv_bfloat16* __restrict__ x, int T, int H, __half* __restrict__ x16,
                           float* __restrict__ scale) {
    const int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    float amax = 0.0f;
    for (int c = lane; c < H / 8; c += 32) {
        const uint4 q = src[c];
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
    }
    amax = warp_max(amax);
    int e = 0;
    if (amax > 0.0f) frexpf(amax, &e);         // amax in [2^(e-1), 2^e)
    const int p = (amax > 0.0f) ? e - 15 : 0;  // amax * 2^-p in [2^14, 2^15)
    const float down = ldexpf(1.0f, -p);
    for (int c = lane; c < H / 8; c += 32) {
        const uint4 q = src[c];
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            o[i] = h2_bits(__floats2half2_rn(bf16_lo(w[i]) * down, bf16_hi(w[i]) * down));
        reinterpret_cast<uint4*>(x16 + (size_t)t * H)[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (lane == 0) scale[t] = ldexpf(1.0f, p);
}

// Rows of the gate/up token operand in permuted order: xp[p] = xq[perm[p] / k]
// (16-byte copies; one thread per 8 columns).
__global__ void k_gather_rows(const __nv_bfloat16* __restrict__ xq, const int32_t* __restrict__ perm, int slots,
                              int H, int k, __nv_bfloat16* __restrict__ xp) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int per_row = H / 8;
    if (i >= (long long)slots * per_row) return;
    const int p = (int)(i / per_row), c = (int)(i % per_row);
    const int t = __ldg(perm + p) / k;
    reinterpret_cast<uint4*>(xp + (size_t)p * H)[c] = __ldg(reinterpret_cast<const uint4*>(xq + (size_t)t * H) + c);
}

// NVFP4 activations: x -> bf16 values q * s_b (the global scale is applied in
// the GEMM epilogue); one thread per 16-element block.
__global__ void k_act_fp4_values(const __nv_bfloat16* __restrict__ x, int T, int H, float g,
                                 __nv_bfloat16* __restrict__ xq) {
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int nblk = H / kFp4Blk;
    if (t >= (long long)T * nblk) return;
    const __nv_bfloat16* src = x + (size_t)t * kFp4Blk;
    float v[16];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) { v[i] = __bfloat162float(src[i]); amax = fmaxf(amax, fabsf(v[i])); }
    float sbv = 0.0f, r = 0.0f;
    if (g != 0.0f) {
        sbv = e4m3_to_f32(f32_to_e4m3(__fdiv_rn(amax, __fmul_rn(6.0f, g))));
        r = (sbv == 0.0f) ? 0.0f : __fdiv_rn(1.0f, __fmul_rn(sbv, g));
    }
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        const uint32_t c = f32x2_to_e2m1(__fmul_rn(v[i], r), __fmul_rn(v[i + 1], r));
        o[i / 2] = pack_bf16x2(e2m1_to_f32(c & 0xFu) * sbv, e2m1_to_f32(c >> 4) * sbv);
    }
    uint4* d = reinterpret_cast<uint4*>(xq + (size_t)t * kFp4Blk);
    d[0] = make_uint4(o[0], o[1], o[2], o[3]);
    d[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

// ----------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2D 16-bit map over [rows, cols] (cols contiguous), box 64 x box_rows, 128-byte swizzle
static bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                     CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t prefill_tile_capacity(int max_tokens, int k, int E, int H, int I) {
    const int RB = (H > I ? H : I) / kBlkN;
    return (size_t)((max_tokens * (size_t)k + kBN - 1) / kBN + E + (max_tokens + kBN - 1) / kBN + 1) * RB;
}

static int num_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

cudaError_t launch_prefill(const PrefillArgs& p, cudaStream_t st) {
    const ExpertArgs& ex = p.ex;
    const int T = p.T, k = ex.k, H = ex.H, I = ex.I, E = ex.E;
    const int slots = T * k;
    cudaError_t err = launch_permute(p.ids, T, k, E, p.counts, p.offsets, p.perm, p.inv, p.perm_scratch, st);
    if (err != cudaSuccess) return err;
    const bool fp4 = ex.quant == Q_NVFP4;
    const __nv_bfloat16* xin = nullptr;
    CUtensorMapDataType xdt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (fp4) {
        const long long nblk = (long long)T * (H / kFp4Blk);
        k_act_fp4_values<<<(unsigned)((nblk + 255) / 256), 256, 0, st>>>((const __nv_bfloat16*)p.x, T, H, ex.g_x,
                                                                         p.xq);
        xin = p.xq;
    } else {
        k_x_to_f16<<<(T + 7) / 8, 256, 0, st>>>((const __nv_bfloat16*)p.x, T, H, reinterpret_cast<__half*>(p.xq),
                                                 p.tok_scale);
        xin = p.xq;
        xdt = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    }
    {
        const long long n8 = (long long)slots * (H / 8);
        k_gather_rows<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(xin, p.perm, slots, H, k, p.xp);
    }
    const bool has_sh = ex.sh_gate != nullptr;
    CUtensorMap m_routed, m_shared;
    // ---- gate / up
    if (!make_map(&m_routed, p.xp, (uint64_t)slots, (uint64_t)H, kBN, xdt) ||
        !make_map(&m_shared, p.x, (uint64_t)T, (uint64_t)H, kBN))
        return cudaErrorInvalidValue;
    k_build_tiles<<<1, 1024, 0, st>>>(p.counts, p.offsets, E, T, I / kBlkN, has_sh ? 1 : 0, p.tiles, p.num_tiles);
    GemmArgs g{};
    g.quant = ex.quant;
    g.w0 = ex.gate;
    g.w1 = ex.up;
    g.sh0 = ex.sh_gate;
    g.sh1 = ex.sh_up;
    g.perm = p.perm;
    g.tiles = p.tiles;
    g.num_tiles = p.num_tiles;
    g.K = H;
    g.k_top = k;
    g.out_ld = I;
    g.out = p.a_perm;
    g.out_sh = p.a_sh;
    g.g_w = fp4 ? ex.g_gate : nullptr;
    g.g_act = fp4 ? ex.g_x : 1.0f;
    g.g_req = ex.g_a;
    g.tok_scale = fp4 ? nullptr : p.tok_scale;
    g.err = p.err;
    const int grid = num_sms();
    err = cudaFuncSetAttribute(k_grouped_gemm<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, SmemLayout<0>::ALLOC);
    if (err != cudaSuccess) return err;
    if (p.ev_gu0) cudaEventRecord(p.ev_gu0, st);
    k_grouped_gemm<0><<<grid, kGemmThreads, SmemLayout<0>::ALLOC, st>>>(m_routed, m_shared, g);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (p.ev_gu1) cudaEventRecord(p.ev_gu1, st);
    // ---- down
    if (!make_map(&m_routed, p.a_perm, (uint64_t)slots, (uint64_t)I, kBN) ||
        !make_map(&m_shared, p.a_sh, (uint64_t)T, (uint64_t)I, kBN))
        return cudaErrorInvalidValue;
    k_build_tiles<<<1, 1024, 0, st>>>(p.counts, p.offsets, E, T, H / kBlkN, has_sh ? 1 : 0, p.tiles, p.num_tiles);
    g.w0 = ex.down;
    g.w1 = ex.down;
    g.sh0 = ex.sh_down;
    g.sh1 = nullptr;
    g.K = I;
    g.out_ld = H;
    g.out = nullptr;
    g.out_sh = nullptr;
    g.o16 = p.o;
    g.o16_sh = p.o_sh;
    g.topk_w = p.w;
    g.g_w = fp4 ? ex.g_down : nullptr;
    g.g_act = fp4 ? ex.g_a : 1.0f;
    g.tok_scale = nullptr;
    err = cudaFuncSetAttribute(k_grouped_gemm<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, SmemLayout<1>::ALLOC);
    if (err != cudaSuccess) return err;
    if (p.ev_dn0) cudaEventRecord(p.ev_dn0, st);
    k_grouped_gemm<1><<<grid, kGemmThreads, SmemLayout<1>::ALLOC, st>>>(m_routed, m_shared, g);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (p.ev_dn1) cudaEventRecord(p.ev_dn1, st);
    // ---- combine
    const long long threads = (long long)T * (H / 8);
    k_combine<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(p.o, has_sh ? p.o_sh : nullptr, T, H, k,
                                                               (__nv_bfloat16*)p.y);
    return cudaGetLastError();
}

}  // namespace moe
