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
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tiles.cuh"

namespace moe {

using namespace sm100;

constexpr int kBN = kTileTokens;    // tokens per tile (MMA N <= 128)
constexpr int kEpiWarps = 8;        // two warps per TMEM lane quarter, 64 token columns each
constexpr int kWarpProducer = 0, kWarpMma = 1;   // gate/up: warps 1 and 2 issue the MMAs
constexpr uint32_t kTmemCols = 512;

constexpr int kATile = kBlkN * 128;          // 16 KB: 128 rows x 64 16-bit

// MODE 0: gate + up (two matrices, SwiGLU epilogue); MODE 1: down; MODE 2:
// the router logits x . Wr^T (fp32 out, A = Wr rows by TMA, no tile list).
// SH = false: routed tiles, packed weights dequantized into TMEM (the MMA
// reads A from TMEM); SH = true: shared-expert tiles, bf16 weight images in
// shared memory (the MMA reads A from shared memory).
template <int MODE, bool SH>
struct Cfg {
    static constexpr int NMAT = MODE == 0 ? 2 : 1;
    // k-blocks (64 columns) per pipeline stage: routed stages cover 128
    // columns, which halves the barrier round trips and commits per MMA
    static constexpr int KSTEP = SH ? 1 : 2;
    // tokens per tile: the router launch takes 256 (each Wr byte it streams
    // serves twice the tokens: 31 -> 21 us at T = 8192); the shared-expert
    // launches measured slower with 256 (one accumulator, two stages) and
    // keep 128, as the routed ones
    static constexpr int TN = MODE == 2 ? 2 * kBN : kBN;
    static constexpr int B_TILE = TN * 128;           // one k-block of the token operand
    // S: stages of the token operand ring, which for routed tiles are also
    // the TMEM slots of the dequantized weights (a slot and its token tile
    // are released by the same MMA commit)
    static constexpr int S = SH ? (MODE == 0 ? 3 : 4) : (MODE == 0 ? 2 : 4);
    // SC: stages of the packed-weight ring (routed), decoupled from the TMEM
    // slots so that the HBM reads of the codes run several stages ahead
    static constexpr int SC = SH ? 0 : 6;
    // MMA-issuing warps: one per matrix (each stage gets NMAT commits).  A
    // second issuer taking alternate down tiles was measured slower: the
    // down GEMM shares shared-memory bandwidth and issue slots between the
    // MMA operand reads, the staged codes and the epilogue staging.
    static constexpr int MMA_WARPS = NMAT;
    // routed: a second producer warp loads the token operand, the first the
    // packed weights
    static constexpr int BPROD = kWarpMma + MMA_WARPS;
    static constexpr int DEQ0 = BPROD + (SH ? 0 : 1);                  // first dequant warp
    // dequant warps: one per (TMEM lane quarter, matrix, k-block of the
    // stage), one thread per weight row; all of them convert every stage
    static constexpr int DEQ_WARPS = SH ? 0 : 4 * NMAT * KSTEP;
    static constexpr int EPI0 = DEQ0 + DEQ_WARPS;                    // first epilogue warp
    static constexpr int THREADS = (EPI0 + kEpiWarps) * 32;
    // accumulators: NMAT x TN columns per buffer; routed gate/up keeps one
    // buffer so that its A slots fit in the 512 columns
    static constexpr int ACC_BUFS = (SH || MODE == 1) ? 2 : 1;
    static constexpr bool ACC_SPLIT = MODE == 0 && !SH;   // routed gate/up: halves for small tiles
    static constexpr int ACC_COLS = NMAT * TN;
    static constexpr int A_COL0 = ACC_BUFS * ACC_COLS;   // TMEM column of A slot 0 (routed)
    static constexpr int A_STAGE_COLS = NMAT * KSTEP * 32;
    static_assert(SH || A_COL0 + S * A_STAGE_COLS <= (int)kTmemCols, "TMEM budget");
    // staged packed bytes of one matrix and stage: KSTEP blocks of codes,
    // then the scales (INT4/INT2: the one 128-column group; NVFP4: KSTEP x
    // 512), then the INT2 zero points
    static constexpr int STG_MAT = KSTEP * 4096 + KSTEP * 512;
    // shared memory
    static constexpr int A = 0;                                           // SH: [S][NMAT][16 KB]
    static constexpr int B = A + (SH ? S * NMAT * kATile : 0);            // [S][KSTEP][B_TILE]
    static constexpr int STG = B + S * KSTEP * B_TILE;                    // routed: [SC][NMAT][STG_MAT]
    static constexpr int OUT = STG + SC * NMAT * STG_MAT;                 // [OUT_BUFS][TN][128] 16-bit
    static constexpr int OUT_TILE = TN * kBlkN * 2;
    // down writes its staged rows with TMA stores: the shared-expert launch
    // has room for two staging buffers (a tile's stores overlap the next
    // tile's staging), the routed one for one
    static constexpr int OUT_BUFS = (MODE == 1 && SH) ? 2 : 1;
    static constexpr int BYTES = OUT + (MODE == 2 ? 0 : OUT_BUFS * OUT_TILE);
    static constexpr int ALLOC = BYTES + 1024;                            // slack for 1024-byte alignment
    static_assert(ALLOC <= 227 * 1024 - 8192, "shared memory budget (static arrays take up to 8 KB)");
};

// Token-operand tensor maps with boxes of 128, 64, 32 and 16 rows: a tile
// of n (a multiple of 16) tokens loads only its n rows, as at most three
// boxes at 16-row (2 KB, swizzle-atom aligned) offsets.
struct BMaps {
    CUtensorMap m[4];
};
MOE_DEV uint32_t load_token_rows(uint8_t* dst, const BMaps& mb, int x, int y, int n, uint64_t* bar) {
    int off = 0;
    for (; n - off >= 128; off += 128) tma_load_2d(dst + off * 128, &mb.m[0], x, y + off, bar);
    const int n16 = (n - off) >> 4;
#pragma unroll
    for (int b = 2; b >= 0; --b)
        if (n16 & (1 << b)) {
            tma_load_2d(dst + off * 128, &mb.m[3 - b], x, y + off, bar);
            off += 16 << b;
        }
    return (uint32_t)off * 128u;
}

// Store maps of a 16-bit output [rows][H] (the per-slot outputs by permuted
// position, the shared expert's output by token) with boxes of 128 / 2^i
// rows x 128 columns: a tile's n consecutive rows leave as at most eight TMA
// stores.
struct OMaps {
    CUtensorMap m[8];
};
// TMA stores of a tile's n staged rows ([n][128] 16-bit, row-major) to rows
// y .. y+n-1, columns x .. x+127, as one bulk group (issued by one thread).
MOE_DEV void store_tile_rows(const OMaps& mo, int x, int y, int n, const uint8_t* src) {
    int off = 0;
    for (; n - off >= 128; off += 128) tma_store_2d(&mo.m[0], x, y + off, src + off * (kBlkN * 2));
    const int rem = n - off;                     // < 128: one box per set bit
#pragma unroll
    for (int b = 6; b >= 0; --b)
        if ((rem >> b) & 1) {
            tma_store_2d(&mo.m[7 - b], x, y + off, src + off * (kBlkN * 2));
            off += 1 << b;
        }
    bulk_commit();
}

struct GemmArgs {
    int quant;                // routed weight format
    MatView w0, w1;           // gate/up (mode 0) or down (w0, mode 1)
    const uint8_t* sh0;       // shared expert bf16 images (gate/up or down)
    const uint8_t* sh1;
    const int32_t* perm;      // slot at each permuted position
    const GemmTile* tiles;
    const int* num_tiles;     // [0]: routed tiles, [1]: all tiles (shared ones last), [2]: routed
                              // groups, [3]: 1 when routed launches take the group order
    const int2* groups;       // routed groups: first tile, tiles
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
    float* logits;            // mode 2: [n_tok, n_rows] fp32
    int n_tok, n_rows;        // mode 2: tokens, router rows (experts)
    int n_tiles;              // mode 2: (row blocks) x (token blocks)
    const float* w_perm;      // routing weight of each permuted position (down)
    const float* ts_perm;     // INT4/INT2 gate/up: token scale of each permuted position
    uint8_t* out4;            // NVFP4 gate/up: e2m1 intermediate [slots, I/2] (permuted rows)
    uint8_t* out_sf;          // NVFP4 gate/up: its e4m3 block scales, stage-major [I/256][slots][16]
    // NVFP4 block-scaled GEMMs: the weight image (per expert, 128-row block
    // and 256-value stage one block of NMAT swizzled 16 KB code tiles and
    // NMAT 2 KB scale tiles), and the e4m3 scales of the token operand,
    // stage-major [K/256][rows][16 B] with sfb_rows = slots rows per stage
    const uint8_t* wimg;
    const uint8_t* sfb;
    long long sfb_rows;
    long long sfb_rows_out;   // NVFP4 gate/up: rows per stage of out_sf (the slots)
    int* err;
};

// ------------------------------------------------------------------ dequant
MOE_DEV uint32_t bf16x2_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t*>(&v); }

MOE_DEV uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }
MOE_DEV __half f16_sat(float v) { return __float2half_rn(fminf(fmaxf(v, -65504.0f), 65504.0f)); }

// Dequantization of one half (32 columns, h = 0 / 1) of row r of a 128x64
// block: codes of the block (device layout of layout.cuh), the block's
// scales (INT4/INT2: fp16 per row of its 128-column group; NVFP4: four e4m3
// per row) and INT2 zero points.  v[i] holds columns 32h + 2i and
// 32h + 2i + 1 (low, high), the A-operand layout of one TMEM lane.
//
// INT4 / INT2 -> fp16 (u - 8) * s or (u - z) * s: the integer is exact in
// fp16 and so is the fp16 scale, so each weight is rounded once (2^-12).
MOE_DEV void dequant_half_f16(int quant, const uint8_t* codes, const uint8_t* scales, const uint8_t* zeros, int r,
                              int h, uint32_t (&v)[16]) {
    const __half2 s2 = __half2half2(reinterpret_cast<const __half*>(scales)[r]);
    if (is_int4(quant)) {
        // even nibbles j = 0, 2 at bits 0..3 give 1024 + u; odd ones j = 1, 3
        // are masked in place at bits 4..7, giving 1024 + 16u, and take
        // (1024 + 16u - 1152) * (s / 16): exact steps before the one rounding
        // of (u - 8) * s, as for the even nibbles, while s / 16 is a normal
        // fp16 (s >= 2^-10; below that s / 16 keeps one bit less)
        const __half2 off = __float2half2_rn(1032.0f);
        const __half2 off16 = __float2half2_rn(1152.0f);
        const __half2 s16 = __hmul2(s2, __float2half2_rn(0.0625f));                    // exact
        const uint4 q = *reinterpret_cast<const uint4*>(codes + (h * kBlkN + r) * 16);   // chunk h
        const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const uint32_t x = jj ? wv[w] >> 8 : wv[w];
                const uint32_t te = (x & 0x000F000Fu) | 0x64006400u;                      // 1024 + u
                const uint32_t to = (x & 0x00F000F0u) | 0x64006400u;                      // 1024 + 16u
                v[4 * w + 2 * jj] = h2_bits(__hmul2(__hsub2(*reinterpret_cast<const __half2*>(&te), off), s2));
                v[4 * w + 2 * jj + 1] =
                    h2_bits(__hmul2(__hsub2(*reinterpret_cast<const __half2*>(&to), off16), s16));
            }
        }
    } else {
        const __half2 off = __float2half2_rn(1024.0f + (float)zeros[r]);
        const uint2 q = *reinterpret_cast<const uint2*>(codes + r * 16 + h * 8);          // words 2h, 2h+1
        const uint32_t wv[2] = {q.x, q.y};
#pragma unroll
        for (int w = 0; w < 2; ++w)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t t = ((wv[w] >> (2 * j)) & 0x00030003u) | 0x64006400u;   // 1024 + u
                v[8 * w + j] = h2_bits(__hmul2(__hsub2(*reinterpret_cast<const __half2*>(&t), off), s2));
            }
    }
}

// bf16 variant (down projection, NVFP4): (u - 8) * s and (u - z) * s in
// bf16; e2m1 * e4m3 block scale is exact in bf16 (the global scales are
// applied in the epilogue).
MOE_DEV void dequant_half(int quant, const uint8_t* codes, const uint8_t* scales, const uint8_t* zeros, int r, int h,
                          uint32_t (&v)[16]) {
    if (is_int4(quant)) {
        const __half s16 = reinterpret_cast<const __half*>(scales)[r];
        const __nv_bfloat162 s2 = __bfloat162bfloat162(__float2bfloat16_rn(__half2float(s16)));
        const __nv_bfloat162 off = __bfloat162bfloat162(__float2bfloat16_rn(136.0f));
        const uint4 q = *reinterpret_cast<const uint4*>(codes + (h * kBlkN + r) * 16);
        const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t t = ((wv[w] >> (4 * j)) & 0x000F000Fu) | 0x43004300u;   // 128 + u
                const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&t);
                v[4 * w + j] = bf16x2_bits(__hmul2(__hsub2(b, off), s2));             // (u - 8) * s
            }
    } else if (quant == Q_INT2) {
        const __half s16 = reinterpret_cast<const __half*>(scales)[r];
        const __nv_bfloat162 s2 = __bfloat162bfloat162(__float2bfloat16_rn(__half2float(s16)));
        const __nv_bfloat162 off = __bfloat162bfloat162(__float2bfloat16_rn(128.0f + (float)zeros[r]));
        const uint2 q = *reinterpret_cast<const uint2*>(codes + r * 16 + h * 8);
        const uint32_t wv[2] = {q.x, q.y};
#pragma unroll
        for (int w = 0; w < 2; ++w)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t t = ((wv[w] >> (2 * j)) & 0x00030003u) | 0x43004300u;   // 128 + u
                const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&t);
                v[8 * w + j] = bf16x2_bits(__hmul2(__hsub2(b, off), s2));             // (u - z) * s
            }
    } else {  // NVFP4: two 16-column blocks per half, one e4m3 scale each
        const uint32_t sb4 = reinterpret_cast<const uint32_t*>(scales)[r];
        const uint4 q = *reinterpret_cast<const uint4*>(codes + (h * kBlkN + r) * 16);
        const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
        const uint32_t sb2[2] = {bf16x2_splat(e4m3_to_f32((sb4 >> (16 * h)) & 0xffu)),
                                 bf16x2_splat(e4m3_to_f32((sb4 >> (16 * h + 8)) & 0xffu))};
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int j = 0; j < 4; ++j) v[4 * w + j] = fp4_pair(wv[w], j, sb2[w >> 1]);
    }
}

// bytes of the packed codes of one 128x64 block
__host__ __device__ constexpr int block_code_bytes(int quant) {
    return quant == Q_INT2 ? 2048 : (quant == Q_FP8 ? 8192 : (quant == Q_FP6 ? 6144 : 4096));
}

// FP6 (e2m3, fp16 scale per 32 inputs): chunk h of row r from the two
// planes of the block; e2m3 values are exact in fp16, w = e2m3 * s is
// rounded once to fp16 (f16) or bf16.  v[4w + j] = columns 8w + 2j, +1.
MOE_DEV void dequant_half_fp6(const uint8_t* codes, const uint8_t* scales, int r, int h, bool f16,
                              uint32_t (&v)[16]) {
    const uint4 q = *reinterpret_cast<const uint4*>(codes + (h * kBlkN + r) * 16);
    const uint2 hq = *reinterpret_cast<const uint2*>(codes + 4096 + (h * kBlkN + r) * 8);
    const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
    const uint32_t hv[4] = {hq.x & 0xffffu, hq.x >> 16, hq.y & 0xffffu, hq.y >> 16};
    const __half s16 = reinterpret_cast<const __half*>(scales)[r];
    const __half2 up = __float2half2_rn(16384.0f), s2 = __half2half2(s16);
    const float sf = __half2float(s16);
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t nib = (wv[w] >> (4 * j)) & 0x000F000Fu;
            const uint32_t x = hv[w] >> (2 * j);
            const uint32_t h2 = e2m3x2_to_f16x2_scaled(nib, (x & 0x3u) | ((x & 0x300u) << 8));
            const __half2 e = __hmul2(*reinterpret_cast<const __half2*>(&h2), up);      // exact e2m3 values
            v[4 * w + j] = f16 ? h2_bits(__hmul2(e, s2)) : pack_bf16x2(__low2float(e) * sf, __high2float(e) * sf);
        }
}

// FP8 (E4M3, one fp32 scale per 128x128 block): chunk h (32 columns, two
// 16-column chunks of the block's layout) of row r; the E4M3 values are
// exact in fp16, w = e4m3 * s is rounded once to fp16 (f16) or bf16.
MOE_DEV void dequant_half_fp8(const uint8_t* codes, float s, int r, int h, bool f16, uint32_t (&v)[16]) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const uint4 w4 = *reinterpret_cast<const uint4*>(codes + ((2 * h + q) * kBlkN + r) * 16);
        const uint32_t wd[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const uint32_t h2 = e4m3x2_to_f16x2(wd[p >> 1] >> (16 * (p & 1)));
            const __half2 hv = *reinterpret_cast<const __half2*>(&h2);
            const float lo = __low2float(hv) * s, hi = __high2float(hv) * s;
            v[q * 8 + p] = f16 ? h2_bits(__floats2half2_rn(lo, hi)) : pack_bf16x2(lo, hi);
        }
    }
}

// Bounded mbarrier wait by a whole warp with a warp-uniform result (every
// lane returns from mbar_wait, so every lane reaches the vote): a warp that
// synchronises with __syncwarp never has lanes on both sides of a stop.
MOE_DEV bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err, int code) {
    const bool ok = mbar_wait(bar, parity, abort_flag, err, code);
    return __all_sync(0xffffffffu, ok);
}

// named barrier of the epilogue warps
MOE_DEV void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory"); }
template <int NW>
MOE_DEV void epi_sync_n() { asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory"); }

// SwiGLU of one accumulator pair: silu(g) * u with the fast exponential and
// division (relative error ~1e-6, far below the bf16 / e2m1 rounding of
// the stored intermediate)
MOE_DEV float swiglu_fast(float g, float u) { return __fdividef(g * u, 1.0f + __expf(-g)); }

// Accumulator placement. ACC_BUFS == 2: tile j takes buffer j & 1 (NMAT x
// 128 columns each). Routed gate/up keeps one 256-column buffer: a tile of
// at most 64 tokens takes one 128-column half (gate, then up 64 columns
// further), so that two such tiles alternate and the epilogue of one
// overlaps the MMAs of the next; a larger tile takes both halves (gate at
// 0, up at 128). The MMA warps and the epilogue walk the same sequence.
struct AccSeq {
    uint32_t uses0 = 0, uses1 = 0;
    int next = 0;
};
struct AccUse {
    int mask;               // bit b: buffer (half) b
    uint32_t col;           // first column of the matrix-0 accumulator
    uint32_t mat_stride;    // columns from matrix 0 to matrix 1
    uint32_t par0, par1;    // phase parity of this use of buffer 0 / 1
};
template <int ACC_BUFS, int ACC_COLS, int TN, bool SPLIT>
MOE_DEV AccUse acc_next(AccSeq& q, int n_mma) {
    AccUse u;
    if (ACC_BUFS == 2) {
        u.mask = 1 << q.next;
        u.col = (uint32_t)(q.next * ACC_COLS);
        u.mat_stride = TN;
    } else if (!SPLIT) {
        u.mask = 1;                              // one buffer, gate at 0 and up at TN
        u.col = 0;
        u.mat_stride = TN;
    } else if (n_mma > 64) {
        u.mask = 3;
        u.col = 0;
        u.mat_stride = kBN;
    } else {
        u.mask = 1 << q.next;
        u.col = (uint32_t)(q.next * kBN);
        u.mat_stride = 64;
    }
    u.par0 = q.uses0 & 1u;
    u.par1 = q.uses1 & 1u;
    q.uses0 += (uint32_t)(u.mask & 1);
    q.uses1 += (uint32_t)(u.mask >> 1);
    q.next = (u.mask == 3 || (ACC_BUFS == 1 && !SPLIT)) ? 0 : (q.next ^ 1);
    return u;
}

struct PermMeta {
    const float* topk_w;      // [T*k] routing weight of each slot
    const float* tok_scale;   // [T] fp16 activation scale of each token, or null
    float* w_perm;            // [T*k] out: routing weight of each permuted position
    float* ts_perm;           // [T*k] out: token scale of each permuted position
};

// A CTA's tile sequence is copied into shared memory once, so that no role
// waits on a global load at the start of a tile.  The block-scaled NVFP4
// launches take groups (up to kGroupTiles consecutive token tiles of one expert and weight
// block, which read the same weights) in the order g = blockIdx.x + j *
// gridDim.x, so that a CTA reads a weight block for its second token tile
// while it is still in L2; otherwise (or when a CTA's tiles would not fit
// the list) tiles go round robin, ti = first + j * gridDim.x.
struct TileCache {
    GemmTile t[kTileCache];
    int n;          // tiles of this CTA
    int grouped;    // 1: group order (all n tiles in t), 0: round robin
};
MOE_DEV void cache_tiles(TileCache& tc, const GemmTile* tiles, int first, int end) {
    for (int j = threadIdx.x; j < kTileCache; j += blockDim.x) {
        const int ti = first + j * gridDim.x;
        if (ti < end) tc.t[j] = tiles[ti];
    }
    if (threadIdx.x == 0) {
        tc.n = first < end ? (end - first + gridDim.x - 1) / gridDim.x : 0;
        tc.grouped = 0;
    }
}
// Group order (needs blockDim.x >= kTileCache): thread i takes this CTA's
// i-th group, an exclusive scan of the group sizes places its tiles.
MOE_DEV void cache_groups(TileCache& tc, const GemmTile* tiles, const int2* groups, int ngroups, int* scan) {
    const int i = threadIdx.x;
    int2 gr = make_int2(0, 0);
    if (i < kTileCache) {
        const int g = blockIdx.x + i * gridDim.x;
        if (g < ngroups) gr = groups[g];
    }
    // inclusive scan of gr.y over threads 0 .. kTileCache-1
    const int lane = i & 31, w = i >> 5;
    int v = gr.y;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (i < kTileCache && lane == 31) scan[w] = v;
    __syncthreads();
    if (i < kTileCache) {
        int base = 0;
        for (int k = 0; k < w; ++k) base += scan[k];
        const int pos = base + v - gr.y;
        for (int k = 0; k < gr.y && pos + k < kTileCache; ++k) tc.t[pos + k] = tiles[gr.x + k];
        if (i == kTileCache - 1) {
            tc.n = min(base + v, kTileCache);
            tc.grouped = 1;
        }
    }
}

// Tile ti: from the device-built list, or (router) row block ti % RB of
// token block ti / RB.
template <int MODE>
MOE_DEV GemmTile load_tile(const GemmArgs& a, int ti, const TileCache* tc = nullptr, int first = 0, int j = -1) {
    if constexpr (MODE == 2) {
        constexpr int TN = 2 * kBN;              // the router launch's token tiles
        const int RB = (a.n_rows + kBlkN - 1) / kBlkN;
        GemmTile t;
        t.expert = -1;
        t.rb = ti % RB;
        t.seg = (ti / RB) * TN;
        t.count = min(TN, a.n_tok - t.seg);
        return t;
    } else {
        if (tc && tc->grouped) return tc->t[j];
        const int jj = (ti - first) / (int)gridDim.x;
        return (tc && jj < kTileCache) ? tc->t[jj] : a.tiles[ti];
    }
}

// ------------------------------------------------------------------ kernel
// Q: the routed weights' format (a compile-time constant, so that each
// instantiation holds only its own dequantization and ring geometry); the
// shared-expert and router launches take Q_BF16.
template <int MODE, bool SH, int Q>
__global__ void __launch_bounds__(Cfg<MODE, SH>::THREADS, 1)
k_grouped_gemm(const __grid_constant__ BMaps map_b, const __grid_constant__ CUtensorMap map_a,
               const __grid_constant__ OMaps map_o, GemmArgs a) {
    using C = Cfg<MODE, SH>;
    constexpr int NMAT = C::NMAT, S = C::S, KSTEP = C::KSTEP;
    constexpr int SC = C::SC > 0 ? C::SC : 1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t cfull[SC], cempty[SC], full[S], empty[S], acc_full[2], acc_empty[2];
    __shared__ uint32_t tmem_base_slot;
    __shared__ volatile int abort_flag;
    __shared__ float ep_scale[C::TN];           // epilogue: per token column of the current tile
    __shared__ int ep_row[C::TN];
    __shared__ int ep_stop;
    __shared__ TileCache tcache;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    {
        const int tb = (SH && MODE != 2) ? __ldcg(a.num_tiles) : 0;
        const int te = MODE == 2 ? a.n_tiles : SH ? __ldcg(a.num_tiles + 1) : __ldcg(a.num_tiles);
        // round robin: with the dequantizing pipeline the skewed tile sizes
        // of Zipf routing balance better than in the group order
        if (MODE != 2) cache_tiles(tcache, a.tiles, tb + blockIdx.x, te);
    }
    if (threadIdx.x == 0) {
        for (int c = 0; c < SC; ++c) {
            mbar_init(&cfull[c], 1);                      // codes producer (bytes)
            mbar_init(&cempty[c], C::DEQ_WARPS);          // every dequant warp has read its part
        }
        for (int s = 0; s < S; ++s) {
            // token producer (bytes) [+ one arrival per dequant warp]
            mbar_init(&full[s], 1 + C::DEQ_WARPS);
            mbar_init(&empty[s], NMAT);                   // one commit per matrix
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], NMAT);
            mbar_init(&acc_empty[b], kEpiWarps);          // one arrival per epilogue warp
        }
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) tmem_alloc(&tmem_base_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_slot;
    const int t_begin = (SH && MODE != 2) ? __ldcg(a.num_tiles) : 0;
    const int t_end = MODE == 2 ? a.n_tiles : SH ? __ldcg(a.num_tiles + 1) : __ldcg(a.num_tiles);
    const int t_first = t_begin + blockIdx.x;
    const int NS = a.K / (kBlkK * KSTEP);                 // stages per tile
    // this CTA's tile sequence
    const int nseq = MODE == 2 ? (t_first < t_end ? (t_end - t_first + (int)gridDim.x - 1) / (int)gridDim.x : 0)
                               : tcache.n;
    auto tile_at = [&](int j) { return load_tile<MODE>(a, t_first + j * (int)gridDim.x, &tcache, t_first, j); };

    if (warp == kWarpProducer && !SH) {
        // ------------------------------------------- producer: packed weights
        // the codes of KSTEP consecutive blocks are contiguous, and so are
        // their NVFP4 scales
        const int KB = a.K / kBlkK, G = scale_stride(Q, a.K);
        constexpr bool fp8 = Q == Q_FP8;
        const int cb = block_code_bytes(Q) * KSTEP;
        // scales of a stage: NVFP4 KSTEP x 512 bytes; INT4/INT2 group 128 one
        // group (128 rows x fp16); INT4 group 32 the stage's 2 KSTEP groups;
        // FP8 the one block scale, stored by this thread
        constexpr bool g32 = Q == Q_INT4G32 || Q == Q_FP6;
        constexpr int sb = Q == Q_NVFP4 ? 512 * KSTEP : g32 ? 256 * 2 * KSTEP : fp8 ? 0 : 256;
        constexpr int zb = Q == Q_INT2 ? 128 : 0;
        // FP8 and FP6 stages take more of the ring
        constexpr int stg_mat = fp8 ? KSTEP * 8192 + 16 : Q == Q_FP6 ? KSTEP * 6144 + KSTEP * 512 : C::STG_MAT;
        constexpr int SCr = stg_mat > C::STG_MAT ? (SC * C::STG_MAT) / stg_mat : SC;
        int g = 0;
        for (int jt = 0; jt < nseq && !abort_flag; ++jt) {
            const GemmTile t = tile_at(jt);
            bool ok = true;
            for (int ks = 0; ks < NS; ++ks, ++g) {
                const int c = g % SCr;
                if (!warp_wait(&cempty[c], ((uint32_t)(g / SCr) & 1u) ^ 1u, &abort_flag, a.err, 1)) { ok = false; break; }
                if (lane == 0) {
                    const int kb0 = ks * KSTEP;
                    uint8_t* stg = smem + C::STG + c * NMAT * stg_mat;
                    if (fp8)      // plain stores, released by the arrive below
                        for (int m = 0; m < NMAT; ++m)
                            *reinterpret_cast<float*>(stg + m * stg_mat + cb) =
                                __ldg(reinterpret_cast<const float*>(expert_matrix(m == 0 ? a.w0 : a.w1, t.expert).scales) +
                                      (size_t)t.rb * G + kb0 / 2);
                    mbar_arrive_expect_tx(&cfull[c], (uint32_t)(NMAT * (cb + sb + zb)));
                    for (int m = 0; m < NMAT; ++m) {
                        const ExpertMat em = expert_matrix(m == 0 ? a.w0 : a.w1, t.expert);
                        uint8_t* d = stg + m * stg_mat;
                        bulk_g2s(d, em.codes + ((size_t)t.rb * KB + kb0) * (size_t)block_code_bytes(Q), cb,
                                 &cfull[c]);
                        if constexpr (Q == Q_NVFP4) {
                            bulk_g2s(d + cb, em.scales + ((size_t)t.rb * KB + kb0) * 512, sb, &cfull[c]);
                        } else if (!fp8) {
                            // first group of the stage (kb0 even: one group-128)
                            const size_t go = ((size_t)t.rb * G + (g32 ? 2 * kb0 : kb0 / 2)) * 256;
                            bulk_g2s(d + cb, em.scales + go, sb, &cfull[c]);
                            if (zb) bulk_g2s(d + cb + sb, em.zeros + go / 2, zb, &cfull[c]);
                        }
                    }
                }
                __syncwarp();
            }
            if (!ok) break;
        }
    } else if ((SH && warp == kWarpProducer) || (!SH && warp == C::BPROD)) {
        // ---------------------------------------- producer: token operand
        // (+ the router / shared-expert weight tiles)
        int g = 0;
        for (int jt = 0; jt < nseq && !abort_flag; ++jt) {
            const GemmTile t = tile_at(jt);
            const int n_mma = (t.count + 15) & ~15;
            bool ok = true;
            for (int ks = 0; ks < NS; ++ks, ++g) {
                const int s = g % S;
                const uint32_t r = (uint32_t)(g / S);
                if (!warp_wait(&empty[s], (r & 1u) ^ 1u, &abort_flag, a.err, 1)) { ok = false; break; }
                if (lane == 0) {
                    const int kb0 = ks * KSTEP;
                    uint8_t* B = smem + C::B + s * KSTEP * C::B_TILE;
                    const uint32_t tb = (uint32_t)KSTEP * (uint32_t)n_mma * 128u;
                    if constexpr (MODE == 2) {
                        mbar_arrive_expect_tx(&full[s], tb + kATile);
                        tma_load_2d(smem + C::A + s * kATile, &map_a, kb0 * kBlkK, t.rb * kBlkN, &full[s]);
                    } else if constexpr (SH) {
                        uint8_t* A = smem + C::A + s * NMAT * kATile;
                        mbar_arrive_expect_tx(&full[s], tb + NMAT * kATile);
                        for (int m = 0; m < NMAT; ++m) {
                            const uint8_t* img = (m == 0 ? a.sh0 : a.sh1) + ((size_t)t.rb * (a.K / kBlkK) + kb0) * kATile;
                            bulk_g2s(A + m * kATile, img, kATile, &full[s]);
                        }
                    } else {
                        mbar_arrive_expect_tx(&full[s], tb);
                    }
                    // token rows t.seg .. t.seg + n_mma - 1 (rows past the
                    // end of the operand read as zero)
                    for (int j = 0; j < KSTEP; ++j)
                        load_token_rows(B + j * C::B_TILE, map_b, (kb0 + j) * kBlkK, t.seg, n_mma, &full[s]);
                }
                __syncwarp();
            }
            if (!ok) break;
        }
    } else if (warp >= kWarpMma && warp < kWarpMma + C::MMA_WARPS) {
        // --------------------------------------------------------- MMA issue
        // warp kWarpMma + m issues the MMAs of matrix m (gate/up: two warps)
        const int mi = warp - kWarpMma;
        int g = 0;
        AccSeq aseq;
        for (int jt = 0; jt < nseq && !abort_flag; ++jt) {
            const GemmTile t = tile_at(jt);
            const int n_mma = (t.count + 15) & ~15;
            // INT/FP8/FP6 routed tiles, gate/up and down: fp16 operands
            constexpr bool f16 = MODE != 2 && !SH && Q != Q_NVFP4;
            const uint32_t idesc = f16 ? idesc_f16_f32(128, n_mma) : idesc_bf16_f32(128, n_mma);
            const AccUse au = acc_next<C::ACC_BUFS, C::ACC_COLS, C::TN, C::ACC_SPLIT>(aseq, n_mma);
            if ((au.mask & 1) && !warp_wait(&acc_empty[0], au.par0 ^ 1u, &abort_flag, a.err, 2)) break;
            if ((au.mask & 2) && !warp_wait(&acc_empty[1], au.par1 ^ 1u, &abort_flag, a.err, 2)) break;
            tc_fence_after();
            bool ok = true;
            const uint32_t d = tmem + au.col + mi * au.mat_stride;
            for (int ks = 0; ks < NS; ++ks, ++g) {
                const int s = g % S;
                const uint32_t r = (uint32_t)(g / S);
                if (!warp_wait(&full[s], r & 1u, &abort_flag, a.err, 3)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int j = 0; j < KSTEP; ++j) {
                        const uint64_t bdesc = desc_kmajor_sw128(smem_u32(smem + C::B + (s * KSTEP + j) * C::B_TILE));
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t acc = (ks | j | kk) != 0;
                            if constexpr (SH) {
                                const uint64_t adesc = desc_kmajor_sw128(smem_u32(smem + C::A + (s * NMAT + mi) * kATile));
                                mma_bf16(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, acc);
                            } else {
                                const uint32_t at = tmem + C::A_COL0 + s * C::A_STAGE_COLS + (mi * KSTEP + j) * 32 + kk * 8;
                                mma_f16_tmem_a(d, at, bdesc + 2 * kk, idesc, acc);
                            }
                        }
                    }
                    mma_commit(&empty[s]);
                    if (ks == NS - 1) {
                        if (au.mask & 1) mma_commit(&acc_full[0]);
                        if (au.mask & 2) mma_commit(&acc_full[1]);
                    }
                }
                __syncwarp();
            }
            if (!ok) break;
        }
    } else if (warp >= C::DEQ0 && warp < C::EPI0) {
        // ------------------------------------------------------------ dequant
        // routed tiles only: thread (row r, matrix m, k-block j of the stage)
        // writes TMEM lane r (its warp's lane quarter)
        if constexpr (!SH) {
            const int quarter = warp & 3;
            const int r = quarter * 32 + lane;                 // weight row = TMEM lane
            const int wi = (warp - C::DEQ0) >> 2;
            const int m = wi % NMAT, j = wi / NMAT;
            const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
            constexpr bool f16 = Q != Q_NVFP4;
            constexpr int cb = block_code_bytes(Q);
            constexpr bool fp8 = Q == Q_FP8, fp6 = Q == Q_FP6;
            // as the producer
            constexpr int stg_mat = fp8 ? KSTEP * 8192 + 16 : fp6 ? KSTEP * 6144 + KSTEP * 512 : C::STG_MAT;
            constexpr int SCr = stg_mat > C::STG_MAT ? (SC * C::STG_MAT) / stg_mat : SC;
            int g = 0;
            for (int jt = 0; jt < nseq && !abort_flag; ++jt) {
                bool ok = true;
                for (int ks = 0; ks < NS; ++ks, ++g) {
                    const int c = g % SCr, s = g % S;
                    // the packed codes arrived, and the MMAs that read this
                    // TMEM slot before have completed
                    if (!warp_wait(&cfull[c], (uint32_t)(g / SCr) & 1u, &abort_flag, a.err, 4) ||
                        !warp_wait(&empty[s], ((uint32_t)(g / S) & 1u) ^ 1u, &abort_flag, a.err, 6)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t* stg = smem + C::STG + (c * NMAT + m) * stg_mat;
                    const uint8_t* sc = stg + cb * KSTEP;
                    const uint8_t* zr = sc + 256;
                    uint32_t v[16];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        // chunk h of block j: NVFP4 scales of the block, INT4 group
                        // 32 the chunk's own group, else the stage's one group
                        const uint8_t* scj = Q == Q_NVFP4 ? sc + j * 512
                                           : (Q == Q_INT4G32 || fp6) ? sc + (2 * j + h) * 256 : sc;
                        if constexpr (fp8) dequant_half_fp8(stg + j * cb, *reinterpret_cast<const float*>(sc), r, h, f16, v);
                        else if constexpr (fp6) dequant_half_fp6(stg + j * cb, scj, r, h, f16, v);
                        else if constexpr (f16) dequant_half_f16(Q, stg + j * cb, scj, zr, r, h, v);
                        else dequant_half(Q, stg + j * cb, scj, zr, r, h, v);
                        tmem_st16(tmem + lane_addr + C::A_COL0 + s * C::A_STAGE_COLS + (m * KSTEP + j) * 32 + 16 * h, v);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&cempty[c]);       // this warp's staged bytes are consumed
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full[s]);
                }
                if (!ok) break;
            }
        }
    } else if (warp >= C::EPI0) {
        // ----------------------------------------------------------- epilogue
        // TMEM -> registers -> (SwiGLU / routing weight) -> 16-bit staging
        // tile [token][128 outputs] in shared memory; the accumulator is
        // released as soon as it is read, then the staged rows are written
        // to global memory with 16-byte stores.
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;                 // weight row within the block = output column
        const int ej = threadIdx.x - C::EPI0 * 32;           // 0 .. 32 * kEpiWarps - 1
        const int cset = (warp - C::EPI0) >> 2;              // this warp's half of the token columns
        uint16_t* out_s = reinterpret_cast<uint16_t*>(smem + C::OUT);
        // The epilogue warps leave the loop together (named barriers): the
        // stop decision is taken by one thread between two barriers.
        // token info of the next tile (scale factor, output row) is loaded
        // while the current one is processed
        // (of the tiles two and one ahead)
        struct TileInfo {
            float sc, gw;
            int row;
        };
        auto fetch = [&](int jn) {
            TileInfo f{1.0f, 1.0f, 0};
            if (MODE == 2 || jn >= nseq) return f;
            const GemmTile tn = tile_at(jn);
            if (!SH && a.g_w) f.gw = __ldg(a.g_w + tn.expert);     // the expert's global scale
            if (ej >= tn.count) return f;
            if constexpr (SH) {
                f.row = tn.seg + ej;
            } else if (MODE == 0) {
                f.sc = a.ts_perm ? __ldg(a.ts_perm + tn.seg + ej) : 1.0f;
                f.row = tn.seg + ej;
            } else {
                // per-slot outputs are stored by permuted position (the
                // combine finds them through the inverse permutation)
                f.sc = __ldg(a.w_perm + tn.seg + ej);
                f.row = tn.seg + ej;
            }
            return f;
        };
        TileInfo nx = fetch(0), nx2 = fetch(1);
        AccSeq aseq;
        for (int jt = 0; jt < nseq; ++jt) {
            const GemmTile t = tile_at(jt);
            const int n_mma = (t.count + 15) & ~15;
            const AccUse au = acc_next<C::ACC_BUFS, C::ACC_COLS, C::TN, C::ACC_SPLIT>(aseq, n_mma);
            const float gsc = (!SH && a.g_w) ? nx.gw * a.g_act : 1.0f;
            // down: the staging buffer of this tile was last read by the TMA
            // stores of the tile OUT_BUFS back
            if (MODE == 1 && ej == 0) {
                if (C::OUT_BUFS == 2) bulk_wait_read<1>();
                else bulk_wait_read<0>();
            }
            epi_sync();                                      // the previous tile's readers are done
            if (ej == 0) ep_stop = abort_flag;
            if (MODE != 2 && ej < t.count) {
                ep_scale[ej] = nx.sc * gsc;
                ep_row[ej] = nx.row;
            }
            nx = nx2;
            nx2 = fetch(jt + 2);
            epi_sync();
            if (ep_stop) break;
            // a failed wait sets abort_flag: this tile is skipped and all four
            // warps stop at the next tile's decision
            if ((au.mask & 1) && !warp_wait(&acc_full[0], au.par0, &abort_flag, a.err, 5)) continue;
            if ((au.mask & 2) && !warp_wait(&acc_full[1], au.par1, &abort_flag, a.err, 5)) continue;
            tc_fence_after();
            // the two warps of a lane quarter split the columns (16-aligned)
            const int chalf = (((n_mma >> 4) + 1) >> 1) << 4;
            const int cbeg = cset ? chalf : 0, cend = cset ? n_mma : chalf;
            const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + au.col;
            if constexpr (MODE == 2) {
                // logits: for each token, the 32 lanes store 32 consecutive
                // experts (128 contiguous bytes)
                const int e = t.rb * kBlkN + row;
                for (int c0 = cbeg; c0 < cend; c0 += 16) {
                    float v0[16];
                    tmem_ld16(lane_base + c0, v0);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c0 + i < t.count && e < a.n_rows) a.logits[(size_t)(t.seg + c0 + i) * a.n_rows + e] = v0[i];
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[au.mask >> 1]);
                continue;
            }
            if constexpr (MODE == 1) {
                // all of this warp's columns (at most 64) in one batch
                uint32_t r[64];
                const int nch = (cend - cbeg) >> 4;
                tmem_ld_chunks(lane_base + cbeg, nch, r);
                uint16_t* ob = out_s + (jt % C::OUT_BUFS) * (C::OUT_TILE / 2);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (q < nch) {
                        // per-slot outputs are fp16 (saturating at +-65504):
                        // their rounding error stays well below the final bf16 one
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int col = cbeg + 16 * q + i;
                            const float sc = col < t.count ? ep_scale[col] : 0.0f;
                            ob[col * kBlkN + row] = __half_as_ushort(f16_sat(__uint_as_float(r[16 * q + i]) * sc));
                        }
                    }
                }
                fence_proxy_async_smem();                    // the TMA stores read what this thread wrote
            }
            if constexpr (MODE == 0) {
                for (int c0 = cbeg; c0 < cend; c0 += 16) {
                    float v0[16];
                    if constexpr (MODE == 0) {
                        float v1[16];
                        tmem_ld16x2(lane_base + c0, lane_base + au.mat_stride + c0, v0, v1);
    #pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int col = c0 + i;
                            const float tsc = col < t.count ? ep_scale[col] : 0.0f;
                            const float gg = v0[i] * tsc, uu = v1[i] * tsc;
                            float act = swiglu_fast(gg, uu);
                            if constexpr (!SH && Q == Q_NVFP4) {
                                // W4A4: requantize the intermediate per 16 consecutive outputs
                                float amax = fabsf(act);
    #pragma unroll
                                for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                                const float gq = a.g_req;
                                float sbv = 0.0f, rcp = 0.0f;
                                if (gq != 0.0f) {
                                    sbv = e4m3_to_f32(f32_to_e4m3(__fdiv_rn(amax, __fmul_rn(6.0f, gq))));
                                    rcp = (sbv == 0.0f) ? 0.0f : __fdiv_rn(1.0f, __fmul_rn(sbv, gq));
                                }
                                act = e2m1_to_f32(f32x2_to_e2m1(__fmul_rn(act, rcp), 0.0f) & 0xFu) * sbv;
                            }
                            // the routed INT/FP8/FP6 intermediate is the fp16 B operand
                            // of the down GEMM (saturating at +-65504); the shared expert's
                            // and the W4A4 values stay bf16
                            if constexpr (!SH && Q != Q_NVFP4)
                                out_s[col * kBlkN + row] = __half_as_ushort(f16_sat(act));
                            else
                                out_s[col * kBlkN + row] = __bfloat16_as_ushort(__float2bfloat16_rn(act));
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {                                 // the MMA may refill this accumulator
                if (au.mask & 1) mbar_arrive(&acc_empty[0]);
                if (au.mask & 2) mbar_arrive(&acc_empty[1]);
            }
            epi_sync();                                      // staging tile complete
            if constexpr (MODE == 1) {
                // the tile's rows (permuted positions, or tokens of the shared
                // expert) are seg .. seg+count-1
                if (ej == 0)
                    store_tile_rows(map_o, t.rb * kBlkN, t.seg, t.count,
                                    reinterpret_cast<const uint8_t*>(out_s + (jt % C::OUT_BUFS) * (C::OUT_TILE / 2)));
            } else {
                uint16_t* dst = reinterpret_cast<uint16_t*>(SH ? a.out_sh : a.out);
                const int col0 = t.rb * kBlkN;
                for (int i = ej; i < t.count * 16; i += kEpiWarps * 32) {
                    const int col = i >> 4, ch = i & 15;
                    const uint4 q = *reinterpret_cast<const uint4*>(out_s + col * kBlkN + ch * 8);
                    *reinterpret_cast<uint4*>(dst + (size_t)ep_row[col] * a.out_ld + col0 + ch * 8) = q;
                }
            }
        }
        if (MODE == 1 && ej == 0) bulk_wait_all();          // every store done before the CTA leaves
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) tmem_dealloc(tmem, kTmemCols);
}

// --------------------------------------------------------------- combine
// y[t] = sum_{j<k} O[inv[t*k + j]] + S[t], fp32 sum in fixed j order, one
// bf16 rounding; O holds the weighted expert outputs by permuted position.
// A slot without a position (id outside [0, E): inv < 0) has no expert
// output and contributes zero.
MOE_DEV float h_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu))); }
MOE_DEV float h_hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }

// Slot rows per batch of loads: the top-10 workloads issue every slot row
// and the shared row at once (one round trip per thread; 70.4 -> 67.3 us
// against batches of 8 at T = 8192).
constexpr int kCombineBatch = 12;
template <int KB>
__global__ void k_combine(const __half* __restrict__ O, const __half* __restrict__ S, const int32_t* __restrict__ inv,
                          int T, int H, int k, __nv_bfloat16* __restrict__ y) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // one thread per 8 columns
    const int per_row = H / 8;
    if (i >= (long long)T * per_row) return;
    const int t = (int)(i / per_row), c = (int)(i % per_row) * 8;
    // the permuted position of each of the token's slots (-1: no expert
    // output); KB 16-byte slot rows and the shared row in flight per thread,
    // summed in the fixed j order
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j0 = 0; j0 < k; j0 += KB) {
        int pos[KB];
#pragma unroll
        for (int u = 0; u < KB; ++u) pos[u] = j0 + u < k ? __ldg(inv + (size_t)t * k + j0 + u) : -1;
        uint4 q[KB];
#pragma unroll
        for (int u = 0; u < KB; ++u)
            q[u] = pos[u] >= 0 ? ldg_stream_v4(O + (size_t)pos[u] * H + c) : make_uint4(0, 0, 0, 0);
        uint4 sq = make_uint4(0, 0, 0, 0);
        const bool last = j0 + KB >= k;
        if (S && last) sq = ldg_stream_v4(S + (size_t)t * H + c);
#pragma unroll
        for (int u = 0; u < KB; ++u) {
            if (pos[u] >= 0) {
                const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
                for (int p = 0; p < 4; ++p) { acc[2 * p] += h_lo(w[p]); acc[2 * p + 1] += h_hi(w[p]); }
            }
        }
        if (S && last) {
            const uint32_t w[4] = {sq.x, sq.y, sq.z, sq.w};
#pragma unroll
            for (int p = 0; p < 4; ++p) { acc[2 * p] += h_lo(w[p]); acc[2 * p + 1] += h_hi(w[p]); }
        }
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
// GEMM epilogue.  The row is written straight into the permuted operand: the
// warp of token t converts it once and stores it at the k positions
// inv[t*k + j] of its slots (with each position's routing weight and token
// scale for the GEMM epilogues).  Dropped slots (inv < 0) are skipped.
__global__ void k_x_to_f16_perm(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ inv, int T, int H,
                                int k, __half* __restrict__ xp, float* __restrict__ scale, const float* __restrict__ topk_w,
                                float* __restrict__ w_perm, float* __restrict__ ts_perm) {
    const int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    const int mypos = lane < k ? __ldg(inv + (size_t)t * k + lane) : -1;
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
        const uint4 ov = make_uint4(o[0], o[1], o[2], o[3]);
        for (int j = 0; j < k; ++j) {
            const int pos = __shfl_sync(0xffffffffu, mypos, j);
            if (pos >= 0) reinterpret_cast<uint4*>(xp + (size_t)pos * H)[c] = ov;
        }
    }
    const float sc = ldexpf(1.0f, p);
    if (lane < k && mypos >= 0) {
        w_perm[mypos] = __ldg(topk_w + (size_t)t * k + lane);
        ts_perm[mypos] = sc;
    }
    if (lane == 0) scale[t] = sc;
}

// Routing weight and token scale of permuted position p, read by the GEMM
// epilogues as one independent load per token column.
MOE_DEV void perm_meta(int p, int slot, int k, const PermMeta& m) {
    m.w_perm[p] = __ldg(m.topk_w + slot);
    if (m.tok_scale) m.ts_perm[p] = __ldg(m.tok_scale + slot / k);
}

// Rows of the gate/up token operand in permuted order: xp[p] = xq[perm[p] / k]
// (16-byte copies; one thread per 8 columns); also the per-position meta.
__global__ void k_gather_rows(const __nv_bfloat16* __restrict__ xq, const int32_t* __restrict__ perm, int slots,
                              int H, int k, __nv_bfloat16* __restrict__ xp, PermMeta meta) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int per_row = H / 8;
    if (i >= (long long)slots * per_row) return;
    const int p = (int)(i / per_row), c = (int)(i % per_row);
    const int slot = __ldg(perm + p), t = slot / k;
    if (c == 0) perm_meta(p, slot, k, meta);
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
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __bfloat162float(src[i]);
    nvfp4_block16_values(v, g);
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 16; i += 2) o[i / 2] = pack_bf16x2(v[i], v[i + 1]);
    uint4* d = reinterpret_cast<uint4*>(xq + (size_t)t * kFp4Blk);
    d[0] = make_uint4(o[0], o[1], o[2], o[3]);
    d[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

// ------------------------------------------------------------ NVFP4 native
// W4A4 routed tiles on the block-scaled tensor-core path.  A (weights, e2m1)
// and B (tokens, e2m1) are TMA tiles of 128 rows x 256 values (128 bytes,
// 128-byte swizzle) read from natural-layout images; their e4m3 block scales
// (one per 16 values) are TMA tiles of 128 rows x 16 bytes that four warps
// store into TMEM in the layout the MMA reads (for each K = 64 instruction,
// four 32-bit columns: column c, lane l holds the four scales of row 32c + l,
// replicated in every lane quarter), and
// tcgen05.mma.kind::mxf4nvf4.block_scale.block16 multiplies 64 values of K
// per instruction.  The fp32 global scales of weights and activations are
// applied in the epilogue.  The gate/up epilogue requantizes the SwiGLU
// intermediate to NVFP4 (codes and scales) for the down GEMM.
constexpr int kFp4KS = 256;                  // K values per stage
constexpr int kFp4Tile = 128 * 128;          // 16 KB: 128 rows x 128 bytes
constexpr int kFp4SfTile = 128 * 16;         // 2 KB: 128 rows x 16 scale bytes

// Token-operand maps of the block-scaled GEMM (e2m1 codes, 128-byte rows,
// 128-byte swizzle) with boxes of 16, 32, ..., 176 rows: a tile of n (a
// multiple of 16) tokens loads exactly its rows with one TMA request (the
// copy engine's requests per SM, not bytes, bound these GEMMs' streaming).
struct Fp4BMaps {
    CUtensorMap codes[11];  // box rows 16 (i + 1), up to a gate/up tile's 176
};
MOE_DEV void load_fp4_token_rows(uint8_t* dst_codes, const Fp4BMaps& mb, int x_codes, int y, int n, uint64_t* bar) {
    tma_load_2d(dst_codes, &mb.codes[(n >> 4) - 1], x_codes, y, bar);
}


// Tokens per tile of the block-scaled GEMMs (the MMA's N, at most 256): an
// expert's ~160 tokens of the uniform workload are one tile, so each weight
// block streams once and each (expert, row block) pays one epilogue.
constexpr int kFp4GuN = 176;

// The accumulator of the next tile, walked identically by the MMA warps and
// the epilogue: buffer, first column, matrix stride and phase parity.
struct Fp4Acc {
    int buf;
    uint32_t col, mat_stride, parity;
};
struct Fp4AccSeq {
    uint32_t uses0 = 0u, uses1 = 0u;   // completed uses of buffer 0 / 1
    int local = 0;
};
template <int MODE>
MOE_DEV Fp4Acc fp4_acc_next(Fp4AccSeq& q, int n_mma) {
    Fp4Acc a;
    (void)n_mma;
    if (MODE == 1) {
        a.buf = q.local & 1;
        a.col = (uint32_t)(a.buf * kFp4GuN);
        a.mat_stride = kFp4GuN;
    } else {
        a.buf = 0;
        a.col = 0;
        a.mat_stride = kFp4GuN;
    }
    a.parity = (a.buf ? q.uses1 : q.uses0) & 1u;
    q.uses0 += a.buf == 0 ? 1u : 0u;
    q.uses1 += a.buf == 1 ? 1u : 0u;
    ++q.local;
    return a;
}

template <int MODE>
struct Fp4Cfg {
    static constexpr int NMAT = MODE == 0 ? 2 : 1;
    // stages: down takes two (a tile is two stages) so that two staging
    // buffers fit, which let a tile's TMA stores overlap the next staging
    static constexpr int S = MODE == 0 ? 3 : 2;
    static constexpr int SF0 = kWarpMma + NMAT;                       // four scale-factor warps
    static constexpr int EPI0 = SF0 + 4;
    // epilogue warps: four per TMEM lane quarter, each taking
    // a part of the tile's token columns (the SwiGLU + requantization or the fp16
    // staging of a tile is the longest step of these kernels)
    static constexpr int EPI_WARPS = 16;
    static constexpr int THREADS = (EPI0 + EPI_WARPS) * 32;
    // token rows per tile
    static constexpr int BROWS = kFp4GuN;
    // accumulators: gate/up one of 2 x BROWS columns (the epilogue reads it
    // and releases it before the requantization); down alternates two of
    // BROWS
    static constexpr int ACC_COLS = NMAT * BROWS;
    // scale factors in TMEM: per slot, A (4 columns per MMA and matrix), then
    // B (ceil(rows / 32) columns per MMA, at 8-column steps); two slots, each
    // released by its own MMA commits
    static constexpr int SFB_KK = 8;
    static constexpr int SF_STAGE_COLS = NMAT * 16 + 4 * SFB_KK;
    static constexpr int SF_SLOTS = 2;
    static constexpr int SF_COL0 = MODE == 0 ? ACC_COLS : 2 * ACC_COLS;
    static_assert(SF_COL0 + SF_SLOTS * SF_STAGE_COLS <= (int)kTmemCols, "TMEM budget");
    // weights: per stage one block of the image, [NMAT][16 KB codes] then
    // [NMAT][2 KB scales] (a multiple of 1 KB: every code tile stays aligned
    // for the 128-byte swizzle)
    static constexpr int W_STAGE = NMAT * (kFp4Tile + kFp4SfTile);
    static constexpr int B_STAGE = BROWS * 128;                       // a multiple of 1 KB
    // token scales: rows 32c + lane of each 32-row column group are read, so
    // a stage's tile spans whole groups
    static constexpr int SFB_STAGE = ((BROWS + 31) / 32) * 32 * 16;
    static constexpr int W = 0;                                       // [S][W_STAGE]
    static constexpr int B = W + S * W_STAGE;                         // [S][B_STAGE]
    static constexpr int SFB = B + S * B_STAGE;                       // [S][SFB_STAGE]
    static constexpr int OUT = SFB + S * SFB_STAGE;                   // gate/up: [BROWS][80 B]; down: 2 x [BROWS][128] fp16
    static constexpr int OUT_TILE = BROWS * kBlkN * 2;
    static constexpr int OUT_BYTES = MODE == 0 ? BROWS * 80 : 2 * OUT_TILE;
    static constexpr int SCR = OUT + OUT_BYTES;                       // gate/up: per epilogue warp [8 tok][32] fp32
    static constexpr int SCR_BYTES = MODE == 0 ? EPI_WARPS * 8 * 32 * 4 : 0;
    static constexpr int ALLOC = SCR + SCR_BYTES + 1024;
    static_assert(ALLOC <= 227 * 1024 - 8192, "shared memory budget (static arrays take up to 8 KB)");
};

template <int MODE>
__global__ void __launch_bounds__(Fp4Cfg<MODE>::THREADS, 1)
k_fp4_gemm(const __grid_constant__ Fp4BMaps map_b, const __grid_constant__ OMaps map_o, GemmArgs a) {
    using C = Fp4Cfg<MODE>;
    constexpr int NMAT = C::NMAT, S = C::S;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[S], sfready[S], empty[S], acc_full[2], acc_empty[2], sffree[2];
    __shared__ uint32_t tmem_base_slot;
    __shared__ volatile int abort_flag;
    __shared__ float ep_scale[kFp4GuN];
    __shared__ int ep_row[kFp4GuN];
    __shared__ int ep_stop;
    __shared__ float rcp_tab[256];              // gate/up: 1 / (e4m3(code) * g_req), IEEE division, 0 for zero
    __shared__ TileCache tcache;
    __shared__ int gscan[kTileCache / 32];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (__ldcg(a.num_tiles + 3)) cache_groups(tcache, a.tiles, a.groups, __ldcg(a.num_tiles + 2), gscan);
    else cache_tiles(tcache, a.tiles, blockIdx.x, __ldcg(a.num_tiles));
    if (MODE == 0 && threadIdx.x < 256) {
        const float sbv = e4m3_to_f32((uint32_t)threadIdx.x);
        rcp_tab[threadIdx.x] = (sbv == 0.0f || a.g_req == 0.0f) ? 0.0f : __fdiv_rn(1.0f, __fmul_rn(sbv, a.g_req));
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);                       // producer (bytes)
            mbar_init(&sfready[s], 4);                    // the four scale-factor warps
            mbar_init(&empty[s], NMAT);                   // one commit per MMA warp
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], NMAT);
            mbar_init(&acc_empty[b], C::EPI_WARPS);
            mbar_init(&sffree[b], NMAT);                  // one commit per MMA warp
        }
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) tmem_alloc(&tmem_base_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_slot;
    const int t_end = __ldcg(a.num_tiles);                // routed tiles only
    const int nseq = tcache.n;                            // this CTA's tile sequence
    auto tile_at = [&](int j) { return load_tile<MODE>(a, (int)blockIdx.x + j * (int)gridDim.x, &tcache, blockIdx.x, j); };
    const int NS = a.K / kFp4KS;

    if (warp == kWarpProducer) {
        // ---------------------------------------------------------- producer
        int g = 0;
        for (int jt = 0; jt < nseq && !abort_flag; ++jt) {
            const GemmTile t = tile_at(jt);
            // this (expert, row block)'s NS consecutive image blocks
            const uint8_t* wblk = a.wimg + ((size_t)t.expert * (a.n_rows / kBlkN) + t.rb) * NS * C::W_STAGE;
            bool ok = true;
            for (int ks = 0; ks < NS; ++ks, ++g) {
                const int s = g % S;
                const uint32_t r = (uint32_t)(g / S);
                if (!warp_wait(&empty[s], (r & 1u) ^ 1u, &abort_flag, a.err, 11)) { ok = false; break; }
                if (lane == 0) {
                    // the stage's weight codes and scales (one bulk copy),
                    // then the tile's token rows and their scales
                    const int n_mma = (t.count + 15) & ~15;
                    mbar_arrive_expect_tx(&full[s], (uint32_t)C::W_STAGE + (uint32_t)n_mma * 144u);
                    bulk_g2s(smem + C::W + s * C::W_STAGE, wblk + (size_t)ks * C::W_STAGE, (uint32_t)C::W_STAGE,
                             &full[s]);
                    // the token rows' scales: n_mma x 16 B, contiguous (rows past
                    // the end of the slots read workspace slack, never used)
                    bulk_g2s(smem + C::SFB + s * C::SFB_STAGE, a.sfb + ((size_t)ks * a.sfb_rows + t.seg) * 16,
                             (uint32_t)n_mma * 16u, &full[s]);
                    load_fp4_token_rows(smem + C::B + s * C::B_STAGE, map_b, ks * 128, t.seg, n_mma, &full[s]);
                }
                __syncwarp();
            }
            if (!ok) break;
        }
    } else if (warp >= kWarpMma && warp < C::SF0) {
        // --------------------------------------------------------- MMA issue
        const int mi = warp - kWarpMma;
        int g = 0;
        Fp4AccSeq aseq;
        for (int jt = 0; jt < nseq && !abort_flag; ++jt) {
            const GemmTile t = tile_at(jt);
            const int n_mma = (t.count + 15) & ~15;
            const uint32_t idesc = idesc_nvfp4(128, n_mma);
            const Fp4Acc acc = fp4_acc_next<MODE>(aseq, n_mma);
            const int ab = acc.buf;
            if (!warp_wait(&acc_empty[ab], acc.parity ^ 1u, &abort_flag, a.err, 12)) break;
            tc_fence_after();
            bool ok = true;
            const uint32_t d = tmem + acc.col + mi * acc.mat_stride;
            for (int ks = 0; ks < NS; ++ks, ++g) {
                const int s = g % S;
                const uint32_t r = (uint32_t)(g / S);
                if (!warp_wait(&full[s], r & 1u, &abort_flag, a.err, 13)) { ok = false; break; }
                if (!warp_wait(&sfready[s], r & 1u, &abort_flag, a.err, 14)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint64_t adesc = desc_kmajor_sw128(smem_u32(smem + C::W + s * C::W_STAGE + mi * kFp4Tile));
                    const uint64_t bdesc = desc_kmajor_sw128(smem_u32(smem + C::B + s * C::B_STAGE));
                    const int slot = g % C::SF_SLOTS;
                    const uint32_t sf = tmem + C::SF_COL0 + slot * C::SF_STAGE_COLS;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_fp4_block16(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, sf + mi * 16 + kk * 4,
                                        sf + NMAT * 16 + kk * C::SFB_KK, (ks | kk) != 0);
                    mma_commit(&empty[s]);
                    mma_commit(&sffree[slot]);                    // this slot's scales are consumed
                    if (ks == NS - 1) mma_commit(&acc_full[ab]);
                }
                __syncwarp();
            }
            if (!ok) break;
        }
    } else if (warp >= C::SF0 && warp < C::EPI0) {
        // ---------------------------------------------- scale factors -> TMEM
        const int quarter = warp & 3;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        int g = 0;
        for (int jt = 0; jt < nseq && !abort_flag; ++jt) {
            bool ok = true;
            for (int ks = 0; ks < NS; ++ks, ++g) {
                const int s = g % S;
                const uint32_t r = (uint32_t)(g / S);
                if (!warp_wait(&full[s], r & 1u, &abort_flag, a.err, 15)) { ok = false; break; }
                // the TMEM slot is free once the MMAs of stage g - 2 are done
                const int slot = g % C::SF_SLOTS;
                if (g >= C::SF_SLOTS &&
                    !warp_wait(&sffree[slot], (uint32_t)((g / C::SF_SLOTS - 1) & 1), &abort_flag, a.err, 17)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sf = tmem + lane_addr + C::SF_COL0 + slot * C::SF_STAGE_COLS;
                // column 4 kk + cc (A) / SFB_KK kk + cc (B): the scales of
                // K-blocks 4kk..4kk+3 of row 32cc + lane
#pragma unroll
                for (int q = 0; q < NMAT; ++q) {
                    const uint8_t* tile = smem + C::W + s * C::W_STAGE + NMAT * kFp4Tile + q * kFp4SfTile;
                    uint32_t v[16];
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        const uint4 w = *reinterpret_cast<const uint4*>(tile + (32 * cc + lane) * 16);
                        v[0 * 4 + cc] = w.x;
                        v[1 * 4 + cc] = w.y;
                        v[2 * 4 + cc] = w.z;
                        v[3 * 4 + cc] = w.w;
                    }
                    tmem_st16(sf + q * 16, v);
                }
                {
                    const uint8_t* tile = smem + C::SFB + s * C::SFB_STAGE;
                    constexpr int CB = C::SFB_STAGE / (32 * 16);           // 32-row groups of the B tile
                    uint32_t v[4 * C::SFB_KK];
#pragma unroll
                    for (int i = 0; i < 4 * C::SFB_KK; ++i) v[i] = 0u;
#pragma unroll
                    for (int cc = 0; cc < CB; ++cc) {
                        const uint4 w = *reinterpret_cast<const uint4*>(tile + (32 * cc + lane) * 16);
                        v[0 * C::SFB_KK + cc] = w.x;
                        v[1 * C::SFB_KK + cc] = w.y;
                        v[2 * C::SFB_KK + cc] = w.z;
                        v[3 * C::SFB_KK + cc] = w.w;
                    }
#pragma unroll
                    for (int h = 0; h < C::SFB_KK / 4; ++h) {
                        uint32_t u[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) u[i] = v[16 * h + i];
                        tmem_st16(sf + NMAT * 16 + 16 * h, u);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfready[s]);
            }
            if (!ok) break;
        }
    } else if (warp >= C::EPI0) {
        // ----------------------------------------------------------- epilogue
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int ej = threadIdx.x - C::EPI0 * 32;
        const int cset = (warp - C::EPI0) >> 2;              // this warp's quarter of the token columns
        uint8_t* out_s = smem + C::OUT;
        // token info (routing weight, output row) and expert global scale
        // of the tiles two and one ahead, loaded while the current tile is
        // processed (the routing weights are HBM reads by then)
        struct TileInfo {
            float sc, gw;
            int row;
        };
        auto fetch = [&](int jn) {
            TileInfo f{1.0f, 0.0f, 0};
            if (jn >= nseq) return f;
            const GemmTile tn = tile_at(jn);
            f.gw = __ldg(a.g_w + tn.expert);
            if (ej >= tn.count) return f;
            f.sc = MODE == 0 ? 1.0f : __ldg(a.w_perm + tn.seg + ej);
            f.row = tn.seg + ej;
            return f;
        };
        // (gate/up reads only the small table of global scales: one tile ahead)
        TileInfo nx = fetch(0), nx2 = MODE == 1 ? fetch(1) : TileInfo{1.0f, 0.0f, 0};
        int local = 0;
        Fp4AccSeq aseq;
        for (int jt = 0; jt < nseq; ++jt, ++local) {
            const GemmTile t = tile_at(jt);
            const Fp4Acc acc = fp4_acc_next<MODE>(aseq, (t.count + 15) & ~15);
            const int ab = acc.buf;
            const float gsc = nx.gw * a.g_act;
            // down: this tile's staging buffer was last read by the TMA
            // stores of the tile two back (one bulk group per tile)
            if (MODE == 1 && ej == 0) bulk_wait_read<1>();
            epi_sync_n<C::EPI_WARPS>();
            if (ej == 0) ep_stop = abort_flag;
            if (ej < t.count) {
                ep_scale[ej] = nx.sc * gsc;
                ep_row[ej] = nx.row;
            }
            if constexpr (MODE == 1) {
                nx = nx2;
                nx2 = fetch(jt + 2);
            } else {
                nx = fetch(jt + 1);
            }
            epi_sync_n<C::EPI_WARPS>();
            if (ep_stop) break;
            if (!warp_wait(&acc_full[ab], acc.parity, &abort_flag, a.err, 16)) continue;
            tc_fence_after();
            const int n_mma = (t.count + 15) & ~15;
            // the warps of a lane quarter split the columns (16-aligned parts)
            constexpr int NSET = C::EPI_WARPS / 4;
            const int cpart = (((n_mma >> 4) + NSET - 1) / NSET) << 4;
            const int cbeg = min(n_mma, cset * cpart), cend = min(n_mma, cbeg + cpart);
            const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + acc.col;
            const int nch = (cend - cbeg) >> 4;
            // Every warp first copies its accumulator columns into registers
            // and releases the accumulator, so that the MMAs of the next tile
            // start while this tile's SwiGLU / requantization or fp16
            // conversion runs.
            if constexpr (MODE == 1) {
                static_assert(C::EPI_WARPS == 16 && kFp4GuN <= 192, "down: at most 48 columns per warp");
                // 16 columns at a time (the two accumulators alternate, so
                // this one is released after the conversion)
                uint16_t* ob = reinterpret_cast<uint16_t*>(out_s + (local & 1) * C::OUT_TILE);
#pragma unroll 1
                for (int q = 0; q < nch; ++q) {
                    uint32_t r[32];
                    tmem_ld_x16c(lane_base + cbeg + 16 * q, r);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int col = cbeg + 16 * q + i;
                        const float sc = col < t.count ? ep_scale[col] : 0.0f;
                        ob[col * kBlkN + row] = __half_as_ushort(f16_sat(__uint_as_float(r[i]) * sc));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[ab]);
                fence_proxy_async_smem();        // the TMA store reads what this thread wrote
            } else {
                static_assert(C::EPI_WARPS == 16 && kFp4GuN <= 192, "gate/up: at most 48 columns per warp");
                // SwiGLU as each 16-column chunk is read: only the 3 x 16
                // results stay live across the release
                float act[3][16];
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                    if (q < nch) {
                        const int c0 = cbeg + 16 * q;
                        float vg[16], vu[16];
                        tmem_ld16x2(lane_base + c0, lane_base + acc.mat_stride + c0, vg, vu);
                        // one scale for the whole tile (the expert's and the
                        // activations' global scales); padding columns give 0
                        const float sct = ep_scale[0];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float sc = c0 + i < t.count ? sct : 0.0f;
                            act[q][i] = swiglu_fast(vg[i] * sc, vu[i] * sc);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[ab]);
                // the warp's scratch [8 tokens][32 outputs] turns the results
                // into 16-output blocks for the requantization, eight tokens
                // at a time: lane = (token i, block b, half hf) takes eight
                // values of the block, the two halves share the block's amax
                float* scr = reinterpret_cast<float*>(smem + C::SCR) + (warp - C::EPI0) * 8 * 32;
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                    if (q < nch) {
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int c0 = cbeg + 16 * q + 8 * hh;
#pragma unroll
                            for (int i = 0; i < 8; ++i) scr[i * 32 + lane] = act[q][8 * hh + i];
                            __syncwarp();
                            // NVFP4 with the static global scale; code decisions in
                            // fp32 as the format defines them
                            {
                                const int i = lane & 7, b = (lane >> 3) & 1, hf = lane >> 4;
                                const float4* src = reinterpret_cast<const float4*>(scr + i * 32 + b * 16 + hf * 8);
                                const float4 f0 = src[0], f1 = src[1];
                                const float v[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
                                float amax = 0.0f;
#pragma unroll
                                for (int qq = 0; qq < 8; ++qq) amax = fmaxf(amax, fabsf(v[qq]));
                                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 16));
                                const uint32_t sbc = a.g_req != 0.0f ? f32_to_e4m3(__fdiv_rn(amax, __fmul_rn(6.0f, a.g_req))) : 0u;
                                const float rcp = rcp_tab[sbc];
                                uint32_t w = 0u;
#pragma unroll
                                for (int qq = 0; qq < 4; ++qq)
                                    w |= f32x2_to_e2m1(__fmul_rn(v[2 * qq], rcp), __fmul_rn(v[2 * qq + 1], rcp)) << (8 * qq);
                                const int col = c0 + i, o0 = (quarter * 32 + b * 16) >> 1;   // byte of output row quarter*32 + 16b
                                *reinterpret_cast<uint32_t*>(out_s + col * 80 + o0 + 4 * hf) = w;
                                if (hf == 0) out_s[col * 80 + 64 + quarter * 2 + b] = (uint8_t)sbc;
                            }
                            __syncwarp();
                        }
                    }
                }
            }
            epi_sync_n<C::EPI_WARPS>();
            if constexpr (MODE == 0) {
                // per token: 64 code bytes and 8 scale bytes of this 128-row block
                const int I2 = a.out_ld / 2;
                for (int i = ej; i < t.count * 5; i += C::EPI_WARPS * 32) {
                    const int col = i / 5, part = i % 5;
                    const size_t r = (size_t)ep_row[col];
                    if (part < 4)
                        *reinterpret_cast<uint4*>(a.out4 + r * I2 + t.rb * 64 + part * 16) =
                            *reinterpret_cast<const uint4*>(out_s + col * 80 + part * 16);
                    else   // stage-major scales: stage rb / 2, bytes 8 (rb % 2) .. +8
                        *reinterpret_cast<uint2*>(a.out_sf + ((size_t)(t.rb >> 1) * a.sfb_rows_out + r) * 16 + (t.rb & 1) * 8) =
                            *reinterpret_cast<const uint2*>(out_s + col * 80 + 64);
                }
            } else if (ej == 0) {
                // the tile's rows are the permuted positions seg .. seg+count-1:
                // TMA stores of boxes of 128, 64, ..., 1 rows, one bulk group
                store_tile_rows(map_o, t.rb * kBlkN, t.seg, t.count, out_s + (local & 1) * C::OUT_TILE);
            }
        }
        if (MODE == 1 && ej == 0) bulk_wait_all();     // every store done before the CTA leaves
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) tmem_dealloc(tmem, kTmemCols);
}

// W4A4 activations of the gate/up GEMM in permuted order, quantized per 16
// values with the static global scale g (codes [slots][H/2]; scales
// stage-major [H/256][slots][16 B], so that a GEMM stage's scale rows are
// contiguous).  The warp of token t quantizes its row once and stores it
// at the k positions inv[t*k + j] of its slots, with each position's
// routing weight; dropped slots (inv < 0) are skipped.
__global__ void k_x_fp4_perm(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ inv, int T, int H, int k,
                             float g, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, long long slots,
                             const float* __restrict__ topk_w, float* __restrict__ w_perm) {
    const int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    const int mypos = lane < k ? __ldg(inv + (size_t)t * k + lane) : -1;
    for (int b = lane; b < H / 16; b += 32) {
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H + b * 16);
        const uint4 q0 = src[0], q1 = src[1];
        const uint32_t wv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        float v[16];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            v[2 * q] = bf16_lo(wv[q]);
            v[2 * q + 1] = bf16_hi(wv[q]);
        }
        uint32_t w[2];
        const uint32_t sbc = nvfp4_quant_block16(v, g, w);
        for (int j = 0; j < k; ++j) {
            const int pos = __shfl_sync(0xffffffffu, mypos, j);
            if (pos < 0) continue;
            *reinterpret_cast<uint2*>(codes + (size_t)pos * (H / 2) + b * 8) = make_uint2(w[0], w[1]);
            sf[((size_t)(b >> 4) * slots + pos) * 16 + (b & 15)] = (uint8_t)sbc;
        }
    }
    if (lane < k && mypos >= 0) w_perm[mypos] = __ldg(topk_w + (size_t)t * k + lane);
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

// Token-operand maps with 128-, 64-, 32- and 16-row boxes
static bool make_bmaps(BMaps* mb, const void* base, uint64_t rows, uint64_t cols,
                       CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    for (int i = 0; i < 4; ++i)
        if (!make_map(&mb->m[i], base, rows, cols, (uint32_t)(kBN >> i), dt)) return false;
    return true;
}

// 2D map over bytes [rows, row_bytes]: box box_bytes x box_rows, 128-byte
// swizzle for operand tiles, none for scale tiles
static bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t row_bytes, uint32_t box_bytes,
                        uint32_t box_rows, bool sw128) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {row_bytes, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_bytes, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool prefill_native_fp4(int H, int I) { return H % kFp4KS == 0 && I % kFp4KS == 0; }

// Token-operand maps of the block-scaled GEMM over codes [rows][K/2], boxes
// of 16, 32, ..., 176 rows
static bool make_fp4_bmaps(Fp4BMaps* mb, const void* codes, uint64_t rows, int K) {
    for (int i = 0; i < 11; ++i)
        if (!make_map_u8(&mb->codes[i], codes, rows, K / 2, 128, (uint32_t)(16 * (i + 1)), true)) return false;
    return true;
}

// 2D fp16 map over [rows, cols] for TMA stores: box 128 columns x box_rows,
// no swizzle (the smem image is row-major)
static bool make_map_store16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {128, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The eight store maps (boxes of 128 / 2^i rows) of a 16-bit [rows][cols] output.
static bool make_omaps(OMaps* mo, const void* base, uint64_t rows, uint64_t cols) {
    for (int i = 0; i < 8; ++i)
        if (!make_map_store16(&mo->m[i], base, rows, cols, (uint32_t)(kBN >> i))) return false;
    return true;
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

// One persistent CTA per SM over the routed (SH = false) or the shared (SH =
// true) tiles of the list.
// map_o: the down launches' output store maps (unused by the others).
template <int MODE, bool SH, int Q>
static cudaError_t launch_gemm_q(const BMaps& map_b, const GemmArgs& g, cudaStream_t st, const CUtensorMap* map_a,
                                 int grid, const OMaps& map_o) {
    constexpr int bytes = Cfg<MODE, SH>::ALLOC;
    cudaError_t err =
        cudaFuncSetAttribute(k_grouped_gemm<MODE, SH, Q>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (err != cudaSuccess) return err;
    k_grouped_gemm<MODE, SH, Q><<<grid > 0 ? grid : num_sms(), Cfg<MODE, SH>::THREADS, bytes, st>>>(
        map_b, map_a ? *map_a : map_b.m[0], map_o, g);
    return cudaGetLastError();
}

template <int MODE, bool SH>
static cudaError_t launch_gemm(const BMaps& map_b, const GemmArgs& g, cudaStream_t st,
                               const CUtensorMap* map_a = nullptr, int grid = 0, const OMaps* map_o = nullptr) {
    OMaps none;
    memset(&none, 0, sizeof(none));
    const OMaps& mo = map_o ? *map_o : none;
    if (MODE == 1 && !map_o) return cudaErrorInvalidValue;
    if constexpr (SH) {
        return launch_gemm_q<MODE, true, Q_BF16>(map_b, g, st, map_a, grid, mo);
    } else {
        switch (g.quant) {
            case Q_INT4: return launch_gemm_q<MODE, false, Q_INT4>(map_b, g, st, map_a, grid, mo);
            case Q_INT4G32: return launch_gemm_q<MODE, false, Q_INT4G32>(map_b, g, st, map_a, grid, mo);
            case Q_INT2: return launch_gemm_q<MODE, false, Q_INT2>(map_b, g, st, map_a, grid, mo);
            case Q_NVFP4: return launch_gemm_q<MODE, false, Q_NVFP4>(map_b, g, st, map_a, grid, mo);
            case Q_FP8: return launch_gemm_q<MODE, false, Q_FP8>(map_b, g, st, map_a, grid, mo);
            case Q_FP6: return launch_gemm_q<MODE, false, Q_FP6>(map_b, g, st, map_a, grid, mo);
            default: return cudaErrorInvalidValue;
        }
    }
}

// Router logits on the tensor cores: logits[T, E] = x[T, H] . Wr[E, H]^T in
// fp32 (bf16 products, fp32 accumulation); tiles of 128 experts x 128 tokens.
cudaError_t launch_router_tc(const void* x, const void* wr, int T, int H, int E, float* logits, int* err,
                             cudaStream_t st) {
    BMaps m_x;
    CUtensorMap m_w;
    if (!make_bmaps(&m_x, x, (uint64_t)T, (uint64_t)H) || !make_map(&m_w, wr, (uint64_t)E, (uint64_t)H, kBlkN))
        return cudaErrorInvalidValue;
    GemmArgs g{};
    g.K = H;
    g.logits = logits;
    g.n_tok = T;
    g.n_rows = E;
    constexpr int TN = Cfg<2, true>::TN;
    g.n_tiles = ((E + kBlkN - 1) / kBlkN) * ((T + TN - 1) / TN);
    g.err = err;
    return launch_gemm<2, true>(m_x, g, st, &m_w, g.n_tiles < num_sms() ? g.n_tiles : num_sms());
}

// Block-scaled NVFP4 GEMM over the routed tiles; maps: A of gate (or down),
// A of up, their scale tiles, B and its scale tiles.
template <int MODE>
static cudaError_t launch_fp4(const Fp4BMaps& mb, const OMaps& mo, const GemmArgs& g, cudaStream_t st) {
    constexpr int bytes = Fp4Cfg<MODE>::ALLOC;
    cudaError_t err = cudaFuncSetAttribute(k_fp4_gemm<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (err != cudaSuccess) return err;
    k_fp4_gemm<MODE><<<num_sms(), Fp4Cfg<MODE>::THREADS, bytes, st>>>(mb, mo, g);
    return cudaGetLastError();
}

// The prefill path of NVFP4 layers: activations quantized into permuted
// rows, block-scaled gate/up (intermediate requantized to NVFP4), block-scaled
// down; the bf16 shared expert and the combine as in the other formats.
static cudaError_t launch_prefill_fp4(const PrefillArgs& p, cudaStream_t st) {
    const ExpertArgs& ex = p.ex;
    const int T = p.T, k = ex.k, H = ex.H, I = ex.I, E = ex.E;
    const int slots = T * k;
    const bool has_sh = ex.sh_gate != nullptr;
    uint8_t* xc = reinterpret_cast<uint8_t*>(p.xp);                  // [slots][H/2] e2m1
    uint8_t* xs = xc + (size_t)slots * H / 2;                          // [slots][H/16] e4m3
    uint8_t* a4 = reinterpret_cast<uint8_t*>(p.a_perm);               // [slots][I/2]
    uint8_t* as = a4 + (size_t)slots * I / 2;                          // [slots][I/16]
    {
        k_x_fp4_perm<<<(T + 7) / 8, 256, 0, st>>>((const __nv_bfloat16*)p.x, p.inv, T, H, k, ex.g_x, xc, xs,
                                                   (long long)slots, p.w, p.w_perm);
    }
    // ---- gate / up
    Fp4BMaps mb;
    BMaps m_shared;
    if (!make_fp4_bmaps(&mb, xc, (uint64_t)slots, H) ||
        !make_bmaps(&m_shared, p.x, (uint64_t)T, (uint64_t)H))
        return cudaErrorInvalidValue;
    GemmArgs g{};
    g.quant = ex.quant;
    g.sh0 = ex.sh_gate;
    g.sh1 = ex.sh_up;
    g.perm = p.perm;
    g.tiles = p.tiles;
    g.num_tiles = p.num_tiles;
    g.groups = p.groups;
    g.K = H;
    g.k_top = k;
    g.n_rows = I;
    g.out_ld = I;
    g.out_sh = p.a_sh;
    g.out4 = a4;
    g.out_sf = as;
    g.g_w = ex.g_gate;
    g.g_act = ex.g_x;
    g.g_req = ex.g_a;
    g.err = p.err;
    g.wimg = p.fp4_img[0];
    g.sfb = xs;
    g.sfb_rows = (long long)slots;
    g.sfb_rows_out = (long long)slots;
    if (p.ev_gu0) cudaEventRecord(p.ev_gu0, st);
    OMaps mo;                         // the down GEMM's output maps (unused by gate/up)
    memset(&mo, 0, sizeof(mo));
    cudaError_t err = launch_fp4<0>(mb, mo, g, st);
    if (err == cudaSuccess && p.ev_gu_r) cudaEventRecord(p.ev_gu_r, st);
    if (err == cudaSuccess && has_sh) err = launch_gemm<0, true>(m_shared, g, st);
    if (err != cudaSuccess) return err;
    if (p.ev_gu1) cudaEventRecord(p.ev_gu1, st);
    // ---- down
    if (!make_fp4_bmaps(&mb, a4, (uint64_t)slots, I) ||
        !make_bmaps(&m_shared, p.a_sh, (uint64_t)T, (uint64_t)I))
        return cudaErrorInvalidValue;
    g.wimg = p.fp4_img[1];
    g.sfb = as;
    g.tiles = p.tiles + p.tile_cap;          // the down list
    g.groups = p.groups + p.tile_cap;
    g.num_tiles = p.num_tiles + 4;
    g.sh0 = ex.sh_down;
    g.sh1 = nullptr;
    g.K = I;
    g.n_rows = H;
    g.out_ld = H;
    g.out_sh = nullptr;
    g.o16 = p.o;
    g.o16_sh = p.o_sh;
    g.topk_w = p.w;
    g.w_perm = p.w_perm;
    g.g_w = ex.g_down;
    g.g_act = ex.g_a;
    if (p.ev_dn0) cudaEventRecord(p.ev_dn0, st);
    OMaps mo_sh;
    if (!make_omaps(&mo, p.o, (uint64_t)slots, (uint64_t)H) ||
        (has_sh && !make_omaps(&mo_sh, p.o_sh, (uint64_t)T, (uint64_t)H)))
        return cudaErrorInvalidValue;
    err = launch_fp4<1>(mb, mo, g, st);
    if (err == cudaSuccess && p.ev_dn_r) cudaEventRecord(p.ev_dn_r, st);
    if (err == cudaSuccess && has_sh) err = launch_gemm<1, true>(m_shared, g, st, nullptr, 0, &mo_sh);
    if (err != cudaSuccess) return err;
    if (p.ev_dn1) cudaEventRecord(p.ev_dn1, st);
    const long long threads = (long long)T * (H / 8);
    k_combine<kCombineBatch><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(p.o, has_sh ? p.o_sh : nullptr, p.inv, T, H, k,
                                                               (__nv_bfloat16*)p.y);
    return cudaGetLastError();
}

cudaError_t launch_prefill(const PrefillArgs& p, cudaStream_t st) {
    const ExpertArgs& ex = p.ex;
    const int T = p.T, k = ex.k, H = ex.H, I = ex.I, E = ex.E;
    const int slots = T * k;
    const bool fp4 = ex.quant == Q_NVFP4;
    // NVFP4 W4A4 on the block-scaled tensor cores when the shapes allow
    // 256-value stages (else the exact bf16 dequantization path below)
    const bool native = fp4 && p.fp4_img[0] && p.fp4_img[1] && prefill_native_fp4(H, I);
    // the permutation launch also builds both tile lists (gate/up: I / 128
    // row blocks, down: H / 128)
    TileListArgs tl{};
    tl.tiles = p.tiles;
    tl.groups = p.groups;
    tl.num_tiles = p.num_tiles;
    tl.cap = p.tile_cap;
    tl.T = T;
    tl.RB0 = I / kBlkN;
    tl.RB1 = H / kBlkN;
    tl.has_shared = ex.sh_gate != nullptr ? 1 : 0;
    tl.tok0 = native ? kFp4GuN : kBN;        // the block-scaled GEMMs take wider tiles
    tl.tok1 = native ? kFp4GuN : kBN;
    tl.tok_sh = Cfg<0, true>::TN;            // the shared expert's launches
    tl.grid = num_sms();
    cudaError_t err = launch_permute(p.ids, T, k, E, p.counts, p.offsets, p.perm, p.inv, p.perm_scratch, st, &tl);
    if (err != cudaSuccess) return err;
    if (native) return launch_prefill_fp4(p, st);
    const __nv_bfloat16* xin = nullptr;
    CUtensorMapDataType xdt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (fp4) {
        const long long nblk = (long long)T * (H / kFp4Blk);
        k_act_fp4_values<<<(unsigned)((nblk + 255) / 256), 256, 0, st>>>((const __nv_bfloat16*)p.x, T, H, ex.g_x,
                                                                         p.xq);
        xin = p.xq;
        const long long n8 = (long long)slots * (H / 8);
        const PermMeta meta{p.w, nullptr, p.w_perm, p.ts_perm};
        k_gather_rows<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(xin, p.perm, slots, H, k, p.xp, meta);
    } else {
        // fp16 scaling and the permuted copy in one pass over x
        k_x_to_f16_perm<<<(T + 7) / 8, 256, 0, st>>>((const __nv_bfloat16*)p.x, p.inv, T, H, k,
                                                      reinterpret_cast<__half*>(p.xp), p.tok_scale, p.w, p.w_perm,
                                                      p.ts_perm);
        xdt = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    }
    const bool has_sh = ex.sh_gate != nullptr;
    BMaps m_routed, m_shared;
    // ---- gate / up
    if (!make_bmaps(&m_routed, p.xp, (uint64_t)slots, (uint64_t)H, xdt) ||
        !make_bmaps(&m_shared, p.x, (uint64_t)T, (uint64_t)H))
        return cudaErrorInvalidValue;
    GemmArgs g{};
    g.quant = ex.quant;
    g.w0 = ex.gate;
    g.w1 = ex.up;
    g.sh0 = ex.sh_gate;
    g.sh1 = ex.sh_up;
    g.perm = p.perm;
    g.tiles = p.tiles;
    g.num_tiles = p.num_tiles;
    g.groups = p.groups;
    g.K = H;
    g.k_top = k;
    g.out_ld = I;
    g.out = p.a_perm;
    g.out_sh = p.a_sh;
    g.g_w = fp4 ? ex.g_gate : nullptr;
    g.g_act = fp4 ? ex.g_x : 1.0f;
    g.g_req = ex.g_a;
    g.tok_scale = fp4 ? nullptr : p.tok_scale;
    g.ts_perm = fp4 ? nullptr : p.ts_perm;
    g.err = p.err;
    if (p.ev_gu0) cudaEventRecord(p.ev_gu0, st);
    err = launch_gemm<0, false>(m_routed, g, st);
    if (err == cudaSuccess && p.ev_gu_r) cudaEventRecord(p.ev_gu_r, st);
    if (err == cudaSuccess && has_sh) err = launch_gemm<0, true>(m_shared, g, st);
    if (err != cudaSuccess) return err;
    if (p.ev_gu1) cudaEventRecord(p.ev_gu1, st);
    // ---- down
    if (!make_bmaps(&m_routed, p.a_perm, (uint64_t)slots, (uint64_t)I, xdt) ||
        !make_bmaps(&m_shared, p.a_sh, (uint64_t)T, (uint64_t)I))
        return cudaErrorInvalidValue;
    g.tiles = p.tiles + p.tile_cap;          // the down list
    g.groups = p.groups + p.tile_cap;
    g.num_tiles = p.num_tiles + 4;
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
    g.w_perm = p.w_perm;
    g.g_w = fp4 ? ex.g_down : nullptr;
    g.g_act = fp4 ? ex.g_a : 1.0f;
    g.tok_scale = nullptr;
    g.ts_perm = nullptr;
    OMaps mo, mo_sh;
    if (!make_omaps(&mo, p.o, (uint64_t)slots, (uint64_t)H) ||
        (has_sh && !make_omaps(&mo_sh, p.o_sh, (uint64_t)T, (uint64_t)H)))
        return cudaErrorInvalidValue;
    if (p.ev_dn0) cudaEventRecord(p.ev_dn0, st);
    err = launch_gemm<1, false>(m_routed, g, st, nullptr, 0, &mo);
    if (err == cudaSuccess && p.ev_dn_r) cudaEventRecord(p.ev_dn_r, st);
    if (err == cudaSuccess && has_sh) err = launch_gemm<1, true>(m_shared, g, st, nullptr, 0, &mo_sh);
    if (err != cudaSuccess) return err;
    if (p.ev_dn1) cudaEventRecord(p.ev_dn1, st);
    // ---- combine
    const long long threads = (long long)T * (H / 8);
    k_combine<kCombineBatch><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(p.o, has_sh ? p.o_sh : nullptr, p.inv, T, H, k,
                                                               (__nv_bfloat16*)p.y);
    return cudaGetLastError();
}

}  // namespace moe
