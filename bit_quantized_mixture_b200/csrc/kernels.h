// Host-side launchers of the MoE kernels (internal to the library).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "layout.cuh"

namespace moe {

// quantize.cu
cudaError_t launch_quantize(int quant, const float* w, int N, int K, float g, void* codes, void* scales,
                            void* zeros, cudaStream_t st);
cudaError_t launch_quantize_act_nvfp4(const void* x, int T, int K, float g, void* codes, void* scales,
                                      cudaStream_t st);
cudaError_t launch_absmax(const float* x, long long n, float* out, cudaStream_t st);
// g[e] = gate/up and g[E + e] = down global scale read from each table block at offset off
cudaError_t launch_gather_global_scales(const uint8_t* const* table, size_t off, int E, float* g, cudaStream_t st);
// NVFP4 block-scaled GEMM weight image (see k_fp4_block_image): one matrix of
// one expert into slot `slot` of its nmat-matrix blocks (N % 128 == 0, K % 256 == 0)
cudaError_t launch_fp4_block_image(const uint8_t* codes, const uint8_t* scales, int N, int K, int slot, int nmat,
                                   uint8_t* dst, cudaStream_t st);
// bytes of one expert's image of nmat matrices of N rows and K columns
inline size_t fp4_block_image_bytes(int N, int K, int nmat) {
    return (size_t)(N / 128) * (K / 256) * nmat * (16384 + 2048);
}
cudaError_t launch_relayout(const MatGeom& gm, const uint8_t* src_codes, const uint8_t* src_scales,
                            const uint8_t* src_zeros, uint8_t* dst_codes, uint8_t* dst_scales,
                            uint8_t* dst_zeros, cudaStream_t st);
cudaError_t launch_unpack(const MatGeom& gm, const uint8_t* dev_codes, const uint8_t* dev_scales,
                          const uint8_t* dev_zeros, uint8_t* codes, uint8_t* scales, uint8_t* zeros,
                          cudaStream_t st);

// route.cu
struct RouteArgs {
    const void* x;          // bf16 [T, H]
    const void* wr;         // bf16 [E, H]
    const float* logits_in; // fp32 [T, E] (route from logits) or null
    float* logits;          // fp32 [T, E] workspace or caller buffer
    int32_t* ids;           // [T, k]
    float* w;               // [T, k]
    unsigned int* counter;  // zero-initialised grid counter (decode router)
    int* err;               // device error word (bounded waits of the tensor-core router)
    int T, H, E, k;
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t st);
// grouped_gemm.cu: router logits on the tensor cores (any T, E; H % 64 == 0)
cudaError_t launch_router_tc(const void* x, const void* wr, int T, int H, int E, float* logits, int* err,
                             cudaStream_t st);

// moe_api.cu: text returned by moe_last_error(NULL) on this host thread
void set_thread_error(const char* msg);

// permute.cu
// One tile of a grouped GEMM: (expert, 128-row weight block, up to 128
// consecutive permuted positions).
struct GemmTile {
    int expert;   // routed expert, or -1 for the shared expert
    int rb;       // 128-row block of the weight matrix
    int seg;      // first row of the segment (permuted position, or token for shared)
    int count;    // tokens in this tile
};
// The grouped GEMMs' tile lists, built by the permutation launch from the
// expert counts it computes: list 0 (gate/up, RB0 row blocks) and list 1
// (down, RB1 row blocks), each of cap entries with its group list and four
// counts (routed tiles, all tiles, routed groups, group order).
struct TileListArgs {
    GemmTile* tiles;               // [2][cap]
    int2* groups;                  // [2][cap]
    int* num_tiles;                // [2][4]
    size_t cap;
    int T, RB0, RB1, has_shared;
    int tok0, tok1;                // tokens per routed tile of each list
    int tok_sh;                    // tokens per shared-expert tile
    int grid;                      // CTAs of the GEMM launches
};
// tl may be null (permutation only)
cudaError_t launch_permute(const int32_t* ids, int T, int k, int E, int32_t* counts, int32_t* offsets,
                           int32_t* perm, int32_t* inv, int32_t* chunk_scratch, cudaStream_t st,
                           const TileListArgs* tl = nullptr);
size_t permute_scratch_ints(int slots, int E);

// decode.cu (small-T path) and segment path
struct ExpertArgs {
    MatView gate, up, down;        // routed experts (device layout)
    const uint8_t* sh_gate;        // shared expert bf16 device layout, or null
    const uint8_t* sh_up;
    const uint8_t* sh_down;
    const float* g_gate;           // NVFP4 per-expert global scales, [E]
    const float* g_down;
    float g_x, g_a;                // NVFP4 activation global scales
    int quant, H, I, E, k;
};
struct DecodeArgs {
    ExpertArgs ex;
    const void* x;                 // bf16 [T, H]
    const int32_t* ids;            // [T, k]
    const float* w;                // [T, k]
    void* y;                       // bf16 [T, H]
    float* a;                      // workspace fp32 [T*k, I]
    float* a_sh;                   // workspace fp32 [T, I]
    float* part;                   // workspace fp32 [T*k, H]
    float* part_sh;                // workspace fp32 [T, H]
    unsigned int* counters;        // workspace, H/16 zero-initialised counters
    int T;
    cudaEvent_t ev_mid;            // optional: recorded between the two kernels
};
bool decode_supported(int T, int k);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st);

// decode_fused.cu: the whole decode step in one cooperative kernel
struct FusedArgs {
    DecodeArgs d;                  // ids / w are inputs when wr is null
    const void* wr;                // bf16 [E, H] router, or null
    float* logits;                 // workspace [T, E]
    int32_t* ids_out;              // [T, k] (when wr is set)
    float* w_out;                  // [T, k]
    unsigned long long* bar;       // workspace: monotonically increasing arrival count, zero-initialised
    float* gu_sh;                  // workspace [4][T][2 * I]: partial shared gate/up sums by K part
    int* err;                      // device error word
    // test hook of the bounded grid-barrier waits: CTA withhold_cta (>= 0)
    // skips its arrival at the first grid barrier; wait_limit (> 0) replaces
    // the default limit of the waits, in SM clock cycles
    int withhold_cta = -1;
    long long wait_limit = 0;
};
size_t fused_smem_bytes(int H, int I);
cudaError_t launch_decode_fused(const FusedArgs& f, cudaStream_t st);   // cudaErrorNotSupported: shapes too large
bool fused_supported(int T, int H, int I, int quant);

// grouped_gemm.cu (prefill path)
struct PrefillArgs {
    ExpertArgs ex;
    const void* x;                 // bf16 [T, H]
    const int32_t* ids;            // [T, k]
    const float* w;                // [T, k]
    void* y;                       // bf16 [T, H]
    int T;
    int32_t *counts, *offsets, *perm, *inv, *perm_scratch;
    GemmTile* tiles;               // two lists of tile_cap entries: gate/up, then down
    int2* groups;                  // routed tile groups (same layout as tiles)
    int* num_tiles;                // 4 ints per list
    size_t tile_cap;               // entries per list (prefill_tile_capacity)
    __nv_bfloat16* xq;             // [T, H]: NVFP4 W4A4 activation values, else fp16 scaled x
    float* tok_scale;              // [T]: power of two of each token's fp16 activations
    __nv_bfloat16* xp;             // [T*k, H]: rows of xq in permuted (expert-major) order
    float* w_perm;                 // [T*k]: routing weight of each permuted position
    float* ts_perm;                // [T*k]: token scale of each permuted position (INT4/INT2)
    // NVFP4: block-scaled GEMM weight images (k_fp4_block_image), gate/up
    // (two matrices per block) and down, or null
    const uint8_t* fp4_img[2];
    __nv_bfloat16* a_perm;         // [T*k, I] intermediate in permuted order
    __nv_bfloat16* a_sh;           // [T, I] shared-expert intermediate
    __half* o;                     // [T*k, H] weighted expert outputs by slot (fp16)
    __half* o_sh;                  // [T, H] shared-expert output (fp16)
    int* err;                      // device error word (bounded waits)
    // profiling events (may be null): before / after the gate-up grouped
    // GEMM, before / after the down grouped GEMM
    cudaEvent_t ev_gu0, ev_gu1, ev_dn0, ev_dn1;
    // after the routed gate/up and the routed down launch (before the
    // shared-expert launch of each)
    cudaEvent_t ev_gu_r, ev_dn_r;
};
size_t prefill_tile_capacity(int max_tokens, int k, int E, int H, int I);
// NVFP4 prefill runs on the block-scaled tensor cores when H and I allow
// 256-value stages (else the exact bf16 dequantization path)
bool prefill_native_fp4(int H, int I);
cudaError_t launch_prefill(const PrefillArgs& p, cudaStream_t st);

}  // namespace moe
