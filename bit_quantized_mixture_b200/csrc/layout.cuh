// Device layout of the expert weights held in a layer's arena.
//
// Every matrix W [N, K] is cut into blocks of 128 rows x 64 columns
// (nb = N/128 row blocks, kb = K/64 column blocks), stored block after block
// (row block major).  Inside a block the packed codes of one row occupy
// 32 bytes (INT4, NVFP4), 16 bytes (INT2) or 128 bytes (bf16):
//
//   INT4 / NVFP4 / INT2 : [16-byte chunk c][row r (128)][16 bytes]
//       so 32 consecutive rows of one chunk are 512 contiguous bytes (one
//       coalesced warp load).  Inside each 32-bit word the codes of eight
//       (INT4/NVFP4) or sixteen (INT2) consecutive columns are stored in the
//       order that lets one shift-and-mask pull out two neighbouring columns
//       into the two 16-bit halves of a register:
//         INT4  nibble p of the word holds column 2*(p%4) + p/4
//         INT2  crumb  p of the word holds column 2*(p%8) + p/8
//       Chunk c of an INT4/NVFP4 row covers columns [32c, 32c+32); word w of
//       a chunk covers [8w, 8w+8) (INT4) or [16w, 16w+16) (INT2, one chunk).
//   FP8  : [16-byte chunk q (4)][row r (128)][16 bytes]: chunk q of a row
//       holds the E4M3 codes of columns [16q, 16q+16) in natural order.
//   FP6  : two planes.  Low plane (4096 bytes): bits 0-3 of every e2m3 code
//       exactly as the INT4 nibbles.  High plane (2048 bytes): bits 4-5 as
//       [chunk c][row r][4 x 16 bits]: 16-bit word w of (c, r) holds, at
//       bits 2p..2p+1, the high bits of the column whose low bits are
//       nibble p of INT4 word w.
//   bf16 : the 16 KB image of a 128x64 K-major tile in the 128-byte swizzle
//       the tensor cores read: row r, 16-byte chunk c (columns 8c..8c+7) at
//       byte (r/8)*1024 + (r%8)*128 + ((c ^ (r%8)) * 16).
//
// Scales (INT4/INT2): fp16 [nb][K/g][128 rows] with g the group size (128;
// 32 for INT4 group 32); zeros (INT2): uint8, one zero per byte,
// [nb][K/128][128]; FP8 block scales: fp32 [nb][align4(K/128)] (one per
// 128x128 block, rows padded to 16 bytes); NVFP4 block scales: E4M3 bytes
// [nb][kb][128 rows][4] (the four 16-column blocks of the 64-column block).
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace moe {

constexpr int kBlkN = 128;      // rows per block
constexpr int kBlkK = 64;       // columns per block
constexpr int kGroup = 128;     // INT4/INT2 quantization group
constexpr int kGroup32 = 32;    // INT4 group-32 quantization group
constexpr int kFp4Blk = 16;     // NVFP4 scale block

// Q_INT4G32: INT4 symmetric with one fp16 scale per 32 inputs; codes exactly
// as Q_INT4 (one 32-column chunk of a block = one group)
// Q_FP8: E4M3 codes with one fp32 scale per 128x128 block; Q_FP6: e2m3
// codes with one fp16 scale per 32 inputs (scales as Q_INT4G32)
enum Quant : int { Q_INT4 = 0, Q_INT2 = 1, Q_NVFP4 = 2, Q_BF16 = 3, Q_INT4G32 = 4, Q_FP8 = 5, Q_FP6 = 6 };

__host__ __device__ constexpr bool is_int4(int q) { return q == Q_INT4 || q == Q_INT4G32; }
__host__ __device__ constexpr int group_size(int q) { return (q == Q_INT4G32 || q == Q_FP6) ? kGroup32 : kGroup; }
// scale entries per row (INT4/INT2: per weight row; FP8: per 128-row block,
// padded to a multiple of four) in the device layout
__host__ __device__ constexpr int scale_stride(int q, int K) {
    return q == Q_FP8 ? (((K / 128) + 3) & ~3) : K / group_size(q);
}

__host__ __device__ constexpr int row_bytes_per_kblock(int q) {
    return q == Q_INT2 ? 16 : (q == Q_BF16 ? 128 : (q == Q_FP8 ? 64 : (q == Q_FP6 ? 48 : 32)));
}

struct MatGeom {
    int N = 0, K = 0, quant = 0;
    __host__ __device__ int nb() const { return N / kBlkN; }
    __host__ __device__ int kbs() const { return K / kBlkK; }
    __host__ __device__ int groups() const { return K / group_size(quant); }
    __host__ __device__ size_t block_bytes() const { return (size_t)kBlkN * row_bytes_per_kblock(quant); }
    __host__ __device__ size_t codes_bytes() const { return (size_t)nb() * kbs() * block_bytes(); }
    __host__ __device__ size_t scales_bytes() const {
        if (is_int4(quant) || quant == Q_INT2 || quant == Q_FP6) return (size_t)N * groups() * 2;
        if (quant == Q_NVFP4) return (size_t)N * (K / kFp4Blk);
        if (quant == Q_FP8) return (size_t)nb() * fp8_scale_stride() * 4;
        return 0;
    }
    // FP8: fp32 scales per row block, padded to a multiple of four
    __host__ __device__ int fp8_scale_stride() const { return ((K / 128) + 3) & ~3; }
    __host__ __device__ size_t zeros_bytes() const { return quant == Q_INT2 ? (size_t)N * groups() : 0; }
};

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// One matrix kind (gate, up or down) of every routed expert.
struct MatView {
    const uint8_t* codes;   // expert e at codes + e * stride
    const uint8_t* scales;  // expert e at scales + e * stride
    const uint8_t* zeros;   // expert e at zeros + e * stride (INT2)
    size_t stride;          // bytes between consecutive experts
    // per-expert address table: when set, expert e's block (all three
    // matrices, the arena's per-expert layout) starts at table[e] and this
    // matrix's codes / scales / zeros lie at the offsets below inside it
    const uint8_t* const* table;
    size_t off_codes, off_scales, off_zeros;
    int N, K;
};

// codes / scales / zeros (null when absent) of expert e
struct ExpertMat {
    const uint8_t* codes;
    const uint8_t* scales;
    const uint8_t* zeros;
};
__host__ __device__ inline ExpertMat expert_matrix(const MatView& v, int e) {
    ExpertMat m;
    if (v.table) {
        const uint8_t* b = v.table[e];
        m.codes = b + v.off_codes;
        m.scales = v.scales ? b + v.off_scales : nullptr;
        m.zeros = v.zeros ? b + v.off_zeros : nullptr;
    } else {
        m.codes = v.codes + (size_t)e * v.stride;
        m.scales = v.scales ? v.scales + (size_t)e * v.stride : nullptr;
        m.zeros = v.zeros ? v.zeros + (size_t)e * v.stride : nullptr;
    }
    return m;
}

// byte offset of block (rb, kb) inside the codes of one matrix
__host__ __device__ inline size_t block_offset(const MatGeom& g, int rb, int kb) {
    return ((size_t)rb * g.kbs() + kb) * g.block_bytes();
}

}  // namespace moe
