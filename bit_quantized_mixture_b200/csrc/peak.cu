// Tensor-core throughput loops: the peak against which the block-scaled
// NVFP4 GEMM's tensor-pipe fraction is reported, measured on the device
// itself rather than taken as a nominal ratio to the bf16 peak.
//
// One CTA per SM.  Each issuing warp's elected lane issues `iters` MMAs
// back to back into its own TMEM accumulator from operand tiles resident in
// shared memory (filled with a hash of the index, so the data toggles as in
// real work), then commits to an mbarrier and waits (bounded) for them.
//   kind 0: tcgen05.mma kind::f16, bf16 A/B, M = 128, N = 256, K = 16
//   kind 1: tcgen05.mma kind::mxf4nvf4.block_scale.block16, e2m1 A/B with
//           e4m3 scales (all 1.0) in TMEM, M = 128, N = 128, K = 64
#include "../../include/moe_b200.h"
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace moe {

using namespace sm100;

constexpr int kPeakThreads = 128;
// A 16 KB and B up to 32 KB (the rest only keeps a second CTA off the SM, so
// that each SM runs exactly one loop and one TMEM allocation)
constexpr int kPeakSmem = 120 * 1024;

__host__ __device__ constexpr int peak_n(int kind) { return kind == 0 ? 256 : 128; }
__host__ __device__ constexpr int peak_k(int kind) { return kind == 0 ? 16 : 64; }

MOE_DEV uint32_t mix32(uint32_t x) {
    x ^= x >> 16;
    x *= 0x7feb352du;
    x ^= x >> 15;
    x *= 0x846ca68bu;
    x ^= x >> 16;
    return x;
}

template <int KIND>
__global__ void __launch_bounds__(kPeakThreads, 1) k_mma_peak(long long iters, int issuers, int* err) {
    constexpr int N = peak_n(KIND);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* A = smem;                   // 128 rows x 128 bytes
    uint8_t* B = smem + 16384;           // N rows x 128 bytes
    __shared__ uint64_t done[4];
    __shared__ uint32_t tmem_slot;
    __shared__ volatile int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // operands: bf16 values in (-1, 1) with random mantissas / random e2m1 codes
    const int words = (16384 + N * 128) / 4;
    for (int i = threadIdx.x; i < words; i += kPeakThreads) {
        uint32_t h = mix32((uint32_t)i * 2654435761u + blockIdx.x);
        if (KIND == 0) h = (h & 0x807F807Fu) | 0x3E803E80u;    // sign, mantissa random; exponent 2^-2
        reinterpret_cast<uint32_t*>(smem)[i] = h;
    }
    fence_proxy_async_smem();            // the tensor core reads what these threads wrote
    if (threadIdx.x == 0) {
        for (int w = 0; w < 4; ++w) mbar_init(&done[w], 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(&tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    // accumulators: issuer w at column w * N; kind 1: scale factors (e4m3
    // 1.0 everywhere) in the 16 columns after the accumulators
    const uint32_t sf_col = (uint32_t)(issuers * N);
    if (KIND == 1) {
        uint32_t v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0x38383838u;
        tmem_st16(tmem + ((uint32_t)(warp * 32) << 16) + sf_col, v);
        tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp < issuers) {
        if (lane == 0) {
            const uint64_t adesc = desc_kmajor_sw128(smem_u32(A));
            const uint64_t bdesc = desc_kmajor_sw128(smem_u32(B));
            const uint32_t d = tmem + (uint32_t)(warp * N);
            for (long long i = 0; i < iters; ++i) {
                const int kk = (int)(i & 3);
                if constexpr (KIND == 0)
                    mma_bf16(d, adesc + 2 * kk, bdesc + 2 * kk, idesc_bf16_f32(128, N), i != 0);
                else
                    mma_fp4_block16(d, adesc + 2 * kk, bdesc + 2 * kk, idesc_nvfp4(128, N), tmem + sf_col + kk * 4,
                                    tmem + sf_col + kk * 4, i != 0);
            }
            mma_commit(&done[warp]);
        }
        __syncwarp();
        mbar_wait(&done[warp], 0, &abort_flag, err, 30);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_mma_peak_loop(int32_t kind, int32_t issuers, int64_t iters, int32_t* err_dev,
                                        double* flops_out, moe_stream_t stream) {
    if ((kind != 0 && kind != 1) || iters < 1 || !err_dev || !flops_out) {
        set_thread_error("moe_mma_peak_loop: kind must be 0 or 1, iters >= 1, pointers non-null");
        return MOE_ERR_INVALID_ARG;
    }
    const int max_issuers = kind == 0 ? 2 : 3;      // accumulators (+ scale columns) within 512 TMEM columns
    if (issuers < 1 || issuers > max_issuers) {
        set_thread_error("moe_mma_peak_loop: issuers outside 1..2 (kind 0) or 1..3 (kind 1)");
        return MOE_ERR_INVALID_ARG;
    }
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
        return MOE_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e;
    if (kind == 0) {
        e = cudaFuncSetAttribute(k_mma_peak<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPeakSmem);
        if (e == cudaSuccess) k_mma_peak<0><<<sms, kPeakThreads, kPeakSmem, st>>>(iters, issuers, err_dev);
    } else {
        e = cudaFuncSetAttribute(k_mma_peak<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPeakSmem);
        if (e == cudaSuccess) k_mma_peak<1><<<sms, kPeakThreads, kPeakSmem, st>>>(iters, issuers, err_dev);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_thread_error(cudaGetErrorString(e));
        return MOE_ERR_CUDA;
    }
    *flops_out = 2.0 * 128.0 * peak_n(kind) * peak_k(kind) * (double)iters * issuers * sms;
    return MOE_OK;
}
