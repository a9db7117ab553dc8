// moe_permute_noalloc: the token permutation without any device allocation.
//
// moe_permute takes its per-chunk histogram scratch from the stream-ordered
// allocator.  Some callers cannot allocate device memory at call time: a
// runtime that reserves its whole memory budget at start-up and forbids later
// allocations, a host framework whose caching pool already owns the device
// memory (a stray allocation fails or fragments it), or a latency-critical
// path that must not risk the implicit synchronisation of cudaMalloc and
// cudaFree.  This variant runs the same three kernels with its scratch in a
// file-scope device array instead; the caller still passes every input and
// output.
//
// The array is a module global: every GPU that loads the library holds it
// until the process exits, and all calls on one device share it.
#include <stdio.h>

#include <mutex>

#include "../../include/moe_b200.h"
#include "kernels.h"

namespace {

constexpr int kChunkSlots = 1024;                  // slots per histogram chunk (permute.cu)
constexpr int kNoAllocMaxSlots = 1 << 18;          // largest T * k accepted (262,144)
constexpr int kNoAllocMaxExperts = 1024;           // largest E accepted
constexpr int kMaxDevices = 64;

// one int per (chunk, expert): 256 chunks x 1024 experts = 1 MiB
static __device__ __align__(256) int32_t g_permute_scratch[(kNoAllocMaxSlots / kChunkSlots) * kNoAllocMaxExperts];

std::mutex g_mu;
int32_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The host-side
// symbol is only a stand-in; the address is looked up once per device.
cudaError_t scratch_address(int32_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_permute_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = static_cast<int32_t*>(p);
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

// the message is reported by moe_last_error(NULL) on this host thread
moe_status noalloc_fail(moe_status s, const char* msg) {
    moe::set_thread_error(msg);
    return s;
}

}  // namespace

extern "C" moe_status moe_permute_noalloc(const int32_t* topk_ids, int32_t T, int32_t k, int32_t E, int32_t* counts,
                                          int32_t* offsets, int32_t* perm, int32_t* inv, moe_stream_t stream) {
    if (!topk_ids || !counts || !offsets || !perm || !inv)
        return noalloc_fail(MOE_ERR_INVALID_ARG, "moe_permute_noalloc: null pointer");
    if (T <= 0 || k <= 0 || E <= 0)
        return noalloc_fail(MOE_ERR_INVALID_ARG, "moe_permute_noalloc: sizes must be positive");
    if ((int64_t)T * k > kNoAllocMaxSlots)
        return noalloc_fail(MOE_ERR_INVALID_ARG,
                            "moe_permute_noalloc: T*k exceeds the static scratch limit of 262144 slots");
    if (E > kNoAllocMaxExperts)
        return noalloc_fail(MOE_ERR_INVALID_ARG, "moe_permute_noalloc: E exceeds the limit of 1024 experts");
    int32_t* scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) return noalloc_fail(MOE_ERR_CUDA, "moe_permute_noalloc: cannot resolve the scratch address");
    // every entry the scan and scatter read is written by the histogram pass
    // of the same call, so the array needs no clearing between calls
    e = moe::launch_permute(topk_ids, T, k, E, counts, offsets, perm, inv, scratch, (cudaStream_t)stream);
    if (e != cudaSuccess) return noalloc_fail(MOE_ERR_CUDA, "moe_permute_noalloc: launch failed");
    return MOE_OK;
}
