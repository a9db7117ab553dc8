/*
 * moe_b200.h - C ABI of the B200 (sm_100a) routed-expert MoE layer.
 *
 * The layer is the mixture-of-experts block of a sparse MoE LLM whose routed
 * experts are stored with low-bit group quantization:
 *   1. router logits x Wr^T (bf16 router, fp32 logits), softmax and top-k
 *      with the k weights renormalised to sum to one
 *      ("Qwen3.8-Flash-Next on one 24 GB GPU", "What the patch does": ten of
 *      512 experts per token; "Qwen3.8-Flash-Next-FP6-INT8", "Precision map":
 *      routers stay bf16);
 *   2. token-to-expert permutation;
 *   3. each selected expert's SwiGLU MLP a = silu(x Wg^T) * (x Wu^T),
 *      o = a Wd^T, with dequantization fused into the products, in three
 *      weight formats: INT4 symmetric group-128 W4A16
 *      ("albucino/Qwen3.8-Flash-Next-W4A16-FP8PLE", "Composition"), INT2
 *      group-128 with fp16 scale and 2-bit zero ("Qwen3.8-Flash-Next on one
 *      24 GB GPU", "Hardware and software requirements"), and NVFP4 W4A4
 *      E2M1 with one E4M3 scale per 16 elements
 *      ("meshapplied/Qwen3.8-Flash-Next-NVFP4-Latest", "Format");
 *   4. y_t = sum_j w_tj o_tj + shared(x_t), the bf16 shared expert added
 *      with weight one (same NVFP4 card, "Format": shared experts stay BF16).
 *
 * Conventions for every entry point
 *   - Pointers named *_dev are device pointers of the handle's device.
 *     Pointers named *_any may be host or device memory (copied with
 *     cudaMemcpyDefault).  All other data pointers are device pointers; the
 *     device address of mapped pinned host memory (cudaHostAllocMapped,
 *     cudaHostGetDevicePointer) is one too, and the kernels then read or
 *     write host memory across the bus (worth it for the few kilobytes of a
 *     decode step's y, not for operands that many CTAs read).
 *   - All calls are asynchronous on the given stream unless stated.
 *     Argument and state errors are detected on the host before any work is
 *     enqueued and return without side effects.  A failed launch returns
 *     MOE_ERR_CUDA; moe_last_error() gives the text.
 *   - A handle is not reentrant: calls on one handle must not overlap in
 *     host threads.  Device work of one handle must not overlap in time
 *     (the handle owns one workspace), i.e. use one stream per handle or
 *     order the streams.
 *   - bf16 tensors are row-major, 16-byte aligned, with rows of H (or I)
 *     contiguous elements.
 *
 * Interchange formats (the layout the load and quantize calls exchange).
 * A matrix W is [N, K] (output rows, input columns); groups run along K.
 *   INT4  codes  uint8 [N, K/2]; element k = 2j in the low nibble of byte j;
 *                stored code u = q + 8 with q = clamp(rne(w/s), -8, 7)
 *         scales fp16  [N, K/128]; s = fp16(amax/7)
 *   INT4_G32  as INT4 with scales fp16 [N, K/32] (one scale per 32 inputs)
 *   FP8_B128  codes uint8 [N, K] E4M3FN; scales fp32 [N/128, K/128];
 *             s = amax_block / 448, q = e4m3(w / s); N and K multiples of 128
 *   FP6_E2M3  codes uint8 [N, K], one e2m3 code per byte (bit 5 sign, bits
 *             3-4 exponent with bias 1, bits 0-2 mantissa); scales fp16
 *             [N, K/32]; s = fp16(amax/7.5), q = e2m3(w / s), saturating
 *   INT2  codes  uint8 [N, K/4]; element k = 4j + i at bits 2i..2i+1;
 *                u = clamp(rne(w/s) + z, 0, 3)
 *         scales fp16  [N, K/128]; s = fp16((max - min)/3), min <= 0 <= max
 *         zeros  uint8 [N/4, K/128]; zero of row n at bits 2(n%4) of byte
 *                (n/4, group); z = clamp(rne(-min/s), 0, 3)
 *   NVFP4 codes  uint8 [N, K/2]; low nibble = even k; E2M1 sign-magnitude
 *         scales uint8 [N, K/16]; E4M3FN block scale per 16 elements
 *         global fp32 g per matrix (gate and up share one); w ~ e2m1 * s * g
 *   BF16  codes  bf16 [N, K] (shared expert only)
 * Every rounding is round-half-to-even; every code decision is taken in IEEE
 * fp32.  The library re-lays loaded weights into its own tiled device layout;
 * moe_debug_unpack_matrix() returns them in the interchange layout.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t;   /* same type as cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or index */
    MOE_ERR_UNSUPPORTED = 2,   /* shape or format the library does not handle */
    MOE_ERR_STATE = 3,         /* e.g. forward before the weights are loaded */
    MOE_ERR_OOM = 4,           /* device allocation failed in moe_create     */
    MOE_ERR_CUDA = 5,          /* a CUDA call or launch failed               */
    MOE_ERR_TIMEOUT = 6        /* a bounded device-side wait gave up         */
} moe_status;

typedef enum {
    MOE_Q_INT4 = 0,            /* INT4 symmetric, group 128, fp16 scales (W4A16) */
    MOE_Q_INT2 = 1,            /* INT2 asymmetric, group 128, fp16 scale + 2-bit zero (W2A16) */
    MOE_Q_NVFP4 = 2,           /* E2M1 + E4M3 per-16 scale + fp32 global (W4A4) */
    MOE_Q_BF16 = 3,            /* unquantized bf16 (shared expert) */
    MOE_Q_INT4_G32 = 4,        /* INT4 symmetric, group 32, fp16 scales (the MTP-draft experts of
                                  "Qwen3.8-Flash-Next on 2x RTX 3090", storage-format table) */
    MOE_Q_FP8_B128 = 5,        /* E4M3FN with one fp32 scale per 128x128 block (W8A16; the MTP-draft
                                  experts of "meshapplied/Qwen3.8-Flash-Next-NVFP4-Latest", Format) */
    MOE_Q_FP6_E2M3 = 6         /* FP6 E2M3 with one fp16 scale per 32 inputs (W6A16; the routed experts
                                  of "Qwen3.8-Flash-Next-FP6-INT8") */
} moe_quant;

#define MOE_SHARED_EXPERT (-1)

typedef struct {
    int32_t hidden;        /* H: multiple of 128 */
    int32_t inter;         /* I: multiple of 128 */
    int32_t num_experts;   /* E: 1 .. 1024 */
    int32_t top_k;         /* k: 1 .. min(E, 32) */
    int32_t quant;         /* moe_quant of the routed experts (not BF16) */
    int32_t has_shared;    /* 1: one always-on bf16 shared expert of width I */
    int32_t max_tokens;    /* largest T any call will pass; sizes the workspace */
    int32_t device;        /* CUDA device ordinal */
} moe_config;

typedef struct moe_layer* moe_handle;

/* One quantized matrix in interchange layout (see above). */
typedef struct {
    const void* codes;     /* required */
    const void* scales;    /* INT4/INT2: fp16; NVFP4: E4M3 bytes; BF16: NULL */
    const void* zeros;     /* INT2 only, else NULL */
    float global_scale;    /* NVFP4 only */
} moe_qmatrix;

typedef struct {
    moe_qmatrix gate;      /* [I, H] */
    moe_qmatrix up;        /* [I, H] */
    moe_qmatrix down;      /* [H, I] */
} moe_expert_weights;

/* ------------------------------------------------------------------ setup */

/* Validate cfg, allocate the weight arena and the workspace for max_tokens on
 * cfg->device.  On success *out owns all device memory until moe_destroy.
 * NVFP4 layers whose hidden and inter sizes are multiples of 256 also keep,
 * in the arena, the block-scaled prefill GEMM's weight images: a second copy
 * of the routed experts' codes and scales (the same number of bytes), laid
 * out per 128-row block and 256-value stage.
 * Errors: INVALID_ARG (bad cfg/null), UNSUPPORTED (shape), OOM, CUDA. */
moe_status moe_create(const moe_config* cfg, moe_handle* out);

/* Synchronize the handle's device, free everything; NULL is a no-op. */
moe_status moe_destroy(moe_handle h);

/* Copy the bf16 router matrix Wr [E, H] (host or device) into the arena. */
moe_status moe_load_router(moe_handle h, const void* w_router_any, moe_stream_t stream);

/* Copy one expert's three matrices (host or device, interchange layout) into
 * the arena, re-laid for the kernels (NVFP4: and into the block-scaled weight
 * images described at moe_create).  expert in [0, E) takes the routed
 * format of the handle; MOE_SHARED_EXPERT takes BF16 codes.  The caller may
 * free its arrays once the stream has passed this call.  Errors:
 * INVALID_ARG (index, null codes/scales/zeros for the format). */
moe_status moe_load_expert_weights(moe_handle h, int32_t expert,
                                   const moe_expert_weights* w, moe_stream_t stream);

/* NVFP4 (W4A4) only: the static per-layer fp32 global scales of the input
 * activations (g_x) and of the SwiGLU intermediate (g_a), each amax/(6*448)
 * of a calibration pass. */
moe_status moe_set_act_global_scales(moe_handle h, float g_x, float g_a);

/* ---------------------------------------------------------------- hot path */

/* Router: logits = x Wr^T (fp32), then per token the k largest logits in
 * order (logit descending, expert index ascending on ties) and weights
 * w_j = exp(l_j - l_max) / sum_selected exp(l - l_max).
 *   x          bf16 [T, H]           topk_ids int32 [T, k]
 *   topk_w     fp32 [T, k]           logits_out fp32 [T, E] or NULL
 * topk_ids and topk_w may both be NULL when logits_out is given: only the
 * logits are computed (e.g. when the routing itself comes from elsewhere).
 * 1 <= T <= max_tokens.  Errors: INVALID_ARG, STATE (router not loaded). */
moe_status moe_route(moe_handle h, const void* x, int32_t T, int32_t* topk_ids,
                     float* topk_w, float* logits_out, moe_stream_t stream);

/* The softmax/top-k half of moe_route on caller-supplied fp32 logits [T, E]. */
moe_status moe_route_from_logits(moe_handle h, const float* logits, int32_t T,
                                 int32_t* topk_ids, float* topk_w, moe_stream_t stream);

/* Expert computation and combine:
 *   y_t = sum_{j<k} topk_w[t,j] * Expert_{topk_ids[t,j]}(x_t) + Shared(x_t)
 * x bf16 [T, H] in, y bf16 [T, H] out (single rounding of the fp32 sum).
 * T <= 8 runs the fused decode kernel or the two GEMV kernels as
 * moe_set_decode_path selects; larger T the grouped GEMMs.
 * Every id must lie in [0, E); ids of one token should be distinct.
 * Errors: INVALID_ARG, STATE (experts/shared/scales not loaded). */
moe_status moe_forward(moe_handle h, const void* x, int32_t T, const int32_t* topk_ids,
                       const float* topk_w, void* y, moe_stream_t stream);

/* The whole layer, moe_route followed by moe_forward, as one call: writes
 * topk_ids / topk_w (as moe_route) and y (as moe_forward).  For T <= 8 an
 * eager call runs one cooperative kernel (router, top-k, experts, shared
 * expert and combine, separated by bounded grid-wide barriers) and a call
 * under stream capture runs moe_route then moe_forward (see
 * moe_set_decode_path); larger T, a format or shape the fused kernel does
 * not take, or a refused cooperative launch, runs moe_route then
 * moe_forward.  Errors as those two. */
moe_status moe_route_forward(moe_handle h, const void* x, int32_t T, int32_t* topk_ids,
                             float* topk_w, void* y, moe_stream_t stream);

/* ------------------------------------------------- format kernels (no handle) */

/* Quantize W fp32 [N, K] (device) into interchange layout (device outputs).
 * quant INT4/INT2/NVFP4; global_scale is used for NVFP4 only.
 * INT4/INT2 need K % 128 == 0 (INT2 also N % 4 == 0); NVFP4 K % 16 == 0. */
moe_status moe_quantize(int32_t quant, const float* w, int32_t N, int32_t K, float global_scale,
                        void* codes, void* scales, void* zeros, moe_stream_t stream);

/* *amax_inout_dev = max(*amax_inout_dev, max_i |x_i|) over n fp32 values. */
moe_status moe_absmax(const float* x, int64_t n, float* amax_inout_dev, moe_stream_t stream);

/* NVFP4 global scale of a tensor with the given amax: amax / (6 * 448) in
 * fp32 (host function, no device work). */
float moe_nvfp4_global_scale(float amax);

/* NVFP4 activation quantization of bf16 rows x [T, K] with global scale g:
 * codes uint8 [T, K/2], scales uint8 [T, K/16] (interchange layout). */
moe_status moe_quantize_act_nvfp4(const void* x, int32_t T, int32_t K, float g,
                                  void* codes, void* scales, moe_stream_t stream);

/* Token permutation of the flat slots s = t*k + j into expert-major order,
 * stable in s: counts int32 [E], offsets int32 [E+1], perm int32 [T*k]
 * (slot at each permuted position), inv int32 [T*k] (position of each slot).
 * A slot whose id lies outside [0, E) gets no position: its inv entry is -1,
 * it is not counted, and only the first offsets[E] entries of perm are
 * written.  T*k <= 2^30, 1 <= E <= 1024.  Uses no handle; deterministic. */
moe_status moe_permute(const int32_t* topk_ids, int32_t T, int32_t k, int32_t E,
                       int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                       moe_stream_t stream);

/* moe_permute without any device allocation.  The pages have no counterpart:
 * this entry point exists for callers that cannot allocate device memory at
 * call time - runtimes that reserve their whole budget at start-up, hosts
 * whose caching allocator already owns the device memory, or latency-critical
 * paths that must not risk the implicit synchronisation of cudaMalloc and
 * cudaFree.  Same arguments, outputs and determinism as moe_permute; the
 * per-chunk histogram scratch lives in a file-scope device array of 1 MiB that
 * every GPU loading the library keeps until the process exits.
 * Limits: T*k <= 262144 and E <= 1024, else MOE_ERR_INVALID_ARG (message in
 * moe_last_error(NULL)) before any device work.  The first call on a device
 * looks up the array's device address (with that device current); make that
 * first call before any stream capture.  All calls on a device share the one
 * array: calls whose kernels overlap in time on the GPU (different streams
 * without ordering) race and give wrong results.  Nothing in the array has to
 * start at zero: each call writes every entry it reads. */
moe_status moe_permute_noalloc(const int32_t* topk_ids, int32_t T, int32_t k, int32_t E,
                               int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                               moe_stream_t stream);

/* Path of moe_route_forward and moe_forward for T <= 16 (decode and the
 * few-token verify steps of speculative decoding):
 *   MOE_DECODE_AUTO     (default) T <= 8: the fused cooperative kernel for
 *                       eager calls; inside a stream capture (CUDA graph) the
 *                       router kernel and the two GEMV kernels, which overlap
 *                       through programmatic launch and have no grid
 *                       barriers.  9 <= T <= 16: the grouped-GEMM path (the
 *                       faster one there, measured on the decode-b1 layer)
 *   MOE_DECODE_FUSED    the fused kernel for T <= 8 (where the format fits it)
 *   MOE_DECODE_KERNELS  the router + two GEMV kernels for T <= 16 (two
 *                       8-column MMA groups above 8 tokens)
 *   MOE_DECODE_GEMM     the grouped-GEMM (prefill) path for every T, e.g. to
 *                       find the token count where it overtakes the GEMVs
 * All paths compute the same layer; their fp32 sums may round differently.
 * Errors: INVALID_ARG (unknown path). */
#define MOE_DECODE_AUTO 0
#define MOE_DECODE_FUSED 1
#define MOE_DECODE_KERNELS 2
#define MOE_DECODE_GEMM 3
moe_status moe_set_decode_path(moe_handle h, int32_t path);

/* ------------------------------------------------- expert address table
 *
 * Experts read where they are: after moe_set_expert_table, the kernels read
 * routed expert e's weights from blocks[e] instead of the handle's arena
 * (the arena stays allocated; moe_load_expert_weights keeps writing it).
 * A block holds one expert's three matrices in the library's device layout
 * (NVFP4: and the expert's two fp32 global scales), moe_expert_block_bytes
 * bytes, as moe_export_expert writes it; blocks may
 * lie anywhere in device memory of the handle's device, in any order, and
 * several entries may point at the same block.  Blocks must stay valid and
 * unchanged while calls that read them are in flight. */

/* Bytes of one expert block (a multiple of 256). */
moe_status moe_expert_block_bytes(moe_handle h, size_t* bytes);

/* Copy expert `expert`'s block from the arena to dst (device memory of the
 * handle's device, 256-byte aligned), ordered on `stream`.
 * Errors: INVALID_ARG (null or misaligned dst, expert out of range), CUDA. */
moe_status moe_export_expert(moe_handle h, int32_t expert, void* dst, moe_stream_t stream);

/* blocks: host array of E device addresses (each 256-byte aligned, not
 * null), or NULL to read the arena again.  The call synchronizes `stream`
 * (work already queued keeps the old table), copies the E addresses to the
 * device (NVFP4: and reads each block's global scales on `stream`) and
 * synchronizes again before it returns; the caller's array may be freed then.  With
 * a table, NVFP4 layers run prefill on the exact bf16-dequantization path
 * (their block-scaled weight images stay in the arena).
 * Errors: INVALID_ARG (null or misaligned entry: nothing changes), CUDA. */
moe_status moe_set_expert_table(moe_handle h, const void* const* blocks, moe_stream_t stream);

/* ---------------------------------------------------------------- debug */

/* Write loaded matrix `which` (0 gate, 1 up, 2 down) of `expert` back in
 * interchange layout into device buffers sized as above (NVFP4: the global
 * scale is written to *global_scale_out when non-NULL). */
moe_status moe_debug_unpack_matrix(moe_handle h, int32_t expert, int32_t which,
                                   void* codes, void* scales, void* zeros,
                                   float* global_scale_out, moe_stream_t stream);

/* Copy the token permutation of the last grouped-GEMM forward (T > 8) of this
 * handle: counts [E], offsets [E+1], perm [T*k] (the flat slot s = t*k + j at
 * each expert-major position, ascending s inside an expert) and inv [T*k]
 * (the position of each slot; -1 for a slot whose id lies outside [0, E)).
 * Only the first offsets[E] entries of perm are written by the forward.  The
 * order is the expert-major gather of the selected experts of each token
 * ("Qwen3.8-Flash-Next on one 24 GB GPU", section "What the patch does").
 * Buffers may be host or device memory; the copies are asynchronous on
 * `stream` (synchronize before reading host buffers).
 * Errors: INVALID_ARG (null), STATE (no grouped-GEMM forward yet), CUDA. */
moe_status moe_debug_get_permutation(moe_handle h, int32_t* counts, int32_t* offsets, int32_t* perm,
                                     int32_t* inv, moe_stream_t stream);

/* Copy the W4A4 activation operand of the last block-scaled NVFP4
 * grouped-GEMM forward: in permuted order (position p holds the row of token
 * perm[p] / k), codes [T*k][H/2] (E2M1, even column in the low nibble) and
 * scales [T*k][H/16] (E4M3, one per 16 values), quantized with the static
 * global scale g_x ("meshapplied/Qwen3.8-Flash-Next-NVFP4-Latest", section
 * "Format").  Positions from offsets[E] on are not written by the forward.
 * Buffers host or device, copies asynchronous on `stream`.
 * Errors: INVALID_ARG (null), STATE (no such forward yet), CUDA. */
moe_status moe_debug_get_act_nvfp4(moe_handle h, void* codes, void* scales, moe_stream_t stream);

/* Test hook of the bounded device-side waits (no counterpart on the pages;
 * it exists so that the timeout path can be exercised without a fault): the
 * next launch of the fused decode kernel on this handle (moe_route_forward
 * or moe_forward with T <= 8 outside stream capture) has CTA `withhold_cta`
 * skip its arrival at its first grid barrier, and every grid-barrier wait of
 * that launch gives up after `wait_limit_cycles` SM clock cycles (0: the
 * default limit of about 2 s).  That launch then stops every CTA at the
 * barrier and reports MOE_ERR_TIMEOUT through moe_sync_status, which also
 * resets the barrier so that the next call is correct.  One-shot: the
 * setting applies to one launch and then clears; withhold_cta < 0 clears it.
 * Errors: INVALID_ARG (null handle, negative limit). */
moe_status moe_debug_set_wait_test(moe_handle h, int32_t withhold_cta, int64_t wait_limit_cycles);

/* Profiling aid: when events != NULL, every later call records, on its
 * stream, the events of the slots it has:
 *   [0] before and [1] after the routing kernels of moe_route;
 *   [2] before the expert kernels and [4] after the last kernel of
 *       moe_forward and moe_route_forward (the fused decode kernel takes
 *       [0] and [4] for moe_route_forward);
 *   [3] decode, two-kernel path: between the gate/up and the down kernel;
 *       grouped-GEMM path: after the gate/up grouped GEMM;
 *   [5] / [6] / [7] grouped-GEMM path only: before the gate/up grouped GEMM,
 *       before the down grouped GEMM, after the down grouped GEMM;
 *   [8] / [9] grouped-GEMM path only: after the routed-expert gate/up and
 *       after the routed-expert down launch (before the shared-expert
 *       launch of each, which [3] and [7] close).
 * events are cudaEvent_t handles created by the caller; n >= 5 of them are
 * read (slots n..9 are not recorded); NULL turns recording off.  Recording
 * an event between two kernels removes their launch overlap, so time the
 * layer itself with recording off. */
moe_status moe_set_profile_events(moe_handle h, void* const* events, int32_t n);

/* Measurement aid (no counterpart on the pages): a tensor-core throughput
 * loop on every SM of the current device, the denominator of the tensor-pipe
 * fraction of the grouped GEMMs.  Each CTA (one per SM) has `issuers` warps
 * issue `iters` MMAs each, back to back, from operand tiles resident in
 * shared memory into their own TMEM accumulators:
 *   kind 0: tcgen05.mma kind::f16, bf16 operands, M = 128, N = 256, K = 16
 *           (issuers 1..2);
 *   kind 1: tcgen05.mma kind::mxf4nvf4.block_scale.block16, E2M1 operands
 *           with E4M3 scales, M = 128, N = 128, K = 64 (issuers 1..3).
 * *flops_out (host) receives the FLOPs of the launch (2 M N K per MMA); time
 * the launch on `stream` with events.  A wait that gives up writes a code to
 * *err_dev (device int, zero on entry).  Asynchronous.
 * Errors: INVALID_ARG (kind, issuers, iters, null), CUDA. */
moe_status moe_mma_peak_loop(int32_t kind, int32_t issuers, int64_t iters, int32_t* err_dev,
                             double* flops_out, moe_stream_t stream);

/* Synchronize `stream` and report device-side failures of earlier calls on
 * this handle: MOE_ERR_TIMEOUT when a kernel gave up a bounded wait (the
 * kernel stopped and its outputs are invalid; the flag is cleared), or
 * MOE_ERR_CUDA for an asynchronous CUDA error.  MOE_OK otherwise. */
moe_status moe_sync_status(moe_handle h, moe_stream_t stream);

/* Static text of a status code. */
const char* moe_status_str(moe_status s);

/* Text of the last error on this handle (or of the last handle-free call
 * made by this host thread when h is NULL). */
const char* moe_last_error(moe_handle h);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
