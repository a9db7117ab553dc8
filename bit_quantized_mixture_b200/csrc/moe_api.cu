// C ABI of the routed-expert MoE layer: handle, arena, workspace, argument
// validation and dispatch to the kernels.  Declarations and the contract of
// every entry point are in include/moe_b200.h.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <new>

#include "../../include/moe_b200.h"
#include "kernels.h"
#include "layout.cuh"

using namespace moe;

constexpr int kProfEvents = 10;  // see moe_set_profile_events

struct moe_layer {
    moe_config cfg;
    // arena
    uint8_t* arena = nullptr;
    size_t arena_bytes = 0;
    MatGeom geom[3];               // gate, up, down of a routed expert
    size_t off_codes[3], off_scales[3], off_zeros[3];
    size_t off_gs = 0;             // NVFP4: the expert's two global scales inside its block
    size_t expert_stride = 0;      // bytes per routed expert
    uint8_t* experts = nullptr;    // expert e at experts + e * expert_stride
    uint8_t* router = nullptr;     // bf16 [E, H]
    uint8_t* shared[3] = {nullptr, nullptr, nullptr};   // bf16 device layout
    // NVFP4: the block-scaled prefill GEMM's weight images (gate/up, down),
    // when H and I allow 256-value stages
    uint8_t* fp4_img[2] = {nullptr, nullptr};
    float* g_gate = nullptr;       // NVFP4 global scales [E]
    float* g_down = nullptr;
    // workspace
    uint8_t* ws = nullptr;
    size_t ws_bytes = 0;
    float* logits = nullptr;       // [max_tokens, E]
    unsigned int* route_counter = nullptr;
    float* dec_a = nullptr;        // [8*k, I]
    float* dec_a_sh = nullptr;     // [8, I]
    float* dec_part = nullptr;     // [8*k, H]
    float* dec_part_sh = nullptr;  // [8, H]
    unsigned int* dec_counters = nullptr;   // [H/16]
    unsigned long long* fused_bar = nullptr;   // arrival count of the fused decode kernel's grid barrier
    float* fused_gu_sh = nullptr;              // [4][8][2I] partial shared gate/up sums of the fused decode kernel
    uint8_t* staging = nullptr;    // interchange copy of one matrix
    size_t staging_bytes = 0;
    // prefill path
    int32_t *counts = nullptr, *offsets = nullptr, *perm = nullptr, *inv = nullptr, *perm_scratch = nullptr;
    GemmTile* tiles = nullptr;
    int* num_tiles = nullptr;
    int2* groups = nullptr;
    size_t tile_cap = 0;
    int* dev_err = nullptr;
    // per-expert address table (moe_set_expert_table): device [E], in use when set
    const uint8_t** table = nullptr;
    bool table_set = false;
    int decode_path = 0;           // MOE_DECODE_AUTO / _FUSED / _KERNELS
    float* g_tab = nullptr;        // NVFP4: [2E] global scales gathered from the table's blocks
    __nv_bfloat16 *xq = nullptr, *xp = nullptr, *a_perm = nullptr, *a_sh = nullptr;
    float *w_perm = nullptr, *ts_perm = nullptr;
    __half *o = nullptr, *o_sh = nullptr;
    float* tok_scale = nullptr;
    // state
    bool router_loaded = false;
    bool shared_loaded = false;
    int experts_loaded = 0;
    uint8_t* expert_flag = nullptr;   // host, [E]
    float* g_host = nullptr;          // host copies of the NVFP4 global scales, [2E]
    float g_x = 0.0f, g_a = 0.0f;
    bool act_scales_set = false;
    cudaEvent_t prof[kProfEvents] = {};
    // the last grouped-GEMM forward: its token count and whether it took the
    // block-scaled NVFP4 path (read by the debug getters)
    int last_prefill_T = 0;
    bool last_prefill_fp4 = false;
    // moe_debug_set_wait_test: one-shot test hook of the next fused decode launch
    int dbg_withhold_cta = -1;
    long long dbg_wait_limit = 0;
    char err[512] = {0};
};

static thread_local char g_err[512];

static moe_status fail(moe_layer* h, moe_status s, const char* fmt, ...) {
    char* buf = h ? h->err : g_err;
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, 512, fmt, ap);
    va_end(ap);
    return s;
}

void moe::set_thread_error(const char* msg) { snprintf(g_err, sizeof g_err, "%s", msg); }

static moe_status cuda_fail(moe_layer* h, cudaError_t e, const char* where) {
    return fail(h, MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// Switches to the handle's device for the scope of an entry point.
struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(int dev) {
        cudaGetDevice(&prev);
        if (prev != dev) cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        int cur;
        cudaGetDevice(&cur);
        if (prev >= 0 && cur != prev) cudaSetDevice(prev);
    }
};

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

extern "C" {

const char* moe_status_str(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported";
        case MOE_ERR_STATE: return "invalid state";
        case MOE_ERR_OOM: return "out of device memory";
        case MOE_ERR_CUDA: return "cuda error";
        case MOE_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

const char* moe_last_error(moe_handle h) { return h ? h->err : g_err; }

float moe_nvfp4_global_scale(float amax) { return amax / (6.0f * 448.0f); }

moe_status moe_create(const moe_config* cfg, moe_handle* out) {
    if (!cfg || !out) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_create: null argument");
    *out = nullptr;
    const moe_config c = *cfg;
    if (c.hidden <= 0 || c.inter <= 0 || c.num_experts <= 0 || c.top_k <= 0 || c.max_tokens <= 0)
        return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_create: sizes must be positive");
    if (c.hidden % 128 || c.inter % 128)
        return fail(nullptr, MOE_ERR_UNSUPPORTED, "moe_create: hidden and inter must be multiples of 128");
    if (c.num_experts > 1024 || c.top_k > 32 || c.top_k > c.num_experts)
        return fail(nullptr, MOE_ERR_UNSUPPORTED, "moe_create: need E <= 1024 and k <= min(E, 32)");
    if (c.quant != MOE_Q_INT4 && c.quant != MOE_Q_INT4_G32 && c.quant != MOE_Q_INT2 && c.quant != MOE_Q_NVFP4 &&
        c.quant != MOE_Q_FP8_B128 && c.quant != MOE_Q_FP6_E2M3)
        return fail(nullptr, MOE_ERR_UNSUPPORTED,
                    "moe_create: routed quant must be INT4, INT4_G32, INT2, NVFP4, FP8_B128 or FP6_E2M3");
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || c.device < 0 || c.device >= ndev)
        return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_create: no CUDA device %d", c.device);
    DeviceGuard dg(c.device);

    moe_layer* h = new (std::nothrow) moe_layer();
    if (!h) return fail(nullptr, MOE_ERR_OOM, "moe_create: host allocation failed");
    h->cfg = c;
    const int H = c.hidden, I = c.inter, E = c.num_experts, k = c.top_k;
    h->geom[0] = {I, H, c.quant};
    h->geom[1] = {I, H, c.quant};
    h->geom[2] = {H, I, c.quant};
    size_t off = 0;
    for (int m = 0; m < 3; ++m) { h->off_codes[m] = off; off = align_up(off + h->geom[m].codes_bytes(), 256); }
    for (int m = 0; m < 3; ++m) { h->off_scales[m] = off; off = align_up(off + h->geom[m].scales_bytes(), 256); }
    for (int m = 0; m < 3; ++m) { h->off_zeros[m] = off; off = align_up(off + h->geom[m].zeros_bytes(), 256); }
    if (c.quant == MOE_Q_NVFP4) { h->off_gs = off; off = align_up(off + 2 * sizeof(float), 256); }
    h->expert_stride = off;
    size_t a = 0;
    const size_t experts_off = a; a = align_up(a + h->expert_stride * E, 4096);
    const size_t router_off = a; a = align_up(a + (size_t)E * H * 2, 256);
    size_t shared_off[3] = {0, 0, 0};
    if (c.has_shared)
        for (int m = 0; m < 3; ++m) { shared_off[m] = a; a = align_up(a + (size_t)H * I * 2, 256); }
    const size_t g_off = a; a = align_up(a + sizeof(float) * 2 * E, 256);
    // NVFP4: the interchange codes and scales, kept again as the block-scaled
    // prefill GEMM's weight images (per 128-row block and 256-value stage one
    // contiguous block of swizzled codes and scales; gate and up share blocks)
    const bool fp4_images = c.quant == MOE_Q_NVFP4 && prefill_native_fp4(H, I);
    size_t img_off[2] = {0, 0};
    if (fp4_images) {
        img_off[0] = a; a = align_up(a + (size_t)E * fp4_block_image_bytes(I, H, 2), 256);
        img_off[1] = a; a = align_up(a + (size_t)E * fp4_block_image_bytes(H, I, 1), 256);
    }
    h->arena_bytes = a;
    if (cudaMalloc(&h->arena, h->arena_bytes) != cudaSuccess) {
        cudaGetLastError();
        delete h;
        return fail(nullptr, MOE_ERR_OOM, "moe_create: arena of %zu bytes", a);
    }
    h->experts = h->arena + experts_off;
    if (fp4_images)
        for (int i = 0; i < 2; ++i) h->fp4_img[i] = h->arena + img_off[i];
    h->router = h->arena + router_off;
    if (c.has_shared)
        for (int m = 0; m < 3; ++m) h->shared[m] = h->arena + shared_off[m];
    h->g_gate = reinterpret_cast<float*>(h->arena + g_off);
    h->g_down = h->g_gate + E;

    // workspace
    const int MT = 16;  // tokens per launch of the two-kernel decode path
    size_t w = 0;
    auto carve = [&](size_t bytes) { size_t o = w; w = align_up(w + bytes, 256); return o; };
    const size_t o_logits = carve(sizeof(float) * (size_t)c.max_tokens * E);
    const size_t o_rc = carve(256);
    const size_t o_a = carve(sizeof(float) * (size_t)MT * k * I);
    const size_t o_ash = carve(sizeof(float) * (size_t)MT * I);
    const size_t o_part = carve(sizeof(float) * (size_t)MT * k * H);
    const size_t o_psh = carve(sizeof(float) * (size_t)MT * H);
    const size_t o_cnt = carve(sizeof(unsigned int) * (size_t)(H / 16));
    const size_t o_fbar = carve(sizeof(unsigned long long));
    const size_t o_gush = carve(sizeof(float) * 4 * (size_t)MT * 2 * I);
    h->staging_bytes = (size_t)2 * H * I + 65536;
    const size_t o_stage = carve(h->staging_bytes);
    const size_t Tm = (size_t)c.max_tokens, slots = Tm * k;
    const size_t o_counts = carve(sizeof(int32_t) * E);
    const size_t o_offsets = carve(sizeof(int32_t) * (E + 1));
    const size_t o_perm = carve(sizeof(int32_t) * slots);
    const size_t o_inv = carve(sizeof(int32_t) * slots);
    const size_t o_pscr = carve(sizeof(int32_t) * permute_scratch_ints((int)slots, E));
    // two tile lists (gate/up, down), each with its group list and four counts:
    // routed tiles, all tiles, routed groups, group order
    const size_t tile_cap = prefill_tile_capacity(c.max_tokens, k, E, H, I);
    const size_t o_tiles = carve(sizeof(GemmTile) * 2 * tile_cap);
    const size_t o_groups = carve(sizeof(int2) * 2 * tile_cap);
    const size_t o_ntiles = carve(8 * sizeof(int));
    const size_t o_err = carve(sizeof(int));
    const size_t o_table = carve(sizeof(void*) * (size_t)E);
    const size_t o_gtab = carve(sizeof(float) * 2 * (size_t)E);
    const size_t o_xq = carve(Tm * H * 2);
    const size_t o_tsc = carve(Tm * sizeof(float));
    const size_t o_xp = carve(slots * H * 2);
    const size_t o_wperm = carve(slots * sizeof(float));
    const size_t o_tsperm = carve(slots * sizeof(float));
    const size_t o_aperm = carve(slots * I * 2);
    const size_t o_ash16 = carve(c.has_shared ? Tm * I * 2 : 0);
    const size_t o_o = carve(slots * H * 2);
    const size_t o_osh = carve(c.has_shared ? Tm * H * 2 : 0);
    h->ws_bytes = w;
    if (cudaMalloc(&h->ws, h->ws_bytes) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(h->arena);
        delete h;
        return fail(nullptr, MOE_ERR_OOM, "moe_create: workspace of %zu bytes", w);
    }
    h->logits = reinterpret_cast<float*>(h->ws + o_logits);
    h->route_counter = reinterpret_cast<unsigned int*>(h->ws + o_rc);
    h->dec_a = reinterpret_cast<float*>(h->ws + o_a);
    h->dec_a_sh = reinterpret_cast<float*>(h->ws + o_ash);
    h->dec_part = reinterpret_cast<float*>(h->ws + o_part);
    h->dec_part_sh = reinterpret_cast<float*>(h->ws + o_psh);
    h->dec_counters = reinterpret_cast<unsigned int*>(h->ws + o_cnt);
    h->fused_bar = reinterpret_cast<unsigned long long*>(h->ws + o_fbar);
    h->fused_gu_sh = reinterpret_cast<float*>(h->ws + o_gush);
    h->staging = h->ws + o_stage;
    h->counts = reinterpret_cast<int32_t*>(h->ws + o_counts);
    h->offsets = reinterpret_cast<int32_t*>(h->ws + o_offsets);
    h->perm = reinterpret_cast<int32_t*>(h->ws + o_perm);
    h->inv = reinterpret_cast<int32_t*>(h->ws + o_inv);
    h->perm_scratch = reinterpret_cast<int32_t*>(h->ws + o_pscr);
    h->tiles = reinterpret_cast<GemmTile*>(h->ws + o_tiles);
    h->tile_cap = tile_cap;
    h->num_tiles = reinterpret_cast<int*>(h->ws + o_ntiles);
    h->groups = reinterpret_cast<int2*>(h->ws + o_groups);
    h->dev_err = reinterpret_cast<int*>(h->ws + o_err);
    h->table = reinterpret_cast<const uint8_t**>(h->ws + o_table);
    h->g_tab = reinterpret_cast<float*>(h->ws + o_gtab);
    h->xq = reinterpret_cast<__nv_bfloat16*>(h->ws + o_xq);
    h->tok_scale = reinterpret_cast<float*>(h->ws + o_tsc);
    h->xp = reinterpret_cast<__nv_bfloat16*>(h->ws + o_xp);
    h->w_perm = reinterpret_cast<float*>(h->ws + o_wperm);
    h->ts_perm = reinterpret_cast<float*>(h->ws + o_tsperm);
    h->a_perm = reinterpret_cast<__nv_bfloat16*>(h->ws + o_aperm);
    h->a_sh = reinterpret_cast<__nv_bfloat16*>(h->ws + o_ash16);
    h->o = reinterpret_cast<__half*>(h->ws + o_o);
    h->o_sh = reinterpret_cast<__half*>(h->ws + o_osh);
    cudaError_t e1 = cudaMemset(h->ws, 0, h->ws_bytes);
    cudaError_t e2 = cudaMemset(h->arena, 0, h->arena_bytes);
    if (e1 != cudaSuccess || e2 != cudaSuccess) {
        cudaFree(h->ws);
        cudaFree(h->arena);
        delete h;
        return fail(nullptr, MOE_ERR_CUDA, "moe_create: memset failed");
    }
    h->expert_flag = new (std::nothrow) uint8_t[E]();
    h->g_host = new (std::nothrow) float[2 * (size_t)E]();
    if (!h->expert_flag || !h->g_host) {
        delete[] h->expert_flag;
        delete[] h->g_host;
        cudaFree(h->ws);
        cudaFree(h->arena);
        delete h;
        return fail(nullptr, MOE_ERR_OOM, "moe_create: host allocation failed");
    }
    *out = h;
    return MOE_OK;
}

moe_status moe_destroy(moe_handle h) {
    if (!h) return MOE_OK;
    DeviceGuard dg(h->cfg.device);
    cudaDeviceSynchronize();
    cudaFree(h->ws);
    cudaFree(h->arena);
    delete[] h->expert_flag;
    delete[] h->g_host;
    delete h;
    return MOE_OK;
}

moe_status moe_load_router(moe_handle h, const void* w_router_any, moe_stream_t stream) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_load_router: null handle");
    if (!w_router_any) return fail(h, MOE_ERR_INVALID_ARG, "moe_load_router: null router");
    DeviceGuard dg(h->cfg.device);
    const size_t bytes = (size_t)h->cfg.num_experts * h->cfg.hidden * 2;
    cudaError_t e = cudaMemcpyAsync(h->router, w_router_any, bytes, cudaMemcpyDefault, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "moe_load_router");
    h->router_loaded = true;
    return MOE_OK;
}

static moe_status load_matrix(moe_layer* h, const MatGeom& gm, const moe_qmatrix& q, uint8_t* dst_codes,
                              uint8_t* dst_scales, uint8_t* dst_zeros, cudaStream_t st, uint8_t* img = nullptr,
                              int img_slot = 0, int img_nmat = 1) {
    const size_t codes_in = gm.quant == Q_BF16 ? (size_t)gm.N * gm.K * 2
                                               : (size_t)gm.N * gm.K /
                                                     (gm.quant == Q_INT2 ? 4 : ((gm.quant == Q_FP8 || gm.quant == Q_FP6) ? 1 : 2));
    // interchange scales (the device layout pads FP8 scale rows to 16 bytes)
    const size_t scales_in = gm.quant == Q_FP8 ? (size_t)gm.nb() * (gm.K / 128) * 4 : gm.scales_bytes();
    const size_t zeros_in = gm.quant == Q_INT2 ? (size_t)(gm.N / 4) * gm.groups() : 0;
    const size_t o_s = align_up(codes_in, 256), o_z = align_up(o_s + scales_in, 256);
    if (align_up(o_z + zeros_in, 256) > h->staging_bytes) return fail(h, MOE_ERR_UNSUPPORTED, "staging too small");
    cudaError_t e = cudaMemcpyAsync(h->staging, q.codes, codes_in, cudaMemcpyDefault, st);
    if (e == cudaSuccess && scales_in) e = cudaMemcpyAsync(h->staging + o_s, q.scales, scales_in, cudaMemcpyDefault, st);
    if (e == cudaSuccess && zeros_in) e = cudaMemcpyAsync(h->staging + o_z, q.zeros, zeros_in, cudaMemcpyDefault, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "moe_load_expert_weights: copy");
    e = launch_relayout(gm, h->staging, h->staging + o_s, h->staging + o_z, dst_codes, dst_scales, dst_zeros, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "moe_load_expert_weights: relayout");
    if (img) {
        // NVFP4: the prefill GEMM's weight image, built from the interchange
        // codes and scales still in the staging buffer
        e = launch_fp4_block_image(h->staging, h->staging + o_s, gm.N, gm.K, img_slot, img_nmat, img, st);
        if (e != cudaSuccess) return cuda_fail(h, e, "moe_load_expert_weights: NVFP4 image");
    }
    return MOE_OK;
}

moe_status moe_load_expert_weights(moe_handle h, int32_t expert, const moe_expert_weights* w,
                                   moe_stream_t stream) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_load_expert_weights: null handle");
    if (!w) return fail(h, MOE_ERR_INVALID_ARG, "moe_load_expert_weights: null weights");
    const moe_config& c = h->cfg;
    const bool shared = expert == MOE_SHARED_EXPERT;
    if (!shared && (expert < 0 || expert >= c.num_experts))
        return fail(h, MOE_ERR_INVALID_ARG, "moe_load_expert_weights: expert %d out of range", expert);
    if (shared && !c.has_shared)
        return fail(h, MOE_ERR_INVALID_ARG, "moe_load_expert_weights: layer has no shared expert");
    const moe_qmatrix* mats[3] = {&w->gate, &w->up, &w->down};
    for (int m = 0; m < 3; ++m) {
        if (!mats[m]->codes) return fail(h, MOE_ERR_INVALID_ARG, "moe_load_expert_weights: null codes");
        if (!shared && !mats[m]->scales) return fail(h, MOE_ERR_INVALID_ARG, "moe_load_expert_weights: null scales");
        if (!shared && c.quant == MOE_Q_INT2 && !mats[m]->zeros)
            return fail(h, MOE_ERR_INVALID_ARG, "moe_load_expert_weights: INT2 needs zeros");
    }
    if (!shared && c.quant == MOE_Q_NVFP4) {
        if (w->gate.global_scale != w->up.global_scale)
            return fail(h, MOE_ERR_INVALID_ARG, "moe_load_expert_weights: gate and up must share one global scale");
        if (!(w->gate.global_scale >= 0.0f) || !(w->down.global_scale >= 0.0f))
            return fail(h, MOE_ERR_INVALID_ARG, "moe_load_expert_weights: bad NVFP4 global scale");
    }
    DeviceGuard dg(c.device);
    cudaStream_t st = (cudaStream_t)stream;
    for (int m = 0; m < 3; ++m) {
        MatGeom gm = h->geom[m];
        moe_status s;
        if (shared) {
            gm.quant = Q_BF16;
            s = load_matrix(h, gm, *mats[m], h->shared[m], nullptr, nullptr, st);
        } else {
            uint8_t* base = h->experts + (size_t)expert * h->expert_stride;
            // gate and up fill slots 0 and 1 of the gate/up image's blocks
            const int im = m == 2 ? 1 : 0, nmat = m == 2 ? 1 : 2;
            uint8_t* img = h->fp4_img[im] ? h->fp4_img[im] + (size_t)expert * fp4_block_image_bytes(gm.N, gm.K, nmat)
                                          : nullptr;
            s = load_matrix(h, gm, *mats[m], base + h->off_codes[m], base + h->off_scales[m], base + h->off_zeros[m], st,
                            img, m == 1 ? 1 : 0, nmat);
        }
        if (s != MOE_OK) return s;
    }
    if (!shared && c.quant == MOE_Q_NVFP4) {
        // copied from host arrays owned by the handle, so the caller's struct
        // need not outlive the asynchronous copy
        h->g_host[expert] = w->gate.global_scale;
        h->g_host[c.num_experts + expert] = w->down.global_scale;
        cudaError_t e = cudaMemcpyAsync(h->g_gate + expert, h->g_host + expert, sizeof(float),
                                        cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(h->g_down + expert, h->g_host + c.num_experts + expert, sizeof(float),
                                cudaMemcpyHostToDevice, st);
        // and inside the expert's block, which moe_export_expert copies
        uint8_t* gb = h->experts + (size_t)expert * h->expert_stride + h->off_gs;
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(gb, h->g_host + expert, sizeof(float), cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(gb + sizeof(float), h->g_host + c.num_experts + expert, sizeof(float),
                                cudaMemcpyHostToDevice, st);
        if (e != cudaSuccess) return cuda_fail(h, e, "moe_load_expert_weights: global scales");
    }
    if (shared) h->shared_loaded = true;
    else if (!h->expert_flag[expert]) { h->expert_flag[expert] = 1; ++h->experts_loaded; }
    return MOE_OK;
}

moe_status moe_set_act_global_scales(moe_handle h, float g_x, float g_a) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_set_act_global_scales: null handle");
    if (h->cfg.quant != MOE_Q_NVFP4) return fail(h, MOE_ERR_STATE, "moe_set_act_global_scales: layer is not NVFP4");
    if (!(g_x > 0.0f) || !(g_a > 0.0f)) return fail(h, MOE_ERR_INVALID_ARG, "moe_set_act_global_scales: scales must be > 0");
    h->g_x = g_x;
    h->g_a = g_a;
    h->act_scales_set = true;
    return MOE_OK;
}

static moe_status check_tokens(moe_layer* h, const char* fn, int32_t T) {
    if (T < 1 || T > h->cfg.max_tokens)
        return fail(h, MOE_ERR_INVALID_ARG, "%s: T=%d outside [1, max_tokens=%d]", fn, T, h->cfg.max_tokens);
    return MOE_OK;
}

moe_status moe_route(moe_handle h, const void* x, int32_t T, int32_t* topk_ids, float* topk_w, float* logits_out,
                     moe_stream_t stream) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_route: null handle");
    moe_status s = check_tokens(h, "moe_route", T);
    if (s != MOE_OK) return s;
    if (!x || (!topk_ids) != (!topk_w) || (!topk_ids && !logits_out))
        return fail(h, MOE_ERR_INVALID_ARG, "moe_route: null pointer");
    if (!aligned16(x)) return fail(h, MOE_ERR_INVALID_ARG, "moe_route: x must be 16-byte aligned");
    if (!h->router_loaded) return fail(h, MOE_ERR_STATE, "moe_route: router not loaded");
    DeviceGuard dg(h->cfg.device);
    RouteArgs a{};
    a.x = x;
    a.wr = h->router;
    a.logits_in = nullptr;
    a.logits = logits_out ? logits_out : h->logits;
    a.ids = topk_ids;
    a.w = topk_w;
    a.counter = h->route_counter;
    a.err = h->dev_err;
    a.T = T; a.H = h->cfg.hidden; a.E = h->cfg.num_experts; a.k = h->cfg.top_k;
    cudaStream_t st = (cudaStream_t)stream;
    if (h->prof[0]) cudaEventRecord(h->prof[0], st);
    cudaError_t e = launch_route(a, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "moe_route");
    if (h->prof[1]) cudaEventRecord(h->prof[1], st);
    return MOE_OK;
}

moe_status moe_route_from_logits(moe_handle h, const float* logits, int32_t T, int32_t* topk_ids, float* topk_w,
                                 moe_stream_t stream) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_route_from_logits: null handle");
    moe_status s = check_tokens(h, "moe_route_from_logits", T);
    if (s != MOE_OK) return s;
    if (!logits || !topk_ids || !topk_w) return fail(h, MOE_ERR_INVALID_ARG, "moe_route_from_logits: null pointer");
    DeviceGuard dg(h->cfg.device);
    RouteArgs a{};
    a.logits_in = logits;
    a.logits = nullptr;
    a.ids = topk_ids;
    a.w = topk_w;
    a.T = T; a.H = h->cfg.hidden; a.E = h->cfg.num_experts; a.k = h->cfg.top_k;
    cudaError_t e = launch_route(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "moe_route_from_logits");
    return MOE_OK;
}

static ExpertArgs expert_args(moe_layer* h) {
    ExpertArgs ex{};
    const moe_config& c = h->cfg;
    MatView* v[3] = {&ex.gate, &ex.up, &ex.down};
    for (int m = 0; m < 3; ++m) {
        v[m]->codes = h->experts + h->off_codes[m];
        v[m]->scales = h->experts + h->off_scales[m];
        v[m]->zeros = c.quant == MOE_Q_INT2 ? h->experts + h->off_zeros[m] : nullptr;
        v[m]->stride = h->expert_stride;
        v[m]->table = h->table_set ? h->table : nullptr;
        v[m]->off_codes = h->off_codes[m];
        v[m]->off_scales = h->off_scales[m];
        v[m]->off_zeros = h->off_zeros[m];
        v[m]->N = h->geom[m].N;
        v[m]->K = h->geom[m].K;
    }
    ex.sh_gate = c.has_shared ? h->shared[0] : nullptr;
    ex.sh_up = c.has_shared ? h->shared[1] : nullptr;
    ex.sh_down = c.has_shared ? h->shared[2] : nullptr;
    ex.g_gate = h->table_set ? h->g_tab : h->g_gate;
    ex.g_down = h->table_set ? h->g_tab + c.num_experts : h->g_down;
    ex.g_x = h->g_x;
    ex.g_a = h->g_a;
    ex.quant = c.quant;
    ex.H = c.hidden; ex.I = c.inter; ex.E = c.num_experts; ex.k = c.top_k;
    return ex;
}

// Decode (T <= 8) on the fused cooperative kernel?  It saves the launch gaps
// of eager calls; inside a CUDA graph the GEMV kernels (programmatic launch
// overlap, no grid barriers) are faster.  false with an error on failure.
static bool use_fused_decode(moe_layer* h, cudaStream_t st, cudaError_t* err) {
    *err = cudaSuccess;
    if (h->decode_path == MOE_DECODE_FUSED) return true;
    if (h->decode_path == MOE_DECODE_KERNELS || h->decode_path == MOE_DECODE_GEMM) return false;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    *err = cudaStreamIsCapturing(st, &cs);
    return *err == cudaSuccess && cs == cudaStreamCaptureStatusNone;
}

// the one-shot test hook of the bounded waits goes to this launch only
static void take_wait_test(moe_layer* h, FusedArgs& f) {
    f.withhold_cta = h->dbg_withhold_cta;
    f.wait_limit = h->dbg_wait_limit;
    h->dbg_withhold_cta = -1;
    h->dbg_wait_limit = 0;
}

static DecodeArgs decode_args(moe_layer* h) {
    DecodeArgs a{};
    a.ex = expert_args(h);
    a.a = h->dec_a;
    a.a_sh = h->dec_a_sh;
    a.part = h->dec_part;
    a.part_sh = h->dec_part_sh;
    a.counters = h->dec_counters;
    return a;
}

moe_status moe_forward(moe_handle h, const void* x, int32_t T, const int32_t* topk_ids, const float* topk_w, void* y,
                       moe_stream_t stream) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_forward: null handle");
    moe_status s = check_tokens(h, "moe_forward", T);
    if (s != MOE_OK) return s;
    if (!x || !topk_ids || !topk_w || !y) return fail(h, MOE_ERR_INVALID_ARG, "moe_forward: null pointer");
    if (!aligned16(x) || !aligned16(y)) return fail(h, MOE_ERR_INVALID_ARG, "moe_forward: x and y must be 16-byte aligned");
    const moe_config& c = h->cfg;
    if (h->experts_loaded != c.num_experts)
        return fail(h, MOE_ERR_STATE, "moe_forward: %d of %d experts loaded", h->experts_loaded, c.num_experts);
    if (c.has_shared && !h->shared_loaded) return fail(h, MOE_ERR_STATE, "moe_forward: shared expert not loaded");
    if (c.quant == MOE_Q_NVFP4 && !h->act_scales_set)
        return fail(h, MOE_ERR_STATE, "moe_forward: NVFP4 activation global scales not set");
    DeviceGuard dg(c.device);
    cudaStream_t st = (cudaStream_t)stream;
    // the grouped-GEMM path: more tokens than the GEMVs take, the GEMM path
    // forced, or 9 to 16 tokens by default (measured: from 8 tokens per call
    // the grouped GEMM is the faster of the two on the decode-b1 INT4 layer)
    const bool gemv_ok = decode_supported(T, c.top_k) && (T <= 8 || h->decode_path == MOE_DECODE_KERNELS);
    if (!gemv_ok || h->decode_path == MOE_DECODE_GEMM) {
        PrefillArgs p{};
        p.ex = expert_args(h);
        p.x = x; p.ids = topk_ids; p.w = topk_w; p.y = y; p.T = T;
        p.counts = h->counts; p.offsets = h->offsets; p.perm = h->perm; p.inv = h->inv;
        p.perm_scratch = h->perm_scratch;
        p.tiles = h->tiles; p.groups = h->groups; p.num_tiles = h->num_tiles; p.tile_cap = h->tile_cap;
        p.xq = h->xq; p.tok_scale = h->tok_scale; p.xp = h->xp; p.w_perm = h->w_perm; p.ts_perm = h->ts_perm;
        p.a_perm = h->a_perm; p.a_sh = h->a_sh; p.o = h->o; p.o_sh = h->o_sh;
        p.err = h->dev_err;
        // the block-scaled NVFP4 images live in the arena: with an address
        // table the exact bf16-dequantization path reads the table's blocks
        for (int i = 0; i < 2; ++i) p.fp4_img[i] = h->table_set ? nullptr : h->fp4_img[i];
        p.ev_gu0 = h->prof[5]; p.ev_gu1 = h->prof[3]; p.ev_dn0 = h->prof[6]; p.ev_dn1 = h->prof[7];
        p.ev_gu_r = h->prof[8]; p.ev_dn_r = h->prof[9];
        h->last_prefill_T = T;
        h->last_prefill_fp4 = c.quant == MOE_Q_NVFP4 && !h->table_set && prefill_native_fp4(c.hidden, c.inter);
        if (h->prof[2]) cudaEventRecord(h->prof[2], st);
        cudaError_t e = launch_prefill(p, st);
        if (e != cudaSuccess) return cuda_fail(h, e, "moe_forward (grouped GEMM path)");
        if (h->prof[4]) cudaEventRecord(h->prof[4], st);
        return MOE_OK;
    }
    DecodeArgs a = decode_args(h);
    cudaError_t pe = cudaSuccess;
    const bool fused = T <= 8 && use_fused_decode(h, st, &pe);
    if (pe != cudaSuccess) return cuda_fail(h, pe, "moe_forward");
    if (fused) {
        FusedArgs f{};
        f.d = a;
        f.d.x = x; f.d.ids = topk_ids; f.d.w = topk_w; f.d.y = y; f.d.T = T;
        f.wr = nullptr;
        f.bar = h->fused_bar;
        f.gu_sh = h->fused_gu_sh;
        f.err = h->dev_err;
        take_wait_test(h, f);
        if (h->prof[2]) cudaEventRecord(h->prof[2], st);
        cudaError_t e = launch_decode_fused(f, st);
        if (e == cudaSuccess) {
            if (h->prof[4]) cudaEventRecord(h->prof[4], st);
            return MOE_OK;
        }
        // a refused cooperative launch falls back to the two-kernel decode path
        if (e != cudaErrorCooperativeLaunchTooLarge && e != cudaErrorNotSupported) return cuda_fail(h, e, "moe_forward");
        cudaGetLastError();
    }
    a.ex = expert_args(h);
    a.a = h->dec_a;
    a.a_sh = h->dec_a_sh;
    a.part = h->dec_part;
    a.part_sh = h->dec_part_sh;
    a.counters = h->dec_counters;
    a.ev_mid = h->prof[3];
    if (h->prof[2]) cudaEventRecord(h->prof[2], st);
    for (int t0 = 0; t0 < T;) {
        int tc = T - t0 < 16 ? T - t0 : 16;
        while (!decode_supported(tc, c.top_k)) --tc;
        a.x = reinterpret_cast<const uint8_t*>(x) + (size_t)t0 * c.hidden * 2;
        a.ids = topk_ids + (size_t)t0 * c.top_k;
        a.w = topk_w + (size_t)t0 * c.top_k;
        a.y = reinterpret_cast<uint8_t*>(y) + (size_t)t0 * c.hidden * 2;
        a.T = tc;
        cudaError_t e = launch_decode(a, st);
        if (e != cudaSuccess) return cuda_fail(h, e, "moe_forward");
        t0 += tc;
    }
    if (h->prof[4]) cudaEventRecord(h->prof[4], st);
    return MOE_OK;
}

moe_status moe_route_forward(moe_handle h, const void* x, int32_t T, int32_t* topk_ids, float* topk_w, void* y,
                             moe_stream_t stream) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_route_forward: null handle");
    moe_status s = check_tokens(h, "moe_route_forward", T);
    if (s != MOE_OK) return s;
    if (!x || !topk_ids || !topk_w || !y) return fail(h, MOE_ERR_INVALID_ARG, "moe_route_forward: null pointer");
    if (!aligned16(x) || !aligned16(y))
        return fail(h, MOE_ERR_INVALID_ARG, "moe_route_forward: x and y must be 16-byte aligned");
    const moe_config& c = h->cfg;
    if (!h->router_loaded) return fail(h, MOE_ERR_STATE, "moe_route_forward: router not loaded");
    if (h->experts_loaded != c.num_experts)
        return fail(h, MOE_ERR_STATE, "moe_route_forward: %d of %d experts loaded", h->experts_loaded, c.num_experts);
    if (c.has_shared && !h->shared_loaded) return fail(h, MOE_ERR_STATE, "moe_route_forward: shared expert not loaded");
    if (c.quant == MOE_Q_NVFP4 && !h->act_scales_set)
        return fail(h, MOE_ERR_STATE, "moe_route_forward: NVFP4 activation global scales not set");
    DeviceGuard dg(c.device);
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t pe = cudaSuccess;
    const bool fused = use_fused_decode(h, st, &pe);
    if (pe != cudaSuccess) return cuda_fail(h, pe, "moe_route_forward");
    if (!fused || T > 8 || !decode_supported(T, c.top_k)) {
        s = moe_route(h, x, T, topk_ids, topk_w, nullptr, stream);
        if (s != MOE_OK) return s;
        return moe_forward(h, x, T, topk_ids, topk_w, y, stream);
    }
    FusedArgs f{};
    f.d = decode_args(h);
    f.d.x = x; f.d.ids = topk_ids; f.d.w = topk_w; f.d.y = y; f.d.T = T;
    f.wr = h->router;
    f.logits = h->logits;
    f.ids_out = topk_ids;
    f.w_out = topk_w;
    f.bar = h->fused_bar;
    f.gu_sh = h->fused_gu_sh;
    f.err = h->dev_err;
    take_wait_test(h, f);
    if (h->prof[0]) cudaEventRecord(h->prof[0], st);
    cudaError_t e = launch_decode_fused(f, st);
    if (e == cudaSuccess) {
        if (h->prof[4]) cudaEventRecord(h->prof[4], st);
        return MOE_OK;
    }
    if (e != cudaErrorCooperativeLaunchTooLarge && e != cudaErrorNotSupported)
        return cuda_fail(h, e, "moe_route_forward");
    cudaGetLastError();
    s = moe_route(h, x, T, topk_ids, topk_w, nullptr, stream);
    if (s != MOE_OK) return s;
    return moe_forward(h, x, T, topk_ids, topk_w, y, stream);
}

moe_status moe_sync_status(moe_handle h, moe_stream_t stream) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_sync_status: null handle");
    DeviceGuard dg(h->cfg.device);
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "moe_sync_status");
    int code = 0;
    e = cudaMemcpy(&code, h->dev_err, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(h, e, "moe_sync_status");
    if (code) {
        // a stopped kernel may leave tickets and the grid barrier half-counted
        const int zero = 0;
        cudaMemcpy(h->dev_err, &zero, sizeof(int), cudaMemcpyHostToDevice);
        cudaMemset(h->dec_counters, 0, sizeof(unsigned int) * (size_t)(h->cfg.hidden / 16));
        cudaMemset(h->fused_bar, 0, sizeof(unsigned long long));
        return fail(h, MOE_ERR_TIMEOUT, "a kernel gave up a bounded wait (site %d); outputs are invalid", code);
    }
    return MOE_OK;
}

moe_status moe_set_profile_events(moe_handle h, void* const* events, int32_t n) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_set_profile_events: null handle");
    if (events && n < 5) return fail(h, MOE_ERR_INVALID_ARG, "moe_set_profile_events: need at least 5 events");
    for (int i = 0; i < kProfEvents; ++i) h->prof[i] = (events && i < n) ? (cudaEvent_t)events[i] : nullptr;
    return MOE_OK;
}

moe_status moe_quantize(int32_t quant, const float* w, int32_t N, int32_t K, float global_scale, void* codes,
                        void* scales, void* zeros, moe_stream_t stream) {
    if (!w || !codes || !scales) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_quantize: null pointer");
    if (N <= 0 || K <= 0) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_quantize: sizes must be positive");
    if (quant == MOE_Q_FP8_B128) {
        if (N % 128 || K % 128)
            return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_quantize: FP8 needs N and K multiples of 128");
    } else if (quant == MOE_Q_INT4 || quant == MOE_Q_INT4_G32 || quant == MOE_Q_INT2 || quant == MOE_Q_FP6_E2M3) {
        if (K % 128) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_quantize: K must be a multiple of 128");
        if (quant == MOE_Q_INT2 && (N % 4 || !zeros))
            return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_quantize: INT2 needs N %% 4 == 0 and zeros");
    } else if (quant == MOE_Q_NVFP4) {
        if (K % 16) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_quantize: K must be a multiple of 16");
        if (!(global_scale >= 0.0f)) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_quantize: bad global scale");
    } else {
        return fail(nullptr, MOE_ERR_UNSUPPORTED, "moe_quantize: quant %d", quant);
    }
    if (!aligned16(w)) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_quantize: w must be 16-byte aligned");
    cudaError_t e = launch_quantize(quant, w, N, K, global_scale, codes, scales, zeros, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(nullptr, e, "moe_quantize");
    return MOE_OK;
}

moe_status moe_absmax(const float* x, int64_t n, float* amax_inout_dev, moe_stream_t stream) {
    if (!x || !amax_inout_dev || n < 0) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_absmax: bad argument");
    if (n == 0) return MOE_OK;
    cudaError_t e = launch_absmax(x, n, amax_inout_dev, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(nullptr, e, "moe_absmax");
    return MOE_OK;
}

moe_status moe_quantize_act_nvfp4(const void* x, int32_t T, int32_t K, float g, void* codes, void* scales,
                                  moe_stream_t stream) {
    if (!x || !codes || !scales || T <= 0 || K <= 0 || K % 16)
        return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_quantize_act_nvfp4: bad argument");
    if (!(g >= 0.0f)) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_quantize_act_nvfp4: bad global scale");
    cudaError_t e = launch_quantize_act_nvfp4(x, T, K, g, codes, scales, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(nullptr, e, "moe_quantize_act_nvfp4");
    return MOE_OK;
}

moe_status moe_permute(const int32_t* topk_ids, int32_t T, int32_t k, int32_t E, int32_t* counts, int32_t* offsets,
                       int32_t* perm, int32_t* inv, moe_stream_t stream) {
    if (!topk_ids || !counts || !offsets || !perm || !inv)
        return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_permute: null pointer");
    if (T <= 0 || k <= 0 || E <= 0 || E > 1024 || (int64_t)T * k > (1 << 30))
        return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_permute: bad sizes");
    cudaStream_t st = (cudaStream_t)stream;
    const size_t n = permute_scratch_ints(T * k, E);
    int32_t* scratch = nullptr;
    cudaError_t e = cudaMallocAsync((void**)&scratch, n * sizeof(int32_t), st);
    if (e != cudaSuccess) return cuda_fail(nullptr, e, "moe_permute: scratch");
    e = launch_permute(topk_ids, T, k, E, counts, offsets, perm, inv, scratch, st);
    cudaError_t e2 = cudaFreeAsync(scratch, st);
    if (e != cudaSuccess) return cuda_fail(nullptr, e, "moe_permute");
    if (e2 != cudaSuccess) return cuda_fail(nullptr, e2, "moe_permute: free");
    return MOE_OK;
}

moe_status moe_debug_unpack_matrix(moe_handle h, int32_t expert, int32_t which, void* codes, void* scales,
                                   void* zeros, float* global_scale_out, moe_stream_t stream) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_debug_unpack_matrix: null handle");
    if (which < 0 || which > 2 || !codes) return fail(h, MOE_ERR_INVALID_ARG, "moe_debug_unpack_matrix: bad argument");
    const moe_config& c = h->cfg;
    const bool shared = expert == MOE_SHARED_EXPERT;
    if (!shared && (expert < 0 || expert >= c.num_experts))
        return fail(h, MOE_ERR_INVALID_ARG, "moe_debug_unpack_matrix: expert out of range");
    if (shared && !c.has_shared) return fail(h, MOE_ERR_INVALID_ARG, "moe_debug_unpack_matrix: no shared expert");
    DeviceGuard dg(c.device);
    cudaStream_t st = (cudaStream_t)stream;
    MatGeom gm = h->geom[which];
    cudaError_t e;
    if (shared) {
        gm.quant = Q_BF16;
        e = launch_unpack(gm, h->shared[which], nullptr, nullptr, (uint8_t*)codes, nullptr, nullptr, st);
    } else {
        if (!scales || (c.quant == MOE_Q_INT2 && !zeros))
            return fail(h, MOE_ERR_INVALID_ARG, "moe_debug_unpack_matrix: null scales/zeros");
        uint8_t* base = h->experts + (size_t)expert * h->expert_stride;
        e = launch_unpack(gm, base + h->off_codes[which], base + h->off_scales[which], base + h->off_zeros[which],
                          (uint8_t*)codes, (uint8_t*)scales, (uint8_t*)zeros, st);
        if (e == cudaSuccess && c.quant == MOE_Q_NVFP4 && global_scale_out)
            e = cudaMemcpyAsync(global_scale_out, (which == 2 ? h->g_down : h->g_gate) + expert, sizeof(float),
                                cudaMemcpyDefault, st);
    }
    if (e != cudaSuccess) return cuda_fail(h, e, "moe_debug_unpack_matrix");
    return MOE_OK;
}

moe_status moe_debug_get_permutation(moe_handle h, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                                     moe_stream_t stream) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_debug_get_permutation: null handle");
    if (!counts || !offsets || !perm || !inv) return fail(h, MOE_ERR_INVALID_ARG, "moe_debug_get_permutation: null pointer");
    if (h->last_prefill_T <= 0) return fail(h, MOE_ERR_STATE, "moe_debug_get_permutation: no grouped-GEMM forward yet");
    DeviceGuard dg(h->cfg.device);
    cudaStream_t st = (cudaStream_t)stream;
    const int E = h->cfg.num_experts;
    const size_t slots = (size_t)h->last_prefill_T * h->cfg.top_k;
    cudaError_t e = cudaMemcpyAsync(counts, h->counts, sizeof(int32_t) * E, cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(offsets, h->offsets, sizeof(int32_t) * (E + 1), cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(perm, h->perm, sizeof(int32_t) * slots, cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(inv, h->inv, sizeof(int32_t) * slots, cudaMemcpyDefault, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "moe_debug_get_permutation");
    return MOE_OK;
}

moe_status moe_debug_get_act_nvfp4(moe_handle h, void* codes, void* scales, moe_stream_t stream) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_debug_get_act_nvfp4: null handle");
    if (!codes || !scales) return fail(h, MOE_ERR_INVALID_ARG, "moe_debug_get_act_nvfp4: null pointer");
    if (h->last_prefill_T <= 0 || !h->last_prefill_fp4)
        return fail(h, MOE_ERR_STATE, "moe_debug_get_act_nvfp4: no block-scaled NVFP4 grouped-GEMM forward yet");
    DeviceGuard dg(h->cfg.device);
    cudaStream_t st = (cudaStream_t)stream;
    const size_t slots = (size_t)h->last_prefill_T * h->cfg.top_k, H = (size_t)h->cfg.hidden;
    // codes [slots][H/2], then the scales stage-major [H/256][slots][16 B]
    const uint8_t* xc = reinterpret_cast<const uint8_t*>(h->xp);
    cudaError_t e = cudaMemcpyAsync(codes, xc, slots * H / 2, cudaMemcpyDefault, st);
    for (size_t ks = 0; e == cudaSuccess && ks < H / 256; ++ks)
        e = cudaMemcpy2DAsync(reinterpret_cast<uint8_t*>(scales) + ks * 16, H / 16, xc + slots * H / 2 + ks * slots * 16, 16,
                              16, slots, cudaMemcpyDefault, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "moe_debug_get_act_nvfp4");
    return MOE_OK;
}

moe_status moe_debug_set_wait_test(moe_handle h, int32_t withhold_cta, int64_t wait_limit_cycles) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_debug_set_wait_test: null handle");
    if (wait_limit_cycles < 0) return fail(h, MOE_ERR_INVALID_ARG, "moe_debug_set_wait_test: negative limit");
    h->dbg_withhold_cta = withhold_cta < 0 ? -1 : withhold_cta;
    h->dbg_wait_limit = wait_limit_cycles;
    return MOE_OK;
}

moe_status moe_set_decode_path(moe_handle h, int32_t path) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_set_decode_path: null handle");
    if (path != MOE_DECODE_AUTO && path != MOE_DECODE_FUSED && path != MOE_DECODE_KERNELS && path != MOE_DECODE_GEMM)
        return fail(h, MOE_ERR_INVALID_ARG, "moe_set_decode_path: unknown path %d", path);
    h->decode_path = path;
    return MOE_OK;
}

moe_status moe_expert_block_bytes(moe_handle h, size_t* bytes) {
    if (!h || !bytes) return fail(h, MOE_ERR_INVALID_ARG, "moe_expert_block_bytes: null pointer");
    *bytes = h->expert_stride;
    return MOE_OK;
}

moe_status moe_export_expert(moe_handle h, int32_t expert, void* dst, moe_stream_t stream) {
    if (!h || !dst) return fail(h, MOE_ERR_INVALID_ARG, "moe_export_expert: null pointer");
    if (expert < 0 || expert >= h->cfg.num_experts)
        return fail(h, MOE_ERR_INVALID_ARG, "moe_export_expert: expert %d out of range", expert);
    if ((reinterpret_cast<uintptr_t>(dst) & 255u) != 0)
        return fail(h, MOE_ERR_INVALID_ARG, "moe_export_expert: dst must be 256-byte aligned");
    DeviceGuard dg(h->cfg.device);
    const cudaError_t e = cudaMemcpyAsync(dst, h->experts + (size_t)expert * h->expert_stride, h->expert_stride,
                                          cudaMemcpyDeviceToDevice, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "moe_export_expert");
    return MOE_OK;
}

moe_status moe_set_expert_table(moe_handle h, const void* const* blocks, moe_stream_t stream) {
    if (!h) return fail(nullptr, MOE_ERR_INVALID_ARG, "moe_set_expert_table: null handle");
    const int E = h->cfg.num_experts;
    if (blocks)
        for (int e = 0; e < E; ++e)
            if (!blocks[e] || (reinterpret_cast<uintptr_t>(blocks[e]) & 255u) != 0)
                return fail(h, MOE_ERR_INVALID_ARG, "moe_set_expert_table: block of expert %d is null or not "
                                                    "256-byte aligned", e);
    DeviceGuard dg(h->cfg.device);
    // earlier work on the stream may still read the old table
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e == cudaSuccess && blocks)
        e = cudaMemcpy(h->table, blocks, sizeof(void*) * (size_t)E, cudaMemcpyHostToDevice);
    // NVFP4: the per-expert global scales travel in the blocks
    if (e == cudaSuccess && blocks && h->cfg.quant == MOE_Q_NVFP4)
        e = launch_gather_global_scales(h->table, h->off_gs, E, h->g_tab, (cudaStream_t)stream);
    if (e == cudaSuccess && blocks) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "moe_set_expert_table");
    h->table_set = blocks != nullptr;
    return MOE_OK;
}

}  // extern "C"
