// C ABI of the e4b library (declared in include/e4b.h): argument validation,
// workspace layout and the launch sequence of each entry point.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/e4b.h"
#include "e4b_internal.h"
#include "lora.h"
#include "router_backward.h"

namespace e4b {

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// ------------------------------------------------------------ kernel timing
struct TimingState {
    std::mutex mu;
    bool on = false;
    uint32_t mask = 0;   // bit k set: launches of kind k are timed
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pending[KK_COUNT];
    cudaEvent_t open[KK_COUNT] = {};
    double total_ms[KK_COUNT] = {};
    uint64_t count[KK_COUNT] = {};
};
static TimingState g_timing;

static cudaEvent_t new_event() {
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// NVTX: every kernel kind's launches sit inside a host range named for the kind
// ("e4b.gemm_gateup", ...), and every entry point inside one named for itself, so a
// profiler can select them (ncu --nvtx --nvtx-include).  Without an attached tool
// the ranges cost a call through a no-op function pointer.
static const char* const kKindRange[KK_COUNT] = {
    "e4b.quantize", "e4b.dequantize", "e4b.route", "e4b.group", "e4b.gather", "e4b.combine",
    "e4b.gemm_gateup", "e4b.gemm_down", "e4b.gemm_dgrad_down", "e4b.gemm_dgrad_gateup",
    "e4b.decode_gateup", "e4b.decode_down"};
static_assert(KK_COUNT == 12, "one range name per kernel kind");

void timing_begin(int kind, cudaStream_t st) {
    nvtxRangePushA(kKindRange[kind]);
    std::lock_guard<std::mutex> lock(g_timing.mu);
    if (!g_timing.on || !((g_timing.mask >> kind) & 1u)) return;
    g_timing.open[kind] = new_event();
    cudaEventRecord(g_timing.open[kind], st);
}

NvtxScope::NvtxScope(const char* name) { nvtxRangePushA(name); }
NvtxScope::~NvtxScope() { nvtxRangePop(); }

void timing_end(int kind, cudaStream_t st) {
    nvtxRangePop();
    std::lock_guard<std::mutex> lock(g_timing.mu);
    if (!g_timing.on || !g_timing.open[kind]) return;
    cudaEvent_t e = new_event();
    cudaEventRecord(e, st);
    g_timing.pending[kind].emplace_back(g_timing.open[kind], e);
    g_timing.open[kind] = nullptr;
}

static void timing_collect() {
    for (int k = 0; k < KK_COUNT; ++k) {
        for (auto& pr : g_timing.pending[k]) {
            float ms = 0.0f;
            cudaEventSynchronize(pr.second);
            if (cudaEventElapsedTime(&ms, pr.first, pr.second) == cudaSuccess) {
                g_timing.total_ms[k] += ms;
                g_timing.count[k] += 1;
            }
            cudaEventDestroy(pr.first);
            cudaEventDestroy(pr.second);
        }
        g_timing.pending[k].clear();
    }
}

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cache[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cache[dev] = n > 0 ? n : 148;
    }
    return cache[dev];
}

// One status word per device, read and cleared by e4b_device_status.
__device__ uint32_t g_device_status;

uint32_t* device_status_ptr() {
    static uint32_t* cache[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_device_status) != cudaSuccess) return nullptr;
        cache[dev] = static_cast<uint32_t*>(ptr);
    }
    return cache[dev];
}

// ------------------------------------------------------------ workspace layout
struct WsLayout {
    size_t chunk_counts, chunk_base, counts, offsets, tile_prefix, sched, perm, inv_perm, a_perm, h, gu, dgu, dec, ones,
        dw_part, lz_gu, lz_d, lv_d, lv_gu, x_perm, lbt_gu, lbt_d, wbf16, total;
};

static size_t align_up(size_t v) { return (v + 255) & ~size_t(255); }

// n-tiles of the input-gradient down^T GEMM (N = I): the per-row dot products of
// the fused routing-weight gradient come one per n-tile.
static int dw_tiles(const e4b_moe_desc* d) { return (d->I + 255) / 256; }

static WsLayout layout_for(const e4b_moe_desc* d, int64_t T) {
    WsLayout L{};
    const int64_t P = T * d->top_k;
    const int64_t nch = (P + kChunkPairs - 1) / kChunkPairs;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
    L.chunk_counts = take((size_t)nch * d->E * 4);
    L.chunk_base = take((size_t)nch * d->E * 4);
    L.counts = take((size_t)d->E * 4);
    L.offsets = take((size_t)(d->E + 1) * 4);
    L.tile_prefix = take((size_t)(d->E + 1) * 4);
    L.sched = take(((size_t)(P + gemm_tile_rows() - 1) / gemm_tile_rows() + d->E) * 16);
    L.perm = take((size_t)P * 4);
    L.inv_perm = take((size_t)P * 4);
    L.a_perm = take((size_t)P * d->H * 2);
    L.h = take((size_t)P * d->I * 2);
    L.gu = take((size_t)P * 2 * d->I * 2);
    L.dgu = take((size_t)P * 2 * d->I * 2);
    L.dec = take(decode_scratch_bytes(d->E, d->H, d->I, T, d->top_k));
    L.ones = take((size_t)P * 4);
    L.dw_part = take((size_t)P * dw_tiles(d) * 4);
    if (d->lora_rank > 0) {   // the thin LoRA operands [P, 64] bf16 and the kept gathered x
        L.lz_gu = take((size_t)P * 64 * 2);
        L.lz_d = take((size_t)P * 64 * 2);
        L.lv_d = take((size_t)P * 64 * 2);
        L.lv_gu = take((size_t)P * 64 * 2);
        L.x_perm = take((size_t)P * d->H * 2);
        L.lbt_gu = take((size_t)d->E * d->lora_rank * 2 * d->I * 2);   // B_gu as [E, r, 2I]
        L.lbt_d = take((size_t)d->E * d->lora_rank * d->H * 2);        // B_d as [E, r, H]
    }
    if (d->codebook == E4B_CODEBOOK_INT8 || d->codebook == E4B_CODEBOOK_FP8)   // one stack dequantized to bf16
        L.wbf16 = take((size_t)d->E * std::max(2 * (int64_t)d->I * d->H, (int64_t)d->H * d->I) * 2);
    L.total = off;
    return L;
}

static e4b_status check_desc(const e4b_moe_desc* d) {
    if (!d) return E4B_ERR_INVALID_ARG;
    if (d->blocksize != (d->codebook == E4B_CODEBOOK_MXFP4 ? 32 : 64)) return E4B_ERR_BLOCKSIZE;
    if (d->codebook < E4B_CODEBOOK_NF4 || d->codebook > E4B_CODEBOOK_BF16) return E4B_ERR_INVALID_ARG;
    if (d->E < 1 || d->E > 256 || d->H <= 0 || d->I <= 0) return E4B_ERR_INVALID_ARG;
    if (d->H % 64 || d->I % 64) return E4B_ERR_BLOCKSIZE;
    if (d->top_k < 1 || d->top_k > 8 || d->top_k > d->E) return E4B_ERR_INVALID_ARG;
    if (d->path < E4B_PATH_AUTO || d->path > E4B_PATH_DECODE) return E4B_ERR_INVALID_ARG;
    if (d->activation != E4B_ACT_SWIGLU && d->activation != E4B_ACT_CLAMPED_GLU) return E4B_ERR_INVALID_ARG;
    if (d->activation == E4B_ACT_CLAMPED_GLU && (!std::isfinite(d->glu_alpha) || !(d->glu_limit > 0.0f)))
        return E4B_ERR_INVALID_ARG;
    if (d->lora_rank < 0 || d->lora_rank > 64 || d->lora_rank % 8) return E4B_ERR_INVALID_ARG;
    if (d->lora_rank > 0 && !std::isfinite(d->lora_scale)) return E4B_ERR_INVALID_ARG;
    return E4B_OK;
}

static e4b_status check_experts(const e4b_moe_desc* d, const e4b_experts* w) {
    if (!w || !w->gate_up || !w->down) return E4B_ERR_INVALID_ARG;
    if (d->codebook == E4B_CODEBOOK_MXFP4 ? (!w->gate_up_scales || !w->down_scales)
        : d->codebook == E4B_CODEBOOK_BF16 ? false
                                           : (!w->gate_up_absmax || !w->down_absmax))
        return E4B_ERR_INVALID_ARG;
    if (d->lora_rank > 0 && (!w->lora_A_gu || !w->lora_B_gu || !w->lora_A_d || !w->lora_B_d))
        return E4B_ERR_INVALID_ARG;
    return E4B_OK;
}

#define E4B_CUDA_TRY(expr)                              \
    do {                                                \
        if ((expr) != cudaSuccess) return E4B_ERR_CUDA; \
    } while (0)

static GemmParams base_params(const e4b_moe_desc* d, uint8_t* ws, const WsLayout& L, const float* topk_w,
                              int64_t P) {
    GemmParams p{};
    p.E = d->E;
    p.tile_prefix = reinterpret_cast<const int*>(ws + L.tile_prefix);
    p.sched = reinterpret_cast<const int4*>(ws + L.sched);
    p.perm = reinterpret_cast<const int*>(ws + L.perm);
    p.topk_w = topk_w;
    p.status = device_status_ptr();
    (void)P;
    return p;
}

// The grouped GEMMs' weight format: the 4-bit codebooks and MXFP4 are decoded in the
// dequantizing warps; the 8-bit codebooks are first dequantized to bf16 (one stack
// at a time, into ws.wbf16), and those and bf16 passthrough stacks are copied as is.
static int gemm_codebook(const e4b_moe_desc* d) { return d->codebook <= E4B_CODEBOOK_MXFP4 ? d->codebook : 3; }

// bf16 weights of one stack (gate_up when up, else down) for the GEMM, or null for
// the decoded formats.
static e4b_status stack_bf16(const e4b_moe_desc* d, const e4b_experts* w, bool up, uint8_t* ws, const WsLayout& L,
                             cudaStream_t st, const __nv_bfloat16** out) {
    *out = nullptr;
    if (d->codebook == E4B_CODEBOOK_BF16) {
        *out = static_cast<const __nv_bfloat16*>(static_cast<const void*>(up ? w->gate_up : w->down));
    } else if (d->codebook == E4B_CODEBOOK_INT8 || d->codebook == E4B_CODEBOOK_FP8) {
        const int64_t n = (int64_t)d->E * (up ? 2 * (int64_t)d->I * d->H : (int64_t)d->H * d->I);
        E4B_CUDA_TRY(launch_dequantize8(up ? w->gate_up : w->down, up ? w->gate_up_absmax : w->down_absmax, n,
                                        d->codebook, 1, ws + L.wbf16, st));
        *out = reinterpret_cast<const __nv_bfloat16*>(ws + L.wbf16);
    }
    return E4B_OK;
}

// MXFP4 stacks: the scale bytes of the stored matrix (cols = its row length).
static void set_mx(const e4b_moe_desc* d, const uint8_t* scales, int64_t cols, GemmParams* p) {
    if (d->codebook != E4B_CODEBOOK_MXFP4) return;
    p->mx_scales = scales;
    p->mx_stride = mxfp4_scale_stride(cols);
}

static int max_m_tiles(int64_t P, int E) { return (int)((P + gemm_tile_rows() - 1) / gemm_tile_rows()) + E; }

// Pairs grouped by expert into the workspace (counts, offsets, m-tile schedule, perm,
// inv_perm); debug builds then check the schedule's consistency.
static cudaError_t group_pairs(const e4b_moe_desc* d, const int32_t* topk_idx, int64_t P, uint8_t* ws,
                               const WsLayout& L, cudaStream_t st) {
    cudaError_t e = launch_group(topk_idx, P, d->E, gemm_tile_rows(), reinterpret_cast<int32_t*>(ws + L.chunk_counts),
                                 reinterpret_cast<int32_t*>(ws + L.chunk_base), reinterpret_cast<int32_t*>(ws + L.counts),
                                 reinterpret_cast<int32_t*>(ws + L.offsets), reinterpret_cast<int32_t*>(ws + L.tile_prefix),
                                 reinterpret_cast<int4*>(ws + L.sched), reinterpret_cast<int32_t*>(ws + L.perm),
                                 reinterpret_cast<int32_t*>(ws + L.inv_perm), st);
#if E4B_DEBUG_CHECKS
    if (e == cudaSuccess && P > 0)
        e = launch_validate_schedule(topk_idx, P, d->E, gemm_tile_rows(), reinterpret_cast<const int32_t*>(ws + L.counts),
                                     reinterpret_cast<const int32_t*>(ws + L.offsets),
                                     reinterpret_cast<const int32_t*>(ws + L.tile_prefix),
                                     reinterpret_cast<const int4*>(ws + L.sched), max_m_tiles(P, d->E),
                                     reinterpret_cast<const int32_t*>(ws + L.perm),
                                     reinterpret_cast<const int32_t*>(ws + L.inv_perm), st);
#endif
    return e;
}

static const __nv_bfloat16* bf(const void* p) { return static_cast<const __nv_bfloat16*>(p); }

// The thin LoRA operand out [P, 64] = s * in [P, K] M_e^T (M an A adapter [E, r, K]
// when q_major, else a B adapter [E, K, r]).
static e4b_status lora_thin(const e4b_moe_desc* d, uint8_t* ws, const WsLayout& L, int64_t P, const void* in, int K,
                            const void* m, bool q_major, size_t out_off, cudaStream_t st) {
    E4B_CUDA_TRY(launch_lora_thin(bf(in), K, bf(m), q_major, d->lora_rank, d->lora_scale,
                                  reinterpret_cast<const int4*>(ws + L.sched),
                                  reinterpret_cast<const int*>(ws + L.tile_prefix), d->E, max_m_tiles(P, d->E),
                                  reinterpret_cast<__nv_bfloat16*>(ws + out_off), st));
    return E4B_OK;
}

// gate_up GEMM + activation over the grouped rows a (ws.a_perm unless given); with
// adapters, the LoRA stage takes ws.lz_gu (made here from a) against B_gu.
static e4b_status run_gateup(const e4b_moe_desc* d, const e4b_experts* w, uint8_t* ws, const WsLayout& L,
                             const float* topk_w, int64_t P, __nv_bfloat16* h_out, __nv_bfloat16* gu_out,
                             cudaStream_t st, const void* a = nullptr) {
    if (!a) a = ws + L.a_perm;
    e4b_status s;
    if (d->lora_rank > 0 && (s = lora_thin(d, ws, L, P, a, d->H, w->lora_A_gu, true, L.lz_gu, st)) != E4B_OK)
        return s;
    GemmParams p = base_params(d, ws, L, topk_w, P);
    p.K = d->H;
    p.N = d->I;
    p.n_tiles = (d->I + 127) / 128;
    p.absmax = w->gate_up_absmax;
    p.b_rows_per_expert = 2 * d->I;
    p.b_rows_total = (int64_t)d->E * 2 * d->I;
    p.b_blocks_per_row = d->H / 64;
    set_mx(d, w->gate_up_scales, d->H, &p);
    p.up_offset = d->I;
    p.out_bf16 = h_out;
    p.gu = gu_out;
    p.ld_out = d->I;
    p.act = (int)d->activation;
    p.alpha = d->glu_alpha;
    p.limit = d->glu_limit;
    p.bias = w->gate_up_bias;
    p.lora_r = d->lora_rank;
    p.lora_b = bf(w->lora_B_gu);
    if ((s = stack_bf16(d, w, true, ws, L, st, &p.bf16_b)) != E4B_OK) return s;
    E4B_CUDA_TRY(launch_grouped_gemm(EPI_GATEUP, gemm_codebook(d), a, P, w->gate_up, p.b_rows_total, d->H / 2, p,
                                     max_m_tiles(P, d->E), st, d->lora_rank > 0 ? ws + L.lz_gu : nullptr));
    return E4B_OK;
}

// down GEMM over h [P, I] into the per-pair rows out (weights w applied); with
// adapters, the LoRA stage takes ws.lz_d = s h A_d^T (made here) against B_d.
static e4b_status run_down(const e4b_moe_desc* d, const e4b_experts* w, uint8_t* ws, const WsLayout& L,
                           const float* wts, int64_t P, const __nv_bfloat16* h, __nv_bfloat16* out,
                           cudaStream_t st) {
    e4b_status s;
    if (d->lora_rank > 0 && (s = lora_thin(d, ws, L, P, h, d->I, w->lora_A_d, true, L.lz_d, st)) != E4B_OK)
        return s;
    GemmParams p = base_params(d, ws, L, wts, P);
    p.K = d->I;
    p.N = d->H;
    p.n_tiles = (d->H + 255) / 256;
    p.absmax = w->down_absmax;
    p.b_rows_per_expert = d->H;
    p.b_rows_total = (int64_t)d->E * d->H;
    p.b_blocks_per_row = d->I / 64;
    set_mx(d, w->down_scales, d->I, &p);
    p.out_bf16 = out;
    p.bias = w->down_bias;
    p.ld_out = d->H;
    p.lora_r = d->lora_rank;
    p.lora_b = bf(w->lora_B_d);
    if ((s = stack_bf16(d, w, false, ws, L, st, &p.bf16_b)) != E4B_OK) return s;
    E4B_CUDA_TRY(launch_grouped_gemm(EPI_DOWN, gemm_codebook(d), h, P, w->down, p.b_rows_total, d->I / 2, p,
                                     max_m_tiles(P, d->E), st, d->lora_rank > 0 ? ws + L.lz_d : nullptr));
    return E4B_OK;
}

}  // namespace e4b

using namespace e4b;

extern "C" {

const char* e4b_status_string(e4b_status s) {
    switch (s) {
        case E4B_OK: return "ok";
        case E4B_ERR_INVALID_ARG: return "invalid argument";
        case E4B_ERR_BLOCKSIZE: return "blocksize must be 64 and divide in_features";
        case E4B_ERR_UNSUPPORTED: return "unsupported request";
        case E4B_ERR_WORKSPACE: return "workspace missing or too small";
        case E4B_ERR_CUDA: return "CUDA error";
        case E4B_ERR_TIMEOUT: return "device wait timed out";
        case E4B_ERR_DEBUG_CHECK: return "debug-build check failed";
    }
    return "unknown status";
}

uint64_t e4b_launch_count(void) { return g_launches.load(); }

void e4b_timing_enable(int on) { e4b_timing_enable_kinds(on ? 0xFFFFFFFFu : 0u); }

void e4b_timing_enable_kinds(uint32_t mask) {
    std::lock_guard<std::mutex> lock(g_timing.mu);
    timing_collect();
    for (int k = 0; k < KK_COUNT; ++k) {   // a kind switched off mid-launch drops its open event
        if (g_timing.open[k] && !((mask >> k) & 1u)) {
            cudaEventDestroy(g_timing.open[k]);
            g_timing.open[k] = nullptr;
        }
    }
    g_timing.mask = mask;
    g_timing.on = mask != 0;
}

void e4b_timing_reset(void) {
    std::lock_guard<std::mutex> lock(g_timing.mu);
    timing_collect();
    for (int k = 0; k < KK_COUNT; ++k) {
        g_timing.total_ms[k] = 0.0;
        g_timing.count[k] = 0;
    }
}

e4b_status e4b_timing_get(int kind, double* total_ms, uint64_t* launches) {
    if (kind < 0 || kind >= KK_COUNT || !total_ms || !launches) return E4B_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_timing.mu);
    timing_collect();
    *total_ms = g_timing.total_ms[kind];
    *launches = g_timing.count[kind];
    return E4B_OK;
}

static std::atomic<uint32_t> g_last_status_word{0};

e4b_status e4b_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return E4B_ERR_CUDA;
    uint32_t* ptr = device_status_ptr();
    if (!ptr) return E4B_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, ptr, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return E4B_ERR_CUDA;
    g_last_status_word.store(v);
    if (v) {
        const uint32_t zero = 0;
        if (cudaMemcpy(ptr, &zero, 4, cudaMemcpyHostToDevice) != cudaSuccess) return E4B_ERR_CUDA;
        return (v & kStatusTimeout) ? E4B_ERR_TIMEOUT : E4B_ERR_DEBUG_CHECK;
    }
    return E4B_OK;
}

uint32_t e4b_last_status_word(void) { return g_last_status_word.load(); }

int e4b_debug_checks(void) { return E4B_DEBUG_CHECKS; }

e4b_status e4b_debug_validate_schedule(const int32_t* topk_idx, int64_t P, int E, int tile_rows, const int32_t* counts,
                                       const int32_t* offsets, const int32_t* tile_prefix, const int32_t* sched,
                                       int64_t n_sched, const int32_t* perm, const int32_t* inv_perm, void* stream) {
    NvtxScope nvtx_scope("e4b_debug_validate_schedule");
    if (!topk_idx || !counts || !offsets || !tile_prefix || !sched || !perm || !inv_perm || P <= 0 || E <= 0 ||
        E > 256 || tile_rows <= 0 || n_sched < 0 || P > INT32_MAX)
        return E4B_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const e4b_status prior = e4b_device_status(stream);   // an earlier kernel's error comes first
    if (prior != E4B_OK) return prior;
    E4B_CUDA_TRY(launch_validate_schedule(topk_idx, P, E, tile_rows, counts, offsets, tile_prefix,
                                          reinterpret_cast<const int4*>(sched), n_sched, perm, inv_perm, st));
    return e4b_device_status(stream);
}

e4b_status e4b_quantize_nf4(const float* w, int64_t E, int64_t out, int64_t in, int blocksize, e4b_codebook cb,
                            uint8_t* packed, float* absmax, void* stream) {
    NvtxScope nvtx_scope("e4b_quantize_nf4");
    if (blocksize != 64) return E4B_ERR_BLOCKSIZE;
    if (E < 0 || out < 0 || in < 0) return E4B_ERR_INVALID_ARG;
    if (in % 64) return E4B_ERR_BLOCKSIZE;
    const bool eight = cb == E4B_CODEBOOK_INT8 || cb == E4B_CODEBOOK_FP8;
    if (cb != E4B_CODEBOOK_NF4 && cb != E4B_CODEBOOK_FP4 && !eight) return E4B_ERR_INVALID_ARG;
    const int64_t n = E * out * in;
    if (n == 0) return E4B_OK;
    if (!w || !packed || !absmax) return E4B_ERR_INVALID_ARG;
    if (eight) E4B_CUDA_TRY(launch_quantize8(w, n / 64, cb, packed, absmax, static_cast<cudaStream_t>(stream)));
    else E4B_CUDA_TRY(launch_quantize(w, n / 64, cb, packed, absmax, static_cast<cudaStream_t>(stream)));
    return E4B_OK;
}

int64_t e4b_mxfp4_scale_stride(int64_t in) { return in < 0 ? 0 : mxfp4_scale_stride(in); }

e4b_status e4b_quantize_mxfp4(const float* w, int64_t E, int64_t out, int64_t in, uint8_t* packed, uint8_t* scales,
                              void* stream) {
    NvtxScope nvtx_scope("e4b_quantize_mxfp4");
    if (E < 0 || out < 0 || in < 0) return E4B_ERR_INVALID_ARG;
    if (in % 32) return E4B_ERR_BLOCKSIZE;
    if (E * out * in == 0) return E4B_OK;
    if (!w || !packed || !scales) return E4B_ERR_INVALID_ARG;
    E4B_CUDA_TRY(launch_quantize_mxfp4(w, E * out, in, packed, scales, static_cast<cudaStream_t>(stream)));
    return E4B_OK;
}

e4b_status e4b_dequantize_mxfp4(const uint8_t* packed, const uint8_t* scales, int64_t E, int64_t out, int64_t in,
                                e4b_dtype out_dtype, void* w_out, void* stream) {
    NvtxScope nvtx_scope("e4b_dequantize_mxfp4");
    if (E < 0 || out < 0 || in < 0) return E4B_ERR_INVALID_ARG;
    if (in % 32) return E4B_ERR_BLOCKSIZE;
    if (out_dtype != E4B_F32 && out_dtype != E4B_BF16) return E4B_ERR_INVALID_ARG;
    if (E * out * in == 0) return E4B_OK;
    if (!packed || !scales || !w_out) return E4B_ERR_INVALID_ARG;
    E4B_CUDA_TRY(launch_dequantize_mxfp4(packed, scales, E * out, in, out_dtype == E4B_BF16, w_out,
                                         static_cast<cudaStream_t>(stream)));
    return E4B_OK;
}

e4b_status e4b_dequantize_nf4(const uint8_t* packed, const float* absmax, int64_t E, int64_t out, int64_t in,
                              int blocksize, e4b_codebook cb, e4b_dtype out_dtype, void* w_out, void* stream) {
    NvtxScope nvtx_scope("e4b_dequantize_nf4");
    if (blocksize != 64) return E4B_ERR_BLOCKSIZE;
    if (E < 0 || out < 0 || in < 0) return E4B_ERR_INVALID_ARG;
    if (in % 64) return E4B_ERR_BLOCKSIZE;
    const bool eight = cb == E4B_CODEBOOK_INT8 || cb == E4B_CODEBOOK_FP8;
    if (cb != E4B_CODEBOOK_NF4 && cb != E4B_CODEBOOK_FP4 && !eight) return E4B_ERR_INVALID_ARG;
    if (out_dtype != E4B_F32 && out_dtype != E4B_BF16) return E4B_ERR_INVALID_ARG;
    const int64_t n = E * out * in;
    if (n == 0) return E4B_OK;
    if (!packed || !absmax || !w_out) return E4B_ERR_INVALID_ARG;
    if (eight)
        E4B_CUDA_TRY(launch_dequantize8(packed, absmax, n, cb, out_dtype == E4B_BF16, w_out,
                                        static_cast<cudaStream_t>(stream)));
    else
        E4B_CUDA_TRY(launch_dequantize(packed, absmax, n, cb, out_dtype == E4B_BF16, w_out,
                                       static_cast<cudaStream_t>(stream)));
    return E4B_OK;
}

size_t e4b_moe_workspace_size(const e4b_moe_desc* d, int64_t T) {
    if (check_desc(d) != E4B_OK || T < 0) return 0;
    return layout_for(d, T).total;
}

e4b_status e4b_moe_forward(const e4b_moe_desc* d, const e4b_experts* w, const void* x, int64_t T,
                           const float* router_logits, int32_t* topk_idx, float* topk_w, void* y, void* saved_gu,
                           void* saved_h, int32_t* offsets_out, int32_t* perm_out, void* workspace, size_t ws_bytes,
                           void* stream) {
    NvtxScope nvtx_scope("e4b_moe_forward");
    e4b_status s = check_desc(d);
    if (s != E4B_OK) return s;
    if ((s = check_experts(d, w)) != E4B_OK) return s;
    if (T < 0 || T * d->top_k > (int64_t)INT32_MAX) return E4B_ERR_INVALID_ARG;
    if (T == 0) return E4B_OK;
    if (!x || !topk_idx || !topk_w || !y) return E4B_ERR_INVALID_ARG;
    const WsLayout L = layout_for(d, T);
    if (!workspace || ws_bytes < L.total) return E4B_ERR_WORKSPACE;
    const bool want_grouped_outputs = saved_gu || saved_h || offsets_out || perm_out;
    // the decode kernels implement SwiGLU without biases
    const bool plain_experts = d->activation == E4B_ACT_SWIGLU && !w->gate_up_bias && !w->down_bias &&
                               d->lora_rank == 0 && d->codebook <= E4B_CODEBOOK_FP4;
    const bool dec_ok = !want_grouped_outputs && plain_experts && decode_supported(d->E, d->H, d->I, T, d->top_k);
    const bool decode = (d->path == E4B_PATH_DECODE) || (d->path == E4B_PATH_AUTO && dec_ok);
    if (d->path == E4B_PATH_DECODE && !dec_ok) return E4B_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int64_t P = T * d->top_k;

    if (decode) {   // routing, gate_up and down in two kernels
        E4B_CUDA_TRY(launch_decode_forward(d->codebook, d->E, d->H, d->I, d->top_k, d->renormalize, T,
                                           static_cast<const __nv_bfloat16*>(x), router_logits, topk_idx, topk_w,
                                           w->gate_up, w->gate_up_absmax, w->down, w->down_absmax, ws + L.dec,
                                           static_cast<__nv_bfloat16*>(y), st));
        return E4B_OK;
    }
    if (router_logits)
        E4B_CUDA_TRY(launch_route(router_logits, T, d->E, d->top_k, d->renormalize, topk_idx, topk_w, st));

    int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
    int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
    E4B_CUDA_TRY(group_pairs(d, topk_idx, P, ws, L, st));
    E4B_CUDA_TRY(launch_gather_rows(static_cast<const __nv_bfloat16*>(x), perm, offsets + d->E, d->top_k, P, d->H,
                                    reinterpret_cast<__nv_bfloat16*>(ws + L.a_perm), st));
    // h goes straight to the caller's saved_h when asked for (the down GEMM reads it there)
    __nv_bfloat16* h = saved_h ? static_cast<__nv_bfloat16*>(saved_h) : reinterpret_cast<__nv_bfloat16*>(ws + L.h);
    __nv_bfloat16* slots = reinterpret_cast<__nv_bfloat16*>(ws + L.a_perm);   // X_perm is dead after gate_up
    if ((s = run_gateup(d, w, ws, L, topk_w, P, h, static_cast<__nv_bfloat16*>(saved_gu), st)) != E4B_OK) return s;

    if ((s = run_down(d, w, ws, L, topk_w, P, h, slots, st)) != E4B_OK) return s;
    E4B_CUDA_TRY(launch_combine(slots, reinterpret_cast<const int32_t*>(ws + L.inv_perm), d->top_k, T, d->H,
                                static_cast<__nv_bfloat16*>(y), st));
    if (offsets_out) E4B_CUDA_TRY(cudaMemcpyAsync(offsets_out, offsets, (d->E + 1) * 4, cudaMemcpyDeviceToDevice, st));
    if (perm_out) E4B_CUDA_TRY(cudaMemcpyAsync(perm_out, perm, P * 4, cudaMemcpyDeviceToDevice, st));
    return E4B_OK;
}

e4b_status e4b_moe_backward(const e4b_moe_desc* d, const e4b_experts* w, const void* x, int64_t T,
                            const float* router_logits, const int32_t* topk_idx, const float* topk_w,
                            const void* grad_out, const void* saved_gu, const void* saved_h, void* grad_x,
                            float* grad_topk_w, float* grad_logits, const e4b_lora_grads* lora_grads,
                            void* workspace, size_t ws_bytes, void* stream) {
    NvtxScope nvtx_scope("e4b_moe_backward");
    e4b_status s = check_desc(d);
    if (s != E4B_OK) return s;
    if ((s = check_experts(d, w)) != E4B_OK) return s;
    if (T < 0 || T * d->top_k > (int64_t)INT32_MAX) return E4B_ERR_INVALID_ARG;
    if (T == 0) return E4B_OK;
    const bool lg = d->lora_rank > 0 && lora_grads;   // adapter gradients asked for
    if (lg && (!lora_grads->dA_gu || !lora_grads->dB_gu || !lora_grads->dA_d || !lora_grads->dB_d))
        return E4B_ERR_INVALID_ARG;
    if (!topk_idx || !topk_w || !grad_out || (!grad_x && !grad_topk_w && !lg)) return E4B_ERR_INVALID_ARG;
    if (!saved_gu && !x) return E4B_ERR_INVALID_ARG;                            // nothing to recompute from
    if ((grad_topk_w || lg) && saved_gu && !saved_h) return E4B_ERR_INVALID_ARG;   // h saved with the derivatives
    if (lg && !x) return E4B_ERR_INVALID_ARG;                                   // dA_gu contracts with x
    if (grad_logits && (!router_logits || !grad_topk_w)) return E4B_ERR_INVALID_ARG;
    const WsLayout L = layout_for(d, T);
    if (!workspace || ws_bytes < L.total) return E4B_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int64_t P = T * d->top_k;
    const bool lora = d->lora_rank > 0;
    int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
    const int32_t* inv_perm = reinterpret_cast<const int32_t*>(ws + L.inv_perm);
    const int32_t* offsets = reinterpret_cast<const int32_t*>(ws + L.offsets);
    E4B_CUDA_TRY(group_pairs(d, topk_idx, P, ws, L, st));
    __nv_bfloat16* a_perm = reinterpret_cast<__nv_bfloat16*>(ws + L.a_perm);
    const int32_t* nrows = offsets + d->E;
    const __nv_bfloat16* gu = static_cast<const __nv_bfloat16*>(saved_gu);
    const __nv_bfloat16* h = static_cast<const __nv_bfloat16*>(saved_h);
    // the gathered x: kept in its own buffer when the adapters need it to the end
    __nv_bfloat16* xg = lora ? reinterpret_cast<__nv_bfloat16*>(ws + L.x_perm) : a_perm;
    if (!gu || lg) {
        E4B_CUDA_TRY(launch_gather_rows(bf(x), perm, nrows, d->top_k, P, d->H, xg, st));
        // s x A_gu^T for dB_gu (recompute mode makes it inside run_gateup)
        if (gu && (s = lora_thin(d, ws, L, P, xg, d->H, w->lora_A_gu, true, L.lz_gu, st)) != E4B_OK) return s;
    }
    if (!gu) {   // recompute the gate/up pre-activations (and h) from x
        __nv_bfloat16* gu_ws = reinterpret_cast<__nv_bfloat16*>(ws + L.gu);
        __nv_bfloat16* h_ws = reinterpret_cast<__nv_bfloat16*>(ws + L.h);
        if ((s = run_gateup(d, w, ws, L, topk_w, P, h_ws, gu_ws, st, xg)) != E4B_OK) return s;
        gu = gu_ws;
        h = h_ws;
    }
    if (lg && (s = lora_thin(d, ws, L, P, h, d->I, w->lora_A_d, true, L.lz_d, st)) != E4B_OK) return s;
    E4B_CUDA_TRY(launch_gather_rows(bf(grad_out), perm, nrows, d->top_k, P, d->H, a_perm, st));
    // LoRA: the down^T GEMM's extra stage is s (grad_out B_d) against A_d (B_d transposed first)
    if (lora) {
        E4B_CUDA_TRY(launch_lora_transpose(bf(w->lora_B_d), d->E, d->H, d->lora_rank,
                                           reinterpret_cast<__nv_bfloat16*>(ws + L.lbt_d), st));
        if ((s = lora_thin(d, ws, L, P, a_perm, d->H, ws + L.lbt_d, true, L.lv_d, st)) != E4B_OK) return s;
    }
    __nv_bfloat16* dgu = reinterpret_cast<__nv_bfloat16*>(ws + L.dgu);

    // dh = w * grad_out W_down (+ the adapter term), then the activation backward; with
    // grad_topk_w the epilogue also leaves <grad_out W_down, h> per row and n-tile
    GemmParams p = base_params(d, ws, L, topk_w, P);
    p.K = d->H;
    p.N = d->I;
    p.n_tiles = dw_tiles(d);
    p.absmax = w->down_absmax;
    p.b_rows_per_expert = d->H;
    p.b_rows_total = (int64_t)d->E * d->H;
    p.b_blocks_per_row = d->I / 64;
    set_mx(d, w->down_scales, d->I, &p);
    p.gu = const_cast<__nv_bfloat16*>(gu);
    p.out_bf16 = dgu;
    p.ld_out = 2 * d->I;
    p.lora_r = d->lora_rank;
    p.lora_b = bf(w->lora_A_d);
    float* dw_part = reinterpret_cast<float*>(ws + L.dw_part);
    if (grad_topk_w) {
        p.h_in = h;
        p.dw_part = dw_part;
    }
    if ((s = stack_bf16(d, w, false, ws, L, st, &p.bf16_b)) != E4B_OK) return s;
    E4B_CUDA_TRY(launch_grouped_gemm(EPI_DGRAD_DOWN, gemm_codebook(d), a_perm, P, w->down, p.b_rows_total, d->I / 2,
                                     p, max_m_tiles(P, d->E), st, lora ? ws + L.lv_d : nullptr));
    if (grad_topk_w)
        E4B_CUDA_TRY(launch_router_grad_parts(bf(grad_out), dw_part, dw_tiles(d), w->down_bias, inv_perm, topk_idx,
                                              topk_w, router_logits, T, d->E, d->top_k, d->H, d->renormalize,
                                              grad_topk_w, grad_logits, st));
    if (lg) {   // down adapter: dB_d = sum w g (x) s z_d,  dA_d = sum w s (g B_d) (x) h
        const __nv_bfloat16* lzd = reinterpret_cast<const __nv_bfloat16*>(ws + L.lz_d);
        const __nv_bfloat16* lvd = reinterpret_cast<const __nv_bfloat16*>(ws + L.lv_d);
        E4B_CUDA_TRY(launch_lora_grad(a_perm, d->H, lzd, d->lora_rank, offsets, d->E, topk_w, perm, true, false,
                                      lora_grads->dB_d, st));
        E4B_CUDA_TRY(launch_lora_grad(h, d->I, lvd, d->lora_rank, offsets, d->E, topk_w, perm, true, true,
                                      lora_grads->dA_d, st));
    }
    // LoRA: the gate_up^T GEMM's extra stage is s (dGU B_gu) against A_gu
    if (lora && (grad_x || lg)) {
        E4B_CUDA_TRY(launch_lora_transpose(bf(w->lora_B_gu), d->E, 2 * d->I, d->lora_rank,
                                           reinterpret_cast<__nv_bfloat16*>(ws + L.lbt_gu), st));
        if ((s = lora_thin(d, ws, L, P, dgu, 2 * d->I, ws + L.lbt_gu, true, L.lv_gu, st)) != E4B_OK) return s;
    }
    if (lg) {   // gate_up adapter: dB_gu = sum dGU (x) s z_gu,  dA_gu = sum s (dGU B_gu) (x) x
        const __nv_bfloat16* lzg = reinterpret_cast<const __nv_bfloat16*>(ws + L.lz_gu);
        const __nv_bfloat16* lvg = reinterpret_cast<const __nv_bfloat16*>(ws + L.lv_gu);
        E4B_CUDA_TRY(launch_lora_grad(dgu, 2 * d->I, lzg, d->lora_rank, offsets, d->E, topk_w, perm, false, false,
                                      lora_grads->dB_gu, st));
        E4B_CUDA_TRY(launch_lora_grad(xg, d->H, lvg, d->lora_rank, offsets, d->E, topk_w, perm, false, true,
                                      lora_grads->dA_gu, st));
    }
    if (!grad_x) return E4B_OK;

    GemmParams q = base_params(d, ws, L, topk_w, P);   // grad_x += [dG, dU] W_gate_up (+ the adapter term)
    q.K = 2 * d->I;
    q.N = d->H;
    q.n_tiles = (d->H + 255) / 256;
    q.absmax = w->gate_up_absmax;
    q.b_rows_per_expert = 2 * d->I;
    q.b_rows_total = (int64_t)d->E * 2 * d->I;
    q.b_blocks_per_row = d->H / 64;
    set_mx(d, w->gate_up_scales, d->H, &q);
    q.out_bf16 = a_perm;   // per-pair rows in grouped order; the gathered grad_out is dead by now
    q.ld_out = d->H;
    q.lora_r = d->lora_rank;
    q.lora_b = bf(w->lora_A_gu);
    if ((s = stack_bf16(d, w, true, ws, L, st, &q.bf16_b)) != E4B_OK) return s;
    E4B_CUDA_TRY(launch_grouped_gemm(EPI_DGRAD_GATEUP, gemm_codebook(d), dgu, P, w->gate_up, q.b_rows_total, d->H / 2,
                                     q, max_m_tiles(P, d->E), st, lora ? ws + L.lv_gu : nullptr));
    E4B_CUDA_TRY(launch_combine(a_perm, inv_perm, d->top_k, T, d->H, static_cast<__nv_bfloat16*>(grad_x), st));
    return E4B_OK;
}

e4b_status e4b_moe_backward_dgrad(const e4b_moe_desc* d, const e4b_experts* w, const void* x, int64_t T,
                                  const int32_t* topk_idx, const float* topk_w, const void* grad_out,
                                  const void* saved_gu, void* grad_x, void* workspace, size_t ws_bytes,
                                  void* stream) {
    NvtxScope nvtx_scope("e4b_moe_backward_dgrad");
    if (T > 0 && !grad_x) return E4B_ERR_INVALID_ARG;
    return e4b_moe_backward(d, w, x, T, nullptr, topk_idx, topk_w, grad_out, saved_gu, nullptr, grad_x, nullptr,
                            nullptr, nullptr, workspace, ws_bytes, stream);
}

e4b_status e4b_moe_backward_router(const e4b_moe_desc* d, const e4b_experts* w, const void* x, int64_t T,
                                   const float* router_logits, const int32_t* topk_idx, const float* topk_w,
                                   const void* grad_out, float* grad_topk_w, float* grad_logits, void* workspace,
                                   size_t ws_bytes, void* stream) {
    NvtxScope nvtx_scope("e4b_moe_backward_router");
    e4b_status s = check_desc(d);
    if (s != E4B_OK) return s;
    if ((s = check_experts(d, w)) != E4B_OK) return s;
    if (T < 0 || T * d->top_k > (int64_t)INT32_MAX) return E4B_ERR_INVALID_ARG;
    if (T == 0) return E4B_OK;
    if (!x || !topk_idx || !topk_w || !grad_out || !grad_topk_w || (grad_logits && !router_logits))
        return E4B_ERR_INVALID_ARG;
    const WsLayout L = layout_for(d, T);
    if (!workspace || ws_bytes < L.total) return E4B_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int64_t P = T * d->top_k;
    // h recomputed through the grouped gate_up GEMM, then the unweighted expert
    // outputs Y (the down GEMM with unit weights), one grouped row per pair
    int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
    E4B_CUDA_TRY(group_pairs(d, topk_idx, P, ws, L, st));
    const int32_t* nrows = reinterpret_cast<const int32_t*>(ws + L.offsets) + d->E;
    __nv_bfloat16* a_perm = reinterpret_cast<__nv_bfloat16*>(ws + L.a_perm);
    E4B_CUDA_TRY(launch_gather_rows(static_cast<const __nv_bfloat16*>(x), perm, nrows, d->top_k, P, d->H, a_perm, st));
    __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(ws + L.h);
    if ((s = run_gateup(d, w, ws, L, topk_w, P, h, nullptr, st)) != E4B_OK) return s;
    float* ones = reinterpret_cast<float*>(ws + L.ones);
    E4B_CUDA_TRY(launch_fill_f32(ones, P, 1.0f, st));
    if ((s = run_down(d, w, ws, L, ones, P, h, a_perm, st)) != E4B_OK) return s;   // Y, one grouped row per pair
    E4B_CUDA_TRY(launch_router_grad(static_cast<const __nv_bfloat16*>(grad_out), a_perm,
                                    reinterpret_cast<const int32_t*>(ws + L.inv_perm), topk_idx, topk_w,
                                    router_logits, T, d->E, d->top_k, d->H, d->renormalize, grad_topk_w, grad_logits,
                                    st));
    return E4B_OK;
}

}  // extern "C"
