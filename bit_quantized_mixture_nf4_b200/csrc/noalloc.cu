// e4b_moe_forward_noalloc: the expert-layer forward for callers that cannot give
// the library device memory.
//
// Who needs it: a caller whose device memory is handed out by its own fixed
// pool, reserved up front (a serving engine that claims all free memory for its
// caches at start-up, or a process held to a hard memory budget), and a caller in
// a latency-critical loop where a per-call cudaMalloc is out of the question
// (allocation can stall or synchronize the device; cudaFree synchronizes it).
// Such callers can pass inputs and outputs they own, but no scratch.
//
// This entry point runs the same launch sequence as e4b_moe_forward, with its
// scratch in a file-scope device array instead of a caller workspace.  It
// allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
#include <mutex>

#include "../../include/e4b.h"
#include "e4b_internal.h"

namespace {

// Largest scratch the no-allocation forward may use.  The array is part of the
// library's device image: every GPU that loads the library holds it until the
// process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;   // 32 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name only stands in for the symbol (it is not a device address), so the
// address is looked up with cudaGetSymbolAddress once per device, with that
// device current, and cached.
void* noalloc_scratch(e4b_status* st) {
    static void* cache[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        *st = E4B_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        void* ptr = nullptr;
        const cudaError_t err = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (err != cudaSuccess || ptr == nullptr) {
            *st = E4B_ERR_CUDA;
            return nullptr;
        }
        cache[dev] = ptr;
    }
    return cache[dev];
}

}  // namespace

extern "C" e4b_status e4b_moe_forward_noalloc(const e4b_moe_desc* d, const e4b_experts* w, const void* x, int64_t T,
                                              const float* router_logits, int32_t* topk_idx, float* topk_w, void* y,
                                              void* stream) {
    e4b::NvtxScope nvtx_scope("e4b_moe_forward_noalloc");
    // Size check first, on the host: nothing is touched for a request that does not fit.
    const size_t need = e4b_moe_workspace_size(d, T);
    if (T > 0 && need > kNoAllocScratchBytes) return E4B_ERR_WORKSPACE;
    e4b_status st = E4B_OK;
    void* scratch = noalloc_scratch(&st);
    if (!scratch) return st;
    // Every byte of the scratch the forward reads is written earlier in the same
    // call, so nothing has to be cleared between calls.
    return e4b_moe_forward(d, w, x, T, router_logits, topk_idx, topk_w, y, nullptr, nullptr, nullptr, nullptr, scratch,
                           kNoAllocScratchBytes, stream);
}
