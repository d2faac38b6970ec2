// Pipelined steps through pinned host buffers (e4b_pipe_*, declared in
// include/e4b.h).
//
// One expert-layer training step (forward routed from router logits, g/u saved,
// then the input gradient with routing held -- "experts4bit-qlora 0.1.0"
// experts.py, Experts4bit.forward, and the recompute-in-backward input gradient
// of bitsandbytes pull request #1965, section "What this adds") for batches that
// live in host memory.  Three streams: copy-in, the caller's compute stream and
// copy-out.  Two device buffer sets alternate, so while batch n's kernels run,
// batch n+1's inputs come in and batch n-1's outputs go out:
//
//   copy-in   [x,l,g](n+1) ......................... [x,l,g](n+2) ...
//   compute   ... fwd(n) ---- dgrad(n) ---- fwd(n+1) ---- dgrad(n+1) ...
//   copy-out  ...  gx(n-1) .......... y(n) ... gx(n) ........ y(n+1) ...
//
// Set b is refilled only after the compute stream is done with it (event
// done[b]) and overwritten by the compute stream only after its previous
// outputs were copied out (event out_done[b]).  The saved g/u and the workspace
// are shared: the compute stream runs the steps one after another.
#include <cuda_runtime.h>

#include <new>

#include <nvtx3/nvToolsExt.h>

#include "../../include/e4b.h"

struct e4b_pipe {
    e4b_moe_desc d;
    e4b_experts w;
    int64_t T_max;
    void* x[2];
    float* logits[2];
    void* go[2];
    void* y[2];
    void* gx[2];
    int32_t* idx[2];
    float* wts[2];
    void* saved;
    void* ws;
    size_t ws_bytes;
    cudaStream_t compute, cin, cout;
    cudaEvent_t in_ready[2], y_ready[2], done[2], out_done[2];
    cudaEvent_t join_in, join_out, fork;
    bool used[2];
    uint64_t n;
};

namespace {

// NVTX range over a submission's host scope (the library's other entry points open
// their own inside it)
struct PipeRange {
    explicit PipeRange(const char* name) { nvtxRangePushA(name); }
    ~PipeRange() { nvtxRangePop(); }
};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Byte offsets of every buffer in the arena for T_max tokens.
struct PipeLayout {
    size_t x[2], logits[2], go[2], y[2], gx[2], idx[2], wts[2], saved, ws, ws_bytes, total;
};

bool pipe_layout(const e4b_moe_desc* d, int64_t T, PipeLayout* L) {
    const size_t ws = e4b_moe_workspace_size(d, T);
    if (ws == 0) return false;   // invalid descriptor
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    const size_t H = (size_t)d->H, E = (size_t)d->E, k = (size_t)d->top_k, I = (size_t)d->I, t = (size_t)T;
    for (int b = 0; b < 2; ++b) {
        L->x[b] = take(t * H * 2);
        L->logits[b] = take(t * E * 4);
        L->go[b] = take(t * H * 2);
        L->y[b] = take(t * H * 2);
        L->gx[b] = take(t * H * 2);
        L->idx[b] = take(t * k * 4);
        L->wts[b] = take(t * k * 4);
    }
    L->saved = take(t * k * 2 * I * 2);
    L->ws = take(ws);
    L->ws_bytes = ws;
    L->total = off;
    return true;
}

}  // namespace

#define PIPE_TRY(expr)                                    \
    do {                                                  \
        if ((expr) != cudaSuccess) return E4B_ERR_CUDA;   \
    } while (0)

extern "C" {

size_t e4b_pipe_arena_size(const e4b_moe_desc* d, int64_t T_max) {
    PipeLayout L;
    if (!d || T_max < 0 || !pipe_layout(d, T_max, &L)) return 0;
    return L.total;
}

e4b_status e4b_pipe_create(const e4b_moe_desc* d, const e4b_experts* w, int64_t T_max, void* arena,
                           size_t arena_bytes, void* stream, e4b_pipe** out) {
    if (!out) return E4B_ERR_INVALID_ARG;
    *out = nullptr;
    if (!d || !w || !arena || T_max < 0 || T_max * d->top_k > (int64_t)INT32_MAX) return E4B_ERR_INVALID_ARG;
    if (!w->gate_up || !w->down || !w->gate_up_absmax || !w->down_absmax) return E4B_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(arena) & 255) return E4B_ERR_INVALID_ARG;
    PipeLayout L;
    if (!pipe_layout(d, T_max, &L)) return E4B_ERR_INVALID_ARG;
    if (arena_bytes < L.total) return E4B_ERR_WORKSPACE;
    e4b_pipe* p = new (std::nothrow) e4b_pipe();
    if (!p) return E4B_ERR_CUDA;
    p->d = *d;
    p->w = *w;
    p->T_max = T_max;
    uint8_t* a = static_cast<uint8_t*>(arena);
    for (int b = 0; b < 2; ++b) {
        p->x[b] = a + L.x[b];
        p->logits[b] = reinterpret_cast<float*>(a + L.logits[b]);
        p->go[b] = a + L.go[b];
        p->y[b] = a + L.y[b];
        p->gx[b] = a + L.gx[b];
        p->idx[b] = reinterpret_cast<int32_t*>(a + L.idx[b]);
        p->wts[b] = reinterpret_cast<float*>(a + L.wts[b]);
    }
    p->saved = a + L.saved;
    p->ws = a + L.ws;
    p->ws_bytes = L.ws_bytes;
    p->compute = static_cast<cudaStream_t>(stream);
    bool ok = cudaStreamCreateWithFlags(&p->cin, cudaStreamNonBlocking) == cudaSuccess;
    ok = ok && cudaStreamCreateWithFlags(&p->cout, cudaStreamNonBlocking) == cudaSuccess;
    cudaEvent_t* evs[] = {&p->in_ready[0], &p->in_ready[1], &p->y_ready[0], &p->y_ready[1], &p->done[0],
                          &p->done[1],     &p->out_done[0], &p->out_done[1], &p->join_in, &p->join_out,
                          &p->fork};
    for (cudaEvent_t* e : evs) ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        e4b_pipe_destroy(p);
        return E4B_ERR_CUDA;
    }
    *out = p;
    return E4B_OK;
}

e4b_status e4b_pipe_submit(e4b_pipe* p, int64_t T, const void* x_host, const float* logits_host,
                           const void* grad_out_host, void* y_host, void* grad_x_host) {
    PipeRange nvtx_scope("e4b_pipe_submit");
    if (!p || T < 0 || T > p->T_max) return E4B_ERR_INVALID_ARG;
    if (T == 0) return E4B_OK;
    if (!x_host || !logits_host || !grad_out_host || !y_host || !grad_x_host) return E4B_ERR_INVALID_ARG;
    const int b = (int)(p->n & 1);
    const size_t row_bytes = (size_t)T * p->d.H * 2, logit_bytes = (size_t)T * p->d.E * 4;
    // inputs of set b: refilled once the compute stream is done with the batch before last
    if (p->used[b]) PIPE_TRY(cudaStreamWaitEvent(p->cin, p->done[b], 0));
    PIPE_TRY(cudaMemcpyAsync(p->logits[b], logits_host, logit_bytes, cudaMemcpyHostToDevice, p->cin));
    PIPE_TRY(cudaMemcpyAsync(p->x[b], x_host, row_bytes, cudaMemcpyHostToDevice, p->cin));
    PIPE_TRY(cudaMemcpyAsync(p->go[b], grad_out_host, row_bytes, cudaMemcpyHostToDevice, p->cin));
    PIPE_TRY(cudaEventRecord(p->in_ready[b], p->cin));
    // kernels: after the inputs landed and set b's previous outputs left
    PIPE_TRY(cudaStreamWaitEvent(p->compute, p->in_ready[b], 0));
    if (p->used[b]) PIPE_TRY(cudaStreamWaitEvent(p->compute, p->out_done[b], 0));
    e4b_status s = e4b_moe_forward(&p->d, &p->w, p->x[b], T, p->logits[b], p->idx[b], p->wts[b], p->y[b], p->saved,
                                   nullptr, nullptr, nullptr, p->ws, p->ws_bytes, p->compute);
    if (s != E4B_OK) return s;
    PIPE_TRY(cudaEventRecord(p->y_ready[b], p->compute));
    s = e4b_moe_backward_dgrad(&p->d, &p->w, p->x[b], T, p->idx[b], p->wts[b], p->go[b], p->saved, p->gx[b], p->ws,
                               p->ws_bytes, p->compute);
    if (s != E4B_OK) return s;
    PIPE_TRY(cudaEventRecord(p->done[b], p->compute));
    // outputs: y under the input gradient's kernels, grad_x after them
    PIPE_TRY(cudaStreamWaitEvent(p->cout, p->y_ready[b], 0));
    PIPE_TRY(cudaMemcpyAsync(y_host, p->y[b], row_bytes, cudaMemcpyDeviceToHost, p->cout));
    PIPE_TRY(cudaStreamWaitEvent(p->cout, p->done[b], 0));
    PIPE_TRY(cudaMemcpyAsync(grad_x_host, p->gx[b], row_bytes, cudaMemcpyDeviceToHost, p->cout));
    PIPE_TRY(cudaEventRecord(p->out_done[b], p->cout));
    p->used[b] = true;
    ++p->n;
    return E4B_OK;
}

e4b_status e4b_pipe_join(e4b_pipe* p) {
    if (!p) return E4B_ERR_INVALID_ARG;
    // compute waits for every copy submitted so far ...
    PIPE_TRY(cudaEventRecord(p->join_in, p->cin));
    PIPE_TRY(cudaEventRecord(p->join_out, p->cout));
    PIPE_TRY(cudaStreamWaitEvent(p->compute, p->join_in, 0));
    PIPE_TRY(cudaStreamWaitEvent(p->compute, p->join_out, 0));
    // ... and later copies wait for what is on the compute stream now
    PIPE_TRY(cudaEventRecord(p->fork, p->compute));
    PIPE_TRY(cudaStreamWaitEvent(p->cin, p->fork, 0));
    PIPE_TRY(cudaStreamWaitEvent(p->cout, p->fork, 0));
    return E4B_OK;
}

e4b_status e4b_pipe_sync(e4b_pipe* p) {
    const e4b_status s = e4b_pipe_join(p);
    if (s != E4B_OK) return s;
    return e4b_device_status(p->compute);
}

void e4b_pipe_destroy(e4b_pipe* p) {
    if (!p) return;
    if (p->cin) cudaStreamSynchronize(p->cin);
    if (p->cout) cudaStreamSynchronize(p->cout);
    cudaStreamSynchronize(p->compute);
    cudaEvent_t evs[] = {p->in_ready[0], p->in_ready[1], p->y_ready[0], p->y_ready[1], p->done[0], p->done[1],
                         p->out_done[0], p->out_done[1], p->join_in, p->join_out, p->fork};
    for (cudaEvent_t e : evs)
        if (e) cudaEventDestroy(e);
    if (p->cin) cudaStreamDestroy(p->cin);
    if (p->cout) cudaStreamDestroy(p->cout);
    delete p;
}

}  // extern "C"
