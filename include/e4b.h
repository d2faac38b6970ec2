/*
 * e4b.h -- C ABI of the e4b library: the NF4 (and FP4) quantized Mixture-of-
 * Experts expert path on NVIDIA B200 (sm_100a).
 *
 * The operations follow the expert-layer pages:
 *   [P4] "experts4bit-qlora 0.1.0" source diff, file _vendor/experts.py, class
 *        Experts4bit: __init__ (storage layout and validation), from_float and
 *        _quantize_stack (quantize), _dequantize_expert (dequantize), forward.
 *   [P5] bitsandbytes pull request #1965 "Add Experts4bit for 4-bit quantization
 *        of fused MoE experts", section "What this adds" (recompute-in-backward
 *        input gradient, frozen base).
 *   [P2] "experts4bit-qlora 0.31.1" PyPI project page, section "Scope": the
 *        gpt-oss experts (per-expert biases and a clamped GLU).
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *     row-major, 16-byte aligned.  The library allocates nothing.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are stream-ordered and asynchronous.
 *   - Argument errors are detected on the host before any launch and return a
 *     status without touching memory.  Launch failures return E4B_ERR_CUDA.
 *   - Device-side waits in the grouped GEMM carry a time limit; if one expires
 *     the kernel records it in a device status word and exits without trapping;
 *     e4b_device_status() reports it as E4B_ERR_TIMEOUT.
 *   - There is no CPU fallback: without a usable sm_100a device every compute
 *     call returns E4B_ERR_CUDA.
 *
 * Storage of one weight stack [E, out, in] (gate_up: out = 2I, in = H, gate
 * rows first; down: out = H, in = I):
 *   packed  uint8 [E, out*in/2]   element 2b of an expert's row-major [out, in]
 *                                 matrix in the HIGH nibble of byte b, element
 *                                 2b+1 in the low nibble;
 *   absmax  fp32  [E, out*in/64]  block j of row o at o*in/64 + j.
 * Codes index the 16-value codebook (NF4: ascending NormalFloat values, code 7
 * = 0; FP4: sign in bit 3, e2m1 magnitude / 6 in bits 2..0).
 */
#ifndef E4B_H_
#define E4B_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define E4B_API __attribute__((visibility("default")))
#else
#define E4B_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    E4B_OK = 0,
    E4B_ERR_INVALID_ARG = 1,   /* null pointer, negative or unsupported size, k > E ... */
    E4B_ERR_BLOCKSIZE = 2,     /* in_features % blocksize != 0, or blocksize != 64      */
    E4B_ERR_UNSUPPORTED = 3,   /* valid request outside what the kernels implement       */
    E4B_ERR_WORKSPACE = 4,     /* workspace NULL or smaller than e4b_moe_workspace_size  */
    E4B_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed                    */
    E4B_ERR_TIMEOUT = 6,       /* a device-side wait hit its time limit                   */
    E4B_ERR_DEBUG_CHECK = 7    /* a debug-build bounds or consistency check failed        */
} e4b_status;

/* NF4 / FP4: 64-element blocks with an fp32 absmax (the 4-bit stacks above).
 * MXFP4: the gpt-oss experts' native storage ([P2] "Scope"), read as the OCP
 * Microscaling Formats v1.0 MXFP4: 32-element blocks sharing an E8M0 scale
 * 2^(s - 127) (one byte s), FP4 E2M1 elements (sign in bit 3, magnitudes
 * {0, .5, 1, 1.5, 2, 3, 4, 6}), packed like the 4-bit stacks; scales uint8
 * [E, out, S] with S = e4b_mxfp4_scale_stride(in) (in/32 rounded up to a multiple
 * of 16, padding bytes 0).  The descriptor's blocksize is 32 for MXFP4. */
/* INT8 / FP8: the 8-bit blockwise modes ([P1] "Storage modes: the support
 * matrix"): 64-element blocks with an fp32 absmax and ONE code byte per element
 * (packed stacks [E, out*in]); int8 is the dynamic tree map (bit 7 the sign; in
 * the 7-bit tail, E leading zeros give 10^-E, then an indicator bit and 6 - E
 * fraction bits on [0.1, 1] at bin centres; tail 0 is 0, or +1 with the sign set),
 * fp8 the E4M3 values divided by 448.  The grouped GEMMs take them as bf16,
 * dequantized one stack at a time into the workspace.
 * BF16: passthrough, the stacks given as bf16 [E, out, in] in gate_up / down (no
 * absmax). */
typedef enum {
    E4B_CODEBOOK_NF4 = 0, E4B_CODEBOOK_FP4 = 1, E4B_CODEBOOK_MXFP4 = 2,
    E4B_CODEBOOK_INT8 = 3, E4B_CODEBOOK_FP8 = 4, E4B_CODEBOOK_BF16 = 5
} e4b_codebook;
typedef enum { E4B_F32 = 0, E4B_BF16 = 1 } e4b_dtype;
typedef enum { E4B_PATH_AUTO = 0, E4B_PATH_GROUPED = 1, E4B_PATH_DECODE = 2 } e4b_path;
/* The experts' gated activation of the pre-activations g (gate rows) and u (up rows):
 *   SWIGLU       h = silu(g) u                                   ([P4] forward)
 *   CLAMPED_GLU  h = (u' + 1) g' sigmoid(alpha g'),  g' = min(g, limit),
 *                u' = clamp(u, -limit, limit)                    ([P2] gpt-oss experts;
 *                the pages give no formula: this is the published gpt-oss expert,
 *                alpha = 1.702 and limit = 7 there).  The clamp passes the gradient
 *                where its input lies inside the closed interval. */
typedef enum { E4B_ACT_SWIGLU = 0, E4B_ACT_CLAMPED_GLU = 1 } e4b_activation;

/* Layer description.  H and I must be multiples of 64 (blocks never straddle a
 * row, [P4] __init__); 1 <= top_k <= min(E, 8); E <= 256; blocksize == 64
 * (32 for E4B_CODEBOOK_MXFP4).
 * path: AUTO takes the weight-streaming decode kernels for T <= 8 when no
 * grouped outputs are requested and the shapes fit them (H <= 8192, and the
 * per-warp stage rings of 16 rows plus the tokens' activation rows fit in
 * shared memory), and the grouped tensor-core kernels otherwise; the other
 * values force one path (DECODE outside that range returns
 * E4B_ERR_UNSUPPORTED).  The decode kernels implement SwiGLU without biases or
 * adapters only: AUTO takes the grouped kernels for the clamped GLU, biased
 * experts or LoRA at every T, and DECODE returns E4B_ERR_UNSUPPORTED for them.
 * activation: E4B_ACT_SWIGLU (zero-initialised descriptors) or
 * E4B_ACT_CLAMPED_GLU with glu_alpha finite and glu_limit > 0 (+inf allowed).
 * lora_rank: 0 (no adapters; zero-initialised descriptors) or the rank r of the
 * per-expert LoRA adapters in e4b_experts, a multiple of 8 up to 64 ([P1]
 * "ExpertsLoRA(base, r, alpha)": the base stays frozen, only the adapters
 * train); lora_scale = alpha / r multiplies each adapter update:
 *   gate_up pre-activations += s (x A_gu^T) B_gu^T,  expert output += s (h A_d^T) B_d^T. */
typedef struct {
    int E, H, I, top_k;
    int renormalize;           /* divide the selected softmax weights by their sum  */
    e4b_codebook codebook;
    int blocksize;             /* must be 64 */
    e4b_path path;
    e4b_activation activation;
    float glu_alpha, glu_limit;   /* E4B_ACT_CLAMPED_GLU only */
    int lora_rank;                /* 0, or 8, 16, ..., 64 */
    float lora_scale;             /* alpha / r, finite */
} e4b_moe_desc;

/* Device pointers to the two quantized stacks (see storage above), the
 * optional per-expert biases ([P2] gpt-oss experts; NULL = none): gate_up_bias
 * is added to the gate_up pre-activations (gate half first, like the rows),
 * down_bias to each expert's output before its routing weight multiplies it;
 * and, when the descriptor's lora_rank r > 0, the four bf16 LoRA adapters of
 * every expert (stacked [E, r, in] / [E, out, r] as in [P2] "Prior art"; all
 * four required then, ignored otherwise).  Pointers are 16-byte aligned. */
typedef struct {
    const uint8_t *gate_up;        /* [E, 2I*H/2] */
    const uint8_t *down;           /* [E, H*I/2]  */
    const float *gate_up_absmax;   /* [E, 2I*H/64] */
    const float *down_absmax;      /* [E, H*I/64]  */
    const float *gate_up_bias;     /* fp32 [E, 2I] or NULL */
    const float *down_bias;        /* fp32 [E, H] or NULL  */
    const void *lora_A_gu;         /* bf16 [E, r, H]  */
    const void *lora_B_gu;         /* bf16 [E, 2I, r] (gate rows first, like the stack) */
    const void *lora_A_d;          /* bf16 [E, r, I]  */
    const void *lora_B_d;          /* bf16 [E, H, r]  */
    const uint8_t *gate_up_scales; /* MXFP4 only (then the absmax pointers are unused): [E, 2I, S(H)] */
    const uint8_t *down_scales;    /*                                                    [E, H, S(I)]  */
} e4b_experts;

/* Gradients of the four adapters (fp32, shaped like them; each fully written),
 * summed over every routed pair of the expert. */
typedef struct {
    float *dA_gu, *dB_gu, *dA_d, *dB_d;
} e4b_lora_grads;

/* Blockwise 4-bit quantization ([P4] from_float / _quantize_stack).
 * w: fp32 [E, out, in].  For every 64-element block of each row: absmax =
 * max|w| (stored as is, fp32); each element is divided by absmax (IEEE fp32
 * division) and takes the code of the nearest codebook value, an exact tie
 * going to the smaller value; an all-zero block stores absmax 0 and the zero
 * code.  Writes packed [E, out*in/2] and absmax [E, out*in/64]; for the 8-bit
 * codebooks (INT8, FP8) packed holds one byte per element, [E, out*in].
 * Errors: E4B_ERR_BLOCKSIZE if blocksize != 64 or in % 64 != 0;
 * E4B_ERR_INVALID_ARG for null pointers, negative sizes or an unknown codebook.
 * Non-finite inputs are outside the contract. */
E4B_API e4b_status e4b_quantize_nf4(const float *w, int64_t E, int64_t out, int64_t in, int blocksize,
                            e4b_codebook codebook, uint8_t *packed, float *absmax, void *stream);

/* MXFP4 quantization (OCP MX v1.0 conversion): for every 32-element block of
 * each row, X = floor(log2(max|w|)) - 2 clamped to [-127, 127] (an all-zero block:
 * -127), scale byte X + 127; each element w / 2^X rounded to the nearest E2M1
 * value, ties to the even code, saturating at 6, a zero result stored as +0.
 * Writes packed [E, out*in/2] and scales [E, out, e4b_mxfp4_scale_stride(in)].
 * Errors: E4B_ERR_BLOCKSIZE if in % 32 != 0; E4B_ERR_INVALID_ARG for null
 * pointers or negative sizes. */
E4B_API int64_t e4b_mxfp4_scale_stride(int64_t in);
E4B_API e4b_status e4b_quantize_mxfp4(const float *w, int64_t E, int64_t out, int64_t in, uint8_t *packed,
                              uint8_t *scales, void *stream);
/* MXFP4 dequantization: e2m1(code) * 2^(s - 127) in fp32 (exact), then bf16
 * nearest-even (exact for these values) when out_dtype == E4B_BF16. */
E4B_API e4b_status e4b_dequantize_mxfp4(const uint8_t *packed, const uint8_t *scales, int64_t E, int64_t out,
                                int64_t in, e4b_dtype out_dtype, void *w_out, void *stream);

/* Dequantization ([P4] _dequantize_expert): value = code_value * absmax with
 * one fp32 multiply, then (out_dtype == E4B_BF16) rounded to bf16 nearest-even.
 * w_out: [E, out, in] of out_dtype.  Same errors as quantize. */
E4B_API e4b_status e4b_dequantize_nf4(const uint8_t *packed, const float *absmax, int64_t E, int64_t out,
                              int64_t in, int blocksize, e4b_codebook codebook, e4b_dtype out_dtype,
                              void *w_out, void *stream);

/* Bytes of device workspace e4b_moe_forward, e4b_moe_backward_dgrad and
 * e4b_moe_backward_router need for T tokens (the largest of them).  Returns 0
 * for an invalid desc. */
E4B_API size_t e4b_moe_workspace_size(const e4b_moe_desc *d, int64_t T);

/* Forward of the expert layer ([P4] Experts4bit.forward):
 *   y_t = sum_j w_{t,j} * (act(x_t W_gate,e^T + bg_e, x_t W_up,e^T + bu_e) W_down,e^T + bd_e),
 * e = topk_idx[t,j], W_gate/W_up = rows [0,I)/[I,2I) of gate_up, act the
 * descriptor's activation (silu(g) * u by default), the biases zero unless
 * given, the weights dequantized to bf16, products accumulated in fp32, the
 * weighted sum over the k slots in fp32, y rounded to bf16.
 *   x            bf16 [T, H]
 *   router_logits fp32 [T, E] or NULL.  If given, the layer routes: top-k by
 *                logit (ties to the lower expert index), weights = softmax over
 *                all E at the chosen experts, divided by their sum when
 *                d->renormalize; topk_idx / topk_w are WRITTEN.  If NULL they
 *                are read as inputs, as in [P4] forward(hidden_states,
 *                top_k_index, top_k_weights).
 *   topk_idx     int32 [T, k];  topk_w fp32 [T, k]
 *   y            bf16 [T, H]
 *   saved_gu     bf16 [T*k, 2I] or NULL: what the input gradient needs from the
 *                forward, in grouped row order (row r holds pair perm[r]): the
 *                activation's derivatives dh/dg in columns [0,I) and dh/du in
 *                columns [I,2I) (SwiGLU: u s(g) (1 + g (1 - s(g))) and silu(g), s
 *                the logistic function), for e4b_moe_backward_dgrad.
 *   saved_h      bf16 [T*k, I] or NULL: the activation output h of every pair in
 *                grouped row order, for the routing-weight gradient of
 *                e4b_moe_backward.  The forward's down GEMM reads h from here.
 *   offsets_out  int32 [E+1] or NULL: first grouped row of each expert.
 *   perm_out     int32 [T*k] or NULL: pair id t*k+j of each grouped row;
 *                experts ascending, tokens ascending inside an expert.
 *   workspace    device scratch of at least e4b_moe_workspace_size(d, T) bytes.
 * T == 0 is a no-op.  topk_idx entries outside [0, E) are outside the contract. */
E4B_API e4b_status e4b_moe_forward(const e4b_moe_desc *d, const e4b_experts *w, const void *x, int64_t T,
                           const float *router_logits, int32_t *topk_idx, float *topk_w, void *y,
                           void *saved_gu, void *saved_h, int32_t *offsets_out, int32_t *perm_out,
                           void *workspace, size_t ws_bytes, void *stream);

/* The layer backward: the input gradient and the routing gradient in one pass.
 *   grad_x       as in e4b_moe_backward_dgrad (written), or NULL;
 *   grad_topk_w  fp32 [T,k] = <grad_out_t, Y_{t,j}> as in e4b_moe_backward_router
 *                (written; 0 for an out-of-range expert), or NULL;
 *   grad_logits  fp32 [T,E] through the routing softmax as in
 *                e4b_moe_backward_router (written), or NULL.
 * The routing-weight gradient is fused into the input gradient's down^T GEMM:
 * its accumulator is grad_out_t W_down,e before the routing weight, so
 *   <grad_out_t, Y_{t,j}> = <grad_out_t W_down,e, h_{t,j}> (+ <grad_out_t, b_e>
 *                                                           with a down bias)
 * and the epilogue leaves one fp32 partial dot product per row and 256-column
 * tile; a per-token kernel adds them in tile order and runs the softmax
 * backward.  No GEMM is repeated for it.  h comes from saved_h (as written by
 * e4b_moe_forward for the same topk_idx, with saved_gu) or, when saved_gu is
 * NULL, is recomputed from x together with the derivatives.
 *   x bf16 [T,H] (read only when saved_gu is NULL); router_logits fp32 [T,E]
 *   (needed only for grad_logits); topk_idx, topk_w, grad_out as for
 *   e4b_moe_backward_dgrad; workspace: e4b_moe_workspace_size(d, T) bytes.
 * With adapters (d->lora_rank > 0), every gradient includes their updates, and
 * lora_grads (or NULL) receives the adapter gradients, with s = lora_scale, dY =
 * w grad_out_t, z_gu = x A_gu^T, z_d = h A_d^T:
 *   dB_d += s dY (x) z_d,   dA_d += s (dY B_d) (x) h,
 *   dB_gu += s dGU (x) z_gu,  dA_gu += s (dGU B_gu) (x) x      (dGU = [dG | dU]).
 * lora_grads needs x (and h: saved_h, or recompute mode).
 * Returns E4B_ERR_INVALID_ARG when no output is asked for, when grad_topk_w or
 * lora_grads is asked for with saved_gu but without saved_h, when lora_grads is
 * asked for without x, or when grad_logits is asked for without router_logits or
 * grad_topk_w. */
E4B_API e4b_status e4b_moe_backward(const e4b_moe_desc *d, const e4b_experts *w, const void *x, int64_t T,
                            const float *router_logits, const int32_t *topk_idx, const float *topk_w,
                            const void *grad_out, const void *saved_gu, const void *saved_h,
                            void *grad_x, float *grad_topk_w, float *grad_logits,
                            const e4b_lora_grads *lora_grads,
                            void *workspace, size_t ws_bytes, void *stream);

/* Input gradient of the forward with routing held constant ([P5] "What this
 * adds": recompute-in-backward; the packed base is frozen, no weight gradient):
 *   dh   = w_{t,j} * grad_out_t W_down,e                 (contract over H)
 *   dG   = dh * dh/dg,  dU = dh * dh/du   (the activation's derivatives; SwiGLU:
 *          u * s(g) * (1 + g (1 - s(g))) and silu(g))
 *   grad_x_t = sum_j  dG W_gate,e + dU W_up,e            (contract over 2I)
 * with the weights re-dequantized inside the kernels and never stored.
 * The SwiGLU derivatives come from saved_gu (as written by e4b_moe_forward for
 * the same topk_idx) or, when saved_gu is NULL, are recomputed from x.
 *   x bf16 [T,H] (read only when saved_gu is NULL), topk_idx int32 [T,k],
 *   topk_w fp32 [T,k], grad_out bf16 [T,H], grad_x bf16 [T,H] (written). */
E4B_API e4b_status e4b_moe_backward_dgrad(const e4b_moe_desc *d, const e4b_experts *w, const void *x,
                                  int64_t T, const int32_t *topk_idx, const float *topk_w,
                                  const void *grad_out, const void *saved_gu, void *grad_x,
                                  void *workspace, size_t ws_bytes, void *stream);

/* Gradient of the layer output with respect to the routing, indices held
 * constant: the other half of the layer backward next to e4b_moe_backward_dgrad.
 * The forward gives y_t = sum_j w_{t,j} Y_{t,j}, with Y_{t,j} the expert output
 * before its routing weight ([P4] Experts4bit.forward), so
 *   grad_topk_w[t,j] = <grad_out_t, Y_{t,j}>                       (fp32 [T,k])
 * and, through the softmax that made the weights from router_logits,
 *   no renormalisation: grad_logits[t,i] = p_i (sum_{j: e_j = i} dw_j - sum_j dw_j p_{e_j}),
 *                       p = softmax of the token's logits over all E;
 *   renormalisation:    grad_logits[t,i] = sum_{j: e_j = i} w_j (dw_j - sum_j' w_j' dw_j'),
 *                       w = topk_w (logits outside the top-k get 0).
 * Y is recomputed from x through the grouped GEMMs (gate_up, then down with unit
 * weights), rounded to bf16 like every per-pair row; the dot products and the
 * softmax backward run in fp32.
 *   x bf16 [T,H], router_logits fp32 [T,E] (needed only for grad_logits),
 *   topk_idx int32 [T,k], topk_w fp32 [T,k] (the forward's), grad_out bf16 [T,H],
 *   grad_topk_w fp32 [T,k] (written; 0 for an out-of-range expert),
 *   grad_logits fp32 [T,E] (written) or NULL,
 *   workspace as for e4b_moe_forward (e4b_moe_workspace_size bytes).
 * Returns E4B_ERR_INVALID_ARG when grad_logits is given without router_logits. */
E4B_API e4b_status e4b_moe_backward_router(const e4b_moe_desc *d, const e4b_experts *w, const void *x,
                                   int64_t T, const float *router_logits, const int32_t *topk_idx,
                                   const float *topk_w, const void *grad_out, float *grad_topk_w,
                                   float *grad_logits, void *workspace, size_t ws_bytes, void *stream);

/* Forward without any device memory from the caller.  The source pages have no
 * counterpart: this is an interface for callers that cannot give the library
 * scratch -- a caller whose device memory all belongs to its own pool, reserved
 * up front (a serving engine that claims free memory for its caches at start-up,
 * a process held to a hard memory budget), or a latency-critical loop that cannot
 * afford a per-call cudaMalloc / cudaFree (both can stall or synchronize the
 * device).  The caller still owns and passes x, topk_idx, topk_w and y.
 *
 * Computes exactly what e4b_moe_forward computes for the same arguments (with
 * saved_gu, offsets_out and perm_out absent), through the same kernels.  Its
 * scratch is a file-scope device array of 32 MiB inside the library, which every
 * GPU that loads the library holds until the process exits.  Requests whose
 * workspace (e4b_moe_workspace_size) exceeds 32 MiB return E4B_ERR_WORKSPACE
 * before anything is launched.  Allocates nothing: no cudaMalloc, no cudaFree,
 * no allocating library call.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  CUDA loads a library's device code lazily, at its first use on a
 * device, and the 32 MiB array is claimed then, not when the library is loaded:
 * a caller that reserves the device's free memory for its own pool must make one
 * call on each device BEFORE reserving it (a call with T = 0 does only this set-up
 * and launches nothing), or that first call can fail with E4B_ERR_CUDA.
 * All calls share the one array and nothing in it needs to start at
 * zero (each call writes what it reads), but calls that can overlap on the GPU
 * -- different streams, or host threads without ordering between their calls --
 * race on it and must be serialized by the caller. */
E4B_API e4b_status e4b_moe_forward_noalloc(const e4b_moe_desc *d, const e4b_experts *w, const void *x,
                                           int64_t T, const float *router_logits, int32_t *topk_idx,
                                           float *topk_w, void *y, void *stream);

/* Pipelined steps through PINNED host buffers: the expert layer's forward
 * (routed from router logits) and its input gradient for a stream of batches
 * that live in host memory.  Each e4b_pipe_submit
 *   - copies the batch's x [T,H] bf16, router logits [T,E] fp32 and grad_out
 *     [T,H] bf16 to the device on the pipe's copy-in stream,
 *   - runs e4b_moe_forward (g/u saved) and e4b_moe_backward_dgrad on the
 *     compute stream given at creation,
 *   - copies y [T,H] and grad_x [T,H] (bf16) back on the pipe's copy-out
 *     stream, y as soon as the forward is done.
 * Two device buffer sets alternate between consecutive submits, so batch n+1's
 * input copies and batch n-1's output copies run under batch n's kernels; the
 * saved g/u and the workspace are shared (the compute stream orders them).
 * Results are exactly those of the two calls on device copies of the inputs.
 *
 * arena: caller-owned device memory of e4b_pipe_arena_size(d, T_max) bytes,
 * 256-byte aligned, alive until e4b_pipe_destroy.  Host pointers passed to
 * submit must be page-locked (cudaHostAlloc / cudaHostRegister); the inputs
 * must stay unchanged and the outputs unread until a later e4b_pipe_join or
 * e4b_pipe_sync covers the submit.  `w` is copied at creation (the weight
 * memory it points to must stay alive).  A pipe is used from one host thread
 * at a time.  Creation makes two non-blocking CUDA streams and a few events
 * (host-side driver objects; no device memory is allocated). */
typedef struct e4b_pipe e4b_pipe;
E4B_API size_t e4b_pipe_arena_size(const e4b_moe_desc *d, int64_t T_max);
E4B_API e4b_status e4b_pipe_create(const e4b_moe_desc *d, const e4b_experts *w, int64_t T_max, void *arena,
                                   size_t arena_bytes, void *stream, e4b_pipe **out);
/* Enqueues one batch (0 <= T <= T_max; T = 0 is a no-op) and returns without
 * waiting for it.  Shape and pointer errors return before anything is enqueued. */
E4B_API e4b_status e4b_pipe_submit(e4b_pipe *p, int64_t T, const void *x_host, const float *logits_host,
                                   const void *grad_out_host, void *y_host, void *grad_x_host);
/* Fork/join point, without waiting on the host: work enqueued on the compute
 * stream after the call runs after every batch submitted so far (copies
 * included), and the pipe's copies of later submits run after the work already
 * enqueued on the compute stream. */
E4B_API e4b_status e4b_pipe_join(e4b_pipe *p);
/* e4b_pipe_join, then waits on the host for the compute stream and returns
 * e4b_device_status of it. */
E4B_API e4b_status e4b_pipe_sync(e4b_pipe *p);
/* Waits for the pipe's streams, then releases its streams and events.  NULL is a no-op. */
E4B_API void e4b_pipe_destroy(e4b_pipe *p);

/* Synchronizes `stream`, then reads and clears the library's device status
 * word: E4B_OK, or E4B_ERR_TIMEOUT if a kernel gave up on a wait since the last
 * call, or else E4B_ERR_DEBUG_CHECK if a check of the debug build failed.
 * E4B_ERR_CUDA if the synchronization itself fails. */
E4B_API e4b_status e4b_device_status(void *stream);

/* The raw status word the last e4b_device_status call read (0 when it returned
 * E4B_OK): bit 0 timeout, bit 1 debug check, bits 8..15 the first failing check's
 * site.  Sites: 1 grouped-GEMM m-tile entry, 2 grouped-GEMM pair id, 3 row-gather
 * pair id, 4 combine inverse-permutation entry, 5 routing-gradient
 * inverse-permutation entry, 6 expert offsets, 7 expert counts, 8 m-tile total,
 * 9 m-tile entry against its expert's rows, 10 perm entry, 11 inv_perm entry. */
E4B_API uint32_t e4b_last_status_word(void);

/* 1 in the debug build (libe4b_debug.so, compiled with E4B_DEBUG_CHECKS=1), else 0.
 * The debug build checks, on the device, every m-tile entry and pair id the
 * grouped GEMMs use, the pair ids of the row gather, the inverse-permutation
 * entries of the combine and the routing gradient, and, after every grouping, the
 * whole schedule (e4b_debug_validate_schedule).  A failed check records its site
 * in the status word and skips the access it guards; nothing traps.  This is the
 * stand-in for a memory checker on the expert layer's pages' "fails loudly"
 * contract (bitsandbytes PR #1965, "Correctness & coverage").  Release builds
 * compile the checks out. */
E4B_API int e4b_debug_checks(void);

/* Diagnostic, in every build: checks a grouping schedule on the device.  Given the
 * routing topk_idx [P] (P = T * top_k pairs), E experts and the m-tile height
 * tile_rows, the schedule is counts [E], offsets [E+1] (expert e owns the grouped
 * rows [offsets[e], offsets[e+1])), tile_prefix [E+1] (tile_prefix[E] = number of
 * m-tiles), sched [n_sched][4] int32 m-tile entries (expert, first row, rows, 0),
 * perm [P] (pair id of each grouped row) and inv_perm [P] (grouped row of each pair,
 * -1 for a pair whose expert is outside [0, E)).  All pointers are device memory
 * the caller owns.  Every value read is range-checked before it serves as an index.
 * Returns E4B_OK for a consistent schedule; E4B_ERR_DEBUG_CHECK otherwise, with the
 * first failing property in e4b_last_status_word (sites 6-11); an earlier kernel's
 * pending error is returned first.  E4B_ERR_INVALID_ARG for null pointers, P <= 0,
 * E outside 1..256, tile_rows <= 0 or n_sched < 0.  Synchronizes `stream`. */
E4B_API e4b_status e4b_debug_validate_schedule(const int32_t *topk_idx, int64_t P, int E, int tile_rows,
                                               const int32_t *counts, const int32_t *offsets,
                                               const int32_t *tile_prefix, const int32_t *sched, int64_t n_sched,
                                               const int32_t *perm, const int32_t *inv_perm, void *stream);

/* Diagnostic: launches one kernel whose single thread waits, through the same
 * bounded mbarrier wait every pipelined kernel uses, on a barrier nothing
 * arrives at.  After the wait's 2 s limit the kernel records the timeout in the
 * device status word and returns (nothing faults, traps or hangs), so the next
 * e4b_device_status() returns E4B_ERR_TIMEOUT and clears it; the context stays
 * usable.  Returns E4B_OK once the kernel is launched. */
E4B_API e4b_status e4b_watchdog_selftest(void *stream);

/* Static description of a status code. */
E4B_API const char *e4b_status_string(e4b_status s);

/* Number of kernels the library launched since load (a host-side counter,
 * for benchmarks that report their launch count). */
E4B_API uint64_t e4b_launch_count(void);

/* Optional per-kernel timing for benchmarks (off by default).  When enabled,
 * every launch of the library is bracketed by two CUDA events on its stream;
 * e4b_timing_get synchronizes on the recorded events and returns, for one
 * kernel kind, the summed device time (ms) and the number of timed launches.
 * Kinds: 0 quantize, 1 dequantize, 2 route, 3 group, 4 gather, 5 combine,
 * 6 grouped gate_up GEMM, 7 grouped down GEMM, 8 dgrad down GEMM,
 * 9 dgrad gate_up GEMM, 10 decode gate_up GEMV, 11 decode down GEMV. */
E4B_API void e4b_timing_enable(int on);
/* Times only the kinds whose bit is set in mask (bit k = kind k above); 0 turns
 * timing off.  e4b_timing_enable(1) equals a mask with every bit set.  A kind
 * left untimed records no events, so its launches run back to back. */
E4B_API void e4b_timing_enable_kinds(uint32_t mask);
E4B_API void e4b_timing_reset(void);
E4B_API e4b_status e4b_timing_get(int kind, double *total_ms, uint64_t *launches);

#ifdef __cplusplus
}
#endif
#endif /* E4B_H_ */
