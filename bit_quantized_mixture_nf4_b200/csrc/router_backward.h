// Launchers of the routing-gradient kernels (router_backward.cu).
#pragma once
#include "e4b_internal.h"

namespace e4b {

cudaError_t launch_fill_f32(float* p, int64_t n, float v, cudaStream_t st);
// dw [T*k] = <grad_out_t, Y[inv_perm[p]]> for every pair p = t*k + j (Y in grouped
// row order; 0 for an out-of-range expert); dlogits [T, E] (skipped when null)
// through the routing softmax.
cudaError_t launch_router_grad(const __nv_bfloat16* grad_out, const __nv_bfloat16* Y, const int32_t* inv_perm,
                               const int32_t* idx, const float* wts, const float* logits, int64_t T, int E, int k,
                               int H, int renorm, float* dw, float* dlogits, cudaStream_t st);

// The same from the per-tile dot products parts [P, n_parts] (grouped row order)
// that the input-gradient down^T GEMM writes: dw = sum of the row's parts, plus
// <grad_out_t, b_e> when down_bias is given.
cudaError_t launch_router_grad_parts(const __nv_bfloat16* grad_out, const float* parts, int n_parts,
                                     const float* down_bias, const int32_t* inv_perm, const int32_t* idx,
                                     const float* wts, const float* logits, int64_t T, int E, int k, int H,
                                     int renorm, float* dw, float* dlogits, cudaStream_t st);

}  // namespace e4b
