// Launchers of the LoRA kernels (lora.cu).
#pragma once
#include "e4b_internal.h"

namespace e4b {

// out [rows, 64] bf16 = s * in [rows, K] M_e^T for the rows of every m-tile of the
// grouped schedule (expert e of the tile), ranks >= r zero.  M: the A adapter
// [E, r, K] (m_q_major) or the B adapter [E, K, r], bf16.  K a multiple of 64.
cudaError_t launch_lora_thin(const __nv_bfloat16* in, int K, const __nv_bfloat16* m, bool m_q_major, int r, float s,
                             const int4* sched, const int* tile_prefix, int E, int max_m_tiles, __nv_bfloat16* out,
                             cudaStream_t st);
// t [E, r, K] = the B adapter m [E, K, r] transposed (K a multiple of 64).
cudaError_t launch_lora_transpose(const __nv_bfloat16* m, int E, int K, int r, __nv_bfloat16* t, cudaStream_t st);
// out (fp32) for each expert e = sum over its grouped rows p (offsets[e] .. offsets[e+1])
// of coef_p U[p, :] (x) V[p, :r], U [rows, N] bf16, V [rows, 64] bf16; coef_p =
// topk_w[perm[p]] when coef_w, else 1; out [E, N, r], or [E, r, N] when q_major_out.
cudaError_t launch_lora_grad(const __nv_bfloat16* U, int N, const __nv_bfloat16* V, int r, const int* offsets,
                             int E, const float* topk_w, const int* perm, bool coef_w, bool q_major_out, float* out,
                             cudaStream_t st);

}  // namespace e4b
