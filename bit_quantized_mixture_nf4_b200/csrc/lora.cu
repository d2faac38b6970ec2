// Per-expert LoRA over the frozen 4-bit base: the thin projections and the
// adapter gradients ("experts4bit-qlora" 0.4.0 description, "ExpertsLoRA(base,
// r, alpha)": only the adapters train; stacked per-expert adapters
// [num_experts, r, in] / [num_experts, out, r] as in the pages' prior art).
// The update of each projection is s (x A^T) B^T with s = alpha / r.  Inside the
// grouped GEMMs it is one more 64-deep k-stage: the thin operand s (x A^T) (rank
// padded to 64 with zeros, bf16) against the adapter B.  The two input
// gradients take s (dy B) against A the same way.  The kernels here make those
// thin operands and the four adapter gradients, which are sums over each
// expert's rows in grouped order (a fixed order: deterministic).
#include "lora.h"

namespace e4b {

// out[row, q] = s * sum_c in[row, c] * M_e(q, c) for the rows of one m-tile (one
// expert), q < r; columns r..63 of out are zero.  M_e(q, c) = m[e][q][c]
// (Q_MAJOR, an A adapter [E, r, K]) or m[e][c][q] (a B adapter [E, K, r]).
// One thread per row; the adapter goes through shared memory in chunks of 64
// columns of K as fp32 [64][r].
template <bool Q_MAJOR>
__global__ void __launch_bounds__(256) lora_thin_kernel(const __nv_bfloat16* __restrict__ in, int K,
                                                        const __nv_bfloat16* __restrict__ m, int r, float s,
                                                        const int4* __restrict__ sched,
                                                        const int* __restrict__ tile_prefix, int E,
                                                        __nv_bfloat16* __restrict__ out) {
    __shared__ __align__(16) float ms[64 * 64];
    const int mt = blockIdx.x;
    if (mt >= __ldg(tile_prefix + E)) return;
    const int4 tl = __ldg(sched + mt);   // (expert, first row, rows, 0)
    const int e = tl.x, row = tl.y + (int)threadIdx.x;
    const bool valid = (int)threadIdx.x < tl.z;
    float acc[64];
#pragma unroll
    for (int q = 0; q < 64; ++q) acc[q] = 0.0f;
    const __nv_bfloat16* me = m + (int64_t)e * r * K;
    const uint4* xin = reinterpret_cast<const uint4*>(in + (int64_t)row * K);
    for (int c0 = 0; c0 < K; c0 += 64) {
        __syncthreads();
        for (int i = threadIdx.x; i < 64 * r; i += blockDim.x) {   // ms[c][q] = M_e(q, c0 + c)
            const int c = i / r, q = i - c * r;
            const float v = Q_MAJOR ? __bfloat162float(me[(int64_t)q * K + c0 + c])
                                    : __bfloat162float(me[(int64_t)(c0 + c) * r + q]);
            ms[c * r + q] = v;
        }
        __syncthreads();
        if (!valid) continue;
#pragma unroll 1
        for (int c8 = 0; c8 < 64; c8 += 8) {
            const uint4 xv = __ldg(xin + (c0 + c8) / 8);
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float x = __uint_as_float(j & 1 ? (xw[j >> 1] & 0xFFFF0000u) : (xw[j >> 1] << 16));
                const float* mr = ms + (c8 + j) * r;
#pragma unroll
                for (int q = 0; q < 64; ++q)
                    if (q < r) acc[q] = fmaf(x, mr[q], acc[q]);
            }
        }
    }
    if (!valid) return;
    uint4* o = reinterpret_cast<uint4*>(out + (int64_t)row * 64);
#pragma unroll
    for (int q8 = 0; q8 < 8; ++q8) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int q = 8 * q8 + 2 * j;
            w[j] = pack_bf16x2(q < r ? s * acc[q] : 0.0f, q + 1 < r ? s * acc[q + 1] : 0.0f);
        }
        o[q8] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// out for expert e = sum over its grouped rows p (ascending) of coef_p * U[p, a] *
// V[p, q], a < N (the big dimension), q < r; coef_p = topk_w[perm[p]] when
// coef_w, else 1.  Written as out[e][a][q] (B adapters) or, with Q_MAJOR_OUT,
// out[e][q][a] (A adapters), fp32.  Block (e, 256 columns): one thread per
// column a, V rows staged through shared memory 32 at a time.
template <bool Q_MAJOR_OUT>
__global__ void __launch_bounds__(256) lora_grad_kernel(const __nv_bfloat16* __restrict__ U, int N,
                                                        const __nv_bfloat16* __restrict__ V, int r,
                                                        const int* __restrict__ offsets,
                                                        const float* __restrict__ topk_w,
                                                        const int* __restrict__ perm, int coef_w,
                                                        float* __restrict__ out) {
    __shared__ float vs[32][65];
    __shared__ float cs[32];
    const int e = blockIdx.y, a = blockIdx.x * 256 + (int)threadIdx.x;
    const int p0 = __ldg(offsets + e), p1 = __ldg(offsets + e + 1);
    float acc[64];
#pragma unroll
    for (int q = 0; q < 64; ++q) acc[q] = 0.0f;
    for (int pb = p0; pb < p1; pb += 32) {
        const int np = min(32, p1 - pb);
        __syncthreads();
        for (int i = threadIdx.x; i < np * 64; i += blockDim.x) {
            const int pp = i >> 6, q = i & 63;
            vs[pp][q] = __bfloat162float(V[(int64_t)(pb + pp) * 64 + q]);
        }
        if ((int)threadIdx.x < np)
            cs[threadIdx.x] = coef_w ? __ldg(topk_w + __ldg(perm + pb + threadIdx.x)) : 1.0f;
        __syncthreads();
        if (a >= N) continue;
#pragma unroll 1
        for (int pp = 0; pp < np; ++pp) {
            const float u = cs[pp] * __bfloat162float(U[(int64_t)(pb + pp) * N + a]);
#pragma unroll
            for (int q = 0; q < 64; ++q)
                if (q < r) acc[q] = fmaf(u, vs[pp][q], acc[q]);
        }
    }
    if (a >= N) return;
#pragma unroll
    for (int q = 0; q < 64; ++q) {
        if (q >= r) break;
        if (Q_MAJOR_OUT) out[((int64_t)e * r + q) * N + a] = acc[q];
        else out[((int64_t)e * N + a) * r + q] = acc[q];
    }
}

cudaError_t launch_lora_thin(const __nv_bfloat16* in, int K, const __nv_bfloat16* m, bool m_q_major, int r, float s,
                             const int4* sched, const int* tile_prefix, int E, int max_m_tiles, __nv_bfloat16* out,
                             cudaStream_t st) {
    if (max_m_tiles <= 0) return cudaSuccess;
    if (K % 64 || r < 1 || r > 64) return cudaErrorInvalidValue;
    if (m_q_major) lora_thin_kernel<true><<<max_m_tiles, 256, 0, st>>>(in, K, m, r, s, sched, tile_prefix, E, out);
    else lora_thin_kernel<false><<<max_m_tiles, 256, 0, st>>>(in, K, m, r, s, sched, tile_prefix, E, out);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_lora_grad(const __nv_bfloat16* U, int N, const __nv_bfloat16* V, int r, const int* offsets,
                             int E, const float* topk_w, const int* perm, bool coef_w, bool q_major_out, float* out,
                             cudaStream_t st) {
    if (r < 1 || r > 64) return cudaErrorInvalidValue;
    const dim3 grid((N + 255) / 256, E);
    if (q_major_out)
        lora_grad_kernel<true><<<grid, 256, 0, st>>>(U, N, V, r, offsets, topk_w, perm, coef_w ? 1 : 0, out);
    else
        lora_grad_kernel<false><<<grid, 256, 0, st>>>(U, N, V, r, offsets, topk_w, perm, coef_w ? 1 : 0, out);
    count_launch();
    return cudaGetLastError();
}

}  // namespace e4b
