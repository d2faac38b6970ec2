// Routing-weight and router-logit gradient of the expert layer (routing indices
// held).  The layer output is y_t = sum_j w_{t,j} Y_{t,j}, with Y_{t,j} the
// expert output before its routing weight ("experts4bit-qlora 0.1.0"
// experts.py, Experts4bit.forward: the routing weight multiplies the expert
// output).  Hence dL/dw_{t,j} = <grad_out_t, Y_{t,j}>, and the logit gradient
// follows through the softmax that produced the weights:
//   no renormalisation: dL/dl_i = p_i (sum_{j: e_j = i} dw_j - sum_j dw_j p_{e_j}),
//     p = softmax over all E experts;
//   renormalisation: dL/dl_i = sum_{j: e_j = i} w_j (dw_j - sum_j' w_j' dw_j').
// The unweighted Y comes from the grouped down GEMM run with unit weights, or,
// fused into the input gradient, dL/dw = <grad_out_t W_d, h_{t,j}> (+ <grad_out_t,
// b_e> with a down bias) from the dot products the down^T GEMM leaves per tile.
#include "router_backward.h"

namespace e4b {

__global__ void __launch_bounds__(256) fill_f32_kernel(float* __restrict__ p, int64_t n, float v) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        p[i] = v;
}

// One warp per token: the k routing-weight gradients of the token, then its
// logit gradient.  FROM_PARTS = false: dw_j = <grad_out_t, Y_{t,j}> over H
// (fp32, a fixed order: per-lane sums over 16-byte chunks, then a butterfly).
// FROM_PARTS = true: dw_j = the sum of the pair's per-tile dot products
// <grad_out_t W_d, h> (written by the input-gradient down^T GEMM; lane-strided
// over the tiles, then a butterfly) plus, with a down bias, <grad_out_t, b_e>.
template <bool FROM_PARTS>
__global__ void __launch_bounds__(256) router_grad_kernel(const __nv_bfloat16* __restrict__ grad_out,
                                                          const __nv_bfloat16* __restrict__ Y,
                                                          const float* __restrict__ parts, int n_parts,
                                                          const float* __restrict__ down_bias,
                                                          const int32_t* __restrict__ inv_perm,
                                                          const int32_t* __restrict__ idx,
                                                          const float* __restrict__ wts,
                                                          const float* __restrict__ logits, int64_t T, int E,
                                                          int k, int H, int renorm, float* __restrict__ dw_out,
                                                          float* __restrict__ dl_out, uint32_t* __restrict__ status) {
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    float dw[8];
    int ej[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        dw[j] = 0.0f;
        ej[j] = -1;
        if (j >= k) continue;
        const int64_t p = t * k + j;
        const int e = __ldg(idx + p);
        bool valid = e >= 0 && e < E;
        float acc = 0.0f;
        const int64_t r = valid ? __ldg(inv_perm + p) : -1;
#if E4B_DEBUG_CHECKS
        if (valid && (r < 0 || r >= T * k)) {   // a routed pair has a grouped row
            if (lane == 0) debug_fail(status, kSiteRouterInv);
            valid = false;
        }
#endif
        if (valid) {
            const uint4* g4 = reinterpret_cast<const uint4*>(grad_out + t * H);
            if (FROM_PARTS) {
                for (int c = lane; c < n_parts; c += 32) acc += __ldcs(parts + r * n_parts + c);
                if (down_bias) {
                    float b = 0.0f;
                    const float4* b4 = reinterpret_cast<const float4*>(down_bias + (int64_t)e * H);
                    for (int c = lane; c < H / 8; c += 32) {
                        const uint4 gv = __ldg(g4 + c);
                        const float4 bl = __ldg(b4 + 2 * c), bh = __ldg(b4 + 2 * c + 1);
                        const float bv[8] = {bl.x, bl.y, bl.z, bl.w, bh.x, bh.y, bh.z, bh.w};
                        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            b = fmaf(__uint_as_float(gw[q] << 16), bv[2 * q], b);
                            b = fmaf(__uint_as_float(gw[q] & 0xFFFF0000u), bv[2 * q + 1], b);
                        }
                    }
                    acc += b;
                }
            } else {
                const uint4* y4 = reinterpret_cast<const uint4*>(Y + r * H);
                for (int c = lane; c < H / 8; c += 32) {
                    const uint4 gv = __ldg(g4 + c), yv = __ldcs(y4 + c);
                    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, yw[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        acc = fmaf(__uint_as_float(gw[q] << 16), __uint_as_float(yw[q] << 16), acc);
                        acc = fmaf(__uint_as_float(gw[q] & 0xFFFF0000u), __uint_as_float(yw[q] & 0xFFFF0000u), acc);
                    }
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        dw[j] = acc;
        ej[j] = valid ? e : -1;
        if (lane == 0) dw_out[p] = acc;
    }
    if (!dl_out) return;
    const float* l = logits + t * E;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (lane + 32 * i < E) ? __ldg(l + lane + 32 * i) : __int_as_float(0xff800000);
    float dl[8];
    if (renorm) {
        float a = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < k && ej[j] >= 0) a = fmaf(__ldg(wts + t * k + j), dw[j], a);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            dl[i] = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j < k && ej[j] == lane + 32 * i) dl[i] = fmaf(__ldg(wts + t * k + j), dw[j] - a, dl[i]);
        }
    } else {
        float top = v[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) top = fmaxf(top, v[i]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, off));
        float z = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (lane + 32 * i < E) z += expf(v[i] - top);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
        float a = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < k && ej[j] >= 0) a = fmaf(dw[j], expf(__ldg(l + ej[j]) - top) / z, a);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float pi = (lane + 32 * i < E) ? expf(v[i] - top) / z : 0.0f;
            float sel = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j < k && ej[j] == lane + 32 * i) sel += dw[j];
            dl[i] = pi * (sel - a);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (lane + 32 * i < E) dl_out[t * E + lane + 32 * i] = dl[i];
}

cudaError_t launch_fill_f32(float* p, int64_t n, float v, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    const int grid = (int)std::min<int64_t>((n + 255) / 256, 1184);
    fill_f32_kernel<<<grid, 256, 0, st>>>(p, n, v);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_router_grad(const __nv_bfloat16* grad_out, const __nv_bfloat16* Y, const int32_t* inv_perm,
                               const int32_t* idx, const float* wts, const float* logits, int64_t T, int E, int k,
                               int H, int renorm, float* dw, float* dlogits, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int64_t grid = (T * 32 + 255) / 256;
    router_grad_kernel<false><<<(unsigned)grid, 256, 0, st>>>(grad_out, Y, nullptr, 0, nullptr, inv_perm, idx, wts,
                                                              logits, T, E, k, H, renorm, dw, dlogits,
                                                              device_status_ptr());
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_router_grad_parts(const __nv_bfloat16* grad_out, const float* parts, int n_parts,
                                     const float* down_bias, const int32_t* inv_perm, const int32_t* idx,
                                     const float* wts, const float* logits, int64_t T, int E, int k, int H,
                                     int renorm, float* dw, float* dlogits, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int64_t grid = (T * 32 + 255) / 256;
    router_grad_kernel<true><<<(unsigned)grid, 256, 0, st>>>(grad_out, nullptr, parts, n_parts, down_bias, inv_perm,
                                                             idx, wts, logits, T, E, k, H, renorm, dw, dlogits,
                                                             device_status_ptr());
    count_launch();
    return cudaGetLastError();
}

}  // namespace e4b
