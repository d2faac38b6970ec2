// Small-batch (T <= 8) forward: weight-streaming GEMVs on the CUDA cores.
//
// At a handful of tokens the layer is bound by reading the touched experts'
// packed weights once (0.5625 B per weight), so tensor cores do not help.  This
// is the decode fast path of the expert-layer pages ("experts4bit-qlora" 0.4.0
// description, section "Inference": single-token forward over the token's top-k
// experts with no host synchronisation, 4-bit GEMV reading packed NF4 directly),
// written for B200: 16-byte coalesced loads, a shared 256-entry byte -> code-pair
// table, fp32 FMAs, warp-shuffle reductions, no dequantized weight ever stored.
#include "e4b_internal.h"

namespace e4b {

constexpr int DEC_THREADS = 256;
constexpr int DEC_GU_FEATS = 8;     // features per CTA in the gate_up kernel (one per warp)
constexpr int DEC_DN_ROWS = 32;     // output rows per CTA in the down kernel (4 per warp)

template <int CB>
__device__ __forceinline__ void build_pair_lut(float2* lut) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) lut[b] = make_float2(c_code[CB][b >> 4], c_code[CB][b & 15]);
}

// Dot of 32 elements (16 packed bytes) with x[0..31] (fp32, shared memory).
__device__ __forceinline__ float dot32(const float2* lut, uint4 pk, const float* x) {
    const uint32_t w[4] = {pk.x, pk.y, pk.z, pk.w};
    const float4* x4 = reinterpret_cast<const float4*>(x);
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 xa = x4[2 * i], xb = x4[2 * i + 1];
        const float2 c0 = lut[w[i] & 0xFFu], c1 = lut[(w[i] >> 8) & 0xFFu];
        const float2 c2 = lut[(w[i] >> 16) & 0xFFu], c3 = lut[w[i] >> 24];
        acc = fmaf(c0.x, xa.x, acc); acc = fmaf(c0.y, xa.y, acc);
        acc = fmaf(c1.x, xa.z, acc); acc = fmaf(c1.y, xa.w, acc);
        acc = fmaf(c2.x, xb.x, acc); acc = fmaf(c2.y, xb.y, acc);
        acc = fmaf(c3.x, xb.z, acc); acc = fmaf(c3.y, xb.w, acc);
    }
    return acc;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// h[p, f] = silu(x_t . W_gate,e[f]) * (x_t . W_up,e[f]) for pair p = (t, j), e = idx[p].
// The block-scale is applied per 32-element half block: sum_b a_b * sum_{i in b} c[q_i] x_i.
template <int CB>
__global__ void __launch_bounds__(DEC_THREADS) decode_gateup_kernel(
    const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ idx, int E, int k, int H, int I,
    const uint8_t* __restrict__ packed, const float* __restrict__ absmax, float* __restrict__ h) {
    extern __shared__ float dsm[];
    float2* lut = reinterpret_cast<float2*>(dsm);          // 256 x float2
    float* xs = dsm + 512;                                  // H floats
    const int p = blockIdx.x;
    const int t = p / k;
    const int e = __ldg(idx + p);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int f = blockIdx.y * DEC_GU_FEATS + warp;
    if (e < 0 || e >= E) {   // out-of-range expert: contributes nothing
        if (lane == 0 && f < I) h[(int64_t)p * I + f] = 0.0f;
        return;
    }
    build_pair_lut<CB>(lut);
    for (int i = threadIdx.x; i < H; i += blockDim.x) xs[i] = __bfloat162float(x[(int64_t)t * H + i]);
    __syncthreads();
    if (f >= I) return;
    const int64_t rows = 2LL * I;
    const int nch = H / 32, bpr = H / 64;
    const uint4* rg = reinterpret_cast<const uint4*>(packed + ((int64_t)e * rows + f) * (H / 2));
    const uint4* ru = reinterpret_cast<const uint4*>(packed + ((int64_t)e * rows + I + f) * (H / 2));
    const float* ag = absmax + ((int64_t)e * rows + f) * bpr;
    const float* au = absmax + ((int64_t)e * rows + I + f) * bpr;
    float g = 0.0f, u = 0.0f;
    for (int c = lane; c < nch; c += 32) {
        const uint4 pg = __ldcs(rg + c), pu = __ldcs(ru + c);
        const float* xc = xs + c * 32;
        g = fmaf(__ldg(ag + (c >> 1)), dot32(lut, pg, xc), g);
        u = fmaf(__ldg(au + (c >> 1)), dot32(lut, pu, xc), u);
    }
    g = warp_sum(g);
    u = warp_sum(u);
    if (lane == 0) h[(int64_t)p * I + f] = g / (1.0f + expf(-g)) * u;
}

// y[t, c] = sum_j w[t,j] * (W_down,e[c] . h[t*k+j]), summed over j in slot order.
template <int CB>
__global__ void __launch_bounds__(DEC_THREADS) decode_down_kernel(
    const float* __restrict__ h, const int32_t* __restrict__ idx, const float* __restrict__ wts, int E, int k, int T,
    int H, int I, const uint8_t* __restrict__ packed, const float* __restrict__ absmax,
    __nv_bfloat16* __restrict__ y) {
    extern __shared__ float dsm[];
    float2* lut = reinterpret_cast<float2*>(dsm);
    float* hs = dsm + 512;                                  // I floats
    build_pair_lut<CB>(lut);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nch = I / 32, bpr = I / 64;
    constexpr int RPW = DEC_DN_ROWS / 8;                    // rows per warp
    float acc[RPW][8];
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int tt = 0; tt < 8; ++tt) acc[r][tt] = 0.0f;
    const int P = T * k;
    for (int p = 0; p < P; ++p) {
        __syncthreads();
        for (int i = threadIdx.x; i < I; i += blockDim.x) hs[i] = h[(int64_t)p * I + i];
        __syncthreads();
        const int e = __ldg(idx + p);
        if (e < 0 || e >= E) continue;
        const float wp = __ldg(wts + p);
        const int t = p / k;
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
            const int c = blockIdx.x * DEC_DN_ROWS + warp * RPW + r;
            if (c >= H) break;
            const uint4* rw = reinterpret_cast<const uint4*>(packed + ((int64_t)e * H + c) * (I / 2));
            const float* ar = absmax + ((int64_t)e * H + c) * bpr;
            float d = 0.0f;
            for (int ch = lane; ch < nch; ch += 32) d = fmaf(__ldg(ar + (ch >> 1)), dot32(lut, __ldcs(rw + ch), hs + ch * 32), d);
            d = warp_sum(d);
#pragma unroll
            for (int tt = 0; tt < 8; ++tt)
                if (tt == t) acc[r][tt] = fmaf(wp, d, acc[r][tt]);
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
            const int c = blockIdx.x * DEC_DN_ROWS + warp * RPW + r;
            if (c >= H) break;
#pragma unroll
            for (int tt = 0; tt < 8; ++tt)
                if (tt < T) y[(int64_t)tt * H + c] = __float2bfloat16_rn(acc[r][tt]);
        }
    }
}

template <int CB>
static cudaError_t decode_impl(int E, int H, int I, int k, int64_t T, const __nv_bfloat16* x, const int32_t* idx,
                               const float* w, const uint8_t* gu_packed, const float* gu_absmax,
                               const uint8_t* d_packed, const float* d_absmax, float* h, __nv_bfloat16* y,
                               cudaStream_t st) {
    const int P = (int)(T * k);
    const size_t sm1 = (512 + (size_t)H) * sizeof(float);
    const size_t sm2 = (512 + (size_t)I) * sizeof(float);
    static bool attr = false;
    if (!attr) {
        cudaFuncSetAttribute(decode_gateup_kernel<CB>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
        cudaFuncSetAttribute(decode_down_kernel<CB>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
        attr = true;
    }
    dim3 g1(P, (I + DEC_GU_FEATS - 1) / DEC_GU_FEATS);
    timing_begin(KK_DECODE_GATEUP, st);
    decode_gateup_kernel<CB><<<g1, DEC_THREADS, sm1, st>>>(x, idx, E, k, H, I, gu_packed, gu_absmax, h);
    timing_end(KK_DECODE_GATEUP, st);
    count_launch();
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    timing_begin(KK_DECODE_DOWN, st);
    decode_down_kernel<CB><<<(H + DEC_DN_ROWS - 1) / DEC_DN_ROWS, DEC_THREADS, sm2, st>>>(h, idx, w, E, k, (int)T, H, I,
                                                                                           d_packed, d_absmax, y);
    timing_end(KK_DECODE_DOWN, st);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_decode_forward(int codebook, int E, int H, int I, int k, int64_t T, const __nv_bfloat16* x,
                                  const int32_t* idx, const float* w, const uint8_t* gu_packed,
                                  const float* gu_absmax, const uint8_t* d_packed, const float* d_absmax,
                                  float* h_scratch, __nv_bfloat16* y, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    if (codebook == 0)
        return decode_impl<0>(E, H, I, k, T, x, idx, w, gu_packed, gu_absmax, d_packed, d_absmax, h_scratch, y, st);
    return decode_impl<1>(E, H, I, k, T, x, idx, w, gu_packed, gu_absmax, d_packed, d_absmax, h_scratch, y, st);
}

}  // namespace e4b
