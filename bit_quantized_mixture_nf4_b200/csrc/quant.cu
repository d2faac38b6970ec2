// Blockwise 4-bit quantize and dequantize kernels (HBM-bound).
//
// Quantize follows "experts4bit-qlora 0.1.0" experts.py, Experts4bit.from_float /
// _quantize_stack: per 64 contiguous in-features of each row, absmax = max|w|,
// every element divided by absmax and mapped to the nearest codebook value (an
// exact tie goes to the smaller value), two codes per byte with the first
// element in the high nibble.  Dequantize follows _dequantize_expert: code value
// times absmax in fp32, optionally rounded to bf16 (nearest-even).
#include <cmath>
#include <limits>
#include <mutex>
#include <utility>

#include "e4b_internal.h"

namespace e4b {

// Codes in ascending order of their value (NF4: identity; FP4: -1 .. -1/12,
// +0, 1/12 .. 1; the -0 code is never produced).
__device__ __forceinline__ int sorted_code(int cb, int r) {
    if (cb == 0) return r;
    return r < 7 ? 15 - r : r - 7;
}

// 4 threads per 64-element block; thread q of a quad holds elements
// 16*i + 4*q + {0..3}, i = 0..3, so each quad reads 64 contiguous bytes per load.
template <int CB>
__global__ void __launch_bounds__(256) quantize_kernel(const float* __restrict__ w, int64_t nblocks,
                                                       uint8_t* __restrict__ packed, float* __restrict__ absmax) {
    __shared__ __align__(16) uint16_t s_out[8][128];   // per warp: 8 blocks x 32 packed bytes
    constexpr int NV = (CB == 0) ? 16 : 15;   // distinct codebook values
    // the 15 midpoints between consecutive sorted codebook values, in registers (+inf past
    // the last one); the nearest-value search below selects among them without memory loads
    float m[15];
#pragma unroll
    for (int r = 0; r < 15; ++r) {
        if (r < NV - 1) {
            const float lo = c_code[CB][sorted_code(CB, r)], hi = c_code[CB][sorted_code(CB, r + 1)];
            m[r] = __fmul_rn(__fadd_rn(lo, hi), 0.5f);
        } else {
            m[r] = __int_as_float(0x7f800000);   // +inf: never below a finite value
        }
    }
    const int q = threadIdx.x & 3;
    const int zero_code = (CB == 0) ? 7 : 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x / 4;
    // the loop bound is taken per warp (8 blocks; every lane runs the same
    // iterations, for the __syncwarp in the body); out-of-range lanes skip work
    const int lb = (threadIdx.x & 31) >> 2;   // block within the warp
    for (int64_t bw = ((int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31)) / 4; bw < nblocks; bw += stride) {
        const int64_t b = bw + lb;
        const bool valid = b < nblocks;
        const float4* src = reinterpret_cast<const float4*>(w + b * 64);
        float v[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 f = valid ? __ldcs(src + i * 4 + q) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
        }
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[i]));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
        if (q == 0 && valid) absmax[b] = a;
        uint32_t code[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (a == 0.0f) {
                code[i] = zero_code;
            } else {
                const float n = __fdiv_rn(v[i], a);
                // r = number of midpoints strictly below n: a 4-level binary search whose
                // pivots m[7], m[r+3], m[r+1], m[r] are picked by selects on r's bits
                const bool b3 = m[7] < n;
                const bool b2 = (b3 ? m[11] : m[3]) < n;
                const float p1 = b3 ? (b2 ? m[13] : m[9]) : (b2 ? m[5] : m[1]);
                const bool b1 = p1 < n;
                const float p0 = b3 ? (b2 ? (b1 ? m[14] : m[12]) : (b1 ? m[10] : m[8]))
                                    : (b2 ? (b1 ? m[6] : m[4]) : (b1 ? m[2] : m[0]));
                const int r = (b3 ? 8 : 0) + (b2 ? 4 : 0) + (b1 ? 2 : 0) + ((p0 < n) ? 1 : 0);
                code[i] = (uint32_t)sorted_code(CB, r);
            }
        }
        // The warp's 8 blocks are 256 contiguous packed bytes: assemble them in
        // shared memory, then each lane stores 8 bytes (one coalesced 256-byte store).
        uint16_t* stage = s_out[threadIdx.x >> 5];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t b0 = (code[4 * i] << 4) | code[4 * i + 1];
            const uint32_t b1 = (code[4 * i + 2] << 4) | code[4 * i + 3];
            stage[(lb * 32 + i * 8 + q * 2) / 2] = (uint16_t)(b0 | (b1 << 8));
        }
        __syncwarp();
        const int lane = threadIdx.x & 31;
        if (bw + lane / 4 < nblocks)
            *reinterpret_cast<uint2*>(packed + bw * 32 + lane * 8) = reinterpret_cast<const uint2*>(stage)[lane];
        __syncwarp();
    }
}

// One thread per 16 packed bytes (32 elements, half a block).
// CB 2 (MXFP4): chunk c is one 32-element block; its scale byte is mx[row * S + j]
// with row = c / nb, j = c % nb (nb = in / 32 blocks per row).
template <int CB, bool BF16>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint8_t* __restrict__ packed,
                                                         const float* __restrict__ absmax, int64_t nchunks,
                                                         void* __restrict__ out, const uint8_t* __restrict__ mx,
                                                         int64_t nb, int64_t S) {
    __shared__ float s_val[16];
    __shared__ uint4 s_stage[8][128];   // per warp: 32 lanes x 4 pieces of 16 bytes
    if (threadIdx.x < 16) s_val[threadIdx.x] = c_code[CB][threadIdx.x];
    __syncthreads();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // the loop bound is taken per warp (every lane of a warp runs the same
    // iterations, for the __syncwarp in the body); out-of-range lanes only skip work
    for (int64_t cw = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); cw < nchunks; cw += stride) {
        const int64_t c = cw + (threadIdx.x & 31);
        const bool valid = c < nchunks;
        const uint4 pk = valid ? __ldcs(reinterpret_cast<const uint4*>(packed) + c) : make_uint4(0u, 0u, 0u, 0u);
        float a = 0.0f;
        if (valid) a = (CB == 2) ? mx_scale(__ldg(mx + (c / nb) * S + c % nb)) : __ldg(absmax + (c >> 1));
        const uint32_t words[4] = {pk.x, pk.y, pk.z, pk.w};
        if (BF16) {
            // A warp's 32 chunks are 2 KB of contiguous output.  Each lane decodes
            // its 64 bytes into shared memory (16-byte piece s of lane l at slot
            // (s + l/2) mod 4: conflict-free), then the warp stores 512 contiguous
            // bytes per instruction.
            const BlockTable tb = make_table<CB>(a);
            const int lane = threadIdx.x & 31;
            uint4* stage = s_stage[threadIdx.x >> 5];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t o[4];
                decode_word(tb, words[i], o);
                stage[lane * 4 + ((i + (lane >> 1)) & 3)] = make_uint4(o[0], o[1], o[2], o[3]);
            }
            __syncwarp();
            const int64_t c0 = c - lane;   // first chunk of this warp
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + c0 * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int p = 32 * i + lane, t = p >> 2, sub = p & 3;   // piece p of the warp's output
                if (c0 + t < nchunks) __stcs(dst + p, stage[t * 4 + ((sub + (t >> 1)) & 3)]);
            }
            __syncwarp();
        } else {
            if (!valid) continue;
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t x = words[i];
                float f[8];
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) {
                    const uint32_t byte = (x >> (8 * bb)) & 0xFFu;
                    f[2 * bb] = __fmul_rn(s_val[byte >> 4], a);
                    f[2 * bb + 1] = __fmul_rn(s_val[byte & 15u], a);
                }
                __stcs(dst + 2 * i, make_float4(f[0], f[1], f[2], f[3]));
                __stcs(dst + 2 * i + 1, make_float4(f[4], f[5], f[6], f[7]));
            }
        }
    }
}

static int grid_for(int64_t work_items, int threads) {
    const int64_t blocks = (work_items + threads - 1) / threads;
    return (int)std::max<int64_t>(1, std::min<int64_t>(blocks, (int64_t)num_sms() * 8));
}

cudaError_t launch_quantize(const float* w, int64_t nblocks, int codebook, uint8_t* packed, float* absmax,
                            cudaStream_t st) {
    if (nblocks == 0) return cudaSuccess;
    const int grid = grid_for(nblocks * 4, 256);
    timing_begin(KK_QUANT, st);
    if (codebook == 0) quantize_kernel<0><<<grid, 256, 0, st>>>(w, nblocks, packed, absmax);
    else quantize_kernel<1><<<grid, 256, 0, st>>>(w, nblocks, packed, absmax);
    timing_end(KK_QUANT, st);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* packed, const float* absmax, int64_t n, int codebook, int out_bf16,
                              void* out, cudaStream_t st) {
    const int64_t nchunks = n / 32;
    if (nchunks == 0) return cudaSuccess;
    const int grid = grid_for(nchunks, 256);
    timing_begin(KK_DEQUANT, st);
    if (codebook == 0) {
        if (out_bf16) dequantize_kernel<0, true><<<grid, 256, 0, st>>>(packed, absmax, nchunks, out, nullptr, 1, 1);
        else dequantize_kernel<0, false><<<grid, 256, 0, st>>>(packed, absmax, nchunks, out, nullptr, 1, 1);
    } else {
        if (out_bf16) dequantize_kernel<1, true><<<grid, 256, 0, st>>>(packed, absmax, nchunks, out, nullptr, 1, 1);
        else dequantize_kernel<1, false><<<grid, 256, 0, st>>>(packed, absmax, nchunks, out, nullptr, 1, 1);
    }
    timing_end(KK_DEQUANT, st);
    count_launch();
    return cudaGetLastError();
}

int64_t mxfp4_scale_stride(int64_t in) { return ((in / 32) + 15) / 16 * 16; }

// MXFP4 quantize (OCP Microscaling Formats v1.0, the gpt-oss expert storage):
// one thread per (row, scale byte j); j < in/32 quantizes the 32-element block j:
// X = floor(log2 amax) - 2 = (biased exponent of amax) - 129, at least -127 (an
// all-zero block: -127); each element v * 2^-X (exact) goes to the nearest E2M1
// value, ties to the even code, saturating at 6; a zero result is +0.  Bytes
// j >= in/32 are the row's zero padding.
__global__ void __launch_bounds__(256) quantize_mxfp4_kernel(const float* __restrict__ w, int64_t rows, int64_t in,
                                                             int64_t S, uint8_t* __restrict__ packed,
                                                             uint8_t* __restrict__ scales) {
    const int64_t nb = in / 32, total = rows * S;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / S, j = i - r * S;
        if (j >= nb) {
            scales[i] = 0;
            continue;
        }
        const float4* src = reinterpret_cast<const float4*>(w + r * in + j * 32);
        float v[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float4 f = __ldcs(src + k);
            v[4 * k] = f.x; v[4 * k + 1] = f.y; v[4 * k + 2] = f.z; v[4 * k + 3] = f.w;
        }
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < 32; ++k) amax = fmaxf(amax, fabsf(v[k]));
        const int eb = (int)((__float_as_uint(amax) >> 23) & 0xFFu);   // biased exponent (0: zero / subnormal)
        const int X = max(eb - 129, -127);
        scales[i] = (uint8_t)(X + 127);
        const float inv = __int_as_float((127 - X) << 23);   // 2^-X, a normal float for X in [-127, 125]
        uint32_t words[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint32_t wv = 0;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const float p = __fmul_rn(v[8 * k + t], inv);
                const float a = fabsf(p);
                // nearest E2M1 magnitude: ties at 0.25, 1.25, 2.5, 5 go down (even code below),
                // at 0.75, 1.75, 3.5 up (even code above); 6 and beyond saturate to code 7
                uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) +
                             (a > 5.0f);
                if (amax == 0.0f) c = 0;
                if (c != 0 && p < 0.0f) c |= 8u;
                // element 2b in the high nibble of byte b: byte t/2 of the word, high nibble for even t
                wv |= c << (8 * (t >> 1) + ((t & 1) ? 0 : 4));
            }
            words[k] = wv;
        }
        *reinterpret_cast<uint4*>(packed + (r * in + j * 32) / 2) = make_uint4(words[0], words[1], words[2], words[3]);
    }
}

cudaError_t launch_quantize_mxfp4(const float* w, int64_t rows, int64_t in, uint8_t* packed, uint8_t* scales,
                                  cudaStream_t st) {
    if (rows == 0 || in == 0) return cudaSuccess;
    if (in % 32) return cudaErrorInvalidValue;
    const int64_t S = mxfp4_scale_stride(in);
    const int grid = grid_for(rows * S, 256);
    timing_begin(KK_QUANT, st);
    quantize_mxfp4_kernel<<<grid, 256, 0, st>>>(w, rows, in, S, packed, scales);
    timing_end(KK_QUANT, st);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_dequantize_mxfp4(const uint8_t* packed, const uint8_t* scales, int64_t rows, int64_t in,
                                    int out_bf16, void* out, cudaStream_t st) {
    if (in % 32) return cudaErrorInvalidValue;
    const int64_t nchunks = rows * (in / 32);
    if (nchunks == 0) return cudaSuccess;
    const int grid = grid_for(nchunks, 256);
    const int64_t nb = in / 32, S = mxfp4_scale_stride(in);
    timing_begin(KK_DEQUANT, st);
    if (out_bf16) dequantize_kernel<2, true><<<grid, 256, 0, st>>>(packed, nullptr, nchunks, out, scales, nb, S);
    else dequantize_kernel<2, false><<<grid, 256, 0, st>>>(packed, nullptr, nchunks, out, scales, nb, S);
    timing_end(KK_DEQUANT, st);
    count_launch();
    return cudaGetLastError();
}

}  // namespace e4b

namespace e4b {

// ------------------------------------------------------- 8-bit blockwise modes
// int8: the dynamic tree map (Dettmers et al. 2022, block-wise 8-bit
// quantization): bit 7 the sign; in the 7-bit tail, E leading zeros give the
// decimal exponent 10^-E, then an indicator bit, then F = 6 - E bits of a linear
// fraction on [0.1, 1] at bin centres; tail 0 is 0, or +1 with the sign set.
// fp8: the E4M3 values (bias 7, subnormals, S.1111.111 NaN) divided by 448.  Both
// normalised to max 1 and used with 64-element blocks and fp32 absmax like the
// 4-bit codebooks ("experts4bit-qlora" 0.4.0, "Storage modes: the support
// matrix": int8 a blockwise dynamic map, fp8 an e4m3 codebook).
static float code8_value(int cb, int q) {
    if (cb == 3) {
        static const double kPow10[7] = {1.0, 0.1, 0.01, 0.001, 0.0001, 0.00001, 0.000001};
        const int s = q >> 7, t = q & 127;
        if (t == 0) return s ? 1.0f : 0.0f;
        int E = 0;
        while (!(t & (64 >> E))) ++E;
        const int F = 6 - E, j = t & ((1 << F) - 1);
        const double v = kPow10[E] * (0.1 + 0.9 * (j + 0.5) / (double)(1 << F));
        return (float)(s ? -v : v);
    }
    const int s = q >> 7, e = (q >> 3) & 15, m = q & 7;
    if (e == 15 && m == 7) return std::numeric_limits<float>::quiet_NaN();
    const double mag = (e == 0) ? (m / 8.0) * std::ldexp(1.0, -6) : (1.0 + m / 8.0) * std::ldexp(1.0, e - 7);
    const float v = (float)(mag / 448.0);
    return s ? -v : v;
}

// Per codebook: the value of every code, the sorted distinct values' midpoints
// (+inf padded) and the code of each sorted value.
struct Table8 {
    float value[256];
    float mid[256];
    uint8_t code[256];
    int n;
};
static __constant__ Table8 c_t8[2];   // [0] int8, [1] fp8

static Table8 make_table8(int cb) {
    Table8 t{};
    float v[256];
    int c[256], n = 0;
    for (int q = 0; q < 256; ++q) {
        t.value[q] = code8_value(cb, q);
        if (t.value[q] != t.value[q] || (cb == 4 && q == 0x80)) continue;   // NaN and -0 never produced
        v[n] = t.value[q];
        c[n] = q;
        ++n;
    }
    for (int i = 1; i < n; ++i)
        for (int k = i; k > 0 && v[k - 1] > v[k]; --k) {
            std::swap(v[k], v[k - 1]);
            std::swap(c[k], c[k - 1]);
        }
    for (int i = 0; i < 256; ++i) {
        t.mid[i] = i + 1 < n ? (v[i] + v[i + 1]) * 0.5f : std::numeric_limits<float>::infinity();
        t.code[i] = (uint8_t)(i < n ? c[i] : 0);
    }
    t.n = n;
    return t;
}

static cudaError_t ensure_tables8() {
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (done[dev]) return cudaSuccess;
    Table8 t[2] = {make_table8(3), make_table8(4)};
    e = cudaMemcpyToSymbol(c_t8, t, sizeof(t));
    if (e == cudaSuccess) done[dev] = true;
    return e;
}

// One thread per 64-element block: n = w / absmax (IEEE division), code of the
// sorted value r = the number of midpoints strictly below n (an exact tie goes to
// the smaller value), found by an 8-step binary search in shared memory.
template <int T8>
__global__ void __launch_bounds__(256) quantize8_kernel(const float* __restrict__ w, int64_t nblocks,
                                                        uint8_t* __restrict__ codes, float* __restrict__ absmax) {
    __shared__ float mid[256];
    __shared__ uint8_t cds[256];
    mid[threadIdx.x] = c_t8[T8].mid[threadIdx.x];
    cds[threadIdx.x] = c_t8[T8].code[threadIdx.x];
    __syncthreads();
    uint8_t zero_code = 0;
    for (int i = 0; i < 256; ++i)
        if (c_t8[T8].value[i] == 0.0f && !(T8 == 1 && i == 0x80)) { zero_code = (uint8_t)i; break; }
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks; b += (int64_t)gridDim.x * blockDim.x) {
        const float4* src = reinterpret_cast<const float4*>(w + b * 64);
        float a = 0.0f;
        for (int k = 0; k < 16; ++k) {
            const float4 f = __ldg(src + k);
            a = fmaxf(a, fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w))));
        }
        absmax[b] = a;
        uint32_t* dst = reinterpret_cast<uint32_t*>(codes + b * 64);
        for (int k = 0; k < 16; ++k) {
            const float4 f = __ldcs(src + k);
            const float x[4] = {f.x, f.y, f.z, f.w};
            uint32_t word = 0;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                uint32_t code = zero_code;
                if (a != 0.0f) {
                    const float n = __fdiv_rn(x[t], a);
                    int r = 0;   // midpoints below n: the largest r with mid[r - 1] < n
#pragma unroll
                    for (int step = 128; step >= 1; step >>= 1)
                        if (mid[r + step - 1] < n) r += step;
                    code = cds[r];
                }
                word |= code << (8 * t);
            }
            dst[k] = word;
        }
    }
}

// value = code value * absmax (fp32), then bf16 nearest-even or fp32; one thread
// per 16 codes.
template <int T8, bool BF16>
__global__ void __launch_bounds__(256) dequantize8_kernel(const uint8_t* __restrict__ codes,
                                                          const float* __restrict__ absmax, int64_t nchunks,
                                                          void* __restrict__ out) {
    __shared__ float val[256];
    val[threadIdx.x] = c_t8[T8].value[threadIdx.x];
    __syncthreads();
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < nchunks; c += (int64_t)gridDim.x * blockDim.x) {
        const uint4 q = __ldcs(reinterpret_cast<const uint4*>(codes) + c);
        const float a = __ldg(absmax + c / 4);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
        float f[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) f[i] = __fmul_rn(val[(w[i >> 2] >> (8 * (i & 3))) & 0xFFu], a);
        if (BF16) {
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = pack_bf16x2(f[2 * i], f[2 * i + 1]);
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + c * 16);
            __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
            __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
        } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + c * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) __stcs(dst + i, make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]));
        }
    }
}

cudaError_t launch_quantize8(const float* w, int64_t nblocks, int codebook, uint8_t* codes, float* absmax,
                             cudaStream_t st) {
    if (nblocks == 0) return cudaSuccess;
    cudaError_t e = ensure_tables8();
    if (e != cudaSuccess) return e;
    const int grid = grid_for(nblocks, 256);
    timing_begin(KK_QUANT, st);
    if (codebook == 3) quantize8_kernel<0><<<grid, 256, 0, st>>>(w, nblocks, codes, absmax);
    else quantize8_kernel<1><<<grid, 256, 0, st>>>(w, nblocks, codes, absmax);
    timing_end(KK_QUANT, st);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_dequantize8(const uint8_t* codes, const float* absmax, int64_t n, int codebook, int out_bf16,
                               void* out, cudaStream_t st) {
    const int64_t nchunks = n / 16;
    if (nchunks == 0) return cudaSuccess;
    cudaError_t e = ensure_tables8();
    if (e != cudaSuccess) return e;
    const int grid = grid_for(nchunks, 256);
    timing_begin(KK_DEQUANT, st);
    if (codebook == 3) {
        if (out_bf16) dequantize8_kernel<0, true><<<grid, 256, 0, st>>>(codes, absmax, nchunks, out);
        else dequantize8_kernel<0, false><<<grid, 256, 0, st>>>(codes, absmax, nchunks, out);
    } else {
        if (out_bf16) dequantize8_kernel<1, true><<<grid, 256, 0, st>>>(codes, absmax, nchunks, out);
        else dequantize8_kernel<1, false><<<grid, 256, 0, st>>>(codes, absmax, nchunks, out);
    }
    timing_end(KK_DEQUANT, st);
    count_launch();
    return cudaGetLastError();
}

}  // namespace e4b
