// Per-expert LoRA over the frozen 4-bit base: the thin projections and the
// adapter gradients ("experts4bit-qlora" 0.4.0 description, "ExpertsLoRA(base,
// r, alpha)": only the adapters train; stacked per-expert adapters
// [num_experts, r, in] / [num_experts, out, r] as in the pages' prior art).
// The update of each projection is s (x A^T) B^T with s = alpha / r.  Inside the
// grouped GEMMs it is one more 64-deep k-stage: the thin operand s (x A^T) (rank
// padded to 64 with zeros, bf16) against the adapter B.  The two input
// gradients take s (dy B) against A the same way.  The kernels here make those
// thin operands and the four adapter gradients, which are sums over each
// expert's rows in grouped order (a fixed order: deterministic).  Both are
// small-N contractions (N = r <= 64): mma.sync m16n8k16 tiles fed from
// cp.async-staged shared memory, fp32 accumulation.
#include <mutex>

#include "lora.h"

namespace e4b {

namespace {

__device__ __forceinline__ void mma16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t r[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t r[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t& r0, uint32_t& r1, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t& r0, uint32_t& r1, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
// 16-byte copy global -> shared; src_bytes = 0 fills zeros
__device__ __forceinline__ void cp16z(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

constexpr int THIN_ROWS = 128, THIN_SA = 72;   // rows per CTA (8 warps x 16); smem row stride (bf16)
constexpr int THIN_STAGES = 4;                 // K chunks in the cp.async ring (3 in flight)
constexpr int THIN_SMEM = THIN_STAGES * (THIN_ROWS + 64) * THIN_SA * 2;
constexpr int GR_P = 32, GR_A = 128, GR_SU = GR_A + 8, GR_SV = 72;   // rows per chunk, columns per CTA

}  // namespace

// out[row, q] = s * sum_k in[row, k] * M_e(q, k) for the rows of half an m-tile
// (one expert, up to 128 of the m-tile's up to 256 rows; block 2 mt + h takes half h
// of m-tile mt), q < r; columns r..63 of out are zero.  M_e(q, k) = m[e][q][k]
// (Q_MAJOR, an A adapter [E, r, K]) or m[e][k][q] (a B adapter [E, K, r]).  K in
// chunks of 64 through a 4-deep cp.async ring (three chunks in flight: the kernel
// streams its rows from HBM once), the rows' chunk and M_e's chunk as [q][k] in
// shared memory; warp w owns rows 16w..16w+15 (one m16 tile).
template <bool Q_MAJOR>
__global__ void __launch_bounds__(256) lora_thin_kernel(const __nv_bfloat16* __restrict__ in, int K,
                                                        const __nv_bfloat16* __restrict__ m, int r, float s,
                                                        const int4* __restrict__ sched,
                                                        const int* __restrict__ tile_prefix, int E,
                                                        __nv_bfloat16* __restrict__ out) {
    extern __shared__ __align__(16) uint8_t sm[];
    const int mt = blockIdx.x >> 1, half = blockIdx.x & 1;
    if (mt >= __ldg(tile_prefix + E)) return;
    const int4 tl = __ldg(sched + mt);   // (expert, first row, rows, 0)
    const int e = tl.x, row0 = tl.y + THIN_ROWS * half, rows = min(tl.z - THIN_ROWS * half, THIN_ROWS);
    if (rows <= 0) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    __nv_bfloat16* sA = reinterpret_cast<__nv_bfloat16*>(sm);                 // [STAGES][128][72]
    __nv_bfloat16* sM = sA + THIN_STAGES * THIN_ROWS * THIN_SA;               // [STAGES][64][72]
    const __nv_bfloat16* me = m + (int64_t)e * r * K;
    const int nch = K / 64;
    auto stage = [&](int c, int b) {
        __nv_bfloat16* a = sA + b * THIN_ROWS * THIN_SA;
        for (int i = tid; i < THIN_ROWS * 8; i += 256) {
            const int rr = i >> 3, sg = i & 7;
            const bool ok = rr < rows;
            cp16z(smem_u32(a + rr * THIN_SA + sg * 8), in + (int64_t)(row0 + (ok ? rr : 0)) * K + c * 64 + sg * 8,
                  ok ? 16u : 0u);
        }
        __nv_bfloat16* mm = sM + b * 64 * THIN_SA;
        if (Q_MAJOR) {
            for (int i = tid; i < 64 * 8; i += 256) {
                const int q = i >> 3, sg = i & 7;
                const bool ok = q < r;
                cp16z(smem_u32(mm + q * THIN_SA + sg * 8), me + (int64_t)(ok ? q : 0) * K + c * 64 + sg * 8,
                      ok ? 16u : 0u);
            }
        } else {   // m[e][k][q]: transposed through registers, zeros past r
            for (int i = tid; i < 64 * 8; i += 256) {
                const int k = i >> 3, q0 = (i & 7) * 8;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (q0 < r) v = __ldg(reinterpret_cast<const uint4*>(me + (int64_t)(c * 64 + k) * r + q0));
                const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
                for (int j = 0; j < 8; ++j) mm[(q0 + j) * THIN_SA + k] = hv[j];
            }
        }
        cp_commit();
    };
    float acc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
    const int nt_n = r / 8;
#pragma unroll
    for (int c = 0; c < THIN_STAGES - 1; ++c) {   // prologue: chunks 0 .. STAGES-2 in flight
        if (c < nch) stage(c, c);
        else cp_commit();
    }
    for (int c = 0; c < nch; ++c) {
        const int cn = c + THIN_STAGES - 1;
        if (cn < nch) stage(cn, cn % THIN_STAGES);   // its slot was read in iteration c - 1
        else cp_commit();
        cp_wait<THIN_STAGES - 1>();                   // chunk c has landed (this thread's part)
        __syncthreads();                              // ... and everyone's
        const __nv_bfloat16* a = sA + (c % THIN_STAGES) * THIN_ROWS * THIN_SA;
        const __nv_bfloat16* mm = sM + (c % THIN_STAGES) * 64 * THIN_SA;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t af[4];
            ldsm_x4(af, smem_u32(a + (16 * warp + (lane & 15)) * THIN_SA + kk * 16 + (lane >> 4) * 8));
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                if (nt >= nt_n) break;
                uint32_t b0, b1;
                ldsm_x2(b0, b1, smem_u32(mm + (8 * nt + (lane & 7)) * THIN_SA + kk * 16 + ((lane >> 3) & 1) * 8));
                mma16816(acc[nt], af, b0, b1);
            }
        }
        __syncthreads();                              // slot c % STAGES is free for chunk c + STAGES
    }
    const int g = lane >> 2, c2 = (lane & 3) * 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int rr = 16 * warp + g + 8 * h;
        if (rr >= rows) continue;
        uint32_t* o = reinterpret_cast<uint32_t*>(out + (int64_t)(row0 + rr) * 64);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const float v0 = nt < nt_n ? s * acc[nt][2 * h] : 0.0f;
            const float v1 = nt < nt_n ? s * acc[nt][2 * h + 1] : 0.0f;
            o[(8 * nt + c2) >> 1] = pack_bf16x2(v0, v1);
        }
    }
}

// out for expert e = sum over its grouped rows p (offsets[e] .. offsets[e+1], in
// chunks of 32, ascending) of coef_p U[p, a] V[p, q], a < N, q < r: out[e][a][q],
// or out[e][q][a] with Q_MAJOR_OUT; fp32.  coef_p = topk_w[perm[p]] when coef_w,
// else 1 (applied to V's rows while they are staged).  Block: 128 columns a of
// one expert; warp w owns a = 16w..16w+15 as an m16 tile of U^T.
template <bool Q_MAJOR_OUT>
__global__ void __launch_bounds__(256) lora_grad_kernel(const __nv_bfloat16* __restrict__ U, int N,
                                                        const __nv_bfloat16* __restrict__ V, int r,
                                                        const int* __restrict__ offsets,
                                                        const float* __restrict__ topk_w,
                                                        const int* __restrict__ perm, int coef_w,
                                                        float* __restrict__ out) {
    __shared__ __align__(16) __nv_bfloat16 sU[2][GR_P][GR_SU];
    __shared__ __align__(16) __nv_bfloat16 sV[2][GR_P][GR_SV];
    const int e = blockIdx.y, a0 = blockIdx.x * GR_A;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int p0 = __ldg(offsets + e), p1 = __ldg(offsets + e + 1);
    const int nchunks = (p1 - p0 + GR_P - 1) / GR_P;
    auto stage = [&](int c, int b) {
        const int pb = p0 + c * GR_P;
        for (int i = tid; i < GR_P * (GR_A / 8); i += 256) {   // U rows: 32 x 128 columns
            const int pp = i / (GR_A / 8), sg = i % (GR_A / 8);
            const int a = a0 + sg * 8;
            const bool ok = pb + pp < p1 && a < N;
            cp16z(smem_u32(&sU[b][pp][sg * 8]), U + (int64_t)(ok ? pb + pp : p0) * N + (ok ? a : 0), ok ? 16u : 0u);
        }
        cp_commit();
        {   // V rows scaled by coef_p: 32 x 64 (ranks past r are zero in V already)
            const int pp = tid >> 3, q0 = (tid & 7) * 8;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (pb + pp < p1) {
                v = __ldg(reinterpret_cast<const uint4*>(V + (int64_t)(pb + pp) * 64 + q0));
                if (coef_w) {
                    const float cf = __ldg(topk_w + __ldg(perm + pb + pp));
                    uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        w[j] = pack_bf16x2(cf * __uint_as_float(w[j] << 16), cf * __uint_as_float(w[j] & 0xFFFF0000u));
                }
            }
            *reinterpret_cast<uint4*>(&sV[b][pp][q0]) = v;
        }
    };
    float acc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
    const int nt_n = r / 8;
    if (nchunks > 0) stage(0, 0);
    for (int c = 0; c < nchunks; ++c) {
        if (c + 1 < nchunks) stage(c + 1, (c + 1) & 1);
        else cp_commit();
        cp_wait1();
        __syncthreads();
        const int b = c & 1;
#pragma unroll
        for (int kk = 0; kk < GR_P / 16; ++kk) {
            uint32_t af[4];   // A = U^T: 16 columns a x 16 rows p
            const int mtx = lane >> 3;
            ldsm_x4_t(af, smem_u32(&sU[b][kk * 16 + (mtx >> 1) * 8 + (lane & 7)][16 * warp + (mtx & 1) * 8]));
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                if (nt >= nt_n) break;
                uint32_t b0, b1;   // B = V: 16 rows p x 8 ranks q
                ldsm_x2_t(b0, b1, smem_u32(&sV[b][kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7)][8 * nt]));
                mma16816(acc[nt], af, b0, b1);
            }
        }
        __syncthreads();
    }
    const int g = lane >> 2, c2 = (lane & 3) * 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int a = a0 + 16 * warp + g + 8 * h;
        if (a >= N) continue;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            if (nt >= nt_n) break;
            const int q = 8 * nt + c2;
            if (Q_MAJOR_OUT) {
                out[((int64_t)e * r + q) * N + a] = acc[nt][2 * h];
                out[((int64_t)e * r + q + 1) * N + a] = acc[nt][2 * h + 1];
            } else {
                *reinterpret_cast<float2*>(out + ((int64_t)e * N + a) * r + q) =
                    make_float2(acc[nt][2 * h], acc[nt][2 * h + 1]);
            }
        }
    }
}

// t[e][q][k] = m[e][k][q]: a B adapter [E, K, r] in the [E, r, K] layout of the thin
// kernel (tiled through shared memory; K a multiple of 64).
__global__ void __launch_bounds__(256) lora_transpose_kernel(const __nv_bfloat16* __restrict__ m, int K, int r,
                                                             __nv_bfloat16* __restrict__ t) {
    __shared__ __nv_bfloat16 tile[64][65];
    const int e = blockIdx.y, k0 = blockIdx.x * 64;
    const __nv_bfloat16* me = m + (int64_t)e * K * r;
    for (int i = threadIdx.x; i < 64 * r; i += blockDim.x) {   // rows k0..k0+63, r contiguous each
        const int k = i / r, q = i - k * r;
        tile[q][k] = me[(int64_t)(k0 + k) * r + q];
    }
    __syncthreads();
    __nv_bfloat16* te = t + (int64_t)e * r * K;
    for (int i = threadIdx.x; i < 64 * r; i += blockDim.x) {   // rows q, 64 contiguous k each
        const int q = i >> 6, k = i & 63;
        te[(int64_t)q * K + k0 + k] = tile[q][k];
    }
}

cudaError_t launch_lora_transpose(const __nv_bfloat16* m, int E, int K, int r, __nv_bfloat16* t, cudaStream_t st) {
    if (K % 64 || r < 8 || r > 64) return cudaErrorInvalidValue;
    lora_transpose_kernel<<<dim3(K / 64, E), 256, 0, st>>>(m, K, r, t);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_lora_thin(const __nv_bfloat16* in, int K, const __nv_bfloat16* m, bool m_q_major, int r, float s,
                             const int4* sched, const int* tile_prefix, int E, int max_m_tiles, __nv_bfloat16* out,
                             cudaStream_t st) {
    if (max_m_tiles <= 0) return cudaSuccess;
    if (K % 64 || r < 8 || r > 64 || r % 8) return cudaErrorInvalidValue;
    static std::mutex mu;
    static bool set[64][2] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!set[dev][m_q_major]) {
            err = m_q_major ? cudaFuncSetAttribute(lora_thin_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   THIN_SMEM)
                            : cudaFuncSetAttribute(lora_thin_kernel<false>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, THIN_SMEM);
            if (err != cudaSuccess) return err;
            set[dev][m_q_major] = true;
        }
    }
    if (m_q_major)
        lora_thin_kernel<true><<<2 * max_m_tiles, 256, THIN_SMEM, st>>>(in, K, m, r, s, sched, tile_prefix, E, out);
    else
        lora_thin_kernel<false><<<2 * max_m_tiles, 256, THIN_SMEM, st>>>(in, K, m, r, s, sched, tile_prefix, E, out);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_lora_grad(const __nv_bfloat16* U, int N, const __nv_bfloat16* V, int r, const int* offsets,
                             int E, const float* topk_w, const int* perm, bool coef_w, bool q_major_out, float* out,
                             cudaStream_t st) {
    if (r < 8 || r > 64 || r % 8 || N % 64) return cudaErrorInvalidValue;
    const dim3 grid((N + GR_A - 1) / GR_A, E);
    if (q_major_out)
        lora_grad_kernel<true><<<grid, 256, 0, st>>>(U, N, V, r, offsets, topk_w, perm, coef_w ? 1 : 0, out);
    else
        lora_grad_kernel<false><<<grid, 256, 0, st>>>(U, N, V, r, offsets, topk_w, perm, coef_w ? 1 : 0, out);
    count_launch();
    return cudaGetLastError();
}

}  // namespace e4b
