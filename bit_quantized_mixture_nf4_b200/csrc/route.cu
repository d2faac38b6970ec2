// Router and grouping kernels.
//
// Routing (softmax, top-k, optional renormalisation) produces the top_k_index /
// top_k_weights that "experts4bit-qlora 0.1.0" experts.py Experts4bit.forward
// takes as inputs.  Grouping replaces that forward's one-hot expert mask, hit
// list and per-expert torch.where (each a host synchronisation) with a
// histogram, a prefix scan and a stable counting-sort permutation that stay on
// the device: rows of expert e are [offsets[e], offsets[e+1]), tokens ascending.
#include "e4b_internal.h"

namespace e4b {

// One warp per token (the per-token routing is route_token_warp, shared with
// the small-batch kernels).
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, int64_t T, int E, int k,
                                                    int renorm, int32_t* __restrict__ idx,
                                                    float* __restrict__ wts) {
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    int e;
    float p;
    route_token_warp(logits + t * E, E, k, renorm, lane, &e, &p);
    if (lane < k) {
        idx[t * k + lane] = e;
        wts[t * k + lane] = p;
    }
}

// Per-chunk expert histogram (order-independent, so atomics keep it exact).
__global__ void __launch_bounds__(256) hist_kernel(const int32_t* __restrict__ idx, int64_t P, int E,
                                                   int32_t* __restrict__ chunk_counts) {
    __shared__ int cnt[256];
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const int64_t p0 = (int64_t)blockIdx.x * kChunkPairs;
    for (int i = threadIdx.x; i < kChunkPairs; i += blockDim.x) {
        const int64_t pp = p0 + i;
        if (pp < P) {
            const int e = __ldg(idx + pp);
            if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);   // out-of-range experts are dropped
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_counts[(int64_t)blockIdx.x * E + e] = cnt[e];
}

// Single block: totals, exclusive scan over experts, per-chunk bases, m-tile prefix.
__global__ void __launch_bounds__(256) scan_kernel(const int32_t* __restrict__ chunk_counts, int nchunks, int E,
                                                   int tile_rows, int32_t* __restrict__ chunk_base,
                                                   int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                   int32_t* __restrict__ tile_prefix, int4* __restrict__ sched) {
    __shared__ int s_tot[256], s_tiles[256];
    const int e = threadIdx.x;
    int tot = 0;
    if (e < E)
        for (int c = 0; c < nchunks; ++c) tot += chunk_counts[(int64_t)c * E + e];
    s_tot[e] = (e < E) ? tot : 0;
    s_tiles[e] = (e < E) ? (tot + tile_rows - 1) / tile_rows : 0;
    __syncthreads();
    if (e == 0) {   // E <= 256: a serial scan is short and exact
        int run = 0, trun = 0;
        for (int i = 0; i < E; ++i) {
            const int a = s_tot[i], b = s_tiles[i];
            s_tot[i] = run;
            s_tiles[i] = trun;
            run += a;
            trun += b;
        }
        offsets[E] = run;
        tile_prefix[E] = trun;
    }
    __syncthreads();
    if (e < E) {
        counts[e] = tot;
        offsets[e] = s_tot[e];
        tile_prefix[e] = s_tiles[e];
        int run = s_tot[e];
        for (int c = 0; c < nchunks; ++c) {
            chunk_base[(int64_t)c * E + e] = run;
            run += chunk_counts[(int64_t)c * E + e];
        }
        // m-tile schedule: (expert, first row, rows) of every m-tile, experts ascending
        const int nt = (tot + tile_rows - 1) / tile_rows;
        for (int m = 0; m < nt; ++m)
            sched[s_tiles[e] + m] = make_int4(e, s_tot[e] + m * tile_rows, min(tile_rows, tot - m * tile_rows), 0);
    }
}

// Stable scatter: pairs of a chunk keep their order inside each expert.
__global__ void __launch_bounds__(256) scatter_kernel(const int32_t* __restrict__ idx, int64_t P, int E,
                                                      const int32_t* __restrict__ chunk_base,
                                                      int32_t* __restrict__ perm) {
    constexpr int WARPS = 8, PER_WARP = kChunkPairs / WARPS;
    __shared__ int wbase[WARPS][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < WARPS * 256; i += blockDim.x) (&wbase[0][0])[i] = 0;
    __syncthreads();
    const int64_t p0 = (int64_t)blockIdx.x * kChunkPairs + warp * PER_WARP;
    for (int it = 0; it < PER_WARP; it += 32) {
        const int64_t pp = p0 + it + lane;
        if (pp < P) {
            const int e = __ldg(idx + pp);
            if (e >= 0 && e < E) atomicAdd(&wbase[warp][e], 1);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = chunk_base[(int64_t)blockIdx.x * E + e];
        for (int w = 0; w < WARPS; ++w) {
            const int c = wbase[w][e];
            wbase[w][e] = run;
            run += c;
        }
    }
    __syncthreads();
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int it = 0; it < PER_WARP; it += 32) {
        const int64_t pp = p0 + it + lane;
        int e = (pp < P) ? __ldg(idx + pp) : -1;
        if (e >= E) e = -1;
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & lt_mask);
        const int base = (e >= 0) ? wbase[warp][e] : 0;
        __syncwarp();
        if (e >= 0) {
            perm[base + rank] = (int32_t)pp;
            if (rank == 0) wbase[warp][e] = base + __popc(peers);
        }
        __syncwarp();
    }
}

// dst[r] = src[perm[r] / k]: one warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256) gather_rows_kernel(const __nv_bfloat16* __restrict__ src,
                                                          const int32_t* __restrict__ perm,
                                                          const int32_t* __restrict__ nrows, int k, int64_t P,
                                                          int H, __nv_bfloat16* __restrict__ dst) {
    const int lane = threadIdx.x & 31;
    P = min(P, (int64_t)__ldg(nrows));   // rows that belong to a valid expert
    const int64_t wstride = (int64_t)gridDim.x * blockDim.x / 32;
    const int vec = H / 8;
    for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; r < P; r += wstride) {
        const int64_t t = __ldg(perm + r) / k;
        const uint4* s = reinterpret_cast<const uint4*>(src + t * H);
        uint4* d = reinterpret_cast<uint4*>(dst + r * H);
        for (int i = lane; i < vec; i += 32) d[i] = __ldg(s + i);
    }
}

// y[t] = bf16( sum_j fp32(slot[t*k + j]) ), j ascending: the weighted combine of
// the k expert outputs of each token in fp32 (experts4bit-qlora 0.1.0 experts.py,
// Experts4bit.forward: per-expert outputs in the compute dtype, index_add_ into an
// fp32 buffer).  Slots of out-of-range experts are skipped.
__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16* __restrict__ slots,
                                                      const int32_t* __restrict__ idx, int E, int k, int64_t T,
                                                      int H, __nv_bfloat16* __restrict__ y) {
    const int h8 = H / 8;
    const int64_t n = T * h8;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const int64_t t = i / h8;
        const int c = (int)(i - t * h8);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < k; ++j) {
            const int e = __ldg(idx + t * k + j);
            if (e < 0 || e >= E) continue;
            const uint4 v = __ldcs(reinterpret_cast<const uint4*>(slots + (t * k + j) * H) + c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc[2 * q] += __uint_as_float(w[q] << 16);
                acc[2 * q + 1] += __uint_as_float(w[q] & 0xFFFF0000u);
            }
        }
        reinterpret_cast<uint4*>(y)[i] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                                    pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    }
}

static int capped_grid(int64_t blocks) {
    return (int)std::max<int64_t>(1, std::min<int64_t>(blocks, (int64_t)num_sms() * 16));
}

cudaError_t launch_route(const float* logits, int64_t T, int E, int k, int renorm, int32_t* idx, float* w,
                         cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int64_t blocks = (T * 32 + 255) / 256;
    timing_begin(KK_ROUTE, st);
    route_kernel<<<(unsigned)blocks, 256, 0, st>>>(logits, T, E, k, renorm, idx, w);
    timing_end(KK_ROUTE, st);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_group(const int32_t* idx, int64_t P, int E, int tile_rows, int32_t* chunk_counts,
                         int32_t* chunk_base, int32_t* counts, int32_t* offsets, int32_t* tile_prefix,
                         int4* sched, int32_t* perm, cudaStream_t st) {
    const int nchunks = (int)((P + kChunkPairs - 1) / kChunkPairs);
    if (nchunks == 0) return cudaSuccess;
    timing_begin(KK_GROUP, st);
    hist_kernel<<<nchunks, 256, 0, st>>>(idx, P, E, chunk_counts);
    scan_kernel<<<1, 256, 0, st>>>(chunk_counts, nchunks, E, tile_rows, chunk_base, counts, offsets, tile_prefix,
                                   sched);
    scatter_kernel<<<nchunks, 256, 0, st>>>(idx, P, E, chunk_base, perm);
    timing_end(KK_GROUP, st);
    count_launch();
    count_launch();
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_gather_rows(const __nv_bfloat16* src, const int32_t* perm, const int32_t* nrows, int k,
                               int64_t P, int H, __nv_bfloat16* dst, cudaStream_t st) {
    if (P == 0) return cudaSuccess;
    timing_begin(KK_GATHER, st);
    gather_rows_kernel<<<capped_grid((P * 32 + 255) / 256), 256, 0, st>>>(src, perm, nrows, k, P, H, dst);
    timing_end(KK_GATHER, st);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_combine(const __nv_bfloat16* slots, const int32_t* idx, int E, int k, int64_t T, int H,
                           __nv_bfloat16* y, cudaStream_t st) {
    const int64_t n = T * (H / 8);
    if (n == 0) return cudaSuccess;
    timing_begin(KK_COMBINE, st);
    combine_kernel<<<capped_grid((n + 255) / 256), 256, 0, st>>>(slots, idx, E, k, T, H, y);
    timing_end(KK_COMBINE, st);
    count_launch();
    return cudaGetLastError();
}

}  // namespace e4b
