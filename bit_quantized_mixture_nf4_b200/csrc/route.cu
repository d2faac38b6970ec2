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

// Programmatic dependent launch: the grouping chain (route, histogram, scan,
// scatter, gather) is launched with programmatic stream serialization, so a
// kernel's blocks are resident while its predecessor drains.  Every kernel of
// the chain waits for its predecessor's completion (and memory) before it reads
// anything the predecessor wrote; since each one waits before it can finish,
// completion is ordered along the whole chain.  A chained kernel's lifetime
// overlaps its predecessors', so what they write is not read-only for it: the
// chain reads through L2 (ld.global.cg), never through the non-coherent path.
__device__ __forceinline__ void chain_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void chain_release() { asm volatile("griddepcontrol.launch_dependents;"); }

constexpr int kMaxTopK = 8;   // the entry points reject top_k > 8

// One warp per token (the per-token routing is route_token_warp, shared with
// the small-batch kernels).
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, int64_t T, int E, int k,
                                                    int renorm, int32_t* __restrict__ idx,
                                                    float* __restrict__ wts) {
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    chain_release();
    chain_wait();
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
// chunk_counts is expert-major: [E][nchunks].
__global__ void __launch_bounds__(256) hist_kernel(const int32_t* __restrict__ idx, int64_t P, int E,
                                                   int32_t* __restrict__ chunk_counts) {
    __shared__ int cnt[256];
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    chain_release();
    chain_wait();
    __syncthreads();
    const int64_t p0 = (int64_t)blockIdx.x * kChunkPairs;
    for (int i = threadIdx.x; i < kChunkPairs; i += blockDim.x) {
        const int64_t pp = p0 + i;
        if (pp < P) {
            const int e = __ldcg(idx + pp);
            if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);   // out-of-range experts are dropped
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_counts[(int64_t)e * gridDim.x + blockIdx.x] = cnt[e];
}

__device__ __forceinline__ int warp_inclusive_scan(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

// Single block of 1024 threads: expert totals, exclusive scans over experts (rows
// and m-tiles), per-chunk bases and the m-tile schedule.  A warp owns experts
// warp, warp+32, ...; it walks an expert's chunk counts (contiguous, expert-major)
// 32 at a time with a running carry.
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* __restrict__ chunk_counts, int nchunks, int E,
                                                    int tile_rows, int32_t* __restrict__ chunk_base,
                                                    int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ tile_prefix, int4* __restrict__ sched) {
    __shared__ int s_tot[256], s_off[256], s_toff[256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    chain_release();
    chain_wait();
    for (int e = warp; e < E; e += nw) {
        const int32_t* c = chunk_counts + (int64_t)e * nchunks;
        int sum = 0;
        for (int i = lane; i < nchunks; i += 32) sum += __ldcg(c + i);
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0) s_tot[e] = sum;
    }
    __syncthreads();
    if (warp == 0) {   // exclusive scans of the row counts and m-tile counts over experts
        int run = 0, trun = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int v = e < E ? s_tot[e] : 0;
            const int tv = (v + tile_rows - 1) / tile_rows;
            const int x = warp_inclusive_scan(v, lane), tx = warp_inclusive_scan(tv, lane);
            if (e < E) {
                s_off[e] = run + x - v;
                s_toff[e] = trun + tx - tv;
            }
            run += __shfl_sync(0xffffffffu, x, 31);
            trun += __shfl_sync(0xffffffffu, tx, 31);
        }
        if (lane == 0) {
            offsets[E] = run;
            tile_prefix[E] = trun;
        }
    }
    __syncthreads();
    for (int e = warp; e < E; e += nw) {
        const int32_t* c = chunk_counts + (int64_t)e * nchunks;
        int32_t* b = chunk_base + (int64_t)e * nchunks;
        const int tot = s_tot[e], off = s_off[e], toff = s_toff[e];
        int run = off;
        for (int i0 = 0; i0 < nchunks; i0 += 32) {
            const int i = i0 + lane;
            const int v = i < nchunks ? __ldcg(c + i) : 0;
            const int x = warp_inclusive_scan(v, lane);
            if (i < nchunks) b[i] = run + x - v;
            run += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0) {
            counts[e] = tot;
            offsets[e] = off;
            tile_prefix[e] = toff;
        }
        // m-tile schedule: (expert, first row, rows) of every m-tile, experts ascending
        const int nt = (tot + tile_rows - 1) / tile_rows;
        for (int m = lane; m < nt; m += 32)
            sched[toff + m] = make_int4(e, off + m * tile_rows, min(tile_rows, tot - m * tile_rows), 0);
    }
}

// Stable scatter: pairs of a chunk keep their order inside each expert.  Also the
// inverse map pair -> grouped row (-1 for pairs of out-of-range experts).
__global__ void __launch_bounds__(256) scatter_kernel(const int32_t* __restrict__ idx, int64_t P, int E,
                                                      const int32_t* __restrict__ chunk_base,
                                                      int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm) {
    constexpr int WARPS = 8, PER_WARP = kChunkPairs / WARPS;
    __shared__ int wbase[WARPS][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < WARPS * 256; i += blockDim.x) (&wbase[0][0])[i] = 0;
    chain_release();
    chain_wait();
    __syncthreads();
    const int64_t p0 = (int64_t)blockIdx.x * kChunkPairs + warp * PER_WARP;
    for (int it = 0; it < PER_WARP; it += 32) {
        const int64_t pp = p0 + it + lane;
        if (pp < P) {
            const int e = __ldcg(idx + pp);
            if (e >= 0 && e < E) atomicAdd(&wbase[warp][e], 1);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = __ldcg(chunk_base + (int64_t)e * gridDim.x + blockIdx.x);
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
        int e = (pp < P) ? __ldcg(idx + pp) : -1;
        if (e >= E) e = -1;
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & lt_mask);
        const int base = (e >= 0) ? wbase[warp][e] : 0;
        __syncwarp();
        if (e >= 0) {
            perm[base + rank] = (int32_t)pp;
            inv_perm[pp] = base + rank;
            if (rank == 0) wbase[warp][e] = base + __popc(peers);
        } else if (pp < P) {
            inv_perm[pp] = -1;
        }
        __syncwarp();
    }
}

// dst[r] = src[perm[r] / k]: one warp per row, 16-byte vectors, four loads in
// flight per lane before the stores.
__global__ void __launch_bounds__(256) gather_rows_kernel(const __nv_bfloat16* __restrict__ src,
                                                          const int32_t* __restrict__ perm,
                                                          const int32_t* __restrict__ nrows, int k, int64_t P,
                                                          int H, __nv_bfloat16* __restrict__ dst,
                                                          uint32_t* __restrict__ status) {
    const int lane = threadIdx.x & 31;
    chain_release();
    chain_wait();
    const int64_t n = min(P, (int64_t)__ldcg(nrows));   // rows that belong to a valid expert
    const int64_t wstride = (int64_t)gridDim.x * blockDim.x / 32;
    const int vec = H / 8;
    for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; r < n; r += wstride) {
        const int64_t pid = __ldcg(perm + r);
#if E4B_DEBUG_CHECKS
        if (pid < 0 || pid >= P) {
            if (lane == 0) debug_fail(status, kSiteGatherPerm);
            continue;
        }
#endif
        const int64_t t = pid / k;
        const uint4* s = reinterpret_cast<const uint4*>(src + t * H);
        uint4* d = reinterpret_cast<uint4*>(dst + r * H);
#pragma unroll 1
        for (int i0 = lane; i0 < vec; i0 += 128) {
            uint4 v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (i0 + 32 * q < vec) v[q] = __ldcg(s + i0 + 32 * q);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (i0 + 32 * q < vec) d[i0 + 32 * q] = v[q];
        }
    }
}

// y[t] = bf16( sum_j fp32(rows[inv_perm[t*k + j]]) ), j ascending: the weighted
// combine of the k expert outputs of each token in fp32 (experts4bit-qlora 0.1.0
// experts.py, Experts4bit.forward: per-expert outputs in the compute dtype,
// index_add_ into an fp32 buffer).  Pairs of out-of-range experts (inv_perm -1)
// are skipped.
__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16* __restrict__ rows,
                                                      const int32_t* __restrict__ inv_perm, int k, int64_t T,
                                                      int H, __nv_bfloat16* __restrict__ y,
                                                      uint32_t* __restrict__ status) {
    const int h8 = H / 8;
    const int64_t n = T * h8;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const int64_t t = i / h8;
        const int c = (int)(i - t * h8);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        uint4 v[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {   // every slot's vector in flight before the sums
            v[j] = make_uint4(0u, 0u, 0u, 0u);
            if (j < k) {
                const int r = __ldg(inv_perm + t * k + j);
#if E4B_DEBUG_CHECKS
                if (r < -1 || r >= T * k) {
                    debug_fail(status, kSiteCombineInv);
                    continue;
                }
#endif
                if (r >= 0) v[j] = __ldcs(reinterpret_cast<const uint4*>(rows + (int64_t)r * H) + c);
            }
        }
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            if (j >= k) break;
            const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
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

// Consistency checks of a grouping schedule (the output of the three grouping
// kernels): expert offsets and counts, the m-tile total and entries, and perm /
// inv_perm as inverse maps that respect the experts.  A violated property records
// its site in the status word (debug_fail).  Every value read from the schedule is
// range-checked before it is used as an index, so a corrupt schedule is reported,
// never followed.
__global__ void __launch_bounds__(256) validate_schedule_kernel(const int32_t* __restrict__ idx, int64_t P, int E,
                                                                int tile_rows, const int32_t* __restrict__ counts,
                                                                const int32_t* __restrict__ offsets,
                                                                const int32_t* __restrict__ tile_prefix,
                                                                const int4* __restrict__ sched, int64_t n_sched,
                                                                const int32_t* __restrict__ perm,
                                                                const int32_t* __restrict__ inv_perm,
                                                                uint32_t* __restrict__ status) {
    __shared__ unsigned long long s_tiles;
    if (blockIdx.x == 0) {   // per-expert properties
        if (threadIdx.x == 0) {
            s_tiles = 0ull;
            if (offsets[0] != 0) debug_fail(status, kSiteOffsets);
        }
        __syncthreads();
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            const int64_t a = offsets[e], b = offsets[e + 1];
            if (b < a || b > P) debug_fail(status, kSiteOffsets);
            if (counts[e] != b - a) debug_fail(status, kSiteCounts);
            if (b > a) atomicAdd(&s_tiles, (unsigned long long)((b - a + tile_rows - 1) / tile_rows));
        }
        __syncthreads();
        if (threadIdx.x == 0 && (int64_t)s_tiles != (int64_t)tile_prefix[E]) debug_fail(status, kSiteTilePrefix);
    }
    const int64_t n = min(max((int64_t)offsets[E], (int64_t)0), P);   // grouped rows
    int64_t nt = tile_prefix[E];
    if (nt < 0 || nt > n_sched) {
        if (blockIdx.x == 0 && threadIdx.x == 0) debug_fail(status, kSiteTilePrefix);
        nt = nt < 0 ? 0 : n_sched;
    }
    const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x, stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t m = i0; m < nt; m += stride) {   // m-tile entries
        const int4 v = sched[m];
        if (v.x < 0 || v.x >= E) {
            debug_fail(status, kSiteSchedule);
            continue;
        }
        const int64_t a = offsets[v.x], b = offsets[v.x + 1];
        if (v.y < a || v.z < 1 || v.z > tile_rows || (int64_t)v.y + v.z > b || (v.y - a) % tile_rows != 0)
            debug_fail(status, kSiteSchedule);
    }
    for (int64_t r = i0; r < n; r += stride) {   // grouped row -> pair of the row's expert
        const int64_t pid = perm[r];
        if (pid < 0 || pid >= P) {
            debug_fail(status, kSitePerm);
            continue;
        }
        const int e = idx[pid];
        if (e < 0 || e >= E || r < offsets[e] || r >= offsets[e + 1]) debug_fail(status, kSitePerm);
        if (inv_perm[pid] != r) debug_fail(status, kSiteInvPerm);
    }
    for (int64_t pid = i0; pid < P; pid += stride) {   // pair -> its grouped row, -1 for a dropped pair
        const int64_t r = inv_perm[pid];
        const int e = idx[pid];
        if (e >= 0 && e < E) {
            if (r < 0 || r >= n || perm[r] != pid) debug_fail(status, kSiteInvPerm);
        } else if (r != -1) {
            debug_fail(status, kSiteInvPerm);
        }
    }
}

static int capped_grid(int64_t blocks) {
    return (int)std::max<int64_t>(1, std::min<int64_t>(blocks, (int64_t)num_sms() * 16));
}

// Launch with programmatic stream serialization (the kernel calls chain_wait
// before it reads its predecessors' output).
template <typename... KArgs, typename... Args>
static cudaError_t launch_chained(void (*kernel)(KArgs...), unsigned grid, unsigned block, cudaStream_t st,
                                  Args... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

cudaError_t launch_route(const float* logits, int64_t T, int E, int k, int renorm, int32_t* idx, float* w,
                         cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int64_t blocks = (T * 32 + 255) / 256;
    timing_begin(KK_ROUTE, st);
    const cudaError_t err = launch_chained(route_kernel, (unsigned)blocks, 256, st, logits, T, E, k, renorm, idx, w);
    timing_end(KK_ROUTE, st);
    count_launch();
    return err;
}

cudaError_t launch_group(const int32_t* idx, int64_t P, int E, int tile_rows, int32_t* chunk_counts,
                         int32_t* chunk_base, int32_t* counts, int32_t* offsets, int32_t* tile_prefix,
                         int4* sched, int32_t* perm, int32_t* inv_perm, cudaStream_t st) {
    const int nchunks = (int)((P + kChunkPairs - 1) / kChunkPairs);
    if (nchunks == 0) return cudaSuccess;
    timing_begin(KK_GROUP, st);
    cudaError_t err = launch_chained(hist_kernel, nchunks, 256, st, idx, P, E, chunk_counts);
    if (err == cudaSuccess)
        err = launch_chained(scan_kernel, 1, 1024, st, chunk_counts, nchunks, E, tile_rows, chunk_base, counts, offsets,
                             tile_prefix, sched);
    if (err == cudaSuccess)
        err = launch_chained(scatter_kernel, nchunks, 256, st, idx, P, E, chunk_base, perm, inv_perm);
    timing_end(KK_GROUP, st);
    count_launch();
    count_launch();
    count_launch();
    return err;
}

cudaError_t launch_gather_rows(const __nv_bfloat16* src, const int32_t* perm, const int32_t* nrows, int k,
                               int64_t P, int H, __nv_bfloat16* dst, cudaStream_t st) {
    if (P == 0) return cudaSuccess;
    timing_begin(KK_GATHER, st);
    const cudaError_t err =
        launch_chained(gather_rows_kernel, capped_grid((P * 32 + 255) / 256), 256, st, src, perm, nrows, k, P, H, dst,
                       device_status_ptr());
    timing_end(KK_GATHER, st);
    count_launch();
    return err;
}

cudaError_t launch_combine(const __nv_bfloat16* rows, const int32_t* inv_perm, int k, int64_t T, int H,
                           __nv_bfloat16* y, cudaStream_t st) {
    const int64_t n = T * (H / 8);
    if (n == 0) return cudaSuccess;
    timing_begin(KK_COMBINE, st);
    combine_kernel<<<capped_grid((n + 255) / 256), 256, 0, st>>>(rows, inv_perm, k, T, H, y, device_status_ptr());
    timing_end(KK_COMBINE, st);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_validate_schedule(const int32_t* idx, int64_t P, int E, int tile_rows, const int32_t* counts,
                                     const int32_t* offsets, const int32_t* tile_prefix, const int4* sched,
                                     int64_t n_sched, const int32_t* perm, const int32_t* inv_perm, cudaStream_t st) {
    uint32_t* status = device_status_ptr();
    if (!status) return cudaErrorUnknown;
    const int grid = capped_grid((std::max<int64_t>(std::max<int64_t>(P, n_sched), E) + 255) / 256);
    validate_schedule_kernel<<<grid, 256, 0, st>>>(idx, P, E, tile_rows, counts, offsets, tile_prefix, sched, n_sched,
                                                   perm, inv_perm, status);
    count_launch();
    return cudaGetLastError();
}

}  // namespace e4b
