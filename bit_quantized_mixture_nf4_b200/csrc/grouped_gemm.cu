// Grouped expert GEMMs with in-kernel 4-bit dequantization on the 5th-generation
// tensor cores (tcgen05, TMEM accumulators), sm_100a.
//
// One persistent kernel template serves the four contractions of the expert
// layer (expert-layer pages: "experts4bit-qlora 0.1.0" experts.py,
// Experts4bit.forward; bitsandbytes PR #1965, "What this adds": recompute-in-
// backward input gradient).  Rows are routed (token, slot) pairs in grouped
// order, so expert e owns the contiguous rows [offsets[e], offsets[e+1]).
//
//   EPI_GATEUP        D = X_e W_gu,e^T ; epilogue h = silu(g)*u (+ saves g,u)
//   EPI_DOWN          D = h_e W_d,e^T  ; epilogue y32[token] += w * D (atomic fp32)
//   EPI_DGRAD_DOWN    D = dY_e W_d,e   ; epilogue dh = w*D, dG/dU (SwiGLU backward)
//   EPI_DGRAD_GATEUP  D = dGU_e W_gu,e ; epilogue gx32[token] += D (atomic fp32)
//
// Tile: 128 rows x 256 columns x 64-deep k-stages, 4-stage smem ring.
//   warp 4      TMA producer: A tile (bf16, 128B swizzle) + packed 4-bit weight tile
//   warps 8-15  dequantize the packed tile into a bf16 operand tile in smem, in the
//               tensor cores' 128B-swizzled layout: K-major for the forward (weights
//               stored [N, K]) and MN-major for the input gradient (weights used
//               transposed, stored [K, N]); the transposition costs nothing
//   warp 5      one thread issues tcgen05.mma (M=128, N=256, K=16) into TMEM
//   warps 0-3   epilogue: tcgen05.ld from TMEM (double-buffered accumulator, 2x256
//               columns) and the fused elementwise/scatter work
// Every wait is bounded; on expiry the kernel records a timeout and exits.
#include "e4b_internal.h"

namespace e4b {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_STAGE_BYTES = BM * BK * 2;       // 16 KB
constexpr int B_STAGE_BYTES = BN * BK * 2;       // 32 KB
constexpr int RAW_STAGE_BYTES = BN * BK / 2;     //  8 KB
constexpr int GEMM_THREADS = 512;
constexpr int PRODUCER_WARP = 4, MMA_WARP = 5, DEQ_WARP0 = 8;
constexpr int TMEM_COLS = 2 * BN;                // two accumulator buffers
constexpr int SMEM_DATA = STAGES * (A_STAGE_BYTES + B_STAGE_BYTES + RAW_STAGE_BYTES);
constexpr int GEMM_SMEM_BYTES = SMEM_DATA + 1024 /*alignment slack*/ + 256 /*barriers*/;

struct SmemCtl {
    uint64_t full_tma[STAGES];
    uint64_t full_b[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(SmemCtl) <= 256, "control block");

struct TileInfo {
    int e, row0, rows, nt;
};

__device__ __forceinline__ TileInfo decode_tile(const GemmParams& p, int tile) {
    const int mt = tile / p.n_tiles;
    TileInfo ti;
    ti.nt = tile - mt * p.n_tiles;
    int lo = 0, hi = p.E;   // tile_prefix[lo] <= mt < tile_prefix[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(p.tile_prefix + mid) <= mt) lo = mid; else hi = mid;
    }
    ti.e = lo;
    ti.row0 = __ldg(p.offsets + lo) + (mt - __ldg(p.tile_prefix + lo)) * BM;
    ti.rows = min(BM, __ldg(p.offsets + lo + 1) - ti.row0);
    return ti;
}

// Stored weight row (within one expert) that feeds operand row n (K-major mode).
template <int EPI>
__device__ __forceinline__ int kmajor_row(const GemmParams& p, const TileInfo& ti, int n) {
    if (EPI == EPI_GATEUP)   // 128 gate rows, then the matching 128 up rows
        return (n < 128) ? ti.nt * 128 + n : p.up_offset + ti.nt * 128 + (n - 128);
    return ti.nt * BN + n;
}

// absmax feeding this dequant thread's 64-element block for k-stage ks.
template <int EPI>
__device__ __forceinline__ float load_absmax(const GemmParams& p, const TileInfo& ti, int ks, int t) {
    int64_t row;
    int blk;
    if (EPI == EPI_GATEUP || EPI == EPI_DOWN) {         // blocks run along K
        row = (int64_t)ti.e * p.b_rows_per_expert + kmajor_row<EPI>(p, ti, t);
        blk = ks;
    } else {                                           // blocks run along N
        row = (int64_t)ti.e * p.b_rows_per_expert + (int64_t)ks * BK + (t >> 2);
        blk = ti.nt * (BN / 64) + (t & 3);
        if (blk >= p.b_blocks_per_row) return 0.0f;
    }
    if (row >= p.b_rows_total) return 0.0f;
    return __ldg(p.absmax + row * p.b_blocks_per_row + blk);
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

template <int EPI, int CB>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_raw,
                    const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_STAGE_BYTES;
    uint8_t* sRaw = sB + STAGES * B_STAGE_BYTES;
    SmemCtl* ctl = reinterpret_cast<SmemCtl*>(sRaw + STAGES * RAW_STAGE_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool kMajorB = (EPI == EPI_GATEUP || EPI == EPI_DOWN);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&ctl->full_tma[s]), 1);
            mbar_init(smem_u32(&ctl->full_b[s]), 8);      // one arrival per dequant warp
            mbar_init(smem_u32(&ctl->empty[s]), 1);       // tcgen05.commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&ctl->acc_full[b]), 1);
            mbar_init(smem_u32(&ctl->acc_empty[b]), 4);   // one arrival per epilogue warp
        }
        ctl->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == PRODUCER_WARP && lane == 0) {
        tma_prefetch_desc(&tmap_a);
        tma_prefetch_desc(&tmap_raw);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    volatile int* abort_flag = &ctl->abort_flag;

    const int total_tiles = __ldg(p.tile_prefix + p.E) * p.n_tiles;
    const int nk = p.K / BK;

    if (warp == PRODUCER_WARP) {
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile(p, tile);
                for (int ks = 0; ks < nk; ++ks, ++it) {
                    const int s = it % STAGES;
                    const uint32_t r = it / STAGES;
                    if (!mbar_wait(smem_u32(&ctl->empty[s]), (r & 1) ^ 1, abort_flag, p.status)) { ok = false; break; }
                    const uint32_t fb = smem_u32(&ctl->full_tma[s]);
                    mbar_arrive_expect_tx(fb, A_STAGE_BYTES + RAW_STAGE_BYTES);
                    tma_load_2d(smem_u32(sA + s * A_STAGE_BYTES), &tmap_a, fb, ks * BK, ti.row0);
                    const uint32_t raw = smem_u32(sRaw + s * RAW_STAGE_BYTES);
                    if (kMajorB) {
                        const int y0 = ti.e * p.b_rows_per_expert + kmajor_row<EPI>(p, ti, 0);
                        const int y1 = ti.e * p.b_rows_per_expert + kmajor_row<EPI>(p, ti, 128);
                        tma_load_2d(raw, &tmap_raw, fb, ks * (BK / 2), y0);
                        tma_load_2d(raw + RAW_STAGE_BYTES / 2, &tmap_raw, fb, ks * (BK / 2), y1);
                    } else {
                        tma_load_2d(raw, &tmap_raw, fb, ti.nt * (BN / 2), ti.e * p.b_rows_per_expert + ks * BK);
                    }
                }
            }
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(BM, BN, kMajorB ? 0 : 1);
            uint32_t it = 0, lt = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++lt) {
                const uint32_t ab = lt & 1, ar = lt >> 1;
                if (!mbar_wait(smem_u32(&ctl->acc_empty[ab]), (ar & 1) ^ 1, abort_flag, p.status)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + ab * BN;
                for (int ks = 0; ks < nk; ++ks, ++it) {
                    const int s = it % STAGES;
                    const uint32_t r = it / STAGES;
                    if (!mbar_wait(smem_u32(&ctl->full_tma[s]), r & 1, abort_flag, p.status) ||
                        !mbar_wait(smem_u32(&ctl->full_b[s]), r & 1, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sA + s * A_STAGE_BYTES);
                    const uint32_t b_addr = smem_u32(sB + s * B_STAGE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
                        const uint64_t bdesc = kMajorB ? smem_desc_sw128(b_addr + kk * 32, 16, 1024)
                                                       : smem_desc_sw128(b_addr + kk * 2048, 8192, 1024);
                        mma_bf16_ss(d_tmem, adesc, bdesc, idesc, (ks | kk) != 0);
                    }
                    mma_commit(smem_u32(&ctl->empty[s]));
                }
                if (ok) mma_commit(smem_u32(&ctl->acc_full[ab]));
            }
        }
    } else if (warp >= DEQ_WARP0) {
        const int t = threadIdx.x - DEQ_WARP0 * 32;   // 0..255
        uint32_t it = 0;
        int tile = blockIdx.x, ks = 0;
        TileInfo ti{};
        float a_next = 0.0f;
        if (tile < total_tiles) {
            ti = decode_tile(p, tile);
            a_next = load_absmax<EPI>(p, ti, 0, t);
        }
        while (tile < total_tiles) {
            const float a_cur = a_next;
            const int s = it % STAGES;
            const uint32_t r = it / STAGES;
            // prefetch the next stage's absmax before waiting on this one
            if (++ks == nk) {
                ks = 0;
                tile += gridDim.x;
                if (tile < total_tiles) ti = decode_tile(p, tile);
            }
            if (tile < total_tiles) a_next = load_absmax<EPI>(p, ti, ks, t);

            if (!mbar_wait(smem_u32(&ctl->full_tma[s]), r & 1, abort_flag, p.status)) break;
            const uint8_t* raw = sRaw + s * RAW_STAGE_BYTES + (kMajorB ? t * 32 : (t >> 2) * 128 + (t & 3) * 32);
            const uint4 p0 = *reinterpret_cast<const uint4*>(raw);
            const uint4 p1 = *reinterpret_cast<const uint4*>(raw + 16);
            const BlockTable tb = make_table<CB>(a_cur);
            uint8_t* dst_tile = sB + s * B_STAGE_BYTES;
            const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t o[4];
                decode_word(tb, words[c], o);
                const uint32_t off = kMajorB ? sw128_offset(t, c) : (t & 3) * 8192 + sw128_offset(t >> 2, c);
                *reinterpret_cast<uint4*>(dst_tile + off) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl->full_b[s]));
            ++it;
        }
    } else if (warp < 4) {
        // ------------------------------------------------------------ epilogue
        const int rloc = warp * 32 + lane;   // TMEM lane == tile row
        uint32_t lt = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++lt) {
            const TileInfo ti = decode_tile(p, tile);
            const uint32_t ab = lt & 1, ar = lt >> 1;
            if (!mbar_wait(smem_u32(&ctl->acc_full[ab]), ar & 1, abort_flag, p.status)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(warp * 32) << 16) + ab * BN;
            const bool valid = rloc < ti.rows;
            const int row = ti.row0 + rloc;
            if (EPI == EPI_GATEUP) {
                const int I = p.up_offset;
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    float g[32], u[32];
                    tmem_load32(tbase + 32 * q, g);
                    tmem_load32(tbase + 128 + 32 * q, u);
                    const int f0 = ti.nt * 128 + 32 * q;
                    if (valid && f0 < I) {
                        uint32_t hv[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            hv[i] = pack_bf16x2(silu_f(g[2 * i]) * u[2 * i], silu_f(g[2 * i + 1]) * u[2 * i + 1]);
                        uint4* dst = reinterpret_cast<uint4*>(p.out_bf16 + (int64_t)row * p.ld_out + f0);
#pragma unroll
                        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
                        if (p.gu) {
                            uint4* dg = reinterpret_cast<uint4*>(p.gu + (int64_t)row * 2 * I + f0);
                            uint4* du = reinterpret_cast<uint4*>(p.gu + (int64_t)row * 2 * I + I + f0);
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                dg[i] = make_uint4(pack_bf16x2(g[8 * i], g[8 * i + 1]), pack_bf16x2(g[8 * i + 2], g[8 * i + 3]),
                                                   pack_bf16x2(g[8 * i + 4], g[8 * i + 5]), pack_bf16x2(g[8 * i + 6], g[8 * i + 7]));
                                du[i] = make_uint4(pack_bf16x2(u[8 * i], u[8 * i + 1]), pack_bf16x2(u[8 * i + 2], u[8 * i + 3]),
                                                   pack_bf16x2(u[8 * i + 4], u[8 * i + 5]), pack_bf16x2(u[8 * i + 6], u[8 * i + 7]));
                            }
                        }
                    }
                }
            } else {
                int pair = 0;
                float wgt = 1.0f;
                if (valid) {
                    pair = __ldg(p.perm + row);
                    if (EPI != EPI_DGRAD_GATEUP) wgt = __ldg(p.topk_w + pair);
                }
                const int tok = pair / p.k_top;
#pragma unroll 1
                for (int q = 0; q < BN / 32; ++q) {
                    float v[32];
                    tmem_load32(tbase + 32 * q, v);
                    const int c0 = ti.nt * BN + 32 * q;
                    if (!valid || c0 >= p.N) continue;
                    if (EPI == EPI_DOWN || EPI == EPI_DGRAD_GATEUP) {
                        float4* dst = reinterpret_cast<float4*>(p.out_f32 + (int64_t)tok * p.ld_out + c0);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            atomicAdd(dst + i, make_float4(v[4 * i] * wgt, v[4 * i + 1] * wgt, v[4 * i + 2] * wgt, v[4 * i + 3] * wgt));
                    } else {   // EPI_DGRAD_DOWN: SwiGLU backward with the saved pre-activations
                        const int I = p.N;
                        const uint4* gsrc = reinterpret_cast<const uint4*>(p.gu + (int64_t)row * 2 * I + c0);
                        const uint4* usrc = reinterpret_cast<const uint4*>(p.gu + (int64_t)row * 2 * I + I + c0);
                        uint4* dgo = reinterpret_cast<uint4*>(p.out_bf16 + (int64_t)row * 2 * I + c0);
                        uint4* duo = reinterpret_cast<uint4*>(p.out_bf16 + (int64_t)row * 2 * I + I + c0);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint4 gq = __ldg(gsrc + i), uq = __ldg(usrc + i);
                            const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w}, uw[4] = {uq.x, uq.y, uq.z, uq.w};
                            uint32_t dgw[4], duw[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                float dG[2], dU[2];
#pragma unroll
                                for (int h = 0; h < 2; ++h) {
                                    const float gg = __uint_as_float(h ? (gw[j] & 0xFFFF0000u) : (gw[j] << 16));
                                    const float uu = __uint_as_float(h ? (uw[j] & 0xFFFF0000u) : (uw[j] << 16));
                                    const float dh = v[8 * i + 2 * j + h] * wgt;
                                    const float sg = 1.0f / (1.0f + __expf(-gg));
                                    dG[h] = dh * uu * sg * (1.0f + gg * (1.0f - sg));
                                    dU[h] = dh * gg * sg;
                                }
                                dgw[j] = pack_bf16x2(dG[0], dG[1]);
                                duw[j] = pack_bf16x2(dU[0], dU[1]);
                            }
                            dgo[i] = make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]);
                            duo[i] = make_uint4(duw[0], duw[1], duw[2], duw[3]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl->acc_empty[ab]));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

static bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                        uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, int CB>
static cudaError_t launch_one(const CUtensorMap& ma, const CUtensorMap& mr, const GemmParams& p, int grid,
                              cudaStream_t st) {
    auto kern = grouped_gemm_kernel<EPI, CB>;
    static bool attr_set = false;   // per instantiation
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM_SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    timing_begin(KK_GEMM_GATEUP + EPI, st);
    kern<<<grid, GEMM_THREADS, GEMM_SMEM_BYTES, st>>>(ma, mr, p);
    timing_end(KK_GEMM_GATEUP + EPI, st);
    count_launch();
    return cudaGetLastError();
}

int gemm_tile_rows() { return BM; }

cudaError_t launch_grouped_gemm(int epi, int codebook, const void* a, int64_t a_rows, const uint8_t* packed,
                                int64_t packed_rows_total, int packed_row_bytes, GemmParams p, int max_m_tiles,
                                cudaStream_t st) {
    CUtensorMap ma, mr;
    if (!make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a, (uint64_t)p.K, (uint64_t)a_rows, (uint64_t)p.K * 2, 64,
                     BM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const bool kmaj = (epi == EPI_GATEUP || epi == EPI_DOWN);
    if (!make_map_2d(&mr, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)packed_row_bytes,
                     (uint64_t)packed_rows_total, (uint64_t)packed_row_bytes, kmaj ? BK / 2 : BN / 2,
                     kmaj ? 128 : BK, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const int64_t tiles = (int64_t)max_m_tiles * p.n_tiles;
    const int grid = (int)std::min<int64_t>(tiles, num_sms());
    if (grid <= 0) return cudaSuccess;
#define E4B_LAUNCH(E_, C_) return launch_one<E_, C_>(ma, mr, p, grid, st)
    if (codebook == 0) {
        switch (epi) {
            case EPI_GATEUP: E4B_LAUNCH(EPI_GATEUP, 0);
            case EPI_DOWN: E4B_LAUNCH(EPI_DOWN, 0);
            case EPI_DGRAD_DOWN: E4B_LAUNCH(EPI_DGRAD_DOWN, 0);
            default: E4B_LAUNCH(EPI_DGRAD_GATEUP, 0);
        }
    } else {
        switch (epi) {
            case EPI_GATEUP: E4B_LAUNCH(EPI_GATEUP, 1);
            case EPI_DOWN: E4B_LAUNCH(EPI_DOWN, 1);
            case EPI_DGRAD_DOWN: E4B_LAUNCH(EPI_DGRAD_DOWN, 1);
            default: E4B_LAUNCH(EPI_DGRAD_GATEUP, 1);
        }
    }
#undef E4B_LAUNCH
}

}  // namespace e4b
