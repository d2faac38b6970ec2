// Grouped expert GEMMs with in-kernel 4-bit dequantization on the 5th-generation
// tensor cores (tcgen05, TMEM accumulators), sm_100a.
//
// One persistent kernel template serves the four contractions of the expert
// layer (expert-layer pages: "experts4bit-qlora 0.1.0" experts.py,
// Experts4bit.forward; bitsandbytes PR #1965, "What this adds": recompute-in-
// backward input gradient).  Rows are routed (token, slot) pairs in grouped
// order, so expert e owns the contiguous rows [offsets[e], offsets[e+1]).
//
//   EPI_GATEUP        D = X_e W_gu,e^T ; epilogue h = silu(g)*u (+ saves dh/dg, dh/du)
//   EPI_DOWN          D = h_e W_d,e^T  ; epilogue out[row] = bf16(w * D)
//   EPI_DGRAD_DOWN    D = dY_e W_d,e   ; epilogue dh = w*D, dG = dh*dh/dg, dU = dh*dh/du, and
//                                        optionally the per-tile dot products <D, h> of the
//                                        routing-weight gradient
//   EPI_DGRAD_GATEUP  D = dGU_e W_gu,e ; epilogue out[row] = bf16(D)
// Every output row is the grouped row itself (a contiguous slab per tile); the
// k rows of a token are found through the inverse permutation and summed in
// fp32, in slot order, by combine_kernel.
//
// Tile: (128*CTAS) rows x 256 columns, 64-deep k-stages.  With CTAS = 2 a
// cluster of two CTAs on two SMs computes one 256-row tile with
// tcgen05.mma.cta_group::2 (M = 256): each CTA holds 128 rows of A and HALF of
// the dequantized B tile, so each SM dequantizes only 128 x 64 weights per
// 512-clock stage and the B operand is read from shared memory once for both.
// Roles per CTA (512 threads):
//   warp 4      TMA producer of the A tile (bf16, 128B swizzle), 6-stage ring
//   warp 6      producer of the packed 4-bit B tile (TMA) and its absmax values
//               (cp.async), 8-stage ring, prefetched far ahead
//   warps 8, 10, 11, 12, 14, 15   dequantization, 3 groups of 2 warps taking every
//               third k-stage (none of them shares a scheduler with the MMA
//               thread): each thread turns 64-element blocks (one absmax each) of
//               packed codes into bf16 in the tensor cores' 128B-swizzled layout --
//               K-major for the forward (weights stored [N, K]), MN-major for the
//               input gradient (weights used transposed, stored [K, N]; the
//               transposition costs nothing); 4-stage ring of dequantized tiles
//   warp 5      one thread of the first CTA issues the MMAs into TMEM
//               (double-buffered accumulator, 2 x 256 columns)
//   warps 0-3   epilogue: tcgen05.ld of this CTA's 128 accumulator rows; a warp's
//               32 x 32 output chunks go through shared memory (64B-swizzled)
//               and leave with TMA tensor stores, so the epilogue issues no
//               per-thread global stores that would compete with the
//               dequantizing warps for the load/store pipeline
//   warps 7, 9, 13 idle
// Every mbarrier wait is bounded; on expiry the kernel records a timeout and exits.
#include <mutex>

#include "e4b_internal.h"

namespace e4b {

constexpr int BN = 256, BK = 64;
constexpr int GEMM_THREADS = 512;
constexpr int PRODUCER_WARP = 4, MMA_WARP = 5, RAW_WARP = 6, DEQ_WARP0 = 8;
constexpr int TMEM_COLS = 2 * BN;   // two accumulator buffers

template <int CTAS, int EPI = 0>
struct Cfg {
    static constexpr int TILE_M = 128 * CTAS;            // rows per tile (all CTAs of the cluster)
    static constexpr int N_CTA = BN / CTAS;              // B columns dequantized by one CTA
    static constexpr int A_BYTES = 128 * BK * 2;         // this CTA's 128 A rows
    static constexpr int B_BYTES = N_CTA * BK * 2;
    static constexpr int RAW_BYTES = N_CTA * BK / 2;
    static constexpr int ASTAGES = (CTAS == 2) ? 6 : 4;    // A (activation) ring: TMA latency under load
    static constexpr int STAGES = (CTAS == 2) ? 4 : 3;     // dequantized-B ring
    // packed-weight ring, prefetched far ahead (the input gradient's down^T GEMM gives two
    // stages to the epilogue buffers that bring in the saved SwiGLU derivatives).  The
    // single-SM tiles (twice the B columns per SM) have room for 3: one per dequantizing
    // group, so each group reuses its own slot.
    static constexpr int RSTAGES = (CTAS == 2) ? (EPI == EPI_DGRAD_DOWN ? 6 : 8) : 3;
    static constexpr int AM_BYTES = N_CTA * 4;             // the stage's absmax values, one per block
    static constexpr int RAW_STAGE = RAW_BYTES + AM_BYTES;
    // dequantizing warps: 6 warps (none on the MMA thread's scheduler), 3 groups of 2
    // taking every third k-stage; a thread owns N_CTA / 64 blocks of 64 elements
    static constexpr int DEQ_GROUPS = 3, DEQ_GROUP_WARPS = 2;
    static constexpr int BLK_PER_THREAD = N_CTA / (32 * DEQ_GROUP_WARPS);
    // A group's next stage reuses a ring slot whose previous use is at most one barrier
    // phase old only if each ring has a slot per group: with fewer, a parity wait could
    // pass on a phase two behind while another group's stage is still in use.
    static_assert(STAGES >= DEQ_GROUPS && RSTAGES >= DEQ_GROUPS, "ring slots per dequantizing group");
    // epilogue staging: per epilogue warp three 32 x 32 bf16 buffers (2 KB each); four (two
    // pairs of saved-derivative chunks, loaded and stored in place) for the down^T GEMM
    static constexpr int STAGE_BUF = 2048, STAGE_BUFS = (EPI == EPI_DGRAD_DOWN) ? 4 : 3;
    static constexpr int STAGE_WARP = STAGE_BUF * STAGE_BUFS;
    static constexpr int RINGS_BYTES = ASTAGES * A_BYTES + STAGES * B_BYTES + RSTAGES * RAW_STAGE;
    static constexpr int SMEM_BYTES = RINGS_BYTES + 1024 + 4 * STAGE_WARP + 1024;
};
static_assert(Cfg<2, EPI_GATEUP>::RINGS_BYTES % 1024 == 0 && Cfg<2, EPI_DGRAD_DOWN>::RINGS_BYTES % 1024 == 0,
              "staging buffers stay 1024-byte aligned");
static_assert(Cfg<2, EPI_GATEUP>::SMEM_BYTES <= 232448 && Cfg<2, EPI_DGRAD_DOWN>::SMEM_BYTES <= 232448,
              "shared memory per block");
static_assert(Cfg<1, EPI_GATEUP>::RINGS_BYTES % 1024 == 0 && Cfg<1, EPI_DGRAD_DOWN>::RINGS_BYTES % 1024 == 0,
              "staging buffers stay 1024-byte aligned (single-SM tiles)");
static_assert(Cfg<1, EPI_GATEUP>::SMEM_BYTES <= 232448 && Cfg<1, EPI_DGRAD_DOWN>::SMEM_BYTES <= 232448,
              "shared memory per block (single-SM tiles)");

// TMA tensor store of a 32 x 32 bf16 box from shared memory, and its bulk-group
// bookkeeping (issued and awaited by one thread).
// The outputs stream through L2 once (the next kernel reads them from HBM at these
// sizes), so the stores carry an evict-first policy: they do not push out the weight
// columns and activation rows the neighbouring tiles are still reading.
constexpr bool kStoreEvictFirst = true;
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, uint32_t src, int x, int y) {
    if (kStoreEvictFirst) {
        asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;"
                     ::"l"(reinterpret_cast<uint64_t>(m)), "r"(src), "r"(x), "r"(y), "l"(l2_evict_first_policy())
                     : "memory");
    } else {
        asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                     ::"l"(reinterpret_cast<uint64_t>(m)), "r"(src), "r"(x), "r"(y)
                     : "memory");
    }
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

struct SmemCtl {
    uint64_t a_full[8];
    uint64_t b_full[8];
    uint64_t empty[8];        // dequantized-B stage consumed (MMA commit)
    uint64_t a_empty[8];      // A stage consumed (MMA commit)
    uint64_t raw_full[16];
    uint64_t raw_empty[16];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t ld_full[4][2];   // EPI_DGRAD_DOWN: saved-derivative chunk pair landed (per epilogue warp)
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(SmemCtl) <= 1024, "control block");

struct TileInfo {
    int e, row0, rows, nt;
};

// Tile order.  Tiles are numbered expert by expert.  Inside an expert, its n-tiles
// go in groups of kTileGroup; inside a group, the expert's m-tiles are the outer
// loop and the group's n-tiles the inner one.  The tiles that run at the same time
// on neighbouring clusters then share one group of weight columns (re-read from L2
// by every m-tile of the expert) and a few m-tiles of activation rows, instead of
// sweeping all of the expert's weights once per m-tile.  16 measured best on the
// Mixtral shape (HBM reads of the gate_up GEMM 4.3 -> 1.8 GB per launch; 8 re-reads
// the long activation rows of the K = 14336 and 28672 GEMMs); where an expert has
// at most 16 n-tiles this is the plain (m-tile, n-tile) order.
constexpr int kTileGroup = 16;

// Tile -> (m-tile entry of the grouping scan's schedule, n-tile); one schedule load.
// max_rows: the tile height.  Debug builds check the entry; a bad one becomes an
// empty tile of expert 0 (every role of the CTA decodes the same entry, so they all
// skip it alike).
__device__ __forceinline__ TileInfo decode_tile(const GemmParams& p, const int4* sched, int tile, int max_rows) {
    const int n = p.n_tiles;
    const int mt_tile = tile / n;   // m-tile that the plain (m, n) order would give: locates the expert
    int lo = 0, hi = p.E;           // the last expert whose first m-tile is at or before mt_tile
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(p.tile_prefix + mid) <= mt_tile) lo = mid;
        else hi = mid;
    }
    const int m0 = __ldg(p.tile_prefix + lo), me = __ldg(p.tile_prefix + lo + 1) - m0;
    const int l = tile - m0 * n;    // the tile's index inside its expert: [0, me * n)
    const int g = min(kTileGroup, n), full = n / g;
    int m, nt;
    if (l < full * g * me) {
        const int grp = l / (g * me), r = l - grp * g * me;
        m = r / g;
        nt = grp * g + (r - m * g);
    } else {                        // the last, narrower group
        const int gw = n - full * g, r = l - full * g * me;
        m = r / gw;
        nt = full * g + (r - m * gw);
    }
    const int4 v = __ldg(sched + m0 + m);
#if E4B_DEBUG_CHECKS
    if (v.x < 0 || v.x >= p.E || v.z < 1 || v.z > max_rows || v.y < 0 || (int64_t)v.y + v.z > p.a_rows) {
        debug_fail(p.status, kSiteGemmTile);
        return TileInfo{0, 0, 0, nt};
    }
#endif
    return TileInfo{v.x, v.y, v.z, nt};
}

// Stored weight row (within one expert) feeding B column `n` (0..255) of tile nt (K-major mode).
template <int EPI>
__device__ __forceinline__ int kmajor_row(const GemmParams& p, int nt, int n) {
    if (EPI == EPI_GATEUP)   // 128 gate rows, then the matching 128 up rows
        return (n < 128) ? nt * 128 + n : p.up_offset + nt * 128 + (n - 128);
    return nt * BN + n;
}

// Index into the absmax array of 64-element block b (0..N_CTA-1) of this CTA's B
// half at k-stage ks, or -1 outside the stored matrix.
//   K-major:  block b = B column (rank*N_CTA + b), k-block ks
//   MN-major: block b = (k-row b & 63, n-block b >> 6 of this CTA's half)
template <int EPI, int CTAS>
__device__ __forceinline__ int64_t absmax_index(const GemmParams& p, const TileInfo& ti, int ks, int b, int rank) {
    int64_t row;
    int blk;
    if (EPI == EPI_GATEUP || EPI == EPI_DOWN) {
        row = (int64_t)ti.e * p.b_rows_per_expert + kmajor_row<EPI>(p, ti.nt, rank * Cfg<CTAS>::N_CTA + b);
        blk = ks;
    } else {
        row = (int64_t)ti.e * p.b_rows_per_expert + (int64_t)ks * BK + (b & 63);
        blk = (ti.nt * BN + rank * Cfg<CTAS>::N_CTA) / 64 + (b >> 6);
        if (blk >= p.b_blocks_per_row) return -1;
    }
    if (row >= p.b_rows_total) return -1;
    return row * p.b_blocks_per_row + blk;
}

// MXFP4: byte offset, in p.mx_scales, of the 4 scale bytes the raw warp copies for
// block b at k-stage 0 (-1 outside the stack).  K-major: row b's bytes for 32-blocks
// 0..3 (k-stage ks reads bytes 2ks, 2ks+1 of the group starting at 4 (ks / 2));
// MN-major: k-row (b & 63)'s bytes for the 32-column groups 4 j .. 4 j + 3 of this
// CTA's columns, j = (b >> 6) / 2 (n-block b >> 6 takes bytes 2 ((b >> 6) & 1), +1).
template <int EPI, int CTAS>
__device__ __forceinline__ int64_t mx_offset(const GemmParams& p, const TileInfo& ti, int b, int rank) {
    if (absmax_index<EPI, CTAS>(p, ti, 0, b, rank) < 0) return -1;
    if (EPI == EPI_GATEUP || EPI == EPI_DOWN) {
        const int64_t row = (int64_t)ti.e * p.b_rows_per_expert + kmajor_row<EPI>(p, ti.nt, rank * Cfg<CTAS>::N_CTA + b);
        return row * p.mx_stride;
    }
    const int64_t row = (int64_t)ti.e * p.b_rows_per_expert + (b & 63);
    return row * p.mx_stride + (ti.nt * BN + rank * Cfg<CTAS>::N_CTA) / 32 + 4 * ((b >> 6) >> 1);
}

// This row's part of the routing-weight gradient over one 32-column chunk:
// acc += sum_j v[j] * h[row, c0 + j] (fp32, columns in order).
__device__ __forceinline__ void dw_dot_chunk(const GemmParams& p, int64_t row, int c0, const float (&v)[32],
                                             float& acc) {
    const uint4* hs = reinterpret_cast<const uint4*>(p.h_in + row * p.N + c0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 hv = __ldg(hs + i);
        const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc = fmaf(v[8 * i + 2 * j], __uint_as_float(hw[j] << 16), acc);
            acc = fmaf(v[8 * i + 2 * j + 1], __uint_as_float(hw[j] & 0xFFFF0000u), acc);
        }
    }
}

// XACT, the extended epilogue: EPI_GATEUP handles per-expert biases and the clamped
// GLU (p.bias, p.act); EPI_DGRAD_DOWN also takes the dot products of the
// routing-weight gradient (p.h_in, p.dw_part).  The plain instances carry none of
// that code.
template <int EPI, int CB, int CTAS, bool XACT = false>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_raw,
                    const __grid_constant__ CUtensorMap tmap_out, const __grid_constant__ CUtensorMap tmap_gu,
                    const __grid_constant__ CUtensorMap tmap_lora, const GemmParams p) {
    using C = Cfg<CTAS, EPI>;
    constexpr int STAGES = C::STAGES;
    constexpr int ASTAGES = C::ASTAGES;
    constexpr bool kMajorB = (EPI == EPI_GATEUP || EPI == EPI_DOWN);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + ASTAGES * C::A_BYTES;
    uint8_t* sRaw = sB + STAGES * C::B_BYTES;
    SmemCtl* ctl = reinterpret_cast<SmemCtl*>(sRaw + C::RSTAGES * C::RAW_STAGE);
    uint8_t* sStage = reinterpret_cast<uint8_t*>(ctl) + 1024;
    constexpr int RSTAGES = C::RSTAGES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = (CTAS == 2) ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int cluster_id = blockIdx.x / CTAS, nclusters = gridDim.x / CTAS;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ASTAGES; ++s) {
            mbar_init(smem_u32(&ctl->a_full[s]), 1);               // producer of the first CTA
            mbar_init(smem_u32(&ctl->a_empty[s]), 1);              // MMA commit
        }
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&ctl->b_full[s]), C::DEQ_GROUP_WARPS * CTAS);   // one dequant group per CTA
            mbar_init(smem_u32(&ctl->empty[s]), 1);                // MMA commit
        }
        for (int s = 0; s < RSTAGES; ++s) {
            mbar_init(smem_u32(&ctl->raw_full[s]), 1 + 32);        // TMA + the producer warp's absmax copies
            mbar_init(smem_u32(&ctl->raw_empty[s]), C::DEQ_GROUP_WARPS);       // the dequant group that read it
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&ctl->acc_full[b]), 1);
            mbar_init(smem_u32(&ctl->acc_empty[b]), 4 * CTAS);     // epilogue warps of all CTAs
            for (int w = 0; w < 4; ++w) mbar_init(smem_u32(&ctl->ld_full[w][b]), 1);
        }
        ctl->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == MMA_WARP) {
        if (CTAS == 2) {
            tmem_alloc_pair(smem_u32(&ctl->tmem_base), TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
            tmem_relinquish();
        }
    }
    if (warp == PRODUCER_WARP && lane == 0) {
        tma_prefetch_desc(&tmap_a);
        tma_prefetch_desc(&tmap_raw);
    }
    tc_fence_before();
    __syncthreads();
    if (CTAS == 2) cluster_sync_all();   // peer barriers initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    volatile int* abort_flag = &ctl->abort_flag;
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        return mbar_wait(smem_u32(bar), parity, abort_flag, p.status);
    };
    // arrive on a barrier of the cluster's first CTA
    auto arrive_leader = [&](uint64_t* bar) {
        if (CTAS == 2 && !leader) mbar_arrive_cluster(mapa_shared(smem_u32(bar), 0));
        else mbar_arrive(smem_u32(bar));
    };

    const int4* sched = p.sched;
    const int total_tiles = __ldg(p.tile_prefix + p.E) * p.n_tiles;
    const int nk = p.K / BK;              // k-stages of the quantized weights
    const int nkt = nk + (p.lora_r > 0);  // plus the LoRA stage (the last one of a tile)

    if (warp == PRODUCER_WARP) {
        // A tiles: refilled as soon as the MMA has released a stage.  Each tile is also
        // prefetched into L2 APF stages before its load, which hides the long HBM
        // latency of the gathered activation rows without more shared memory.
        if (lane == 0) {
            constexpr int APF = 8;
            const int a_off = 128 * (int)rank;
            int pf_tile = cluster_id, pf_ks = 0;
            TileInfo pf_ti{};
            if (pf_tile < total_tiles) pf_ti = decode_tile(p, sched, pf_tile, C::TILE_M);
            auto prefetch_next = [&]() {
                if (pf_tile >= total_tiles) return;
                if (pf_ks < nk) tma_prefetch_l2_2d(&tmap_a, pf_ks * BK, pf_ti.row0 + a_off);
                if (++pf_ks == nkt) {
                    pf_ks = 0;
                    pf_tile += nclusters;
                    if (pf_tile < total_tiles) pf_ti = decode_tile(p, sched, pf_tile, C::TILE_M);
                }
            };
            for (int i = 0; i < APF; ++i) prefetch_next();
            uint32_t it = 0;
            bool ok = true;
            for (int tile = cluster_id; tile < total_tiles && ok; tile += nclusters) {
                const TileInfo ti = decode_tile(p, sched, tile, C::TILE_M);
                for (int ks = 0; ks < nkt; ++ks, ++it) {
                    prefetch_next();
                    const int s = it % ASTAGES;
                    const uint32_t r = it / ASTAGES;
                    if (!wait(&ctl->a_empty[s], (r & 1) ^ 1)) { ok = false; break; }
                    const uint32_t a_dst = smem_u32(sA + s * C::A_BYTES);
                    const int a_row = ti.row0 + a_off;
                    // the LoRA stage reads the thin operand [rows, 64] instead of A
                    const CUtensorMap* am = ks < nk ? &tmap_a : &tmap_lora;
                    const int ax = ks < nk ? ks * BK : 0;
                    if (CTAS == 2) {
                        if (leader) mbar_arrive_expect_tx(smem_u32(&ctl->a_full[s]), 2 * C::A_BYTES);
                        tma_load_2d_pair(a_dst, am, mapa_shared(smem_u32(&ctl->a_full[s]), 0), ax, a_row);
                    } else {
                        mbar_arrive_expect_tx(smem_u32(&ctl->a_full[s]), C::A_BYTES);
                        tma_load_2d(a_dst, am, smem_u32(&ctl->a_full[s]), ax, a_row);
                    }
                }
            }
        }
    } else if (warp == RAW_WARP) {
        // packed 4-bit tiles and their absmax values: a deep ring released by the
        // dequantizing threads, so the weight loads run many stages ahead of the MMAs.
        // Lane 0 issues the TMA; every lane copies N_CTA/32 absmax values (cp.async),
        // so the dequantizing threads never wait on global memory.
        constexpr int PER_LANE = C::N_CTA / 32;   // absmax values this lane copies per stage
        uint32_t it = 0;
        for (int tile = cluster_id; tile < total_tiles; tile += nclusters) {
            const TileInfo ti = decode_tile(p, sched, tile, C::TILE_M);
            const int ebase = ti.e * p.b_rows_per_expert;
            // per-tile source of each of this lane's absmax values at k-stage 0, and the
            // step per k-stage (K-major: next block of the row; MN-major: 64 rows down)
            // (MXFP4: the 4 E8M0 scale bytes that hold this block's two 32-block scales)
            const uint8_t* src[PER_LANE];
            bool valid[PER_LANE];
#pragma unroll
            for (int i = 0; i < PER_LANE; ++i) {
                if (CB == 2) {
                    const int64_t off = mx_offset<EPI, CTAS>(p, ti, lane + 32 * i, (int)rank);
                    valid[i] = off >= 0;
                    src[i] = p.mx_scales + (valid[i] ? off : 0);
                } else {
                    const int64_t ix = absmax_index<EPI, CTAS>(p, ti, 0, lane + 32 * i, (int)rank);
                    valid[i] = ix >= 0;
                    src[i] = reinterpret_cast<const uint8_t*>(p.absmax + (valid[i] ? ix : 0));
                }
            }
            const int64_t step = CB == 2 ? (kMajorB ? 0 : (int64_t)BK * p.mx_stride)
                                         : 4 * (kMajorB ? 1 : (int64_t)BK * p.b_blocks_per_row);
            bool ok = true;
            for (int ks = 0; ks < nkt; ++ks, ++it) {
                const int s = it % RSTAGES;
                const uint32_t r = it / RSTAGES;
                if (lane == 0) ok = mbar_wait(smem_u32(&ctl->raw_empty[s]), (r & 1) ^ 1, abort_flag, p.status);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                const uint32_t rb = smem_u32(&ctl->raw_full[s]);
                if (CB == 3 || ks == nk) {   // bf16 weights or the LoRA stage: no packed bytes, the same 1 + 32 arrivals
                    if (lane == 0) mbar_arrive(rb);
                    mbar_arrive(rb);
                    continue;
                }
                uint8_t* stage = sRaw + s * C::RAW_STAGE;
                if (lane == 0) {
                    mbar_arrive_expect_tx(rb, C::RAW_BYTES);
                    const uint32_t raw = smem_u32(stage);
                    if (kMajorB) {
#pragma unroll
                        for (int h = 0; h < C::N_CTA / 128; ++h)
                            tma_load_2d(raw + h * 4096, &tmap_raw, rb, ks * (BK / 2),
                                        ebase + kmajor_row<EPI>(p, ti.nt, (int)rank * C::N_CTA + 128 * h));
                    } else {
                        tma_load_2d(raw, &tmap_raw, rb, (ti.nt * BN + (int)rank * C::N_CTA) / 2, ebase + ks * BK);
                    }
                }
                const uint32_t am = smem_u32(stage + C::RAW_BYTES) + 4u * lane;
#pragma unroll
                for (int i = 0; i < PER_LANE; ++i) {
                    const uint8_t* a = src[i] + ks * step + ((CB == 2 && kMajorB) ? 4 * (ks >> 1) : 0);
                    cp_async_4(am + 128u * i, valid[i] ? a : src[i], valid[i] ? 4u : 0u);
                }
                cp_async_mbar_arrive_noinc(rb);
            }
            if (!ok) break;
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0 && leader) {
            constexpr uint32_t idesc = idesc_bf16(C::TILE_M, BN, kMajorB ? 0 : 1);
            uint32_t it = 0, lt = 0;
            bool ok = true;
            for (int tile = cluster_id; tile < total_tiles && ok; tile += nclusters, ++lt) {
                const uint32_t ab = lt & 1, ar = lt >> 1;
                if (!wait(&ctl->acc_empty[ab], (ar & 1) ^ 1)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + ab * BN;
                for (int ks = 0; ks < nkt; ++ks, ++it) {
                    const int s = it % STAGES, sa = it % ASTAGES;
                    const uint32_t r = it / STAGES, ra = it / ASTAGES;
                    if (!wait(&ctl->a_full[sa], ra & 1) || !wait(&ctl->b_full[s], r & 1)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sA + sa * C::A_BYTES);
                    const uint32_t b_addr = smem_u32(sB + s * C::B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
                        const uint64_t bdesc = kMajorB ? smem_desc_sw128(b_addr + kk * 32, 16, 1024)
                                                       : smem_desc_sw128(b_addr + kk * 2048, 8192, 1024);
                        if (CTAS == 2) mma_bf16_ss_pair(d_tmem, adesc, bdesc, idesc, (ks | kk) != 0);
                        else mma_bf16_ss(d_tmem, adesc, bdesc, idesc, (ks | kk) != 0);
                    }
                    if (CTAS == 2) {
                        mma_commit_pair(smem_u32(&ctl->empty[s]));
                        mma_commit_pair(smem_u32(&ctl->a_empty[sa]));
                    } else {
                        mma_commit(smem_u32(&ctl->empty[s]));
                        mma_commit(smem_u32(&ctl->a_empty[sa]));
                    }
                }
                if (ok) {
                    if (CTAS == 2) mma_commit_pair(smem_u32(&ctl->acc_full[ab]));
                    else mma_commit(smem_u32(&ctl->acc_full[ab]));
                }
            }
        }
    } else if (warp >= DEQ_WARP0 && (warp & 3) != (MMA_WARP & 3)) {
        // warps 8, 10, 11, 12, 14, 15: the MMA-issuing thread's scheduler stays free of
        // dequantization work.  Group g takes k-stages g, g+3, ...; thread tg owns blocks
        // tg + 64*i of this CTA's half.
        const int dq = (warp - DEQ_WARP0) - ((warp - DEQ_WARP0) > (MMA_WARP & 3)) - ((warp - DEQ_WARP0) > 4 + (MMA_WARP & 3));
        const int grp = dq / C::DEQ_GROUP_WARPS;
        const int tg = (dq % C::DEQ_GROUP_WARPS) * 32 + lane;   // 0..63
        constexpr int NB = C::BLK_PER_THREAD;
        constexpr int TPG = 32 * C::DEQ_GROUP_WARPS;             // threads per group
        uint32_t it = grp;
        int tile = cluster_id, ks = grp;
        auto normalize = [&]() {   // carry ks past the end of a tile into the next tile(s)
            while (ks >= nkt && tile < total_tiles) {
                ks -= nkt;
                tile += nclusters;
            }
        };
        normalize();
        while (tile < total_tiles) {
            const int s = it % STAGES;
            const uint32_t r = it / STAGES;
            const int cur_tile = tile, cur_ks = ks;
            ks += C::DEQ_GROUPS;   // this group's next stage
            normalize();
            const int rs = it % RSTAGES;
            const uint32_t rr = it / RSTAGES;
            if (!mbar_wait(smem_u32(&ctl->raw_full[rs]), rr & 1, abort_flag, p.status)) break;
            if (CB == 3 || cur_ks == nk) {
                // bf16 weights (CB 3) or the LoRA stage: the tile in bf16 straight from global
                // memory, in the same shared-memory layout as a dequantized tile
                const bool lora_stage = cur_ks == nk;
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&ctl->raw_empty[rs]));
                if (!wait(&ctl->empty[s], (r & 1) ^ 1)) break;
                const TileInfo ti = decode_tile(p, sched, cur_tile, C::TILE_M);
                uint8_t* dst_tile = sB + s * C::B_BYTES;
                if (CB == 3 && !lora_stage) {
                    // bf16 weights: the group's first warp loads this CTA's part of the tile by
                    // TMA (tmap_raw maps the bf16 stack, 128B-swizzled: the operand layout),
                    // completing on the first CTA's barrier; the other warps only arrive.
                    // Rows or columns outside the stack read as zero; those of a neighbouring
                    // expert only feed output columns that are never stored.
                    if (lane == 0) {
                        if (tg == 0) {
                            const uint32_t bar = smem_u32(&ctl->b_full[s]);
                            if (leader) mbar_arrive_expect_tx(bar, CTAS * C::B_BYTES);
                            else mbar_arrive_cluster(mapa_shared(bar, 0));
                            const int ebase = ti.e * p.b_rows_per_expert;
                            auto load = [&](uint32_t dst, int x, int y) {
                                if (CTAS == 2) tma_load_2d_pair(dst, &tmap_raw, mapa_shared(bar, 0), x, y);
                                else tma_load_2d(dst, &tmap_raw, bar, x, y);
                            };
                            if (kMajorB) {   // boxes of 128 stored rows x 64 k
#pragma unroll
                                for (int h = 0; h < C::N_CTA / 128; ++h)
                                    load(smem_u32(dst_tile) + h * 16384, cur_ks * BK,
                                         ebase + kmajor_row<EPI>(p, ti.nt, (int)rank * C::N_CTA + 128 * h));
                            } else {         // boxes of 64 k-rows x 64 stored columns
#pragma unroll
                                for (int j = 0; j < C::N_CTA / 64; ++j)
                                    load(smem_u32(dst_tile) + j * 8192, ti.nt * BN + (int)rank * C::N_CTA + 64 * j,
                                         ebase + cur_ks * BK);
                            }
                        } else {
                            arrive_leader(&ctl->b_full[s]);
                        }
                    }
                    it += C::DEQ_GROUPS;
                    continue;
                }
#pragma unroll
                for (int i = 0; i < NB; ++i) {
                    const int b = tg + TPG * i;
                    const __nv_bfloat16* src = nullptr;   // 64 consecutive bf16 of the tile row b, or null
                    int nvalid = 0;                        // of which the first nvalid are in range
                    if (kMajorB) {   // row b of this CTA's half
                        const int n = (int)rank * C::N_CTA + b;
                        const int row = kmajor_row<EPI>(p, ti.nt, n);
                        const bool in = (EPI == EPI_GATEUP) ? (ti.nt * 128 + (n & 127) < p.up_offset)
                                                            : (row < p.b_rows_per_expert);
                        if (in && lora_stage) {   // the adapter's r values, zeros after
                            src = p.lora_b + ((int64_t)ti.e * p.b_rows_per_expert + row) * p.lora_r;
                            nvalid = p.lora_r;
                        } else if (in) {          // 64 weights of the row at this k-stage
                            src = p.bf16_b + ((int64_t)ti.e * p.b_rows_per_expert + row) * p.K + cur_ks * BK;
                            nvalid = 64;
                        }
                    } else {         // k-row q = b & 63, columns of block b >> 6
                        const int q = b & 63, col = ti.nt * BN + (int)rank * C::N_CTA + (b >> 6) * 64;
                        if (lora_stage) {   // q is the rank index
                            if (q < p.lora_r && col < p.N) {
                                src = p.lora_b + ((int64_t)ti.e * p.lora_r + q) * p.N + col;
                                nvalid = min(64, p.N - col);
                            }
                        } else if (col < p.N) {   // stored row ks * 64 + q of the expert
                            src = p.bf16_b + ((int64_t)ti.e * p.b_rows_per_expert + cur_ks * BK + q) * p.N + col;
                            nvalid = min(64, p.N - col);
                        }
                    }
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint4 v = make_uint4(0u, 0u, 0u, 0u);
                        if (src && 8 * c < nvalid) v = __ldg(reinterpret_cast<const uint4*>(src) + c);
                        const uint32_t off = kMajorB ? sw128_offset(b, c) : (b >> 6) * 8192 + sw128_offset(b & 63, c);
                        *reinterpret_cast<uint4*>(dst_tile + off) = v;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) arrive_leader(&ctl->b_full[s]);
                it += C::DEQ_GROUPS;
                continue;
            }
            const uint8_t* raw_stage = sRaw + rs * C::RAW_STAGE;
            const float* am = reinterpret_cast<const float*>(raw_stage + C::RAW_BYTES);
            uint4 pk[NB][2];
            float a_cur[NB];
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                const int b = tg + TPG * i;
                a_cur[i] = am[b];
                if (kMajorB) {   // raw [N_CTA rows][32 B]
                    pk[i][0] = *reinterpret_cast<const uint4*>(raw_stage + b * 32);
                    pk[i][1] = *reinterpret_cast<const uint4*>(raw_stage + b * 32 + 16);
                } else {         // raw [64 k-rows][N_CTA/2 B], TMA-swizzled per row
                    const int k = b & 63, j = b >> 6;
                    constexpr int ROWB = C::N_CTA / 2;   // 128 B (128B swizzle) or 64 B (64B swizzle)
                    const int sw = (ROWB == 128) ? (k & 7) : ((k >> 1) & 3);
                    pk[i][0] = *reinterpret_cast<const uint4*>(raw_stage + k * ROWB + (((2 * j) ^ sw) << 4));
                    pk[i][1] = *reinterpret_cast<const uint4*>(raw_stage + k * ROWB + (((2 * j + 1) ^ sw) << 4));
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl->raw_empty[rs]));
            // the bf16 stage is free once the MMAs that read it (STAGES stages ago) are done
            if (!wait(&ctl->empty[s], (r & 1) ^ 1)) break;
            uint8_t* dst_tile = sB + s * C::B_BYTES;
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                const int b = tg + TPG * i;
                // MXFP4: the block's two 32-element halves have their own scales, bytes
                // sel and sel+1 of the 4 copied (K-major: by k-stage; MN-major: by n-block)
                BlockTable tb, tb1;
                if (CB == 2) {
                    const uint32_t sc = __float_as_uint(a_cur[i]);
                    const int sel = kMajorB ? 2 * (cur_ks & 1) : 2 * ((b >> 6) & 1);
                    tb = make_table<2>(mx_scale((sc >> (8 * sel)) & 0xFFu));
                    tb1 = make_table<2>(mx_scale((sc >> (8 * sel + 8)) & 0xFFu));
                } else {
                    tb = make_table<(CB < 3 ? CB : 0)>(a_cur[i]);   // CB 3 never reaches this path
                }
                const uint32_t words[8] = {pk[i][0].x, pk[i][0].y, pk[i][0].z, pk[i][0].w,
                                           pk[i][1].x, pk[i][1].y, pk[i][1].z, pk[i][1].w};
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t o[4];
                    decode_word((CB == 2 && c >= 4) ? tb1 : tb, words[c], o);
                    const uint32_t off = kMajorB ? sw128_offset(b, c) : (b >> 6) * 8192 + sw128_offset(b & 63, c);
                    *reinterpret_cast<uint4*>(dst_tile + off) = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) arrive_leader(&ctl->b_full[s]);
            it += C::DEQ_GROUPS;
        }
    } else if (warp < 4) {
        // ------------------------------------------------------------ epilogue
        // Lane l holds accumulator row (32*warp + l) of this CTA's half.  A warp whose 32
        // rows all lie inside the tile writes each 32 x 32 output chunk into one of its
        // three staging buffers (row l at 64*l, 16-byte chunks 64B-swizzled: chunk c at
        // c ^ ((l >> 1) & 3), which is also conflict-free for the 16-byte stores) and
        // lane 0 sends it out with a TMA tensor store; the tail warp of a partial tile
        // stores its valid rows directly.
        const int rloc = warp * 32 + lane;   // TMEM lane == row of this CTA's half
        uint8_t* stg = sStage + warp * C::STAGE_WARP;
        uint32_t nbuf = 0;                   // staging buffers used so far (rotating)
        // EPI_DGRAD_DOWN, whole-slab warps: the saved dh/dg and dh/du chunks of a 32 x 32
        // output chunk come in by TMA (pair n & 1 of the warp's four buffers, barrier
        // ld_full[warp][n & 1]), are turned into dG, dU in place and leave by TMA
        uint32_t nld = 0, ncons = 0;         // chunk pairs requested / consumed
        auto issue_pair = [&](int c0, int srow) {
            uint8_t* gb = stg + (nld & 1) * 2 * C::STAGE_BUF;
            if (lane == 0) {
                bulk_wait_read<0>();          // the stores that last read this pair are done with it
                const uint32_t bar = smem_u32(&ctl->ld_full[warp][nld & 1]);
                mbar_arrive_expect_tx(bar, 2 * C::STAGE_BUF);
                tma_load_2d(smem_u32(gb), &tmap_gu, bar, c0, srow);
                tma_load_2d(smem_u32(gb + C::STAGE_BUF), &tmap_gu, bar, p.N + c0, srow);
            }
            __syncwarp();
            ++nld;
        };
        bool aborted = false;
        auto stage_store = [&](const uint32_t (&v)[16], const CUtensorMap* m, int x, int y) {
            uint8_t* buf = stg + (nbuf % C::STAGE_BUFS) * C::STAGE_BUF;
            if (nbuf >= (uint32_t)C::STAGE_BUFS) {   // the store that last read this buffer is done reading
                if (lane == 0) bulk_wait_read<C::STAGE_BUFS - 1>();
                __syncwarp();
            }
            const int sw = (lane >> 1) & 3;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4*>(buf + lane * 64 + ((c ^ sw) << 4)) =
                    make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(m, smem_u32(buf), x, y);
                bulk_commit();
            }
            ++nbuf;
        };
        uint32_t lt = 0;
        for (int tile = cluster_id; tile < total_tiles; tile += nclusters, ++lt) {
            const TileInfo ti = decode_tile(p, sched, tile, C::TILE_M);
            const uint32_t ab = lt & 1, ar = lt >> 1;
            const int rtile = 128 * (int)rank + rloc;
            const int wrow0 = 128 * (int)rank + 32 * warp;   // this warp's first row in the tile
            const bool bulk = ti.rows - wrow0 >= 32;          // all 32 rows inside the tile
            const bool any = ti.rows > wrow0;
            const bool valid = rtile < ti.rows;
            const int row = ti.row0 + rtile;
            const int srow = ti.row0 + wrow0;                 // first row of the warp's TMA boxes
            // everything that does not depend on the accumulator is fetched before waiting for it
            float wgt = 1.0f;
            if ((EPI == EPI_DOWN || EPI == EPI_DGRAD_DOWN) && valid) {
                const int pid = __ldg(p.perm + row);
#if E4B_DEBUG_CHECKS
                if (pid < 0 || pid >= p.a_rows) debug_fail(p.status, kSiteGemmPerm);
                else
#endif
                    wgt = __ldg(p.topk_w + pid);
            }
            float dwdot = 0.0f;   // EPI_DGRAD_DOWN, XACT: <grad_out W_d, h> over the tile's columns
            uint4 gq[4], uq[4];   // EPI_DGRAD_DOWN: saved dh/dg, dh/du of the current 32-column chunk
            auto load_gu = [&](int q, uint4 (&g4)[4], uint4 (&u4)[4]) {
                const int c0 = ti.nt * BN + 32 * q;
                if (valid && c0 < p.N) {
                    const uint4* gsrc = reinterpret_cast<const uint4*>(p.gu + (int64_t)row * 2 * p.N + c0);
                    const uint4* usrc = reinterpret_cast<const uint4*>(p.gu + (int64_t)row * 2 * p.N + p.N + c0);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        g4[i] = __ldg(gsrc + i);
                        u4[i] = __ldg(usrc + i);
                    }
                }
            };
            if (EPI == EPI_DGRAD_DOWN) {
                if (bulk) {
                    if (ti.nt * BN < p.N) issue_pair(ti.nt * BN, srow);
                } else {
                    load_gu(0, gq, uq);
                }
            }
            if (!wait(&ctl->acc_full[ab], ar & 1)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(warp * 32) << 16) + ab * BN;
            if (EPI == EPI_GATEUP) {
                const int I = p.up_offset;
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    float g[32], u[32];
                    tmem_load32(tbase + 32 * q, g);
                    tmem_load32(tbase + 128 + 32 * q, u);
                    const int f0 = ti.nt * 128 + 32 * q;
                    if (any && f0 < I) {
                        if (XACT && p.bias) {   // per-expert bias: lane l loads column f0 + l, shuffles share it
                            const float bgl = __ldg(p.bias + (int64_t)ti.e * 2 * I + f0 + lane);
                            const float bul = __ldg(p.bias + (int64_t)ti.e * 2 * I + I + f0 + lane);
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                g[j] += __shfl_sync(0xffffffffu, bgl, j);
                                u[j] += __shfl_sync(0xffffffffu, bul, j);
                            }
                        }
                        if (!XACT) {
                            // h = silu(g) u and the two derivatives the input gradient needs, in place:
                            // u <- dh/dg = u s (1 + g (1 - s)), g <- dh/du = silu(g), s = sigmoid(g).
                            // (This plain instance needs no spill in the in-place form; the extended
                            // instance below packs its outputs as it goes, which spills least there.)
                            uint32_t hv[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                float hh[2];
#pragma unroll
                                for (int h = 0; h < 2; ++h) {
                                    const int j = 2 * i + h;
                                    const float gg = g[j], uu = u[j];
                                    const float sg = __fdividef(1.0f, 1.0f + __expf(-gg));
                                    const float sl = gg * sg;
                                    hh[h] = sl * uu;
                                    u[j] = uu * sg * (1.0f + gg * (1.0f - sg));
                                    g[j] = sl;
                                }
                                hv[i] = pack_bf16x2(hh[0], hh[1]);
                            }
                            auto pack32 = [&](const float (&f)[32], uint32_t (&o)[16]) {
#pragma unroll
                                for (int i = 0; i < 16; ++i) o[i] = pack_bf16x2(f[2 * i], f[2 * i + 1]);
                            };
                            if (bulk) {
                                stage_store(hv, &tmap_out, f0, srow);
                                if (p.gu) {
                                    uint32_t pk[16];
                                    pack32(u, pk);
                                    stage_store(pk, &tmap_gu, f0, srow);
                                    pack32(g, pk);
                                    stage_store(pk, &tmap_gu, I + f0, srow);
                                }
                            } else if (valid) {
                                uint4* dst = reinterpret_cast<uint4*>(p.out_bf16 + (int64_t)row * p.ld_out + f0);
#pragma unroll
                                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
                                if (p.gu) {
                                    uint32_t pk[16];
                                    pack32(u, pk);
                                    uint4* dg = reinterpret_cast<uint4*>(p.gu + (int64_t)row * 2 * I + f0);
#pragma unroll
                                    for (int i = 0; i < 4; ++i) dg[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                                    pack32(g, pk);
                                    uint4* du = reinterpret_cast<uint4*>(p.gu + (int64_t)row * 2 * I + I + f0);
#pragma unroll
                                    for (int i = 0; i < 4; ++i) du[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                                }
                            }
                        } else {
                            // Extended instance: h = act(g, u) and the two derivatives, each packed to
                            // bf16 pairs as soon as its column pair is done.
                            //   SwiGLU: as above
                            //   clamped GLU: g' = min(g, L), u' = clamp(u, -L, L), s = sigmoid(a g'),
                            //     h = (u' + 1) g' s, dh/dg = [g <= L] (u' + 1) s (1 + a g' (1 - s)),
                            //     dh/du = [-L <= u <= L] g' s
                            uint32_t hv[16], pdg[16], pdu[16];
                            const bool clamped = p.act != 0;
                            const float al = clamped ? p.alpha : 1.0f, L = p.limit;
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                float hh[2], dg[2], du[2];
#pragma unroll
                                for (int h = 0; h < 2; ++h) {
                                    const int j = 2 * i + h;
                                    const float gg = g[j], uu = u[j];
                                    if (!clamped) {
                                        const float sg = __fdividef(1.0f, 1.0f + __expf(-gg));
                                        const float sl = gg * sg;
                                        hh[h] = sl * uu;
                                        dg[h] = uu * sg * (1.0f + gg * (1.0f - sg));
                                        du[h] = sl;
                                    } else {
                                        const float gc = fminf(gg, L), uc = fminf(fmaxf(uu, -L), L);
                                        const float sg = __fdividef(1.0f, 1.0f + __expf(-al * gc));
                                        const float gs = gc * sg;
                                        hh[h] = (uc + 1.0f) * gs;
                                        dg[h] = (gg <= L) ? (uc + 1.0f) * sg * (1.0f + al * gc * (1.0f - sg)) : 0.0f;
                                        du[h] = (uu >= -L && uu <= L) ? gs : 0.0f;
                                    }
                                }
                                hv[i] = pack_bf16x2(hh[0], hh[1]);
                                pdg[i] = pack_bf16x2(dg[0], dg[1]);
                                pdu[i] = pack_bf16x2(du[0], du[1]);
                            }
                            if (bulk) {
                                stage_store(hv, &tmap_out, f0, srow);
                                if (p.gu) {
                                    stage_store(pdg, &tmap_gu, f0, srow);
                                    stage_store(pdu, &tmap_gu, I + f0, srow);
                                }
                            } else if (valid) {
                                auto put = [&](__nv_bfloat16* base, const uint32_t (&v)[16]) {
                                    uint4* dst = reinterpret_cast<uint4*>(base);
#pragma unroll
                                    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                                };
                                put(p.out_bf16 + (int64_t)row * p.ld_out + f0, hv);
                                if (p.gu) {
                                    put(p.gu + (int64_t)row * 2 * I + f0, pdg);
                                    put(p.gu + (int64_t)row * 2 * I + I + f0, pdu);
                                }
                            }
                        }
                    }
                }
            } else if (EPI == EPI_DGRAD_DOWN && bulk) {
                const int I = p.N;
#pragma unroll 1
                for (int q = 0; q < BN / 32; ++q) {
                    const int c0 = ti.nt * BN + 32 * q;
                    if (c0 >= I) break;
                    float v[32];
                    tmem_load32(tbase + 32 * q, v);
                    if (q + 1 < BN / 32 && c0 + 32 < I) issue_pair(c0 + 32, srow);   // next pair in flight
                    if (XACT) dw_dot_chunk(p, row, c0, v, dwdot);
                    const uint32_t n = ncons++;
                    if (!wait(&ctl->ld_full[warp][n & 1], (n >> 1) & 1)) {
                        aborted = true;
                        break;
                    }
                    uint8_t* gb = stg + (n & 1) * 2 * C::STAGE_BUF;
                    uint8_t* ub = gb + C::STAGE_BUF;
                    const int sw = (lane >> 1) & 3;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {   // row `lane`, 16-byte chunk c (64B swizzle)
                        uint4* gp = reinterpret_cast<uint4*>(gb + lane * 64 + ((c ^ sw) << 4));
                        uint4* up = reinterpret_cast<uint4*>(ub + lane * 64 + ((c ^ sw) << 4));
                        const uint4 g4 = *gp, u4 = *up;
                        const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
                        const uint32_t uw[4] = {u4.x, u4.y, u4.z, u4.w};
                        uint32_t dgw[4], duw[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float dh0 = v[8 * c + 2 * j] * wgt, dh1 = v[8 * c + 2 * j + 1] * wgt;
                            dgw[j] = pack_bf16x2(dh0 * __uint_as_float(gw[j] << 16),
                                                 dh1 * __uint_as_float(gw[j] & 0xFFFF0000u));
                            duw[j] = pack_bf16x2(dh0 * __uint_as_float(uw[j] << 16),
                                                 dh1 * __uint_as_float(uw[j] & 0xFFFF0000u));
                        }
                        *gp = make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]);
                        *up = make_uint4(duw[0], duw[1], duw[2], duw[3]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmap_out, smem_u32(gb), c0, srow);
                        tma_store_2d(&tmap_out, smem_u32(ub), I + c0, srow);
                        bulk_commit();
                    }
                }
                if (aborted) break;
                if (XACT) p.dw_part[(int64_t)row * p.n_tiles + ti.nt] = dwdot;
            } else {
#pragma unroll 1
                for (int q = 0; q < BN / 32; ++q) {
                    // the partial tile's rows (this path): the chunk's saved derivatives are
                    // loaded with it, not one chunk ahead, which keeps 32 registers free
                    if (EPI == EPI_DGRAD_DOWN && q > 0) load_gu(q, gq, uq);
                    float v[32];
                    tmem_load32(tbase + 32 * q, v);
                    const int c0 = ti.nt * BN + 32 * q;
                    if (any && c0 < p.N) {
                        if (EPI == EPI_DOWN || EPI == EPI_DGRAD_GATEUP) {
                            // this pair's contribution, rounded to bf16, into its grouped row
                            // (summed over the k rows of each token by the combine kernel);
                            // the down projection's per-expert bias joins before the weight
                            if (EPI == EPI_DOWN && p.bias) {
                                const float4* bd = reinterpret_cast<const float4*>(p.bias + (int64_t)ti.e * p.N + c0);
#pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    const float4 b = __ldg(bd + i);
                                    v[4 * i] += b.x; v[4 * i + 1] += b.y; v[4 * i + 2] += b.z; v[4 * i + 3] += b.w;
                                }
                            }
                            uint32_t ov[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) ov[i] = pack_bf16x2(v[2 * i] * wgt, v[2 * i + 1] * wgt);
                            if (bulk) {
                                stage_store(ov, &tmap_out, c0, srow);
                            } else if (valid) {
                                uint4* dst = reinterpret_cast<uint4*>(p.out_bf16 + (int64_t)row * p.ld_out + c0);
#pragma unroll
                                for (int i = 0; i < 4; ++i)
                                    dst[i] = make_uint4(ov[4 * i], ov[4 * i + 1], ov[4 * i + 2], ov[4 * i + 3]);
                            }
                        } else {   // EPI_DGRAD_DOWN: SwiGLU backward with the saved derivatives
                            const int I = p.N;
                            if (XACT && valid) dw_dot_chunk(p, row, c0, v, dwdot);
                            uint32_t dgw[16], duw[16];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const uint32_t gw[4] = {gq[i].x, gq[i].y, gq[i].z, gq[i].w};
                                const uint32_t uw[4] = {uq[i].x, uq[i].y, uq[i].z, uq[i].w};
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    const float dh0 = v[8 * i + 2 * j] * wgt, dh1 = v[8 * i + 2 * j + 1] * wgt;
                                    dgw[4 * i + j] = pack_bf16x2(dh0 * __uint_as_float(gw[j] << 16),
                                                                 dh1 * __uint_as_float(gw[j] & 0xFFFF0000u));
                                    duw[4 * i + j] = pack_bf16x2(dh0 * __uint_as_float(uw[j] << 16),
                                                                 dh1 * __uint_as_float(uw[j] & 0xFFFF0000u));
                                }
                            }
                            if (bulk) {
                                stage_store(dgw, &tmap_out, c0, srow);
                                stage_store(duw, &tmap_out, I + c0, srow);
                            } else if (valid) {
                                uint4* dgo = reinterpret_cast<uint4*>(p.out_bf16 + (int64_t)row * 2 * I + c0);
                                uint4* duo = reinterpret_cast<uint4*>(p.out_bf16 + (int64_t)row * 2 * I + I + c0);
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    dgo[i] = make_uint4(dgw[4 * i], dgw[4 * i + 1], dgw[4 * i + 2], dgw[4 * i + 3]);
                                    duo[i] = make_uint4(duw[4 * i], duw[4 * i + 1], duw[4 * i + 2], duw[4 * i + 3]);
                                }
                            }
                        }
                    }
                }
                if (EPI == EPI_DGRAD_DOWN && XACT && valid) p.dw_part[(int64_t)row * p.n_tiles + ti.nt] = dwdot;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_leader(&ctl->acc_empty[ab]);
        }
        if (lane == 0) {
            bulk_wait_all();   // this warp's tensor stores have left shared memory
            for (; ncons < nld; ++ncons)   // and its derivative loads have landed (bounded)
                mbar_wait_drain(smem_u32(&ctl->ld_full[warp][ncons & 1]), (ncons >> 1) & 1);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (CTAS == 2) cluster_sync_all();   // the peer's smem and TMEM stay alive until the pair is done
    if (warp == MMA_WARP) {
        tc_fence_after();
        if (CTAS == 2) tmem_dealloc_pair(tmem_base, TMEM_COLS);
        else tmem_dealloc(tmem_base, TMEM_COLS);
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

bool make_tensor_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn || rank < 1 || rank > 5) return false;
    cuuint64_t d[5], s[4];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
        if (i + 1 < rank) s[i] = strides_bytes[i];
    }
    return fn(m, dt, rank, const_cast<void*>(base), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

// CTAs per tile of the grouped GEMMs (2: cta_group::2 pairs on two SMs; the kernel
// template also has a single-SM configuration, CTAS = 1, which is not launched).
constexpr int kCtas = 2;
int gemm_tile_rows() { return Cfg<kCtas>::TILE_M; }

template <int EPI, int CB, int CTAS, bool XACT = false>
static cudaError_t launch_one(const CUtensorMap& ma, const CUtensorMap& mr, const CUtensorMap& mo,
                              const CUtensorMap& mg, const CUtensorMap& ml, const GemmParams& p, int grid,
                              cudaStream_t st) {
    using C = Cfg<CTAS, EPI>;
    auto kern = grouped_gemm_kernel<EPI, CB, CTAS, XACT>;
    // The shared-memory limit is a per-device function attribute: set it once per
    // device and instantiation, under a lock.
    {
        static std::mutex mu;
        static bool attr_set[64] = {false};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
        std::lock_guard<std::mutex> lock(mu);
        if (!attr_set[dev]) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
            if (e != cudaSuccess) return e;
            attr_set[dev] = true;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(GEMM_THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CTAS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ma, mr, mo, mg, ml, p);
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// The instance for the epilogue kind and codebook: the extended epilogue (XACT) for the
// gate_up variant (clamped GLU or biases) and for the routing-gradient dot products.
template <int CB, int CTAS>
static cudaError_t launch_cb(int epi, const CUtensorMap& ma, const CUtensorMap& mr, const CUtensorMap& mo,
                             const CUtensorMap& mg, const CUtensorMap& ml, const GemmParams& p, int grid,
                             cudaStream_t st) {
    if (epi == EPI_GATEUP && (p.act != 0 || p.bias != nullptr))
        return launch_one<EPI_GATEUP, CB, CTAS, true>(ma, mr, mo, mg, ml, p, grid, st);
    if (epi == EPI_DGRAD_DOWN && p.dw_part)
        return launch_one<EPI_DGRAD_DOWN, CB, CTAS, true>(ma, mr, mo, mg, ml, p, grid, st);
    switch (epi) {
        case EPI_GATEUP: return launch_one<EPI_GATEUP, CB, CTAS>(ma, mr, mo, mg, ml, p, grid, st);
        case EPI_DOWN: return launch_one<EPI_DOWN, CB, CTAS>(ma, mr, mo, mg, ml, p, grid, st);
        case EPI_DGRAD_DOWN: return launch_one<EPI_DGRAD_DOWN, CB, CTAS>(ma, mr, mo, mg, ml, p, grid, st);
        default: return launch_one<EPI_DGRAD_GATEUP, CB, CTAS>(ma, mr, mo, mg, ml, p, grid, st);
    }
}

// One launch of configuration CTAS over the whole m-tile schedule (max_tiles bounds
// the tiles it can find there).
template <int CTAS>
static cudaError_t launch_cfg(int epi, int codebook, const void* a, int64_t a_rows, const uint8_t* packed,
                              int64_t packed_rows_total, int packed_row_bytes, const GemmParams& p, int64_t max_tiles,
                              cudaStream_t st, const void* lora_a) {
    using C = Cfg<CTAS>;
    CUtensorMap ma, mr;
    if (!make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a, (uint64_t)p.K, (uint64_t)a_rows, (uint64_t)p.K * 2, 64,
                     128, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const bool kmaj = (epi == EPI_GATEUP || epi == EPI_DOWN);
    // K-major: boxes of 128 rows x 32 bytes; MN-major: 64 k-rows x (N_CTA/2) bytes, swizzled so the
    // dequantizing threads read it without bank conflicts.
    const uint32_t mn_row = C::N_CTA / 2;
    if (codebook == 3) {
        // bf16 weights [b_rows_total, cols] (cols = K when K-major, N when MN-major): boxes
        // of 64 columns (128 B, 128B swizzle: the UMMA operand layout) x 128 rows (K-major)
        // or x 64 k-rows (MN-major)
        const uint64_t cols = kmaj ? (uint64_t)p.K : (uint64_t)p.N;
        if (!make_map_2d(&mr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.bf16_b, cols, (uint64_t)p.b_rows_total, cols * 2,
                         64, kmaj ? 128 : BK, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    } else if (!make_map_2d(&mr, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)packed_row_bytes,
                            (uint64_t)packed_rows_total, (uint64_t)packed_row_bytes, kmaj ? BK / 2 : mn_row,
                            kmaj ? 128 : BK,
                            kmaj ? CU_TENSOR_MAP_SWIZZLE_NONE
                                 : (mn_row == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))) {
        return cudaErrorInvalidValue;
    }
    // epilogue outputs: 32 x 32 boxes, 64B-swizzled, of the [rows, ld_out] output (h, the
    // input-gradient halves or the per-pair rows) and of the saved derivatives [rows, 2I]
    CUtensorMap mo, mg;
    if (!make_map_2d(&mo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.out_bf16, (uint64_t)p.ld_out, (uint64_t)a_rows,
                     (uint64_t)p.ld_out * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    mg = mo;
    // saved derivatives [rows, 2I]: written by the gate_up epilogue, read by the down^T epilogue
    const int64_t n_feat = (epi == EPI_GATEUP) ? p.up_offset : p.N;
    if ((epi == EPI_GATEUP || epi == EPI_DGRAD_DOWN) && p.gu &&
        !make_map_2d(&mg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.gu, (uint64_t)n_feat * 2, (uint64_t)a_rows,
                     (uint64_t)n_feat * 4, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    // the LoRA stage's thin A operand [rows, 64] bf16: one 64-deep box per 128 tile rows
    CUtensorMap ml = ma;
    if (p.lora_r > 0 &&
        !make_map_2d(&ml, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora_a, 64, (uint64_t)a_rows, 128, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int grid = (int)std::min<int64_t>(max_tiles * CTAS, (num_sms() / CTAS) * CTAS);
    if (grid <= 0) return cudaSuccess;
    switch (codebook) {
        case 0: return launch_cb<0, CTAS>(epi, ma, mr, mo, mg, ml, p, grid, st);
        case 1: return launch_cb<1, CTAS>(epi, ma, mr, mo, mg, ml, p, grid, st);
        case 2: return launch_cb<2, CTAS>(epi, ma, mr, mo, mg, ml, p, grid, st);
        default: return launch_cb<3, CTAS>(epi, ma, mr, mo, mg, ml, p, grid, st);
    }
}

cudaError_t launch_grouped_gemm(int epi, int codebook, const void* a, int64_t a_rows, const uint8_t* packed,
                                int64_t packed_rows_total, int packed_row_bytes, GemmParams p, int max_m_tiles,
                                cudaStream_t st, const void* lora_a) {
    p.a_rows = a_rows;
    if (p.lora_r > 0 && (!lora_a || !p.lora_b || p.lora_r % 8 || p.lora_r > 64)) return cudaErrorInvalidValue;
    if (epi == EPI_DGRAD_DOWN && p.dw_part && !p.h_in) return cudaErrorInvalidValue;
    if (codebook == 2 && (!p.mx_scales || p.mx_stride < (p.b_blocks_per_row * 2 + 15) / 16 * 16))
        return cudaErrorInvalidValue;
    if (codebook == 3 && !p.bf16_b) return cudaErrorInvalidValue;
    if (max_m_tiles <= 0) return cudaSuccess;
    timing_begin(KK_GEMM_GATEUP + epi, st);
    const cudaError_t e = launch_cfg<kCtas>(epi, codebook, a, a_rows, packed, packed_rows_total, packed_row_bytes, p,
                                            (int64_t)max_m_tiles * p.n_tiles, st, lora_a);
    timing_end(KK_GEMM_GATEUP + epi, st);
    return e;
}

}  // namespace e4b
