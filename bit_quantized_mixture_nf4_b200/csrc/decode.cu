// Small-batch (T <= 8) forward.  At a handful of tokens the layer is a
// weight-streaming GEMV: every touched expert's packed weights are read once,
// so HBM bandwidth bounds it and tensor-core throughput does not matter.
//
// This is the decode fast path of the expert-layer pages ("experts4bit-qlora"
// 0.4.0 description, section "Inference": single-token forward over the token's
// top-k experts with no host synchronisation, 4-bit GEMV reading packed NF4
// directly), designed for B200:
//
//  * Two kernels, gate_up and down, chained with programmatic dependent launch
//    (PDL): each builds its lookup table before it waits on its predecessor.
//    gate_up routes the <= 8 tokens (one warp per token, in every CTA) and CTA
//    0 publishes the routing and its grouping for the down kernel.
//  * Work item = one 8-row weight tile over all of K for one routed expert
//    (gate_up: 4 gate and 4 up rows; down: 8 output rows).  Each warp owns
//    whole items and streams them through its own ring of shared-memory
//    sub-stages (8 blocks of 64 elements of the 8 rows, plus their absmax, and
//    for down the h rows of the expert's tokens) with a multistage cp.async
//    pipeline.  A warp accumulates the full K itself: no CTA barrier and no
//    cross-warp reduction in the main loop, no spin-waits.  The padded sub-stage
//    rows make the reads bank-conflict free.
//  * Weight decode: a 256-entry table maps a packed byte (two 4-bit codes) to a
//    bf16x2 pair of code values.  The table is replicated for each of the 32
//    lanes, so a warp's 32 lookups hit 32 distinct banks.  The lookup address
//    takes one byte permute and one shift.
//  * Math: mma.sync m16n8k16 (bf16 in, fp32 out).  The weight tile is the B
//    operand (8 rows); the activation rows (the tokens routed to the expert,
//    <= 8) are the A operand.  Each MMA covers 16 elements of one 64-element
//    block, so the block's absmax multiplies the fp32 block partial once
//    (w = code * absmax, code in bf16, scale applied in fp32).
#include "e4b_internal.h"

namespace e4b {

constexpr int DK_THREADS = 256;
constexpr int DK_WARPS = DK_THREADS / 32;
constexpr int DK_MAXP = 64;                 // T * k <= 8 * 8 routed pairs
constexpr int DK_MAXE = 256;
constexpr int DK_NS_MAX = 8;                // sub-stages per warp ring
constexpr int DK_KC = 8;                    // 64-element blocks per sub-stage
constexpr int DK_DN_MAX_RT = 8;             // down: 8-row tiles per CTA
constexpr uint32_t DK_LUT_BYTES = 32768;    // 256 byte values x 32 lanes x 4 B
// sub-stage layout: 8 weight rows of DK_KC*32 bytes padded to 288 (72 words = 8 mod 32:
// the 4 rows a half-warp reads fall in distinct banks), 8 absmax rows of DK_KC floats
// padded to 12 words (4 mod 8), then (down) up to 8 activation rows of DK_KC*128
// bytes padded to 1040 (an odd count of 16-byte units)
constexpr int DK_SUB_RS = DK_KC * 32 + 32;
constexpr int DK_SUB_ABS = 8 * DK_SUB_RS;
constexpr int DK_SUB_ASW = DK_KC + 4;
constexpr int DK_SUB_A = DK_SUB_ABS + 8 * DK_SUB_ASW * 4;
constexpr int DK_SUB_AS = DK_KC * 128 + 16;

// e2m1 values (sign in bit 3).  The FP4 codebook is these divided by 6; the
// division is applied to the fp32 result, so the table is exact in bf16.
static __constant__ float c_e2m1[16] = {0.0f,  0.5f,  1.0f,  1.5f,  2.0f,  3.0f,  4.0f,  6.0f,
                                        -0.0f, -0.5f, -1.0f, -1.5f, -2.0f, -3.0f, -4.0f, -6.0f};

struct DecArgs {
    const __nv_bfloat16* x;   // [T, H]
    const float* logits;      // [T, E] or null (routing given in idx / wts)
    int32_t* idx;             // [T, k]
    float* wts;               // [T, k]
    int T, E, k, renorm, H, I;
    const uint8_t* gu_packed;   // [E, 2I, H/2]
    const float* gu_absmax;     // [E, 2I, H/64]
    const uint8_t* d_packed;    // [E, H, I/2]
    const float* d_absmax;      // [E, H, I/64]
    __nv_bfloat16* h;           // [T*k, I] scratch
    __nv_bfloat16* y;           // [T, H]
    struct DecPlan* gplan;      // routing / grouping published by gate_up CTA 0 for the down kernel
    int xs_off, xs_stride;      // gate_up: staged activations
    int gu_ring_off, gu_ns;     // gate_up: per-warp rings (offset, sub-stages)
    int dn_rt;                  // down: 8-row tiles per CTA
    int dn_yslot_off, dn_ring_off, dn_ns, dn_sub;   // down: y slots, per-warp rings, sub-stage bytes
};

// Routing and grouping of the <= 64 pairs.  A "slot" is one expert with up to
// 8 of its pairs (tokens ascending); an expert with more pairs (only possible
// with caller-given routing that repeats an expert within a token) takes
// several slots.
struct __align__(16) DecPlan {
    int n_slots;
    int warp_reps[2];
    int pe[DK_MAXP];
    float pw[DK_MAXP];
    int tslot[DK_MAXP];
    int rep_rank[DK_MAXP];
    int slot_e[DK_MAXP];
    int slot_n[DK_MAXP];
    int slot_pair[DK_MAXP][8];
    int slot_tok[DK_MAXP][8];   // token of slot_pair
};

constexpr uint32_t DK_PLAN_OFF = DK_LUT_BYTES;
constexpr uint32_t DK_FIXED = DK_PLAN_OFF + ((sizeof(DecPlan) + 127) / 128) * 128;

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// cp.async.wait_group takes an immediate: at most n of this thread's groups pending.
__device__ __forceinline__ void cp_async_wait_pending(int n) {
#define DK_WAIT_CASE(N) \
    case N: asm volatile("cp.async.wait_group " #N ";" ::: "memory"); break;
    switch (n) {
        DK_WAIT_CASE(0) DK_WAIT_CASE(1) DK_WAIT_CASE(2) DK_WAIT_CASE(3) DK_WAIT_CASE(4) DK_WAIT_CASE(5)
        DK_WAIT_CASE(6) DK_WAIT_CASE(7) DK_WAIT_CASE(8) DK_WAIT_CASE(9) DK_WAIT_CASE(10) DK_WAIT_CASE(11)
        DK_WAIT_CASE(12) DK_WAIT_CASE(13)
        default: asm volatile("cp.async.wait_group 14;" ::: "memory"); break;
    }
#undef DK_WAIT_CASE
}

template <int CB>
__device__ __forceinline__ float dec_table(int q) {
    return CB == 0 ? c_code[0][q] : c_e2m1[q];
}

// Entry for byte v: bf16x2 {value(high nibble), value(low nibble)} (low half =
// the element that comes first), stored at v*128 + lane*4 for every lane.
template <int CB>
__device__ __forceinline__ void build_lut(uint8_t* lut) {
    const float cv = dec_table<CB>(threadIdx.x & 15);   // lane q (and q+16) holds code value q
#pragma unroll
    for (int k = 0; k < 256 * 8 / DK_THREADS; ++k) {
        const int i = threadIdx.x + k * DK_THREADS, v = i >> 3, q = i & 7;
        const float hi = __shfl_sync(0xffffffffu, cv, v >> 4), lo = __shfl_sync(0xffffffffu, cv, v & 15);
        const uint32_t val = pack_bf16x2(hi, lo);
        *reinterpret_cast<uint4*>(lut + v * 128 + q * 16) = make_uint4(val, val, val, val);
    }
}

// One permute builds (byte << 8) | lane*8 (byte 0 <- lane8.byte0, byte 1 <-
// word.byte[i], bytes 2, 3 <- 0); halved, it is byte*128 + lane*4.
__device__ __forceinline__ uint32_t lut_lookup(const uint8_t* lut, uint32_t word, uint32_t lane8, uint32_t sel) {
    return *reinterpret_cast<const uint32_t*>(lut + (prmt(word, lane8, sel) >> 1));
}

__device__ __forceinline__ void mma_16816(float d[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// Up to 4 consecutive 64-element blocks of an 8-row weight tile against up to 8
// activation rows, accumulated as acc += absmax[block] * (block dot product).
// Lane (g = lane/4, c = lane%4) reads bytes [8c, 8c+8) of each block of weight
// row g (elements 16c..16c+15) and elements 16c..16c+15 of each block of
// activation row g (xrow).  Rows g past the slot's tokens may read any valid
// row: MMA rows are independent and those results are never stored.  MMA m of a block takes elements 16c+4m..16c+4m+3 from every lane:
// the same permutation of k on both operands, so D[g][n] is the block's dot
// product; d[0], d[1] = activation row g against weight rows 2c and 2c+1.  The
// MMAs are issued m-major over the blocks: consecutive MMAs are independent,
// so their latencies overlap.
template <int NB>
__device__ __forceinline__ void mma_batch(const uint8_t* wrow, const uint8_t* xrow, const float* a0, const float* a1,
                                          uint32_t lane8, const uint8_t* lut, float& acc0, float& acc1) {
    uint2 w[NB];
    uint4 xa[NB][2];
#pragma unroll
    for (int j = 0; j < NB; ++j) {
        w[j] = *reinterpret_cast<const uint2*>(wrow + j * 32);
        xa[j][0] = *reinterpret_cast<const uint4*>(xrow + j * 128);
        xa[j][1] = *reinterpret_cast<const uint4*>(xrow + j * 128 + 16);
    }
    float d[NB][4];
#pragma unroll
    for (int j = 0; j < NB; ++j) d[j][0] = d[j][1] = d[j][2] = d[j][3] = 0.0f;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const uint32_t bi = (2 * m) & 3;
        uint32_t b0[NB], b1[NB];
#pragma unroll
        for (int j = 0; j < NB; ++j) {
            const uint32_t word = (m < 2) ? w[j].x : w[j].y;
            b0[j] = lut_lookup(lut, word, lane8, 0x5504u | (bi << 4));
            b1[j] = lut_lookup(lut, word, lane8, 0x5504u | ((bi + 1) << 4));
        }
#pragma unroll
        for (int j = 0; j < NB; ++j) {
            const uint32_t x0 = (m < 2) ? (m == 0 ? xa[j][0].x : xa[j][0].z) : (m == 2 ? xa[j][1].x : xa[j][1].z);
            const uint32_t x1 = (m < 2) ? (m == 0 ? xa[j][0].y : xa[j][0].w) : (m == 2 ? xa[j][1].y : xa[j][1].w);
            mma_16816(d[j], x0, x1, b0[j], b1[j]);
        }
    }
#pragma unroll
    for (int j = 0; j < NB; ++j) {
        acc0 = fmaf(a0[j], d[j][0], acc0);
        acc1 = fmaf(a1[j], d[j][1], acc1);
    }
}

// nb (<= 8) consecutive blocks: batches of 4, then the remainder one block at a time.
__device__ __forceinline__ void mma_blocks(int nb, const uint8_t* wrow, const uint8_t* xrow, const float* a0,
                                           const float* a1, uint32_t lane8, const uint8_t* lut, float& acc0,
                                           float& acc1) {
    int j = 0;
    for (; j + 4 <= nb; j += 4)
        mma_batch<4>(wrow + j * 32, xrow + j * 128, a0 + j, a1 + j, lane8, lut, acc0, acc1);
    for (; j < nb; ++j) mma_batch<1>(wrow + j * 32, xrow + j * 128, a0 + j, a1 + j, lane8, lut, acc0, acc1);
}

// Routing (one warp per token, from logits; or the given routing) and the
// slots.  Inputs are read through L2 (ld.global.cg): the down kernel runs this
// before its dependency wait.  store: write topk_idx / topk_w.
__device__ void dec_build_plan(DecPlan& pl, const DecArgs& a, bool store) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int k = a.k, E = a.E, T = a.T, P = T * k;
    if (a.logits) {
        if (warp < T) {
            const int t = warp;
            int e;
            float p;
            route_token_warp(a.logits + (int64_t)t * E, E, k, a.renorm, lane, &e, &p);
            if (lane < k) {
                pl.pe[t * k + lane] = e;
                pl.pw[t * k + lane] = p;
                if (store) {
                    a.idx[t * k + lane] = e;
                    a.wts[t * k + lane] = p;
                }
            }
        }
    } else {
        for (int p = tid; p < P; p += blockDim.x) {
            pl.pe[p] = __ldcg(a.idx + p);
            pl.pw[p] = __ldcg(a.wts + p);
        }
    }
    __syncthreads();
    int e = -1, ts = 0, cnt = 0;
    bool rep = false;
    if (tid < P) {
        e = pl.pe[tid];
        if (e >= 0 && e < E) {
            for (int q = 0; q < P; ++q)
                if (pl.pe[q] == e) {
                    ts += (q < tid);
                    ++cnt;
                }
            rep = (ts & 7) == 0;
        } else {
            e = -1;
        }
    }
    const unsigned bal = __ballot_sync(0xffffffffu, rep);
    if (lane == 0 && warp < 2) pl.warp_reps[warp] = __popc(bal);
    int r = __popc(bal & ((1u << lane) - 1u));
    __syncthreads();
    if (warp == 1) r += pl.warp_reps[0];
    if (tid < P) {
        pl.rep_rank[tid] = rep ? r : -1;
        pl.tslot[tid] = ts;
    }
    if (tid == 0) pl.n_slots = pl.warp_reps[0] + pl.warp_reps[1];
    __syncthreads();
    if (tid < P && e >= 0) {
        int rq = tid;
        for (int q = 0; q <= tid; ++q)
            if (pl.pe[q] == e && pl.tslot[q] == (ts & ~7)) {
                rq = q;
                break;
            }
        const int s = pl.rep_rank[rq];
        pl.slot_pair[s][ts & 7] = tid;
        pl.slot_tok[s][ts & 7] = tid / k;
        if (rep) {
            pl.slot_e[s] = e;
            pl.slot_n[s] = min(8, cnt - ts);
        }
    }
    __syncthreads();
}

// Copies one sub-stage: blocks [kb0, kb0 + nb) (nb <= DK_KC) of the 8 weight
// rows grow(0..7) of K elements and their absmax.  Lane l takes row l/4 and
// every 4th 16-byte chunk of it; absmax goes as 16-byte chunks when aligned,
// else as 4-byte copies.
template <typename RowFn>
__device__ __forceinline__ void copy_sub(uint32_t st, int K, int kb0, int nb, const uint8_t* packed,
                                         const float* absmax, int lane, RowFn grow) {
    const int r = lane >> 2, part = lane & 3, kbr = K / 64;
    const size_t gr = grow(r);
    const uint8_t* src = packed + gr * (size_t)(K / 2) + kb0 * 32;
    for (int q = part; q < 2 * nb; q += 4) cp_async16(st + r * DK_SUB_RS + q * 16, src + q * 16);
    const float* asrc = absmax + gr * (size_t)kbr + kb0;
    const uint32_t adst = st + DK_SUB_ABS + r * DK_SUB_ASW * 4;
    if ((kbr & 3) == 0 && (kb0 & 3) == 0 && (nb & 3) == 0) {
        for (int q = part; q < nb / 4; q += 4) cp_async16(adst + q * 16, asrc + q * 4);
    } else {
        for (int q = part; q < nb; q += 4) cp_async_4(adst + q * 4, asrc + q, 4);
    }
}

// ------------------------------------------------------------------ gate_up
// h[p, f] = silu(x_t . W_gate,e[f]) * (x_t . W_up,e[f]) for every routed pair
// p = (t, j).  Item = (slot, 4 features): its 8-row tile holds gate rows
// f0..f0+3 at tile rows 0, 2, 4, 6 and up rows at 1, 3, 5, 7, so after the MMA
// each lane holds G and U of one feature for one token.  Items go round-robin
// to all warps of the grid.
template <int CB>
__global__ void __launch_bounds__(DK_THREADS, 2) dec_gateup_kernel(DecArgs a) {
    extern __shared__ __align__(128) uint8_t dsm[];
    DecPlan& pl = *reinterpret_cast<DecPlan*>(dsm + DK_PLAN_OFF);
    build_lut<CB>(dsm);
    griddep_wait();
    dec_build_plan(pl, a, a.logits != nullptr && blockIdx.x == 0);
    if (blockIdx.x == 0) {   // publish the plan for the down kernel
        const int* src = reinterpret_cast<const int*>(&pl);
        int* dst = reinterpret_cast<int*>(a.gplan);
        for (int i = threadIdx.x; i < (int)(sizeof(DecPlan) / 4); i += DK_THREADS) dst[i] = src[i];
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H, I = a.I, KB = H / 64, FT = I / 4;
    // activations of the T tokens
    const uint32_t xs = smem_u32(dsm + a.xs_off);
    for (int i = tid; i < a.T * (H / 8); i += DK_THREADS) {
        const int t = i / (H / 8), q = i - t * (H / 8);
        cp_async16(xs + t * a.xs_stride + q * 16, a.x + (size_t)t * H + q * 8);
    }
    cp_async_wait_all();
    __syncthreads();
    griddep_launch_dependents();

    const int N = pl.n_slots * FT, W = gridDim.x * DK_WARPS, gw = blockIdx.x * DK_WARPS + warp;
    const int nsub = (KB + DK_KC - 1) / DK_KC;
    const int n_items = gw < N ? (N - gw + W - 1) / W : 0;
    const int total = n_items * nsub;   // this warp's sub-stages
    const int ns = a.gu_ns;
    const uint32_t ring = smem_u32(dsm + a.gu_ring_off) + warp * ns * DK_SUB_A;
    const uint8_t* ring_p = dsm + a.gu_ring_off + warp * ns * DK_SUB_A;

    // issue cursor: item m, sub-stage sb
    int im = 0, isb = 0;
    auto issue = [&]() {
        const int it = gw + im * W, s = it / FT, f0 = (it - s * FT) * 4;
        const size_t r0 = (size_t)pl.slot_e[s] * 2 * I + f0;
        const int kb0 = isb * DK_KC;
        copy_sub(ring + ((im * nsub + isb) % ns) * DK_SUB_A, H, kb0, min(DK_KC, KB - kb0), a.gu_packed, a.gu_absmax,
                 lane, [&](int r) { return r0 + (r & 1) * I + (r >> 1); });
        if (++isb == nsub) {
            isb = 0;
            ++im;
        }
    };
    for (int j = 0; j < ns - 1; ++j) {
        if (j < total) issue();
        cp_async_commit();
    }
    const int g = lane >> 2, c = lane & 3;
    const uint32_t lane8 = (uint32_t)lane * 8u;
    const float mu = CB == 0 ? 1.0f : (1.0f / 6.0f);
    float acc0 = 0.0f, acc1 = 0.0f;
    int s = 0, f0 = 0, sb = 0, m = 0;
    const uint8_t* xrow = dsm;
    for (int i = 0; i < total; ++i) {
        if (sb == 0) {   // new item
            const int it = gw + m * W;
            s = it / FT;
            f0 = (it - s * FT) * 4;
            xrow = dsm + a.xs_off + pl.slot_tok[s][g < pl.slot_n[s] ? g : 0] * a.xs_stride + c * 32;
        }
        cp_async_wait_pending(ns - 2);
        __syncwarp();   // this warp's copies of sub-stage i landed; sub-stage i-1 consumed by every lane
        if (i + ns - 1 < total) issue();
        cp_async_commit();
        const uint8_t* st = ring_p + (i % ns) * DK_SUB_A;
        const int kb0 = sb * DK_KC, nb = min(DK_KC, KB - kb0);
        const uint8_t* wrow = st + g * DK_SUB_RS + c * 8;
        const float* ag = reinterpret_cast<const float*>(st + DK_SUB_ABS) + (2 * c) * DK_SUB_ASW;
        const float* au = ag + DK_SUB_ASW;
        mma_blocks(nb, wrow, xrow + kb0 * 128, ag, au, lane8, dsm, acc0, acc1);
        if (++sb == nsub) {   // item done: SwiGLU, store h
            if (g < pl.slot_n[s]) {
                const float G = acc0 * mu, U = acc1 * mu;
                const float hv = G / (1.0f + expf(-G)) * U;
                a.h[(int64_t)pl.slot_pair[s][g] * I + f0 + c] = __float2bfloat16_rn(hv);
            }
            acc0 = acc1 = 0.0f;
            sb = 0;
            ++m;
        }
    }
    cp_async_wait_all();
}

// --------------------------------------------------------------------- down
// y[t, r] = sum_j w[t,j] * (W_down,e_j[r] . h[t*k+j]), summed over j in slot order.
// A CTA owns dn_rt 8-row tiles of the output for all routed experts.  Item =
// (slot, tile); items go round-robin to the CTA's warps, and an item's
// sub-stages also carry the h rows of the slot's pairs.  Weighted per-pair rows
// go to shared memory and are summed per token in j order.
template <int CB>
__global__ void __launch_bounds__(DK_THREADS, 1) dec_down_kernel(DecArgs a) {
    extern __shared__ __align__(128) uint8_t dsm[];
    DecPlan& pl = *reinterpret_cast<DecPlan*>(dsm + DK_PLAN_OFF);
    build_lut<CB>(dsm);
    griddep_launch_dependents();   // the next layer's gate_up may build its table meanwhile
    griddep_wait();                // routing plan and h come from gate_up
    {
        const int* src = reinterpret_cast<const int*>(a.gplan);
        int* dst = reinterpret_cast<int*>(&pl);
        for (int i = threadIdx.x; i < (int)(sizeof(DecPlan) / 4); i += DK_THREADS) dst[i] = __ldcg(src + i);
    }
    __syncthreads();

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H, I = a.I, KB = I / 64, RW = a.dn_rt * 8;
    const int r0 = blockIdx.x * RW;
    const int nt = min(RW, H - r0) / 8;   // 8-row tiles in this CTA
    float* yslot = reinterpret_cast<float*>(dsm + a.dn_yslot_off);   // [P][RW]
    const int N = pl.n_slots * nt;
    const int nsub = (KB + DK_KC - 1) / DK_KC;
    const int n_items = warp < N ? (N - warp + DK_WARPS - 1) / DK_WARPS : 0;
    const int total = n_items * nsub;
    const int ns = a.dn_ns, sub = a.dn_sub;
    const uint32_t ring = smem_u32(dsm + a.dn_ring_off) + warp * ns * sub;
    const uint8_t* ring_p = dsm + a.dn_ring_off + warp * ns * sub;

    int im = 0, isb = 0;
    auto issue = [&]() {
        const int it = warp + im * DK_WARPS, s = it / nt, t = it - s * nt;
        const size_t rb = (size_t)pl.slot_e[s] * H + r0 + t * 8;
        const int kb0 = isb * DK_KC, nb = min(DK_KC, KB - kb0);
        const uint32_t st = ring + ((im * nsub + isb) % ns) * sub;
        copy_sub(st, I, kb0, nb, a.d_packed, a.d_absmax, lane, [&](int r) { return rb + r; });
        const int n = pl.slot_n[s];
        for (int gg = 0; gg < n; ++gg) {   // h rows of the slot's pairs, these blocks
            const __nv_bfloat16* hsrc = a.h + (size_t)pl.slot_pair[s][gg] * I + kb0 * 64;
            for (int q = lane; q < nb * 8; q += 32) cp_async16(st + DK_SUB_A + gg * DK_SUB_AS + q * 16, hsrc + q * 8);
        }
        if (++isb == nsub) {
            isb = 0;
            ++im;
        }
    };
    for (int j = 0; j < ns - 1; ++j) {
        if (j < total) issue();
        cp_async_commit();
    }
    const int g = lane >> 2, c = lane & 3;
    const uint32_t lane8 = (uint32_t)lane * 8u;
    const float mu = CB == 0 ? 1.0f : (1.0f / 6.0f);
    float acc0 = 0.0f, acc1 = 0.0f;
    int s = 0, t = 0, sb = 0, m = 0, n = 0;
    for (int i = 0; i < total; ++i) {
        if (sb == 0) {
            const int it = warp + m * DK_WARPS;
            s = it / nt;
            t = it - s * nt;
            n = pl.slot_n[s];
        }
        cp_async_wait_pending(ns - 2);
        __syncwarp();
        if (i + ns - 1 < total) issue();
        cp_async_commit();
        const uint8_t* st = ring_p + (i % ns) * sub;
        const int kb0 = sb * DK_KC, nb = min(DK_KC, KB - kb0);
        const uint8_t* wrow = st + g * DK_SUB_RS + c * 8;
        const float* a0p = reinterpret_cast<const float*>(st + DK_SUB_ABS) + (2 * c) * DK_SUB_ASW;
        const float* a1p = a0p + DK_SUB_ASW;
        const uint8_t* hrow = st + DK_SUB_A + (g < n ? g : 0) * DK_SUB_AS + c * 32;
        mma_blocks(nb, wrow, hrow, a0p, a1p, lane8, dsm, acc0, acc1);
        if (++sb == nsub) {   // item done: weight by the routing weight, stash per pair
            if (g < n) {
                const int p = pl.slot_pair[s][g];
                yslot[p * RW + t * 8 + 2 * c] = pl.pw[p] * (acc0 * mu);
                yslot[p * RW + t * 8 + 2 * c + 1] = pl.pw[p] * (acc1 * mu);
            }
            acc0 = acc1 = 0.0f;
            sb = 0;
            ++m;
        }
    }
    cp_async_wait_all();
    __syncthreads();
    const int rows = nt * 8;
    for (int i = tid; i < a.T * rows; i += DK_THREADS) {
        const int tt = i / rows, rl = i - tt * rows;
        float v = 0.0f;
        for (int j = 0; j < a.k; ++j) {
            const int p = tt * a.k + j;
            const int e = pl.pe[p];
            if (e >= 0 && e < a.E) v += yslot[p * RW + rl];
        }
        a.y[(int64_t)tt * H + r0 + rl] = __float2bfloat16_rn(v);
    }
}

// ------------------------------------------------------------------- host side

static int sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

static int xs_stride(int H) { return (H * 2 / 16) % 2 ? H * 2 : H * 2 + 16; }
static int align128(int v) { return (v + 127) / 128 * 128; }
// h rows per down sub-stage: a slot holds at most T pairs when the routing comes
// from logits (distinct experts per token), at most 8 with caller-given routing.
static int down_arows(int64_t T, int k, bool routed) { return routed ? (int)T : (int)std::min<int64_t>(8, T * k); }

struct DecLaunch {
    int gu_grid, gu_smem, dn_grid, dn_smem;
};

// Shared-memory plan of both kernels: gate_up two CTAs per SM (up to 112 KB
// each) while a 3-deep per-warp ring fits, else one; down one CTA per SM.
static bool decode_plan_launch(int H, int I, int64_t T, int k, bool routed, DecArgs* a, DecLaunch* l) {
    if (T < 1 || T > 8 || T * k > DK_MAXP) return false;
    const int nsm = sm_count();
    const int sub_g = DK_SUB_A;   // already a multiple of 128
    const int xs_off = (int)DK_FIXED, xst = xs_stride(H);
    const int gu_ring = align128(xs_off + (int)T * xst);
    int gu_ns = std::min(DK_NS_MAX, (112 * 1024 - gu_ring) / (DK_WARPS * sub_g));
    int gu_grid = 2 * nsm;
    if (gu_ns < 3) {
        gu_ns = std::min(DK_NS_MAX, (220 * 1024 - gu_ring) / (DK_WARPS * sub_g));
        gu_grid = nsm;
    }
    const int rt = std::max(1, std::min(DK_DN_MAX_RT, (H / 8 + nsm - 1) / nsm));
    const int yslot_off = (int)DK_FIXED;
    const int dn_ring = align128(yslot_off + (int)(T * k) * rt * 8 * 4);
    const int sub_d = align128(DK_SUB_A + down_arows(T, k, routed) * DK_SUB_AS);
    const int dn_ns = std::min(DK_NS_MAX, (220 * 1024 - dn_ring) / (DK_WARPS * sub_d));
    if (gu_ns < 2 || dn_ns < 2) return false;
    if (a) {
        a->xs_off = xs_off;
        a->xs_stride = xst;
        a->gu_ring_off = gu_ring;
        a->gu_ns = gu_ns;
        a->dn_rt = rt;
        a->dn_yslot_off = yslot_off;
        a->dn_ring_off = dn_ring;
        a->dn_ns = dn_ns;
        a->dn_sub = sub_d;
    }
    if (l) {
        l->gu_grid = gu_grid;
        l->gu_smem = gu_ring + DK_WARPS * gu_ns * sub_g;
        l->dn_grid = (H / 8 + rt - 1) / rt;
        l->dn_smem = dn_ring + DK_WARPS * dn_ns * sub_d;
    }
    return true;
}

bool decode_supported(int H, int I, int64_t T, int k, bool routed) {
    return decode_plan_launch(H, I, T, k, routed, nullptr, nullptr);
}

template <typename K>
static cudaError_t launch_pdl(K kernel, int grid, int smem, cudaStream_t st, const DecArgs& a) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(DK_THREADS);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, a);
}

template <int CB>
static cudaError_t decode_impl(const DecArgs& a, const DecLaunch& l, cudaStream_t st) {
    cudaError_t err =
        cudaFuncSetAttribute(dec_gateup_kernel<CB>, cudaFuncAttributeMaxDynamicSharedMemorySize, l.gu_smem);
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(dec_down_kernel<CB>, cudaFuncAttributeMaxDynamicSharedMemorySize, l.dn_smem);
    // the whole unified L1 / shared array as shared memory, so two gate_up CTAs fit per SM
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(dec_gateup_kernel<CB>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                   (int)cudaSharedmemCarveoutMaxShared);
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(dec_down_kernel<CB>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                   (int)cudaSharedmemCarveoutMaxShared);
    if (err != cudaSuccess) return err;
    timing_begin(KK_DECODE_GATEUP, st);
    err = launch_pdl(dec_gateup_kernel<CB>, l.gu_grid, l.gu_smem, st, a);
    timing_end(KK_DECODE_GATEUP, st);
    count_launch();
    if (err != cudaSuccess) return err;
    timing_begin(KK_DECODE_DOWN, st);
    err = launch_pdl(dec_down_kernel<CB>, l.dn_grid, l.dn_smem, st, a);
    timing_end(KK_DECODE_DOWN, st);
    count_launch();
    return err;
}

size_t decode_plan_bytes() { return sizeof(DecPlan); }

cudaError_t launch_decode_forward(int codebook, int E, int H, int I, int k, int renorm, int64_t T,
                                  const __nv_bfloat16* x, const float* logits, int32_t* idx, float* w,
                                  const uint8_t* gu_packed, const float* gu_absmax, const uint8_t* d_packed,
                                  const float* d_absmax, __nv_bfloat16* h_scratch, void* plan_scratch,
                                  __nv_bfloat16* y, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    DecArgs a;
    DecLaunch l;
    if (E > DK_MAXE || !decode_plan_launch(H, I, T, k, logits != nullptr, &a, &l)) return cudaErrorInvalidValue;
    a.x = x;
    a.logits = logits;
    a.idx = idx;
    a.wts = w;
    a.T = (int)T;
    a.E = E;
    a.k = k;
    a.renorm = renorm;
    a.H = H;
    a.I = I;
    a.gu_packed = gu_packed;
    a.gu_absmax = gu_absmax;
    a.d_packed = d_packed;
    a.d_absmax = d_absmax;
    a.h = h_scratch;
    a.gplan = static_cast<DecPlan*>(plan_scratch);
    a.y = y;
    return codebook == 0 ? decode_impl<0>(a, l, st) : decode_impl<1>(a, l, st);
}

}  // namespace e4b
