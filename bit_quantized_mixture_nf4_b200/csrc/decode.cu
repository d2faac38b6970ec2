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
//  * Work unit = one weight tile of 8 (gate_up) or 16 (down) rows over all of K,
//    for one routed expert.  A CTA's units stream through a ring of shared-memory
//    stages with a classic multistage cp.async pipeline: each warp copies whole
//    rows as 16-byte chunks NS-1 units ahead, then cp.async.wait_group and one
//    CTA barrier per unit.  There are no spin-waits, and the padded stage rows
//    make the reads bank-conflict free.  gate_up runs two CTAs per SM.
//  * Weight decode: a 256-entry table maps a packed byte (two 4-bit codes) to a
//    bf16x2 pair of code values.  The table is replicated for each of the 32
//    lanes, so a warp's 32 lookups hit 32 distinct banks.  The lookup address
//    takes one byte permute and one shift.
//  * Math: mma.sync m16n8k16 (bf16 in, fp32 out).  The weight tile is the B
//    operand (8 rows); the activation rows (the tokens routed to the expert,
//    <= 8) are the A operand.  Each MMA covers 16 elements of one 64-element
//    block, so the block's absmax multiplies the fp32 block partial once
//    (w = code * absmax, code in bf16, scale applied in fp32).  The warps of a
//    CTA split K; their partials are summed in shared memory in warp order.
#include "e4b_internal.h"

namespace e4b {

constexpr int DK_THREADS = 256;
constexpr int DK_WARPS = DK_THREADS / 32;
constexpr int DK_MAXP = 64;                 // T * k <= 8 * 8 routed pairs
constexpr int DK_MAXE = 256;
constexpr int DK_NS_MAX = 16;               // ring stages
constexpr int DK_DN_MAX_ROWS = 64;          // down: output rows per CTA
constexpr uint32_t DK_LUT_BYTES = 32768;    // 256 byte values x 32 lanes x 4 B

// e2m1 values (sign in bit 3).  The FP4 codebook is these divided by 6; the
// division is applied to the fp32 result, so the table is exact in bf16.
static __constant__ float c_e2m1[16] = {0.0f,  0.5f,  1.0f,  1.5f,  2.0f,  3.0f,  4.0f,  6.0f,
                                        -0.0f, -0.5f, -1.0f, -1.5f, -2.0f, -3.0f, -4.0f, -6.0f};

// Layout of one ring stage: R packed weight rows, R absmax rows, then (down
// only) up to 8 activation rows.
struct StageLayout {
    int rows;        // R
    int rowstride;   // bytes between weight rows: K/2 + pad, (rowstride/4) = 8 (mod 32)
    int absoff;      // offset of the absmax rows
    int absw;        // words between absmax rows: odd, 2 (mod 4) or 4 (mod 8)
    int aoff;        // offset of the activation rows
    int astride;     // bytes between activation rows: (astride/16) odd
    int bytes;       // stage size (multiple of 128)
    int ns;          // stages in the ring
    int ring_off;    // offset of the ring in dynamic shared memory
    int smem;        // dynamic shared memory of the kernel
};

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
    int dn_rows;                // down: output rows per CTA (multiple of 16, <= 64)
    int xs_off, xs_stride;      // gate_up: staged activations
    StageLayout gl, dl;         // gate_up / down stage layouts
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
constexpr uint32_t DK_PART_OFF = DK_PLAN_OFF + ((sizeof(DecPlan) + 127) / 128) * 128;
constexpr uint32_t DK_PART_BYTES = 2 * DK_WARPS * 32 * 8;                  // [2][WARPS][32] float2
constexpr uint32_t DK_YSLOT_OFF = DK_PART_OFF + DK_PART_BYTES;
constexpr uint32_t DK_YSLOT_BYTES = DK_MAXP * DK_DN_MAX_ROWS * 4;           // down: [MAXP][rows] fp32

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
// activation row g (xrow; null: the row is zero).  MMA m of a block takes elements 16c+4m..16c+4m+3 from every lane:
// the same permutation of k on both operands, so D[g][n] is the block's dot
// product; d[0], d[1] = activation row g against weight rows 2c and 2c+1.  The
// MMAs are issued m-major over the blocks: consecutive MMAs are independent,
// so their latencies overlap.
__device__ __forceinline__ void mma_batch4(int nb, const uint8_t* wrow, const uint8_t* xrow, const float* a0,
                                           const float* a1, uint32_t lane8, const uint8_t* lut, float& acc0,
                                           float& acc1) {
    uint2 w[4];
    uint4 xa[4][2];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        w[j] = (j < nb) ? *reinterpret_cast<const uint2*>(wrow + j * 32) : make_uint2(0u, 0u);
        if (xrow && j < nb) {
            xa[j][0] = *reinterpret_cast<const uint4*>(xrow + j * 128);
            xa[j][1] = *reinterpret_cast<const uint4*>(xrow + j * 128 + 16);
        } else {
            xa[j][0] = xa[j][1] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    float d[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) d[j][0] = d[j][1] = d[j][2] = d[j][3] = 0.0f;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const uint32_t bi = (2 * m) & 3;
        uint32_t b0[4], b1[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t word = (m < 2) ? w[j].x : w[j].y;
            b0[j] = lut_lookup(lut, word, lane8, 0x5504u | (bi << 4));
            b1[j] = lut_lookup(lut, word, lane8, 0x5504u | ((bi + 1) << 4));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (j < nb) {
                const uint32_t x0 = (m < 2) ? (m == 0 ? xa[j][0].x : xa[j][0].z) : (m == 2 ? xa[j][1].x : xa[j][1].z);
                const uint32_t x1 = (m < 2) ? (m == 0 ? xa[j][0].y : xa[j][0].w) : (m == 2 ? xa[j][1].y : xa[j][1].w);
                mma_16816(d[j], x0, x1, b0[j], b1[j]);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (j < nb) {
            acc0 = fmaf(a0[j], d[j][0], acc0);
            acc1 = fmaf(a1[j], d[j][1], acc1);
        }
    }
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

// Copies weight rows grow(0) .. grow(R-1) (K/2 bytes each) and their absmax
// rows (K/64 floats each) into a stage: warp w copies rows w, w+8, ... as 16-byte
// chunks (absmax rows whose length is not a multiple of 16 bytes go as 4-byte
// copies).
template <typename RowFn>
__device__ __forceinline__ void stage_rows(uint32_t st, const StageLayout& L, int K, const uint8_t* packed,
                                           const float* absmax, RowFn grow) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rc = K / 32, kb = K / 64;   // 16-byte chunks per row, absmax per row
    for (int r = warp; r < L.rows; r += DK_WARPS) {
        const size_t gr = grow(r);
        const uint8_t* src = packed + gr * (size_t)(K / 2);
        const uint32_t dst = st + r * L.rowstride;
        for (int q = lane; q < rc; q += 32) cp_async16(dst + q * 16, src + q * 16);
        const float* asrc = absmax + gr * (size_t)kb;
        const uint32_t adst = st + L.absoff + r * L.absw * 4;
        if (kb % 4 == 0) {
            for (int q = lane; q < kb / 4; q += 32) cp_async16(adst + q * 16, asrc + q * 4);
        } else {
            for (int q = lane; q < kb; q += 32) cp_async_4(adst + q * 4, asrc + q, 4);
        }
    }
}

// ------------------------------------------------------------------ gate_up
// h[p, f] = silu(x_t . W_gate,e[f]) * (x_t . W_up,e[f]) for every routed pair
// p = (t, j).  Unit = (slot, 4 features): its 8-row tile holds gate rows
// f0..f0+3 at tile rows 0, 2, 4, 6 and up rows at 1, 3, 5, 7, so after the MMA
// each lane holds G and U of one feature for one token.  Units are split evenly
// over the CTAs (one per SM); the 8 warps split K.
template <int CB>
__global__ void __launch_bounds__(DK_THREADS, 2) dec_gateup_kernel(DecArgs a) {
    extern __shared__ __align__(128) uint8_t dsm[];
    DecPlan& pl = *reinterpret_cast<DecPlan*>(dsm + DK_PLAN_OFF);
    float2* part = reinterpret_cast<float2*>(dsm + DK_PART_OFF);   // [2][WARPS][32]
    const StageLayout& L = a.gl;
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
    const int N = pl.n_slots * FT;
    const int u0 = (int)((int64_t)blockIdx.x * N / gridDim.x);
    const int n_units = (int)((int64_t)(blockIdx.x + 1) * N / gridDim.x) - u0;
    const uint32_t ring = smem_u32(dsm + L.ring_off), xs = smem_u32(dsm + a.xs_off);

    // activations of the T tokens (first copy group, with unit 0)
    for (int i = tid; i < a.T * (H / 8); i += DK_THREADS) {
        const int t = i / (H / 8), q = i - t * (H / 8);
        cp_async16(xs + t * a.xs_stride + q * 16, a.x + (size_t)t * H + q * 8);
    }
    griddep_launch_dependents();
    // Unit cursors (slot, first feature, ring stage) advance by one unit at a
    // time: no divisions in the loop.
    struct Cur {
        int s, f0, stg;
    };
    const int ns = L.ns;
    auto advance = [&](Cur& q) {
        q.f0 += 4;
        if (q.f0 == I) {
            q.f0 = 0;
            ++q.s;
        }
        q.stg = (q.stg + 1 == ns) ? 0 : q.stg + 1;
    };
    const Cur first = {u0 / FT, (u0 % FT) * 4, 0};
    auto issue = [&](const Cur& q) {
        const size_t r0 = (size_t)pl.slot_e[q.s] * 2 * I + q.f0;
        stage_rows(ring + q.stg * L.bytes, L, H, a.gu_packed, a.gu_absmax,
                   [&](int r) { return r0 + (r & 1) * I + (r >> 1); });
    };
    Cur iq = first;
    for (int j = 0; j < ns - 1; ++j) {
        if (j < n_units) {
            issue(iq);
            advance(iq);
        }
        cp_async_commit();
    }

    const int g = lane >> 2, c = lane & 3;
    const int kb0 = warp * KB / DK_WARPS, kb1 = (warp + 1) * KB / DK_WARPS;
    const uint32_t lane8 = (uint32_t)lane * 8u;
    const float mu = CB == 0 ? 1.0f : (1.0f / 6.0f);
    // Sum of the 8 warps' partials of a unit (one warp does it), SwiGLU, store h.
    auto reduce = [&](const Cur& q, int parity) {
        const float2* pb = part + (size_t)parity * DK_WARPS * 32;
        float G = 0.0f, U = 0.0f;
#pragma unroll
        for (int w = 0; w < DK_WARPS; ++w) {
            const float2 v = pb[w * 32 + lane];
            G += v.x;
            U += v.y;
        }
        if (g < pl.slot_n[q.s]) {
            G *= mu;
            U *= mu;
            const float hv = G / (1.0f + expf(-G)) * U;
            a.h[(int64_t)pl.slot_pair[q.s][g] * I + q.f0 + c] = __float2bfloat16_rn(hv);
        }
    };
    Cur cq = first, prev = first;
    for (int i = 0; i < n_units; ++i) {
        cp_async_wait_pending(ns - 2);
        __syncthreads();   // unit i's stage complete; unit i-1's partials written, its stage free
        if (i > 0 && warp == (i & (DK_WARPS - 1))) reduce(prev, (i - 1) & 1);
        if (i + ns - 1 < n_units) {
            issue(iq);
            advance(iq);
        }
        cp_async_commit();

        const uint8_t* xrow =   // activation row of token slot g (staged x)
            (g < pl.slot_n[cq.s]) ? dsm + a.xs_off + pl.slot_tok[cq.s][g] * a.xs_stride + c * 32 : nullptr;
        const uint8_t* st = dsm + L.ring_off + cq.stg * L.bytes;
        const uint8_t* wrow = st + g * L.rowstride + c * 8;
        const float* ag = reinterpret_cast<const float*>(st + L.absoff) + (2 * c) * L.absw;
        const float* au = ag + L.absw;
        float acc0 = 0.0f, acc1 = 0.0f;
        for (int kb = kb0; kb < kb1; kb += 4)
            mma_batch4(min(4, kb1 - kb), wrow + kb * 32, xrow ? xrow + kb * 128 : nullptr, ag + kb, au + kb, lane8,
                       dsm, acc0, acc1);
        part[((size_t)(i & 1) * DK_WARPS + warp) * 32 + lane] = make_float2(acc0, acc1);
        prev = cq;
        advance(cq);
    }
    cp_async_wait_all();
    __syncthreads();
    if (n_units > 0 && warp == (n_units & (DK_WARPS - 1))) reduce(prev, (n_units - 1) & 1);
}

// --------------------------------------------------------------------- down
// y[t, r] = sum_j w[t,j] * (W_down,e_j[r] . h[t*k+j]), summed over j in slot order.
// A CTA owns dn_rows output rows for all routed experts.  Unit = (slot, 16
// rows): warps 0-3 take rows 0-7 and warps 4-7 rows 8-15, each a quarter of K.
// The unit's stage also holds the h rows of the slot's pairs.  Weighted
// per-pair rows go to shared memory and are summed per token in j order.
template <int CB>
__global__ void __launch_bounds__(DK_THREADS, 2) dec_down_kernel(DecArgs a) {
    extern __shared__ __align__(128) uint8_t dsm[];
    DecPlan& pl = *reinterpret_cast<DecPlan*>(dsm + DK_PLAN_OFF);
    float2* part = reinterpret_cast<float2*>(dsm + DK_PART_OFF);   // [2][WARPS][32]
    float* yslot = reinterpret_cast<float*>(dsm + DK_YSLOT_OFF);    // [MAXP][dn_rows]
    const StageLayout& L = a.dl;
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
    const int H = a.H, I = a.I, KB = I / 64, RW = a.dn_rows;
    const int r0 = blockIdx.x * RW;
    const int ng = min(RW, H - r0) / 16;   // 16-row groups in this CTA
    const int n_units = pl.n_slots * ng;
    const uint32_t ring = smem_u32(dsm + L.ring_off);
    struct Cur {
        int s, tg, stg;
    };
    const int ns = L.ns;
    auto advance = [&](Cur& q) {
        if (++q.tg == ng) {
            q.tg = 0;
            ++q.s;
        }
        q.stg = (q.stg + 1 == ns) ? 0 : q.stg + 1;
    };
    auto issue = [&](const Cur& q) {   // weight rows and the h rows of the unit's pairs
        const size_t rb = (size_t)pl.slot_e[q.s] * H + r0 + q.tg * 16;
        const uint32_t st = ring + q.stg * L.bytes;
        stage_rows(st, L, I, a.d_packed, a.d_absmax, [&](int r) { return rb + r; });
        const int n = pl.slot_n[q.s], rc = I / 8;
        for (int gg = warp; gg < n; gg += DK_WARPS) {
            const __nv_bfloat16* src = a.h + (size_t)pl.slot_pair[q.s][gg] * I;
            for (int qq = lane; qq < rc; qq += 32) cp_async16(st + L.aoff + gg * L.astride + qq * 16, src + qq * 8);
        }
    };
    Cur iq = {0, 0, 0};
    for (int j = 0; j < ns - 1; ++j) {
        if (j < n_units) {
            issue(iq);
            advance(iq);
        }
        cp_async_commit();
    }

    const int g = lane >> 2, c = lane & 3, t8 = warp >> 2, kp = warp & 3;
    const int kb0 = kp * KB / 4, kb1 = (kp + 1) * KB / 4;
    const uint32_t lane8 = (uint32_t)lane * 8u;
    const float mu = CB == 0 ? 1.0f : (1.0f / 6.0f);
    // Sum of the 4 K-part partials of each of a unit's two 8-row tiles (two warps), weight, stash.
    auto reduce = [&](const Cur& q, int parity) {
        const int t = (warp & 1);
        const float2* pb = part + (size_t)parity * DK_WARPS * 32;
        float v0 = 0.0f, v1 = 0.0f;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            const float2 v = pb[(t * 4 + qq) * 32 + lane];
            v0 += v.x;
            v1 += v.y;
        }
        if (g < pl.slot_n[q.s]) {
            const int p = pl.slot_pair[q.s][g];
            yslot[p * RW + q.tg * 16 + t * 8 + 2 * c] = pl.pw[p] * (v0 * mu);
            yslot[p * RW + q.tg * 16 + t * 8 + 2 * c + 1] = pl.pw[p] * (v1 * mu);
        }
    };
    Cur cq = {0, 0, 0}, prev = cq;
    for (int i = 0; i < n_units; ++i) {
        cp_async_wait_pending(ns - 2);
        __syncthreads();
        if (i > 0 && (warp >> 1) == (i & 3)) reduce(prev, (i - 1) & 1);
        if (i + ns - 1 < n_units) {
            issue(iq);
            advance(iq);
        }
        cp_async_commit();

        const int n = pl.slot_n[cq.s];
        const uint8_t* st = dsm + L.ring_off + cq.stg * L.bytes;
        const uint8_t* wrow = st + (t8 * 8 + g) * L.rowstride + c * 8;
        const float* a0p = reinterpret_cast<const float*>(st + L.absoff) + (t8 * 8 + 2 * c) * L.absw;
        const float* a1p = a0p + L.absw;
        const uint8_t* hrow = (g < n) ? st + L.aoff + g * L.astride + c * 32 : nullptr;
        float acc0 = 0.0f, acc1 = 0.0f;
        for (int kb = kb0; kb < kb1; kb += 4)
            mma_batch4(min(4, kb1 - kb), wrow + kb * 32, hrow ? hrow + kb * 128 : nullptr, a0p + kb, a1p + kb, lane8,
                       dsm, acc0, acc1);
        part[((size_t)(i & 1) * DK_WARPS + warp) * 32 + lane] = make_float2(acc0, acc1);
        prev = cq;
        advance(cq);
    }
    cp_async_wait_all();
    __syncthreads();
    if (n_units > 0 && (warp >> 1) == (n_units & 3)) reduce(prev, (n_units - 1) & 1);
    __syncthreads();
    const int rows = ng * 16;
    for (int i = tid; i < a.T * rows; i += DK_THREADS) {
        const int t = i / rows, rl = i - t * rows;
        float v = 0.0f;
        for (int j = 0; j < a.k; ++j) {
            const int p = t * a.k + j;
            const int e = pl.pe[p];
            if (e >= 0 && e < a.E) v += yslot[p * RW + rl];
        }
        a.y[(int64_t)t * H + r0 + rl] = __float2bfloat16_rn(v);
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

// Stage layout for R weight rows of K elements (+ a_rows activation rows).
// Weight rows are padded so that (row stride / 4) = 8 (mod 32): the lanes of
// 4 consecutive rows then read distinct banks.  Absmax rows use a word stride
// that is odd, 2 (mod 4) or 4 (mod 8) (the last keeps rows 16-byte aligned for
// 16-byte copies): the lanes reading rows 2c (or 2c+1), c = 0..3, hit distinct
// banks.  Activation rows use a 16-byte stride count that is odd.
static StageLayout stage_layout(int K, int R, int a_rows, int ring_off, int ring_budget) {
    StageLayout L{};
    const int rowb = K / 2, kb = K / 64;
    L.rows = R;
    L.rowstride = rowb + 4 * (((8 - rowb / 4) % 32 + 32) % 32);
    L.absoff = R * L.rowstride;
    L.absw = (kb % 4 != 0) ? kb : (kb % 8 == 0 ? kb + 4 : kb);   // odd, 2 or 4 (mod 8): distinct banks
    L.aoff = (L.absoff + R * L.absw * 4 + 15) / 16 * 16;
    L.astride = (K * 2 / 16) % 2 ? K * 2 : K * 2 + 16;
    L.bytes = (L.aoff + a_rows * L.astride + 127) / 128 * 128;
    L.ns = std::max(2, std::min(DK_NS_MAX, ring_budget / L.bytes));
    L.ring_off = ring_off;
    L.smem = ring_off + L.ns * L.bytes;
    return L;
}

static int xs_stride(int H) { return (H * 2 / 16) % 2 ? H * 2 : H * 2 + 16; }

// h rows per down stage: a slot holds at most T pairs when the routing comes from
// logits (distinct experts per token), at most 8 with caller-given routing.
static int down_arows(int64_t T, int k, bool routed) { return routed ? (int)T : (int)std::min<int64_t>(8, T * k); }

bool decode_supported(int H, int I, int64_t T, int k, bool routed) {
    if (T < 1 || T > 8 || T * k > DK_MAXP) return false;
    const int gu = (int)DK_PART_OFF + (int)DK_PART_BYTES + (int)T * xs_stride(H) + 128;
    return stage_layout(H, 8, 0, gu, 0).smem <= 200 * 1024 &&
           stage_layout(I, 16, down_arows(T, k, routed), (int)(DK_YSLOT_OFF + DK_YSLOT_BYTES), 0).smem <= 200 * 1024;
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
static cudaError_t decode_impl(const DecArgs& a, cudaStream_t st) {
    cudaError_t err = cudaFuncSetAttribute(dec_gateup_kernel<CB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           a.gl.smem);
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(dec_down_kernel<CB>, cudaFuncAttributeMaxDynamicSharedMemorySize, a.dl.smem);
    // the whole unified L1 / shared array as shared memory, so two CTAs fit per SM
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(dec_gateup_kernel<CB>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                   (int)cudaSharedmemCarveoutMaxShared);
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(dec_down_kernel<CB>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                   (int)cudaSharedmemCarveoutMaxShared);
    if (err != cudaSuccess) return err;
    timing_begin(KK_DECODE_GATEUP, st);
    err = launch_pdl(dec_gateup_kernel<CB>, 2 * sm_count(), a.gl.smem, st, a);
    timing_end(KK_DECODE_GATEUP, st);
    count_launch();
    if (err != cudaSuccess) return err;
    timing_begin(KK_DECODE_DOWN, st);
    err = launch_pdl(dec_down_kernel<CB>, (a.H + a.dn_rows - 1) / a.dn_rows, a.dl.smem, st, a);
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
    if (E > DK_MAXE || !decode_supported(H, I, T, k, logits != nullptr)) return cudaErrorInvalidValue;
    DecArgs a;
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
    const int nsm = sm_count();
    // down: 16-row groups spread over about one CTA per SM (H is a multiple of 64)
    const int groups = H / 16;
    a.dn_rows = 16 * std::min(DK_DN_MAX_ROWS / 16, (groups + nsm - 1) / nsm);
    a.xs_off = (int)(DK_PART_OFF + DK_PART_BYTES);
    a.xs_stride = xs_stride(H);
    const int gu_ring = (a.xs_off + (int)T * a.xs_stride + 127) / 128 * 128;
    // gate_up: two CTAs per SM, each up to 112 KB (an SM has 228 KB, 1 KB per CTA
    // reserved); down: one CTA per SM with up to about 150 KB.
    a.gl = stage_layout(H, 8, 0, gu_ring, 112 * 1024 - gu_ring);
    const int dn_fixed = (int)(DK_YSLOT_OFF + DK_YSLOT_BYTES);
    a.dl = stage_layout(I, 16, down_arows(T, k, logits != nullptr), dn_fixed, 150 * 1024 - dn_fixed);
    return codebook == 0 ? decode_impl<0>(a, st) : decode_impl<1>(a, st);
}

}  // namespace e4b
