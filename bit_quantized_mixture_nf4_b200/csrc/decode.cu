// Small-batch (T <= 8) forward.  At a handful of tokens the expert layer is a
// weight-streaming GEMV: each touched expert's packed weights are read once, so
// HBM bandwidth bounds it, and at ~20 MB per layer the fixed latencies (routing,
// the first bytes, the gate_up -> down dependency) weigh as much as the stream.
//
// This is the decode fast path of the expert-layer pages ("experts4bit-qlora"
// 0.4.0 description, section "Inference": single-token forward over the token's
// top-k experts, a 4-bit GEMV that reads the packed codes directly), designed for
// B200:
//
//  * Two kernels, gate_up then down (a programmatic dependent), one CTA per SM.
//  * Both kernels route the tokens themselves (one warp per token, from fp32
//    logits, the routing of the grouped path) and build the same "slots": the
//    distinct routed experts, ascending.  Every slot is computed for all T tokens
//    (the MMA's 8 columns); a token's weight for a slot is 0 when it does not
//    route there, and only routed tokens' h rows are stored and read.
//  * gate_up: unit = (slot, 8 features) = 8 gate + 8 up rows over all of K = H;
//    the units are split evenly over the CTAs and round-robin over the 8 warps.
//    While it streams its own weights it asks L2 for the down weights of the
//    down CTA with the same index.
//  * down: CTA c owns whole output tiles (16 rows of H); unit = (tile, slot),
//    tile-major.  It starts streaming its weights before it waits for gate_up
//    (only the h rows wait); each warp keeps its own sums per output tile and
//    the warps' sums are added in warp order, so the result is deterministic and
//    no CTA waits for another.
//  * Each warp computes whole units: it streams a unit's 16 rows (codes and
//    absmax; for down also the h rows) in chunks of KC 64-element blocks from
//    global memory with 16-byte cp.async into its own ring of shared-memory
//    stages, lanes running along a row so every copy instruction reads whole
//    128-byte lines, and computes on the stage copied D-1 chunks earlier.
//  * Math: mma.sync m16n8k16 (bf16 in, fp32 out) with the WEIGHTS as the A
//    operand (16 rows) and the <= 8 tokens' activations as B (8 columns): one MMA
//    covers 256 weights.  K is permuted identically on both operands so a lane
//    reads 8 contiguous bytes of a row per 64-element block.  Codes become bf16
//    code values through a 256-entry byte -> bf16x2 table replicated per lane
//    (conflict-free).  Every MMA starts from zero (no accumulation chain between
//    MMAs); a block's partial sums are added and scaled by its absmax in fp32.
#include <mutex>

#include "e4b_internal.h"

namespace e4b {

constexpr int DV_WARPS = 8;
constexpr int DV_THREADS = 32 * DV_WARPS;
constexpr int DV_MAXT = 8, DV_MAXP = 64, DV_MAXS = 64, DV_MAXE = 256;
constexpr int DV_MAXTL = 8;        // output tiles per down CTA
constexpr int DV_MAXD = 8;         // ring stages per warp
constexpr int DV_LUT_WORDS = 256 * 32;   // byte value x lane
static_assert(DV_MAXE <= DV_THREADS, "one thread per expert in the slot builder");

struct DvArgs {
    const __nv_bfloat16* x;   // [T, H]
    const float* logits;      // [T, E] or null (routing given in idx / wts)
    int32_t* idx;             // [T, k]
    float* wts;               // [T, k]
    int T, E, k, renorm, H, I;
    const uint8_t* gu_packed;   // [E, 2I, H/2]
    const float* gu_absmax;     // [E, 2I, H/64]
    const uint8_t* d_packed;    // [E, H, I/2]
    const float* d_absmax;      // [E, H, I/64]
    __nv_bfloat16* h;         // [n_slots, T, I] (scratch)
    __nv_bfloat16* y;         // [T, H]
    int kc;                   // 64-element blocks per streamed chunk of a unit
    int depth;                // ring stages per warp
    int stage_bytes;          // one stage: codes [16][rs] + absmax [16][ss] (+ h [T][hrs])
    int rs, ss, hrs;          // row strides of a stage (bytes, floats, bytes)
    int ring_off;             // shared-memory offset of the rings
};

// The slots: distinct routed experts, ascending, with each token's summed
// routing weight (0 where the token does not route there).
struct __align__(16) DvSlots {
    int n_slots;
    int pad[3];
    int slot_e[DV_MAXS];
    unsigned slot_tmask[DV_MAXS];
    float slot_w[DV_MAXS][DV_MAXT];
};

// Dynamic shared memory of both kernels: the slots, the routing pairs and
// bookkeeping; then
// (gate_up) the activations or (down) the warps' tile sums; then the warps'
// rings.
constexpr int DV_SLOTS_OFF = 0, DV_PAIRS_OFF = 3072, DV_MISC_OFF = 3584;
constexpr int DV_HDR = 4096;
static_assert(sizeof(DvSlots) <= DV_PAIRS_OFF, "slots");
static_assert(DV_PAIRS_OFF + 2 * DV_MAXP * 4 <= DV_MISC_OFF, "pairs");
struct DvMisc {
    int warp_cnt[DV_WARPS];   // slot builder: routed experts per warp
};
static_assert(sizeof(DvMisc) <= DV_HDR - DV_MISC_OFF, "misc");

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

__device__ __forceinline__ uint32_t bfe15(uint32_t v) {   // (v >> 1) & 0x7fff
    uint32_t d;
    asm("bfe.u32 %0, %1, 1, 15;" : "=r"(d) : "r"(v));
    return d;
}

__device__ __forceinline__ void dv_cp16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void dv_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void dv_wait_groups() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// At most n (0 <= n < DV_MAXD) of this thread's copy groups still pending.
__device__ __forceinline__ void dv_wait_pending(int n) {
    switch (n) {
        case 0: dv_wait_groups<0>(); break;
        case 1: dv_wait_groups<1>(); break;
        case 2: dv_wait_groups<2>(); break;
        case 3: dv_wait_groups<3>(); break;
        case 4: dv_wait_groups<4>(); break;
        case 5: dv_wait_groups<5>(); break;
        case 6: dv_wait_groups<6>(); break;
        default: dv_wait_groups<7>(); break;
    }
}
// Request the 128-byte line at p into L2 (no data returned to the thread).
__device__ __forceinline__ void dv_prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// D = A * B with zero accumulator input (every MMA independent of the others).
__device__ __forceinline__ void mma_16816_z(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// Code value q of the codebook (NF4: the NormalFloat values; FP4: the e2m1
// values, divided by 6 in fp32 after the dot product so they stay exact in bf16).
template <int CB>
__device__ __forceinline__ float dv_code(int q) {
    if (CB == 1) {
        const float m = (q & 7) < 4 ? 0.5f * (q & 7) : ((q & 7) == 4 ? 2.0f : ((q & 7) == 5 ? 3.0f : ((q & 7) == 6 ? 4.0f : 6.0f)));
        return (q & 8) ? -m : m;
    }
    float v;
    switch (q & 15) {
        case 0: v = -1.0f; break;
        case 1: v = -0.6961928009986877f; break;
        case 2: v = -0.5250730514526367f; break;
        case 3: v = -0.39491748809814453f; break;
        case 4: v = -0.28444138169288635f; break;
        case 5: v = -0.18477343022823334f; break;
        case 6: v = -0.09105003625154495f; break;
        case 7: v = 0.0f; break;
        case 8: v = 0.07958029955625534f; break;
        case 9: v = 0.16093020141124725f; break;
        case 10: v = 0.24611230194568634f; break;
        case 11: v = 0.33791524171829224f; break;
        case 12: v = 0.44070982933044434f; break;
        case 13: v = 0.5626170039176941f; break;
        case 14: v = 0.7229568362236023f; break;
        default: v = 1.0f; break;
    }
    return v;
}

// Table entry of byte v for lane l at word v*32 + l: bf16x2 {value(high nibble),
// value(low nibble)} (low half = the element that comes first).  The 16 code
// values go through the small table cv first.  Ends with a block barrier.
template <int CB>
__device__ __forceinline__ void dv_build_lut(uint32_t* lut, float* cv) {
    if (threadIdx.x < 16) cv[threadIdx.x] = dv_code<CB>((int)threadIdx.x);
    __syncthreads();
    for (int i = threadIdx.x; i < 256 * 8; i += DV_THREADS) {
        const int v = i >> 3;
        const uint32_t val = pack_bf16x2(cv[v >> 4], cv[v & 15]);
        reinterpret_cast<uint4*>(lut)[i] = make_uint4(val, val, val, val);
    }
    __syncthreads();
}

// Four table lookups for the bytes of w: byte b's entry for this lane sits at
// byte offset b*128 + lane*4.  One byte permute builds two offsets at once
// ([lane8, b_i, lane8, b_j], lane8 = lane*8).
__device__ __forceinline__ void dv_lut4(const uint32_t* lut, uint32_t w, uint32_t lane8, uint32_t& v0, uint32_t& v1,
                                        uint32_t& v2, uint32_t& v3) {
    const uint8_t* base = reinterpret_cast<const uint8_t*>(lut);
    const uint32_t d01 = prmt(w, lane8, 0x1404u);
    const uint32_t d23 = prmt(w, lane8, 0x3424u);
    v0 = *reinterpret_cast<const uint32_t*>(base + bfe15(d01));
    v1 = *reinterpret_cast<const uint32_t*>(base + (d01 >> 17));
    v2 = *reinterpret_cast<const uint32_t*>(base + bfe15(d23));
    v3 = *reinterpret_cast<const uint32_t*>(base + (d23 >> 17));
}

// One 64-element block (column bl of the slot) of the 16 slot rows against the
// activation fragments of its two halves; h0 / h1: the half is in range.
// acc += absmax * (block dot products).
__device__ __forceinline__ void dv_block(const uint8_t* slot, const float* sabs, int rs, int nbs, int bl, bool h0,
                                         bool h1, uint4 x0, uint4 x1, const uint32_t* lut, uint32_t lane8, int g, int c,
                                         float acc[4]) {
    const uint2 wlo = *reinterpret_cast<const uint2*>(slot + g * rs + bl * 32 + c * 8);
    const uint2 whi = *reinterpret_cast<const uint2*>(slot + (g + 8) * rs + bl * 32 + c * 8);
    const float alo = sabs[g * nbs + bl], ahi = sabs[(g + 8) * nbs + bl];
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    if (h0) {
        uint32_t l0, l1, l2, l3, m0, m1, m2, m3;
        dv_lut4(lut, wlo.x, lane8, l0, l1, l2, l3);
        dv_lut4(lut, whi.x, lane8, m0, m1, m2, m3);
        float d0[4], d1[4];
        mma_16816_z(d0, l0, m0, l1, m1, x0.x, x0.y);
        mma_16816_z(d1, l2, m2, l3, m3, x0.z, x0.w);
#pragma unroll
        for (int j = 0; j < 4; ++j) s[j] += d0[j] + d1[j];
    }
    if (h1) {
        uint32_t l0, l1, l2, l3, m0, m1, m2, m3;
        dv_lut4(lut, wlo.y, lane8, l0, l1, l2, l3);
        dv_lut4(lut, whi.y, lane8, m0, m1, m2, m3);
        float d0[4], d1[4];
        mma_16816_z(d0, l0, m0, l1, m1, x1.x, x1.y);
        mma_16816_z(d1, l2, m2, l3, m3, x1.z, x1.w);
#pragma unroll
        for (int j = 0; j < 4; ++j) s[j] += d0[j] + d1[j];
    }
    acc[0] = fmaf(alo, s[0], acc[0]);
    acc[1] = fmaf(alo, s[1], acc[1]);
    acc[2] = fmaf(ahi, s[2], acc[2]);
    acc[3] = fmaf(ahi, s[3], acc[3]);
}

// First unit of CTA c when U units are split evenly over G CTAs (c * U < 2^31).
__device__ __forceinline__ int dv_lo(int c, int U, int G) { return c * U / G; }

// Stored row (within the stack) of row r of a unit.  gate_up unit u = (slot,
// 8 features): rows 0..7 the gate rows, 8..15 the up rows.  down unit u =
// (tile of 16 output rows, slot), tile-major over S slots.
__device__ __forceinline__ int64_t dv_gu_row(const DvSlots& sl, int I, int u, int r) {
    const int FT = I / 8, s = u / FT, f0 = (u - s * FT) * 8;
    return (int64_t)sl.slot_e[s] * 2 * I + (r < 8 ? f0 + r : I + f0 + r - 8);
}
__device__ __forceinline__ int64_t dv_dn_row(const DvSlots& sl, int H, int S, int u, int r) {
    const int tile = u / S, s = u - tile * S;
    return (int64_t)sl.slot_e[s] * H + tile * 16 + r;
}


// i / d for 0 <= i < 1024 and 1 <= d <= 64, with inv = ceil(65536 / d).
__device__ __forceinline__ int dv_div(int i, uint32_t inv) { return (int)(((uint32_t)i * inv) >> 16); }
__device__ __forceinline__ uint32_t dv_inv(int d) { return (65536u + (uint32_t)d - 1u) / (uint32_t)d; }

// One warp: cp.async copies of blocks [b0, b0 + nb) of a unit's 16 rows into the
// stage at shared address st: codes (row r at codes + row_of(r) * rb) into
// [16][rs] and absmax (absmax + row_of(r) * kb) into [16][ss].  Lanes run along
// a row, so each copy instruction reads whole 128-byte lines.
template <typename RowFn>
__device__ __forceinline__ void dv_copy_chunk(uint32_t st, int lane, int b0, int nb, const uint8_t* codes, int rb,
                                              const float* absmax, int kb, int rs, int ss, RowFn row_of) {
    const int cpr = 2 * nb;   // 16-byte units per row
    const uint32_t inv = dv_inv(cpr);
    for (int i = lane; i < 16 * cpr; i += 32) {
        const int r = dv_div(i, inv), j = i - r * cpr;
        dv_cp16(st + r * rs + j * 16, codes + row_of(r) * rb + b0 * 32 + j * 16);
    }
    const uint32_t sab = st + 16 * rs;
    if (((kb | b0 | nb) & 3) == 0) {   // 16-byte aligned absmax runs
        const int cpa = nb >> 2;
        const uint32_t inva = dv_inv(cpa);
        for (int i = lane; i < 16 * cpa; i += 32) {
            const int r = dv_div(i, inva), j = i - r * cpa;
            dv_cp16(sab + r * ss * 4 + j * 16, absmax + row_of(r) * kb + b0 + j * 4);
        }
    } else {
        const uint32_t inva = dv_inv(nb);
        for (int i = lane; i < 16 * nb; i += 32) {
            const int r = dv_div(i, inva), j = i - r * nb;
            cp_async_4(sab + (r * ss + j) * 4, absmax + row_of(r) * kb + b0 + j, 4);
        }
    }
}

// Chunk geometry of a kernel: kc blocks of 64 K per chunk (nc chunks per unit),
// ring of `depth` stages of stage_bytes per warp.
__device__ __forceinline__ int dv_chunk_blocks(int c, int kc, int kb) { return min(kc, kb - c * kc); }

// -------------------------------------------------------------------- routing
// The routing and the slots of the T tokens, computed identically by every CTA
// of both kernels (shared memory only; ends with a block barrier).  From
// logits: one warp per token (route_token_warp, the routing of the grouped
// path).  Given routing: the pairs are read from idx / wts.  Slots: the
// distinct routed experts in ascending order; a token's weight for a slot is
// the sum of its pairs' weights there, in pair order.
__device__ __forceinline__ void dv_plan(const DvArgs& a, uint8_t* dsm, bool write_out) {
    DvSlots& sl = *reinterpret_cast<DvSlots*>(dsm + DV_SLOTS_OFF);
    int* pe = reinterpret_cast<int*>(dsm + DV_PAIRS_OFF);
    float* pw = reinterpret_cast<float*>(dsm + DV_PAIRS_OFF + DV_MAXP * 4);
    DvMisc& misc = *reinterpret_cast<DvMisc*>(dsm + DV_MISC_OFF);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = a.T, E = a.E, k = a.k, P = T * k;
    if (a.logits) {
        if (warp < T) {
            int e;
            float p;
            route_token_warp(a.logits + (int64_t)warp * E, E, k, a.renorm, lane, &e, &p);
            if (lane < k) {
                pe[warp * k + lane] = e;
                pw[warp * k + lane] = p;
                if (write_out) {
                    a.idx[warp * k + lane] = e;
                    a.wts[warp * k + lane] = p;
                }
            }
        }
    } else if (tid < P) {
        pe[tid] = __ldcg(a.idx + tid);
        pw[tid] = __ldcg(a.wts + tid);
    }
    __syncthreads();
    // thread e marks the tokens routed to expert e
    const int e = tid;
    unsigned tm = 0u;
    if (e < E) {
        int t = 0, j = 0;
        for (int p = 0; p < P; ++p) {
            if (pe[p] == e) tm |= 1u << t;
            if (++j == k) {
                j = 0;
                ++t;
            }
        }
    }
    const unsigned bal = __ballot_sync(0xffffffffu, tm != 0u);
    if (lane == 0) misc.warp_cnt[warp] = __popc(bal);
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += misc.warp_cnt[w];
    if (tm) {
        const int s = base + __popc(bal & ((1u << lane) - 1u));
        sl.slot_e[s] = e;
        sl.slot_tmask[s] = tm;
        for (int t = 0; t < T; ++t) {
            float wsum = 0.0f;
            for (int j = 0; j < k; ++j)
                if (pe[t * k + j] == e) wsum += pw[t * k + j];
            sl.slot_w[s][t] = wsum;
        }
    }
    if (tid == DV_THREADS - 1) {
        int n = 0;
        for (int w = 0; w < DV_WARPS; ++w) n += misc.warp_cnt[w];
        sl.n_slots = n;
    }
    __syncthreads();
}

// The compute of one streamed chunk of KC blocks (all of them in range): the
// unit's 16 rows in the stage against the activation rows at act (row stride
// ars bytes, token g of the lane).
template <int KC>
__device__ __forceinline__ void dv_chunk(const uint8_t* st, const float* sabs, int rs, int ss, const uint8_t* act,
                                         bool gvalid, const uint32_t* lut, uint32_t lane8, int g, int q4,
                                         float acc[4]) {
#pragma unroll
    for (int bl = 0; bl < KC; ++bl) {
        const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
        const uint4 x0 = gvalid ? *reinterpret_cast<const uint4*>(act + bl * 128) : zero;
        const uint4 x1 = gvalid ? *reinterpret_cast<const uint4*>(act + bl * 128 + 16) : zero;
        dv_block(st, sabs, rs, ss, bl, true, true, x0, x1, lut, lane8, g, q4, acc);
    }
}
// A chunk of nb < KC blocks (the last of a unit whose K is not a multiple of KC).
__device__ __forceinline__ void dv_chunk_tail(int nb, const uint8_t* st, const float* sabs, int rs, int ss,
                                              const uint8_t* act, bool gvalid, const uint32_t* lut, uint32_t lane8,
                                              int g, int q4, float acc[4]) {
#pragma unroll 1
    for (int bl = 0; bl < nb; ++bl) {
        const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
        const uint4 x0 = gvalid ? *reinterpret_cast<const uint4*>(act + bl * 128) : zero;
        const uint4 x1 = gvalid ? *reinterpret_cast<const uint4*>(act + bl * 128 + 16) : zero;
        dv_block(st, sabs, rs, ss, bl, true, true, x0, x1, lut, lane8, g, q4, acc);
    }
}

// Code table and zeroed slot records (both kernels, before the wait on the
// preceding grid: shared memory only).
template <int CB>
__device__ __forceinline__ void dv_prologue(uint32_t* lut, float* cv, uint8_t* dsm) {
    DvSlots& sl = *reinterpret_cast<DvSlots*>(dsm + DV_SLOTS_OFF);
    const int tid = threadIdx.x;
    if (tid < DV_MAXS) sl.slot_tmask[tid] = 0u;
    dv_build_lut<CB>(lut, cv);   // ends with a barrier
}

// ------------------------------------------------------------------ gate_up
// h[s, t, f] = silu(x_t . W_gate,e[f]) * (x_t . W_up,e[f]) for every slot s
// (expert e) and every token t.  Unit = (slot, 8 features): a warp computes a
// whole unit (all of K = H), streaming it in chunks of KC blocks through its
// ring.
template <int CB, int KC>
__global__ void __launch_bounds__(DV_THREADS, 1) dv_gateup_kernel(DvArgs a) {
    __shared__ __align__(16) uint32_t lut[DV_LUT_WORDS];
    __shared__ float cv[16];
    extern __shared__ __align__(128) uint8_t dsm[];
    DvSlots& sl = *reinterpret_cast<DvSlots*>(dsm + DV_SLOTS_OFF);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int I = a.I, H = a.H, T = a.T, G = gridDim.x;

    dv_prologue<CB>(lut, cv, dsm);
    griddep_wait();               // everything before this kernel (inputs included) is complete
    griddep_launch_dependents();  // the down kernel may take the SMs this grid leaves

    // activations x [T][H] into shared memory (rows of H*2 + 16 bytes), one copy group
    uint8_t* xs = dsm + DV_HDR;
    const int xrs = H * 2 + 16;
    {
        const int cpr = H / 8;
        for (int i = tid; i < T * cpr; i += DV_THREADS) {
            const int t = i / cpr, j = i - t * cpr;
            dv_cp16(smem_u32(xs) + t * xrs + j * 16, a.x + (int64_t)t * H + j * 8);
        }
        dv_commit();
    }
    dv_plan(a, dsm, blockIdx.x == 0);

    const int FT = I / 8, KB = H / 64, RB = H / 2, S = sl.n_slots, NC = (KB + KC - 1) / KC;
    const int U = S * FT;
    const int u0 = dv_lo(blockIdx.x, U, G), u1 = dv_lo(blockIdx.x + 1, U, G);
    const int nu = u1 - u0 > warp ? (u1 - u0 - warp + DV_WARPS - 1) / DV_WARPS : 0;   // this warp's units
    const int L = nu * NC;                                                           // its chunk stream
    const int D = a.depth;
    const uint32_t ring = smem_u32(dsm + a.ring_off) + warp * D * a.stage_bytes;
    int ij = 0, ic = 0;   // issue cursor: unit index j of this warp, chunk c
    auto issue = [&]() {
        if (ij < nu) {
            const int u = u0 + warp + ij * DV_WARPS, s = u / FT, f0 = (u - s * FT) * 8;
            const int64_t gb = (int64_t)sl.slot_e[s] * 2 * I + f0, ub = gb + I;
            const int i = ij * NC + ic;
            dv_copy_chunk(ring + (i % D) * a.stage_bytes, lane, ic * KC, dv_chunk_blocks(ic, KC, KB), a.gu_packed, RB,
                          a.gu_absmax, KB, a.rs, a.ss, [&](int r) { return r < 8 ? gb + r : ub + r - 8; });
            if (++ic == NC) {
                ic = 0;
                ++ij;
            }
        }
        dv_commit();
    };
    for (int i = 0; i < D - 1; ++i) issue();
    // The weights of the down CTA of this index, requested into L2 while this
    // grid streams its own: output tiles [t0, t1) of every slot.
    if (S > 0) {
        const int NT = H / 16, t0 = dv_lo(blockIdx.x, NT, G), t1 = dv_lo(blockIdx.x + 1, NT, G);
        const int lcode = 16 * (I / 2) / 128, labs = (16 * (I / 64) * 4 + 127) / 128, lpu = lcode + labs;
        const int n = (t1 - t0) * S * lpu;
        for (int i = tid; i < n; i += DV_THREADS) {
            const int uu = i / lpu, l = i - uu * lpu, tile = t0 + uu / S, s = uu - (uu / S) * S;
            const int64_t row0 = (int64_t)sl.slot_e[s] * H + tile * 16;
            if (l < lcode) dv_prefetch_l2(a.d_packed + row0 * (I / 2) + l * 128);
            else dv_prefetch_l2(reinterpret_cast<const uint8_t*>(a.d_absmax + row0 * (I / 64)) + (l - lcode) * 128);
        }
    }
    dv_wait_pending(D - 1);   // this thread's part of the activations has landed ...
    __syncthreads();          // ... and everyone's

    const int g = lane >> 2, q4 = lane & 3;
    const bool gvalid = g < T;
    const uint32_t lane8 = (uint32_t)lane * 8u;
    const float mu = CB == 0 ? 1.0f : (1.0f / 6.0f);
    const uint8_t* xrow = xs + g * xrs + 32 * q4;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int cj = 0, cc = 0;   // compute cursor
    for (int i = 0; i < L; ++i) {
        __syncwarp();               // every lane is done with the stage chunk i-1 used
        issue();
        dv_wait_pending(D - 1);     // this lane's copies of chunk i landed
        __syncwarp();               // ... and every lane's
        const uint8_t* st = dsm + a.ring_off + (warp * D + (i % D)) * a.stage_bytes;
        const float* sabs = reinterpret_cast<const float*>(st + 16 * a.rs);
        const int nb = dv_chunk_blocks(cc, KC, KB);
        if (nb == KC) dv_chunk<KC>(st, sabs, a.rs, a.ss, xrow + cc * KC * 128, gvalid, lut, lane8, g, q4, acc);
        else dv_chunk_tail(nb, st, sabs, a.rs, a.ss, xrow + cc * KC * 128, gvalid, lut, lane8, g, q4, acc);
        if (++cc == NC) {   // unit done: SwiGLU, store h
            const int u = u0 + warp + cj * DV_WARPS, s = u / FT, f = (u - s * FT) * 8 + g;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int t = 2 * q4 + jj;
                if (t < T && ((sl.slot_tmask[s] >> t) & 1u)) {   // h of the tokens routed here
                    const float gv = acc[jj] * mu, uv = acc[2 + jj] * mu;
                    const float hv = gv / (1.0f + expf(-gv)) * uv;
                    a.h[((int64_t)s * T + t) * I + f] = __float2bfloat16_rn(hv);
                }
            }
            acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
            cc = 0;
            ++cj;
        }
    }
    dv_wait_groups<0>();
}

// --------------------------------------------------------------------- down
// y[t, r] = sum over slots s of w[s, t] * (W_down,e_s[r] . h[s, t]).  CTA c owns
// whole output tiles of 16 rows, [c NT / G, (c+1) NT / G) of NT = H / 16; a unit
// is (tile, slot), tile-major, and a warp computes whole units (all of K = I).
// The kernel repeats the routing itself and starts its weight stream before it
// waits for gate_up; only the h rows wait.
template <int CB, int KC>
__global__ void __launch_bounds__(DV_THREADS, 1) dv_down_kernel(DvArgs a) {
    __shared__ __align__(16) uint32_t lut[DV_LUT_WORDS];
    __shared__ float cv[16];
    extern __shared__ __align__(128) uint8_t dsm[];
    DvSlots& sl = *reinterpret_cast<DvSlots*>(dsm + DV_SLOTS_OFF);
    float* yw = reinterpret_cast<float*>(dsm + DV_HDR);   // [warp][ntl][16][8] per-warp tile sums
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int I = a.I, H = a.H, T = a.T, KBI = I / 64, RB = I / 2, G = gridDim.x;
    const int NT = H / 16, t0 = dv_lo(blockIdx.x, NT, G), t1 = dv_lo(blockIdx.x + 1, NT, G);
    const int ntl = (NT + G - 1) / G;   // output tiles per CTA at most

    for (int i = tid; i < DV_WARPS * ntl * 128; i += DV_THREADS) yw[i] = 0.0f;
    dv_prologue<CB>(lut, cv, dsm);
    // This grid starts once every gate_up CTA has passed its own wait, so the
    // inputs of the layer are complete here; the routing is recomputed.
    dv_plan(a, dsm, false);
    const int S = sl.n_slots;
    const int n = (t1 - t0) * S, u0 = t0 * S;   // this CTA's units [u0, u0 + n)
    const int NC = (KBI + KC - 1) / KC;
    const int nu = n > warp ? (n - warp + DV_WARPS - 1) / DV_WARPS : 0;
    const int L = nu * NC;
    const int D = a.depth;
    const uint32_t ring = smem_u32(dsm + a.ring_off) + warp * D * a.stage_bytes;
    const int h_off = 16 * a.rs + 16 * a.ss * 4;
    // chunk i of this warp's stream: weights (part & 1) and h rows (part & 2)
    auto copy = [&](int i, int part) {
        const int ij = i / NC, ic = i - ij * NC;
        const int u = u0 + warp + ij * DV_WARPS, s = u % S;
        const int b0 = ic * KC, nb = dv_chunk_blocks(ic, KC, KBI);
        const uint32_t st = ring + (i % D) * a.stage_bytes;
        if (part & 1) {
            const int64_t rb0 = dv_dn_row(sl, H, S, u, 0);
            dv_copy_chunk(st, lane, b0, nb, a.d_packed, RB, a.d_absmax, KBI, a.rs, a.ss,
                          [&](int r) { return rb0 + r; });
        }
        if (part & 2) {   // the h rows of the tokens routed to this slot (the others stay unread)
            const int cpr = nb * 8;   // 16-byte units of a token's h row in this chunk
            const uint32_t inv = dv_inv(cpr);
            const unsigned tms = sl.slot_tmask[s];
            const __nv_bfloat16* src = a.h + (int64_t)s * T * I + b0 * 64;
            for (int q = lane; q < T * cpr; q += 32) {
                const int t = dv_div(q, inv), j = q - t * cpr;
                if ((tms >> t) & 1u) dv_cp16(st + h_off + t * a.hrs + j * 16, src + (int64_t)t * I + j * 8);
            }
        }
    };
    const int npre = min(D - 1, L);
    for (int i = 0; i < D - 1; ++i) {   // weights of the first chunks: inputs, ready now
        if (i < npre) copy(i, 1);
        dv_commit();
    }
    griddep_wait();   // gate_up is complete: h is visible
    griddep_launch_dependents();
    for (int i = 0; i < D - 1; ++i) {
        if (i < npre) copy(i, 2);
        dv_commit();
    }

    if (S == 0) {   // no valid expert anywhere: y = 0 on this CTA's tiles
        for (int i = tid; i < (t1 - t0) * 16 * T; i += DV_THREADS) {
            const int t = i / ((t1 - t0) * 16), r = i - t * (t1 - t0) * 16;
            a.y[(int64_t)t * H + t0 * 16 + r] = __float2bfloat16_rn(0.0f);
        }
        dv_wait_groups<0>();
        return;
    }
    const int g = lane >> 2, q4 = lane & 3;
    const bool gvalid = g < T;
    const uint32_t lane8 = (uint32_t)lane * 8u;
    const float mu = CB == 0 ? 1.0f : (1.0f / 6.0f);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int cj = 0, cc = 0;
    for (int i = 0; i < L; ++i) {
        __syncwarp();
        if (i + D - 1 < L) copy(i + D - 1, 3);
        dv_commit();
        dv_wait_pending(D - 1);
        __syncwarp();
        const uint8_t* st = dsm + a.ring_off + (warp * D + (i % D)) * a.stage_bytes;
        const float* sabs = reinterpret_cast<const float*>(st + 16 * a.rs);
        const uint8_t* hrow = st + h_off + g * a.hrs + 32 * q4;
        const int nb = dv_chunk_blocks(cc, KC, KBI);
        const int su = (u0 + warp + cj * DV_WARPS) % S;
        const bool hv = gvalid && ((sl.slot_tmask[su] >> g) & 1u);   // token g routed to this slot
        if (nb == KC) dv_chunk<KC>(st, sabs, a.rs, a.ss, hrow, hv, lut, lane8, g, q4, acc);
        else dv_chunk_tail(nb, st, sabs, a.rs, a.ss, hrow, hv, lut, lane8, g, q4, acc);
        if (++cc == NC) {   // unit done: weight by the routing and add into this warp's tile sums
            const int u = u0 + warp + cj * DV_WARPS, tile = u / S, s = u - tile * S, tl = tile - t0;
            const unsigned tms = sl.slot_tmask[s];
            float* yb = yw + (warp * ntl + tl) * 128;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int t = 2 * q4 + jj;
                if (t < T && ((tms >> t) & 1u)) {
                    const float wgt = sl.slot_w[s][t] * mu;
                    yb[g * 8 + t] += wgt * acc[jj];
                    yb[(g + 8) * 8 + t] += wgt * acc[2 + jj];
                }
            }
            acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
            cc = 0;
            ++cj;
        }
    }
    dv_wait_groups<0>();
    __syncthreads();
    // this CTA's tiles: the warps' sums added in warp order
    for (int i = tid; i < (t1 - t0) * 16 * T; i += DV_THREADS) {
        const int tl = i / (16 * T), rem = i - tl * 16 * T, t = rem >> 4, r = rem & 15;
        float v = 0.0f;
        for (int w = 0; w < DV_WARPS; ++w) v += yw[(w * ntl + tl) * 128 + r * 8 + t];
        a.y[(int64_t)t * H + (t0 + tl) * 16 + r] = __float2bfloat16_rn(v);
    }
}

// ------------------------------------------------------------------- host side

struct DvGeom {
    int kc, depth, stage_bytes, rs, ss, hrs, ring_off, smem;
};
struct DvCfg {
    int G;
    DvGeom a, b;
};

constexpr int DV_SMEM_MAX = 227 * 1024 - DV_LUT_WORDS * 4;   // dynamic shared memory per CTA

// Stage geometry for chunks of kc blocks: code rows of an odd number of 32-byte
// units keep the warp's 8-byte row reads at two wavefronts; an absmax stride of
// 4 mod 8 floats and h rows of an odd number of 16-byte units keep those reads
// conflict-free.  fixed: shared bytes before the rings.
static bool dv_geom(int K, int hrows, int fixed, DvGeom* g) {
    const int kb = K / 64;
    for (int kc = std::min(kb, 8); kc >= 1; kc = kc > 2 ? kc / 2 : kc - 1) {
        DvGeom t{};
        t.kc = kc;
        t.rs = kc * 32 + ((kc & 1) ? 0 : 32);
        t.ss = 4;
        while (t.ss < kc || t.ss % 8 != 4) t.ss += 4;
        t.hrs = kc * 128 + 16;
        t.stage_bytes = (16 * t.rs + 16 * t.ss * 4 + hrows * t.hrs + 127) / 128 * 128;
        t.ring_off = (fixed + 127) / 128 * 128;
        t.depth = std::min(DV_MAXD, (DV_SMEM_MAX - t.ring_off) / (DV_WARPS * t.stage_bytes));
        if (t.depth >= 3 || (t.depth >= 2 && kc == 1)) {
            t.smem = t.ring_off + t.depth * DV_WARPS * t.stage_bytes;
            *g = t;
            return true;
        }
    }
    return false;
}

static bool dv_config(int E, int H, int I, int64_t T, int k, DvCfg* c) {
    if (T < 1 || T > DV_MAXT || T * k > DV_MAXP || E > DV_MAXE) return false;
    if (H % 64 || I % 64 || H > 8192) return false;
    DvCfg d{};
    d.G = num_sms();
    if ((H / 16 + d.G - 1) / d.G > DV_MAXTL) return false;   // output tiles per down CTA
    // gate_up: the activations [T][H*2 + 16] after the header; down: the warps' tile sums
    if (!dv_geom(H, 0, DV_HDR + (int)T * (H * 2 + 16), &d.a)) return false;
    const int ntl = (H / 16 + d.G - 1) / d.G;
    if (!dv_geom(I, (int)T, DV_HDR + DV_WARPS * ntl * 128 * 4, &d.b)) return false;
    if (c) *c = d;
    return true;
}

bool decode_supported(int E, int H, int I, int64_t T, int k) { return dv_config(E, H, I, T, k, nullptr); }

static size_t al256(size_t v) { return (v + 255) & ~size_t(255); }

// h per (slot, token).
size_t decode_scratch_bytes(int E, int H, int I, int64_t T, int k) {
    if (!decode_supported(E, H, I, T, k)) return 0;
    const int64_t slots = std::min<int64_t>(E, T * k);
    return al256((size_t)slots * T * I * 2);
}

template <typename K>
static cudaError_t dv_launch(K kernel, int grid, int smem, cudaStream_t st, const DvArgs& a) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(DV_THREADS);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, a);
}

// Per-device function attributes: the largest dynamic shared memory any call
// asked for so far, and the whole unified L1 / shared array as shared memory.
// kind: one slot per kernel instance.
constexpr int DV_KINDS = 16;
template <typename K>
static cudaError_t dv_attr(K kernel, int smem, int kind) {
    static std::mutex mu;
    static int set_bytes[64][DV_KINDS] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (set_bytes[dev][kind] >= smem) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) set_bytes[dev][kind] = smem;
    return e;
}

static void dv_apply(DvArgs& a, const DvGeom& g) {
    a.kc = g.kc;
    a.depth = g.depth;
    a.stage_bytes = g.stage_bytes;
    a.rs = g.rs;
    a.ss = g.ss;
    a.hrs = g.hrs;
    a.ring_off = g.ring_off;
}

// Kernel instances by chunk size (kc in {1, 2, 4, 8}).
template <int CB, int KC>
static cudaError_t dv_launch_gateup(const DvCfg& c, const DvArgs& a, cudaStream_t st) {
    cudaError_t err = dv_attr(dv_gateup_kernel<CB, KC>, c.a.smem, CB * 8 + (KC == 8 ? 3 : KC == 4 ? 2 : KC - 1));
    if (err != cudaSuccess) return err;
    return dv_launch(dv_gateup_kernel<CB, KC>, c.G, c.a.smem, st, a);
}
template <int CB, int KC>
static cudaError_t dv_launch_down(const DvCfg& c, const DvArgs& a, cudaStream_t st) {
    cudaError_t err = dv_attr(dv_down_kernel<CB, KC>, c.b.smem, CB * 8 + 4 + (KC == 8 ? 3 : KC == 4 ? 2 : KC - 1));
    if (err != cudaSuccess) return err;
    return dv_launch(dv_down_kernel<CB, KC>, c.G, c.b.smem, st, a);
}

template <int CB>
static cudaError_t dv_impl(const DvCfg& c, const DvArgs& a, cudaStream_t st) {
    DvArgs aa = a;
    dv_apply(aa, c.a);
    timing_begin(KK_DECODE_GATEUP, st);
    cudaError_t err;
    switch (c.a.kc) {
        case 8: err = dv_launch_gateup<CB, 8>(c, aa, st); break;
        case 4: err = dv_launch_gateup<CB, 4>(c, aa, st); break;
        case 2: err = dv_launch_gateup<CB, 2>(c, aa, st); break;
        default: err = dv_launch_gateup<CB, 1>(c, aa, st); break;
    }
    timing_end(KK_DECODE_GATEUP, st);
    count_launch();
    if (err != cudaSuccess) return err;
    DvArgs ab = a;
    dv_apply(ab, c.b);
    timing_begin(KK_DECODE_DOWN, st);
    switch (c.b.kc) {
        case 8: err = dv_launch_down<CB, 8>(c, ab, st); break;
        case 4: err = dv_launch_down<CB, 4>(c, ab, st); break;
        case 2: err = dv_launch_down<CB, 2>(c, ab, st); break;
        default: err = dv_launch_down<CB, 1>(c, ab, st); break;
    }
    timing_end(KK_DECODE_DOWN, st);
    count_launch();
    return err;
}

cudaError_t launch_decode_forward(int codebook, int E, int H, int I, int k, int renorm, int64_t T,
                                  const __nv_bfloat16* x, const float* logits, int32_t* idx, float* w,
                                  const uint8_t* gu_packed, const float* gu_absmax, const uint8_t* d_packed,
                                  const float* d_absmax, void* scratch, __nv_bfloat16* y, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    DvCfg c;
    if (!dv_config(E, H, I, T, k, &c)) return cudaErrorInvalidValue;
    DvArgs a{};
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
    a.h = static_cast<__nv_bfloat16*>(scratch);
    a.y = y;
    return codebook == 0 ? dv_impl<0>(c, a, st) : dv_impl<1>(c, a, st);
}

}  // namespace e4b
