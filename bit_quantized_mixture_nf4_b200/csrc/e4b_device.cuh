// Device-side building blocks for the e4b kernels (sm_100a only): codebooks,
// the exact per-block dequantization, mbarrier / TMA / tcgen05 wrappers written
// as inline PTX.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ != 1000)
#error "e4b kernels are written for sm_100a only"
#endif

namespace e4b {

// Device status word (read and cleared by e4b_device_status): bit 0 a bounded wait
// timed out; bit 1 a debug-build bounds check failed, with the first failing
// check's site in bits 8..15.
enum : uint32_t { kStatusTimeout = 1u, kStatusDebugCheck = 2u };

// Debug-build bounds checks (E4B_DEBUG_CHECKS=1): a check that fails records its
// site and the kernel skips the access it guarded (nothing traps).  The sites:
enum : uint32_t {
    kSiteGemmTile = 1,       // grouped GEMM: an m-tile entry outside the experts or the grouped rows
    kSiteGemmPerm = 2,       // grouped GEMM epilogue: a grouped row's pair id outside [0, rows)
    kSiteGatherPerm = 3,     // row gather: a pair id outside [0, P)
    kSiteCombineInv = 4,     // combine: an inverse-permutation entry outside [-1, P)
    kSiteRouterInv = 5,      // routing gradient: an inverse-permutation entry outside [-1, P)
    kSiteOffsets = 6,        // schedule: expert offsets not ascending from 0, or past P
    kSiteCounts = 7,         // schedule: counts[e] != offsets[e+1] - offsets[e]
    kSiteTilePrefix = 8,     // schedule: m-tile total != sum of ceil(counts / tile rows)
    kSiteSchedule = 9,       // schedule: an m-tile entry outside its expert's rows
    kSitePerm = 10,          // schedule: perm[r] outside [0, P), or of another expert
    kSiteInvPerm = 11,       // schedule: inv_perm not the inverse of perm
};
#ifndef E4B_DEBUG_CHECKS
#define E4B_DEBUG_CHECKS 0
#endif

// Records a failed check: sets bit 1 and, if no site is recorded yet, this site.
// A compare-and-swap loop with a bound (it only repeats while other threads change
// the word).
__device__ __forceinline__ void debug_fail(uint32_t* status, uint32_t site) {
    uint32_t cur = *reinterpret_cast<volatile uint32_t*>(status);
    for (int i = 0; i < 64; ++i) {
        const uint32_t nv = cur | kStatusDebugCheck | ((cur & 0xFF00u) ? 0u : ((site & 0xFFu) << 8));
        const uint32_t prev = atomicCAS(status, cur, nv);
        if (prev == cur) return;
        cur = prev;
    }
    atomicOr(status, kStatusDebugCheck);
}

// ----------------------------------------------------------------- codebooks
// NF4: the 16 NormalFloat values (QLoRA appendix, the "standard" table the
// expert-layer pages refer to via get_4bit_type("nf4")), ascending, code 7 = 0.
// FP4: e2m1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} / 6 with the sign in bit 3.
// MXFP4 (index 2): the same codes unscaled, {0, .5, ..., 6}; a 32-element block's
// E8M0 scale 2^(s - 127) multiplies them (OCP Microscaling Formats v1.0).
static __constant__ float c_code[3][16] = {
    {-1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,
     -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,
     0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f, 0.33791524171829224f,
     0.44070982933044434f, 0.5626170039176941f, 0.7229568362236023f, 1.0f},
    {0.0f, 0.5f / 6.0f, 1.0f / 6.0f, 1.5f / 6.0f, 2.0f / 6.0f, 3.0f / 6.0f, 4.0f / 6.0f, 1.0f,
     -0.0f, -0.5f / 6.0f, -1.0f / 6.0f, -1.5f / 6.0f, -2.0f / 6.0f, -3.0f / 6.0f, -4.0f / 6.0f, -1.0f},
    {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f, -0.0f, -0.5f, -1.0f, -1.5f, -2.0f, -3.0f, -4.0f, -6.0f}};

// The E8M0 scale byte s as the fp32 value 2^(s - 127) (s = 0: the subnormal 2^-127;
// s = 255, the format's NaN, is never produced by the quantizer).
__device__ __forceinline__ float mx_scale(uint32_t s) {
    return s == 0u ? __int_as_float(0x00400000) : __int_as_float((int)(s << 23));
}

// --------------------------------------------------------------- small utils
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// (a & ~m) | (b & m): per-bit select.
__device__ __forceinline__ uint32_t bitsel(uint32_t a, uint32_t b, uint32_t m) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xD8;" : "=r"(d) : "r"(a), "r"(b), "r"(m));
    return d;
}

// Two fp32 -> packed bf16x2 (lo in bits 0..15), round-to-nearest-even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ routing
// Routing weights of one token, computed by one warp once the top-k is known:
// v = the token's logits (lane + 32*i, -inf beyond E), lane j < k holds the
// j-th choice's logit in sel_v, top_v = the largest logit.  softmax over all E
// at the choices (exp(l - top) / sum), optionally divided by their sum.  The
// summation order is fixed (per-lane sums over i, then a butterfly), so every
// kernel that routes gets bit-identical weights.
__device__ __forceinline__ float route_weights_warp(const float (&v)[8], int E, int k, int renorm, int lane,
                                                    float sel_v, float top_v) {
    float z = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (lane + 32 * i < E) z += expf(v[i] - top_v);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    float p = (lane < k) ? expf(sel_v - top_v) / z : 0.0f;
    if (renorm) {
        float s = p;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        p = p / s;
    }
    return p;
}

// Order-preserving 32-bit key of a finite float (-0 is taken as +0): a > b as
// floats iff key(a) > key(b).  0 is below every key of a float, -inf included.
__device__ __forceinline__ uint32_t float_key(float f) {
    uint32_t b = __float_as_uint(f);
    if ((b & 0x7fffffffu) == 0u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

struct NoPickHook {
    __device__ __forceinline__ void operator()(int, int) const {}
};

// Routing of one token by one warp: top-k on the fp32 logits (descending, ties
// to the lower expert index; E <= 256), then route_weights_warp.  Each of the k
// rounds takes the warp-wide maximum key and, among the lanes holding it, the
// lowest expert index (two redux.sync).  Lane j < k receives the j-th choice in
// *e_out / *w_out.  on_pick(expert, j) runs on every lane as soon as round j has
// picked its expert (the decode kernels start that expert's weight stream there).
template <typename PickHook = NoPickHook>
__device__ __forceinline__ void route_token_warp(const float* __restrict__ l, int E, int k, int renorm, int lane,
                                                 int* e_out, float* w_out, const PickHook& on_pick = PickHook()) {
    float v[8];
    uint32_t key[8];
    const float NEG_INF = __int_as_float(0xff800000);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        v[i] = (e < E) ? __ldcg(l + e) : NEG_INF;
        key[i] = (e < E) ? float_key(v[i]) : 0u;
    }
    uint32_t taken = 0;
    int sel_e = -1;
    float sel_v = 0.0f, top_v = 0.0f;
    for (int j = 0; j < k; ++j) {
        uint32_t bk = 0u;
        int bi = -1;
#pragma unroll
        for (int i = 0; i < 8; ++i)   // first (lowest index) maximum among this lane's free experts
            if (lane + 32 * i < E && !((taken >> i) & 1u) && (bi < 0 || key[i] > bk)) {
                bk = key[i];
                bi = i;
            }
        const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t win = __reduce_min_sync(0xffffffffu, (bi >= 0 && bk == mk) ? (uint32_t)(lane + 32 * bi) : 0xffffffffu);
        if ((int)(win & 31u) == lane) taken |= 1u << (win >> 5);
        on_pick((int)win, j);
        const float wv = key_float(mk);
        if (j == 0) top_v = wv;
        if (lane == j) {
            sel_e = (int)win;
            sel_v = wv;
        }
    }
    *e_out = sel_e;
    *w_out = route_weights_warp(v, E, k, renorm, lane, sel_v, top_v);
}

// ------------------------------------------------- exact per-block dequantize
// A 64-element block shares one absmax a, so its 16 possible outputs are
// bf16_rn(code[q] * a).  Build those 16 values once (16 fp32 multiplies), keep
// their low and high bytes as two 16-byte register tables, and decode each
// 4-bit code with byte permutes.  The result is bit-identical to converting
// every element separately.
struct BlockTable {
    uint32_t lo[4], hi[4];
};

template <int CB>
__device__ __forceinline__ BlockTable make_table(float a) {
    uint32_t t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        t[i] = pack_bf16x2(__fmul_rn(c_code[CB][2 * i], a), __fmul_rn(c_code[CB][2 * i + 1], a));
    BlockTable b;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        b.lo[j] = prmt(t[2 * j], t[2 * j + 1], 0x6420);  // low bytes of entries 4j..4j+3
        b.hi[j] = prmt(t[2 * j], t[2 * j + 1], 0x7531);  // high bytes
    }
    return b;
}

// Decode one packed word (4 bytes = 8 elements in storage order, element 2b in
// the high nibble of byte b) into four bf16x2 words in element order.
__device__ __forceinline__ void decode_word(const BlockTable& tb, uint32_t x, uint32_t out[4]) {
    const uint32_t s = x & 0x77777777u;   // low 3 bits of every code
    const uint32_t x4 = x << 4;           // puts bit 3 of even nibbles at bit 7 of their byte
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t sel = h ? (s >> 16) : s;
        // byte i = 0xFF when nibble 4h+i has its top bit set (sign-replicate mode)
        const uint32_t m = prmt(x, x4, h ? 0xBFAEu : 0x9D8Cu);
        const uint32_t l = bitsel(prmt(tb.lo[0], tb.lo[1], sel), prmt(tb.lo[2], tb.lo[3], sel), m);
        const uint32_t g = bitsel(prmt(tb.hi[0], tb.hi[1], sel), prmt(tb.hi[2], tb.hi[3], sel), m);
        // nibble 4h+1 is element 4h (high nibble of byte 2h), nibble 4h is element 4h+1
        out[2 * h + 0] = prmt(l, g, 0x4051);
        out[2 * h + 1] = prmt(l, g, 0x6273);
    }
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t addr, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(addr), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t addr) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(addr) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t addr, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(addr), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait: returns false (after recording a timeout in *status and in the
// CTA-wide abort flag) if the phase does not complete within the time limit or
// another role of the CTA has already given up.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s: far above any legitimate wait
__device__ __forceinline__ bool mbar_wait(uint32_t addr, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status) {
    if (mbar_try_wait(addr, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(addr, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}

// Bounded wait that does not give up early on the abort flag: used to let a
// CTA's own bulk copies land before it exits.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t addr, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(addr, parity))
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    return true;
}

// Contiguous global -> shared bulk copy (no tensor map), completing on an
// mbarrier.  dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(mbar)
                 : "memory");
}

// Barrier over the first nthreads threads of the CTA (id != 0; 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// 4-byte asynchronous global->shared copy; src_bytes = 0 writes zero without reading.
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// Arrive on the mbarrier when this thread's earlier cp.async copies have landed
// (the arrival is not added to the expected count: the barrier's init count has it).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint32_t mbar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m, uint32_t mbar, int x,
                                            int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(mbar), "r"(x), "r"(y)
        : "memory");
}

// Bring a tensor tile into L2 ahead of its load (no shared memory, no completion).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* m, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(m)),
                 "r"(x), "r"(y)
                 : "memory");
}

// ------------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D(tmem) (+)= A(smem desc) * B(smem desc), kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on an mbarrier when all previously issued tcgen05 ops complete.
__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     mbar)
                 : "memory");
}

// 32 lanes x 32 columns of 32-bit: thread i gets lane (base_lane + i), columns c..c+31.
// The raw registers must go through tmem_ld_wait() before use.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// tcgen05.wait::ld with the loaded registers as in/out operands, so no use of
// them can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;"
        : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
          "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
          "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
          "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
          "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
        :
        : "memory");
}

// Load 32 fp32 accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_load32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(taddr, r);
    tmem_ld_wait(r);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}


// ------------------------------------------------------------------ clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t local_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
    return r;
}
// Arrive on an mbarrier of another CTA of the cluster, given by its shared::cluster
// address (default semantics: release at CTA scope; the data the arrival announces
// stays in the arriving CTA's own shared memory and is made visible to the tensor
// cores by a proxy fence before the arrival).  A cluster-scope release here costs
// thousands of cycles per arrival and is not needed.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t addr, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    return done != 0;
}
// Bounded wait with cluster-scope acquire (barriers that receive remote arrivals).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t addr, uint32_t parity, volatile int* abort_flag,
                                                  uint32_t* status) {
    if (mbar_try_wait_cluster(addr, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_cluster(addr, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on the
// mbarrier of the pair's first CTA (2-SM operand loads).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* m, uint32_t leader_mbar, int x,
                                                 int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(leader_mbar), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// 2-SM MMA issued by the pair's first CTA: A rows and B columns split between the two CTAs.
__device__ __forceinline__ void mma_bf16_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on the mbarrier at the same offset in both CTAs of the pair.
__device__ __forceinline__ void mma_commit_pair(uint32_t mbar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(mbar),
        "h"((uint16_t)0x3)
        : "memory");
}

// Shared-memory matrix descriptor (sm_100 format, version 1): start address,
// leading / stride byte offsets, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version for sm_100
    d |= (uint64_t)2 << 61;   // SWIZZLE_128B
    return d;
}

// Instruction descriptor for kind::f16: bf16 A and B, fp32 accumulator, A
// K-major, B K-major (b_mn_major = 0) or MN-major (1), shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int b_mn_major) {
    return (1u << 4)                        // D format: f32
           | (1u << 7)                      // A format: bf16
           | (1u << 10)                     // B format: bf16
           | ((uint32_t)b_mn_major << 16)   // B major-ness
           | ((uint32_t)(N >> 3) << 17)     // N / 8
           | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// Byte offset of 16-byte chunk `chunk` (0..7) of 128-byte row `row` inside a
// 1024-byte-aligned tile stored with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

}  // namespace e4b
