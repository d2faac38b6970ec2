// Internal host/device interfaces shared by the e4b translation units.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <algorithm>

#include "e4b_device.cuh"

namespace e4b {

enum Epi { EPI_GATEUP = 0, EPI_DOWN = 1, EPI_DGRAD_DOWN = 2, EPI_DGRAD_GATEUP = 3 };

struct GemmParams {
    int E, K, N, n_tiles;
    const int* tile_prefix;   // [E+1] prefix of ceil(M_e / tile_rows); [E] = total m-tiles
    const int4* sched;        // per m-tile: (expert, first row, rows, 0)
    const int* perm;          // [P] pair id of each grouped row
    const float* topk_w;      // [P] routing weight by pair id
    const float* absmax;      // absmax of the weight stack
    int64_t b_rows_total;     // rows of the stored [rows, cols] weight matrix, all experts
    int b_rows_per_expert;
    int b_blocks_per_row;     // stored cols / 64
    int up_offset;            // I (EPI_GATEUP: first up row; also the feature count)
    int act;                  // EPI_GATEUP: 0 SwiGLU, 1 clamped GLU (alpha, limit below)
    __nv_bfloat16* out_bf16;  // h [P, I], dGU [P, 2I], or the per-pair rows [P, H] (down / dgrad gate_up)
    __nv_bfloat16* gu;        // saved activation derivatives [P, 2I]: dh/dg | dh/du (written by
                              // EPI_GATEUP, read by EPI_DGRAD_DOWN)
    const float* bias;        // optional per-expert bias: [E, 2I] (EPI_GATEUP) or [E, H] (EPI_DOWN)
    int ld_out;
    float alpha, limit;
    uint32_t* status;         // device status word
    const __nv_bfloat16* h_in;   // EPI_DGRAD_DOWN, optional: the forward's h [P, I] in grouped order
    float* dw_part;           // with h_in: [P, n_tiles] fp32, row r / n-tile nt: sum over the tile's
                              // columns c of (grad_out_r W_d,e)[c] * h[r, c] (before the routing weight)
    // Per-expert LoRA as one more 64-deep k-stage: A gets the thin operand [rows, 64] bf16
    // (the lora_a argument of launch_grouped_gemm), B the adapter: K-major B (gate_up, down)
    // reads lora_b as [E, b_rows_per_expert, lora_r] (the B_gu / B_d adapter rows), MN-major
    // B (the two input-gradient GEMMs) as [E, lora_r, N] (A_d / A_gu).  Ranks above lora_r
    // and rows or columns outside the expert read as 0.  lora_r = 0: no extra stage.
    const __nv_bfloat16* lora_b;
    int lora_r;               // 0 or a multiple of 8 up to 64
    // MXFP4 weights (codebook 2): the E8M0 scale bytes [rows, mx_stride] replace absmax
    const uint8_t* mx_scales;
    int64_t mx_stride;
    // bf16 weights (GEMM codebook 3: the 8-bit modes after their dequantization, or
    // bf16 passthrough): [b_rows_total, stored cols] row-major; copied into the operand
    // ring by the dequantizing warps
    const __nv_bfloat16* bf16_b;
    int64_t a_rows;           // rows of A and of the per-row arrays (set by launch_grouped_gemm;
                              // the debug-build bounds checks compare against it)
};

// launch bookkeeping
void count_launch();
// Optional per-kernel-kind event timing (off by default): brackets one launch
// with CUDA events on its stream.
enum KernelKind { KK_QUANT = 0, KK_DEQUANT, KK_ROUTE, KK_GROUP, KK_GATHER, KK_COMBINE, KK_GEMM_GATEUP, KK_GEMM_DOWN,
                  KK_GEMM_DGRAD_DOWN, KK_GEMM_DGRAD_GATEUP, KK_DECODE_GATEUP, KK_DECODE_DOWN, KK_COUNT };
// Also opens / closes the kind's NVTX range (api.cu).
void timing_begin(int kind, cudaStream_t st);
void timing_end(int kind, cudaStream_t st);
int num_sms();
// NVTX range over an entry point's host scope (api.cu)
struct NvtxScope {
    explicit NvtxScope(const char* name);
    ~NvtxScope();
    NvtxScope(const NvtxScope&) = delete;
    NvtxScope& operator=(const NvtxScope&) = delete;
};
uint32_t* device_status_ptr();

// quant.cu
cudaError_t launch_quantize(const float* w, int64_t nblocks, int codebook, uint8_t* packed, float* absmax,
                            cudaStream_t st);
cudaError_t launch_dequantize(const uint8_t* packed, const float* absmax, int64_t n, int codebook, int out_bf16,
                              void* out, cudaStream_t st);
// 8-bit blockwise codebooks (3 int8, 4 fp8): one code byte per element, fp32 absmax per 64
cudaError_t launch_quantize8(const float* w, int64_t nblocks, int codebook, uint8_t* codes, float* absmax,
                             cudaStream_t st);
cudaError_t launch_dequantize8(const uint8_t* codes, const float* absmax, int64_t n, int codebook, int out_bf16,
                               void* out, cudaStream_t st);
// MXFP4 (32-element blocks, E8M0 scales [rows, S], S = mxfp4_scale_stride(in) bytes per row)
int64_t mxfp4_scale_stride(int64_t in);
cudaError_t launch_quantize_mxfp4(const float* w, int64_t rows, int64_t in, uint8_t* packed, uint8_t* scales,
                                  cudaStream_t st);
cudaError_t launch_dequantize_mxfp4(const uint8_t* packed, const uint8_t* scales, int64_t rows, int64_t in,
                                    int out_bf16, void* out, cudaStream_t st);

// route.cu
constexpr int kChunkPairs = 256;   // pairs per grouping block (one per thread of a 256-thread block)
cudaError_t launch_route(const float* logits, int64_t T, int E, int k, int renorm, int32_t* idx, float* w,
                         cudaStream_t st);
// counts/offsets/tile_prefix/perm from topk_idx; chunk scratch: [nchunks * E] ints x2
// sched: [ceil(P/tile_rows) + E] m-tile entries (expert, first row, rows, 0)
// inv_perm[pair] = grouped row of the pair, -1 for a pair of an out-of-range expert
cudaError_t launch_group(const int32_t* idx, int64_t P, int E, int tile_rows, int32_t* chunk_counts,
                         int32_t* chunk_base, int32_t* counts, int32_t* offsets, int32_t* tile_prefix,
                         int4* sched, int32_t* perm, int32_t* inv_perm, cudaStream_t st);
// Consistency checks of a grouping schedule (sched has n_sched entries); a violated
// property records its site in the device status word.  Debug builds run it after
// every grouping.
cudaError_t launch_validate_schedule(const int32_t* idx, int64_t P, int E, int tile_rows, const int32_t* counts,
                                     const int32_t* offsets, const int32_t* tile_prefix, const int4* sched,
                                     int64_t n_sched, const int32_t* perm, const int32_t* inv_perm, cudaStream_t st);
// nrows: device pointer to the number of grouped rows (offsets[E])
cudaError_t launch_gather_rows(const __nv_bfloat16* src, const int32_t* perm, const int32_t* nrows, int k,
                               int64_t P, int H, __nv_bfloat16* dst, cudaStream_t st);
// y[t] = sum over the grouped rows inv_perm[t*k + j] of token t (fp32 sum in slot
// order j, bf16 result; rows of out-of-range experts skipped)
cudaError_t launch_combine(const __nv_bfloat16* rows, const int32_t* inv_perm, int k, int64_t T, int H,
                           __nv_bfloat16* y, cudaStream_t st);

// grouped_gemm.cu
int gemm_tile_rows();
// codebook: 0 NF4, 1 FP4, 2 MXFP4 (packed + E8M0 scales), 3 bf16 weights in p.bf16_b.
// lora_a: the thin A operand of the LoRA k-stage, [a_rows, 64] bf16 (rank padded with
// zeros), when p.lora_r > 0; otherwise null.
cudaError_t launch_grouped_gemm(int epi, int codebook, const void* a, int64_t a_rows, const uint8_t* packed,
                                int64_t packed_rows_total, int packed_row_bytes, GemmParams p, int max_m_tiles,
                                cudaStream_t st, const void* lora_a = nullptr);

// Tiled TMA descriptor of a rank-`rank` tensor (dims innermost first, strides in bytes of
// dims 1..rank-1); grouped_gemm.cu.
bool make_tensor_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle sw);

// decode.cu (T <= 8): the weight-streaming forward.  decode_supported: the shapes the
// kernels take (H, I multiples of 64, H <= 8192, the stage rings fit in shared memory).
bool decode_supported(int E, int H, int I, int64_t T, int k);
// Scratch bytes of the decode path: h per (slot, token) [min(E, T*k), T, I] bf16.
size_t decode_scratch_bytes(int E, int H, int I, int64_t T, int k);
cudaError_t launch_decode_forward(int codebook, int E, int H, int I, int k, int renorm, int64_t T,
                                  const __nv_bfloat16* x, const float* logits, int32_t* idx, float* w,
                                  const uint8_t* gu_packed, const float* gu_absmax, const uint8_t* d_packed,
                                  const float* d_absmax, void* scratch, __nv_bfloat16* y, cudaStream_t st);

}  // namespace e4b
