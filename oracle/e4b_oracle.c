/*
 * e4b oracle: a plain, slow, obviously-correct CPU statement of the NF4
 * Mixture-of-Experts expert path.  TEST INFRASTRUCTURE ONLY: the tests, the
 * package smoke check and the CPU-baseline leg of the benchmark call it; the
 * product path never does.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * Sources (cited by page title and section):
 *   [P4]  "experts4bit-qlora 0.1.0" source diff, file _vendor/experts.py,
 *         class Experts4bit (__init__, from_float, _quantize_stack,
 *         _dequantize_expert, forward).
 *   [P5]  bitsandbytes pull request #1965 "Add Experts4bit for 4-bit
 *         quantization of fused MoE experts", sections "What this adds" and
 *         "Correctness & coverage".
 *   [P1]  "experts4bit-qlora" 0.4.0 package description, section "Storage
 *         modes: the support matrix".
 *   [QLoRA] Dettmers et al. 2023, "QLoRA", appendix on the NormalFloat data
 *         type (the 16 NF4 values; the pages only call get_4bit_type("nf4")).
 *   [P2]  "experts4bit-qlora 0.31.1" PyPI project page, section "Scope": the
 *         gpt-oss experts carry per-expert biases and a clamped GLU.  The pages
 *         give no formula; the reading taken is the published gpt-oss expert
 *         (gpt-oss model card, OpenAI 2025): g' = min(g, limit), u' = clamp(u,
 *         -limit, limit), h = (u' + 1) g' sigmoid(alpha g'), with alpha and limit
 *         parameters (1.702 and 7 in gpt-oss), biases added to g, u and to the
 *         down projection's output, and the clamp passing the gradient where its
 *         input lies inside the closed interval.
 *
 * Precision.  Quantize takes its decisions in fp32 (the pages quantize fp32
 * weights with fp32 absmax); dequantize multiplies in fp32 and rounds once to
 * bf16 (round-to-nearest-even); routing weights, forward and input gradient
 * are computed in fp64.  Readings where the pages are silent:
 *   - codes are chosen by strict comparison with the fp32 midpoints of the
 *     sorted codebook, so an exact tie goes to the smaller value;
 *   - an all-zero block stores absmax 0 and the zero code;
 *   - the FP4 codebook is OCP e2m1 {0,.5,1,1.5,2,3,4,6}/6 with the sign in
 *     bit 3 (parity with bitsandbytes' own fp4 table is unpinned);
 *   - routing selects top-k on the fp32 logits (descending, ties to the lower
 *     expert index), weights are softmax over all experts, optionally divided
 *     by their sum over the selected k.
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_BLOCKSIZE 2

/* ---- codebooks ---------------------------------------------------------- */

/* NF4: the 16 NormalFloat values of [QLoRA], ascending, index 7 is zero.  The
 * code of a value is its index. */
static const float kNF4[16] = {
    -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,
    -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,
    0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f,
    0.33791524171829224f, 0.44070982933044434f, 0.5626170039176941f,
    0.7229568362236023f, 1.0f};

/* FP4 (e2m1, max-normalised): value of a 4-bit code = sign(bit 3) * e2m1(bits
 * 2..0) / 6.  e2m1 magnitudes: 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
static float fp4_value(int code) {
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    float m = (float)(mag[code & 7] / 6.0);
    return (code & 8) ? -m : m;
}

/* Value of code q (0..15) under codebook cb (0 = NF4, 1 = FP4). */
float e4bo_code_value(int cb, int q) {
    if (cb == 0) return kNF4[q & 15];
    return fp4_value(q & 15);
}

/* The 15 distinct codebook values in ascending order and the code of each.
 * NF4: 16 distinct values, the code is the index.  FP4: -0 is dropped (it is
 * never produced), so 15 values remain. */
static int sorted_codebook(int cb, float *vals, int *codes) {
    if (cb == 0) {
        for (int i = 0; i < 16; ++i) { vals[i] = kNF4[i]; codes[i] = i; }
        return 16;
    }
    int n = 0;
    for (int m = 7; m >= 1; --m) { vals[n] = fp4_value(8 | m); codes[n] = 8 | m; ++n; }
    vals[n] = 0.0f; codes[n] = 0; ++n;
    for (int m = 1; m <= 7; ++m) { vals[n] = fp4_value(m); codes[n] = m; ++n; }
    return n;
}

/* Copy the 16 code values (indexed by code) for a test to inspect. */
void e4bo_codebook(int cb, float *out16) {
    for (int q = 0; q < 16; ++q) out16[q] = e4bo_code_value(cb, q);
}

/* ---- bf16 round-to-nearest-even from the IEEE bit definition ------------- */

uint16_t e4bo_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) {           /* inf / nan */
        if (u & 0x007fffffu) return (uint16_t)((u >> 16) | 0x40u); /* quiet nan */
        return (uint16_t)(u >> 16);
    }
    uint32_t upper = u >> 16, lower = u & 0xffffu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
    return (uint16_t)upper;
}

float e4bo_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ---- quantize ([P4] _quantize_stack; [P5] "What this adds") -------------- */

/* w: fp32 [E, out, in] row-major.  packed: [E, out*in/2] bytes, element 2b in
 * the high nibble of byte b.  absmax: [E, out*in/blocksize], block j of row o
 * at o*in/blocksize + j.  in % blocksize must be 0 ([P4] __init__ raises
 * otherwise).  Only blocksize 64 is part of the contract. */
int e4bo_quantize(const float *w, int64_t E, int64_t out, int64_t in, int blocksize,
                  int cb, uint8_t *packed, float *absmax) {
    if (!w || !packed || !absmax || E < 0 || out < 0 || in < 0) return ORC_ERR_ARG;
    if (cb != 0 && cb != 1) return ORC_ERR_ARG;
    if (blocksize != 64) return ORC_ERR_BLOCKSIZE;
    if (in % blocksize != 0) return ORC_ERR_BLOCKSIZE;
    float vals[16];
    int codes[16];
    int nv = sorted_codebook(cb, vals, codes);
    float mid[15];
    for (int i = 0; i + 1 < nv; ++i) mid[i] = (vals[i] + vals[i + 1]) * 0.5f;
    const int zero_code = (cb == 0) ? 7 : 0;
    const int64_t nblocks = E * out * in / blocksize;
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nblocks; ++b) {
        const float *src = w + b * blocksize;
        float a = 0.0f;
        for (int i = 0; i < blocksize; ++i) {
            float m = fabsf(src[i]);
            if (m > a) a = m;
        }
        absmax[b] = a;
        uint8_t *dst = packed + b * (blocksize / 2);
        for (int i = 0; i < blocksize; i += 2) {
            int q[2];
            for (int t = 0; t < 2; ++t) {
                if (a == 0.0f) { q[t] = zero_code; continue; }
                float n = src[i + t] / a;   /* IEEE fp32 division, correctly rounded */
                int r = 0;
                for (int m = 0; m < nv - 1; ++m) r += (mid[m] < n) ? 1 : 0;
                q[t] = codes[r];
            }
            dst[i / 2] = (uint8_t)((q[0] << 4) | q[1]);
        }
    }
    return ORC_OK;
}

/* ---- dequantize ([P4] _dequantize_expert) -------------------------------- */

/* fp32 value of element i: code value * absmax, one fp32 rounding. */
static inline float deq_one(const uint8_t *packed, const float *absmax, int64_t i,
                            int blocksize, int cb) {
    uint8_t byte = packed[i >> 1];
    int q = (i & 1) ? (byte & 15) : (byte >> 4);
    return e4bo_code_value(cb, q) * absmax[i / blocksize];
}

int e4bo_dequantize_f32(const uint8_t *packed, const float *absmax, int64_t n,
                        int blocksize, int cb, float *out) {
    if (!packed || !absmax || !out || n < 0 || n % blocksize) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = deq_one(packed, absmax, i, blocksize, cb);
    return ORC_OK;
}

int e4bo_dequantize_bf16(const uint8_t *packed, const float *absmax, int64_t n,
                         int blocksize, int cb, uint16_t *out) {
    if (!packed || !absmax || !out || n < 0 || n % blocksize) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = e4bo_f32_to_bf16(deq_one(packed, absmax, i, blocksize, cb));
    return ORC_OK;
}

/* ---- 8-bit blockwise modes ([P1] "Storage modes: the support matrix") -----
 * int8 is a "blockwise dynamic map" and fp8 a "bnb e4m3 codebook"; the pages
 * print neither table.  Readings taken, both normalised to max 1 and used like
 * the 4-bit codebooks (64-element blocks, fp32 absmax, nearest value with an
 * exact tie going to the smaller value, one byte per element):
 *   int8: the dynamic tree quantization of Dettmers et al. (2022, "8-bit
 *     optimizers via block-wise quantization"): bit 7 the sign; in the 7-bit tail
 *     the number E of leading zeros is a decimal exponent, the first 1 bit an
 *     indicator, and the F = 6 - E bits after it a linear fraction j on
 *     [0.1, 1]: |value| = 10^-E (0.1 + 0.9 (j + 1/2) / 2^F), the centres of 2^F
 *     equal bins.  Tail 0 is 0 (sign clear) or +1 (sign set: the absmax element);
 *   fp8: the E4M3 values (OCP 8-bit floating point: bias 7, subnormals, 448 the
 *     largest, S.1111.111 NaN) divided by 448; the code is the E4M3 bit pattern
 *     (the two NaNs and -0 are never produced).
 * With these, the reconstruction error ordering of the support matrix holds:
 * int8 < fp8 < nf4 < fp4. */

static float int8_value(int code) {
    const int s = code >> 7, t = code & 127;
    if (t == 0) return s ? 1.0f : 0.0f;
    int E = 0;
    while (!(t & (64 >> E))) ++E;              /* leading zeros of the 7-bit tail */
    const int F = 6 - E, j = t & ((1 << F) - 1);
    const double v = pow(10.0, -E) * (0.1 + 0.9 * (j + 0.5) / (double)(1 << F));
    return (float)(s ? -v : v);
}

static float fp8_value(int code) {   /* NaN patterns give NaN, never produced */
    const int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    const double mag = (e == 0) ? (m / 8.0) * pow(2.0, -6) : (1.0 + m / 8.0) * pow(2.0, e - 7);
    const float v = (float)(mag / 448.0);
    return s ? -v : v;
}

/* codebook 3 = int8, 4 = fp8: value of a byte code */
float e4bo_code_value8(int cb, int q) { return cb == 3 ? int8_value(q & 255) : fp8_value(q & 255); }

/* The distinct values in ascending order with their codes (fp8: NaNs and -0
 * dropped). */
static int sorted_codebook8(int cb, float *vals, int *codes) {
    int n = 0;
    for (int q = 0; q < 256; ++q) {
        const float v = e4bo_code_value8(cb, q);
        if (v != v) continue;
        if (cb == 4 && q == 0x80) continue;
        vals[n] = v;
        codes[n] = q;
        ++n;
    }
    for (int i = 1; i < n; ++i)   /* insertion sort by value */
        for (int k = i; k > 0 && vals[k - 1] > vals[k]; --k) {
            float tv = vals[k]; vals[k] = vals[k - 1]; vals[k - 1] = tv;
            int tc = codes[k]; codes[k] = codes[k - 1]; codes[k - 1] = tc;
        }
    return n;
}

void e4bo_codebook8(int cb, float *out256) {
    for (int q = 0; q < 256; ++q) out256[q] = e4bo_code_value8(cb, q);
}

/* w fp32 [E, out, in] -> codes [E, out*in] (one byte per element), absmax
 * [E, out*in/64]; the quantization rule of e4bo_quantize with the 8-bit table. */
int e4bo_quantize8(const float *w, int64_t E, int64_t out, int64_t in, int cb, uint8_t *codes, float *absmax) {
    if (!w || !codes || !absmax || E < 0 || out < 0 || in < 0 || (cb != 3 && cb != 4)) return ORC_ERR_ARG;
    if (in % 64) return ORC_ERR_BLOCKSIZE;
    float vals[256], mid[255];
    int cds[256];
    const int nv = sorted_codebook8(cb, vals, cds);
    for (int i = 0; i + 1 < nv; ++i) mid[i] = (vals[i] + vals[i + 1]) * 0.5f;
    int zero_code = 0;
    for (int i = 0; i < nv; ++i)
        if (vals[i] == 0.0f) zero_code = cds[i];
    const int64_t nblocks = E * out * in / 64;
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nblocks; ++b) {
        const float *src = w + b * 64;
        float a = 0.0f;
        for (int i = 0; i < 64; ++i) a = fmaxf(a, fabsf(src[i]));
        absmax[b] = a;
        for (int i = 0; i < 64; ++i) {
            if (a == 0.0f) { codes[b * 64 + i] = (uint8_t)zero_code; continue; }
            const float n = src[i] / a;
            int r = 0;
            for (int m = 0; m < nv - 1; ++m) r += (mid[m] < n) ? 1 : 0;
            codes[b * 64 + i] = (uint8_t)cds[r];
        }
    }
    return ORC_OK;
}

/* value = code value * absmax in fp32, then bf16 (bf16 != 0) or fp32 */
int e4bo_dequantize8(const uint8_t *codes, const float *absmax, int64_t n, int cb, int bf16, void *dst) {
    if (!codes || !absmax || !dst || n < 0 || n % 64 || (cb != 3 && cb != 4)) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const float v = e4bo_code_value8(cb, codes[i]) * absmax[i / 64];
        if (bf16) ((uint16_t *)dst)[i] = e4bo_f32_to_bf16(v);
        else ((float *)dst)[i] = v;
    }
    return ORC_OK;
}

/* ---- MXFP4 ([P2] "Scope": the gpt-oss experts ship MXFP4 weights) --------
 * The pages name the format only; the reading taken is the OCP Microscaling
 * Formats (MX) v1.0 specification: blocks of 32 consecutive elements of a row
 * share one E8M0 scale 2^X (stored as the byte X + 127), and each element is an
 * FP4 E2M1 value (sign in bit 3, magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} in bits
 * 2..0).  Quantization (the spec's conversion): X = floor(log2(amax)) - 2 (2 is
 * the largest E2M1 exponent), clamped to [-127, 127]; each element is v / 2^X
 * rounded to the nearest E2M1 value, ties to the even code, saturating at 6.
 * Readings where the spec leaves room: an all-zero block stores X = -127 and zero
 * codes; a value that rounds to zero is stored as +0.  Storage: codes packed like
 * the 4-bit stacks (element 2b in the high nibble of byte b); scales uint8
 * [E, out, S] with S = in/32 rounded up to a multiple of 16 (padding bytes 0). */

static const float kE2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

int64_t e4bo_mxfp4_scale_stride(int64_t in) { return ((in / 32) + 15) / 16 * 16; }

/* nearest E2M1 magnitude code of |p| (p finite), ties to the even code, saturating */
static int e2m1_code(float a) {
    if (a >= 6.0f) return 7;
    int best = 0;
    for (int c = 1; c < 8; ++c) {
        float dc = fabsf(a - kE2M1[c]), db = fabsf(a - kE2M1[best]);
        if (dc < db || (dc == db && (c & 1) == 0)) best = c;
    }
    return best;
}

int e4bo_quantize_mxfp4(const float *w, int64_t E, int64_t out, int64_t in, uint8_t *packed, uint8_t *scales) {
    if (!w || !packed || !scales || E < 0 || out < 0 || in < 0) return ORC_ERR_ARG;
    if (in % 32 != 0) return ORC_ERR_BLOCKSIZE;
    const int64_t S = e4bo_mxfp4_scale_stride(in), rows = E * out;
    memset(scales, 0, (size_t)(rows * S));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < in / 32; ++j) {
            const float *src = w + r * in + j * 32;
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(src[i]));
            int X = -127;
            if (amax > 0.0f) {
                int e;
                frexpf(amax, &e);          /* amax = m 2^e, m in [0.5, 1): floor(log2 amax) = e - 1 */
                X = (e - 1) - 2;
                if (X < -127) X = -127;
                if (X > 127) X = 127;
            }
            scales[r * S + j] = (uint8_t)(X + 127);
            uint8_t *dst = packed + (r * in + j * 32) / 2;
            for (int i = 0; i < 32; i += 2) {
                int q[2];
                for (int t = 0; t < 2; ++t) {
                    float p = ldexpf(src[i + t], -X);   /* exact scaling by a power of two */
                    int c = amax > 0.0f ? e2m1_code(fabsf(p)) : 0;
                    q[t] = (c != 0 && p < 0.0f) ? (8 | c) : c;
                }
                dst[i / 2] = (uint8_t)((q[0] << 4) | q[1]);
            }
        }
    }
    return ORC_OK;
}

static inline float mx_one(const uint8_t *packed, const uint8_t *scales, int64_t in, int64_t S, int64_t i) {
    const int64_t r = i / in, c = i % in;
    const uint8_t byte = packed[i >> 1];
    const int q = (i & 1) ? (byte & 15) : (byte >> 4);
    const float m = kE2M1[q & 7];
    return ldexpf((q & 8) ? -m : m, (int)scales[r * S + c / 32] - 127);
}

int e4bo_dequantize_mxfp4(const uint8_t *packed, const uint8_t *scales, int64_t E, int64_t out, int64_t in,
                          int bf16, void *dst) {
    if (!packed || !scales || !dst || E < 0 || out < 0 || in < 0 || in % 32) return ORC_ERR_ARG;
    const int64_t S = e4bo_mxfp4_scale_stride(in), n = E * out * in;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const float v = mx_one(packed, scales, in, S, i);
        if (bf16) ((uint16_t *)dst)[i] = e4bo_f32_to_bf16(v);
        else ((float *)dst)[i] = v;
    }
    return ORC_OK;
}

/* ---- routing ------------------------------------------------------------- */

/* logits fp32 [T, E] -> idx [T, k] (descending logit, ties to lower index) and
 * weights [T, k] = softmax over all E at the chosen experts, optionally divided
 * by their sum over the k. */
int e4bo_route(const float *logits, int64_t T, int E, int k, int renorm,
               int32_t *idx, double *wts) {
    if (!logits || !idx || !wts || T < 0 || E <= 0 || k <= 0 || k > E) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        int32_t *o = idx + t * k;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                int taken = 0;
                for (int jj = 0; jj < j; ++jj) taken |= (o[jj] == e);
                if (taken) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict: ties keep lower index */
            }
            o[j] = best;
        }
        double mx = (double)l[o[0]];
        double z = 0.0;
        for (int e = 0; e < E; ++e) z += exp((double)l[e] - mx);
        double s = 0.0;
        for (int j = 0; j < k; ++j) {
            wts[t * k + j] = exp((double)l[o[j]] - mx) / z;
            s += wts[t * k + j];
        }
        if (renorm)
            for (int j = 0; j < k; ++j) wts[t * k + j] /= s;
    }
    return ORC_OK;
}

/* ---- grouping ([P4] forward: expert mask, hit list, token gather) --------- */

/* Stable counting sort of the pair ids p = t*k + j by expert: rows of expert e
 * are [offsets[e], offsets[e+1]) and hold pair ids in ascending order. */
int e4bo_permute(const int32_t *idx, int64_t T, int k, int E, int32_t *counts,
                 int32_t *offsets, int32_t *perm) {
    if (!idx || !counts || !offsets || !perm || T < 0 || k <= 0 || E <= 0) return ORC_ERR_ARG;
    int64_t P = T * k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t p = 0; p < P; ++p) {
        if (idx[p] < 0 || idx[p] >= E) return ORC_ERR_ARG;
        counts[idx[p]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    if (!fill) return ORC_ERR_ARG;
    for (int e = 0; e < E; ++e) fill[e] = offsets[e];
    for (int64_t p = 0; p < P; ++p) perm[fill[idx[p]]++] = (int32_t)p;
    free(fill);
    return ORC_OK;
}

/* ---- forward ([P4] Experts4bit.forward) ---------------------------------- */

/* The expert's gated activation of the pre-activations g, u and its two partial
 * derivatives.  act 0 (SwiGLU, [P4] forward): h = silu(g) u.  act 1 (the clamped
 * GLU of [P2], reading above): h = (u' + 1) g' sigmoid(alpha g').  dhdg / dhdu may
 * be NULL. */
static double expert_act(int act, double alpha, double limit, double g, double u, double *dhdg, double *dhdu) {
    if (act == 0) {
        double s = 1.0 / (1.0 + exp(-g));
        if (dhdg) *dhdg = u * s * (1.0 + g * (1.0 - s));
        if (dhdu) *dhdu = g * s;
        return g * s * u;
    }
    double gc = g <= limit ? g : limit;                 /* min(g, limit) */
    double uc = u < -limit ? -limit : (u > limit ? limit : u);
    double s = 1.0 / (1.0 + exp(-alpha * gc));
    if (dhdg) *dhdg = (g <= limit) ? (uc + 1.0) * s * (1.0 + alpha * gc * (1.0 - s)) : 0.0;
    if (dhdu) *dhdu = (u >= -limit && u <= limit) ? gc * s : 0.0;
    return (uc + 1.0) * gc * s;
}

/* For each token t in tokens[0..nt) (all tokens when tokens == NULL) and each
 * slot j with expert e = idx[t,j]:
 *   g = x_t W_gate,e^T + bg_e,  u = x_t W_up,e^T + bu_e   (W_gate = rows [0,I),
 *   W_up = rows [I,2I) of gate_up, i.e. proj.chunk(2) with gate first; the
 *   biases bgu [E,2I] in the same order, zero when bgu == NULL),
 *   h = expert_act(g, u)   (silu(g) * u for act 0),
 *   y_t += w_{t,j} * (h W_down,e^T + bd_e),  summed over j in slot order
 *   (bd [E,H], zero when NULL).
 * x: [T,H] fp64, wgu: [E,2I,H] fp32 (dequantized), wd: [E,H,I] fp32,
 * y: [nt,H] fp64 (row i belongs to tokens[i]). */
int e4bo_forward(const double *x, int64_t T, int E, int H, int I, int k,
                 const int32_t *idx, const double *wts, const float *wgu,
                 const float *wd, const int64_t *tokens, int64_t nt, int act, double alpha, double limit,
                 const float *bgu, const float *bd, double *y) {
    if (!x || !idx || !wts || !wgu || !wd || !y || T < 0 || E <= 0 || k <= 0 || act < 0 || act > 1) return ORC_ERR_ARG;
    if (!tokens) nt = T;
#pragma omp parallel
    {
        double *h = (double *)malloc(sizeof(double) * (size_t)I);
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nt; ++i) {
            int64_t t = tokens ? tokens[i] : i;
            const double *xt = x + t * H;
            double *yt = y + i * H;
            for (int c = 0; c < H; ++c) yt[c] = 0.0;
            for (int j = 0; j < k; ++j) {
                int e = idx[t * k + j];
                const float *Wg = wgu + (int64_t)e * 2 * I * H;
                const float *Wu = Wg + (int64_t)I * H;
                const float *Wd = wd + (int64_t)e * H * I;
                for (int r = 0; r < I; ++r) {
                    double g = bgu ? (double)bgu[(int64_t)e * 2 * I + r] : 0.0;
                    double u = bgu ? (double)bgu[(int64_t)e * 2 * I + I + r] : 0.0;
                    for (int c = 0; c < H; ++c) {
                        g += xt[c] * (double)Wg[(int64_t)r * H + c];
                        u += xt[c] * (double)Wu[(int64_t)r * H + c];
                    }
                    h[r] = expert_act(act, alpha, limit, g, u, NULL, NULL);
                }
                double w = wts[t * k + j];
                for (int c = 0; c < H; ++c) {
                    double acc = bd ? (double)bd[(int64_t)e * H + c] : 0.0;
                    for (int r = 0; r < I; ++r) acc += h[r] * (double)Wd[(int64_t)c * I + r];
                    yt[c] += w * acc;
                }
            }
        }
        free(h);
    }
    return ORC_OK;
}

/* ---- input gradient ([P5] "What this adds": recompute-in-backward) -------- */

/* grad_x_t = sum_j dx_{t,j}, routing held constant:
 *   dY   = w_{t,j} * grad_out_t
 *   dh   = dY W_down,e                    (contract over H; the down bias drops out)
 *   dG   = dh * dh/dg,  dU = dh * dh/du   (expert_act's partials; for SwiGLU
 *          dh/dg = u s(g) (1 + g (1 - s(g))), dh/du = silu(g), s the logistic function)
 *   dx   = dG W_gate,e + dU W_up,e        (contract over 2I)
 * with g, u (biases included) recomputed from x and the dequantized weights. */
int e4bo_dgrad(const double *x, const double *gout, int64_t T, int E, int H, int I, int k,
               const int32_t *idx, const double *wts, const float *wgu, const float *wd,
               const int64_t *tokens, int64_t nt, int act, double alpha, double limit, const float *bgu,
               double *gx) {
    if (!x || !gout || !idx || !wts || !wgu || !wd || !gx || T < 0 || E <= 0 || k <= 0 || act < 0 || act > 1)
        return ORC_ERR_ARG;
    if (!tokens) nt = T;
#pragma omp parallel
    {
        double *dG = (double *)malloc(sizeof(double) * (size_t)I);
        double *dU = (double *)malloc(sizeof(double) * (size_t)I);
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nt; ++i) {
            int64_t t = tokens ? tokens[i] : i;
            const double *xt = x + t * H;
            const double *go = gout + t * H;
            double *gt = gx + i * H;
            for (int c = 0; c < H; ++c) gt[c] = 0.0;
            for (int j = 0; j < k; ++j) {
                int e = idx[t * k + j];
                const float *Wg = wgu + (int64_t)e * 2 * I * H;
                const float *Wu = Wg + (int64_t)I * H;
                const float *Wd = wd + (int64_t)e * H * I;
                double w = wts[t * k + j];
                for (int r = 0; r < I; ++r) {
                    double g = bgu ? (double)bgu[(int64_t)e * 2 * I + r] : 0.0;
                    double u = bgu ? (double)bgu[(int64_t)e * 2 * I + I + r] : 0.0;
                    double dh = 0.0;
                    for (int c = 0; c < H; ++c) {
                        g += xt[c] * (double)Wg[(int64_t)r * H + c];
                        u += xt[c] * (double)Wu[(int64_t)r * H + c];
                        dh += w * go[c] * (double)Wd[(int64_t)c * I + r];
                    }
                    double dhdg, dhdu;
                    expert_act(act, alpha, limit, g, u, &dhdg, &dhdu);
                    dG[r] = dh * dhdg;
                    dU[r] = dh * dhdu;
                }
                for (int c = 0; c < H; ++c) {
                    double acc = 0.0;
                    for (int r = 0; r < I; ++r)
                        acc += dG[r] * (double)Wg[(int64_t)r * H + c] + dU[r] * (double)Wu[(int64_t)r * H + c];
                    gt[c] += acc;
                }
            }
        }
        free(dG);
        free(dU);
    }
    return ORC_OK;
}

/* ---- routing gradient (the other half of the layer backward) ------------- */

/* With the routing indices held, the layer output is y_t = sum_j w_{t,j} Y_{t,j},
 * Y_{t,j} = h_{t,j} W_down,e^T the expert output before its routing weight
 * ([P4] forward: the routing weight multiplies the expert output).  So
 *   dL/dw_{t,j} = <grad_out_t, Y_{t,j}>.
 * The weights come from the logits (e4bo_route):
 *   no renormalisation: w_j = p_{e_j}, p = softmax(l) over all E, and
 *     dL/dl_i = p_i * (sum_{j: e_j = i} dw_j - sum_j dw_j p_{e_j});
 *   renormalisation: w_j = exp(l_{e_j}) / sum_j' exp(l_{e_j'}) (the full softmax
 *     denominator cancels), and
 *     dL/dl_i = sum_{j: e_j = i} w_j * (dw_j - sum_j' w_j' dw_j').
 * dw: [nt, k]; dlogits (may be NULL): [nt, E]; row i belongs to tokens[i]. */
int e4bo_router_grad(const double *x, const double *gout, const float *logits, int64_t T, int E, int H, int I,
                     int k, int renorm, const int32_t *idx, const float *wgu, const float *wd,
                     const int64_t *tokens, int64_t nt, int act, double alpha, double limit, const float *bgu,
                     const float *bd, double *dw, double *dlogits) {
    if (!x || !gout || !idx || !wgu || !wd || !dw || T < 0 || E <= 0 || k <= 0 || act < 0 || act > 1)
        return ORC_ERR_ARG;
    if (dlogits && !logits) return ORC_ERR_ARG;
    if (!tokens) nt = T;
    for (int64_t p = 0; p < T * k; ++p)
        if (idx[p] < 0 || idx[p] >= E) return ORC_ERR_ARG;
#pragma omp parallel
    {
        double *h = (double *)malloc(sizeof(double) * (size_t)I);
        double *pr = (double *)malloc(sizeof(double) * (size_t)E);
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nt; ++i) {
            int64_t t = tokens ? tokens[i] : i;
            const double *xt = x + t * H;
            const double *go = gout + t * H;
            for (int j = 0; j < k; ++j) {
                int e = idx[t * k + j];
                const float *Wg = wgu + (int64_t)e * 2 * I * H;
                const float *Wu = Wg + (int64_t)I * H;
                const float *Wd = wd + (int64_t)e * H * I;
                for (int r = 0; r < I; ++r) {
                    double g = bgu ? (double)bgu[(int64_t)e * 2 * I + r] : 0.0;
                    double u = bgu ? (double)bgu[(int64_t)e * 2 * I + I + r] : 0.0;
                    for (int c = 0; c < H; ++c) {
                        g += xt[c] * (double)Wg[(int64_t)r * H + c];
                        u += xt[c] * (double)Wu[(int64_t)r * H + c];
                    }
                    h[r] = expert_act(act, alpha, limit, g, u, NULL, NULL);
                }
                double d = 0.0;
                for (int c = 0; c < H; ++c) {
                    double yc = bd ? (double)bd[(int64_t)e * H + c] : 0.0;
                    for (int r = 0; r < I; ++r) yc += h[r] * (double)Wd[(int64_t)c * I + r];
                    d += go[c] * yc;
                }
                dw[i * k + j] = d;
            }
            if (!dlogits) continue;
            const float *l = logits + t * E;
            const int32_t *o = idx + t * k;
            double *dl = dlogits + i * E;
            for (int e = 0; e < E; ++e) dl[e] = 0.0;
            if (renorm) {
                double mx = (double)l[o[0]];
                for (int j = 1; j < k; ++j) mx = fmax(mx, (double)l[o[j]]);
                double z = 0.0;
                for (int j = 0; j < k; ++j) z += exp((double)l[o[j]] - mx);
                double a = 0.0;
                for (int j = 0; j < k; ++j) a += exp((double)l[o[j]] - mx) / z * dw[i * k + j];
                for (int j = 0; j < k; ++j) {
                    double wj = exp((double)l[o[j]] - mx) / z;
                    dl[o[j]] += wj * (dw[i * k + j] - a);
                }
            } else {
                double mx = (double)l[0];
                for (int e = 1; e < E; ++e) mx = fmax(mx, (double)l[e]);
                double z = 0.0;
                for (int e = 0; e < E; ++e) z += exp((double)l[e] - mx);
                for (int e = 0; e < E; ++e) pr[e] = exp((double)l[e] - mx) / z;
                double a = 0.0;
                for (int j = 0; j < k; ++j) a += dw[i * k + j] * pr[o[j]];
                for (int e = 0; e < E; ++e) dl[e] = -pr[e] * a;
                for (int j = 0; j < k; ++j) dl[o[j]] += pr[o[j]] * dw[i * k + j];
            }
        }
        free(h);
        free(pr);
    }
    return ORC_OK;
}

/* ---- per-expert LoRA over the frozen base ([P1] "ExpertsLoRA(base, r, alpha)",
 * "only the LoRA adapters train"; [P2] section "Prior art": stacked per-expert
 * adapters [num_experts, r, in] / [num_experts, out, r]).  Reading: both stacks
 * carry an adapter, the update is the standard LoRA one, scale = alpha / r, no
 * dropout:
 *   gu   = x W_gu,e^T + s (x A_gu,e^T) B_gu,e^T          A_gu [E,r,H], B_gu [E,2I,r]
 *   h    = expert_act(g, u)        (g = gu[0,I), u = gu[I,2I), biases as above)
 *   Y    = h W_d,e^T + s (h A_d,e^T) B_d,e^T + bd_e       A_d [E,r,I],  B_d [E,H,r]
 *   y_t  = sum_j w_{t,j} Y_{t,j}
 * Backward, routing held, base frozen (gradients summed over the pairs of each expert):
 *   dY = w grad_out_t
 *   dB_d += s dY (h A_d^T)^T   [H,r];   dA_d += s (dY B_d)^T h   [r,I]
 *   dh  = dY W_d + s (dY B_d) A_d
 *   dG, dU = dh * dh/dg, dh * dh/du;  dGU = [dG | dU]
 *   dB_gu += s dGU (x A_gu^T)^T [2I,r]; dA_gu += s (dGU B_gu)^T x [r,H]
 *   dx  = dGU W_gu + s (dGU B_gu) A_gu
 * All in fp64 over the fp32 inputs. */
static void lora_pair(const double *xt, int H, int I, int r, double s, const float *Wg, const float *Wd,
                      const float *Ag, const float *Bg, const float *Ad, const float *Bd, int act, double alpha,
                      double limit, const float *bg, const float *bd, double *za, double *gu, double *h,
                      double *zd, double *Y) {
    /* za = x A_gu^T [r]; gu = x W^T + s za B^T (+ bias) [2I] */
    for (int q = 0; q < r; ++q) {
        double a = 0.0;
        for (int c = 0; c < H; ++c) a += xt[c] * (double)Ag[(int64_t)q * H + c];
        za[q] = a;
    }
    for (int o = 0; o < 2 * I; ++o) {
        double a = bg ? (double)bg[o] : 0.0;
        for (int c = 0; c < H; ++c) a += xt[c] * (double)Wg[(int64_t)o * H + c];
        double l = 0.0;
        for (int q = 0; q < r; ++q) l += za[q] * (double)Bg[(int64_t)o * r + q];
        gu[o] = a + s * l;
    }
    for (int i = 0; i < I; ++i) h[i] = expert_act(act, alpha, limit, gu[i], gu[I + i], NULL, NULL);
    for (int q = 0; q < r; ++q) {
        double a = 0.0;
        for (int i = 0; i < I; ++i) a += h[i] * (double)Ad[(int64_t)q * I + i];
        zd[q] = a;
    }
    if (!Y) return;
    for (int c = 0; c < H; ++c) {
        double a = bd ? (double)bd[c] : 0.0;
        for (int i = 0; i < I; ++i) a += h[i] * (double)Wd[(int64_t)c * I + i];
        double l = 0.0;
        for (int q = 0; q < r; ++q) l += zd[q] * (double)Bd[(int64_t)c * r + q];
        Y[c] = a + s * l;
    }
}

int e4bo_lora_forward(const double *x, int64_t T, int E, int H, int I, int k, const int32_t *idx,
                      const double *wts, const float *wgu, const float *wd, const float *agu, const float *bgu_l,
                      const float *ad, const float *bd_l, int r, double scale, int act, double alpha,
                      double limit, const float *bgu, const float *bd, double *y) {
    if (!x || !idx || !wts || !wgu || !wd || !agu || !bgu_l || !ad || !bd_l || !y || T < 0 || E <= 0 || k <= 0 ||
        r <= 0 || act < 0 || act > 1)
        return ORC_ERR_ARG;
#pragma omp parallel
    {
        double *za = (double *)malloc(sizeof(double) * (size_t)r);
        double *zd = (double *)malloc(sizeof(double) * (size_t)r);
        double *gu = (double *)malloc(sizeof(double) * (size_t)(2 * I));
        double *h = (double *)malloc(sizeof(double) * (size_t)I);
        double *Y = (double *)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < T; ++t) {
            double *yt = y + t * H;
            for (int c = 0; c < H; ++c) yt[c] = 0.0;
            for (int j = 0; j < k; ++j) {
                int e = idx[t * k + j];
                lora_pair(x + t * H, H, I, r, scale, wgu + (int64_t)e * 2 * I * H, wd + (int64_t)e * H * I,
                          agu + (int64_t)e * r * H, bgu_l + (int64_t)e * 2 * I * r, ad + (int64_t)e * r * I,
                          bd_l + (int64_t)e * H * r, act, alpha, limit, bgu ? bgu + (int64_t)e * 2 * I : NULL,
                          bd ? bd + (int64_t)e * H : NULL, za, gu, h, zd, Y);
                for (int c = 0; c < H; ++c) yt[c] += wts[t * k + j] * Y[c];
            }
        }
        free(za); free(zd); free(gu); free(h); free(Y);
    }
    return ORC_OK;
}

/* Gradients of L = <grad_out, y>: gx [T,H], and the adapter gradients dagu [E,r,H],
 * dbgu [E,2I,r], dad [E,r,I], dbd [E,H,r] (zeroed here, summed over pairs in token
 * order, so the result does not depend on the thread count). */
int e4bo_lora_backward(const double *x, const double *gout, int64_t T, int E, int H, int I, int k,
                       const int32_t *idx, const double *wts, const float *wgu, const float *wd, const float *agu,
                       const float *bgu_l, const float *ad, const float *bd_l, int r, double scale, int act,
                       double alpha, double limit, const float *bgu, double *gx, double *dagu, double *dbgu,
                       double *dad, double *dbd) {
    if (!x || !gout || !idx || !wts || !wgu || !wd || !agu || !bgu_l || !ad || !bd_l || !gx || !dagu || !dbgu ||
        !dad || !dbd || T < 0 || E <= 0 || k <= 0 || r <= 0 || act < 0 || act > 1)
        return ORC_ERR_ARG;
    memset(dagu, 0, sizeof(double) * (size_t)E * r * H);
    memset(dbgu, 0, sizeof(double) * (size_t)E * 2 * I * r);
    memset(dad, 0, sizeof(double) * (size_t)E * r * I);
    memset(dbd, 0, sizeof(double) * (size_t)E * H * r);
    double *za = (double *)malloc(sizeof(double) * (size_t)r);
    double *zd = (double *)malloc(sizeof(double) * (size_t)r);
    double *gu = (double *)malloc(sizeof(double) * (size_t)(2 * I));
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    double *dY = (double *)malloc(sizeof(double) * (size_t)H);
    double *vb = (double *)malloc(sizeof(double) * (size_t)r);   /* dY B_d, then dGU B_gu */
    double *dh = (double *)malloc(sizeof(double) * (size_t)I);
    double *dgu = (double *)malloc(sizeof(double) * (size_t)(2 * I));
    for (int64_t t = 0; t < T; ++t) {
        const double *xt = x + t * H;
        double *gt = gx + t * H;
        for (int c = 0; c < H; ++c) gt[c] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = idx[t * k + j];
            const float *Wg = wgu + (int64_t)e * 2 * I * H, *Wd = wd + (int64_t)e * H * I;
            const float *Ag = agu + (int64_t)e * r * H, *Bg = bgu_l + (int64_t)e * 2 * I * r;
            const float *Ad = ad + (int64_t)e * r * I, *Bd = bd_l + (int64_t)e * H * r;
            double *dAg = dagu + (int64_t)e * r * H, *dBg = dbgu + (int64_t)e * 2 * I * r;
            double *dAd = dad + (int64_t)e * r * I, *dBd = dbd + (int64_t)e * H * r;
            lora_pair(xt, H, I, r, scale, Wg, Wd, Ag, Bg, Ad, Bd, act, alpha, limit,
                      bgu ? bgu + (int64_t)e * 2 * I : NULL, NULL, za, gu, h, zd, NULL);
            double w = wts[t * k + j];
            for (int c = 0; c < H; ++c) dY[c] = w * gout[t * H + c];
            /* down adapter */
            for (int q = 0; q < r; ++q) {
                double a = 0.0;
                for (int c = 0; c < H; ++c) a += dY[c] * (double)Bd[(int64_t)c * r + q];
                vb[q] = a;
            }
            for (int c = 0; c < H; ++c)
                for (int q = 0; q < r; ++q) dBd[(int64_t)c * r + q] += scale * dY[c] * zd[q];
            for (int q = 0; q < r; ++q)
                for (int i = 0; i < I; ++i) dAd[(int64_t)q * I + i] += scale * vb[q] * h[i];
            for (int i = 0; i < I; ++i) {
                double a = 0.0;
                for (int c = 0; c < H; ++c) a += dY[c] * (double)Wd[(int64_t)c * I + i];
                double l = 0.0;
                for (int q = 0; q < r; ++q) l += vb[q] * (double)Ad[(int64_t)q * I + i];
                dh[i] = a + scale * l;
            }
            /* activation */
            for (int i = 0; i < I; ++i) {
                double dg, du;
                expert_act(act, alpha, limit, gu[i], gu[I + i], &dg, &du);
                dgu[i] = dh[i] * dg;
                dgu[I + i] = dh[i] * du;
            }
            /* gate_up adapter and the input gradient */
            for (int q = 0; q < r; ++q) {
                double a = 0.0;
                for (int o = 0; o < 2 * I; ++o) a += dgu[o] * (double)Bg[(int64_t)o * r + q];
                vb[q] = a;
            }
            for (int o = 0; o < 2 * I; ++o)
                for (int q = 0; q < r; ++q) dBg[(int64_t)o * r + q] += scale * dgu[o] * za[q];
            for (int q = 0; q < r; ++q)
                for (int c = 0; c < H; ++c) dAg[(int64_t)q * H + c] += scale * vb[q] * xt[c];
            for (int c = 0; c < H; ++c) {
                double a = 0.0;
                for (int o = 0; o < 2 * I; ++o) a += dgu[o] * (double)Wg[(int64_t)o * H + c];
                double l = 0.0;
                for (int q = 0; q < r; ++q) l += vb[q] * (double)Ag[(int64_t)q * H + c];
                gt[c] += a + scale * l;
            }
        }
    }
    free(za); free(zd); free(gu); free(h); free(dY); free(vb); free(dh); free(dgu);
    return ORC_OK;
}

int e4bo_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
