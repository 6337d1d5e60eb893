/*
 * gnf4_oracle.c -- CPU oracle for the grouped NF4 W4A16 expert GEMM.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the slow, plain reference that the
 * CUDA path is checked against. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load it. It shares no code, header, table
 * or helper with the CUDA library, and the CUDA library never calls it.
 *
 * What it computes, and where the pages state it:
 *  - The grouped expert GEMM on NF4-packed weights: for every activation row
 *    m of group g (expert e = expert_ids[g]),
 *        y[m,n] = sum_k x[m,k] * NF4[code(e,n,k)] * absmax[e,n,k/64]
 *    ("grouped-nf4-gemm -- single-launch W4A16 GEMM over fused NF4 MoE expert
 *    stacks", opening section: one launch over all active experts, LUT decode,
 *    blockwise fp32 absmax, fp32 accumulation, bf16 epilogue, [E,N,K/2] uint8
 *    plus fp32 absmax with (sizes, expert_ids) after the token->expert sort).
 *    The oracle computes this definition in fp64: bf16 x widens exactly, and
 *    NF4[c]*absmax is exact in fp64 (24 + 24 significant bits < 53).
 *  - The dequantise-then-matmul baseline the method replaces (same section:
 *    the bf16 weight copy is written and read again; fp32 accumulation makes
 *    the fused path more accurate than that baseline). Emulated here as
 *    w_bf16 = RNE_bf16(fl32(NF4[c]*absmax)), fp32 accumulation in ascending k,
 *    one bf16 rounding of the result.
 *  - The token->expert sort that produces (sizes, expert_ids) (same section:
 *    "the usual token->expert sort"). Reading taken: a stable counting sort of
 *    the flat slots s = t*top_k + j by expert id; groups are the non-empty
 *    experts in ascending id; within a group slots keep ascending s.
 *  - NF4 quantisation (bitsandbytes gemm_4bit conventions, named in the same
 *    section and on the "grouped-nf4-gemm" package page, "Direct answer"):
 *    64-element blocks along K, absmax = max |w| in fp32, code = nearest NF4
 *    value to w/absmax (ties to the lower index), byte j of a row holds k=2j in
 *    the high nibble and k=2j+1 in the low nibble. Only used to make inputs.
 *  - SwiGLU on the gate_up output ("grouped-nf4-gemm" package page, "Owns":
 *    decode glue kernels including swiglu). Reading taken: gate = columns
 *    [0, N/2), up = [N/2, N), silu(g) = g / (1 + exp(-g)).
 *
 * Build flags matter: -ffp-contract=off keeps every product a separately
 * rounded single multiply (no silent fusing into an FMA).
 *
 * The NF4 code table is the one published with the NF4 data type (QLoRA,
 * Dettmers et al. 2023) and used by bitsandbytes; the pages name the
 * bitsandbytes layout but do not print the table. The tests pin it against
 * its closed form (normal quantiles), independently of this file.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define GNF4O_BLOCK 64

/* Status codes returned by the oracle (0 = ok). */
enum { ORC_OK = 0, ORC_BAD_SHAPE = 1, ORC_BAD_SIZES = 2, ORC_BAD_EXPERT = 3, ORC_BAD_TOPK = 4,
       ORC_BAD_SLOT = 5 };

static const float NF4_TABLE[16] = {
    -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,
    -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,
    0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f, 0.33791524171829224f,
    0.44070982933044434f, 0.5626170039176941f, 0.7229568362236023f, 1.0f};

void oracle_nf4_table(float *out16) { memcpy(out16, NF4_TABLE, sizeof(NF4_TABLE)); }

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Code of element k in a packed row: high nibble for even k, low for odd k. */
static inline int code_at(const uint8_t *row, int64_t k) {
    uint8_t b = row[k >> 1];
    return (k & 1) ? (b & 0x0F) : (b >> 4);
}

/* ---------------------------------------------------------------- bf16 */
/* Round an fp32 value to bf16, round-to-nearest-even on the bit pattern. */
static inline uint16_t bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40u); /* quiet NaN */
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static inline float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

void oracle_f32_to_bf16(const float *in, int64_t n, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_rne(in[i]);
}

/* ----------------------------------------------------------- quantiser */
/* Quantise R rows of K fp32 weights (K % 64 == 0) to packed NF4 + absmax. */
int oracle_quantize_nf4(const float *w, int64_t R, int64_t K, uint8_t *packed, float *absmax) {
    if (R < 0 || K <= 0 || K % GNF4O_BLOCK) return ORC_BAD_SHAPE;
    const int64_t nb = K / GNF4O_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        const float *wr = w + r * K;
        uint8_t *pr = packed + r * (K / 2);
        for (int64_t b = 0; b < nb; ++b) {
            float amax = 0.0f;
            for (int64_t i = 0; i < GNF4O_BLOCK; ++i) {
                float a = fabsf(wr[b * GNF4O_BLOCK + i]);
                if (a > amax) amax = a;
            }
            absmax[r * nb + b] = amax;
            for (int64_t i = 0; i < GNF4O_BLOCK; i += 2) {
                int c[2];
                for (int h = 0; h < 2; ++h) {
                    int best = 7; /* all-zero block: every code is the 0.0 entry */
                    if (amax > 0.0f) {
                        float v = wr[b * GNF4O_BLOCK + i + h] / amax;
                        float bd = INFINITY;
                        for (int q = 0; q < 16; ++q) {
                            float d = fabsf(NF4_TABLE[q] - v);
                            if (d < bd) { bd = d; best = q; } /* strict: ties keep lower index */
                        }
                    }
                    c[h] = best;
                }
                pr[(b * GNF4O_BLOCK + i) / 2] = (uint8_t)((c[0] << 4) | c[1]);
            }
        }
    }
    return ORC_OK;
}

/* -------------------------------------------------------------- dequant */
/* fp32 dequantisation: one IEEE single multiply per element. */
int oracle_dequant_f32(const uint8_t *packed, const float *absmax, int64_t R, int64_t K, float *out) {
    if (R < 0 || K <= 0 || K % GNF4O_BLOCK) return ORC_BAD_SHAPE;
    const int64_t nb = K / GNF4O_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        const uint8_t *pr = packed + r * (K / 2);
        for (int64_t k = 0; k < K; ++k) {
            out[r * K + k] = NF4_TABLE[code_at(pr, k)] * absmax[r * nb + k / GNF4O_BLOCK];
        }
    }
    return ORC_OK;
}

/* bf16 dequantisation: the fp32 product above, rounded once to bf16. */
int oracle_dequant_bf16(const uint8_t *packed, const float *absmax, int64_t R, int64_t K, uint16_t *out) {
    if (R < 0 || K <= 0 || K % GNF4O_BLOCK) return ORC_BAD_SHAPE;
    const int64_t nb = K / GNF4O_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        const uint8_t *pr = packed + r * (K / 2);
        for (int64_t k = 0; k < K; ++k) {
            const float prod = NF4_TABLE[code_at(pr, k)] * absmax[r * nb + k / GNF4O_BLOCK];
            out[r * K + k] = bf16_rne(prod);
        }
    }
    return ORC_OK;
}

/* ----------------------------------------------------------- moe_align */
/* Stable counting sort of the T*top_k slots by expert id.
 * Outputs: sorted_idx[T*top_k] (flat slot indices, grouped, ascending within a
 * group), sizes[E], expert_ids[E] (first num_groups entries describe the
 * non-empty experts in ascending id; the rest are sizes=0, expert_ids=-1) and
 * num_groups. Returns ORC_BAD_TOPK if an id is outside [0, E). */
int oracle_moe_align(const int32_t *topk_ids, int64_t T, int32_t top_k, int32_t E,
                     int32_t *sorted_idx, int32_t *sizes, int32_t *expert_ids, int32_t *num_groups) {
    if (T < 0 || top_k <= 0 || E <= 0) return ORC_BAD_SHAPE;
    const int64_t S = T * top_k;
    int64_t *count = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    int64_t *cursor = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    if (!count || !cursor) { free(count); free(cursor); return ORC_BAD_SHAPE; }
    for (int64_t s = 0; s < S; ++s) {
        int32_t e = topk_ids[s];
        if (e < 0 || e >= E) { free(count); free(cursor); return ORC_BAD_TOPK; }
        count[e]++;
    }
    int32_t g = 0;
    int64_t start = 0;
    for (int32_t e = 0; e < E; ++e) {
        cursor[e] = start;
        start += count[e];
        if (count[e] > 0) { sizes[g] = (int32_t)count[e]; expert_ids[g] = e; ++g; }
    }
    for (int32_t q = g; q < E; ++q) { sizes[q] = 0; expert_ids[q] = -1; }
    *num_groups = g;
    for (int64_t s = 0; s < S; ++s) sorted_idx[cursor[topk_ids[s]]++] = (int32_t)s;
    free(count);
    free(cursor);
    return ORC_OK;
}

/* ------------------------------------------------------- group lookup */
/* Validate (sizes, expert_ids) against M and E and fill row -> expert. */
static int rows_to_expert(const int32_t *sizes, const int32_t *expert_ids, int32_t G, int64_t M,
                          int32_t E, int32_t *row_expert) {
    int64_t off = 0;
    for (int32_t g = 0; g < G; ++g) {
        if (sizes[g] < 0) return ORC_BAD_SIZES;
        if (sizes[g] > 0 && (expert_ids[g] < 0 || expert_ids[g] >= E)) return ORC_BAD_EXPERT;
        if (off + sizes[g] > M) return ORC_BAD_SIZES;
        for (int64_t i = 0; i < sizes[g]; ++i) row_expert[off + i] = expert_ids[g];
        off += sizes[g];
    }
    return off == M ? ORC_OK : ORC_BAD_SIZES;
}

/* -------------------------------------------------- grouped GEMM (fp64) */
/* y[r, n] for the requested rows (rows == NULL: all M rows, in order).
 * x: bf16 bits [M, K]; w: [E, N, K/2]; absmax: [E, N, K/64]; y: fp64 [nrows, N]. */
int oracle_grouped_gemm_f64(const uint16_t *x, const uint8_t *w, const float *absmax,
                            const int32_t *sizes, const int32_t *expert_ids, int32_t G, int64_t M,
                            int32_t N, int32_t K, int32_t E, const int64_t *rows, int64_t nrows,
                            double *y) {
    if (M < 0 || N <= 0 || K <= 0 || K % GNF4O_BLOCK || E <= 0 || G < 0) return ORC_BAD_SHAPE;
    int32_t *row_expert = (int32_t *)malloc((size_t)(M > 0 ? M : 1) * sizeof(int32_t));
    if (!row_expert) return ORC_BAD_SHAPE;
    int st = rows_to_expert(sizes, expert_ids, G, M, E, row_expert);
    if (st != ORC_OK) { free(row_expert); return st; }
    if (!rows) nrows = M;
    for (int64_t i = 0; i < nrows; ++i) {
        if (rows && (rows[i] < 0 || rows[i] >= M)) { free(row_expert); return ORC_BAD_SHAPE; }
    }
    const int64_t nb = K / GNF4O_BLOCK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t m = rows ? rows[i] : i;
        const int32_t e = row_expert[m];
        double *xr = (double *)malloc((size_t)K * sizeof(double));
        for (int32_t k = 0; k < K; ++k) xr[k] = (double)bf16_to_f32(x[m * K + k]);
        for (int32_t n = 0; n < N; ++n) {
            const int64_t row = (int64_t)e * N + n;
            const uint8_t *wr = w + row * (K / 2);
            const float *ar = absmax + row * nb;
            double acc = 0.0;
            for (int32_t k = 0; k < K; ++k) {
                double wv = (double)NF4_TABLE[code_at(wr, k)] * (double)ar[k / GNF4O_BLOCK];
                acc += xr[k] * wv;
            }
            y[i * N + n] = acc;
        }
        free(xr);
    }
    free(row_expert);
    return ORC_OK;
}

/* ------------------------------------------------ MXFP4 grouped GEMM (fp64) */
/* The same grouped GEMM over native MXFP4 weights ("grouped-nf4-gemm" package
 * page, "Direct answer": e2m1 codes with e8m0 scales, multiplied as released,
 * no requantisation). Format (OCP microscaling FP4, the layout of the
 * released gpt-oss expert blocks): byte j of a row holds element k = 2j in the
 * LOW nibble and k = 2j+1 in the HIGH nibble; each code is an e2m1 number
 * (1 sign, 2 exponent bits with bias 1, 1 mantissa bit; exponent field 0 is
 * the subnormal 0 or 0.5); scales[e][n][b] is one e8m0 byte per 32
 * consecutive elements, the power of two 2^(s-127) (255 is NaN). The
 * product code * scale is exact in fp64. */
static double e2m1_value(int c) {
    const int sgn = (c >> 3) & 1, ex = (c >> 1) & 3, man = c & 1;
    double mag = ex == 0 ? 0.5 * man : ldexp(1.0 + 0.5 * man, ex - 1);
    return sgn ? -mag : mag;
}

static double e8m0_value(uint8_t s) { return s == 255 ? NAN : ldexp(1.0, (int)s - 127); }

void oracle_e2m1_table(double *out16) {
    for (int c = 0; c < 16; ++c) out16[c] = e2m1_value(c);
}

int oracle_grouped_gemm_mxfp4_f64(const uint16_t *x, const uint8_t *w, const uint8_t *scales,
                                  const int32_t *sizes, const int32_t *expert_ids, int32_t G,
                                  int64_t M, int32_t N, int32_t K, int32_t E, const int64_t *rows,
                                  int64_t nrows, double *y) {
    if (M < 0 || N <= 0 || K <= 0 || K % 32 || E <= 0 || G < 0) return ORC_BAD_SHAPE;
    int32_t *row_expert = (int32_t *)malloc((size_t)(M > 0 ? M : 1) * sizeof(int32_t));
    if (!row_expert) return ORC_BAD_SHAPE;
    int st = rows_to_expert(sizes, expert_ids, G, M, E, row_expert);
    if (st != ORC_OK) { free(row_expert); return st; }
    if (!rows) nrows = M;
    for (int64_t i = 0; i < nrows; ++i) {
        if (rows && (rows[i] < 0 || rows[i] >= M)) { free(row_expert); return ORC_BAD_SHAPE; }
    }
    const int64_t nb = K / 32;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t m = rows ? rows[i] : i;
        const int32_t e = row_expert[m];
        double *xr = (double *)malloc((size_t)K * sizeof(double));
        for (int32_t k = 0; k < K; ++k) xr[k] = (double)bf16_to_f32(x[m * K + k]);
        for (int32_t n = 0; n < N; ++n) {
            const int64_t row = (int64_t)e * N + n;
            const uint8_t *wr = w + row * (K / 2);
            const uint8_t *sr = scales + row * nb;
            double acc = 0.0;
            for (int32_t k = 0; k < K; ++k) {
                const uint8_t byte = wr[k >> 1];
                const int code = (k & 1) ? (byte >> 4) : (byte & 0x0F);
                acc += xr[k] * (e2m1_value(code) * e8m0_value(sr[k / 32]));
            }
            y[i * N + n] = acc;
        }
        free(xr);
    }
    free(row_expert);
    return ORC_OK;
}

/* -------------------------------- SwiGLU on interleaved gate/up, clamped */
/* The gpt-oss form of the gated activation (its published model definition),
 * listed with the absmax variants among the next steps of this path: gate =
 * even columns, up = odd columns of the gate_up output y [M, N]; the gate is
 * clamped from above at `limit`, the up value to [-limit, limit];
 * out[m, j] = g * sigmoid(alpha * g) * (u + 1), in fp64. */
int oracle_swiglu_interleaved_f64(const double *y, int64_t M, int32_t N, double alpha,
                                  double limit, double *out) {
    if (M < 0 || N <= 0 || N % 2) return ORC_BAD_SHAPE;
    const int32_t H = N / 2;
    for (int64_t m = 0; m < M; ++m)
        for (int32_t j = 0; j < H; ++j) {
            double g = y[m * N + 2 * j], u = y[m * N + 2 * j + 1];
            if (g > limit) g = limit;
            if (u > limit) u = limit;
            if (u < -limit) u = -limit;
            out[m * H + j] = g / (1.0 + exp(-alpha * g)) * (u + 1.0);
        }
    return ORC_OK;
}

/* ------------------------------------------------------------ row gather */
/* The activation rows of the sorted order: x[i] = hidden[sorted_idx[i] / top_k]
 * (bf16 bits; the gather the token->expert sort implies, "grouped-nf4-gemm"
 * package page, "Use this when", folded into the GEMM). */
int oracle_gather_rows(const uint16_t *hidden, int64_t T, int32_t K, const int32_t *sorted_idx,
                       int64_t M, int32_t top_k, uint16_t *x) {
    if (T < 0 || K <= 0 || M < 0 || top_k < 1) return ORC_BAD_SHAPE;
    for (int64_t i = 0; i < M; ++i) {
        const int32_t s = sorted_idx[i];
        if (s < 0 || (int64_t)s >= T * top_k) return ORC_BAD_SLOT;
        memcpy(x + i * K, hidden + (int64_t)(s / top_k) * K, (size_t)K * sizeof(uint16_t));
    }
    return ORC_OK;
}

/* SwiGLU on an fp64 [M, N] gate_up output: out[m, j] = silu(y[m, j]) * y[m, j + N/2]. */
int oracle_swiglu_f64(const double *y, int64_t M, int32_t N, double *out) {
    if (M < 0 || N <= 0 || N % 2) return ORC_BAD_SHAPE;
    const int32_t H = N / 2;
    for (int64_t m = 0; m < M; ++m)
        for (int32_t j = 0; j < H; ++j) {
            double g = y[m * N + j], u = y[m * N + H + j];
            out[m * H + j] = g / (1.0 + exp(-g)) * u;
        }
    return ORC_OK;
}

/* ------------------------------------- dequant-to-bf16-then-matmul baseline */
/* Emulates the path the method replaces: bf16 weights materialised from the
 * fp32 product, fp32 accumulation in ascending k (one fused multiply-add per
 * step), one bf16 rounding of the result. Output: bf16 bits [nrows, N]. */
int oracle_baseline_bf16(const uint16_t *x, const uint8_t *w, const float *absmax,
                         const int32_t *sizes, const int32_t *expert_ids, int32_t G, int64_t M,
                         int32_t N, int32_t K, int32_t E, const int64_t *rows, int64_t nrows,
                         uint16_t *y) {
    if (M < 0 || N <= 0 || K <= 0 || K % GNF4O_BLOCK || E <= 0 || G < 0) return ORC_BAD_SHAPE;
    int32_t *row_expert = (int32_t *)malloc((size_t)(M > 0 ? M : 1) * sizeof(int32_t));
    if (!row_expert) return ORC_BAD_SHAPE;
    int st = rows_to_expert(sizes, expert_ids, G, M, E, row_expert);
    if (st != ORC_OK) { free(row_expert); return st; }
    if (!rows) nrows = M;
    const int64_t nb = K / GNF4O_BLOCK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t m = rows ? rows[i] : i;
        const int32_t e = row_expert[m];
        for (int32_t n = 0; n < N; ++n) {
            const int64_t row = (int64_t)e * N + n;
            const uint8_t *wr = w + row * (K / 2);
            const float *ar = absmax + row * nb;
            float acc = 0.0f;
            for (int32_t k = 0; k < K; ++k) {
                const float prod = NF4_TABLE[code_at(wr, k)] * ar[k / GNF4O_BLOCK];
                float wb = bf16_to_f32(bf16_rne(prod));
                acc = fmaf(bf16_to_f32(x[m * K + k]), wb, acc);
            }
            y[i * N + n] = bf16_rne(acc);
        }
    }
    free(row_expert);
    return ORC_OK;
}

/* SwiGLU of the dequantise-then-matmul baseline, applied to its bf16 gate_up
 * output yb [M, N] (bf16 bits): the gate and up values as the baseline
 * materialised them (bf16, widened exactly to fp32), silu(g) = g / (1 + e^-g)
 * and the product with up in fp32, one bf16 rounding. Output: bf16 bits
 * [M, N/2]. This is the baseline side of the fidelity comparison for a fused
 * SwiGLU ("grouped-nf4-gemm -- single-launch W4A16 GEMM ...", "The claim":
 * fused error below the dequantise-then-matmul path's; the package page's
 * "Owns" names swiglu among the glue that follows gate_up). Reading taken:
 * the baseline rounds its GEMM output to bf16 before the activation. */
int oracle_baseline_swiglu_bf16(const uint16_t *yb, int64_t M, int32_t N, uint16_t *out) {
    if (M < 0 || N <= 0 || N % 2) return ORC_BAD_SHAPE;
    const int32_t H = N / 2;
    for (int64_t m = 0; m < M; ++m)
        for (int32_t j = 0; j < H; ++j) {
            const float g = bf16_to_f32(yb[m * N + j]);
            const float u = bf16_to_f32(yb[m * N + H + j]);
            const float silu = g / (1.0f + expf(-g));
            out[m * H + j] = bf16_rne(silu * u);
        }
    return ORC_OK;
}

/* ------------------------------------------------------ router top-k */
/* Per token: the top_k experts by logit, picked one at a time as the largest
   remaining logit (equal logits: the lower expert id; a NaN logit counts as
   -inf), and their softmax weights in fp64, exp(l - l_max) over the sum of
   exp(l_e - l_max) for all E experts (renorm == 0) or for the selected ones
   (renorm == 1). Package page "grouped-nf4-gemm", "Use this when" (router
   softmax and top-k). */
int oracle_router_topk(const float *logits, int64_t T, int32_t E, int32_t k, int32_t renorm,
                       int32_t *ids, double *weights) {
  if (T < 0 || E < 1 || k < 1 || k > E) return ORC_BAD_SHAPE;
  for (int64_t t = 0; t < T; ++t) {
    const float *row = logits + t * E;
    int32_t *sel = ids + t * k;
    for (int j = 0; j < k; ++j) {
      int best = -1;
      double bv = 0.0;
      for (int e = 0; e < E; ++e) {
        int taken = 0;
        for (int i = 0; i < j; ++i) taken |= sel[i] == e;
        if (taken) continue;
        const double v = isnan(row[e]) ? -INFINITY : (double)row[e];
        if (best < 0 || v > bv) {   /* strict: an equal logit keeps the lower id */
          best = e;
          bv = v;
        }
      }
      sel[j] = best;
    }
    const double lmax = isnan(row[sel[0]]) ? -INFINITY : (double)row[sel[0]];
    double den = 0.0;
    if (renorm) {
      for (int j = 0; j < k; ++j) den += exp((double)row[sel[j]] - lmax);
    } else {
      for (int e = 0; e < E; ++e) den += exp((double)row[e] - lmax);
    }
    for (int j = 0; j < k; ++j) weights[t * k + j] = exp((double)row[sel[j]] - lmax) / den;
  }
  return ORC_OK;
}

/* ---------------------------------------------------- weighted combine */
/* out[t][h] = sum_{j < k} w[t][j] * y[p(t*k + j)][h] in fp64, where p(s) is
   the position of slot s in sorted_idx (entries of -1 are slots left out and
   contribute nothing). Package page "grouped-nf4-gemm", "Owns" and "Use this
   when" (the top-k combine). */
int oracle_moe_combine(const uint16_t *y, const int32_t *sorted_idx, const float *w, int64_t T,
                       int32_t k, int32_t H, double *out) {
  if (T < 0 || k < 1 || H < 1) return ORC_BAD_SHAPE;
  const int64_t S = T * k;
  int64_t *pos = (int64_t *)malloc((size_t)(S > 0 ? S : 1) * sizeof(int64_t));
  if (!pos) return ORC_BAD_SHAPE;
  for (int64_t s = 0; s < S; ++s) pos[s] = -1;
  for (int64_t i = 0; i < S; ++i) {
    const int32_t s = sorted_idx[i];
    if (s == -1) continue;
    if (s < 0 || s >= S) {
      free(pos);
      return ORC_BAD_SLOT;
    }
    pos[s] = i;
  }
  for (int64_t t = 0; t < T; ++t) {
    for (int32_t h = 0; h < H; ++h) {
      double acc = 0.0;
      for (int32_t j = 0; j < k; ++j) {
        const int64_t p = pos[t * k + j];
        if (p < 0) continue;
        acc += (double)w[t * k + j] * (double)bf16_to_f32(y[p * H + h]);
      }
      out[t * H + h] = acc;
    }
  }
  free(pos);
  return ORC_OK;
}

/* ------------------------------------------------ grouped dgrad (fp64) */
/* The gradient of the grouped GEMM with respect to its activations:
   dx[m, k] = sum_n dy[m, n] * NF4[code(e, n, k)] * absmax[e, n, k/64], e the
   expert of row m's group, in fp64 (the same weight values as the forward
   oracle). Package page "grouped-nf4-gemm", header block ("Owns": the grouped
   packed GEMM and its dgrad).
   dy: bf16 bits [M, N]; w: [E, N, K/2]; absmax: [E, N, K/64]; dx: fp64 [M, K]. */
int oracle_grouped_dgrad_f64(const uint16_t *dy, const uint8_t *w, const float *absmax,
                             const int32_t *sizes, const int32_t *expert_ids, int32_t G,
                             int64_t M, int32_t N, int32_t K, int32_t E, double *dx) {
    if (M < 0 || N <= 0 || K <= 0 || K % GNF4O_BLOCK || E <= 0 || G < 0) return ORC_BAD_SHAPE;
    int32_t *row_expert = (int32_t *)malloc((size_t)(M > 0 ? M : 1) * sizeof(int32_t));
    if (!row_expert) return ORC_BAD_SHAPE;
    int st = rows_to_expert(sizes, expert_ids, G, M, E, row_expert);
    if (st != ORC_OK) { free(row_expert); return st; }
    const int64_t nb = K / GNF4O_BLOCK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        const int32_t e = row_expert[m];
        double *acc = dx + m * K;
        for (int32_t k = 0; k < K; ++k) acc[k] = 0.0;
        for (int32_t n = 0; n < N; ++n) {
            const double g = (double)bf16_to_f32(dy[m * N + n]);
            const int64_t row = (int64_t)e * N + n;
            const uint8_t *wr = w + row * (K / 2);
            const float *ar = absmax + row * nb;
            for (int32_t k = 0; k < K; ++k)
                acc[k] += g * ((double)NF4_TABLE[code_at(wr, k)] * (double)ar[k / GNF4O_BLOCK]);
        }
    }
    free(row_expert);
    return ORC_OK;
}
