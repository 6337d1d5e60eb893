/*
 * gnf4.h -- C ABI of libgnf4: the grouped MoE expert GEMM computed directly on
 * NF4-packed weights, for NVIDIA B200 (sm_100a).
 *
 * Source of the operation: "grouped-nf4-gemm -- single-launch W4A16 GEMM over
 * fused NF4 MoE expert stacks" (PyPI README of grouped_nf4_gemm 0.1.0), opening
 * section: one launch over all active experts; LUT decode of 4-bit NF4 codes,
 * blockwise fp32 absmax, fp32 accumulation, bf16 epilogue; no per-expert
 * dequantise-then-matmul and no bf16 weight copy; inputs in the bitsandbytes
 * gemm_4bit layout, [E, N, K/2] uint8 plus fp32 blockwise absmax, with
 * (sizes, expert_ids) supplied after the token->expert sort. The package page
 * "grouped-nf4-gemm" ("Do not use this when") adds that nothing falls back
 * silently: host tensors are refused with an error.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Plain pointers and sizes only. The caller owns all memory: inputs,
 *    outputs and the workspace. The library allocates nothing.
 *  - All work is enqueued asynchronously on `stream` (NULL = legacy default
 *    stream). No entry point synchronises the stream or copies to the host,
 *    except gnf4_read_device_status, which exists to do exactly that.
 *  - Host-side checks run first and synchronously; on failure nothing is
 *    launched and a status != GNF4_OK is returned. Pointers that are not
 *    device memory (host or unregistered) give GNF4_ERR_HOST_POINTER.
 *  - Data that only the device knows (sizes, expert_ids, topk_ids, sorted_idx) is checked
 *    on the device. A violation sets a bit in the workspace's error word (see
 *    GNF4_DEVERR_*) and the kernel skips the affected work; it never traps.
 *    Read the word with gnf4_read_device_status.
 *  - Every device-side wait is bounded; a wait that runs out sets
 *    GNF4_DEVERR_TIMEOUT and the kernel returns.
 *  - bf16 tensors are passed as uint16_t bit patterns.
 *
 * Weight layout (NF4, bitsandbytes gemm_4bit conventions):
 *    w[e][n][j]        uint8, j < K/2: element k=2j in the HIGH nibble (bits
 *                      7..4), element k=2j+1 in the LOW nibble (bits 3..0).
 *    absmax[e][n][b]   fp32, b < K/64: scale of elements k in [64b, 64b+64).
 *    value(e,n,k)      = NF4[code] * absmax[e][n][k/64], NF4 = the 16-entry
 *                        normal-float table of QLoRA/bitsandbytes.
 */
#ifndef GNF4_H
#define GNF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GNF4_VERSION 120 /* 1.2.0: + gnf4_grouped_gemm_ex (MXFP4, bf16 absmax, gather, gpt-oss SwiGLU) */

/* Exported entry points (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define GNF4_API __attribute__((visibility("default")))
#else
#define GNF4_API
#endif

/* A CUDA stream handle (identical to cudaStream_t). */
typedef struct CUstream_st *gnf4_stream_t;

typedef enum {
    GNF4_OK = 0,
    GNF4_ERR_INVALID_ARGUMENT = 1,    /* null pointer, bad enum, negative size */
    GNF4_ERR_HOST_POINTER = 2,        /* a pointer is not device memory */
    GNF4_ERR_UNSUPPORTED_SHAPE = 3,   /* K % 64, blocksize != 64, odd N with SwiGLU, limits */
    GNF4_ERR_WORKSPACE_TOO_SMALL = 4, /* ws_bytes < gnf4_workspace_bytes(...) */
    GNF4_ERR_CUDA = 5,                /* a CUDA runtime call or launch failed */
    GNF4_ERR_DEVICE_METADATA = 6,     /* (read_device_status) device data was invalid */
    GNF4_ERR_TIMEOUT = 7,             /* (read_device_status) a bounded device wait ran out */
    GNF4_ERR_MISALIGNED = 8,          /* a pointer breaks the alignment rule below */
    GNF4_ERR_SCRATCH_LIMIT = 9        /* problem needs more than the fixed scratch of
                                         gnf4_grouped_gemm_noalloc */
} gnf4_status;

typedef enum {
    GNF4_EPI_NONE = 0,
    GNF4_EPI_SWIGLU = 1,              /* silu(gate) * up, gate = columns [0, N/2), up = [N/2, N) */
    GNF4_EPI_SWIGLU_INTERLEAVED = 2   /* gate = even columns, up = odd columns, clamped; see
                                         gnf4_grouped_gemm_ex */
} gnf4_epilogue;
typedef enum {
    GNF4_FMT_NF4 = 0,                 /* NF4 codes (bitsandbytes layout) + absmax per 64 */
    GNF4_FMT_MXFP4 = 1                /* e2m1 codes + e8m0 scale per 32 (OCP microscaling) */
} gnf4_format;
typedef enum {
    GNF4_SCALE_F32 = 0,               /* NF4 absmax as fp32 */
    GNF4_SCALE_BF16 = 1,              /* NF4 absmax as bf16 */
    GNF4_SCALE_E8M0 = 2               /* MXFP4 scales: one byte 2^(s-127) per 32 elements */
} gnf4_scale_dtype;
typedef enum { GNF4_MODE_AUTO = 0, GNF4_MODE_DECODE = 1, GNF4_MODE_PREFILL = 2 } gnf4_mode;
typedef enum { GNF4_OUT_F32 = 0, GNF4_OUT_BF16 = 1 } gnf4_out_dtype;
typedef enum {
    GNF4_OP_MOE_ALIGN = 0,
    GNF4_OP_GROUPED_GEMM = 1,
    GNF4_OP_MOE_COMBINE = 2,
    GNF4_OP_GROUPED_DGRAD = 3
} gnf4_op;

/* Bits of the device error word (gnf4_read_device_status). */
#define GNF4_DEVERR_SIZES 0x1u      /* a size < 0, or sum(sizes) != M */
#define GNF4_DEVERR_EXPERT 0x2u     /* expert_ids[g] outside [0, E) on a non-empty group */
#define GNF4_DEVERR_TOPK 0x4u       /* a topk id outside [0, E) */
#define GNF4_DEVERR_TIMEOUT 0x8u    /* a bounded wait ran out */
#define GNF4_DEVERR_CAPACITY 0x10u  /* a kernel's on-chip layout did not fit what the
                                       device provides (the decode kernel's shared
                                       memory window; not expected on sm_100a) */
#define GNF4_DEVERR_SLOT 0x20u      /* (moe_combine) a sorted_idx entry outside
                                       [-1, T*top_k) */

/* Limits. */
#define GNF4_MAX_EXPERTS 1024       /* E (and G) */
#define GNF4_BLOCKSIZE 64           /* the only absmax block size */
#define GNF4_MAX_TOPK 32            /* top_k of gnf4_router_topk */

/*
 * gnf4_moe_align -- the token->expert sort that produces (sizes, expert_ids).
 *
 * Passage: README opening section, "(sizes, expert_ids) supplied after the
 * usual token->expert sort". The pages do not define the sort further; this
 * library fixes it as a stable counting sort:
 *   - slots are the flat indices s = t*top_k + j of topk_ids[T][top_k];
 *   - groups are the experts that received at least one slot, in ascending
 *     expert id; sizes[g] = slot count, expert_ids[g] = expert id, for
 *     g < *num_groups; entries g >= *num_groups are sizes=0, expert_ids=-1;
 *   - sorted_idx lists the slots group by group, ascending s within a group;
 *     the caller gathers x_sorted[i] = hidden[sorted_idx[i] / top_k].
 * Arrays sizes/expert_ids have E entries so they feed gnf4_grouped_gemm with
 * G = E and no host synchronisation. Duplicate experts within a token count
 * twice. A topk id outside [0, E) sets GNF4_DEVERR_TOPK; such slots are left
 * out of every group and sorted_idx is padded with -1 at its tail.
 *
 *   topk_ids    device int32 [T*top_k], row-major [T][top_k] (may be NULL if T == 0)
 *   T >= 0, 1 <= top_k, 1 <= E <= GNF4_MAX_EXPERTS, T*top_k < 2^31
 *   sorted_idx  device int32 [T*top_k]    (written; may be NULL if T == 0)
 *   sizes       device int32 [E]          (written)
 *   expert_ids  device int32 [E]          (written)
 *   num_groups  device int32 [1]          (written)
 *   workspace   device, >= gnf4_workspace_bytes(GNF4_OP_MOE_ALIGN, ...) bytes,
 *               zero-filled once by the caller before its first use.
 * One kernel launch.
 */
GNF4_API gnf4_status gnf4_moe_align(const int32_t *topk_ids, int64_t T, int32_t top_k, int32_t E,
                           int32_t *sorted_idx, int32_t *sizes, int32_t *expert_ids,
                           int32_t *num_groups, void *workspace, size_t ws_bytes,
                           gnf4_stream_t stream);

/*
 * gnf4_grouped_gemm -- y = x . W^T per group, on NF4-packed W, one launch.
 *
 * Passage: README opening section (the whole operation, quoted in substance
 * at the top of this file); "The claim" (fp32 accumulation, more accurate than
 * materialising bf16 weights). Rows of x are already sorted by group: group g
 * owns rows [sum(sizes[0..g)), sum(sizes[0..g])) and multiplies expert
 * expert_ids[g]. For every row m of group g and column n:
 *     acc[m][n] = sum_k x[m][k] * NF4[code(e,n,k)] * absmax[e][n][k/64]   (fp32)
 *     epilogue NONE:   y[m][n] = bf16_rne(acc[m][n]),            y is [M][N]
 *     epilogue SWIGLU: y[m][j] = bf16_rne(silu(acc[m][j]) * acc[m][j+N/2]),
 *                      j < N/2, silu(g) = g/(1+exp(-g)),          y is [M][N/2]
 * No bf16 (or other) copy of the weights is written anywhere.
 *
 *   x           device bf16 [M][K] (uint16 bit patterns), row stride K
 *   w           device uint8 [E][N][K/2]
 *   absmax      device fp32 [E][N][K/64]
 *   sizes       device int32 [G]; sizes[g] >= 0, sum == M (checked on device)
 *   expert_ids  device int32 [G]; in [0, E) where sizes[g] > 0, else ignored
 *   1 <= G <= GNF4_MAX_EXPERTS; M >= 0 (M == 0: returns GNF4_OK, no launch)
 *   N >= 1 (even for SWIGLU); K >= 64, K % 64 == 0; 1 <= E <= GNF4_MAX_EXPERTS
 *   blocksize   must be 64
 *   epilogue    gnf4_epilogue
 *   mode        gnf4_mode: AUTO picks DECODE when the mean rows per possible
 *               group, M / min(G, E), is at most 64, else PREFILL. Both modes
 *               accept any group sizes and both epilogues; the mode only
 *               selects the kernel.
 *   y           device bf16 [M][N] or [M][N/2]; fully overwritten; must not
 *               overlap x, w, absmax or the workspace.
 *   workspace   device, >= gnf4_workspace_bytes(GNF4_OP_GROUPED_GEMM, M, N, K, E, G)
 *               bytes (which covers every mode; the call itself only checks
 *               the need of the kernel it runs and refuses less with
 *               GNF4_ERR_WORKSPACE_TOO_SMALL). Its first 256 bytes are the
 *               device status header: zero the whole workspace once before
 *               the first use. Word 2 of the header (bytes 8..11), when not
 *               zero, shortens every bounded wait of the DECODE kernel to
 *               that many nanoseconds (a test hook; 0 = the 2 s default).
 *               DECODE then uses, after the header, one counter per
 *               (SM, unit pair) (zero between calls: each call leaves them
 *               at zero) and the fp32 partial sums of the tiles its stream-K
 *               split cuts (8 KB per SM). PREFILL writes, after the header,
 *               the row-scaled operands of x: an e5m2 copy (M*K bytes,
 *               rounded up to 256), a bf16 copy (twice that) and one fp32
 *               factor per row (M*4 bytes, rounded up to 256). After a call
 *               that ran out of time (GNF4_ERR_TIMEOUT) zero the workspace
 *               again before reusing it. Two calls that may run
 *               concurrently need separate workspaces.
 * Numerics: every product enters an fp32 accumulator. DECODE carries each
 *   NF4 code value as hi = fp16(NF4[code] * 1.677654), a scale that keeps
 *   the rounding error of every value within 6.0e-5 (the elementwise
 *   tolerance above holds with margin on the shapes in scope); with a
 *   fused SwiGLU (which multiplies an up error by silu(gate)) the up rows
 *   also carry the fp16 of the remainder (scaled by 2^13), together within
 *   2^-21 relative of the scaled value; x per row and 64-element block is
 *   scaled by a power of two into fp16 (exact for every element above
 *   2^-28 of that block's largest magnitude); each block sum is scaled by
 *   absmax, the power of two and 1 / 1.677654 in fp32. DECODE's stream-K split
 *   adds the fp32 partial sums of a cut tile in a fixed order: results are
 *   deterministic for a given GPU (SM count).
 *   PREFILL scales each weight row and each row of x by a power of two,
 *   multiplies the bf16 rounding of the fp32 weight NF4[code] * absmax by the
 *   scaled x (exact in bf16), adds the e4m3 rounding of what that rounding
 *   left times the e5m2 rounding of the scaled x (at most about 2^-13 of the
 *   product, whatever the magnitude of the row), and divides both powers of
 *   two out again.
 * Alignment: x, w, y and the workspace 32-byte aligned; absmax 4-byte aligned.
 * On a device-side metadata error no output is written.
 */
GNF4_API gnf4_status gnf4_grouped_gemm(const uint16_t *x, const uint8_t *w, const float *absmax,
                              const int32_t *sizes, const int32_t *expert_ids, int32_t G,
                              int64_t M, int32_t N, int32_t K, int32_t E, int32_t blocksize,
                              int32_t epilogue, int32_t mode, uint16_t *y, void *workspace,
                              size_t ws_bytes, gnf4_stream_t stream);

/*
 * gnf4_grouped_gemm_ex -- the grouped GEMM with its options in a descriptor:
 * the weight format (NF4 or native MXFP4), the scale encoding, the epilogue
 * (none, SwiGLU on halves, SwiGLU on interleaved clamped rows) and the
 * activation gather through the sort's permutation.
 *
 * Passages: README opening section (the operation); package page
 * "grouped-nf4-gemm", "Direct answer" and header block ("Owns": the grouped
 * packed GEMM over NF4 and native MXFP4, e2m1 + e8m0, computed on the
 * released bytes with no requantisation and no bf16 copy); "Use this when"
 * (the small launches around the expert GEMM, the token gather among them,
 * folded into one); the streaming page's bake options (absmax stored as fp32
 * or bf16).
 *
 * For every row m of group g (expert e) and output column n:
 *   NF4:   acc = sum_k x[m][k] * NF4[code(e,n,k)] * absmax[e][n][k/64]
 *          (absmax fp32, or bf16 widened exactly to fp32)
 *   MXFP4: acc = sum_k x[m][k] * E2M1[code(e,n,k)] * 2^(scale[e][n][k/32]-127)
 *          code(e,n,k) = low nibble of w[e][n][k/2] for even k, high for odd
 *          k (the OCP microscaling FP4 packing of the released gpt-oss
 *          blocks); E2M1 = 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives;
 *          scale 255 is NaN.
 *   epilogue NONE / SWIGLU: as gnf4_grouped_gemm.
 *   epilogue SWIGLU_INTERLEAVED (the gpt-oss form): gate = acc of even
 *          column 2j, up = acc of odd column 2j+1; g = min(gate, limit),
 *          u = min(max(up, -limit), limit);
 *          y[m][j] = bf16_rne(g * sigmoid(alpha * g) * (u + 1)), y is [M][N/2].
 *   gather: with x == NULL the rows are taken through the sort's permutation,
 *          row m = hidden[sorted_idx[m] / top_k]: no sorted copy of the
 *          activations is written. sorted_idx comes from gnf4_moe_align (its
 *          first M entries); an entry outside [0, n_tokens*top_k) sets
 *          GNF4_DEVERR_SLOT and nothing is written.
 *
 * Descriptor fields (struct_bytes = sizeof(gnf4_gemm_desc)):
 *   x or (hidden, sorted_idx, n_tokens, top_k): exactly one of x and hidden
 *   is non-NULL; hidden is [n_tokens][K] bf16, n_tokens*top_k < 2^31.
 *   w, scales, sizes, expert_ids, G, M, N, K, E, y, mode: as for
 *   gnf4_grouped_gemm (K % 64 == 0 for both formats; N even for both SwiGLU
 *   forms; swiglu_limit > 0 for the interleaved form).
 *   scale_dtype: GNF4_SCALE_F32 or GNF4_SCALE_BF16 with NF4,
 *   GNF4_SCALE_E8M0 with MXFP4.
 * Kernels: DECODE runs every combination. PREFILL (and AUTO's prefill
 * choice) runs NF4 with fp32 or bf16 absmax, MXFP4, gathered or sorted rows
 * and every epilogue; anything else is refused with
 * GNF4_ERR_UNSUPPORTED_SHAPE. Numerics as gnf4_grouped_gemm; an MXFP4 code
 * value is exact in fp16 and bf16 and enters the MMA whole.
 * Workspace: gnf4_workspace_bytes(GNF4_OP_GROUPED_GEMM, M, N, K, E, G).
 * Alignment: x, hidden, w, y and the workspace 32-byte aligned; scales,
 * sizes, expert_ids and sorted_idx 4-byte aligned.
 */
typedef struct gnf4_gemm_desc {
    uint32_t struct_bytes;      /* sizeof(gnf4_gemm_desc) */
    int32_t format;             /* gnf4_format */
    int32_t scale_dtype;        /* gnf4_scale_dtype */
    int32_t epilogue;           /* gnf4_epilogue */
    float swiglu_alpha;         /* SWIGLU_INTERLEAVED: alpha (gpt-oss: 1.702) */
    float swiglu_limit;         /* SWIGLU_INTERLEAVED: limit (gpt-oss: 7.0) */
    int32_t mode;               /* gnf4_mode */
    int32_t top_k;              /* gather: slots per token */
    const uint16_t *x;          /* [M][K] bf16 rows in sorted order, or NULL to gather */
    const uint16_t *hidden;     /* gather: [n_tokens][K] bf16 */
    const int32_t *sorted_idx;  /* gather: [M] slot t*top_k+j of each row */
    int64_t n_tokens;           /* gather: rows of hidden */
    const uint8_t *w;           /* [E][N][K/2] packed codes */
    const void *scales;         /* NF4: absmax [E][N][K/64]; MXFP4: e8m0 [E][N][K/32] */
    const int32_t *sizes;       /* [G] */
    const int32_t *expert_ids;  /* [G] */
    int32_t G, N, K, E;
    int64_t M;
    uint16_t *y;                /* [M][N] or [M][N/2] bf16 */
} gnf4_gemm_desc;

GNF4_API gnf4_status gnf4_grouped_gemm_ex(const gnf4_gemm_desc *desc, void *workspace,
                                          size_t ws_bytes, gnf4_stream_t stream);

/*
 * gnf4_dequant_debug -- materialise NF4[code] * absmax for inspection/tests.
 *
 * Off the hot path (the GEMM never calls it). It is this library's analogue of
 * the package's pure-torch reference decode ("grouped-nf4-gemm" package page,
 * "Owns": pack and pure-torch reference operations). Each element is one IEEE
 * fp32 multiply NF4[code] * absmax; with GNF4_OUT_BF16 that product is rounded
 * once to bf16 (round to nearest even).
 *
 *   w       device uint8 [rows][K/2]   (rows = E*N for a whole stack)
 *   absmax  device fp32 [rows][K/64]
 *   rows >= 0, K >= 64, K % 64 == 0, blocksize == 64
 *   out     device fp32 or bf16 [rows][K]
 * Alignment: w and out 16-byte aligned.
 */
GNF4_API gnf4_status gnf4_dequant_debug(const uint8_t *w, const float *absmax, int64_t rows, int32_t K,
                               int32_t blocksize, int32_t out_dtype, void *out,
                               gnf4_stream_t stream);

/*
 * gnf4_grouped_dgrad -- the gradient of the grouped GEMM with respect to its
 * activations, over the same packed stack:
 *   dx[m][k] = bf16( sum_n dy[m][n] * NF4[code(e,n,k)] * absmax[e][n][k/64] )
 * with e the expert of row m's group, the weight one fp32 multiply (as in
 * the forward kernels), the sum in fp32 over n ascending, one rounding (RNE).
 *
 * Passage: package page "grouped-nf4-gemm", header block ("Owns": the grouped
 * packed GEMM and its dgrad) and "Do not use this when" (the dgrad refuses
 * tensors that are not on the device, as the GEMM does).
 *
 *   dy          device bf16 [M][N] (the gradient of the GEMM's output y)
 *   w, absmax, sizes, expert_ids, G, E, blocksize: as for gnf4_grouped_gemm
 *   M >= 0, N >= 8 with N % 8 == 0, K % 64 == 0, 1 <= G, E <= GNF4_MAX_EXPERTS,
 *   M < 2^31
 *   dx          device bf16 [M][K] (written; must not overlap dy)
 *   workspace   device, >= gnf4_workspace_bytes(GNF4_OP_GROUPED_DGRAD, ...)
 *               bytes: the 256-byte status header, one counter per (SM,
 *               value) and the fp32 partials of the tiles the stream-K split
 *               cuts (4 KB per SM); zero it once (each call leaves the
 *               counters at zero).
 * One launch of a tensor-core kernel (mma.sync, fp32 accumulation) over
 * batches of up to 8 rows and 64-element blocks of k, split over the SMs by
 * tile-stages of 256 weight rows. Numerics: the weight carried as its fp16
 * rounding (relative error at most 2^-12); dy * absmax, exact in fp32,
 * scaled by a power of two per (row, 16 weight rows) and carried as two fp16
 * parts; fp32 sums, a fixed summation order (deterministic for a given GPU).
 * Alignment: dy and w 16-byte aligned, absmax 4, dx 2, workspace 16.
 * A metadata error (as for gnf4_grouped_gemm) sets the device error word and
 * nothing is written.
 */
GNF4_API gnf4_status gnf4_grouped_dgrad(const uint16_t *dy, const uint8_t *w, const float *absmax,
                                        const int32_t *sizes, const int32_t *expert_ids,
                                        int32_t G, int64_t M, int32_t N, int32_t K, int32_t E,
                                        int32_t blocksize, uint16_t *dx, void *workspace,
                                        size_t ws_bytes, gnf4_stream_t stream);

/*
 * gnf4_router_topk -- the router's choice of experts per token, the input of
 * gnf4_moe_align.
 *
 * Passage: package page "grouped-nf4-gemm", "Use this when" (router softmax
 * and top-k among the small decode launches to fold into one each). The
 * pages fix no formula; this
 * library takes the usual softmax router: per token t, the top_k experts with
 * the largest logits (equal logits: lower expert id first; a NaN logit ranks
 * as -inf) in descending order, and their softmax weights
 *   renormalize == 0: exp(l_e - l_max) / sum over all E experts
 *   renormalize == 1: exp(l_e - l_max) / sum over the top_k selected experts
 * computed in fp32 (weights within about 1e-6 relative of the exact values;
 * weights are unspecified if a logit is infinite or NaN).
 *
 *   logits        device fp32 [T][E], 4-byte aligned
 *   T >= 0, 1 <= E <= GNF4_MAX_EXPERTS, 1 <= top_k <= min(E, GNF4_MAX_TOPK)
 *   topk_ids      device int32 [T][top_k] (written)
 *   topk_weights  device fp32 [T][top_k] (written)
 * One kernel launch, no workspace.
 */
GNF4_API gnf4_status gnf4_router_topk(const float *logits, int64_t T, int32_t E, int32_t top_k,
                                      int32_t renormalize, int32_t *topk_ids, float *topk_weights,
                                      gnf4_stream_t stream);

/*
 * gnf4_moe_combine -- the top-k weighted combine after the down projection:
 *   out[t][h] = bf16( sum_{j < top_k} topk_weights[t][j] * y[p(t*top_k + j)][h] )
 * where p(s) is the row of y that holds slot s (the position of s in
 * sorted_idx), summed in fp32 with j ascending and rounded once (RNE).
 *
 * Passage: package page "grouped-nf4-gemm", header block ("Owns": the decode
 * glue kernels, combine among them) and "Use this when" (the top-k combine
 * among the small decode launches to fold into one each).
 *
 *   y             device bf16 [T*top_k][H]: row i is the down-projection output
 *                 of slot sorted_idx[i] (the grouped GEMM's row order)
 *   sorted_idx    device int32 [T*top_k] from gnf4_moe_align; entries of -1
 *                 (slots left out) contribute nothing; an entry outside
 *                 [-1, T*top_k) sets GNF4_DEVERR_SLOT and is skipped;
 *                 a slot listed twice is the caller's error (one row wins)
 *   topk_weights  device fp32 [T][top_k]
 *   T >= 0, 1 <= top_k <= GNF4_MAX_TOPK, H >= 1, T*top_k < 2^31
 *   out           device bf16 [T][H] (written); must not overlap y
 *   workspace     device, >= gnf4_workspace_bytes(GNF4_OP_MOE_COMBINE, T*top_k, ...)
 *                 bytes (header, then the inverse of sorted_idx); its first 256
 *                 bytes are the device status word, zero-filled once.
 * Alignment: y, out 2-byte aligned (16-byte aligned rows, H % 8 == 0, take the
 * vectorised path); sorted_idx, topk_weights 4-byte aligned; workspace 16-byte.
 * Two kernel launches.
 */
GNF4_API gnf4_status gnf4_moe_combine(const uint16_t *y, const int32_t *sorted_idx,
                                      const float *topk_weights, int64_t T, int32_t top_k,
                                      int32_t H, uint16_t *out, void *workspace, size_t ws_bytes,
                                      gnf4_stream_t stream);

/*
 * gnf4_workspace_bytes -- workspace size for an op and problem size (no GPU
 * work; queries the current device's SM count once). For GNF4_OP_MOE_ALIGN
 * only E matters; for GNF4_OP_GROUPED_GEMM the size covers every mode; for
 * GNF4_OP_MOE_COMBINE, M is T*top_k and nothing else matters; for
 * GNF4_OP_GROUPED_DGRAD it is the status header alone.
 */
GNF4_API size_t gnf4_workspace_bytes(int32_t op, int64_t M, int32_t N, int32_t K, int32_t E, int32_t G);

/*
 * gnf4_read_device_status -- synchronise `stream`, read the device error word
 * from `workspace` into *error_bits (GNF4_DEVERR_* bits; may be NULL) and,
 * if clear != 0, reset it to zero. Returns GNF4_ERR_DEVICE_METADATA if any
 * metadata bit is set, GNF4_ERR_TIMEOUT if only the timeout bit is set,
 * GNF4_ERR_CUDA on a CUDA failure, else GNF4_OK. Not for the hot path.
 */
GNF4_API gnf4_status gnf4_read_device_status(void *workspace, int32_t clear, uint32_t *error_bits,
                                    gnf4_stream_t stream);

/*
 * gnf4_grouped_gemm_noalloc -- gnf4_grouped_gemm (decode kernel) with no
 * caller-provided workspace.
 *
 * No counterpart in the grouped-nf4-gemm pages: this entry point exists for
 * callers that must not allocate device memory themselves, for example a
 * plugin inside a host application that hands out all device memory from its
 * own pre-planned pool and forbids further cudaMalloc calls, or a
 * latency-critical path that cannot afford the implicit synchronisation an
 * allocation may cause.
 *
 * It computes exactly what gnf4_grouped_gemm computes with mode =
 * GNF4_MODE_DECODE (same arguments, minus workspace and mode), using a
 * scratch area that lives inside the library: a fixed device array of
 * GNF4_NOALLOC_SCRATCH_BYTES bytes, reserved on every GPU that loads the
 * library for as long as the process runs. Nothing is allocated or freed.
 *  - The first call on a device looks up that array's device address (one
 *    runtime query, once per device, with that device current).
 *  - Problems whose decode-kernel workspace exceeds
 *    GNF4_NOALLOC_SCRATCH_BYTES are refused with GNF4_ERR_SCRATCH_LIMIT
 *    before anything is launched (the decode kernel's workspace is the
 *    status header plus its stream-K counters and partial sums, about
 *    1.2 MB on a 148-SM GPU whatever the problem size, so the limit is not
 *    reached there; callers should still handle the code).
 *  - All calls share the one array and it keeps the previous call's
 *    contents; each call first clears the part that must start at zero (an
 *    asynchronous memset on `stream`). Calls whose GPU work can overlap (on
 *    different streams, or from different threads) race on the array and
 *    give wrong results: serialise them.
 *  - Device-side metadata errors leave y unwritten, as in gnf4_grouped_gemm,
 *    but the error word stays inside the library's array; use
 *    gnf4_grouped_gemm with a workspace when the error word is needed.
 */
#define GNF4_NOALLOC_SCRATCH_BYTES (8u << 20) /* 8 MiB per device */

GNF4_API gnf4_status gnf4_grouped_gemm_noalloc(const uint16_t *x, const uint8_t *w,
                                               const float *absmax, const int32_t *sizes,
                                               const int32_t *expert_ids, int32_t G, int64_t M,
                                               int32_t N, int32_t K, int32_t E, int32_t blocksize,
                                               int32_t epilogue, uint16_t *y,
                                               gnf4_stream_t stream);

/* Human-readable name of a status code (static storage). */
GNF4_API const char *gnf4_status_string(gnf4_status status);

/* GNF4_VERSION of the loaded library. */
GNF4_API int32_t gnf4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GNF4_H */
