// decode_gemm.cu -- decode-regime grouped 4-bit GEMM (few activation rows per expert).
//
// Passage: "grouped-nf4-gemm -- single-launch W4A16 GEMM over fused NF4 MoE
// expert stacks", opening section (one launch for all active experts, LUT
// decode of the packed codes, blockwise fp32 absmax, fp32 accumulation, bf16
// epilogue, no bf16 weight copy) and "Status / roadmap" (split-K for starved
// grids); package page "grouped-nf4-gemm", "Direct answer" (the same grouped
// GEMM over native MXFP4, e2m1 codes with e8m0 scales) and "Use this when"
// (the token gather folded into the GEMM's launch). At a handful of activation
// rows per expert this GEMM reads every touched weight byte once and is bound
// by HBM bandwidth, so the kernel is built around keeping HBM busy: a TMA
// producer keeps up to six 16 KB stages of packed weights in flight per SM.
//
// Work decomposition
//   batch  = up to 8 consecutive activation rows of one group (the MMA's N).
//   unit   = 16 weight rows of the group's expert for one batch: two row
//            groups of 8 (with SwiGLU: 8 gate rows and the matching 8 up rows).
//   tile   = up to 8 consecutive units of one batch; a tile-stage is 256
//            K-elements of a tile. The tiles of all groups are laid end to end
//            (group by group, batch by batch) on the device from (sizes,
//            expert_ids): the host never learns which experts are active.
//   Stream-K split: the W = tiles x stages tile-stages are cut into one equal
//   contiguous range per CTA (one CTA per SM), so every SM streams the same
//   number of weight bytes whatever the tile count. A tile that lies inside
//   one CTA's range is finished by it; a tile cut by range boundaries is
//   computed in pieces: each piece leaves its fp32 partial sums in the
//   workspace and counts itself in that tile's counter, and the piece that
//   counts last adds the partials in piece order (deterministic), writes y and
//   resets the counter. When tiles outnumber SMs only the few tiles at range
//   boundaries are cut; when SMs outnumber tiles (starved grids) every tile is
//   split across several SMs.
//
// Formats and numerics (per stage, each consumer lane decodes packed bytes
// through a byte-indexed table replicated per lane, so no lookup conflicts)
//   NF4:   code value NF4[c] carried as hi = fp16(NF4[c] * kTableScale), one
//          MMA per 16 K-elements; the block sum is multiplied by
//          1 / kTableScale (see kTableScale). With a fused SwiGLU the up rows
//          also carry the remainder (NF4[c] * kTableScale - hi) * 2^13 as fp16
//          in a second MMA (gate rows 0 there): SwiGLU multiplies an up error
//          by silu(gate), which a near-zero up value leaves unbounded by the
//          relative tolerance, while a one-part gate stays well inside it.
//          The scale is the fp32 (or bf16) absmax of the 64-element block,
//          applied to the block's fp32 sum.
//   MXFP4: e2m1 code values are exact in fp16 (one MMA); the e8m0 scale of
//          each 32-element half-block is applied to its fp32 sum.
//   Activations are staged as bf16 and rewritten in place as fp16 times a
//   power of two per (row, 64-element block), which the block sum divides out.
//
// Inside a CTA (warp 16 = tensor copies; warps 17-19 = scale copies and, when
// the activations are gathered, their row copies, or activation conversion;
// warps 0-15 = consumers)
//   Consumer warp w takes 64-element block w / 4 of every stage for the two
//   units 2 (w % 4), 2 (w % 4) + 1; when a tile piece ends, the four block
//   warps of a unit pair sum their partial results through shared memory
//   (fixed order) and the block-0 warp writes y or the piece's partial.
// Every wait is bounded (2 s unless the workspace header asks for less); on
// expiry the kernel records GNF4_DEVERR_TIMEOUT, lets the producer's copies
// land and returns.
#include <climits>

#include <cuda_fp16.h>

#include "launch.h"
#include "lut_mma.cuh"

namespace gnf4 {
namespace {

constexpr int kConsumerWarps = 16;
constexpr int kTmaWarp = kConsumerWarps;          // issues the tensor copies
// The three other warps copy scales (and gathered activations) or convert
// the staged activations to fp16. With one 16-byte scale copy per row one
// copy warp keeps up and two convert; with 4-byte copies two copy and one
// converts. 20 warps keep 96 registers per thread (each SM sub-partition
// holds 5 of them); a copy warp that also issued the tensor copies delayed
// them behind its own copies.
constexpr int kThreads = (kConsumerWarps + 4) * 32;
template <bool WIDE>
struct WarpRoles {
  static constexpr int kScaleWarps = WIDE ? 1 : 2;
  static constexpr int kXWarps = 3 - kScaleWarps;
  static constexpr int kScaleWarp0 = kTmaWarp + 1;
  static constexpr int kXWarp0 = kScaleWarp0 + kScaleWarps;
};
constexpr int kTileUnits = 8;                 // units per tile (2 row groups each)
constexpr int kStages = 6;
constexpr int kBatch = 8;                     // activation rows per batch (MMA N)
constexpr int kBoxBytes = 1024;               // 8 rows x 128 bytes
constexpr int kStageBlocks = 4;               // 64-element blocks per stage (256 K-elements)
constexpr int kWStage = kTileUnits * 2 * kBoxBytes;              // 16 KB
constexpr int kXStage = kStageBlocks * kBoxBytes;                // 4 KB
constexpr int kXsStage = kStageBlocks * kBatch * 4;              // 128 B: 2^-S per (block, row)
constexpr int kAStage = kTileUnits * 2 * 8 * kStageBlocks * 4;   // 2 KB of scale words
constexpr int kMaxG = GNF4_MAX_EXPERTS;
constexpr int kPairs = kTileUnits / 2;        // unit pairs per tile
constexpr int kPartialSlot = 2 * 32;          // float4 per (pair) partial: 2 units x 32 lanes

// Shared memory layout, as absolute shared-window addresses. The window
// starts with memory the driver reserves and the static tables below; the
// dynamic part must start in [kMinDyn, kDynBase], which the kernel checks.
// The table sits at a multiple of 65536 so that one byte permute forms a
// lookup's whole address.
constexpr int kMinDyn = 1024;
constexpr int kDynBase = 2048;
constexpr int kWOff = kDynBase;                               // 1024-aligned (128-byte swizzle)
constexpr int kXOff = kWOff + kStages * kWStage;              // bf16, converted in place to fp16
constexpr int kXsOff = kXOff + kStages * kXStage;             // float [kStages][4 blocks][8 rows]
constexpr int kRowOffOff = kXsOff + kStages * kXsStage;       // int32 [kMaxG + 1]
constexpr int kBarOff = (kRowOffOff + (kMaxG + 1) * 4 + 7) / 8 * 8;   // mbarriers, see kNumBars
// full[kStages] (copies landed), empty[kStages] (consumers done), xready
// [kStages] (activations converted), then per unit pair: xfull (the three
// partial sums written), xempty (the block-0 warp done reading them), and
// `never`, which nothing arrives at (the wait-limit test hook)
constexpr int kNumBars = 3 * kStages + kTileUnits + 1;
constexpr int kMiscOff = kBarOff + kNumBars * 8;              // int [8]
// table: 256-byte row per packed byte b: lane l's hi pair at l * 4, its
// remainder pair at 128 + l * 4
constexpr int kLutOff = 131072;
constexpr int kLutBytes = 256 * 256;
constexpr int kAOff = kLutOff + kLutBytes;
constexpr int kXchgOff = kAOff + kStages * kAStage;           // float4 [4 pairs][3][2 units][32]
constexpr int kXchgBytes = kPairs * 3 * 2 * 32 * 16;
constexpr int kGExpOff = kXchgOff + kXchgBytes;               // uint16 [kMaxG]
constexpr int kBatchOff = kGExpOff + kMaxG * 2;               // int32 [kMaxG + 1]: first batch per group
constexpr int kSmemEnd = kBatchOff + (kMaxG + 1) * 4;
// dynamic bytes requested: the window reaches kSmemEnd from any start >= kMinDyn
constexpr int kSmemBytes = kSmemEnd - kMinDyn;
static_assert(kMiscOff + 8 * 4 <= kLutOff, "low region overlaps the table");
static_assert(kBarOff % 8 == 0 && kXOff % 1024 == 0 && kLutOff % 65536 == 0, "alignment");
static_assert(kSmemBytes + kDynBase - kMinDyn <= 227 * 1024, "fits one CTA per SM");

// NF4 code values enter the MMAs as fp16(NF4[c] * kTableScale). Of the
// scales in [1, 2) (searched on a 5e-7 grid) this one gives the smallest
// largest rounding error over the 16 values: 6.0e-5 of the code range,
// against 1.9e-4 for the plain fp16 rounding. The consumers' per-block
// factor 2^-S carries the 1 / kTableScale back.
constexpr float kTableScale = 1.6776540f;
constexpr float kTableInv = 1.0f / kTableScale;
constexpr float kLoInv = 1.0f / 8192.0f;      // up-row remainders are carried times 2^13

// Scale encodings of the stack (GemmArgs::scale_kind).
constexpr int kScaleF32 = 0;    // NF4 absmax, fp32
constexpr int kScaleBf16 = 1;   // NF4 absmax, bf16
constexpr int kScaleE8m0 = 2;   // MXFP4: two e8m0 bytes per 64-element block

// e2m1 code value (OCP microscaling FP4: sign, 2 exponent bits, 1 mantissa
// bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), exact in fp16.
__device__ __forceinline__ float e2m1_value(int c) {
  const int m = c & 7;
  const float mag = m < 2 ? 0.5f * m : static_cast<float>(2 + (m & 1)) * exp2f(static_cast<float>((m >> 1) - 2));
  return (c & 8) ? -mag : mag;
}

// 2^(s - 127) for an e8m0 byte (0xFF encodes NaN).
__device__ __forceinline__ float e8m0_value(uint32_t s) {
  if (s == 255u) return __uint_as_float(0x7FC00000u);
  return s == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(s << 23);
}

struct Problem {
  int32_t N, K, E, G;
  int32_t epi;      // 0 none, 1 SwiGLU on the two halves, 2 SwiGLU on interleaved rows, clamped
  int32_t KB;       // 64-element blocks per row
  int32_t KC;       // stages per tile
  int32_t upb;      // units per batch
  int32_t tpb;      // tiles per batch
};

struct Tile {
  int64_t row0;     // first activation row of the batch
  int32_t j0;       // unit index within the batch of the tile's first unit
  int32_t nunits;   // 1..kTileUnits
  int32_t mrows;    // activation rows in the batch (1..8)
  int32_t e;        // expert
};

// Tile t: batch t / tpb, the (t % tpb)-th run of up to 8 units of it.
__device__ __forceinline__ Tile make_tile(int64_t t, const Problem &p, const int *batch_start,
                                          const int *row_off, const uint16_t *gexp) {
  const int64_t bt = div_fast(t, p.tpb);
  const int32_t jt = static_cast<int32_t>(t - bt * p.tpb);
  int lo = 0, hi = p.G;   // invariant: batch_start[lo] <= bt < batch_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (batch_start[mid] <= bt) lo = mid; else hi = mid;
  }
  const int32_t lb = static_cast<int32_t>(bt) - batch_start[lo];
  Tile tl;
  tl.row0 = static_cast<int64_t>(row_off[lo]) + static_cast<int64_t>(lb) * kBatch;
  tl.j0 = jt * kTileUnits;
  tl.nunits = min(kTileUnits, p.upb - tl.j0);
  tl.mrows = min(kBatch, row_off[lo + 1] - row_off[lo] - lb * kBatch);
  tl.e = gexp[lo];
  return tl;
}

// Where piece (tile t, CTA c) keeps its partial sums: slot 0 if t is the
// first tile c touches, slot 1 if it is the last one (a cut tile is always
// one of the two for every CTA that holds a piece of it).
__device__ __forceinline__ int64_t piece_slot(int64_t W, int64_t P, int64_t KC, int64_t t,
                                              int64_t c) {
  return c * 2 + (div_fast(range_lo(W, P, c), KC) == t ? 0 : 1);
}

// Packed-weight tensor maps: boxes of 8, 16, 32, 64 and 128 rows x 128 bytes
// over [E*N rows][K/2 bytes] (2-D), and for interleaved gate/up rows, boxes
// of 8, 16, 32 and 64 rows of one parity over [E*N/2 pairs][2][K/2] (3-D).
constexpr int kNumWMaps = 5;
constexpr int kNumIMaps = 4;
struct WeightMaps {
  CUtensorMap m[kNumWMaps];   // m[i]: boxes of (8 << i) rows
  CUtensorMap im[kNumIMaps];  // im[i]: boxes of (8 << i) rows of one parity (epilogue 2 only)
};

// Copies `nrows` (a multiple of 8) consecutive weight rows, 128 bytes of
// each starting at byte column c0, to dst as row-major 128-byte rows.
__device__ __forceinline__ void load_weight_rows(char *dst, const WeightMaps &wm, int c0,
                                                 int64_t row, int nrows, uint64_t *bar) {
  int done = 0;
#pragma unroll
  for (int i = kNumWMaps - 1; i >= 0; --i) {
    const int h = 8 << i;
    while (nrows - done >= h) {
      tma_load_2d(dst + done * 128, &wm.m[i], c0, static_cast<int>(row + done), bar);
      done += h;
    }
  }
}

// Copies rows 2 (pair0 + i) + parity, i < npairs (a multiple of 8), as
// consecutive 128-byte rows.
__device__ __forceinline__ void load_parity_rows(char *dst, const WeightMaps &wm, int c0,
                                                 int64_t pair0, int parity, int npairs,
                                                 uint64_t *bar) {
  int done = 0;
#pragma unroll
  for (int i = kNumIMaps - 1; i >= 0; --i) {
    const int h = 8 << i;
    while (npairs - done >= h) {
      tma_load_3d(dst + done * 128, &wm.im[i], c0, parity, static_cast<int>(pair0 + done), bar);
      done += h;
    }
  }
}

struct DecodeParams {
  const void *scales;          // fp32 / bf16 absmax [E][N][K/64], or e8m0 [E][N][K/32]
  const int32_t *sizes;
  const int32_t *expert_ids;
  const uint16_t *hidden;      // gathered activations [T][K] (nullptr: x through the tensor map)
  const int32_t *sorted_idx;   // [M] slot of each row (gather)
  int64_t n_slots;             // T * top_k (gather)
  int32_t top_k;               // (gather)
  int32_t G;
  int64_t M;
  int32_t N, K, E;
  int32_t scale_kind;
  int32_t epi;
  float alpha, limit;          // epilogue 2
  uint16_t *y;
  WsHeader *hdr;
  uint32_t *counters;          // [P][kPairs]
  float4 *partials;            // [P][2][kPairs][kPartialSlot]
};

// The output of one unit pair (acc[uu][*], C-fragment order) for tile tl.
__device__ __forceinline__ void store_outputs(uint16_t *y, float alpha, float limit,
                                              const Problem &p, const Tile &tl, int up, int g,
                                              int q, const float (&acc)[2][4], bool act1) {
  const int64_t ncols = p.epi ? p.N / 2 : p.N;
#pragma unroll
  for (int uu = 0; uu < 2; ++uu) {
    if (uu == 1 && !act1) break;
    const int64_t j = tl.j0 + 2 * up + uu;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int m = 2 * q + i;
      if (m >= tl.mrows) continue;
      uint16_t *yr = y + (tl.row0 + m) * ncols;
      const float a0 = acc[uu][i], a1 = acc[uu][2 + i];
      if (p.epi == 0) {
        const int64_t c0 = 16 * j + g, c1 = 16 * j + 8 + g;
        if (c0 < p.N) yr[c0] = bf16_bits(a0);
        if (c1 < p.N) yr[c1] = bf16_bits(a1);
      } else {
        const int64_t c = 8 * j + g;
        if (c >= ncols) continue;
        float o;
        if (p.epi == 1) {
          o = silu(a0) * a1;
        } else {   // clamped gate and up, gate * sigmoid(alpha * gate) * (up + 1)
          const float gt = fminf(a0, limit);
          const float u = fminf(fmaxf(a1, -limit), limit);
          o = gt / (1.0f + expf(-alpha * gt)) * (u + 1.0f);
        }
        yr[c] = bf16_bits(o);
      }
    }
  }
}

// The next stage slot of the ring; its phase parity flips when the slot wraps.
__device__ __forceinline__ void next_stage(int &st, uint32_t &ph) {
  if (++st == kStages) {
    st = 0;
    ph ^= 1u;
  }
}

__device__ __forceinline__ Problem make_problem(const DecodeParams &a) {
  Problem p;
  p.N = a.N; p.K = a.K; p.E = a.E; p.G = a.G; p.epi = a.epi;
  p.KB = a.K / 64;
  p.KC = (p.KB + kStageBlocks - 1) / kStageBlocks;
  p.upb = a.epi ? (a.N / 2 + 7) / 8 : (a.N + 15) / 16;
  p.tpb = (p.upb + kTileUnits - 1) / kTileUnits;
  return p;
}

// Generic pointer of shared-window address `off`.
__device__ __forceinline__ char *shared_ptr(uint32_t off) {
  return static_cast<char *>(__cvta_shared_to_generic(off));
}

// The suspending part of a bounded wait on the mbarrier at shared address
// `bar`: the time limit (shortened by a non-zero header word 2, the test
// hook) and the CTA's abort flag are read here, out of the stage loop.
__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, WsHeader *hdr) {
  const uint32_t hook = hdr->reserved[0];
  const uint64_t limit_ns = hook ? static_cast<uint64_t>(hook) : kTimeoutNs;
  const uint32_t hint = limit_ns < kWaitHintNs ? static_cast<uint32_t>(limit_ns) : kWaitHintNs;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(shared_ptr(kMiscOff)) + 1;
  const uint64_t t0 = global_timer();
  while (true) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint)
        : "memory");
    if (ok) return true;
    if (*abort_flag) return false;
    if (global_timer() - t0 > limit_ns) {
      *abort_flag = 1;
      report_error(hdr, GNF4_DEVERR_TIMEOUT, blockIdx.x);
      return false;
    }
  }
}

// Bounded wait of the whole warp (warp-uniform answer) on the mbarrier at
// shared address `bar`: one non-suspending try, else the loop above.
__device__ __forceinline__ bool warp_wait_sa(uint32_t bar, uint32_t parity, WsHeader *hdr) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  if (!ok) ok = wait_slow(bar, parity, hdr) ? 1u : 0u;
  return __all_sync(0xffffffffu, ok != 0);
}

// One arrival on the mbarrier at shared address `bar` for the whole
// (converged) warp, by an elected lane.
__device__ __forceinline__ void arrive_elect_sa(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
      "@p mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(bar)
      : "memory");
}

// The end of one tile piece for the calling consumer warp (unit pair up =
// warp % 4, block blk = warp / 4) with its sums acc0 (unit 2 up) and acc1
// (unit 2 up + 1) after the ep-th piece of tile t (tl; whole: the piece is
// the whole tile): block warps 1..3 hand their sums to the pair's block-0
// warp, which stores the outputs, or, for a piece of a cut tile, leaves its
// partial sums and counts the piece; the piece that counts last adds all
// pieces in order and stores. Out of line, with the values it needs
// recomputed here from shared memory and the parameters, so that they do
// not stay live across the stage loop. False if a wait gave up.
__device__ __noinline__ bool finish_piece(const DecodeParams &a, float4 acc0, float4 acc1,
                                          int64_t t, Tile tl, bool whole, uint32_t ep) {
  char *smem = shared_ptr(0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int up = warp & 3, blk = warp >> 2, g = lane >> 2, q = lane & 3;
  const Problem p = make_problem(a);
  const uint32_t xfull = kBarOff + (3 * kStages + up) * 8;
  const uint32_t xempty = kBarOff + (3 * kStages + kPairs + up) * 8;
  float4 *xchg = reinterpret_cast<float4 *>(smem + kXchgOff) + up * 3 * 2 * 32 + lane;
  float acc[2][4] = {{acc0.x, acc0.y, acc0.z, acc0.w}, {acc1.x, acc1.y, acc1.z, acc1.w}};
  const bool act1 = 2 * up + 1 < tl.nunits;
  if (blk != 0) {
    // hand the partial sums to the pair's block-0 warp
    if (ep > 0 && !warp_wait_sa(xempty, (ep - 1) & 1u, a.hdr)) return false;
#pragma unroll
    for (int uu = 0; uu < 2; ++uu)
      xchg[((blk - 1) * 2 + uu) * 32] = make_float4(acc[uu][0], acc[uu][1], acc[uu][2], acc[uu][3]);
    __syncwarp();
    if (lane == 0) mbar_arrive(reinterpret_cast<uint64_t *>(smem + xfull));
    return true;
  }
  if (!warp_wait_sa(xfull, ep & 1u, a.hdr)) return false;
#pragma unroll
  for (int b = 1; b < 4; ++b) {
#pragma unroll
    for (int uu = 0; uu < 2; ++uu) {
      const float4 v = xchg[((b - 1) * 2 + uu) * 32];
      acc[uu][0] += v.x;
      acc[uu][1] += v.y;
      acc[uu][2] += v.z;
      acc[uu][3] += v.w;
    }
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(reinterpret_cast<uint64_t *>(smem + xempty));
  if (whole) {
    store_outputs(a.y, a.alpha, a.limit, p, tl, up, g, q, acc, act1);
    return true;
  }
  const int64_t KC = p.KC;
  const int64_t W = static_cast<int64_t>(reinterpret_cast<const int *>(smem + kMiscOff)[2]) * p.tpb * KC;
  const int64_t P = min(static_cast<int64_t>(gridDim.x), W);
  const int64_t b_first = cta_of(W, P, t * KC), b_last = cta_of(W, P, t * KC + KC - 1);
  // a piece of a cut tile: leave the partial sums, count the piece; the
  // piece that counts last adds all pieces in order and stores
  float4 *mine = a.partials + (piece_slot(W, P, KC, t, blockIdx.x) * kPairs + up) * kPartialSlot;
#pragma unroll
  for (int uu = 0; uu < 2; ++uu)
    mine[uu * 32 + lane] = make_float4(acc[uu][0], acc[uu][1], acc[uu][2], acc[uu][3]);
  __syncwarp();
  uint32_t old = 0;
  uint32_t *cnt = a.counters + b_first * kPairs + up;
  if (lane == 0) {
    __threadfence();
    old = atomic_add_acq_rel(cnt, 1u);
  }
  old = __shfl_sync(0xffffffffu, old, 0);
  if (old == static_cast<uint32_t>(b_last - b_first)) {
    __syncwarp();
#pragma unroll
    for (int uu = 0; uu < 2; ++uu)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[uu][i] = 0.0f;
    for (int64_t c = b_first; c <= b_last; ++c) {
      const float4 *pc = a.partials + (piece_slot(W, P, KC, t, c) * kPairs + up) * kPartialSlot;
#pragma unroll
      for (int uu = 0; uu < 2; ++uu) {
        const float4 v = __ldcg(pc + uu * 32 + lane);
        acc[uu][0] += v.x;
        acc[uu][1] += v.y;
        acc[uu][2] += v.z;
        acc[uu][3] += v.w;
      }
    }
    store_outputs(a.y, a.alpha, a.limit, p, tl, up, g, q, acc, act1);
    if (lane == 0) *cnt = 0u;   // reusable by the next launch
  }
  return true;
}

// SK: the scale encoding (kScaleF32, kScaleBf16, or kScaleE8m0 for MXFP4).
// UPLO: the up rows of a SwiGLU unit also carry the code remainders (NF4).
// WIDE: fp32 scales whose 4 blocks of a stage are one 16-byte aligned run in
// every row (K % 256 == 0, scales 16-byte aligned), copied 16 bytes at a time.
template <int SK, bool WIDE, bool UPLO>
__global__ void __launch_bounds__(kThreads, 1)
    decode_gemm_kernel(const __grid_constant__ WeightMaps wmaps,
                       const __grid_constant__ CUtensorMap xmap,
                       const __grid_constant__ DecodeParams a) {
  constexpr bool MX = SK == kScaleE8m0;
  static_assert(!WIDE || SK == kScaleF32, "16-byte scale copies are for fp32 scales");
  constexpr int kScaleWarps = WarpRoles<WIDE>::kScaleWarps;
  constexpr int kXWarps = WarpRoles<WIDE>::kXWarps;
  constexpr int kScaleWarp0 = WarpRoles<WIDE>::kScaleWarp0;
  constexpr int kXWarp0 = WarpRoles<WIDE>::kXWarp0;
  extern __shared__ __align__(1024) char smem_raw[];
  // The parameters the loops use, as locals: the parameter block's address
  // is never taken, so every use is a constant-bank operand, not a load that
  // the asm statements' memory clobbers would force to repeat.
  WsHeader *hdr = a.hdr;
  const void *const scales = a.scales;
  constexpr int scale_kind = SK;
  const uint16_t *const hidden = a.hidden;
  const int32_t *const sorted_idx = a.sorted_idx;
  const int32_t top_k = a.top_k;
  // generic pointer of shared-window address 0: smem + kXxxOff is region kXxx
  const uint32_t dyn0 = smem_u32(smem_raw);
  char *smem = smem_raw - dyn0;
  // the dynamic window [dyn0, dyn0 + its size) must hold [kDynBase, kSmemEnd)
  const uint32_t dyn_size = dynamic_smem_size();
  if (dyn0 > static_cast<uint32_t>(kDynBase) || dyn0 + dyn_size < static_cast<uint32_t>(kSmemEnd)) {
    // the layout cannot be placed (not expected on this architecture)
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      hdr->reserved[60] = dyn0;
      hdr->reserved[61] = dyn_size;
      report_error(hdr, GNF4_DEVERR_CAPACITY, dyn0);
    }
    return;
  }
  int *row_off = reinterpret_cast<int *>(smem + kRowOffOff);
  int *batch_start = reinterpret_cast<int *>(smem + kBatchOff);
  uint16_t *gexp = reinterpret_cast<uint16_t *>(smem + kGExpOff);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kBarOff);
  uint64_t *empty = full + kStages;
  uint64_t *xready = empty + kStages;
  uint64_t *xfull = xready + kStages;          // [kPairs]
  uint64_t *xempty = xfull + kPairs;           // [kPairs]
  uint64_t *never = xempty + kPairs;
  int *misc = reinterpret_cast<int *>(smem + kMiscOff);   // [0] error bits, [1] abort, [2] batches
  volatile int *abort_flag = &misc[1];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();

  const Problem p = make_problem(a);
  const bool gather = hidden != nullptr;

  if (tid == 0) {
    misc[0] = 0;
    misc[1] = 0;
    for (int s = 0; s < kStages; ++s) {
      // one cp.async arrival per scale-warp lane + the byte-count arrival
      mbar_init(&full[s], 32 * kScaleWarps + 1);
      mbar_init(&empty[s], kConsumerWarps);
      mbar_init(&xready[s], kXWarps);
    }
    for (int i = 0; i < kPairs; ++i) {
      mbar_init(&xfull[i], 3);
      mbar_init(&xempty[i], 1);
    }
    mbar_init(never, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int i = 0; i < kNumWMaps; ++i) prefetch_tensormap(&wmaps.m[i]);
    if (a.epi == 2)
      for (int i = 0; i < kNumIMaps; ++i) prefetch_tensormap(&wmaps.im[i]);
    if (!gather) prefetch_tensormap(&xmap);
  }

  // ---- decode table: row b, lane slot l: the fp16 pair of byte b's two code
  //      values (low half = even k) at l * 4 and (UPLO) the pair of their
  //      remainders at 128 + l * 4. NF4 puts even k in the high nibble, MXFP4
  //      in the low nibble.
  for (int i = tid; i < 256 * 8; i += kThreads) {
    const int b = i >> 3, part = i & 7;
    const uint32_t hp =
        MX ? half_bits(e2m1_value(b & 15)) | (half_bits(e2m1_value(b >> 4)) << 16)
           : half_bits(nf4_value(b >> 4) * kTableScale) |
                 (half_bits(nf4_value(b & 15) * kTableScale) << 16);
    uint4 *row = reinterpret_cast<uint4 *>(smem + kLutOff + b * 256);
    row[part] = make_uint4(hp, hp, hp, hp);
    if (UPLO) {
      // remainder of the scaled value: exact in fp32, at most 2^-11 of it
      const float v0 = nf4_value(b >> 4) * kTableScale, v1 = nf4_value(b & 15) * kTableScale;
      const uint32_t lp = half_bits((v0 - __half2float(__ushort_as_half(hp & 0xFFFFu))) * 8192.0f) |
                          (half_bits((v1 - __half2float(__ushort_as_half(hp >> 16))) * 8192.0f) << 16);
      row[8 + part] = make_uint4(lp, lp, lp, lp);
    }
  }

  pdl_wait();   // inputs may come from the previous kernel on the stream
  // Test hook: a non-zero word 2 of the header shortens every bounded wait to
  // that many nanoseconds, and the consumers then start with a wait on a
  // barrier that nothing arrives at, so the timeout path runs for certain.
  const uint32_t hook_ns = hdr->reserved[0];
  const uint64_t limit_ns = hook_ns ? static_cast<uint64_t>(hook_ns) : kTimeoutNs;

  // ---- group table from (sizes, expert_ids), validated on the device: built
  //      by warp 0 alone (its lanes' loads in flight together, one warp scan),
  //      then one block barrier publishes it with the barrier set-up. With a
  //      gather, every row's slot is checked too, before any work.
  if (warp == 0) {
    const int per = (p.G + 31) / 32;
    const int g0 = min(p.G, lane * per), g1 = min(p.G, g0 + per);
    int64_t my_rows = 0, my_batches = 0;
    int bad = 0;
    for (int g = g0; g < g1; ++g) {
      const int sz = a.sizes[g];
      const int e = a.expert_ids[g];
      if (sz < 0) bad |= GNF4_DEVERR_SIZES;
      if (sz > 0 && (e < 0 || e >= p.E)) bad |= GNF4_DEVERR_EXPERT;
      gexp[g] = static_cast<uint16_t>(e);
      row_off[g] = sz;   // kept here until the offsets are known
      my_rows += max(sz, 0);
      my_batches += sz > 0 ? (sz + kBatch - 1) / kBatch : 0;
    }
    int64_t vr = my_rows, vb = my_batches;   // inclusive scan over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t x0 = __shfl_up_sync(0xffffffffu, vr, o);
      const int64_t x1 = __shfl_up_sync(0xffffffffu, vb, o);
      if (lane >= o) { vr += x0; vb += x1; }
    }
    const int64_t tot_r = __shfl_sync(0xffffffffu, vr, 31);
    const int64_t tot_b = __shfl_sync(0xffffffffu, vb, 31);
    int64_t r = vr - my_rows, c = vb - my_batches;
    for (int g = g0; g < g1; ++g) {
      const int sz = max(row_off[g], 0);
      row_off[g] = static_cast<int>(r);
      batch_start[g] = static_cast<int>(c);
      r += sz;
      c += sz > 0 ? (sz + kBatch - 1) / kBatch : 0;
    }
    if (tot_r == a.M && gather) {
      for (int64_t i = lane; i < a.M; i += 32) {
        const int32_t sl = sorted_idx[i];
        if (sl < 0 || sl >= a.n_slots) bad |= GNF4_DEVERR_SLOT;
      }
    }
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (lane == 0) {
      batch_start[p.G] = static_cast<int>(tot_b);
      row_off[p.G] = static_cast<int>(tot_r);
      if (tot_r != a.M) bad |= GNF4_DEVERR_SIZES;
      misc[2] = static_cast<int>(tot_b);
      misc[0] = bad;
    }
  }
  __syncthreads();   // group table, barrier set-up and misc visible
  const int errbits = misc[0];
  if (errbits) {
    if (blockIdx.x == 0 && tid == 0) report_error(hdr, static_cast<uint32_t>(errbits), 0);
    return;
  }
  const int64_t T = static_cast<int64_t>(misc[2]) * p.tpb;   // tiles
  const int64_t KC = p.KC;
  const int64_t W = T * KC;                                 // tile-stages
  // CTAs beyond the tile-stage count take nothing, so every range is non-empty
  // and the pieces of a cut tile are exactly the CTAs cta_of() names
  const int64_t P = min(static_cast<int64_t>(gridDim.x), W);
  if (static_cast<int64_t>(blockIdx.x) >= P) return;
  const int64_t s_lo = range_lo(W, P, blockIdx.x), s_hi = range_lo(W, P, blockIdx.x + 1);

  if (warp >= kXWarp0) {
    // ------------------------------------------------ activation conversion
    // Per stage, each (block b, row r) of the staged bf16 activations is
    // rewritten in place as fp16 x * 2^S, S putting the largest magnitude of
    // its 64 values in [2^14, 2^15) (0 for all zeros, Inf or NaN): exact for
    // every value above 2^-28 of that maximum. 2^-S (NF4: times
    // 1 / kTableScale, one fp32 rounding) goes to the stage's scale table for
    // the consumers' block sums. The kXWarps lanes of one
    // (block, row) take 8 / kXWarps of its 16-byte chunks each.
    constexpr int kChunks = 8 / kXWarps;
    const int xi = (warp - kXWarp0) * 32 + lane;
    const int h = xi % kXWarps, b = (xi / kXWarps) >> 3, r = (xi / kXWarps) & 7;
    int st = 0;          // stage slot and its phase parity, advanced per stage
    uint32_t ph = 0;
    for (int64_t s = s_lo; s < s_hi;) {
      const int64_t t = div_fast(s, KC);
      const int k0 = static_cast<int>(s - t * KC);
      const int k1 = static_cast<int>(min(KC, k0 + (s_hi - s)));
      const Tile tl = make_tile(t, p, batch_start, row_off, gexp);
      // rows past the batch feed only outputs that are never stored: skipped
      const bool live = r < tl.mrows;
      const uint32_t pair_mask = __ballot_sync(0xffffffffu, live);
      for (int kc = k0; kc < k1; ++kc, next_stage(st, ph)) {
        if (!warp_wait_one(&full[st], ph, abort_flag, hdr, limit_ns)) return;
        if (live) {
          char *row = smem + kXOff + st * kXStage + b * kBoxBytes + r * 128;
          uint4 v[kChunks];
          // bf16 magnitudes compare as integers, two per word
          uint32_t m4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            v[c] = *reinterpret_cast<const uint4 *>(row + (((kChunks * h + c) ^ r) << 4));
            m4[0] = __vmaxu2(m4[0], v[c].x & 0x7FFF7FFFu);
            m4[1] = __vmaxu2(m4[1], v[c].y & 0x7FFF7FFFu);
            m4[2] = __vmaxu2(m4[2], v[c].z & 0x7FFF7FFFu);
            m4[3] = __vmaxu2(m4[3], v[c].w & 0x7FFF7FFFu);
          }
          uint32_t mx2 = __vmaxu2(__vmaxu2(m4[0], m4[1]), __vmaxu2(m4[2], m4[3]));
          if (kXWarps == 2) mx2 = __vmaxu2(mx2, __shfl_xor_sync(pair_mask, mx2, 1));
          const uint32_t mx = max(mx2 & 0xFFFFu, mx2 >> 16);
          const int eb = static_cast<int>(mx >> 7);   // biased exponent of the largest magnitude
          int S = 0;
          if (mx != 0 && eb < 255) S = 14 - (eb == 0 ? -126 : eb - 127);
          S = S > 126 ? 126 : S;
          const float sc = __uint_as_float(static_cast<uint32_t>(S + 127) << 23);
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            const uint32_t in[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
            uint32_t out[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const __half2 hv = __floats2half2_rn(__uint_as_float(in[j] << 16) * sc,
                                                   __uint_as_float(in[j] & 0xFFFF0000u) * sc);
              out[j] = *reinterpret_cast<const uint32_t *>(&hv);
            }
            *reinterpret_cast<uint4 *>(row + (((kChunks * h + c) ^ r) << 4)) =
                make_uint4(out[0], out[1], out[2], out[3]);
          }
          if (h == 0)
            reinterpret_cast<float *>(smem + kXsOff + st * kXsStage)[b * 8 + r] =
                __uint_as_float(static_cast<uint32_t>(127 - S) << 23) * (MX ? 1.0f : kTableInv);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&xready[st]);
      }
      s += k1 - k0;
    }
    return;
  }

  if (warp >= kConsumerWarps) {
    // ------------------------------------------------------------ producers
    // Lane 0 of the copy warp issues the tensor copies (one byte-count
    // arrival); the lanes of the scale warps copy scales and, with a gather,
    // activation rows as 16-byte copies (one arrival per lane when its
    // copies land). Scale warp sw takes the units i with i % kScaleWarps ==
    // sw.
    const bool scale_warp = warp >= kScaleWarp0;
    const int sw = warp - kScaleWarp0;
    const bool tma_lane = warp == kTmaWarp && lane == 0;
    // WIDE: one copy per (unit, row group, row); else one 4-byte copy per
    // (unit, row group, row, block)
    constexpr bool wide = WIDE;
    // wide: lane copies row r of row group wrg of units wu + 2 kScaleWarps jj;
    // narrow: lane copies block blk of row r of its units
    const int r = wide ? (lane & 7) : (lane >> 2);
    const int blk = wide ? 0 : (lane & 3);
    const int wrg = (lane >> 3) & 1, wu = sw + kScaleWarps * (lane >> 4);
    const int64_t total_rows = static_cast<int64_t>(p.E) * p.N;
    // scale bytes of the whole stack (2-byte encodings: the last word read
    // must stay inside it)
    const int64_t scale_bytes = total_rows * p.KB * 2;
    // gathered activations: lane copies chunks sw * kGChunks + cc of row
    // gr = lane % 8 of block gb = lane / 8
    constexpr int kGChunks = 8 / kScaleWarps;
    const int gr = lane & 7, gb = lane >> 3;
    uint32_t it = 0;
    bool ok = true;
    for (int64_t s = s_lo; s < s_hi && ok;) {
      const int64_t t = div_fast(s, KC);
      const int k0 = static_cast<int>(s - t * KC);
      const int k1 = static_cast<int>(min(KC, k0 + (s_hi - s)));
      const Tile tl = make_tile(t, p, batch_start, row_off, gexp);
      const int64_t ebase = static_cast<int64_t>(tl.e) * p.N;
      // weight row of unit i, row group rgi, row r within the group
      auto wrow = [&](int i, int rgi, int rr) -> int64_t {
        const int64_t j = tl.j0 + i;
        if (p.epi == 0) return ebase + 16 * j + 8 * rgi + rr;
        if (p.epi == 1) return ebase + 8 * j + rr + rgi * (p.N / 2);
        return ebase + 2 * (8 * j + rr) + rgi;
      };
      uint32_t vmask = 0;   // bit 2i+rgi: row r of that row group exists in the stack
      const uint16_t *hrow = nullptr;
      // scale elements: of row r of unit 0 / row group 0 at block blk, and
      // the steps from one unit and from one row group to the next
      const int64_t e00 = wrow(0, 0, r) * p.KB + blk;
      const int64_t du = (wrow(1, 0, r) - wrow(0, 0, r)) * p.KB;
      const int64_t dg = (wrow(0, 1, r) - wrow(0, 0, r)) * p.KB;
      if (scale_warp)
        for (int i = 0; i < tl.nunits; ++i)
#pragma unroll
          for (int rgi = 0; rgi < 2; ++rgi)
            if (wrow(i, rgi, r) < ebase + p.N) vmask |= 1u << (2 * i + rgi);
      if (scale_warp && gather && gr < tl.mrows) {
        const int32_t slot = sorted_idx[tl.row0 + gr];   // checked in range up front
        hrow = hidden + static_cast<int64_t>(slot / top_k) * p.K;
      }
      for (int kc = k0; kc < k1; ++kc, ++it) {
        const int st = static_cast<int>(it % kStages);
        const uint32_t ph = (it / kStages) & 1u;
        if (!warp_wait_one(&empty[st], ph ^ 1u, abort_flag, hdr, limit_ns)) { ok = false; break; }
        if (tma_lane) {
          mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(tl.nunits * 16 * 128 +
                                                                 (gather ? 0 : kXStage)));
          char *ws = smem + kWOff + st * kWStage;
          if (p.epi == 0) {
            load_weight_rows(ws, wmaps, kc * 128, wrow(0, 0, 0), tl.nunits * 16, &full[st]);
          } else if (p.epi == 1) {   // gate rows, then the matching up rows 8 KB further
            load_weight_rows(ws, wmaps, kc * 128, wrow(0, 0, 0), tl.nunits * 8, &full[st]);
            load_weight_rows(ws + kTileUnits * kBoxBytes, wmaps, kc * 128, wrow(0, 1, 0),
                             tl.nunits * 8, &full[st]);
          } else {                   // interleaved: even rows (gate), then odd rows (up)
            const int64_t pair0 = (ebase >> 1) + 8 * static_cast<int64_t>(tl.j0);
            load_parity_rows(ws, wmaps, kc * 128, pair0, 0, tl.nunits * 8, &full[st]);
            load_parity_rows(ws + kTileUnits * kBoxBytes, wmaps, kc * 128, pair0, 1,
                             tl.nunits * 8, &full[st]);
          }
          // the batch's activations for the stage's 4 blocks in one copy (a
          // block past K is zero-filled by the copy engine)
          if (!gather)
            tma_load_3d(smem + kXOff + st * kXStage, &xmap, 0, static_cast<int>(tl.row0),
                        kc * kStageBlocks, &full[st]);
        }
        if (scale_warp) {
          // stage layout [unit][row group][row][block], one 4-byte word
          // each: the consumer lane of row g reads word g * 4 + blk of the
          // unit's two row groups
          const uint32_t as = smem_u32(smem + kAOff + st * kAStage + r * 16 + blk * 4);
          const int64_t ek = e00 + kc * kStageBlocks;   // element of unit 0, row group 0
          if (wide) {
            const float *fk = static_cast<const float *>(scales) + ek;
#pragma unroll
            for (int jj = 0; jj < 4 / kScaleWarps; ++jj) {
              const int i = wu + 2 * kScaleWarps * jj;
              const bool v = (vmask >> (2 * i + wrg)) & 1u;
              cp_async16(as + i * 256 + wrg * 128, v ? fk + i * du + wrg * dg : scales,
                         v ? 16u : 0u);
            }
          } else if (scale_kind == kScaleF32) {
            const bool kok = kc * kStageBlocks + blk < p.KB;
            const float *fk = static_cast<const float *>(scales) + ek;
            for (int i = sw; i < tl.nunits; i += kScaleWarps) {
#pragma unroll
              for (int rgi = 0; rgi < 2; ++rgi) {
                const bool v = kok && ((vmask >> (2 * i + rgi)) & 1u);
                cp_async4(as + i * 256 + rgi * 128, v ? fk + i * du + rgi * dg : scales,
                          v ? 4u : 0u);
              }
            }
          } else {
            // the 4-byte word that holds the (row, block)'s 2 bytes (the last
            // word of the stack is read only as far as the stack goes)
            const bool kok = kc * kStageBlocks + blk < p.KB;
            const char *cb = static_cast<const char *>(scales);
            for (int i = sw; i < tl.nunits; i += kScaleWarps) {
#pragma unroll
              for (int rgi = 0; rgi < 2; ++rgi) {
                const bool v = kok && ((vmask >> (2 * i + rgi)) & 1u);
                const int64_t wb = ((ek + i * du + rgi * dg) * 2) & ~int64_t{3};
                cp_async4(as + i * 256 + rgi * 128, v ? cb + wb : scales,
                          v ? (wb + 4 <= scale_bytes ? 4u : 2u) : 0u);
              }
            }
          }
          if (gather) {
            // the batch's rows of x for this stage's 4 blocks, through
            // sorted_idx, into the layout the tensor copy gives (128-byte
            // swizzle: chunk c of row r at chunk c ^ r); rows past the batch
            // and blocks past K are zero-filled
            const int kbx = kc * kStageBlocks + gb;
            const bool v = hrow != nullptr && kbx < p.KB;
            const uint32_t dst = smem_u32(smem + kXOff + st * kXStage + gb * kBoxBytes + gr * 128);
#pragma unroll
            for (int cc = 0; cc < kGChunks; ++cc) {
              const int c = kGChunks * sw + cc;
              cp_async16(dst + ((c ^ gr) << 4), v ? hrow + kbx * 64 + c * 8 : hidden,
                         v ? 16u : 0u);
            }
          }
          cp_async_arrive_noinc(&full[st]);
        }
      }
      s += k1 - k0;
    }
    if (scale_warp) cp_async_wait_all();
    if (tma_lane) {
      // the copies of the last stages must land before the CTA exits
      const uint32_t n = it < static_cast<uint32_t>(kStages) ? it : static_cast<uint32_t>(kStages);
      for (uint32_t d = 0; d < n; ++d) {
        const uint32_t gg = it - 1 - d;
        drain_wait(&full[gg % kStages], (gg / kStages) & 1u);
      }
    }
    return;
  }

  // --------------------------------------------------------------- consumers
  // Warp w takes 64-element block w / 4 of every stage for units 2 (w % 4)
  // and 2 (w % 4) + 1 of the tile; the four block warps of a unit pair sum
  // their partial results when the tile piece ends.
  const int g = lane >> 2, q = lane & 3;
  const int up = warp & 3;                  // unit pair
  const int blk = warp >> 2;                // block of the stage
  // This lane's K-elements of a block: the 8 of 16-byte activation chunk cA
  // = q and the 8 of chunk cB = q + 4 (packed bytes 4 cA .. 4 cA + 3 of the
  // block, and 16 bytes on). The first two MMAs of a block take chunks 0..3
  // (the block's first 32 elements), the last two chunks 4..7, which MXFP4's
  // per-32 scales need. With the 128-byte swizzle (chunk ^ row) the packed
  // words of chunk q of rows g = 0..7 fall in 32 distinct banks. The
  // activation chunks are read in the order f, f ^ 4 with f = 0, 5, 2, 7 for
  // q = 0..3 (f is cA or cB): no two values of f differ only in bit 0, so the
  // 8 lanes (rows g, g + 1) that share a 16-byte read's wavefront hit 8
  // distinct chunks; lanes with odd q swap the two reads back afterwards.
  // Both reads run free of bank conflicts.
  // (NF4 sums all four MMAs of a block into one value, so its lanes simply
  // take chunk f for the first two MMAs and f ^ 4 for the last two: no swap.)
  const int f = (q & 2) | ((q & 1) ? 5 : 0);
  const int cA = MX ? q : f, cB = MX ? (q | 4) : (f ^ 4);
  const int offA = g * 128 + (((2 * blk + (cA >> 2)) ^ g) << 4) + 4 * (cA & 3);
  const int offB = g * 128 + (((2 * blk + (cB >> 2)) ^ g) << 4) + 4 * (cB & 3);
  const int xoffF = blk * kBoxBytes + g * 128 + ((f ^ g) << 4);
  const int xoffG = blk * kBoxBytes + g * 128 + ((f ^ 4 ^ g) << 4);
  const bool xswap = MX && (q & 1) != 0;
  const uint32_t lutlane = static_cast<uint32_t>(kLutOff) | (static_cast<uint32_t>(lane) * 4u);
  constexpr bool two_byte = SK != kScaleF32;
  if (hook_ns != 0 && !warp_wait_all(never, 0, abort_flag, hdr, limit_ns)) return;
  int st = 0;            // stage slot and its phase parity, advanced per stage
  uint32_t ph = 0, ep = 0;
  for (int64_t s = s_lo; s < s_hi;) {
    const int64_t t = div_fast(s, KC);
    const int k0 = static_cast<int>(s - t * KC);
    const int k1 = static_cast<int>(min(KC, k0 + (s_hi - s)));
    const Tile tl = make_tile(t, p, batch_start, row_off, gexp);
    const bool act0 = 2 * up < tl.nunits, act1 = 2 * up + 1 < tl.nunits;
    // Two-byte scales: bit 2 uu + r is set if row group r of unit uu finds
    // its 2 bytes in the high half of the copied word (odd element index;
    // the element index of (row, block kc * 4 + blk) has the parity of
    // row * KB + blk).
    uint32_t hsel = 0;
    if (two_byte) {
      const int64_t ebase = static_cast<int64_t>(tl.e) * p.N;
#pragma unroll
      for (int uu = 0; uu < 2; ++uu) {
        const int64_t j = tl.j0 + 2 * up + uu;
        const int64_t w0 = p.epi == 0 ? ebase + 16 * j + g
                           : (p.epi == 1 ? ebase + 8 * j + g : ebase + 2 * (8 * j + g));
        const int64_t w1 = p.epi == 0 ? w0 + 8 : (p.epi == 1 ? w0 + p.N / 2 : w0 + 1);
        hsel |= static_cast<uint32_t>((w0 * p.KB + blk) & 1) << (2 * uu);
        hsel |= static_cast<uint32_t>((w1 * p.KB + blk) & 1) << (2 * uu + 1);
      }
    }
    // C fragment: [0] weight row g, activation row 2q; [1] row g, 2q + 1;
    // [2] row g + 8 (SwiGLU: the matching up row), 2q; [3] row g + 8, 2q + 1
    float acc[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
    for (int kc = k0; kc < k1; ++kc, next_stage(st, ph)) {
      // the activation warps arrive on xready only after they have observed
      // this stage's copies complete (full), so this one wait also orders
      // the copied weights and scales before the reads below
      if (!warp_wait_sa(kBarOff + (2 * kStages + st) * 8, ph, a.hdr)) return;
      // a block past K (the last stage of a row whose K / 64 is not a
      // multiple of 4) would only add the zeros its copies filled in
      if (act0 && kc * kStageBlocks + blk < p.KB) {
        // (Shared-window addresses: region kXxx starts at address kXxx.)
        const uint32_t wst = kWOff + st * kWStage;
        // 2^-S of activation rows 2q and 2q + 1 in this block
        const float2 xs = lds_f2(kXsOff + st * kXsStage + (blk * 4 + q) * 8);
        const uint32_t ast = kAOff + st * kAStage + g * 16 + blk * 4;
        // (rows past the batch feed only outputs that are never stored)
        const uint32_t xst = kXOff + st * kXStage;
        const uint4 xf = lds_u4(xst + xoffF);
        const uint4 xg = lds_u4(xst + xoffG);
        const uint4 xa = xswap ? xg : xf;   // chunk cA
        const uint4 xb = xswap ? xf : xg;   // chunk cB
#pragma unroll
        for (int uu = 0; uu < 2; ++uu) {
          if (uu == 1 && !act1) break;
          const int ui = 2 * up + uu;
          // weight rows g and g + 8 of the unit (1 KB boxes of 8 rows)
          const uint32_t r0 = wst + (p.epi ? ui : 2 * ui) * kBoxBytes;
          const uint32_t r1 = wst + (p.epi ? kTileUnits + ui : 2 * ui + 1) * kBoxBytes;
          const uint32_t wa0 = lds_u32(r0 + offA);
          const uint32_t wb0 = lds_u32(r0 + offB);
          const uint32_t wa1 = lds_u32(r1 + offA);
          const uint32_t wb1 = lds_u32(r1 + offB);
          // scale words of rows g and g + 8 (row groups 0 and 1)
          uint32_t s0 = lds_u32(ast + ui * 256);
          uint32_t s1 = lds_u32(ast + ui * 256 + 128);
          // the 2 scale bytes of (row, block) sit in the low or the high half
          // of the copied 4-byte word, as the element index is even or odd
          if (two_byte) {
            s0 = (s0 >> (16 * ((hsel >> (2 * uu)) & 1u))) & 0xFFFFu;
            s1 = (s1 >> (16 * ((hsel >> (2 * uu + 1)) & 1u))) & 0xFFFFu;
          }
          // MMA k pairs (2q, 2q+1) and (2q+8, 2q+9) <- packed bytes (0, 1)
          // then (2, 3) of each word; activation registers in the same order.
          // (UPLO: rows g + 8, the up rows, with their remainders)
          uint32_t ha0[4], la0[4], ha1[4], la1[4], hb0[4], lb0[4], hb1[4], lb1[4];
          decode_word<1>(lutlane, wa0, ha0, la0);
          decode_word<UPLO ? 2 : 1>(lutlane, wa1, ha1, la1);
          decode_word<1>(lutlane, wb0, hb0, lb0);
          decode_word<UPLO ? 2 : 1>(lutlane, wb1, hb1, lb1);
          if (MX) {
            // the two 32-element halves separately, each times its e8m0
            // scale (byte 0 of the pair: first half, byte 1: second half)
            float c0[4], c1[4];
            mma_f16_z(c0, ha0[0], ha1[0], ha0[1], ha1[1], xa.x, xa.y);
            mma_f16(c0, ha0[2], ha1[2], ha0[3], ha1[3], xa.z, xa.w);
            mma_f16_z(c1, hb0[0], hb1[0], hb0[1], hb1[1], xb.x, xb.y);
            mma_f16(c1, hb0[2], hb1[2], hb0[3], hb1[3], xb.z, xb.w);
            const float e00 = e8m0_value(s0 & 0xFFu), e01 = e8m0_value(s0 >> 8);
            const float e10 = e8m0_value(s1 & 0xFFu), e11 = e8m0_value(s1 >> 8);
            acc[uu][0] = fmaf(fmaf(c1[0], e01, c0[0] * e00), xs.x, acc[uu][0]);
            acc[uu][1] = fmaf(fmaf(c1[1], e01, c0[1] * e00), xs.y, acc[uu][1]);
            acc[uu][2] = fmaf(fmaf(c1[2], e11, c0[2] * e10), xs.x, acc[uu][2]);
            acc[uu][3] = fmaf(fmaf(c1[3], e11, c0[3] * e10), xs.y, acc[uu][3]);
          } else {
            float ch[4];
            mma_f16_z(ch, ha0[0], ha1[0], ha0[1], ha1[1], xa.x, xa.y);
            mma_f16(ch, ha0[2], ha1[2], ha0[3], ha1[3], xa.z, xa.w);
            mma_f16(ch, hb0[0], hb1[0], hb0[1], hb1[1], xb.x, xb.y);
            mma_f16(ch, hb0[2], hb1[2], hb0[3], hb1[3], xb.z, xb.w);
            if (UPLO) {   // the up rows' remainders (gate rows' operands 0)
              float cl[4];
              mma_f16_z(cl, 0u, la1[0], 0u, la1[1], xa.x, xa.y);
              mma_f16(cl, 0u, la1[2], 0u, la1[3], xa.z, xa.w);
              mma_f16(cl, 0u, lb1[0], 0u, lb1[1], xb.x, xb.y);
              mma_f16(cl, 0u, lb1[2], 0u, lb1[3], xb.z, xb.w);
              ch[2] = fmaf(cl[2], kLoInv, ch[2]);
              ch[3] = fmaf(cl[3], kLoInv, ch[3]);
            }
            // absmax of rows g and g + 8 (fp32, or bf16 widened exactly)
            const float am0 = __uint_as_float(two_byte ? s0 << 16 : s0);
            const float am1 = __uint_as_float(two_byte ? s1 << 16 : s1);
            // block sum times absmax(row) and the activation rows' 2^-S
            acc[uu][0] = fmaf(ch[0], am0 * xs.x, acc[uu][0]);
            acc[uu][1] = fmaf(ch[1], am0 * xs.y, acc[uu][1]);
            acc[uu][2] = fmaf(ch[2], am1 * xs.x, acc[uu][2]);
            acc[uu][3] = fmaf(ch[3], am1 * xs.y, acc[uu][3]);
          }
        }
      }
      __syncwarp();
      arrive_elect_sa(kBarOff + (kStages + st) * 8);
    }
    if (act0) {
      if (!finish_piece(a, make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]),
                        make_float4(acc[1][0], acc[1][1], acc[1][2], acc[1][3]), t, tl,
                        k0 == 0 && k1 == KC, ep))
        return;
      ++ep;
    }
    s += k1 - k0;
  }
}

}  // namespace

size_t decode_workspace_bytes(int64_t M, int32_t N, int32_t K, int32_t G, int32_t swiglu) {
  (void)M; (void)N; (void)K; (void)G; (void)swiglu;
  const size_t P = static_cast<size_t>(device_sm_count());
  const size_t counters = (P * kPairs * 4 + 255) / 256 * 256;
  return kWsHeaderBytes + counters + P * 2 * kPairs * kPartialSlot * sizeof(float4);
}

size_t decode_zero_prefix_bytes(int64_t M, int32_t N, int32_t G, int32_t swiglu) {
  (void)M; (void)N; (void)G; (void)swiglu;
  const size_t P = static_cast<size_t>(device_sm_count());
  return kWsHeaderBytes + (P * kPairs * 4 + 255) / 256 * 256;
}

cudaError_t launch_decode_gemm(const GemmArgs &a, cudaStream_t stream) {
  if (static_cast<int64_t>(a.E) * a.N + a.N + 256 >= INT_MAX) return cudaErrorNotSupported;
  const bool mx = a.fmt == GNF4_FMT_MXFP4;
  WeightMaps wm;
  std::memset(&wm, 0, sizeof(wm));
  // packed weights as [E*N rows][K/2 bytes], boxes of (8 << i) rows x 128 bytes
  for (int i = 0; i < kNumWMaps; ++i) {
    if (!encode_tensor_map_2d(&wm.m[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w,
                              static_cast<uint64_t>(a.K / 2),
                              static_cast<uint64_t>(a.E) * static_cast<uint64_t>(a.N),
                              static_cast<uint64_t>(a.K / 2), 128, 8u << i,
                              CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  if (a.epi == GNF4_EPI_SWIGLU_INTERLEAVED) {
    // the same bytes as [E*N/2 pairs][2 parities][K/2]: boxes of one parity
    for (int i = 0; i < kNumIMaps; ++i) {
      const uint64_t dims[3] = {static_cast<uint64_t>(a.K / 2), 2,
                                static_cast<uint64_t>(a.E) * static_cast<uint64_t>(a.N) / 2};
      const uint64_t pitches[2] = {static_cast<uint64_t>(a.K / 2), static_cast<uint64_t>(a.K)};
      const uint32_t box[3] = {128, 1, 8u << i};
      if (!encode_tensor_map(&wm.im[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.w, dims, pitches, box,
                             CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    }
  }
  // activations viewed as [K/64 blocks][M rows][64 bf16]: one box = 4 blocks x
  // 8 rows x 64 elements, laid out in shared memory as 4 swizzled 1 KB tiles
  CUtensorMap xmap;
  std::memset(&xmap, 0, sizeof(xmap));
  if (a.hidden == nullptr) {
    const uint64_t dims[3] = {64, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.K / 64)};
    const uint64_t pitches[2] = {static_cast<uint64_t>(a.K) * 2, 128};
    const uint32_t box[3] = {64, kBatch, kStageBlocks};
    if (!encode_tensor_map(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.x, dims, pitches, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }

  const int P = device_sm_count();
  DecodeParams d;
  d.scales = a.scales;
  d.sizes = a.sizes;
  d.expert_ids = a.expert_ids;
  d.hidden = a.hidden;
  d.sorted_idx = a.sorted_idx;
  d.n_slots = a.n_tokens * a.top_k;
  d.top_k = a.top_k;
  d.G = a.G; d.M = a.M; d.N = a.N; d.K = a.K; d.E = a.E;
  d.scale_kind = mx ? kScaleE8m0 : (a.scale_dtype == GNF4_SCALE_BF16 ? kScaleBf16 : kScaleF32);
  d.epi = a.epi;
  d.alpha = a.alpha;
  d.limit = a.limit;
  d.y = a.y;
  d.hdr = static_cast<WsHeader *>(a.workspace);
  char *ws = static_cast<char *>(a.workspace);
  d.counters = reinterpret_cast<uint32_t *>(ws + kWsHeaderBytes);
  d.partials = reinterpret_cast<float4 *>(ws + decode_zero_prefix_bytes(a.M, a.N, a.G, a.swiglu));

  const bool bf = !mx && a.scale_dtype == GNF4_SCALE_BF16;
  // 16-byte scale copies: fp32 scales, the 4 blocks of a stage one aligned
  // run in every row
  const bool wide = !mx && !bf && (a.K / 64) % kStageBlocks == 0 &&
                    reinterpret_cast<uintptr_t>(a.scales) % 16 == 0;
  // SwiGLU (NF4): the up rows carry their code remainders
  const bool uplo = !mx && a.epi != GNF4_EPI_NONE;
  auto kernel = mx     ? decode_gemm_kernel<kScaleE8m0, false, false>
                : bf   ? (uplo ? decode_gemm_kernel<kScaleBf16, false, true>
                               : decode_gemm_kernel<kScaleBf16, false, false>)
                : wide ? (uplo ? decode_gemm_kernel<kScaleF32, true, true>
                               : decode_gemm_kernel<kScaleF32, true, false>)
                       : (uplo ? decode_gemm_kernel<kScaleF32, false, true>
                               : decode_gemm_kernel<kScaleF32, false, false>);
  const int ki = mx ? 6 : (bf ? 4 : wide ? 2 : 0) + (uplo ? 1 : 0);
  static bool configured[64][7] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev][ki]) {
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kSmemBytes);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64) configured[dev][ki] = true;
  }
  return launch_pdl(kernel, dim3(P), dim3(kThreads), static_cast<size_t>(kSmemBytes), stream, wm,
                    xmap, d);
}

}  // namespace gnf4
