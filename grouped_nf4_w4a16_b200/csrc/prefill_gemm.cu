// prefill_gemm.cu -- prefill-regime grouped NF4 GEMM on the 5th-generation
// tensor cores (tcgen05, TMEM, TMA), as a 2-SM MMA over CTA pairs.
//
// Passage: "grouped-nf4-gemm -- single-launch W4A16 GEMM over fused NF4 MoE
// expert stacks", opening section (one launch for all active experts, LUT
// decode, blockwise fp32 absmax, fp32 accumulation, bf16 epilogue, no bf16
// weight copy in memory) and "The claim" (prefill: compute-bound M, a
// register-LUT M-tile mainloop). With ~1000 activation rows per expert the
// contraction is dense and bound by tensor-core throughput.
//
// Tile = 256 weight rows of one expert x 256 activation rows of one group,
// computed as D[weight row][activation row] = W . x^T by a pair of CTAs on
// two SMs (a cluster of 2): CTA r of the pair owns weight rows 128 r .. +127
// (its TMEM lanes: the MMA's A and D) and activation rows 128 r .. +127 of
// the tile (its shared memory: half of the MMA's B). One tcgen05.mma with
// cta_group::2, issued by the pair's leader (r = 0), reads both halves, so
// every SM loads only half of the activation tile per K-step.
//
// Numerics (the tolerance needs more than one bf16 per weight): each weight
// row is scaled by 2^S, S = beta + 14 with 2^beta * max(absmax of the row) in
// [1, 2) (powers of two scale exactly); the scaled fp32 weight w'' = NF4 *
// absmax * 2^S is split into hi = bf16(w'') and the exact remainder
// w'' - hi, which is below 64 in magnitude and goes to e4m3. Each activation
// row is scaled by 2^s (its largest magnitude into [2^14, 2^15)) by a
// pre-pass that writes its bf16 copy (exact) and its e5m2 copy. Per K-step
// of 64:
//   hi pass: 4 x kind::f16, bf16 hi (TMEM) x bf16 x (shared memory), K = 16
//   lo pass: 2 x kind::f8f6f4, e4m3 remainder (TMEM) x e5m2 x (shared
//            memory), K = 32
// into one fp32 accumulator; the epilogue divides 2^S and 2^s out and rounds
// once to bf16. The lo pass runs at twice the bf16 rate, so a K-step costs
// 1.5 bf16 passes instead of 2.
//
// Roles per CTA (12 warps, one CTA per SM, the pair persistent over tiles):
//   warp 0  TMA: its half of the x tile (bf16, 128-byte swizzle) and of the
//           e5m2 tile (64-byte swizzle); both halves complete on the leader's
//           stage barrier (cta_group::2 copies), whose byte count the leader
//           sets for the pair. Ring of 6 stages.
//   warp 1  (leader) MMA issuer; commits signal both CTAs.
//   warp 2  allocates / frees the 512 TMEM columns (cta_group::2, in both CTAs).
//   warp 3  packed weights: this CTA's 128 rows x 4 K-steps (128 bytes a row)
//           per TMA box (128-byte swizzle), and their absmax values by
//           cp.async, into a 2-slot shared-memory ring. Decoders then read
//           16 contiguous bytes per row per K-step without bank conflicts,
//           instead of scattered global loads (one sector per row).
//   warps 4-11  decoders + epilogue: warp w owns TMEM lanes 32 (w % 4).. and
//           half of the K-step; each lane decodes its row's 32 codes through a
//           per-lane replicated table of the 16 code values, writes hi and
//           remainder to TMEM (tcgen05.st, a 5-stage ring); one lane per warp
//           then arrives on the leader's barrier. The epilogue reads the
//           accumulator back (tcgen05.ld) 32 tokens at a time and writes
//           each chunk through a shared-memory box with one bulk tensor
//           store.
// Every wait is bounded (2 s); on expiry the kernel records
// GNF4_DEVERR_TIMEOUT, lets its asynchronous work drain and returns through
// the final cluster barrier.
#include <cuda_fp8.h>

#include "launch.h"
#include "sm100.cuh"

namespace gnf4 {
namespace {

constexpr int kBM = 128;            // weight rows per CTA (TMEM lanes)
constexpr int kPairM = 256;         // weight rows per pair tile (MMA M)
constexpr int kBN = 256;            // activation rows per tile (MMA N)
constexpr int kBNh = 128;           // activation rows loaded by each CTA
constexpr int kBK = 64;             // K per stage
constexpr int kXStages = 6;         // activation ring (shared memory)
constexpr int kWQuads = 2;          // packed-weight ring: slots of 4 K-steps (shared memory)
constexpr int kWSlotBytes = kBM * 128;       // 16 KB: 128 rows x 128 packed bytes
constexpr int kASlotBytes = 4 * kBM * 4;     // 2 KB: absmax [4 blocks][128 rows]
constexpr int kAStages = 5;         // decoded-weight ring (TMEM)
constexpr int kThreads = 384;       // 12 warps
constexpr int kDecodeWarp0 = 4;
constexpr int kDecodeWarps = 8;     // warps 4..11
constexpr int kMaxG = GNF4_MAX_EXPERTS;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;     // accumulator: columns [0, 256)
constexpr uint32_t kACol = 256;     // stage s: hi at kACol + 48 s (32 columns), lo at +32 (16)
constexpr uint32_t kAStageCols = 48;
constexpr int kXStageBytes = kBNh * kBK * 2;   // 16 KB: this CTA's half of the x tile, bf16
constexpr int kX8StageBytes = kBNh * kBK;      // 8 KB: the same half, e5m2
constexpr uint32_t kPairStageBytes = 2u * (kXStageBytes + kX8StageBytes);
constexpr int kLoShift = 14;        // weights are scaled by 2^(beta + 14)
static_assert(kACol + kAStages * kAStageCols <= kTmemCols, "TMEM columns");

// Shared memory layout (dynamic, 1024-aligned base; identical in both CTAs,
// which the pair MMA relies on: B's second half sits at the same offset in
// the peer).
constexpr int kXOff = 0;                                    // x ring
constexpr int kX8Off = kXOff + kXStages * kXStageBytes;     // e5m2 ring
constexpr int kWOff = kX8Off + kXStages * kX8StageBytes;    // packed-weight ring
constexpr int kAbsOff = kWOff + kWQuads * kWSlotBytes;      // absmax ring
constexpr int kLutOff = kAbsOff + kWQuads * kASlotBytes;    // float [16 codes][32 lanes]
constexpr int kLutBytes = 16 * 32 * 4;
constexpr int kTileStartOff = kLutOff + kLutBytes;          // int[kMaxG + 1]
constexpr int kRowOffOff = kTileStartOff + (kMaxG + 4) * 4;
constexpr int kGSizeOff = kRowOffOff + kMaxG * 4;
constexpr int kGExpOff = kGSizeOff + kMaxG * 4;
constexpr int kBarOff = kGExpOff + kMaxG * 4;               // mbarriers
constexpr int kNumBars = 2 * kXStages + 2 * kAStages + 2 * kWQuads + 3;
constexpr int kMiscOff = kBarOff + kNumBars * 8;            // int[8]
// epilogue staging: per decoder warp one box of 32 tokens x 32 rows bf16
constexpr int kOutChunkBytes = 32 * 32 * 2;
constexpr int kOutOff = ((kMiscOff + 8 * 4 + 1023) / 1024) * 1024;
constexpr int kSmemBytes = kOutOff + kDecodeWarps * kOutChunkBytes + 2048;   // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "fits one CTA per SM");
// The base is 2048-aligned and so is the table: a lookup address is the
// lane's slot OR code * 128 (bits 7..10), with no add.
static_assert(kLutOff % 2048 == 0, "table alignment");

// ------------------------------------------------------------------ PTX
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Both CTAs of the pair, all threads: release our writes, acquire the peer's.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared::cluster address of the object at `p`'s offset in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void *p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

// Arrive on the mbarrier at `p`'s offset in CTA `rank` (possibly this CTA).
// CTA-scope semantics: the arrivals only hand over TMEM contents, which the
// tcgen05 wait and fence order, not generic memory (a cluster-scope release
// would also wait for every load the thread has in flight).
__device__ __forceinline__ void mbar_arrive_cta(const uint64_t *p, uint32_t rank) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr(p, rank))
               : "memory");
}

// Bounded wait on a barrier of this CTA that the peer CTA may also arrive
// on (the arrivals carry no data this wait has to acquire beyond CTA scope).
__device__ __forceinline__ bool wait_bar_cluster(uint64_t *bar, uint32_t parity,
                                                 volatile int *abort_flag, WsHeader *hdr) {
  return wait_bar(bar, parity, abort_flag, hdr);
}

// 2-D tensor copy into this CTA's shared memory whose byte count completes
// on the mbarrier at `bar`'s offset in the pair leader (CTA 0).
__device__ __forceinline__ void tma_load_2d_pair(void *smem_dst, const CUtensorMap *map, int c0,
                                                 int c1, const uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(cluster_addr(bar, 0))
      : "memory");
}

// Bulk tensor store shared -> global of one box (c0 innermost, its byte
// offset a multiple of 16; elements outside the tensor are not written), in
// this thread's bulk group.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *smem_src, int c0,
                                             int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(c0), "r"(c1), "r"(smem_u32(smem_src))
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// none of this thread's bulk groups is still reading shared memory
__device__ __forceinline__ void bulk_wait_read_0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// every bulk group of this thread complete (its writes done)
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// this thread's shared-memory writes visible to the bulk copy engine
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// D[tmem] (+)= A[tmem] . B[smem desc]^T over the pair: kind::f16 (bf16 x bf16).
__device__ __forceinline__ void mma_pair_f16(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same with kind::f8f6f4: e4m3 A (TMEM) x e5m2 B (shared memory), K = 32.
__device__ __forceinline__ void mma_pair_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on the mbarrier at `bar`'s offset in every CTA of `mask` once all
// MMAs issued so far by this thread have completed.
__device__ __forceinline__ void mma_commit_pair(const uint64_t *bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory operand descriptors, K-major, descriptor version 1:
// bf16 tile: 128-byte rows with the 128-byte swizzle, 8-row groups 1024 B apart;
// e5m2 tile: 64-byte rows with the 64-byte swizzle, 8-row groups 512 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}
__device__ __forceinline__ uint64_t sw64_desc(uint32_t smem_addr) {
  return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(512 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(4) << 61);
}

// Instruction descriptors (K-major A and B, fp32 D, M = 256 over the pair,
// N = 256): kind::f16 with bf16 A and B; kind::f8f6f4 with e4m3 A, e5m2 B.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                            (static_cast<uint32_t>(kBN >> 3) << 17) |
                            (static_cast<uint32_t>(kPairM >> 4) << 24);
constexpr uint32_t kIdescF8 = (1u << 4) | (0u << 7) | (1u << 10) |
                              (static_cast<uint32_t>(kBN >> 3) << 17) |
                              (static_cast<uint32_t>(kPairM >> 4) << 24);

struct TileInfo {
  int64_t row0;     // first activation row of the pair tile
  int32_t rows;     // valid activation rows (1..256)
  int32_t n0;       // first output column of the pair tile (256 per tile; 128 with SwiGLU)
  int32_t e;        // expert
};

// Pair tile t: groups in order, within a group weight-row tile j outer and
// token tile i inner (pairs running at the same time share weight tiles).
__device__ __forceinline__ TileInfo tile_info(int t, int G, const int *tile_start,
                                              const int *row_off, const int *gsize,
                                              const int *gexp, int ncols_tile) {
  int lo = 0, hi = G;   // tile_start[lo] <= t < tile_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_start[mid] <= t) lo = mid; else hi = mid;
  }
  const int local = t - tile_start[lo];
  const int tt = (gsize[lo] + kBN - 1) / kBN;   // token tiles of the group
  const int j = local / tt, i = local - j * tt;
  TileInfo ti;
  ti.row0 = static_cast<int64_t>(row_off[lo]) + static_cast<int64_t>(i) * kBN;
  ti.rows = min(kBN, gsize[lo] - i * kBN);
  ti.n0 = j * ncols_tile;
  ti.e = gexp[lo];
  return ti;
}

// Scale encodings (PrefillParams::scale_kind).
constexpr int kScaleF32 = 0;    // NF4 absmax, fp32
constexpr int kScaleBf16 = 1;   // NF4 absmax, bf16
constexpr int kScaleE8m0 = 2;   // MXFP4: one e8m0 byte per 32 elements (a pair per K-step)

struct PrefillParams {
  const uint8_t *w;
  const void *scales;           // fp32 / bf16 absmax [E][N][K/64] or e8m0 [E][N][K/32]
  const float *tok_inv;         // 2^-s per activation row (written by the prep kernel)
  const int32_t *sizes;
  const int32_t *expert_ids;
  const int32_t *sorted_idx;    // gather: every entry must lie in [0, n_slots) (checked)
  int64_t n_slots;
  int32_t G;
  int64_t M;
  int32_t N, K, E;
  int32_t scale_kind;
  int32_t epi;                  // 0 none, 1 SwiGLU on halves, 2 SwiGLU on interleaved rows
  float alpha, limit;
  uint16_t *y;
  int32_t bulk_out;
  WsHeader *hdr;
};

// Weight row (within the expert) of local row rl (0..127) of CTA `rank` in
// a pair tile whose first output column is n0. Without SwiGLU rows are the
// output columns. With SwiGLU a warp's 32 TMEM lanes hold 16 gate rows and
// their 16 up rows: halves layout (epilogue 1): lanes 0-15 gate rows j..j+15,
// lanes 16-31 up rows N/2 + j..; interleaved layout (epilogue 2): lane l row
// 2 j + l (gate rows even, up rows odd), so the 128 rows are contiguous.
// *col: the output column of the row's pair; *valid: the row exists.
__device__ __forceinline__ int64_t weight_row(const PrefillParams &p, int n0, uint32_t rank,
                                              int rl, bool *valid) {
  if (p.epi == 0) {
    const int64_t n = n0 + kBM * static_cast<int64_t>(rank) + rl;
    *valid = n < p.N;
    return n;
  }
  const int qq = rl >> 5, l = rl & 31;
  if (p.epi == 1) {
    const int64_t j = n0 + 64 * static_cast<int64_t>(rank) + 16 * qq + (l & 15);
    *valid = j < p.N / 2;
    return l < 16 ? j : p.N / 2 + j;
  }
  const int64_t j = n0 + 64 * static_cast<int64_t>(rank) + 16 * qq + (l >> 1);
  *valid = j < p.N / 2;
  return 2 * j + (l & 1);
}

// A row maximum of the block scales is gathered from raw loads: the raw bits
// of element idx of the scale array (fp32, bf16, or an e8m0 pair at 2-byte
// element idx), and their magnitude as fp32 (for e8m0 the larger of the
// pair). The two are split so that a load issued ahead is only consumed
// where its value is needed.
__device__ __forceinline__ uint32_t scale_raw_at(const PrefillParams &p, int64_t idx) {
  if (p.scale_kind == kScaleF32)
    return __float_as_uint(__ldg(static_cast<const float *>(p.scales) + idx));
  return __ldg(static_cast<const unsigned short *>(p.scales) + idx);
}
__device__ __forceinline__ float scale_mag(const PrefillParams &p, uint32_t raw) {
  if (p.scale_kind == kScaleF32) return fabsf(__uint_as_float(raw));
  if (p.scale_kind == kScaleBf16) return fabsf(__uint_as_float(raw << 16));
  const uint32_t m = max(raw & 0xFFu, raw >> 8);
  return m == 255u ? __uint_as_float(0x7FC00000u)
                   : (m == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(m << 23));
}
__device__ __forceinline__ float scale_max_at(const PrefillParams &p, int64_t idx) {
  return scale_mag(p, scale_raw_at(p, idx));
}

// Warp-uniform bounded wait with cluster-scope acquire: lane 0 waits, every
// lane gets the same answer (warp-collective instructions follow).
__device__ __forceinline__ bool warp_wait_cluster(uint64_t *bar, uint32_t parity,
                                                  volatile int *abort_flag, WsHeader *hdr) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wait_bar_cluster(bar, parity, abort_flag, hdr) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// SK: the scale encoding (kScaleE8m0 = MXFP4, one bf16 pass); SWIGLU: the
// epilogue pairs gate and up rows (the halves or the interleaved layout,
// chosen at run time).
template <int SK, bool SWIGLU>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_gemm_kernel(const __grid_constant__ CUtensorMap xmap,
                        const __grid_constant__ CUtensorMap x8map,
                        const __grid_constant__ CUtensorMap wmap,
                        const __grid_constant__ CUtensorMap w4map,
                        const __grid_constant__ CUtensorMap ymap,
                        const PrefillParams pin) {
  // A local copy that the helpers take by reference: after inlining it lives
  // in registers; the parameter block's own address is never taken (a use
  // through such an address would be a memory load that every asm memory
  // clobber forces to repeat).
  constexpr bool MX = SK == kScaleE8m0;
  PrefillParams p = pin;
  p.scale_kind = SK;             // compile-time from here on
  if (!SWIGLU) p.epi = 0;
  const float *__restrict__ tok_inv = p.tok_inv;
  const int32_t *__restrict__ sizes = p.sizes;
  const int32_t *__restrict__ expert_ids = p.expert_ids;
  const int32_t G = p.G, N = p.N, K = p.K, E = p.E;
  const int64_t M = p.M;
  uint16_t *__restrict__ y = p.y;
  const int32_t bulk_out = p.bulk_out;
  WsHeader *hdr = p.hdr;
  // output columns per pair tile, and of y
  const int ncols_tile = p.epi ? kPairM / 2 : kPairM;
  const int64_t ncols = p.epi ? N / 2 : N;
  extern __shared__ char smem_raw[];
  char *smem = reinterpret_cast<char *>((reinterpret_cast<uintptr_t>(smem_raw) + 2047) &
                                        ~static_cast<uintptr_t>(2047));
  char *xs = smem + kXOff;
  char *x8s = smem + kX8Off;
  int *tile_start = reinterpret_cast<int *>(smem + kTileStartOff);
  int *row_off = reinterpret_cast<int *>(smem + kRowOffOff);
  int *gsize = reinterpret_cast<int *>(smem + kGSizeOff);
  int *gexp = reinterpret_cast<int *>(smem + kGExpOff);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBarOff);
  uint64_t *x_full = bars;                  // [kXStages] (leader) both halves landed
  uint64_t *x_free = x_full + kXStages;     // [kXStages] (each CTA) the MMA is done with them
  uint64_t *a_full = x_free + kXStages;     // [kAStages] (leader) both CTAs' weights in TMEM
  uint64_t *a_free = a_full + kAStages;     // [kAStages] (each CTA) the MMA is done with them
  uint64_t *w_full = a_free + kAStages;     // [kWQuads] (each CTA) packed bytes + absmax landed
  uint64_t *w_free = w_full + kWQuads;      // [kWQuads] (each CTA) decoders done with the slot
  uint64_t *d_full = w_free + kWQuads;      // (each CTA) accumulator complete
  uint64_t *d_empty = d_full + 1;           // (leader) both CTAs read their accumulators out
  uint64_t *drain = d_full + 2;             // (leader) final MMA drain
  int *misc = reinterpret_cast<int *>(smem + kMiscOff);
  volatile int *abort_flag = &misc[1];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);
  pdl_trigger();

  // ---- set-up: decode table, barriers, TMEM (no global memory yet)
  for (int i = tid; i < 16 * 32; i += kThreads) {
    const int c = i >> 5;
    float v = nf4_value(c);
    if (MX) {   // e2m1: sign, 2 exponent bits (bias 1), 1 mantissa bit
      const int m = c & 7;
      const float mag = m < 2 ? 0.5f * m : static_cast<float>(2 + (m & 1)) * exp2f(static_cast<float>((m >> 1) - 2));
      v = (c & 8) ? -mag : mag;
    }
    reinterpret_cast<float *>(smem + kLutOff)[i] = v;
  }
  if (tid == 0) {
    misc[0] = 0;
    misc[1] = 0;
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(&x_full[s], 1);                  // the leader's byte-count arrival
      mbar_init(&x_free[s], 1);                  // the leader's commit
    }
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(&a_full[s], 2 * kDecodeWarps);   // one per decoder warp of each CTA
      mbar_init(&a_free[s], 1);                  // the leader's commit
    }
    for (int q = 0; q < kWQuads; ++q) {
      mbar_init(&w_full[q], 32 + 1);             // 32 cp.async arrivals + the byte-count arrival
      mbar_init(&w_free[q], kDecodeWarps);
    }
    mbar_init(d_full, 1);
    mbar_init(d_empty, 2 * kDecodeWarps);
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tensormap(&xmap);
    prefetch_tensormap(&x8map);
    prefetch_tensormap(p.epi == 1 ? &w4map : &wmap);
    if (bulk_out) prefetch_tensormap(&ymap);
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&misc[4])),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }

  pdl_wait();   // inputs may come from the previous kernel on the stream

  // ---- group table (validated; both CTAs compute the same one)
  __shared__ int s_wsum[2][kThreads / 32];
  const int NJ = static_cast<int>((ncols + ncols_tile - 1) / ncols_tile);
  const int per = (G + kThreads - 1) / kThreads;
  const int g0 = min(G, tid * per), g1 = min(G, g0 + per);
  int my_rows = 0, my_tiles = 0, bad = 0;
  for (int g = g0; g < g1; ++g) {
    const int sz = sizes[g];
    const int e = expert_ids[g];
    if (sz < 0) bad |= GNF4_DEVERR_SIZES;
    if (sz > 0 && (e < 0 || e >= E)) bad |= GNF4_DEVERR_EXPERT;
    gsize[g] = sz;
    gexp[g] = e;
    my_rows += max(sz, 0);
    my_tiles += sz > 0 ? ((sz + kBN - 1) / kBN) * NJ : 0;
  }
  __syncthreads();
  if (bad) atomicOr(&misc[0], bad);
  int vr = my_rows, vt = my_tiles;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, vr, o);
    const int b = __shfl_up_sync(0xffffffffu, vt, o);
    if (lane >= o) { vr += a; vt += b; }
  }
  if (lane == 31) { s_wsum[0][warp] = vr; s_wsum[1][warp] = vt; }
  __syncthreads();
  int wr = 0, wt = 0, tot_r = 0, tot_t = 0;
  for (int i = 0; i < kThreads / 32; ++i) {
    if (i < warp) { wr += s_wsum[0][i]; wt += s_wsum[1][i]; }
    tot_r += s_wsum[0][i];
    tot_t += s_wsum[1][i];
  }
  {
    int r = wr + vr - my_rows, c = wt + vt - my_tiles;
    for (int g = g0; g < g1; ++g) {
      row_off[g] = r;
      tile_start[g] = c;
      const int sz = max(gsize[g], 0);
      r += sz;
      c += sz > 0 ? ((sz + kBN - 1) / kBN) * NJ : 0;
    }
    if (tid == 0) tile_start[G] = tot_t;
  }
  if (tid == 0 && static_cast<int64_t>(tot_r) != M) atomicOr(&misc[0], GNF4_DEVERR_SIZES);
  if (p.sorted_idx != nullptr) {   // gathered rows: every slot in range before any work
    int badslot = 0;
    for (int64_t i = tid; i < M; i += kThreads) {
      const int32_t sl = __ldg(p.sorted_idx + i);
      if (sl < 0 || sl >= p.n_slots) badslot = 1;
    }
    if (__syncthreads_or(badslot) && tid == 0) atomicOr(&misc[0], GNF4_DEVERR_SLOT);
  }
  // both CTAs: barriers initialised and TMEM allocated before any remote access
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[4]);
  const int errbits = misc[0];
  const int KB = K / kBK;
  const int tiles = tot_t;

  if (errbits == 0) {
    if (warp == 0) {
      // --------------------------------------------------------- TMA producer
      if (lane == 0) {
        uint32_t g = 0;   // stage ring counter
        for (int t = pair; t < tiles && !*abort_flag; t += npairs) {
          const TileInfo ti = tile_info(t, G, tile_start, row_off, gsize, gexp, ncols_tile);
          const int xrow = static_cast<int>(ti.row0) + kBNh * static_cast<int>(rank);
          bool ok = true;
          for (int kb = 0; kb < KB; ++kb, ++g) {
            const int s = g % kXStages;
            const uint32_t ph = (g / kXStages) & 1u;
            if (!wait_bar_cluster(&x_free[s], ph ^ 1u, abort_flag, hdr)) { ok = false; break; }
            if (leader) mbar_arrive_expect_tx(&x_full[s], kPairStageBytes);
            tma_load_2d_pair(xs + s * kXStageBytes, &xmap, kb * kBK, xrow, &x_full[s]);
            tma_load_2d_pair(x8s + s * kX8StageBytes, &x8map, kb * kBK, xrow, &x_full[s]);
          }
          if (!ok) break;
        }
        // the leader's stage barriers count both CTAs' bytes: the last stages
        // issued must have landed before either CTA exits
        if (leader) {
          for (uint32_t d = 0; d < kXStages && d < g; ++d) {
            const uint32_t gg = g - 1 - d;
            drain_wait(&x_full[gg % kXStages], (gg / kXStages) & 1u);
          }
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------- MMA issuer (leader)
      if (leader && lane == 0) {
        uint32_t g = 0;
        uint32_t ntile = 0;
        for (int t = pair; t < tiles && !*abort_flag; t += npairs, ++ntile) {
          if (ntile > 0 && !wait_bar_cluster(d_empty, (ntile - 1) & 1u, abort_flag, hdr)) break;
          tc_fence_after();
          bool ok = true;
          for (int kb = 0; kb < KB; ++kb, ++g) {
            const int s = g % kXStages, sa = g % kAStages;
            if (!wait_bar_cluster(&x_full[s], (g / kXStages) & 1u, abort_flag, hdr) ||
                !wait_bar_cluster(&a_full[sa], (g / kAStages) & 1u, abort_flag, hdr)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t xaddr = smem_u32(xs + s * kXStageBytes);
            const uint32_t x8addr = smem_u32(x8s + s * kX8StageBytes);
            const uint32_t a_hi = tmem + kACol + kAStageCols * sa, a_lo = a_hi + 32u;
            // hi pass: bf16 x bf16, 4 x K=16
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              mma_pair_f16(tmem + kAccCol, a_hi + 8u * kk, sw128_desc(xaddr + kk * 32), kIdesc,
                           (kb > 0 || kk > 0) ? 1u : 0u);
            // lo pass: e4m3 remainders x e5m2 activations, 2 x K=32 (an MXFP4
            // weight is exact in bf16: no remainder)
            if (!MX) {
#pragma unroll
              for (int kk = 0; kk < kBK / 32; ++kk)
                mma_pair_f8(tmem + kAccCol, a_lo + 8u * kk, sw64_desc(x8addr + kk * 32), kIdescF8,
                            1u);
            }
            mma_commit_pair(&x_free[s], 0x3);
            mma_commit_pair(&a_free[sa], 0x3);
          }
          if (!ok) break;
          mma_commit_pair(d_full, 0x3);
        }
        // every MMA this thread issued completes before TMEM is released
        mma_commit_pair(drain, 0x1);
        drain_wait(drain, 0);
      }
    } else if (warp == 3) {
      // -------------------------------------------- packed weights + absmax
      // Per 4 K-steps: this CTA's 128 weight rows x 128 packed bytes (one TMA
      // box, 128-byte swizzle) and their 4 x 128 absmax values ([block][row];
      // cp.async, 4 bytes each: absmax rows need not be 16-byte aligned).
      const int nquads = (KB + 3) / 4;
      uint32_t gq = 0;   // slot ring counter
      bool ok = true;
      for (int t = pair; t < tiles && ok && !*abort_flag; t += npairs) {
        const TileInfo ti = tile_info(t, G, tile_start, row_off, gsize, gexp, ncols_tile);
        const int64_t ebase = static_cast<int64_t>(ti.e) * N;
        // this lane's 4 rows (rr = lane + 32 i): scale element of the row's
        // first block, and whether the row exists
        int64_t rb[4];
        bool rv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          rb[i] = (ebase + weight_row(p, ti.n0, rank, lane + 32 * i, &rv[i])) * KB;
        for (int qd = 0; qd < nquads; ++qd, ++gq) {
          const int slot = static_cast<int>(gq % kWQuads);
          const uint32_t ph = (gq / kWQuads) & 1u;
          if (!warp_wait_cluster(&w_free[slot], ph ^ 1u, abort_flag, hdr)) { ok = false; break; }
          const uint32_t as = smem_u32(smem + kAbsOff + slot * kASlotBytes) + lane * 4;
          if (p.scale_kind == kScaleF32) {
            const float *fb = static_cast<const float *>(p.scales) + 4 * qd;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
              for (int blk = 0; blk < 4; ++blk) {
                const bool v = rv[i] && 4 * qd + blk < KB;
                cp_async4(as + blk * (kBM * 4) + i * 128, v ? fb + rb[i] + blk : p.scales,
                          v ? 4u : 0u);
              }
            }
          } else {   // the 4-byte word holding this (row, K-step)'s 2 bytes
            const char *cb = static_cast<const char *>(p.scales);
            const int64_t total = static_cast<int64_t>(E) * N * KB * 2;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
              for (int blk = 0; blk < 4; ++blk) {
                const bool v = rv[i] && 4 * qd + blk < KB;
                const int64_t wb = ((rb[i] + 4 * qd + blk) * 2) & ~int64_t{3};
                cp_async4(as + blk * (kBM * 4) + i * 128, v ? cb + wb : p.scales,
                          v ? (wb + 4 <= total ? 4u : 2u) : 0u);
              }
            }
          }
          cp_async_arrive_noinc(&w_full[slot]);
          if (lane == 0) {
            mbar_arrive_expect_tx(&w_full[slot], kWSlotBytes);
            char *wdst = smem + kWOff + slot * kWSlotBytes;
            if (p.epi == 1) {   // per TMEM lane quarter: 16 gate rows, then their 16 up rows
#pragma unroll
              for (int qq = 0; qq < 4; ++qq)
                tma_load_4d(wdst + qq * 4096, &w4map, qd * 128,
                            ti.n0 + 64 * static_cast<int>(rank) + 16 * qq, 0, ti.e, &w_full[slot]);
            } else {            // 128 consecutive rows
              bool unused;
              const int64_t row0 = ebase + weight_row(p, ti.n0, rank, 0, &unused);
              tma_load_2d(wdst, &wmap, qd * 128, static_cast<int>(row0), &w_full[slot]);
            }
          }
        }
      }
      cp_async_wait_all();
      if (lane == 0) {   // the last copies must land before the CTA exits
        for (uint32_t d = 0; d < kWQuads && d < gq; ++d) {
          const uint32_t gg = gq - 1 - d;
          drain_wait(&w_full[gg % kWQuads], (gg / kWQuads) & 1u);
        }
      }
    } else if (warp >= kDecodeWarp0) {
      // ---------------------------------------------------- decode + epilogue
      const int dw = warp - kDecodeWarp0;
      const int quarter = warp & 3;          // TMEM lane quarter
      const int half = dw >> 2;              // K half of the stage / token half of the tile
      const int rl = quarter * 32 + lane;                      // row within this CTA's half
      const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
      // shared address of this lane's table slot (bits 7..10 clear): the
      // entry of code c is at lut_lane | c * 128
      const uint32_t lut_lane = smem_u32(smem + kLutOff) + static_cast<uint32_t>(lane) * 4u;
      // absmax row of this thread's weight row in pair tile t (nullptr: no such row)
      // scale-array element index of this thread's weight row in pair tile t
      // (its first block; -1: no such row)
      auto row_scales = [&](int t) -> int64_t {
        if (t >= tiles) return -1;
        const TileInfo tn = tile_info(t, G, tile_start, row_off, gsize, gexp, ncols_tile);
        bool v;
        const int64_t nn = weight_row(p, tn.n0, rank, rl, &v);
        return v ? (static_cast<int64_t>(tn.e) * N + nn) * KB : -1;
      };
      // Row maximum of the block scales for the row scale: for the first
      // tile read here, for every later tile gathered one block per K-step of
      // the tile before.
      float mx = 0.0f;
      {
        const int64_t a0 = row_scales(pair);
        if (a0 >= 0) {
          float m[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
          int b = 0;
          for (; b + 8 <= KB; b += 8) {   // 8 independent loads in flight
#pragma unroll
            for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], scale_max_at(p, a0 + b + i));
          }
          for (; b < KB; ++b) m[0] = fmaxf(m[0], scale_max_at(p, a0 + b));
#pragma unroll
          for (int i = 0; i < 8; ++i) mx = fmaxf(mx, m[i]);
        }
      }
      uint32_t g = 0;    // decoded-weight stage counter
      uint32_t gq = 0;   // packed-weight slot counter
      uint32_t ntile = 0;
      for (int t = pair; t < tiles && !*abort_flag; t += npairs, ++ntile) {
        const TileInfo ti = tile_info(t, G, tile_start, row_off, gsize, gexp, ncols_tile);
        const int64_t ap_next = row_scales(t + npairs);
        float mx_next = 0.0f;
        uint32_t nxq[4];   // next tile's raw block scales, folded 4 K-steps after their load
#pragma unroll
        for (int j = 0; j < 4; ++j) nxq[j] = 0u;
        bool rok;
        const int64_t n = weight_row(p, ti.n0, rank, rl, &rok);
        // scale-array element index of this row's blocks (for the 2-byte
        // encodings: which half of each copied word holds them)
        const int64_t sbase = (static_cast<int64_t>(ti.e) * N + n) * KB;
        // Row scale 2^S, S = beta + 14 with 2^beta * max(absmax of the row) in
        // [1, 2): scaled weights stay below 2^15 and their bf16 remainders
        // below 64, inside the e4m3 range, whatever the row's magnitude.
        const int mexp = static_cast<int>((__float_as_uint(mx) >> 23) & 0xFFu);
        const int beta = mx > 0.0f ? (mexp == 0 ? 126 : 127 - mexp) : 0;
        int S = beta + kLoShift;
        S = S > 127 ? 127 : (S < -126 ? -126 : S);
        const float rscale = __uint_as_float(static_cast<uint32_t>(S + 127) << 23);
        const float rinv = __uint_as_float(static_cast<uint32_t>(127 - S) << 23);
        bool ok = true;
        const int nquads = (KB + 3) / 4;
        for (int qd = 0; qd < nquads && ok; ++qd, ++gq) {
          const int slot = static_cast<int>(gq % kWQuads);
          if (!warp_wait_cluster(&w_full[slot], (gq / kWQuads) & 1u, abort_flag, hdr)) {
            ok = false;
            break;
          }
          // this row's 128 packed bytes (swizzled 16-byte chunks) and 4 absmax values
          const char *wsm = smem + kWOff + slot * kWSlotBytes + rl * 128;
          const float *asm4 = reinterpret_cast<const float *>(smem + kAbsOff + slot * kASlotBytes) + rl;
#pragma unroll
          for (int sub = 0; sub < 4; ++sub) {
            const int kb = 4 * qd + sub;
            if (kb >= KB) break;
            const uint4 pk =
                *reinterpret_cast<const uint4 *>(wsm + (((2 * sub + half) ^ (rl & 7)) << 4));
            float am;
            if (p.scale_kind == kScaleF32) {
              am = asm4[sub * kBM];
            } else {
              const uint32_t wv = __float_as_uint(asm4[sub * kBM]);
              const uint32_t v16 = (wv >> (16 * static_cast<uint32_t>((sbase + kb) & 1))) & 0xFFFFu;
              if (MX) {   // e8m0 of this warp's 32-element half of the K-step
                const uint32_t e = half ? (v16 >> 8) : (v16 & 0xFFu);
                am = e == 255u ? __uint_as_float(0x7FC00000u)
                               : (e == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(e << 23));
              } else {
                am = __uint_as_float(v16 << 16);
              }
            }
            am *= rscale;
            // next tile's block scales, first used 4 K-steps after their load (no wait here)
            mx_next = fmaxf(mx_next, scale_mag(p, nxq[sub]));
            nxq[sub] = ap_next >= 0 ? scale_raw_at(p, ap_next + kb) : 0u;
            const int s = g % kAStages;
            const uint32_t ph = (g / kAStages) & 1u;
            // hi[i]: bf16 pair of k = 32 half + 2i, 2i+1; lo[i]: e4m3 of k = 32 half + 4i .. +3
            uint32_t hi[16], lo[8], lo_even = 0u;
            const uint32_t words[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
#pragma unroll
              for (int pb = 0; pb < 4; ++pb) {
                // codes of byte pb (NF4: high nibble = even k; MXFP4: low
                // nibble = even k), each moved straight to bits 7..10 of its
                // table address
                const uint32_t w = words[q];
                const uint32_t sh = pb == 0 ? (w << 3) : (w >> (8 * pb - 3));   // high nibble
                const uint32_t sl = pb == 0 ? (w << 7) : (w >> (8 * pb - 7));   // low nibble
                const uint32_t s0 = MX ? sl : sh, s1 = MX ? sh : sl;
                float v0, v1;
                asm("ld.shared.f32 %0, [%1];" : "=f"(v0) : "r"(lut_lane | (s0 & 0x780u)));
                asm("ld.shared.f32 %0, [%1];" : "=f"(v1) : "r"(lut_lane | (s1 & 0x780u)));
                const float w0 = __fmul_rn(v0, am), w1 = __fmul_rn(v1, am);
                const __nv_bfloat162 h = __floats2bfloat162_rn(w0, w1);
                const uint32_t hb = *reinterpret_cast<const uint32_t *>(&h);
                hi[q * 4 + pb] = hb;
                if (!MX) {
                  const float h0 = __uint_as_float(hb << 16), h1 = __uint_as_float(hb & 0xFFFF0000u);
                  // remainders (exact in fp32, below 64 in magnitude) to e4m3, RNE
                  const uint32_t l8 = __nv_cvt_float2_to_fp8x2(make_float2(w0 - h0, w1 - h1),
                                                               __NV_SATFINITE, __NV_E4M3);
                  if (pb & 1)
                    lo[q * 2 + (pb >> 1)] = __byte_perm(lo_even, l8, 0x5410u);
                  else
                    lo_even = l8;
                }
              }
            }
            if (!warp_wait_cluster(&a_free[s], ph ^ 1u, abort_flag, hdr)) { ok = false; break; }
            tc_fence_after();
            const uint32_t col = kACol + kAStageCols * s;
            tmem_st16(tmem + lane_base + col + 16u * half, hi);
            if (!MX) tmem_st8(tmem + lane_base + col + 32u + 8u * half, lo);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cta(&a_full[s], 0);
            ++g;
          }
          // done with the slot (every lane has read its bytes)
          __syncwarp();
          if (lane == 0) mbar_arrive(&w_free[slot]);
        }
        if (!ok) break;
#pragma unroll
        for (int j = 0; j < 4; ++j) mx_next = fmaxf(mx_next, scale_mag(p, nxq[j]));
        mx = mx_next;
        // ---- epilogue: accumulator -> bf16 y (this CTA's 128 weight rows).
        // Chunks of 32 tokens: scaled and rounded into a shared-memory box
        // [32 tokens][32 rows] and written by one bulk tensor store; a chunk
        // that runs past the tile's tokens (the group's last tile) is stored
        // element by element instead, so that no other group's rows are
        // touched. The accumulator is released after its last chunk is read.
        if (!warp_wait_cluster(d_full, ntile & 1u, abort_flag, hdr)) break;
        tc_fence_after();
        const int nbox = ti.n0 + kBM * static_cast<int>(rank) + 32 * quarter;   // first row of the box
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
          const int c0 = half * (kBN / 2) + 32 * k;
          uint32_t acc[32];
          tmem_ld32(tmem + lane_base + kAccCol + c0, acc);
          tmem_wait_ld();
          if (k == 3) {   // the accumulator is read out: the next tile's MMAs may start
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cta(d_empty, 0);
          }
          // lane c holds 2^-s of activation row c0 + c of the tile
          const float tinv = c0 + lane < ti.rows ? __ldg(tok_inv + ti.row0 + c0 + lane) : 0.0f;
          if (p.epi != 0) {
            // SwiGLU: the gate lane of each row pair takes its up value from
            // the partner lane and writes one output column of 32 tokens
            const bool halves = p.epi == 1;
            const int partner = halves ? (lane ^ 16) : (lane ^ 1);
            const bool gate_lane = halves ? lane < 16 : (lane & 1) == 0;
            const int jl = halves ? (lane & 15) : (lane >> 1);
            const int64_t jbox = static_cast<int64_t>(ti.n0) + 64 * static_cast<int64_t>(rank) +
                                 16 * quarter;   // first output column of this warp
            const bool use_box = bulk_out && c0 + 32 <= ti.rows;
            if (use_box && jbox >= ncols) continue;   // none of this warp's columns exists
            uint16_t *box = reinterpret_cast<uint16_t *>(smem + kOutOff) + dw * 1024;
            if (use_box) {
              if (lane == 0) bulk_wait_read_0();   // the previous chunk's store has read the box
              __syncwarp();
            }
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float tc = __shfl_sync(0xffffffffu, tinv, c);
              const float v = __uint_as_float(acc[c]) * rinv * tc;
              const float u = __shfl_sync(0xffffffffu, v, partner);
              if (gate_lane) {
                float o;
                if (halves) {
                  o = v / (1.0f + expf(-v)) * u;
                } else {
                  const float gt = fminf(v, p.limit);
                  const float uc = fminf(fmaxf(u, -p.limit), p.limit);
                  o = gt / (1.0f + expf(-p.alpha * gt)) * (uc + 1.0f);
                }
                const __nv_bfloat16 b = __float2bfloat16_rn(o);
                const uint16_t bits = *reinterpret_cast<const uint16_t *>(&b);
                if (use_box) {
                  box[c * 16 + jl] = bits;
                } else if (rok && c0 + c < ti.rows) {
                  y[(ti.row0 + c0 + c) * ncols + jbox + jl] = bits;
                }
              }
            }
            if (use_box) {
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&ymap, box, static_cast<int>(jbox), static_cast<int>(ti.row0) + c0);
                bulk_commit();
              }
            }
            continue;
          }
          if (bulk_out && c0 + 32 <= ti.rows) {
            if (nbox >= N) continue;   // none of this warp's rows exists (nor does its box)
            uint16_t *box = reinterpret_cast<uint16_t *>(smem + kOutOff) + dw * 1024;
            // the previous chunk's store has read the box
            if (lane == 0) bulk_wait_read_0();
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float tc = __shfl_sync(0xffffffffu, tinv, c);
              // 2^-S of the weight row, then 2^-s of the activation row
              const __nv_bfloat16 b = __float2bfloat16_rn(__uint_as_float(acc[c]) * rinv * tc);
              box[c * 32 + lane] = *reinterpret_cast<const uint16_t *>(&b);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&ymap, box, nbox, static_cast<int>(ti.row0) + c0);
              bulk_commit();
            }
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float tc = __shfl_sync(0xffffffffu, tinv, c);
              if (rok && c0 + c < ti.rows) {
                const float v = __uint_as_float(acc[c]) * rinv;
                const __nv_bfloat16 b = __float2bfloat16_rn(v * tc);
                y[(ti.row0 + c0 + c) * N + n] = *reinterpret_cast<const uint16_t *>(&b);
              }
            }
          }
        }
      }
      // every bulk store of this warp has finished before the CTA exits
      if (lane == 0) bulk_wait_all();
      __syncwarp();
    }
  } else if (blockIdx.x == 0 && tid == 0) {
    report_error(hdr, static_cast<uint32_t>(errbits), 0);
  }

  // Neither CTA leaves (or frees TMEM) while the pair's MMAs, copies or
  // remote arrivals may still touch it.
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 2) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// The activation operands, one block per row m of x (rows strided over the
// grid): with s the power of two that puts the row's largest finite
// magnitude in [2^14, 2^15) (0 for a row of zeros or with an infinity;
// clamped to [-126, 127]),
//   xs[m] = bf16(x[m] * 2^s)   (exact: only the exponent changes)
//   x8[m] = e5m2(x[m] * 2^s)   (RNE, saturating)
//   tok_inv[m] = 2^-s
// so the remainder pass keeps e5m2's precision whatever the row's magnitude,
// and the epilogue divides the row's scale back out. A thread keeps its
// kPrepChunks 8-element chunks of the row in registers between the maximum
// and the conversion (K <= 16384 with 256 threads); longer rows are read twice.
constexpr int kPrepThreads = 256;
constexpr int kPrepChunks = 8;

__device__ __forceinline__ float bf16_abs_max2(uint32_t w) {
  return fmaxf(fabsf(__uint_as_float(w << 16)), fabsf(__uint_as_float(w & 0xFFFF0000u)));
}

__device__ __forceinline__ void scale_chunk(const uint4 v, float f, uint4 *dst, uint2 *dst8) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o16[4], o8[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float a = __uint_as_float(w[j] << 16) * f, b = __uint_as_float(w[j] & 0xFFFF0000u) * f;
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    o16[j] = *reinterpret_cast<const uint32_t *>(&h);
    o8[j] = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E5M2);
  }
  *dst = make_uint4(o16[0], o16[1], o16[2], o16[3]);
  *dst8 = make_uint2(o8[0] | (o8[1] << 16), o8[2] | (o8[3] << 16));
}

// With a gather (hidden != nullptr) row m of x is hidden[sorted_idx[m] /
// top_k]; a slot outside [0, n_slots) reads as a row of zeros (the GEMM
// kernel refuses the call on such a slot and writes nothing).
__global__ void __launch_bounds__(kPrepThreads)
    prefill_prep_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ hidden,
                        const int32_t *__restrict__ sorted_idx, int32_t top_k, int64_t n_slots,
                        uint16_t *__restrict__ xs, uint8_t *__restrict__ x8,
                        float *__restrict__ tok_inv, int64_t M, int32_t K) {
  __shared__ float s_max[kPrepThreads / 32];
  pdl_trigger();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c8 = K / 8;   // 8-element chunks per row
  const bool in_regs = c8 <= kPrepThreads * kPrepChunks;
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const uint16_t *row = x + m * K;
    bool zero_row = false;
    if (hidden != nullptr) {
      const int32_t sl = __ldg(sorted_idx + m);
      zero_row = sl < 0 || sl >= n_slots;
      row = hidden + static_cast<int64_t>(zero_row ? 0 : sl / top_k) * K;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(row);
    uint4 v[kPrepChunks];
    float mx = 0.0f;
    const int c8r = zero_row ? 0 : c8;   // chunks read from memory (a zero row reads none)
    if (in_regs) {
#pragma unroll
      for (int u = 0; u < kPrepChunks; ++u) {
        const int i = tid + u * kPrepThreads;
        v[u] = i < c8r ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kPrepChunks; ++u)
        mx = fmaxf(mx, fmaxf(fmaxf(bf16_abs_max2(v[u].x), bf16_abs_max2(v[u].y)),
                             fmaxf(bf16_abs_max2(v[u].z), bf16_abs_max2(v[u].w))));
    } else {
      for (int i = tid; i < c8r; i += kPrepThreads) {
        const uint4 a = __ldg(src + i);
        mx = fmaxf(mx, fmaxf(fmaxf(bf16_abs_max2(a.x), bf16_abs_max2(a.y)),
                             fmaxf(bf16_abs_max2(a.z), bf16_abs_max2(a.w))));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_max[warp] = mx;
    __syncthreads();
    mx = s_max[0];
#pragma unroll
    for (int w = 1; w < kPrepThreads / 32; ++w) mx = fmaxf(mx, s_max[w]);
    __syncthreads();   // s_max is rewritten for the next row
    const uint32_t eb = (__float_as_uint(mx) >> 23) & 0xFFu;
    int sc = 0;
    if (mx > 0.0f && eb != 0xFFu) sc = eb == 0 ? 127 : 14 - (static_cast<int>(eb) - 127);
    sc = sc > 127 ? 127 : (sc < -126 ? -126 : sc);
    const float f = __uint_as_float(static_cast<uint32_t>(sc + 127) << 23);
    if (tid == 0)
      tok_inv[m] = sc == 127 ? __uint_as_float(0x00400000u)   // 2^-127 (subnormal)
                             : __uint_as_float(static_cast<uint32_t>(127 - sc) << 23);
    uint4 *dst = reinterpret_cast<uint4 *>(xs + m * K);
    uint2 *dst8 = reinterpret_cast<uint2 *>(x8 + m * K);
    if (in_regs) {
#pragma unroll
      for (int u = 0; u < kPrepChunks; ++u) {
        const int i = tid + u * kPrepThreads;
        if (i < c8) scale_chunk(v[u], f, dst + i, dst8 + i);
      }
    } else {
      for (int i = tid; i < c8; i += kPrepThreads)
        scale_chunk(i < c8r ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u), f, dst + i, dst8 + i);
    }
  }
}

size_t x8_bytes(int64_t M, int32_t K) {
  return ((static_cast<size_t>(M) * static_cast<size_t>(K) + 255) / 256) * 256;
}

size_t tok_bytes(int64_t M) { return ((static_cast<size_t>(M) * 4 + 255) / 256) * 256; }

}  // namespace

// Header, the e5m2 operand [M][K], the bf16 operand [M][K], the per-row
// factors 2^-s [M].
size_t prefill_workspace_bytes(int64_t M, int32_t N, int32_t K, int32_t G, int32_t swiglu) {
  (void)N; (void)G; (void)swiglu;
  return kWsHeaderBytes + 3 * x8_bytes(M, K) + tok_bytes(M);
}

bool prefill_supports(const GemmArgs &a) {
  const bool nf4 = a.fmt == GNF4_FMT_NF4 &&
                   (a.scale_dtype == GNF4_SCALE_F32 || a.scale_dtype == GNF4_SCALE_BF16);
  const bool mx = a.fmt == GNF4_FMT_MXFP4 && a.scale_dtype == GNF4_SCALE_E8M0;
  return nf4 || mx;
}

cudaError_t launch_prefill_gemm(const GemmArgs &a, cudaStream_t stream) {
  if (!prefill_supports(a)) return cudaErrorNotSupported;
  if (a.ws_bytes < prefill_workspace_bytes(a.M, a.N, a.K, a.G, a.swiglu)) return cudaErrorInvalidValue;
  const bool mx = a.fmt == GNF4_FMT_MXFP4;
  CUtensorMap xmap, x8map, wmap, w4map, ymap;
  std::memset(&w4map, 0, sizeof(w4map));
  // the row-scaled operands live in the workspace after the header
  uint8_t *x8 = static_cast<uint8_t *>(a.workspace) + kWsHeaderBytes;
  uint16_t *xs = reinterpret_cast<uint16_t *>(x8 + x8_bytes(a.M, a.K));
  float *tok_inv = reinterpret_cast<float *>(x8 + 3 * x8_bytes(a.M, a.K));
  // bf16 operand as [M rows][K bf16], boxes of 128 rows x 64 elements
  if (!encode_tensor_map_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, xs,
                            static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M),
                            static_cast<uint64_t>(a.K) * 2, kBK, kBNh, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  // e5m2 operand as [M rows][K bytes], boxes of 128 rows x 64 bytes with the
  // 64-byte swizzle
  if (!encode_tensor_map_2d(&x8map, CU_TENSOR_MAP_DATA_TYPE_UINT8, x8, static_cast<uint64_t>(a.K),
                            static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.K), kBK, kBNh,
                            CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  // output as [M rows][ncols bf16], boxes of 32 rows x 32 elements (16 with
  // SwiGLU), for the epilogue's bulk stores; they need rows of a multiple of
  // 16 bytes (otherwise every output is stored element by element and the map
  // is a placeholder the kernel does not touch)
  const int64_t ncols = a.swiglu ? a.N / 2 : a.N;
  const int32_t bulk_out = ncols % 8 == 0 ? 1 : 0;
  if (bulk_out) {
    if (!encode_tensor_map_2d(&ymap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.y,
                              static_cast<uint64_t>(ncols), static_cast<uint64_t>(a.M),
                              static_cast<uint64_t>(ncols) * 2, a.swiglu ? 16 : 32, 32,
                              CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  // packed weights as [E*N rows][K/2 bytes], boxes of 128 rows x 128 bytes
  // (4 K-steps) with the 128-byte swizzle
  if (!encode_tensor_map_2d(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w,
                            static_cast<uint64_t>(a.K) / 2,
                            static_cast<uint64_t>(a.E) * static_cast<uint64_t>(a.N),
                            static_cast<uint64_t>(a.K) / 2, 128, kBM, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (a.epi == GNF4_EPI_SWIGLU) {
    // the same bytes as [E][2 halves][N/2 rows][K/2]: a box holds 16 rows of
    // the gate half, then the 16 matching rows of the up half
    const uint64_t kh = static_cast<uint64_t>(a.K) / 2, nh = static_cast<uint64_t>(a.N) / 2;
    const uint64_t dims[4] = {kh, nh, 2, static_cast<uint64_t>(a.E)};
    const uint64_t pitches[3] = {kh, nh * kh, 2 * nh * kh};
    const uint32_t box[4] = {128, 16, 2, 1};
    if (!encode_tensor_map(&w4map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, a.w, dims, pitches, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  if (!bulk_out) ymap = wmap;
  if (a.epi != GNF4_EPI_SWIGLU) w4map = wmap;

  const int sk = mx ? kScaleE8m0 : (a.scale_dtype == GNF4_SCALE_BF16 ? kScaleBf16 : kScaleF32);
  using KernelFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
                            PrefillParams);
  static const KernelFn kernels[3][2] = {
      {prefill_gemm_kernel<kScaleF32, false>, prefill_gemm_kernel<kScaleF32, true>},
      {prefill_gemm_kernel<kScaleBf16, false>, prefill_gemm_kernel<kScaleBf16, true>},
      {prefill_gemm_kernel<kScaleE8m0, false>, prefill_gemm_kernel<kScaleE8m0, true>}};
  const int ks = a.swiglu ? 1 : 0;
  const KernelFn kernel = kernels[sk][ks];
  static bool configured[64][3][2] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev][sk][ks]) {
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kSmemBytes);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64) configured[dev][sk][ks] = true;
  }
  // one block per activation row (rows strided over the grid)
  const int64_t want = a.M;   // 4 blocks of 256 threads fit an SM at 64 registers
  const int xblocks = static_cast<int>(want < 4 * device_sm_count() ? want : 4 * device_sm_count());
  cudaError_t err = launch_pdl(prefill_prep_kernel, dim3(xblocks), dim3(kPrepThreads), 0, stream,
                               static_cast<const uint16_t *>(a.x), a.hidden, a.sorted_idx,
                               a.top_k, a.n_tokens * a.top_k, xs, x8, tok_inv, a.M, a.K);
  if (err != cudaSuccess) return err;

  PrefillParams pp;
  pp.w = a.w;
  pp.scales = a.scales;
  pp.tok_inv = tok_inv;
  pp.sizes = a.sizes;
  pp.expert_ids = a.expert_ids;
  pp.sorted_idx = a.hidden != nullptr ? a.sorted_idx : nullptr;
  pp.n_slots = a.n_tokens * a.top_k;
  pp.G = a.G; pp.M = a.M; pp.N = a.N; pp.K = a.K; pp.E = a.E;
  pp.scale_kind = mx ? kScaleE8m0 : (a.scale_dtype == GNF4_SCALE_BF16 ? kScaleBf16 : kScaleF32);
  pp.epi = a.epi;
  pp.alpha = a.alpha;
  pp.limit = a.limit;
  pp.y = a.y;
  pp.bulk_out = bulk_out;
  pp.hdr = static_cast<WsHeader *>(a.workspace);

  // one CTA per SM, in pairs (clusters of 2) for the 2-SM MMA
  const int grid = device_sm_count() & ~1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, xmap, x8map, wmap, w4map, ymap, pp);
}

}  // namespace gnf4
