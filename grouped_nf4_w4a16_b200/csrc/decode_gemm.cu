// decode_gemm.cu -- decode-regime grouped NF4 GEMM (few activation rows per expert).
//
// Passage: "grouped-nf4-gemm -- single-launch W4A16 GEMM over fused NF4 MoE
// expert stacks", opening section (one launch for all active experts, LUT
// decode of the packed codes, blockwise fp32 absmax, fp32 accumulation, bf16
// epilogue, no bf16 weight copy). At a handful of activation rows per expert
// this GEMM reads every touched weight byte exactly once and is bound by HBM
// bandwidth, so the kernel is built around keeping HBM busy: a TMA producer
// keeps up to six 22 KB stages of packed weights in flight per SM.
//
// Work decomposition (no split-K, no cross-CTA reduction)
//   batch  = up to 8 consecutive activation rows of one group (the MMA's N).
//   unit   = 16 weight rows of the group's expert for one batch, over the
//            whole of K: two row groups of 8 (with SwiGLU: 8 gate rows j..j+7
//            and the matching 8 up rows N/2+j..). A unit's output is final
//            when its K loop ends.
//   The units of all groups are laid end to end (group by group, batch by
//   batch, row by row) and every CTA (one per SM) takes an equal contiguous
//   range, so every SM streams the same number of weight bytes. The unit
//   list is derived on the device from (sizes, expert_ids): the host never
//   learns which experts are active (no sync, graph-capturable).
//   tile   = up to 8 consecutive units of one batch.
//
// Numerics: each code value is an fp16 part hi plus the fp16 of the
// remainder times 2^13 (both round to nearest even), together within 1e-7
// relative of the fp32 value. Activations
// are staged as bf16 and rewritten in place as fp16 times a power of two
// per (row, 64-element block), which the block sum divides out in fp32.
//
// Inside a CTA (warp 16 = tensor copies, warp 17 = absmax copies, warp 18 =
// activation conversion, warps 0-15 = consumers)
//   Stage = 256 K-elements of a tile: the tile's weight rows as a few TMA
//   boxes of 128 packed bytes per row (128-byte swizzle), the batch's
//   activations as one box of 4 blocks x 8 rows x 64 bf16, and the 8 x 4
//   absmax values of each row group (cp.async, 4 bytes each: absmax rows
//   need not be 16-byte aligned).
//   Consumer warp w takes 64-element block w / 4 of every stage for the two
//   units 2 (w % 4), 2 (w % 4) + 1, so one set of activation fragments
//   serves both. Per unit, two m16n8k16 fp16 MMAs per 16 K-elements (hi,
//   remainder) cover all 16 weight rows: A rows g and g + 8 are the unit's
//   row groups (with SwiGLU a gate row and its up row, which the epilogue
//   combines in registers). For each packed byte (two codes) one byte
//   permute forms the address of a 256-byte table row replicated per lane
//   (no bank conflicts) holding the hi pair and, 128 bytes on, the
//   remainder pair. The block's fp32 result is scaled by absmax(row, block)
//   and the activations' 2^-S and accumulated in fp32; when a tile's K loop
//   ends, the pair's four block warps sum their partial results through
//   shared memory (fixed order) and the block-0 warp writes y.
// Every wait is bounded (2 s); on expiry the kernel records
// GNF4_DEVERR_TIMEOUT, lets the producer's copies land and returns.
#include <climits>

#include <cuda_fp16.h>

#include "launch.h"
#include "sm100.cuh"

namespace gnf4 {
namespace {

constexpr int kConsumerWarps = 16;
constexpr int kTmaWarp = kConsumerWarps;          // issues the tensor copies
constexpr int kScaleWarp = kConsumerWarps + 1;    // copies the absmax values
constexpr int kXWarp = kConsumerWarps + 2;        // converts the staged activations to fp16
constexpr int kThreads = (kConsumerWarps + 3) * 32;
constexpr int kTileUnits = 8;                 // units per tile (2 row groups each)
constexpr int kStages = 6;
constexpr int kBatch = 8;                     // activation rows per batch (MMA N)
constexpr int kBoxBytes = 1024;               // 8 rows x 128 bytes
constexpr int kStageBlocks = 4;               // absmax blocks per stage (256 K-elements)
constexpr int kWStage = kTileUnits * 2 * kBoxBytes;              // 16 KB
constexpr int kXStage = kStageBlocks * kBoxBytes;                // 4 KB
constexpr int kXsStage = kStageBlocks * kBatch * 4;              // 128 B: 2^-S per (block, row)
constexpr int kAStage = kTileUnits * 2 * 8 * kStageBlocks * 4;   // 2 KB
constexpr int kMaxG = GNF4_MAX_EXPERTS;
constexpr float kLoInv = 1.0f / 8192.0f;      // remainders are carried times 2^13

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
// partial sums written), xempty (the block-0 warp done reading them)
constexpr int kNumBars = 3 * kStages + kTileUnits;
constexpr int kMiscOff = kBarOff + kNumBars * 8;              // int [8]
// table: 256-byte row per packed byte b: lane l's hi pair at l * 4, its
// remainder pair at 128 + l * 4
constexpr int kLutOff = 131072;
constexpr int kLutBytes = 256 * 256;
constexpr int kAOff = kLutOff + kLutBytes;
constexpr int kXchgOff = kAOff + kStages * kAStage;           // float4 [4 pairs][3][2 units][32]
constexpr int kXchgBytes = (kTileUnits / 2) * 3 * 2 * 32 * 16;
constexpr int kUnitStartOff = kXchgOff + kXchgBytes;          // int64 [kMaxG + 1]
constexpr int kGExpOff = kUnitStartOff + (kMaxG + 1) * 8;     // uint16 [kMaxG]
constexpr int kSmemEnd = kGExpOff + kMaxG * 2;
// dynamic bytes requested: the window reaches kSmemEnd from any start >= kMinDyn
constexpr int kSmemBytes = kSmemEnd - kMinDyn;
static_assert(kMiscOff + 8 * 4 <= kLutOff, "low region overlaps the table");
static_assert(kBarOff % 8 == 0 && kXOff % 1024 == 0 && kLutOff % 65536 == 0, "alignment");
static_assert(kSmemBytes + kDynBase - kMinDyn <= 227 * 1024, "fits one CTA per SM");

// ------------------------------------------------------------------ PTX

// Not volatile: the compiler may interleave independent accumulation chains.
__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A.B with a zero accumulator in.
__device__ __forceinline__ void mma_f16_z(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// prmt.b32 in its default mode: result byte i = byte (sel nibble i & 7) of
// {b, a} (the selectors used here never set bit 3 of a nibble).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// hi and lo fp16 pairs of the 4 packed bytes of `word` (pair p: byte p),
// from this lane's slots of the table: lutlane = shared address of the table
// (a multiple of 65536) + lane * 4, so one byte permute forms the whole
// address table + byte * 256 + lane * 4; the lo pair sits 128 bytes on.
__device__ __forceinline__ void decode_word(uint32_t lutlane, uint32_t word, uint32_t (&hi)[4],
                                            uint32_t (&lo)[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t a = prmt(word, lutlane, 0x7604u | (p << 4));
    asm("ld.shared.b32 %0, [%2];\n\tld.shared.b32 %1, [%2+128];"
        : "=r"(hi[p]), "=r"(lo[p])
        : "r"(a));
  }
}

// Bounded wait by every lane of the warp (no divergent branch); the lanes
// agree on the answer by vote.
__device__ __forceinline__ bool warp_wait_all(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag, WsHeader *hdr) {
  return __all_sync(0xffffffffu, wait_bar(bar, parity, abort_flag, hdr));
}

// One arrival on `bar` for the whole (converged) warp, by an elected lane.
__device__ __forceinline__ void mbar_arrive_elect(uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
      "@p mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  const __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<const uint16_t *>(&b);
}

// hi[c]: fp16 bits of the code value (round to nearest even).
__device__ __forceinline__ uint32_t code_hi(int c) {
  const __half h = __float2half_rn(nf4_value(c));
  return static_cast<uint32_t>(*reinterpret_cast<const uint16_t *>(&h));
}

// lo[c]: fp16 bits of (NF4[c] - hi[c]) * 2^13 (round to nearest even). The
// remainder is exact in fp32 and at most 2^-12 in magnitude, so the scaled
// value stays below 2; hi + lo * 2^-13 is within 1e-7 relative of NF4[c].
__device__ __forceinline__ uint32_t code_lo(int c) {
  const __half h = __float2half_rn(nf4_value(c));
  const __half l = __float2half_rn((nf4_value(c) - __half2float(h)) * 8192.0f);
  return static_cast<uint32_t>(*reinterpret_cast<const uint16_t *>(&l));
}

struct Problem {
  int32_t N, K, E, G, swiglu;
  int32_t KB;       // 64-element blocks per row
  int32_t KC;       // stages per unit
  int64_t upb;      // units per batch
};

struct Tile {
  int64_t row0;     // first activation row of the batch
  int64_t j0;       // unit index within the batch of the tile's first unit
  int32_t nunits;   // 1..kTileUnits
  int32_t mrows;    // activation rows in the batch (1..8)
  int32_t e;        // expert
};

// The tile that starts at unit u (never past u_hi or the end of u's batch).
__device__ __forceinline__ Tile make_tile(int64_t u, int64_t u_hi, const Problem &p,
                                          const int64_t *unit_start, const int *row_off,
                                          const uint16_t *gexp) {
  int lo = 0, hi = p.G;   // invariant: unit_start[lo] <= u < unit_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (unit_start[mid] <= u) lo = mid; else hi = mid;
  }
  const int64_t local = u - unit_start[lo];
  const int64_t batch = local < (int64_t{1} << 31)
                            ? static_cast<int64_t>(static_cast<uint32_t>(local) /
                                                   static_cast<uint32_t>(p.upb))
                            : local / p.upb;
  const int64_t run_end = unit_start[lo] + (batch + 1) * p.upb;
  int64_t end = u + kTileUnits;
  if (end > u_hi) end = u_hi;
  if (end > run_end) end = run_end;
  Tile t;
  t.row0 = static_cast<int64_t>(row_off[lo]) + batch * kBatch;
  t.j0 = local - batch * p.upb;
  t.nunits = static_cast<int32_t>(end - u);
  t.mrows = min(kBatch, row_off[lo + 1] - row_off[lo] - static_cast<int32_t>(batch) * kBatch);
  t.e = gexp[lo];
  return t;
}

// Packed-weight tensor maps with boxes of 8, 16, 32, 64 and 128 rows x 128
// bytes: a tile's contiguous rows are fetched with a few large copies.
constexpr int kNumWMaps = 5;
struct WeightMaps {
  CUtensorMap m[kNumWMaps];   // m[i]: boxes of (8 << i) rows
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

__global__ void __launch_bounds__(kThreads, 1)
    decode_gemm_kernel(const __grid_constant__ WeightMaps wmaps,
                       const __grid_constant__ CUtensorMap xmap, const float *__restrict__ absmax,
                       const int32_t *__restrict__ sizes, const int32_t *__restrict__ expert_ids,
                       int32_t G, int64_t M, int32_t N, int32_t K, int32_t E, int32_t swiglu,
                       uint16_t *__restrict__ y, WsHeader *hdr) {
  extern __shared__ __align__(1024) char smem_raw[];
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
  int64_t *unit_start = reinterpret_cast<int64_t *>(smem + kUnitStartOff);
  int *row_off = reinterpret_cast<int *>(smem + kRowOffOff);
  uint16_t *gexp = reinterpret_cast<uint16_t *>(smem + kGExpOff);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kBarOff);
  uint64_t *empty = full + kStages;
  uint64_t *xready = empty + kStages;
  uint64_t *xfull = xready + kStages;          // [kTileUnits / 2]
  uint64_t *xempty = xfull + kTileUnits / 2;   // [kTileUnits / 2]
  int *misc = reinterpret_cast<int *>(smem + kMiscOff);   // [0] error bits, [1] abort
  volatile int *abort_flag = &misc[1];
  __shared__ int64_t s_tot;   // total units (written by warp 0 with the group table)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();

  Problem p;
  p.N = N; p.K = K; p.E = E; p.G = G; p.swiglu = swiglu;
  p.KB = K / 64;
  p.KC = (p.KB + kStageBlocks - 1) / kStageBlocks;
  p.upb = swiglu ? (N / 2 + 7) / 8 : (N + 15) / 16;

  if (tid == 0) {
    misc[0] = 0;
    misc[1] = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 32 + 1);            // 32 cp.async arrivals + the byte-count arrival
      mbar_init(&empty[s], kConsumerWarps);
      mbar_init(&xready[s], 1);
    }
    for (int i = 0; i < kTileUnits / 2; ++i) {
      mbar_init(&xfull[i], 3);
      mbar_init(&xempty[i], 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int i = 0; i < kNumWMaps; ++i) prefetch_tensormap(&wmaps.m[i]);
    prefetch_tensormap(&xmap);
  }

  // ---- decode table: row b, lane slot l: the fp16 pair (hi[b >> 4],
  //      hi[b & 15]) at l * 4 and the pair of remainders at 128 + l * 4 (low
  //      half = even k = high nibble)
  if (tid < 256) {
    const uint32_t hp = code_hi(tid >> 4) | (code_hi(tid & 15) << 16);
    const uint32_t lp = code_lo(tid >> 4) | (code_lo(tid & 15) << 16);
    uint4 *dst = reinterpret_cast<uint4 *>(smem + kLutOff + tid * 256);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      dst[i] = make_uint4(hp, hp, hp, hp);
      dst[8 + i] = make_uint4(lp, lp, lp, lp);
    }
  }

  pdl_wait();   // inputs may come from the previous kernel on the stream

  // ---- group table from (sizes, expert_ids), validated on the device: built
  //      by warp 0 alone (its lanes' loads in flight together, one warp scan),
  //      then one block barrier publishes it with the barrier set-up.
  if (warp == 0) {
    const int per = (G + 31) / 32;
    const int g0 = min(G, lane * per), g1 = min(G, g0 + per);
    int64_t my_rows = 0, my_units = 0;
    int bad = 0;
    for (int g = g0; g < g1; ++g) {
      const int sz = sizes[g];
      const int e = expert_ids[g];
      if (sz < 0) bad |= GNF4_DEVERR_SIZES;
      if (sz > 0 && (e < 0 || e >= E)) bad |= GNF4_DEVERR_EXPERT;
      gexp[g] = static_cast<uint16_t>(e);
      row_off[g] = sz;   // kept here until the offsets are known
      my_rows += max(sz, 0);
      my_units += sz > 0 ? ((sz + kBatch - 1) / kBatch) * p.upb : 0;
    }
    int64_t vr = my_rows, vu = my_units;   // inclusive scan over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t a = __shfl_up_sync(0xffffffffu, vr, o);
      const int64_t b = __shfl_up_sync(0xffffffffu, vu, o);
      if (lane >= o) { vr += a; vu += b; }
    }
    const int64_t tot_r = __shfl_sync(0xffffffffu, vr, 31);
    const int64_t tot_u = __shfl_sync(0xffffffffu, vu, 31);
    int64_t r = vr - my_rows, c = vu - my_units;
    for (int g = g0; g < g1; ++g) {
      const int sz = max(row_off[g], 0);
      row_off[g] = static_cast<int>(r);
      unit_start[g] = c;
      r += sz;
      c += sz > 0 ? ((sz + kBatch - 1) / kBatch) * p.upb : 0;
    }
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (lane == 0) {
      unit_start[G] = tot_u;
      row_off[G] = static_cast<int>(tot_r);
      if (tot_r != M) bad |= GNF4_DEVERR_SIZES;
      s_tot = tot_u;
      misc[0] = bad;
    }
  }
  __syncthreads();   // group table, barrier set-up and misc visible
  const int64_t tot_u = s_tot;
  const int errbits = misc[0];
  if (errbits) {
    if (blockIdx.x == 0 && tid == 0) report_error(hdr, static_cast<uint32_t>(errbits), 0);
    return;
  }
  // Whole tiles, not units, are split across CTAs: a tile costs KC stages
  // whatever its unit count, so a unit range cutting through a batch's tiles
  // would cost its CTA an extra tile (twice the stages when every CTA holds
  // about one tile). Each batch has upb units in tpb = ceil(upb / 8) tiles;
  // this CTA takes tiles [T b / P, T (b + 1) / P) of the T = B tpb, B =
  // tot_u / upb batches (32-bit arithmetic when T fits: q P + r gives
  // q b + r b / P).
  const int64_t tpb = (p.upb + kTileUnits - 1) / kTileUnits;
  const int64_t T = (tot_u / p.upb) * tpb;
  const int64_t P = gridDim.x;
  int64_t u_lo, u_hi;
  if (T < (int64_t{1} << 31) && p.upb < (int64_t{1} << 31)) {
    const uint32_t tt = static_cast<uint32_t>(T), Pu = gridDim.x, bu = blockIdx.x;
    const uint32_t q = tt / Pu, rr = tt - q * Pu;
    const uint32_t t_lo = q * bu + rr * bu / Pu, t_hi = q * (bu + 1) + rr * (bu + 1) / Pu;
    const uint32_t tp = static_cast<uint32_t>(tpb);
    u_lo = static_cast<int64_t>(t_lo / tp) * p.upb + static_cast<int64_t>(t_lo % tp) * kTileUnits;
    u_hi = static_cast<int64_t>(t_hi / tp) * p.upb + static_cast<int64_t>(t_hi % tp) * kTileUnits;
  } else {
    const int64_t t_lo = T * blockIdx.x / P, t_hi = T * (blockIdx.x + 1) / P;
    u_lo = (t_lo / tpb) * p.upb + (t_lo % tpb) * kTileUnits;
    u_hi = (t_hi / tpb) * p.upb + (t_hi % tpb) * kTileUnits;
  }
  if (u_lo >= u_hi) return;

  if (warp == kXWarp) {
    // ------------------------------------------------ activation conversion
    // Per stage, lane (block b = lane / 8, row r = lane % 8) rewrites its 64
    // staged bf16 activations in place as fp16 x * 2^S, S putting the
    // largest magnitude of those 64 in [2^14, 2^15) (0 for all zeros, Inf or
    // NaN): exact for every value above 2^-28 of that maximum. 2^-S goes to
    // the stage's scale table for the consumers' block sums.
    const int b = lane >> 3, r = lane & 7;
    uint32_t it = 0;
    for (int64_t u = u_lo; u < u_hi;) {
      const Tile t = make_tile(u, u_hi, p, unit_start, row_off, gexp);
      for (int kc = 0; kc < p.KC; ++kc, ++it) {
        const int s = static_cast<int>(it % kStages);
        const uint32_t ph = (it / kStages) & 1u;
        if (!warp_wait_bar(&full[s], ph, abort_flag, hdr)) return;
        // rows past the batch feed only outputs that are never stored: skipped
        if (r < t.mrows) {
          char *row = smem + kXOff + s * kXStage + b * kBoxBytes + r * 128;
          uint4 v[8];
          // bf16 magnitudes compare as integers, two per word; four
          // independent chains keep the reduction short
          uint32_t m4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            v[c] = *reinterpret_cast<const uint4 *>(row + ((c ^ r) << 4));
            m4[0] = __vmaxu2(m4[0], v[c].x & 0x7FFF7FFFu);
            m4[1] = __vmaxu2(m4[1], v[c].y & 0x7FFF7FFFu);
            m4[2] = __vmaxu2(m4[2], v[c].z & 0x7FFF7FFFu);
            m4[3] = __vmaxu2(m4[3], v[c].w & 0x7FFF7FFFu);
          }
          const uint32_t mx2 = __vmaxu2(__vmaxu2(m4[0], m4[1]), __vmaxu2(m4[2], m4[3]));
          const uint32_t mx = max(mx2 & 0xFFFFu, mx2 >> 16);
          const int eb = static_cast<int>(mx >> 7);   // biased exponent of the largest magnitude
          int S = 0;
          if (mx != 0 && eb < 255) S = 14 - (eb == 0 ? -126 : eb - 127);
          S = S > 126 ? 126 : S;
          const float sc = __uint_as_float(static_cast<uint32_t>(S + 127) << 23);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t in[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
            uint32_t out[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const __half2 h = __floats2half2_rn(__uint_as_float(in[j] << 16) * sc,
                                                  __uint_as_float(in[j] & 0xFFFF0000u) * sc);
              out[j] = *reinterpret_cast<const uint32_t *>(&h);
            }
            *reinterpret_cast<uint4 *>(row + ((c ^ r) << 4)) = make_uint4(out[0], out[1], out[2], out[3]);
          }
          reinterpret_cast<float *>(smem + kXsOff + s * kXsStage)[lane] =
              __uint_as_float(static_cast<uint32_t>(127 - S) << 23);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&xready[s]);
      }
      u += t.nunits;
    }
    return;
  }

  if (warp >= kTmaWarp) {
    // ------------------------------------------------------------ producers
    // Two warps fill each stage: the copy warp issues the tensor copies (one
    // byte-count arrival), the scale warp the 4-byte absmax copies (one
    // arrival per lane when its copies land). Split so that neither issue
    // stream waits behind the other.
    const bool scale_warp = warp == kScaleWarp;
    const int r = lane >> 2, blk = lane & 3;
    const int64_t total_rows = static_cast<int64_t>(E) * N;
    const int64_t di = swiglu ? 8 : 16;            // rows from one unit to the next
    const int64_t dr = swiglu ? N / 2 : 8;         // rows from row group 0 to row group 1
    uint32_t it = 0;
    bool ok = true;
    for (int64_t u = u_lo; u < u_hi && ok;) {
      const Tile t = make_tile(u, u_hi, p, unit_start, row_off, gexp);
      const int64_t row0 = static_cast<int64_t>(t.e) * N + di * t.j0;   // first weight row
      // absmax source of this lane (row r, block blk) for each row group slot
      const int64_t arow = row0 + r;
      uint32_t vmask = 0;   // bit 2i+rgi: that row exists in the stack
      if (scale_warp) {
        for (int i = 0; i < t.nunits; ++i)
#pragma unroll
          for (int rgi = 0; rgi < 2; ++rgi)
            if (arow + i * di + rgi * dr < total_rows) vmask |= 1u << (2 * i + rgi);
      }
      const float *abase = absmax + arow * p.KB + blk;
      for (int kc = 0; kc < p.KC; ++kc, ++it) {
        const int s = static_cast<int>(it % kStages);
        const uint32_t ph = (it / kStages) & 1u;
        if (!warp_wait_bar(&empty[s], ph ^ 1u, abort_flag, hdr)) { ok = false; break; }
        if (scale_warp) {
          // stage layout [unit][block][row][row group]: a consumer lane reads
          // both row groups of its row in one 8-byte load
          char *as = smem + kAOff + s * kAStage + (blk * 8 + r) * 8;
          const bool kok = kc * kStageBlocks + blk < p.KB;
          for (int i = 0; i < t.nunits; ++i) {
#pragma unroll
            for (int rgi = 0; rgi < 2; ++rgi) {
              const bool v = kok && ((vmask >> (2 * i + rgi)) & 1u);
              const float *src = abase + ((i * di + rgi * dr) * p.KB + kc * kStageBlocks);
              cp_async4(smem_u32(as + i * 256 + rgi * 4), v ? src : absmax, v ? 4u : 0u);
            }
          }
          cp_async_arrive_noinc(&full[s]);
        } else if (lane == 0) {
          mbar_arrive_expect_tx(&full[s],
                                static_cast<uint32_t>(t.nunits * 16 * 128 + kXStage));
          char *ws = smem + kWOff + s * kWStage;
          if (!swiglu) {
            load_weight_rows(ws, wmaps, kc * 128, row0, t.nunits * 16, &full[s]);
          } else {   // gate rows, then the matching up rows 8 KB further
            load_weight_rows(ws, wmaps, kc * 128, row0, t.nunits * 8, &full[s]);
            load_weight_rows(ws + kTileUnits * kBoxBytes, wmaps, kc * 128, row0 + N / 2,
                             t.nunits * 8, &full[s]);
          }
          // the batch's activations for the stage's 4 blocks in one copy (a
          // block past K is zero-filled by the copy engine)
          tma_load_3d(smem + kXOff + s * kXStage, &xmap, 0, static_cast<int>(t.row0),
                      kc * kStageBlocks, &full[s]);
        }
      }
      u += t.nunits;
    }
    if (scale_warp) {
      cp_async_wait_all();
    } else if (lane == 0) {
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
  // their partial results when the tile's K loop ends.
  const int g = lane >> 2, q = lane & 3;
  const int up = warp & 3;                  // unit pair
  const int blk = warp >> 2;                // block of the stage
  // This lane's K-elements of a block: the 8 of 16-byte activation chunk f
  // and the 8 of chunk f ^ 4 (packed bytes 4 f .. 4 f + 3 and 4 (f ^ 4) ..),
  // f = 0, 5, 2, 7 for q = 0..3. With the 128-byte swizzle (chunk ^ row):
  // f & 3 takes every value, so a warp's 4-byte packed-word reads hit 32
  // distinct banks; and no two values of f differ only in bit 0, so the 8
  // lanes (rows g, g + 1) that share a 16-byte activation read's wavefront
  // hit 8 distinct chunks. Both reads run free of bank conflicts.
  const int f = (q & 2) | ((q & 1) ? 5 : 0);
  const int offA = g * 128 + (((2 * blk + (f >> 2)) ^ g) << 4) + 4 * (f & 3);
  const int offB = g * 128 + (((2 * blk + 1 - (f >> 2)) ^ g) << 4) + 4 * (f & 3);
  const int xoffA = blk * kBoxBytes + g * 128 + ((f ^ g) << 4);
  const int xoffB = blk * kBoxBytes + g * 128 + ((f ^ 4 ^ g) << 4);
  const uint32_t lutlane = static_cast<uint32_t>(kLutOff) | (static_cast<uint32_t>(lane) * 4u);
  const int64_t ncols = swiglu ? N / 2 : N;
  // partial sums of block warp b (1..3) for unit uu of the pair
  auto xchg_at = [&](int b, int uu) -> float4 * {
    return reinterpret_cast<float4 *>(smem + kXchgOff) + ((up * 3 + (b - 1)) * 2 + uu) * 32 + lane;
  };
  uint32_t it = 0, ep = 0;
  for (int64_t u = u_lo; u < u_hi;) {
    const Tile t = make_tile(u, u_hi, p, unit_start, row_off, gexp);
    const bool act0 = 2 * up < t.nunits, act1 = 2 * up + 1 < t.nunits;
    // C fragment: [0] weight row g, activation row 2q; [1] row g, 2q + 1;
    // [2] row g + 8 (SwiGLU: the matching up row), 2q; [3] row g + 8, 2q + 1
    float acc[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
    for (int kc = 0; kc < p.KC; ++kc, ++it) {
      const int s = static_cast<int>(it % kStages);
      const uint32_t ph = (it / kStages) & 1u;
      // the activation warp arrives on xready only after it has observed
      // this stage's copies complete (full), so this one wait also orders
      // the copied weights and absmax before the reads below
      if (!warp_wait_all(&xready[s], ph, abort_flag, hdr)) return;
      if (act0) {
        // A block past K reads zero-filled activations and absmax: it adds 0.
        const char *wst = smem + kWOff + s * kWStage;
        // 2^-S of activation rows 2q and 2q + 1 in this block
        const float2 xs = reinterpret_cast<const float2 *>(smem + kXsOff + s * kXsStage)[blk * 4 + q];
        const char *ast = smem + kAOff + s * kAStage + (blk * 8 + g) * 8;
        // (rows past the batch feed only outputs that are never stored)
        const char *xst = smem + kXOff + s * kXStage;
        const uint4 xa = *reinterpret_cast<const uint4 *>(xst + xoffA);
        const uint4 xb = *reinterpret_cast<const uint4 *>(xst + xoffB);
#pragma unroll
        for (int uu = 0; uu < 2; ++uu) {
          if (uu == 1 && !act1) break;
          const int ui = 2 * up + uu;
          // weight rows g and g + 8 of the unit (1 KB boxes of 8 rows)
          const char *r0 = wst + (swiglu ? ui : 2 * ui) * kBoxBytes;
          const char *r1 = wst + (swiglu ? kTileUnits + ui : 2 * ui + 1) * kBoxBytes;
          const uint32_t wa0 = *reinterpret_cast<const uint32_t *>(r0 + offA);
          const uint32_t wb0 = *reinterpret_cast<const uint32_t *>(r0 + offB);
          const uint32_t wa1 = *reinterpret_cast<const uint32_t *>(r1 + offA);
          const uint32_t wb1 = *reinterpret_cast<const uint32_t *>(r1 + offB);
          const float2 amv = *reinterpret_cast<const float2 *>(ast + ui * 256);
          const float am0 = amv.x, am1 = amv.y;   // rows g and g + 8
          // MMA k pairs (2q, 2q+1) and (2q+8, 2q+9) <- packed bytes (0, 1)
          // then (2, 3) of each word; activation registers in the same order.
          uint32_t ha0[4], la0[4], ha1[4], la1[4], hb0[4], lb0[4], hb1[4], lb1[4];
          decode_word(lutlane, wa0, ha0, la0);
          decode_word(lutlane, wa1, ha1, la1);
          decode_word(lutlane, wb0, hb0, lb0);
          decode_word(lutlane, wb1, hb1, lb1);
          float ch[4], cl[4];
          mma_f16_z(ch, ha0[0], ha1[0], ha0[1], ha1[1], xa.x, xa.y);
          mma_f16(ch, ha0[2], ha1[2], ha0[3], ha1[3], xa.z, xa.w);
          mma_f16(ch, hb0[0], hb1[0], hb0[1], hb1[1], xb.x, xb.y);
          mma_f16(ch, hb0[2], hb1[2], hb0[3], hb1[3], xb.z, xb.w);
          mma_f16_z(cl, la0[0], la1[0], la0[1], la1[1], xa.x, xa.y);
          mma_f16(cl, la0[2], la1[2], la0[3], la1[3], xa.z, xa.w);
          mma_f16(cl, lb0[0], lb1[0], lb0[1], lb1[1], xb.x, xb.y);
          mma_f16(cl, lb0[2], lb1[2], lb0[3], lb1[3], xb.z, xb.w);
          // block sum times absmax(row) and the activation rows' 2^-S
          acc[uu][0] = fmaf(fmaf(cl[0], kLoInv, ch[0]), am0 * xs.x, acc[uu][0]);
          acc[uu][1] = fmaf(fmaf(cl[1], kLoInv, ch[1]), am0 * xs.y, acc[uu][1]);
          acc[uu][2] = fmaf(fmaf(cl[2], kLoInv, ch[2]), am1 * xs.x, acc[uu][2]);
          acc[uu][3] = fmaf(fmaf(cl[3], kLoInv, ch[3]), am1 * xs.y, acc[uu][3]);
        }
      }
      __syncwarp();
      mbar_arrive_elect(&empty[s]);
    }
    if (act0) {
      if (blk != 0) {
        // hand the partial sums to the pair's block-0 warp
        if (ep > 0 && !warp_wait_bar(&xempty[up], (ep - 1) & 1u, abort_flag, hdr)) return;
#pragma unroll
        for (int uu = 0; uu < 2; ++uu)
          *xchg_at(blk, uu) = make_float4(acc[uu][0], acc[uu][1], acc[uu][2], acc[uu][3]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&xfull[up]);
      } else {
        if (!warp_wait_bar(&xfull[up], ep & 1u, abort_flag, hdr)) return;
#pragma unroll
        for (int b = 1; b < 4; ++b) {
#pragma unroll
          for (int uu = 0; uu < 2; ++uu) {
            const float4 v = *xchg_at(b, uu);
            acc[uu][0] += v.x;
            acc[uu][1] += v.y;
            acc[uu][2] += v.z;
            acc[uu][3] += v.w;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&xempty[up]);
#pragma unroll
        for (int uu = 0; uu < 2; ++uu) {
          if (uu == 1 && !act1) break;
          const int64_t j = t.j0 + 2 * up + uu;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int m = 2 * q + i;
            if (m >= t.mrows) continue;
            uint16_t *yr = y + (t.row0 + m) * ncols;
            const float a0 = acc[uu][i], a1 = acc[uu][2 + i];
            if (!swiglu) {
              const int64_t c0 = 16 * j + g, c1 = 16 * j + 8 + g;
              if (c0 < N) yr[c0] = bf16_bits(a0);
              if (c1 < N) yr[c1] = bf16_bits(a1);
            } else {
              const int64_t c = 8 * j + g;
              if (c < ncols) yr[c] = bf16_bits(silu(a0) * a1);
            }
          }
        }
      }
      ++ep;
    }
    u += t.nunits;
  }
}

}  // namespace

size_t decode_workspace_bytes(int64_t M, int32_t N, int32_t K, int32_t G, int32_t swiglu) {
  (void)M; (void)N; (void)K; (void)G; (void)swiglu;
  return kWsHeaderBytes;
}

size_t decode_zero_prefix_bytes(int64_t M, int32_t N, int32_t G, int32_t swiglu) {
  (void)M; (void)N; (void)G; (void)swiglu;
  return kWsHeaderBytes;
}

cudaError_t launch_decode_gemm(const GemmArgs &a, cudaStream_t stream) {
  if (static_cast<int64_t>(a.E) * a.N + a.N + 256 >= INT_MAX) return cudaErrorNotSupported;
  WeightMaps wm;
  // packed weights as [E*N rows][K/2 bytes], boxes of (8 << i) rows x 128 bytes
  for (int i = 0; i < kNumWMaps; ++i) {
    if (!encode_tensor_map_2d(&wm.m[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w,
                              static_cast<uint64_t>(a.K / 2),
                              static_cast<uint64_t>(a.E) * static_cast<uint64_t>(a.N),
                              static_cast<uint64_t>(a.K / 2), 128, 8u << i,
                              CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  // activations viewed as [K/64 blocks][M rows][64 bf16]: one box = 4 blocks x
  // 8 rows x 64 elements, laid out in shared memory as 4 swizzled 1 KB tiles
  CUtensorMap xmap;
  {
    const uint64_t dims[3] = {64, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.K / 64)};
    const uint64_t pitches[2] = {static_cast<uint64_t>(a.K) * 2, 128};
    const uint32_t box[3] = {64, kBatch, kStageBlocks};
    if (!encode_tensor_map(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.x, dims, pitches, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }

  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    cudaError_t err = cudaFuncSetAttribute(decode_gemm_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  return launch_pdl(decode_gemm_kernel, dim3(device_sm_count()), dim3(kThreads),
                    static_cast<size_t>(kSmemBytes), stream, wm, xmap, a.absmax, a.sizes,
                    a.expert_ids, a.G, a.M, a.N, a.K, a.E, a.swiglu, a.y,
                    static_cast<WsHeader *>(a.workspace));
}

}  // namespace gnf4
