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
// Inside a CTA (warp 16 = tensor copies, warp 17 = absmax copies, warps 0-15
// = consumers)
//   Stage = 256 K-elements of a tile: the tile's weight rows as a few TMA
//   boxes of 128 packed bytes per row (128-byte swizzle), the batch's
//   activations as one box of 4 blocks x 8 rows x 64 bf16, and the 8 x 4
//   absmax values of each row group (cp.async, 4 bytes each: absmax rows
//   need not be 16-byte aligned).
//   Consumer warp w decodes row group w / 8 of unit w % 8. Lane (g = lane/4,
//   q = lane%4) reads 8 packed bytes of row g per 64-element block. Each byte
//   (two codes) is ONE 8-byte shared-memory load from a 256-entry table
//   replicated per lane (no bank conflicts), addressed by one byte permute;
//   the entry holds (NF4[hi], NF4[lo]) as a bf16 pair plus the bf16 pair of
//   the remainders, so hi + lo equals the fp32 code value to within 2^-18
//   relative. The two halves feed an m16n8k16 bf16 MMA as adjacent
//   A-fragment registers: A rows 0-7 carry the hi parts of the 8 weight rows
//   and rows 8-15 their lo parts, so C rows g and g+8 sum to the exact-code
//   dot product of weight row g. The contraction index inside a block is
//   permuted identically for weights and activations (each lane takes 16
//   contiguous K-elements of the block). The block's fp32 result is scaled
//   by absmax(row, block) and accumulated in fp32. With SwiGLU the up-row
//   warp hands its accumulators to the gate-row warp through shared memory.
// Every wait is bounded (2 s); on expiry the kernel records
// GNF4_DEVERR_TIMEOUT, lets the producer's copies land and returns.
#include <climits>

#include "launch.h"
#include "sm100.cuh"

namespace gnf4 {
namespace {

constexpr int kConsumerWarps = 16;
constexpr int kTmaWarp = kConsumerWarps;          // issues the tensor copies
constexpr int kScaleWarp = kConsumerWarps + 1;    // copies the absmax values
constexpr int kThreads = (kConsumerWarps + 2) * 32;
constexpr int kTileUnits = 8;                 // units per tile (2 row groups each)
constexpr int kStages = 6;
constexpr int kBatch = 8;                     // activation rows per batch (MMA N)
constexpr int kBoxBytes = 1024;               // 8 rows x 128 bytes
constexpr int kStageBlocks = 4;               // absmax blocks per stage (256 K-elements)
constexpr int kWStage = kTileUnits * 2 * kBoxBytes;              // 16 KB
constexpr int kXStage = kStageBlocks * kBoxBytes;                // 4 KB
constexpr int kAStage = kTileUnits * 2 * 8 * kStageBlocks * 4;   // 2 KB
constexpr int kMaxG = GNF4_MAX_EXPERTS;

// Dynamic shared memory layout (bytes from a 1024-aligned base).
constexpr int kWOff = 0;
constexpr int kXOff = kWOff + kStages * kWStage;
constexpr int kLutOff = kXOff + kStages * kXStage;   // uint2 [256 bytes][32 lanes]
constexpr int kLutBytes = 256 * 32 * 8;
constexpr int kAOff = kLutOff + kLutBytes;
constexpr int kUnitStartOff = kAOff + kStages * kAStage;      // int64 [kMaxG + 1]
constexpr int kRowOffOff = kUnitStartOff + (kMaxG + 1) * 8;   // int32 [kMaxG]
constexpr int kGSizeOff = kRowOffOff + kMaxG * 4;             // int32 [kMaxG]
constexpr int kGExpOff = kGSizeOff + kMaxG * 4;               // int32 [kMaxG]
constexpr int kXchgOff = kGExpOff + kMaxG * 4;                // float2 [kTileUnits][32]
constexpr int kBarOff = kXchgOff + kTileUnits * 32 * 8;       // mbarriers, see kNumBars
// full[kStages], empty[kStages], then per unit slot: xfull (up accumulators
// written), xempty (gate warp done reading them)
constexpr int kNumBars = 2 * kStages + 2 * kTileUnits;
constexpr int kMiscOff = kBarOff + kNumBars * 8;              // int [8]
constexpr int kSmemBytes = kMiscOff + 8 * 4 + 1024;           // + alignment slack
static_assert(kBarOff % 8 == 0 && kXchgOff % 8 == 0, "8-byte aligned");
static_assert(kSmemBytes <= 227 * 1024, "fits one CTA per SM");

// ------------------------------------------------------------------ PTX

// Not volatile: the compiler may interleave independent accumulation chains.
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// (hi pair, lo pair) of byte p of `word`, from this lane's table slot.
__device__ __forceinline__ uint2 lut_pair(const char *lut, uint32_t word, uint32_t lane8,
                                          uint32_t p) {
  const uint32_t off = __byte_perm(word, lane8, 0x5504u | (p << 4));   // byte*256 + lane*8
  return *reinterpret_cast<const uint2 *>(lut + off);
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  const __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<const uint16_t *>(&b);
}

// bf16 (hi, lo) split of an fp32 code value: hi = RNE(v), lo = RNE(v - hi),
// as hi | lo << 16.
__device__ __forceinline__ uint32_t code_split(int c) {
  const float v = nf4_value(c);
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
  return static_cast<uint32_t>(*reinterpret_cast<const uint16_t *>(&h)) |
         (static_cast<uint32_t>(*reinterpret_cast<const uint16_t *>(&l)) << 16);
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
                                          const int *gsize, const int *gexp) {
  int lo = 0, hi = p.G;   // invariant: unit_start[lo] <= u < unit_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (unit_start[mid] <= u) lo = mid; else hi = mid;
  }
  const int64_t local = u - unit_start[lo];
  const int64_t batch = local / p.upb;
  const int64_t run_end = unit_start[lo] + (batch + 1) * p.upb;
  int64_t end = u + kTileUnits;
  if (end > u_hi) end = u_hi;
  if (end > run_end) end = run_end;
  Tile t;
  t.row0 = static_cast<int64_t>(row_off[lo]) + batch * kBatch;
  t.j0 = local - batch * p.upb;
  t.nunits = static_cast<int32_t>(end - u);
  t.mrows = min(kBatch, gsize[lo] - static_cast<int32_t>(batch) * kBatch);
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
  extern __shared__ char smem_raw[];
  char *smem = reinterpret_cast<char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~static_cast<uintptr_t>(1023));
  int64_t *unit_start = reinterpret_cast<int64_t *>(smem + kUnitStartOff);
  int *row_off = reinterpret_cast<int *>(smem + kRowOffOff);
  int *gsize = reinterpret_cast<int *>(smem + kGSizeOff);
  int *gexp = reinterpret_cast<int *>(smem + kGExpOff);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kBarOff);
  uint64_t *empty = full + kStages;
  uint64_t *xfull = empty + kStages;      // [kTileUnits]
  uint64_t *xempty = xfull + kTileUnits;  // [kTileUnits]
  int *misc = reinterpret_cast<int *>(smem + kMiscOff);   // [0] error bits, [1] abort
  volatile int *abort_flag = &misc[1];
  __shared__ int64_t s_wsum[2][kThreads / 32];

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
    }
    for (int i = 0; i < kTileUnits; ++i) {
      mbar_init(&xfull[i], 1);
      mbar_init(&xempty[i], 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int i = 0; i < kNumWMaps; ++i) prefetch_tensormap(&wmaps.m[i]);
    prefetch_tensormap(&xmap);
  }

  // ---- decode table: entry byte b, lane slot l = {bf16x2 hi, bf16x2 lo} of
  //      the pair (NF4[b >> 4], NF4[b & 15]) (low half = even k = high nibble)
  if (tid < 256) {
    const uint32_t c0 = code_split(tid >> 4), c1 = code_split(tid & 15);
    const uint32_t hp = (c0 & 0xFFFFu) | (c1 << 16);
    const uint32_t lp = (c0 >> 16) | (c1 & 0xFFFF0000u);
    uint4 *dst = reinterpret_cast<uint4 *>(smem + kLutOff + tid * 256);
#pragma unroll
    for (int i = 0; i < 16; ++i) dst[i] = make_uint4(hp, lp, hp, lp);
  }

  pdl_wait();   // inputs may come from the previous kernel on the stream

  // ---- group table from (sizes, expert_ids), validated on the device
  const int per = (G + kThreads - 1) / kThreads;
  const int g0 = min(G, tid * per), g1 = min(G, g0 + per);
  int64_t my_rows = 0, my_units = 0;
  int bad = 0;
  for (int g = g0; g < g1; ++g) {
    const int sz = sizes[g];
    const int e = expert_ids[g];
    if (sz < 0) bad |= GNF4_DEVERR_SIZES;
    if (sz > 0 && (e < 0 || e >= E)) bad |= GNF4_DEVERR_EXPERT;
    gsize[g] = sz;
    gexp[g] = e;
    my_rows += max(sz, 0);
    my_units += sz > 0 ? ((sz + kBatch - 1) / kBatch) * p.upb : 0;
  }

  __syncthreads();   // barrier init and misc visible
  if (bad) atomicOr(&misc[0], bad);

  int64_t vr = my_rows, vu = my_units;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t a = __shfl_up_sync(0xffffffffu, vr, o);
    const int64_t b = __shfl_up_sync(0xffffffffu, vu, o);
    if (lane >= o) { vr += a; vu += b; }
  }
  if (lane == 31) { s_wsum[0][warp] = vr; s_wsum[1][warp] = vu; }
  __syncthreads();
  int64_t wr = 0, wu = 0, tot_r = 0, tot_u = 0;
  for (int i = 0; i < kThreads / 32; ++i) {
    if (i < warp) { wr += s_wsum[0][i]; wu += s_wsum[1][i]; }
    tot_r += s_wsum[0][i];
    tot_u += s_wsum[1][i];
  }
  {
    int64_t r = wr + vr - my_rows, c = wu + vu - my_units;
    for (int g = g0; g < g1; ++g) {
      const int sz = max(gsize[g], 0);
      row_off[g] = static_cast<int>(r);
      unit_start[g] = c;
      r += sz;
      c += sz > 0 ? ((sz + kBatch - 1) / kBatch) * p.upb : 0;
    }
    if (tid == 0) unit_start[G] = tot_u;
  }
  if (tid == 0 && tot_r != M) atomicOr(&misc[0], GNF4_DEVERR_SIZES);
  __syncthreads();
  const int errbits = misc[0];
  if (errbits) {
    if (blockIdx.x == 0 && tid == 0) report_error(hdr, static_cast<uint32_t>(errbits), 0);
    return;
  }
  const int64_t P = gridDim.x;
  const int64_t u_lo = tot_u * blockIdx.x / P;
  const int64_t u_hi = tot_u * (blockIdx.x + 1) / P;
  if (u_lo >= u_hi) return;

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
      const Tile t = make_tile(u, u_hi, p, unit_start, row_off, gsize, gexp);
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
          char *as = smem + kAOff + s * kAStage + r * 16 + blk * 4;
          const bool kok = kc * kStageBlocks + blk < p.KB;
          for (int i = 0; i < t.nunits; ++i) {
#pragma unroll
            for (int rgi = 0; rgi < 2; ++rgi) {
              const bool v = kok && ((vmask >> (2 * i + rgi)) & 1u);
              const float *src = abase + ((i * di + rgi * dr) * p.KB + kc * kStageBlocks);
              cp_async4(smem_u32(as + (i * 2 + rgi) * 8 * 16), v ? src : absmax, v ? 4u : 0u);
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
  const int g = lane >> 2, q = lane & 3;
  const int ui = warp % kTileUnits;         // unit slot within the tile
  const int rgi = warp / kTileUnits;        // row group of the unit (SwiGLU: 0 gate, 1 up)
  const uint32_t lane8 = static_cast<uint32_t>(lane) * 8u;
  const char *lut = smem + kLutOff;
  const int64_t ncols = swiglu ? N / 2 : N;
  // this warp's 8 weight rows in a stage (SwiGLU: gate rows first, up rows 8 KB on)
  const int wslot = swiglu ? rgi * kTileUnits + ui : 2 * ui + rgi;
  float2 *xchg = reinterpret_cast<float2 *>(smem + kXchgOff) + ui * 32;
  uint32_t it = 0, ep = 0;
  for (int64_t u = u_lo; u < u_hi;) {
    const Tile t = make_tile(u, u_hi, p, unit_start, row_off, gsize, gexp);
    const bool active = ui < t.nunits;
    const int64_t j = t.j0 + ui;
    float acc0 = 0.0f, acc1 = 0.0f;   // weight row g, activation rows 2q and 2q+1
    for (int kc = 0; kc < p.KC; ++kc, ++it) {
      const int s = static_cast<int>(it % kStages);
      const uint32_t ph = (it / kStages) & 1u;
      if (!warp_wait_bar(&full[s], ph, abort_flag, hdr)) return;
      if (active) {
        // 4 blocks = 4 independent accumulation chains, interleaved per k-step.
        // Blocks past K read zero-filled weights, activations and absmax: they add 0.
        const char *wst = smem + kWOff + s * kWStage + wslot * kBoxBytes + g * 128;
        const char *xst = smem + kXOff + s * kXStage + g * 128;
        const char *ast = smem + kAOff + s * kAStage + ((2 * ui + rgi) * 8 + g) * 16;
#pragma unroll 1
        for (int bp = 0; bp < kStageBlocks; bp += 2) {
          uint32_t xr[2][8];
          uint2 wd[2];
          float am[2];
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
            const int b = bp + bb;
            uint4 xa = make_uint4(0u, 0u, 0u, 0u), xb = xa;
            if (g < t.mrows) {
              xa = *reinterpret_cast<const uint4 *>(xst + b * kBoxBytes + (((2 * q) ^ g) << 4));
              xb = *reinterpret_cast<const uint4 *>(xst + b * kBoxBytes + (((2 * q + 1) ^ g) << 4));
            }
            xr[bb][0] = xa.x; xr[bb][1] = xa.y; xr[bb][2] = xa.z; xr[bb][3] = xa.w;
            xr[bb][4] = xb.x; xr[bb][5] = xb.y; xr[bb][6] = xb.z; xr[bb][7] = xb.w;
            const int c = 2 * b + (q >> 1);
            wd[bb] = *reinterpret_cast<const uint2 *>(wst + ((c ^ g) << 4) + 8 * (q & 1));
            am[bb] = *reinterpret_cast<const float *>(ast + b * 4);
          }
          float cc[2][4];
#pragma unroll
          for (int bb = 0; bb < 2; ++bb)
#pragma unroll
            for (int i = 0; i < 4; ++i) cc[bb][i] = 0.0f;
#pragma unroll
          for (int st = 0; st < 4; ++st) {
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
              const uint32_t word = st < 2 ? wd[bb].x : wd[bb].y;
              const uint32_t pp = (st & 1) * 2;
              const uint2 e0 = lut_pair(lut, word, lane8, pp);
              const uint2 e1 = lut_pair(lut, word, lane8, pp + 1);
              mma_bf16(cc[bb], e0.x, e0.y, e1.x, e1.y, xr[bb][2 * st], xr[bb][2 * st + 1]);
            }
          }
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
            acc0 = fmaf(cc[bb][0] + cc[bb][2], am[bb], acc0);
            acc1 = fmaf(cc[bb][1] + cc[bb][3], am[bb], acc1);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (active) {
      if (!swiglu) {
        const int64_t col = 16 * j + 8 * rgi + g;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int m = 2 * q + i;
          if (m < t.mrows && col < N) y[(t.row0 + m) * ncols + col] = bf16_bits(i ? acc1 : acc0);
        }
      } else if (rgi == 1) {
        // up rows: hand the accumulators to the gate warp of the same unit
        if (ep > 0 && !warp_wait_bar(&xempty[ui], (ep - 1) & 1u, abort_flag, hdr)) return;
        xchg[lane] = make_float2(acc0, acc1);
        __syncwarp();
        if (lane == 0) mbar_arrive(&xfull[ui]);
      } else {
        if (!warp_wait_bar(&xfull[ui], ep & 1u, abort_flag, hdr)) return;
        const float2 up = xchg[lane];
        __syncwarp();
        if (lane == 0) mbar_arrive(&xempty[ui]);
        const int64_t col = 8 * j + g;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int m = 2 * q + i;
          if (m < t.mrows && col < ncols)
            y[(t.row0 + m) * ncols + col] = bf16_bits(silu(i ? acc1 : acc0) * (i ? up.y : up.x));
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
