// decode_gemm.cu -- decode-regime grouped NF4 GEMM (few rows per expert).
//
// Passage: "grouped-nf4-gemm -- single-launch W4A16 GEMM over fused NF4 MoE
// expert stacks", opening section (one launch for all active experts, LUT
// decode of the packed codes, blockwise fp32 absmax, fp32 accumulation, bf16
// epilogue, no bf16 weight copy) and "Status / roadmap" (split-K for starved
// grids). At a handful of rows per expert this GEMM streams every touched
// weight byte exactly once and is bound by HBM bandwidth.
//
// Work decomposition
//   tile   = (row chunk, column tile): up to 8 activation rows of one group
//            times 256 weight rows of that group's expert (with SwiGLU: 128
//            gate rows j..j+127 and the matching 128 up rows N/2+j.., so the
//            epilogue pairs them in registers).
//   unit   = one 64-element absmax block of K for a whole tile.
//   Stream-K: the tiles' units are laid end to end and every CTA takes an
//   equal contiguous range. A tile covered by one CTA is finished in
//   registers; a tile split between CTAs is finished by whichever contributor
//   arrives last (per-tile counter in the workspace), which sums the fp32
//   partials in CTA order, so the result does not depend on arrival order.
//   The tile list is derived on the device from (sizes, expert_ids): the
//   host never learns which experts are active (no sync, graph-capturable).
//
// Inside a CTA (8 warps, two CTAs per SM)
//   Warp w owns 32 of the tile's weight rows as four groups of 8 (row group
//   rg). A step covers 2 blocks; for each block, lane (g = lane/4, q = lane%4)
//   loads 8 packed bytes of row g of each group (one 8-byte load per row; the
//   four lanes of a row cover its 32 bytes, so every load instruction reads
//   whole 32-byte sectors) and the block's absmax, one step ahead of use.
//   Decode: each byte (two codes) is ONE 8-byte shared-memory load from a
//   256-entry table, replicated per lane so the warp never hits a bank
//   conflict and addressed by a single byte permute. The entry holds
//   (NF4[hi], NF4[lo]) as a bf16 pair plus the bf16 pair of their
//   remainders, so hi + lo equals the fp32 code value to within 2^-18
//   relative. The two 32-bit halves of the entry feed an m16n8k16 bf16
//   tensor-core MMA directly as adjacent A-fragment registers: A rows 0-7
//   carry the hi parts of the group's 8 weight rows and A rows 8-15 the lo
//   parts of the same rows, so C rows g and g+8 are the hi and lo partial
//   sums of weight row g and their sum is the exact-weight dot product. The
//   multiply-accumulate over a block's 64 elements for all 8 activation rows
//   is then four MMAs per 8x64 weights instead of one FMA per weight per
//   row: the CUDA cores only decode (one permute and one shared load per two
//   weights). The contraction index inside a block is permuted identically
//   for weights and activations so that each lane's weight bytes are
//   contiguous; each lane reads its bf16 activation fragment (16 contiguous
//   values of one row) straight from global memory, where it stays cached in
//   L1 for the whole CTA. The block's fp32 result is scaled by absmax(weight
//   row, block) and added to an fp32 accumulator.
#include "launch.h"

namespace gnf4 {
namespace {

constexpr int kThreads = 256;         // 8 warps
constexpr int kCtasPerSm = 2;
constexpr int kRows = 256;            // weight rows per tile: 8 warps x 2 slices x 16
constexpr int kMT = 8;                // activation rows per tile = MMA N
constexpr int kStepBlocks = 2;        // 64-element blocks per step
constexpr int kMaxG = GNF4_MAX_EXPERTS;
constexpr int kPartialFloats = 8 * kThreads;   // 8 accumulators per thread

// Dynamic shared memory layout (bytes).
constexpr int kLutOff = 0;                                    // uint2 [256 bytes][32 lanes]
constexpr int kLutBytes = 256 * 32 * 8;
constexpr int kChunkStartOff = kLutOff + kLutBytes;           // int[kMaxG + 1]
constexpr int kRowOffOff = kChunkStartOff + (kMaxG + 4) * 4;  // int[kMaxG]
constexpr int kGSizeOff = kRowOffOff + kMaxG * 4;             // int[kMaxG]
constexpr int kGExpOff = kGSizeOff + kMaxG * 4;               // int[kMaxG]
constexpr int kMiscOff = kGExpOff + kMaxG * 4;                // int[16]
constexpr int kSmemBytes = kMiscOff + 16 * 4;

// Named barrier of the split-tile protocol (all kThreads threads take part).
constexpr uint32_t kBarPartial = 1;

// Blocks in a step: at most kStepBlocks, never past the row end or range end.
__device__ __forceinline__ int step_blocks(int64_t left_in_row, int64_t left_in_range) {
  const int64_t n = left_in_row < left_in_range ? left_in_row : left_in_range;
  return static_cast<int>(n < kStepBlocks ? n : kStepBlocks);
}

struct Sched {
  int32_t G, N, K, E, swiglu;
  int32_t KB;        // 64-element blocks per row
  int32_t NT;        // column tiles per row chunk
  int64_t units;     // total units
  int64_t lo, hi;    // this CTA's unit range
};

// Tile-level facts (identical in every thread).
struct TileGroup {
  int64_t row0;      // first activation row
  int32_t mrows;     // activation rows (1..kMT)
  int32_t j;         // column tile
  int32_t e;         // expert
};

// This thread's view of a tile: weight row wrow0 + RowOffsets::dr[rg] for
// row group rg (row g of the group), its activation row (row0 + g, or -1 if
// the tile has no row g), and which row groups exist.
struct ThreadTile {
  int64_t wrow0;
  int64_t xrow;
  int32_t col0;       // output column of row group 0
  uint32_t vmask;     // bit rg: that weight row exists
};

// Row offsets of the four row groups from row group 0 (uniform per launch).
struct RowOffsets {
  int32_t dr[4];      // weight rows
  int32_t dc[4];      // output columns (-1: not an output row)
};

__device__ __forceinline__ RowOffsets make_offsets(int32_t N, int32_t swiglu) {
  RowOffsets o;
#pragma unroll
  for (int rg = 0; rg < 4; ++rg) {
    if (swiglu) {   // rg 0,1: gate rows; rg 2,3: the up rows of the same columns
      o.dr[rg] = 8 * (rg & 1) + (rg < 2 ? 0 : N / 2);
      o.dc[rg] = rg < 2 ? 8 * rg : -1;
    } else {
      o.dr[rg] = 8 * rg;
      o.dc[rg] = 8 * rg;
    }
  }
  return o;
}

__device__ __forceinline__ TileGroup tile_group(int64_t T, const Sched &s, const int *chunk_start,
                                                const int *row_off, const int *gsize,
                                                const int *gexp) {
  TileGroup tg;
  const int64_t c = T / s.NT;
  tg.j = static_cast<int32_t>(T - c * s.NT);
  int lo = 0, hi = s.G;   // invariant: chunk_start[lo] <= c < chunk_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (chunk_start[mid] <= c) lo = mid; else hi = mid;
  }
  const int32_t local = static_cast<int32_t>(c - chunk_start[lo]);
  tg.row0 = static_cast<int64_t>(row_off[lo]) + static_cast<int64_t>(local) * kMT;
  tg.mrows = min(kMT, gsize[lo] - local * kMT);
  tg.e = gexp[lo];
  return tg;
}

__device__ __forceinline__ ThreadTile thread_tile(const TileGroup &tg, const Sched &s, int warp,
                                                  int g) {
  ThreadTile r;
  const int n0 = s.swiglu ? tg.j * 128 + warp * 16 + g : tg.j * kRows + warp * 32 + g;
  const int lim = s.swiglu ? s.N / 2 : s.N;   // columns at or past lim are padding
  uint32_t m;
  if (s.swiglu) {
    m = (n0 < lim ? 5u : 0u) | (n0 + 8 < lim ? 10u : 0u);   // rg 0/2 share n0, rg 1/3 n0+8
  } else {
    m = (n0 < lim ? 1u : 0u) | (n0 + 8 < lim ? 2u : 0u) | (n0 + 16 < lim ? 4u : 0u) |
        (n0 + 24 < lim ? 8u : 0u);
  }
  r.vmask = m;
  r.col0 = n0;
  r.wrow0 = static_cast<int64_t>(tg.e) * s.N + n0;
  r.xrow = g < tg.mrows ? tg.row0 + g : -1;
  return r;
}

// 8 packed bytes (16 codes) of a row; streamed, no L1 allocation.
__device__ __forceinline__ uint2 ldg64_stream(const void *p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.b32 {%0,%1}, [%2];"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p));
  return r;
}

struct StepW {
  uint2 w[kStepBlocks][4];    // [block][row group]: this lane's 8 bytes
  float a[kStepBlocks][4];    // [block][row group]: absmax
};

__device__ __forceinline__ void load_step(const ThreadTile &tt, const RowOffsets &ro,
                                          const uint8_t *__restrict__ w,
                                          const float *__restrict__ absmax, int64_t row_bytes,
                                          int KB, int kb0, int nblk, int q, StepW &d) {
#pragma unroll
  for (int rg = 0; rg < 4; ++rg) {
    const int64_t row = tt.wrow0 + ro.dr[rg];
    const bool ok = (tt.vmask >> rg) & 1u;
    const uint8_t *wp = w + row * row_bytes + kb0 * 32 + 8 * q;
    const float *ap = absmax + row * KB + kb0;
#pragma unroll
    for (int b = 0; b < kStepBlocks; ++b) {
      const bool on = ok && b < nblk;
      d.w[b][rg] = on ? ldg64_stream(wp + b * 32) : make_uint2(0x77777777u, 0x77777777u);
      d.a[b][rg] = on ? __ldg(ap + b) : 0.0f;
    }
  }
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
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

// acc[rg][i] += absmax * (64-element block dot product) for activation row 2q+i.
// b: block within the step.
__device__ __forceinline__ void compute_block(const StepW &d, int b, const ThreadTile &tt,
                                              const uint16_t *__restrict__ x, int64_t K, int kb,
                                              int q, int lane, const char *lut, uint32_t lane8,
                                              float (&acc)[4][2]) {
  // activation fragment: 16 bf16 of row g at k = 16q..16q+15 of this block
  uint4 xa = make_uint4(0u, 0u, 0u, 0u), xb = xa;
  if (tt.xrow >= 0) {
    const uint4 *xp = reinterpret_cast<const uint4 *>(x + tt.xrow * K + kb * 64 + 16 * q);
    xa = __ldg(xp);
    xb = __ldg(xp + 1);
  }
  const uint32_t xr[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
  for (int rg = 0; rg < 4; ++rg) {
    float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int st = 0; st < 4; ++st) {
      const uint32_t word = st < 2 ? d.w[b][rg].x : d.w[b][rg].y;
      const uint32_t p = (st & 1) * 2;
      const uint2 e0 = lut_pair(lut, word, lane8, p);       // k = 16q+4st+{0,1}
      const uint2 e1 = lut_pair(lut, word, lane8, p + 1);   // k = 16q+4st+{2,3}
      mma_bf16(c, e0.x, e0.y, e1.x, e1.y, xr[2 * st], xr[2 * st + 1]);
    }
    const float a = d.a[b][rg];
    acc[rg][0] = fmaf(c[0] + c[2], a, acc[rg][0]);
    acc[rg][1] = fmaf(c[1] + c[3], a, acc[rg][1]);
  }
}

__device__ __forceinline__ int64_t cta_lo(int64_t units, int64_t c, int64_t P) {
  return units * c / P;
}
// CTA whose range contains unit u.
__device__ __forceinline__ int64_t cta_of(int64_t units, int64_t u, int64_t P) {
  return ((u + 1) * P - 1) / units;
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

__device__ __forceinline__ void store_bf16(uint16_t *p, float v) {
  const __nv_bfloat16 b = __float2bfloat16_rn(v);
  *p = *reinterpret_cast<const uint16_t *>(&b);
}

// Epilogue: acc[rg][i] is weight row group rg, activation row 2q + i.
__device__ __forceinline__ void write_tile(const float (&v)[4][2], const TileGroup &tg,
                                           const ThreadTile &tt, const RowOffsets &ro,
                                           const Sched &s, uint16_t *__restrict__ y, int q) {
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int m = 2 * q + i;
    if (m >= tg.mrows) continue;
    if (!s.swiglu) {
#pragma unroll
      for (int rg = 0; rg < 4; ++rg)
        if ((tt.vmask >> rg) & 1u)
          store_bf16(y + (tg.row0 + m) * s.N + tt.col0 + ro.dc[rg], v[rg][i]);
    } else {
#pragma unroll
      for (int rg = 0; rg < 2; ++rg)
        if ((tt.vmask >> rg) & 1u)
          store_bf16(y + (tg.row0 + m) * (s.N / 2) + tt.col0 + ro.dc[rg],
                     silu(v[rg][i]) * v[rg + 2][i]);
    }
  }
}

// bf16 (hi, lo) split of an fp32 value: hi = RNE(v), lo = RNE(v - hi).
__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16 &hi, __nv_bfloat16 &lo) {
  hi = __float2bfloat16_rn(v);
  lo = __float2bfloat16_rn(v - __bfloat162float(hi));
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    decode_gemm_kernel(const uint16_t *__restrict__ x, const uint8_t *__restrict__ w,
                       const float *__restrict__ absmax, const int32_t *__restrict__ sizes,
                       const int32_t *__restrict__ expert_ids, int32_t G, int64_t M, int32_t N,
                       int32_t K, int32_t E, int32_t swiglu, uint16_t *__restrict__ y,
                       WsHeader *hdr, int32_t *__restrict__ tile_cnt, int64_t tile_cap,
                       float *__restrict__ partials) {
  extern __shared__ __align__(1024) char smem[];
  int *chunk_start = reinterpret_cast<int *>(smem + kChunkStartOff);
  int *row_off = reinterpret_cast<int *>(smem + kRowOffOff);
  int *gsize = reinterpret_cast<int *>(smem + kGSizeOff);
  int *gexp = reinterpret_cast<int *>(smem + kGExpOff);
  int *misc = reinterpret_cast<int *>(smem + kMiscOff);   // [0] error bits, [2] last-arriver flag

  const int t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  const int g = lane >> 2, q = lane & 3;

  // ---- 1. decode table: entry byte b, lane slot l = {bf16x2 hi, bf16x2 lo}
  //      of the pair (NF4[b >> 4], NF4[b & 15]) (low half = even k = high nibble).
  for (int i = t; i < 256 * 32; i += kThreads) {
    const int b = i >> 5;
    __nv_bfloat16 h0, l0, h1, l1;
    split_bf16(nf4_value(b >> 4), h0, l0);
    split_bf16(nf4_value(b & 15), h1, l1);
    __nv_bfloat162 hp, lp;
    hp.x = h0; hp.y = h1;
    lp.x = l0; lp.y = l1;
    uint2 e;
    e.x = *reinterpret_cast<const uint32_t *>(&hp);
    e.y = *reinterpret_cast<const uint32_t *>(&lp);
    reinterpret_cast<uint2 *>(smem + kLutOff)[i] = e;
  }
  if (t == 0) misc[0] = 0;
  __syncthreads();

  // ---- 2. group table from (sizes, expert_ids), validated on the device.
  __shared__ int s_wsum[2][kThreads / 32];
  const int per = (G + kThreads - 1) / kThreads;
  const int g0 = min(G, t * per), g1 = min(G, g0 + per);
  int my_rows = 0, my_chunks = 0, bad = 0;
  for (int gi = g0; gi < g1; ++gi) {
    const int sz = sizes[gi];
    const int e = expert_ids[gi];
    if (sz < 0) bad |= GNF4_DEVERR_SIZES;
    if (sz > 0 && (e < 0 || e >= E)) bad |= GNF4_DEVERR_EXPERT;
    gsize[gi] = sz;
    gexp[gi] = e;
    my_rows += max(sz, 0);
    my_chunks += sz > 0 ? (sz + kMT - 1) / kMT : 0;
  }
  if (bad) atomicOr(&misc[0], bad);
  int vr = my_rows, vc = my_chunks;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, vr, o);
    const int b = __shfl_up_sync(0xffffffffu, vc, o);
    if (lane >= o) { vr += a; vc += b; }
  }
  if (lane == 31) { s_wsum[0][warp] = vr; s_wsum[1][warp] = vc; }
  __syncthreads();
  int wr = 0, wc = 0, tot_r = 0, tot_c = 0;
  for (int i = 0; i < kThreads / 32; ++i) {
    if (i < warp) { wr += s_wsum[0][i]; wc += s_wsum[1][i]; }
    tot_r += s_wsum[0][i];
    tot_c += s_wsum[1][i];
  }
  {
    int r = wr + vr - my_rows, c = wc + vc - my_chunks;
    for (int gi = g0; gi < g1; ++gi) {
      row_off[gi] = r;
      chunk_start[gi] = c;
      const int sz = max(gsize[gi], 0);
      r += sz;
      c += sz > 0 ? (sz + kMT - 1) / kMT : 0;
    }
    if (t == 0) chunk_start[G] = tot_c;
  }
  if (t == 0 && static_cast<int64_t>(tot_r) != M) atomicOr(&misc[0], GNF4_DEVERR_SIZES);
  __syncthreads();

  Sched s;
  s.G = G; s.N = N; s.K = K; s.E = E; s.swiglu = swiglu;
  s.KB = K / 64;
  s.NT = swiglu ? (N / 2 + 127) / 128 : (N + kRows - 1) / kRows;
  const int64_t tiles = static_cast<int64_t>(tot_c) * s.NT;
  int errbits = misc[0];
  if (errbits == 0 && tiles > tile_cap) errbits = GNF4_DEVERR_CAPACITY;
  if (errbits) {
    if (blockIdx.x == 0 && t == 0) report_error(hdr, static_cast<uint32_t>(errbits), 0);
    return;
  }
  s.units = tiles * s.KB;
  const int64_t P = gridDim.x;
  s.lo = cta_lo(s.units, blockIdx.x, P);
  s.hi = cta_lo(s.units, blockIdx.x + 1, P);
  if (s.lo >= s.hi) return;

  const uint32_t lane8 = static_cast<uint32_t>(lane) * 8u;
  const char *lut = smem + kLutOff;
  const RowOffsets ro = make_offsets(N, swiglu);
  const int64_t row_bytes = K / 2;

  float acc[4][2];
#pragma unroll
  for (int rg = 0; rg < 4; ++rg) acc[rg][0] = acc[rg][1] = 0.0f;

  // ---- 4. main loop: steps of up to kStepBlocks blocks, never crossing a tile
  int64_t T = s.lo / s.KB;
  int kb0 = static_cast<int>(s.lo - T * s.KB);
  int64_t u = s.lo;
  TileGroup tg = tile_group(T, s, chunk_start, row_off, gsize, gexp);
  ThreadTile tt = thread_tile(tg, s, warp, g);
  int nblk = step_blocks(s.KB - kb0, s.hi - u);
  StepW cur;
  load_step(tt, ro, w, absmax, row_bytes, s.KB, kb0, nblk, q, cur);

  while (true) {
    // issue the next step's loads before consuming this one
    const int64_t un = u + nblk;
    const bool has_next = un < s.hi;
    const bool tile_end = (kb0 + nblk == s.KB) || !has_next;
    int64_t Tn = T;
    int kbn = kb0 + nblk;
    TileGroup tgn = tg;
    ThreadTile ttn = tt;
    int nbn = 0;
    StepW nxt;
    if (has_next) {
      if (kbn == s.KB) {
        kbn = 0;
        Tn = T + 1;
        tgn = tile_group(Tn, s, chunk_start, row_off, gsize, gexp);
        ttn = thread_tile(tgn, s, warp, g);
      }
      nbn = step_blocks(s.KB - kbn, s.hi - un);
      load_step(ttn, ro, w, absmax, row_bytes, s.KB, kbn, nbn, q, nxt);
    }

#pragma unroll
    for (int b = 0; b < kStepBlocks; ++b)
      if (b < nblk) compute_block(cur, b, tt, x, s.K, kb0 + b, q, lane, lut, lane8, acc);

    if (tile_end) {
      const bool whole = (T * s.KB >= s.lo) && ((T + 1) * s.KB <= s.hi);
      if (whole) {
        write_tile(acc, tg, tt, ro, s, y, q);
      } else {
        // split tile: publish the partial, the last contributor finishes it
        const int slot = (T == s.lo / s.KB) ? 0 : 1;
        float *mine = partials + (static_cast<int64_t>(blockIdx.x) * 2 + slot) * kPartialFloats;
#pragma unroll
        for (int rg = 0; rg < 4; ++rg)
#pragma unroll
          for (int i = 0; i < 2; ++i) mine[(rg * 2 + i) * kThreads + t] = acc[rg][i];
        __threadfence();
        named_barrier(kBarPartial, kThreads);
        if (t == 0) {
          // contributors: the CTAs with a non-empty range inside [c0, c1]
          const int64_t c0 = cta_of(s.units, T * s.KB, P);
          const int64_t c1 = cta_of(s.units, (T + 1) * s.KB - 1, P);
          int ncontrib = 0;
          for (int64_t c = c0; c <= c1; ++c)
            ncontrib += cta_lo(s.units, c, P) < cta_lo(s.units, c + 1, P) ? 1 : 0;
          const int old = atomicAdd(&tile_cnt[T], 1);
          misc[2] = (old == ncontrib - 1) ? 1 : 0;
        }
        named_barrier(kBarPartial, kThreads);
        if (misc[2]) {
          __threadfence();
          const int64_t c0 = cta_of(s.units, T * s.KB, P);
          const int64_t c1 = cta_of(s.units, (T + 1) * s.KB - 1, P);
          float sum[4][2];
#pragma unroll
          for (int rg = 0; rg < 4; ++rg) sum[rg][0] = sum[rg][1] = 0.0f;
          for (int64_t c = c0; c <= c1; ++c) {
            const int64_t lo_c = cta_lo(s.units, c, P);
            if (lo_c >= cta_lo(s.units, c + 1, P)) continue;   // empty range: no partial
            const int sl_c = (T == lo_c / s.KB) ? 0 : 1;
            const float *src = partials + (c * 2 + sl_c) * kPartialFloats;
#pragma unroll
            for (int rg = 0; rg < 4; ++rg)
#pragma unroll
              for (int i = 0; i < 2; ++i) sum[rg][i] += __ldcg(src + (rg * 2 + i) * kThreads + t);
          }
          write_tile(sum, tg, tt, ro, s, y, q);
          if (t == 0) tile_cnt[T] = 0;
        }
        named_barrier(kBarPartial, kThreads);   // misc[2] is reused by the next split tile
      }
#pragma unroll
      for (int rg = 0; rg < 4; ++rg) acc[rg][0] = acc[rg][1] = 0.0f;
    }

    if (!has_next) break;
    u = un;
    T = Tn;
    kb0 = kbn;
    nblk = nbn;
    tg = tgn;
    tt = ttn;
    cur = nxt;
  }
}

int decode_grid() { return device_sm_count() * kCtasPerSm; }

int64_t decode_tile_cap(int64_t M, int32_t N, int32_t G, int32_t swiglu) {
  const int64_t nt = swiglu ? (N / 2 + 127) / 128 : (N + kRows - 1) / kRows;
  const int64_t groups = G < M ? G : M;
  return (M / kMT + groups) * nt;
}

}  // namespace

size_t decode_workspace_bytes(int64_t M, int32_t N, int32_t K, int32_t G, int32_t swiglu) {
  (void)K;
  const int64_t tile_cap = decode_tile_cap(M, N, G, swiglu);
  const size_t cnt_bytes = ((static_cast<size_t>(tile_cap) * 4 + 255) / 256) * 256;
  const size_t part_bytes = static_cast<size_t>(decode_grid()) * 2 * kPartialFloats * 4;
  return kWsHeaderBytes + cnt_bytes + part_bytes;
}

size_t decode_zero_prefix_bytes(int64_t M, int32_t N, int32_t G, int32_t swiglu) {
  const int64_t tile_cap = decode_tile_cap(M, N, G, swiglu);
  return kWsHeaderBytes + ((static_cast<size_t>(tile_cap) * 4 + 255) / 256) * 256;
}

cudaError_t launch_decode_gemm(const GemmArgs &a, cudaStream_t stream) {
  const int64_t tile_cap = decode_tile_cap(a.M, a.N, a.G, a.swiglu);
  const size_t cnt_bytes = ((static_cast<size_t>(tile_cap) * 4 + 255) / 256) * 256;
  char *ws = static_cast<char *>(a.workspace);
  WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
  int32_t *cnt = reinterpret_cast<int32_t *>(ws + kWsHeaderBytes);
  float *partials = reinterpret_cast<float *>(ws + kWsHeaderBytes + cnt_bytes);

  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    cudaError_t err = cudaFuncSetAttribute(decode_gemm_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  decode_gemm_kernel<<<decode_grid(), kThreads, kSmemBytes, stream>>>(
      a.x, a.w, a.absmax, a.sizes, a.expert_ids, a.G, a.M, a.N, a.K, a.E, a.swiglu, a.y, hdr, cnt,
      tile_cap, partials);
  return cudaGetLastError();
}

}  // namespace gnf4
