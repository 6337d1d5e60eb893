// dgrad.cu -- the gradient of the grouped NF4 GEMM with respect to its
// activations, on tensor cores:
//   dx[m][k] = sum_n dy[m][n] * w[e][n][k],  w = NF4[code] * absmax[e][n][k/64],
// e the expert of row m's group, accumulated in fp32, rounded once to bf16.
//
// Passage: "grouped-nf4-gemm" package page, header block ("Owns": the grouped
// packed GEMM and its dgrad); "Do not use this when" (the dgrad, like the
// GEMM, refuses tensors that are not on the device).
//
// The contraction runs over n, the weight rows, while two codes of one byte
// are two neighbouring k of one row. As MMA operands (mma.sync m16n8k16, fp32
// accumulation): D[k][m] = W^T[k][n] . B[n][m], B = dy'^T, 16 k x 8 rows x 16
// n per MMA.
//   A (W^T): lane (g, q) holds the rows k = 2 (4 g + t) and + 1 of m-tile t
//   (t = 0..3: one 64-element block of k is four m-tiles) and the columns n
//   = q, q + 4, q + 8, q + 12 of the warp's 16 rows. One 4-byte word of a
//   packed row is byte 4 g + t for t = 0..3, so each lane reads one word of
//   each of its 4 rows and decodes each byte through the per-lane replicated
//   byte -> (fp16 code value of even k, odd k) table; byte permutes then pair
//   the values of two rows for one k (the MMA's A register pairs run along
//   the contraction). Weight values enter as their fp16 rounding (relative
//   error at most 2^-12, as the decode GEMM without SwiGLU; kDgParts = 2
//   adds the remainder times 2^13, within 1e-7 relative of NF4[code]).
//   B: absmax varies with n, so it joins dy: dy'[m][n] = dy[m][n] *
//   absmax[n][block of the tile], exact in fp32, then scaled by a power of
//   two per (row m, 16 n of a warp) into [2^14, 2^15) and split into two
//   fp16 parts (hi and the remainder times 2^11). Each MMA result is
//   multiplied back by that power of two before it joins the fp32 sum.
//
// Work: tile = (batch of up to 8 rows of one group, 64 k); stage = 256 weight
// rows of a tile (8 KB of packed bytes, their 256 absmax values, the batch's
// dy over those 256 n). The tile-stages of all tiles are split into equal
// contiguous ranges, one per CTA (stream-K, as the decode GEMM); a tile cut by
// a range boundary is finished by the piece that counts last, which adds the
// pieces' fp32 partials in order. Inside a CTA: warp 16 issues the tensor
// copies (weights, dy), warp 17 copies absmax; consumer warp w (0..15) takes
// rows 16 w .. 16 w + 15 of every stage, and at a piece's end the 16 warps sum
// their results through shared memory (fixed order). Every wait is bounded.
#include <climits>

#include "launch.h"
#include "lut_mma.cuh"

namespace gnf4 {
namespace {

constexpr int kDgWarps = 16;                 // consumer warps
constexpr int kDgTmaWarp = kDgWarps;
constexpr int kDgScaleWarp = kDgWarps + 1;
constexpr int kDgThreads = (kDgWarps + 2) * 32;
constexpr int kDgStages = 6;
constexpr int kDgRows = 256;                 // weight rows (n) per stage
constexpr int kDgBatch = 8;                  // dy rows per tile (MMA N)
constexpr int kDgWStage = kDgRows * 32;      // 8 KB: 256 rows x 32 packed bytes (64 k)
constexpr int kDyPitch = kDgRows * 2 + 16;   // bytes per dy row in shared memory (padded)
constexpr int kDgYStage = kDgBatch * kDyPitch;
constexpr int kDgAStage = kDgRows * 4;       // absmax of the stage's rows
constexpr int kDgMaxG = GNF4_MAX_EXPERTS;
constexpr int kRedFloats = 16;               // per lane: 4 m-tiles x 4 accumulators
constexpr float kWLoInv = 1.0f / 8192.0f;    // weight remainders carried times 2^13
// fp16 parts per code value: one, the rounding of NF4[code] (relative error at
// most 2^-12, as the decode GEMM without SwiGLU), or two (within 1e-7)
constexpr int kDgParts = 1;
constexpr float kYLoInv = 1.0f / 2048.0f;    // dy' remainders carried times 2^11

// Shared memory, absolute shared-window addresses (the table at a multiple
// of 65536: one byte permute forms a lookup's address), as in the decode GEMM.
constexpr int kDgMinDyn = 1024;
constexpr int kDgDynBase = 2048;
constexpr int kDgWOff = kDgDynBase;
constexpr int kDgYOff = kDgWOff + kDgStages * kDgWStage;
constexpr int kDgAOff = kDgYOff + kDgStages * kDgYStage;
constexpr int kDgRowOffOff = kDgAOff + kDgStages * kDgAStage;       // int32 [G + 1]
constexpr int kDgBatchOff = kDgRowOffOff + (kDgMaxG + 1) * 4;       // int32 [G + 1]
constexpr int kDgGExpOff = kDgBatchOff + (kDgMaxG + 1) * 4;         // uint16 [G]
constexpr int kDgBarOff = (kDgGExpOff + kDgMaxG * 2 + 7) / 8 * 8;
// full[stages], empty[stages], red_full, red_empty
constexpr int kDgNumBars = 2 * kDgStages + 2;
constexpr int kDgMiscOff = kDgBarOff + kDgNumBars * 8;
constexpr int kDgLutOff = 131072;
constexpr int kDgRedOff = kDgLutOff + 256 * 256;                      // float [16 warps][16][32]
constexpr int kDgSmemEnd = kDgRedOff + kDgWarps * kRedFloats * 32 * 4;
constexpr int kDgSmemBytes = kDgSmemEnd - kDgMinDyn;
static_assert(kDgMiscOff + 8 * 4 <= kDgLutOff, "low region overlaps the table");
static_assert(kDgLutOff % 65536 == 0 && kDgBarOff % 8 == 0 && kDgWOff % 128 == 0 &&
              kDgYOff % 16 == 0 && kDgAOff % 16 == 0, "alignment");
static_assert(kDgSmemBytes + kDgDynBase - kDgMinDyn <= 227 * 1024, "fits one CTA per SM");

struct DgradParams {
  const uint16_t *dy;
  const float *absmax;
  const int32_t *sizes;
  const int32_t *expert_ids;
  int32_t G;
  int64_t M;
  int32_t N, K, E;
  uint16_t *dx;
  WsHeader *hdr;
  uint32_t *counters;   // [P][16 values]
  float *partials;      // [P][2][16 values][32 lanes]
};

__global__ void __launch_bounds__(kDgThreads, 1)
    dgrad_tc_kernel(const __grid_constant__ CUtensorMap wmap, const DgradParams prm) {
  extern __shared__ __align__(1024) char smem_raw[];
  const uint16_t *const dy = prm.dy;
  const float *const absmax = prm.absmax;
  const int32_t G = prm.G, N = prm.N, K = prm.K, E = prm.E;
  const int64_t M = prm.M;
  uint16_t *const dx = prm.dx;
  WsHeader *const hdr = prm.hdr;
  uint32_t *const counters = prm.counters;
  float *const partials = prm.partials;

  const uint32_t dyn0 = smem_u32(smem_raw);
  char *smem = smem_raw - dyn0;
  const uint32_t dyn_size = dynamic_smem_size();
  if (dyn0 > static_cast<uint32_t>(kDgDynBase) ||
      dyn0 + dyn_size < static_cast<uint32_t>(kDgSmemEnd)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      hdr->reserved[60] = dyn0;
      hdr->reserved[61] = dyn_size;
      report_error(hdr, GNF4_DEVERR_CAPACITY, dyn0);
    }
    return;
  }
  int *row_off = reinterpret_cast<int *>(smem + kDgRowOffOff);
  int *batch_start = reinterpret_cast<int *>(smem + kDgBatchOff);
  uint16_t *gexp = reinterpret_cast<uint16_t *>(smem + kDgGExpOff);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kDgBarOff);
  uint64_t *empty = full + kDgStages;
  uint64_t *red_full = empty + kDgStages;
  uint64_t *red_empty = red_full + 1;
  int *misc = reinterpret_cast<int *>(smem + kDgMiscOff);
  volatile int *abort_flag = &misc[1];
  __shared__ int s_tot;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();
  const int KB = K / 64;
  const int KC = (N + kDgRows - 1) / kDgRows;   // stages per tile

  if (tid == 0) {
    misc[0] = 0;
    misc[1] = 0;
    for (int s = 0; s < kDgStages; ++s) {
      mbar_init(&full[s], 32 + 1);   // the scale warp's 32 cp.async arrivals + the byte count
      mbar_init(&empty[s], kDgWarps);
    }
    mbar_init(red_full, kDgWarps);
    mbar_init(red_empty, kDgWarps);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tensormap(&wmap);
  }
  // table: row b, lane slot l: fp16 pair (NF4[b >> 4], NF4[b & 15]) (low
  // half = even k) at l * 4, the pair of remainders at 128 + l * 4
  for (int i = tid; i < 256 * 8; i += kDgThreads) {
    const int b = i >> 3, part = i & 7;
    const uint32_t hp = code_hi(b >> 4) | (code_hi(b & 15) << 16);
    uint4 *dst = reinterpret_cast<uint4 *>(smem + kDgLutOff + b * 256);
    dst[part] = make_uint4(hp, hp, hp, hp);
    if (kDgParts == 2) {
      const uint32_t lp = code_lo(b >> 4) | (code_lo(b & 15) << 16);
      dst[8 + part] = make_uint4(lp, lp, lp, lp);
    }
  }

  pdl_wait();

  // ---- group table (warp 0), validated on the device
  if (warp == 0) {
    const int per = (G + 31) / 32;
    const int g0 = min(G, lane * per), g1 = min(G, g0 + per);
    int64_t my_rows = 0, my_batches = 0;
    int bad = 0;
    for (int g = g0; g < g1; ++g) {
      const int sz = prm.sizes[g];
      const int e = prm.expert_ids[g];
      if (sz < 0) bad |= GNF4_DEVERR_SIZES;
      if (sz > 0 && (e < 0 || e >= E)) bad |= GNF4_DEVERR_EXPERT;
      gexp[g] = static_cast<uint16_t>(e);
      row_off[g] = sz;
      my_rows += max(sz, 0);
      my_batches += sz > 0 ? (sz + kDgBatch - 1) / kDgBatch : 0;
    }
    int64_t vr = my_rows, vb = my_batches;
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
      c += sz > 0 ? (sz + kDgBatch - 1) / kDgBatch : 0;
    }
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (lane == 0) {
      batch_start[G] = static_cast<int>(tot_b);
      row_off[G] = static_cast<int>(tot_r);
      if (tot_r != M) bad |= GNF4_DEVERR_SIZES;
      s_tot = static_cast<int>(tot_b);
      misc[0] = bad;
    }
  }
  __syncthreads();
  if (misc[0]) {
    if (blockIdx.x == 0 && tid == 0) report_error(hdr, static_cast<uint32_t>(misc[0]), 0);
    return;
  }
  // tiles: batch-major, 64-element block of k minor
  const int64_t T = static_cast<int64_t>(s_tot) * KB;
  const int64_t W = T * KC;
  const int64_t P = min(static_cast<int64_t>(gridDim.x), W);
  if (static_cast<int64_t>(blockIdx.x) >= P) return;
  const int64_t s_lo = range_lo(W, P, blockIdx.x), s_hi = range_lo(W, P, blockIdx.x + 1);

  // batch of tile t: first row, valid rows, expert
  auto tile_batch = [&](int64_t t, int64_t *row0, int *mrows, int *e) {
    const int64_t bt = div_fast(t, KB);
    int lo = 0, hi = G;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (batch_start[mid] <= bt) lo = mid; else hi = mid;
    }
    const int lb = static_cast<int>(bt) - batch_start[lo];
    *row0 = static_cast<int64_t>(row_off[lo]) + static_cast<int64_t>(lb) * kDgBatch;
    *mrows = min(kDgBatch, row_off[lo + 1] - row_off[lo] - lb * kDgBatch);
    *e = gexp[lo];
  };

  if (warp >= kDgTmaWarp) {
    // ------------------------------------------------------------ producers
    const bool scale_warp = warp == kDgScaleWarp;
    uint32_t it = 0;
    bool ok = true;
    for (int64_t s = s_lo; s < s_hi && ok;) {
      const int64_t t = div_fast(s, KC);
      const int k0 = static_cast<int>(s - t * KC);
      const int k1 = static_cast<int>(min(static_cast<int64_t>(KC), k0 + (s_hi - s)));
      int64_t row0;
      int mrows, e;
      tile_batch(t, &row0, &mrows, &e);
      const int kb = static_cast<int>(t - div_fast(t, KB) * KB);
      const int64_t ebase = static_cast<int64_t>(e) * N;
      for (int kc = k0; kc < k1; ++kc, ++it) {
        const int st = static_cast<int>(it % kDgStages);
        const uint32_t ph = (it / kDgStages) & 1u;
        if (!warp_wait_one(&empty[st], ph ^ 1u, abort_flag, hdr, kTimeoutNs)) { ok = false; break; }
        const int n0 = kc * kDgRows;
        if (scale_warp) {
          // absmax of the stage's 256 rows at the tile's block (rows past
          // the expert: zeros, so their dy' is 0), and the batch's dy over
          // those 256 n as 16-byte copies into rows of kDyPitch bytes (rows
          // past the batch or M, and columns past N: zeros)
          const uint32_t as = smem_u32(smem + kDgAOff + st * kDgAStage);
#pragma unroll
          for (int j = 0; j < kDgRows / 32; ++j) {
            const int n = n0 + lane + 32 * j;
            const bool v = n < N;
            cp_async4(as + (lane + 32 * j) * 4, v ? absmax + (ebase + n) * KB + kb : absmax,
                      v ? 4u : 0u);
          }
          const uint32_t ys = smem_u32(smem + kDgYOff + st * kDgYStage);
#pragma unroll
          for (int j = 0; j < kDgBatch; ++j) {   // lane: 8-element chunk `lane` of row j
            const int n = n0 + 8 * lane;
            const bool v = j < mrows && n < N;
            cp_async16(ys + j * kDyPitch + lane * 16, v ? dy + (row0 + j) * N + n : dy,
                       v ? 16u : 0u);
          }
          cp_async_arrive_noinc(&full[st]);
        } else if (lane == 0) {
          mbar_arrive_expect_tx(&full[st], kDgWStage);
          // 256 rows x 32 packed bytes (the tile's 64 k), rows past the
          // stack zero-filled
          tma_load_2d(smem + kDgWOff + st * kDgWStage, &wmap, kb * 32,
                      static_cast<int>(ebase + n0), &full[st]);
        }
      }
      s += k1 - k0;
    }
    if (scale_warp) {
      cp_async_wait_all();
    } else if (lane == 0) {
      const uint32_t n = it < static_cast<uint32_t>(kDgStages) ? it : static_cast<uint32_t>(kDgStages);
      for (uint32_t d = 0; d < n; ++d) {
        const uint32_t gg = it - 1 - d;
        drain_wait(&full[gg % kDgStages], (gg / kDgStages) & 1u);
      }
    }
    return;
  }

  // --------------------------------------------------------------- consumers
  const int g = lane >> 2, q = lane & 3;
  const uint32_t lutlane = static_cast<uint32_t>(kDgLutOff) | (static_cast<uint32_t>(lane) * 4u);
  // this lane's rows within the stage: 16 w + q + 4 c, c = 0..3 (MMA
  // contraction positions 2q, 2q + 1, 2q + 8, 2q + 9); bank-conflict-free:
  // row pitch 32 bytes, word g of rows differing in q lands in 8 q + g
  const int nrow = 16 * warp + q;
  const int woff = nrow * 32 + 4 * g;
  float *red = reinterpret_cast<float *>(smem + kDgRedOff);
  uint32_t it = 0, ep = 0;
  for (int64_t s = s_lo; s < s_hi;) {
    const int64_t t = div_fast(s, KC);
    const int k0 = static_cast<int>(s - t * KC);
    const int k1 = static_cast<int>(min(static_cast<int64_t>(KC), k0 + (s_hi - s)));
    // D fragments of the 4 m-tiles: [t][0] k = 2 (4 g + t), row 2q; [1] same
    // k, row 2q + 1; [2] k + 1, row 2q; [3] k + 1, row 2q + 1
    float acc[4][4];
#pragma unroll
    for (int t4 = 0; t4 < 4; ++t4)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[t4][i] = 0.0f;
    for (int kc = k0; kc < k1; ++kc, ++it) {
      const int st = static_cast<int>(it % kDgStages);
      const uint32_t ph = (it / kDgStages) & 1u;
      if (!warp_wait_all(&full[st], ph, abort_flag, hdr, kTimeoutNs)) return;
      const char *wst = smem + kDgWOff + st * kDgWStage;
      const char *yst = smem + kDgYOff + st * kDgYStage;
      const float *ast = reinterpret_cast<const float *>(smem + kDgAOff + st * kDgAStage);
      // B: dy' of row g at this lane's 4 rows, in fp32
      float v[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t d16 = *reinterpret_cast<const uint16_t *>(yst + g * kDyPitch + (nrow + 4 * c) * 2);
        v[c] = __uint_as_float(d16 << 16) * ast[nrow + 4 * c];
      }
      // power of two putting row g's largest |dy'| over the warp's 16 rows in
      // [2^14, 2^15) (the four lanes q of row g hold them)
      float mx = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const int eb = static_cast<int>((__float_as_uint(mx) >> 23) & 0xFFu);
      int S = 0;
      if (mx > 0.0f && eb < 255) S = 14 - (eb == 0 ? -126 : eb - 127);
      S = S > 126 ? 126 : (S < -126 ? -126 : S);
      const float sc = __uint_as_float(static_cast<uint32_t>(S + 127) << 23);
      uint32_t bh[2], bl[2];   // b0 = rows (q, q + 4), b1 = rows (q + 8, q + 12)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float u0 = v[2 * j] * sc, u1 = v[2 * j + 1] * sc;
        const __half2 h = __floats2half2_rn(u0, u1);
        const float2 hf = __half22float2(h);
        const __half2 l = __floats2half2_rn((u0 - hf.x) * 2048.0f, (u1 - hf.y) * 2048.0f);
        bh[j] = *reinterpret_cast<const uint32_t *>(&h);
        bl[j] = *reinterpret_cast<const uint32_t *>(&l);
      }
      // 2^-S of the D columns: rows 2q and 2q + 1 (their S sits in lanes 4 (2q) + x)
      const float inv = __uint_as_float(static_cast<uint32_t>(127 - S) << 23);
      const float inv0 = __shfl_sync(0xffffffffu, inv, 8 * q);
      const float inv1 = __shfl_sync(0xffffffffu, inv, 8 * q + 4);
      // A: one word (bytes 4 g .. 4 g + 3 = m-tiles 0..3) of each of the 4 rows
      const uint32_t wa = *reinterpret_cast<const uint32_t *>(wst + woff);
      const uint32_t wb = *reinterpret_cast<const uint32_t *>(wst + woff + 4 * 32);
      const uint32_t wc = *reinterpret_cast<const uint32_t *>(wst + woff + 8 * 32);
      const uint32_t wd = *reinterpret_cast<const uint32_t *>(wst + woff + 12 * 32);
      uint32_t ha[4], la[4], hb[4], lb[4], hc[4], lc[4], hd[4], ld[4];
      decode_word<kDgParts>(lutlane, wa, ha, la);
      decode_word<kDgParts>(lutlane, wb, hb, lb);
      decode_word<kDgParts>(lutlane, wc, hc, lc);
      decode_word<kDgParts>(lutlane, wd, hd, ld);
#pragma unroll
      for (int t4 = 0; t4 < 4; ++t4) {
        // pair two rows' values of one k: a0/a2 even k (MMA row g), a1/a3 odd
        const uint32_t a0 = prmt(ha[t4], hb[t4], 0x5410u), a1 = prmt(ha[t4], hb[t4], 0x7632u);
        const uint32_t a2 = prmt(hc[t4], hd[t4], 0x5410u), a3 = prmt(hc[t4], hd[t4], 0x7632u);
        float chh[4], chl[4];
        mma_f16_z(chh, a0, a1, a2, a3, bh[0], bh[1]);   // weights x hi dy'
        mma_f16_z(chl, a0, a1, a2, a3, bl[0], bl[1]);   // weights x dy' remainders
        float sum[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) sum[i] = fmaf(chl[i], kYLoInv, chh[i]);
        if (kDgParts == 2) {
          const uint32_t r0 = prmt(la[t4], lb[t4], 0x5410u), r1 = prmt(la[t4], lb[t4], 0x7632u);
          const uint32_t r2 = prmt(lc[t4], ld[t4], 0x5410u), r3 = prmt(lc[t4], ld[t4], 0x7632u);
          float clh[4];
          mma_f16_z(clh, r0, r1, r2, r3, bh[0], bh[1]);   // weight remainders x hi dy'
#pragma unroll
          for (int i = 0; i < 4; ++i) sum[i] = fmaf(clh[i], kWLoInv, sum[i]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[t4][i] = fmaf(sum[i], (i & 1) ? inv1 : inv0, acc[t4][i]);
      }
      __syncwarp();
      mbar_arrive_elect(&empty[st]);
    }
    // ---- piece end: the 16 warps' sums through shared memory, fixed order;
    //      warp w then owns value w (m-tile w / 4, accumulator w % 4) of
    //      every lane
    if (ep > 0 && !warp_wait_one(red_empty, (ep - 1) & 1u, abort_flag, hdr, kTimeoutNs)) return;
#pragma unroll
    for (int t4 = 0; t4 < 4; ++t4)
#pragma unroll
      for (int i = 0; i < 4; ++i) red[(warp * kRedFloats + t4 * 4 + i) * 32 + lane] = acc[t4][i];
    __syncwarp();
    mbar_arrive_elect(red_full);
    if (!warp_wait_one(red_full, ep & 1u, abort_flag, hdr, kTimeoutNs)) return;
    float val = 0.0f;
    for (int w2 = 0; w2 < kDgWarps; ++w2) val += red[(w2 * kRedFloats + warp) * 32 + lane];
    __syncwarp();
    mbar_arrive_elect(red_empty);
    ++ep;
    // dx element of (value warp, lane): m-tile t4 = warp / 4, i = warp % 4
    int64_t row0;
    int mrows, e;
    tile_batch(t, &row0, &mrows, &e);
    const int t4 = warp >> 2, i = warp & 3;
    const int kk = static_cast<int>(t - div_fast(t, KB) * KB) * 64 + 2 * (4 * g + t4) + (i >> 1);
    const int m = 2 * q + (i & 1);
    const int64_t b_first = cta_of(W, P, t * KC), b_last = cta_of(W, P, t * KC + KC - 1);
    if (b_first != b_last) {
      // a piece of a cut tile: leave value `warp` of every lane in this
      // CTA's slot (first or last tile of its range), count it; the piece
      // that counts last adds all pieces in order and stores
      auto slot = [&](int64_t c) -> float * {
        const int64_t which = div_fast(range_lo(W, P, c), KC) == t ? 0 : 1;
        return partials + ((c * 2 + which) * kRedFloats + warp) * 32;
      };
      slot(blockIdx.x)[lane] = val;
      __syncwarp();
      uint32_t old = 0;
      uint32_t *cnt = counters + b_first * kRedFloats + warp;
      if (lane == 0) {
        __threadfence();
        old = atomic_add_acq_rel(cnt, 1u);
      }
      old = __shfl_sync(0xffffffffu, old, 0);
      if (old != static_cast<uint32_t>(b_last - b_first)) {
        s += k1 - k0;
        continue;
      }
      __syncwarp();
      val = 0.0f;
      for (int64_t c = b_first; c <= b_last; ++c) val += __ldcg(slot(c) + lane);
      if (lane == 0) *cnt = 0u;   // reusable by the next launch
    }
    if (m < mrows) {
      const __nv_bfloat16 b = __float2bfloat16_rn(val);
      dx[(row0 + m) * K + kk] = *reinterpret_cast<const uint16_t *>(&b);
    }
    s += k1 - k0;
  }
}

}  // namespace

size_t dgrad_zero_prefix_bytes() {
  const size_t P = static_cast<size_t>(device_sm_count());
  return kWsHeaderBytes + (P * kRedFloats * 4 + 255) / 256 * 256;
}

size_t dgrad_workspace_bytes() {
  const size_t P = static_cast<size_t>(device_sm_count());
  return dgrad_zero_prefix_bytes() + P * 2 * kRedFloats * 32 * sizeof(float);
}

cudaError_t launch_grouped_dgrad(const uint16_t *dy, const uint8_t *w, const float *absmax,
                                 const int32_t *sizes, const int32_t *expert_ids, int32_t G,
                                 int64_t M, int32_t N, int32_t K, int32_t E, uint16_t *dx,
                                 WsHeader *hdr, cudaStream_t stream) {
  if (N % 8 != 0 || static_cast<int64_t>(E) * N + kDgRows >= INT_MAX) return cudaErrorNotSupported;
  // packed weights as [E*N rows][K/2 bytes], boxes of 256 rows x 32 bytes.
  // Each 32-byte row piece is fetched into L2 as 64 bytes: the neighbouring
  // 64-element block is the next tile's, read a tile (KC stages) later,
  // while 256-byte fetches were mostly evicted before their other 7 blocks
  // were used (5x the weight bytes from DRAM).
  CUtensorMap wmap;
  if (!encode_tensor_map_2d(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, w,
                            static_cast<uint64_t>(K / 2),
                            static_cast<uint64_t>(E) * static_cast<uint64_t>(N),
                            static_cast<uint64_t>(K / 2), 32, kDgRows,
                            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_64B))
    return cudaErrorInvalidValue;
  DgradParams prm;
  prm.dy = dy;
  prm.absmax = absmax;
  prm.sizes = sizes;
  prm.expert_ids = expert_ids;
  prm.G = G; prm.M = M; prm.N = N; prm.K = K; prm.E = E;
  prm.dx = dx;
  prm.hdr = hdr;
  char *ws = reinterpret_cast<char *>(hdr);
  prm.counters = reinterpret_cast<uint32_t *>(ws + kWsHeaderBytes);
  prm.partials = reinterpret_cast<float *>(ws + dgrad_zero_prefix_bytes());
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    const cudaError_t err = cudaFuncSetAttribute(
        dgrad_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDgSmemBytes);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  return launch_pdl(dgrad_tc_kernel, dim3(device_sm_count()), dim3(kDgThreads),
                    static_cast<size_t>(kDgSmemBytes), stream, wmap, prm);
}

}  // namespace gnf4
