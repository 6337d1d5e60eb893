// decode_gemm.cu -- decode-regime grouped NF4 GEMM (few rows per expert).
//
// Passage: "grouped-nf4-gemm -- single-launch W4A16 GEMM over fused NF4 MoE
// expert stacks", opening section (one launch for all active experts, LUT
// decode to fp32 in registers, blockwise fp32 absmax, fp32 accumulation, bf16
// epilogue, no bf16 weight copy) and "Status / roadmap" (split-K for starved
// grids). At a handful of rows per expert this GEMM streams every touched
// weight byte exactly once and is bound by HBM bandwidth.
//
// Work decomposition
//   tile   = (row chunk, column tile): up to kMT activation rows of one group
//            times 256 weight rows of that group's expert (with SwiGLU: 128
//            gate rows j..j+127 and the matching 128 up rows N/2+j.., so the
//            epilogue can pair them inside the CTA).
//   unit   = one 64-element absmax block of K for a whole tile.
//   Stream-K: the tiles' units are laid end to end and every CTA (one per SM)
//   takes an equal contiguous range. A tile covered by one CTA is finished in
//   registers; a tile split between CTAs is finished by whichever contributor
//   arrives last (per-tile counter in the workspace), which sums the fp32
//   partials in CTA order, so the result does not depend on arrival order.
//   The tile list is derived on the device from (sizes, expert_ids): the
//   host never learns which experts are active (no sync, graph-capturable).
//
// Inside a CTA (8 consumer warps + 1 producer warp)
//   consumer thread t owns weight row t of the tile. It streams its row with
//   32-byte loads straight from HBM into registers (one absmax block per
//   load), one step ahead of use. Each byte (two codes) is decoded with ONE
//   shared-memory load from a 256-entry table of fp32 pairs
//   (NF4[hi], NF4[lo]), replicated per lane so the warp never hits a bank
//   conflict; the byte-to-address step is a single byte permute. The pair
//   multiplies the matching x pair with a packed fp32x2 FMA. After each block
//   the fp32 partial is scaled by that block's absmax and accumulated.
//   producer warp: converts the tile's activation rows for the next steps
//   from bf16 to fp32 into a shared ring (mbarrier handshake); consumers read
//   them as warp-wide broadcasts.
#include "launch.h"

namespace gnf4 {
namespace {

constexpr int kRows = 256;            // weight rows per tile = consumer threads
constexpr int kConsumers = kRows;
constexpr int kThreads = kConsumers + 32;
constexpr int kMT = 8;                // activation rows per tile (row chunk)
constexpr int kStepBlocks = 4;        // 64-element blocks per step (256 k)
constexpr int kStepK = kStepBlocks * 64;
constexpr int kStages = 3;            // activation ring depth
constexpr int kMaxG = GNF4_MAX_EXPERTS;

// Dynamic shared memory layout (bytes).
constexpr int kLutBytes = 256 * 32 * 8;                       // [byte][lane] float2
constexpr int kXsOff = kLutBytes;
constexpr int kXsBytes = kStages * kMT * kStepK * 4;
constexpr int kChunkStartOff = kXsOff + kXsBytes;             // int[kMaxG + 1]
constexpr int kRowOffOff = kChunkStartOff + (kMaxG + 4) * 4;  // int[kMaxG]
constexpr int kGSizeOff = kRowOffOff + kMaxG * 4;             // int[kMaxG]
constexpr int kGExpOff = kGSizeOff + kMaxG * 4;               // int[kMaxG]
constexpr int kExOff = kGExpOff + kMaxG * 4;                  // float[kMT][128]
constexpr int kBarOff = kExOff + kMT * 128 * 4;               // uint64[2*kStages]
constexpr int kMiscOff = kBarOff + 2 * kStages * 8;           // int[16]
constexpr int kSmemBytes = kMiscOff + 16 * 4;

constexpr int64_t kTimeoutNs = 2000000000LL;   // 2 s per wait, then give up

struct Sched {
  int32_t G, N, K, E, swiglu;
  int32_t KB;        // 64-element blocks per row
  int32_t NT;        // column tiles per row chunk
  int64_t units;     // total units
  int64_t lo, hi;    // this CTA's unit range
};

struct Tile {
  int64_t row0;      // first activation row
  int32_t mrows;     // activation rows (1..kMT)
  int32_t j;         // column tile
  int64_t wrow;      // this thread's global weight row (e*N + n)
  int32_t col;       // output column of this thread (or -1 if not an output column)
  bool valid;        // this thread's weight row exists
};

// Blocks in a step: at most kStepBlocks, never past the row end or range end.
__device__ __forceinline__ int step_blocks(int64_t left_in_row, int64_t left_in_range) {
  int64_t n = left_in_row < left_in_range ? left_in_row : left_in_range;
  return static_cast<int>(n < kStepBlocks ? n : kStepBlocks);
}

__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait; after the first timeout in this CTA every later wait gives
// up at once, so a broken pipeline ends quickly instead of hanging.
__device__ __forceinline__ void wait_or_flag(uint64_t *bar, uint32_t parity, int *timed_out,
                                             WsHeader *hdr) {
  if (mbar_try_wait(bar, parity)) return;
  if (*reinterpret_cast<volatile int *>(timed_out)) return;
  const uint64_t t0 = global_timer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return;
    if (global_timer() - t0 > static_cast<uint64_t>(kTimeoutNs)) {
      *reinterpret_cast<volatile int *>(timed_out) = 1;
      report_error(hdr, GNF4_DEVERR_TIMEOUT, blockIdx.x);
      return;
    }
  }
}

__device__ __forceinline__ Tile tile_info(int64_t T, const Sched &s, const int *chunk_start,
                                          const int *row_off, const int *gsize, const int *gexp,
                                          int t) {
  Tile ti;
  const int64_t c = T / s.NT;
  ti.j = static_cast<int32_t>(T - c * s.NT);
  // group g with chunk_start[g] <= c < chunk_start[g+1]
  int lo = 0, hi = s.G;   // invariant: chunk_start[lo] <= c < chunk_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (chunk_start[mid] <= c) lo = mid; else hi = mid;
  }
  const int g = lo;
  const int32_t local = static_cast<int32_t>(c - chunk_start[g]);
  ti.row0 = static_cast<int64_t>(row_off[g]) + static_cast<int64_t>(local) * kMT;
  ti.mrows = min(kMT, gsize[g] - local * kMT);
  const int e = gexp[g];
  int n;
  if (s.swiglu) {
    const int h = s.N / 2;
    const int jj = ti.j * 128 + (t & 127);
    ti.valid = jj < h;
    n = (t < 128) ? jj : h + jj;
    ti.col = (t < 128 && ti.valid) ? jj : -1;
  } else {
    n = ti.j * kRows + t;
    ti.valid = n < s.N;
    ti.col = ti.valid ? n : -1;
  }
  ti.wrow = static_cast<int64_t>(e) * s.N + (ti.valid ? n : 0);
  return ti;
}

// Load this thread's weight bytes and scales for blocks [kb0, kb0+nblk).
__device__ __forceinline__ void load_step(const uint8_t *__restrict__ w,
                                          const float *__restrict__ absmax, const Tile &ti,
                                          const Sched &s, int kb0, int nblk,
                                          uint32_t (&wq)[kStepBlocks][8], float (&aq)[kStepBlocks]) {
  const uint8_t *wr = w + ti.wrow * static_cast<int64_t>(s.K / 2);
  const float *ar = absmax + ti.wrow * static_cast<int64_t>(s.KB);
#pragma unroll
  for (int b = 0; b < kStepBlocks; ++b) {
    if (ti.valid && b < nblk) {
      ldg256_stream(wr + static_cast<int64_t>(kb0 + b) * 32, wq[b]);
      aq[b] = __ldg(ar + kb0 + b);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) wq[b][i] = 0x77777777u;   // codes 7 = 0.0
      aq[b] = 0.0f;
    }
  }
}

// acc[m] += sum over the step's blocks of absmax_b * sum_k x[m,k] * NF4[code_k]
template <int MR>
__device__ __forceinline__ void compute_step(const uint32_t (&wq)[kStepBlocks][8],
                                             const float (&aq)[kStepBlocks], int nblk,
                                             const float *__restrict__ xs, const char *lut,
                                             uint32_t lane8, float (&acc)[kMT]) {
#pragma unroll
  for (int b = 0; b < kStepBlocks; ++b) {
    if (b < nblk) {
      float2 part[MR];
#pragma unroll
      for (int m = 0; m < MR; ++m) part[m] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t word = wq[b][q];
        float2 wv[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          // byte p of the word -> (byte << 8) | lane*8 : offset of this lane's copy
          const uint32_t off = __byte_perm(word, lane8, 0x5504u | (p << 4));
          wv[p] = *reinterpret_cast<const float2 *>(lut + off);
        }
#pragma unroll
        for (int m = 0; m < MR; ++m) {
          const float4 *xp = reinterpret_cast<const float4 *>(xs + m * kStepK + b * 64 + q * 8);
          const float4 xa = xp[0], xb = xp[1];
          part[m] = __ffma2_rn(wv[0], make_float2(xa.x, xa.y), part[m]);
          part[m] = __ffma2_rn(wv[1], make_float2(xa.z, xa.w), part[m]);
          part[m] = __ffma2_rn(wv[2], make_float2(xb.x, xb.y), part[m]);
          part[m] = __ffma2_rn(wv[3], make_float2(xb.z, xb.w), part[m]);
        }
      }
#pragma unroll
      for (int m = 0; m < MR; ++m) acc[m] = fmaf(aq[b], part[m].x + part[m].y, acc[m]);
    }
  }
}

__device__ __forceinline__ void compute_dispatch(int mrows, const uint32_t (&wq)[kStepBlocks][8],
                                                 const float (&aq)[kStepBlocks], int nblk,
                                                 const float *xs, const char *lut, uint32_t lane8,
                                                 float (&acc)[kMT]) {
  switch (mrows) {
    case 1: compute_step<1>(wq, aq, nblk, xs, lut, lane8, acc); break;
    case 2: compute_step<2>(wq, aq, nblk, xs, lut, lane8, acc); break;
    case 3: compute_step<3>(wq, aq, nblk, xs, lut, lane8, acc); break;
    case 4: compute_step<4>(wq, aq, nblk, xs, lut, lane8, acc); break;
    case 5: compute_step<5>(wq, aq, nblk, xs, lut, lane8, acc); break;
    case 6: compute_step<6>(wq, aq, nblk, xs, lut, lane8, acc); break;
    case 7: compute_step<7>(wq, aq, nblk, xs, lut, lane8, acc); break;
    default: compute_step<8>(wq, aq, nblk, xs, lut, lane8, acc); break;
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

// Epilogue for finished accumulators (one activation row set of the tile).
__device__ __forceinline__ void write_tile(const float (&v)[kMT], const Tile &ti, const Sched &s,
                                           uint16_t *__restrict__ y, float *ex, int t) {
  if (!s.swiglu) {
    if (ti.col >= 0) {
#pragma unroll
      for (int m = 0; m < kMT; ++m)
        if (m < ti.mrows) {
          const __nv_bfloat16 b = __float2bfloat16_rn(v[m]);
          y[(ti.row0 + m) * s.N + ti.col] = *reinterpret_cast<const uint16_t *>(&b);
        }
    }
  } else {
    if (t >= 128) {
#pragma unroll
      for (int m = 0; m < kMT; ++m) ex[m * 128 + (t - 128)] = v[m];
    }
    named_barrier(2, kConsumers);
    if (ti.col >= 0) {
      const int h = s.N / 2;
#pragma unroll
      for (int m = 0; m < kMT; ++m)
        if (m < ti.mrows) {
          const float r = silu(v[m]) * ex[m * 128 + t];
          const __nv_bfloat16 b = __float2bfloat16_rn(r);
          y[(ti.row0 + m) * h + ti.col] = *reinterpret_cast<const uint16_t *>(&b);
        }
    }
    named_barrier(2, kConsumers);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    decode_gemm_kernel(const uint16_t *__restrict__ x, const uint8_t *__restrict__ w,
                       const float *__restrict__ absmax, const int32_t *__restrict__ sizes,
                       const int32_t *__restrict__ expert_ids, int32_t G, int64_t M, int32_t N,
                       int32_t K, int32_t E, int32_t swiglu, uint16_t *__restrict__ y,
                       WsHeader *hdr, int32_t *__restrict__ tile_cnt, int64_t tile_cap,
                       float *__restrict__ partials) {
  extern __shared__ __align__(1024) char smem[];
  float *xs = reinterpret_cast<float *>(smem + kXsOff);
  int *chunk_start = reinterpret_cast<int *>(smem + kChunkStartOff);
  int *row_off = reinterpret_cast<int *>(smem + kRowOffOff);
  int *gsize = reinterpret_cast<int *>(smem + kGSizeOff);
  int *gexp = reinterpret_cast<int *>(smem + kGExpOff);
  float *ex = reinterpret_cast<float *>(smem + kExOff);
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + kBarOff);
  uint64_t *empty_bar = full_bar + kStages;
  int *misc = reinterpret_cast<int *>(smem + kMiscOff);
  // misc[0]: error bits, misc[1]: timed out, misc[2]: last-arriver flag,
  // misc[3]: warp sums scratch base not used, misc[4..]: scan scratch

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  // ---- 1. decode table: entry (byte b, lane l) = (NF4[b >> 4], NF4[b & 15])
  for (int i = tid; i < 256 * 32; i += kThreads) {
    const int b = i >> 5;
    reinterpret_cast<float2 *>(smem)[i] = make_float2(nf4_value(b >> 4), nf4_value(b & 15));
  }
  if (tid == 0) {
    misc[0] = 0;
    misc[1] = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full_bar[i], 32);
      mbar_init(&empty_bar[i], kConsumers / 32);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // ---- 2. group table from (sizes, expert_ids), validated on the device
  // Each thread takes a contiguous run of groups; two-level exclusive scan of
  // the row counts and the row-chunk counts.
  __shared__ int s_wsum[2][kThreads / 32];
  const int per = (G + kThreads - 1) / kThreads;
  const int g0 = min(G, tid * per), g1 = min(G, g0 + per);
  int my_rows = 0, my_chunks = 0, bad = 0;
  for (int g = g0; g < g1; ++g) {
    const int sz = sizes[g];
    const int e = expert_ids[g];
    if (sz < 0) bad |= GNF4_DEVERR_SIZES;
    if (sz > 0 && (e < 0 || e >= E)) bad |= GNF4_DEVERR_EXPERT;
    gsize[g] = sz;
    gexp[g] = e;
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
    for (int g = g0; g < g1; ++g) {
      row_off[g] = r;
      chunk_start[g] = c;
      const int sz = max(gsize[g], 0);
      r += sz;
      c += sz > 0 ? (sz + kMT - 1) / kMT : 0;
    }
    if (tid == 0) chunk_start[G] = tot_c;
  }
  if (tid == 0 && static_cast<int64_t>(tot_r) != M) atomicOr(&misc[0], GNF4_DEVERR_SIZES);
  __syncthreads();

  Sched s;
  s.G = G; s.N = N; s.K = K; s.E = E; s.swiglu = swiglu;
  s.KB = K / 64;
  s.NT = swiglu ? (N / 2 + 127) / 128 : (N + kRows - 1) / kRows;
  const int64_t tiles = static_cast<int64_t>(tot_c) * s.NT;
  int errbits = misc[0];
  if (errbits == 0 && tiles > tile_cap) errbits = GNF4_DEVERR_CAPACITY;
  if (errbits) {
    if (blockIdx.x == 0 && tid == 0) report_error(hdr, static_cast<uint32_t>(errbits), 0);
    return;
  }
  s.units = tiles * s.KB;
  const int64_t P = gridDim.x;
  s.lo = cta_lo(s.units, blockIdx.x, P);
  s.hi = cta_lo(s.units, blockIdx.x + 1, P);
  if (s.lo >= s.hi) return;

  int *timed_out = &misc[1];

  if (warp == kConsumers / 32) {
    // ---------------------------------------------------------- producer
    int stage = 0;
    uint32_t phase = 0;
    int64_t curT = -1;
    Tile ti{};
    for (int64_t u = s.lo; u < s.hi;) {
      const int64_t T = u / s.KB;
      const int kb0 = static_cast<int>(u - T * s.KB);
      const int nblk = static_cast<int>(step_blocks(s.KB - kb0, s.hi - u));
      if (T != curT) { ti = tile_info(T, s, chunk_start, row_off, gsize, gexp, 0); curT = T; }
      wait_or_flag(&empty_bar[stage], phase ^ 1u, timed_out, hdr);
      float *dst = xs + stage * kMT * kStepK;
      const int k = kb0 * 64 + lane * 8;
      const bool in = lane * 8 < nblk * 64;
      for (int m = 0; m < ti.mrows; ++m) {
        float4 lo4 = make_float4(0.f, 0.f, 0.f, 0.f), hi4 = lo4;
        if (in) {
          const uint4 v = *reinterpret_cast<const uint4 *>(x + (ti.row0 + m) * K + k);
          lo4 = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                            __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
          hi4 = make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xFFFF0000u),
                            __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xFFFF0000u));
        }
        float4 *d = reinterpret_cast<float4 *>(dst + m * kStepK + lane * 8);
        d[0] = lo4;
        d[1] = hi4;
      }
      mbar_arrive(&full_bar[stage]);
      if (++stage == kStages) { stage = 0; phase ^= 1u; }
      u += nblk;
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int t = tid;
  const uint32_t lane8 = static_cast<uint32_t>(lane) * 8u;
  const char *lut = smem;
  float acc[kMT];
#pragma unroll
  for (int m = 0; m < kMT; ++m) acc[m] = 0.0f;

  int stage = 0;
  uint32_t phase = 0;
  int64_t u = s.lo;
  int64_t T = u / s.KB;
  int kb0 = static_cast<int>(u - T * s.KB);
  int nblk = static_cast<int>(step_blocks(s.KB - kb0, s.hi - u));
  Tile ti = tile_info(T, s, chunk_start, row_off, gsize, gexp, t);
  uint32_t wq[kStepBlocks][8];
  float aq[kStepBlocks];
  load_step(w, absmax, ti, s, kb0, nblk, wq, aq);

  while (u < s.hi) {
    // issue the next step's loads before consuming this one
    const int64_t un = u + nblk;
    const bool has_next = un < s.hi;
    int64_t Tn = T;
    int kbn = 0, nbn = 0;
    Tile tn = ti;
    uint32_t wn[kStepBlocks][8];
    float an[kStepBlocks];
    if (has_next) {
      Tn = un / s.KB;
      kbn = static_cast<int>(un - Tn * s.KB);
      nbn = static_cast<int>(step_blocks(s.KB - kbn, s.hi - un));
      if (Tn != T) tn = tile_info(Tn, s, chunk_start, row_off, gsize, gexp, t);
      load_step(w, absmax, tn, s, kbn, nbn, wn, an);
    }

    wait_or_flag(&full_bar[stage], phase, timed_out, hdr);
    compute_dispatch(ti.mrows, wq, aq, nblk, xs + stage * kMT * kStepK, lut, lane8, acc);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[stage]);
    if (++stage == kStages) { stage = 0; phase ^= 1u; }

    const bool tile_end = (un == (T + 1) * s.KB) || !has_next;
    if (tile_end) {
      const bool whole = (T * s.KB >= s.lo) && ((T + 1) * s.KB <= s.hi);
      if (whole) {
        write_tile(acc, ti, s, y, ex, t);
      } else {
        // split tile: publish the partial, the last contributor finishes it
        const int64_t P2 = P;
        const int slot = (T == s.lo / s.KB) ? 0 : 1;
        float *mine = partials + (static_cast<int64_t>(blockIdx.x) * 2 + slot) * (kMT * kRows);
#pragma unroll
        for (int m = 0; m < kMT; ++m) mine[m * kRows + t] = acc[m];
        __threadfence();
        named_barrier(1, kConsumers);
        if (t == 0) {
          // contributors: the CTAs with a non-empty range inside [c0, c1]
          const int64_t c0 = cta_of(s.units, T * s.KB, P2);
          const int64_t c1 = cta_of(s.units, (T + 1) * s.KB - 1, P2);
          int ncontrib = 0;
          for (int64_t c = c0; c <= c1; ++c)
            ncontrib += cta_lo(s.units, c, P2) < cta_lo(s.units, c + 1, P2) ? 1 : 0;
          const int old = atomicAdd(&tile_cnt[T], 1);
          misc[2] = (old == ncontrib - 1) ? 1 : 0;
        }
        named_barrier(1, kConsumers);
        if (misc[2]) {
          __threadfence();
          const int64_t c0 = cta_of(s.units, T * s.KB, P2);
          const int64_t c1 = cta_of(s.units, (T + 1) * s.KB - 1, P2);
          float sum[kMT];
#pragma unroll
          for (int m = 0; m < kMT; ++m) sum[m] = 0.0f;
          for (int64_t c = c0; c <= c1; ++c) {
            const int64_t lo_c = cta_lo(s.units, c, P2);
            if (lo_c >= cta_lo(s.units, c + 1, P2)) continue;   // empty range: no partial
            const int sl = (T == lo_c / s.KB) ? 0 : 1;
            const float *src = partials + (c * 2 + sl) * (kMT * kRows);
#pragma unroll
            for (int m = 0; m < kMT; ++m) sum[m] += __ldcg(src + m * kRows + t);
          }
          write_tile(sum, ti, s, y, ex, t);
          if (t == 0) tile_cnt[T] = 0;
        }
        named_barrier(1, kConsumers);   // misc[2] is reused by the next split tile
      }
#pragma unroll
      for (int m = 0; m < kMT; ++m) acc[m] = 0.0f;
    }

    if (!has_next) break;
    u = un;
    T = Tn;
    kb0 = kbn;
    nblk = nbn;
    ti = tn;
#pragma unroll
    for (int b = 0; b < kStepBlocks; ++b) {
      aq[b] = an[b];
#pragma unroll
      for (int i = 0; i < 8; ++i) wq[b][i] = wn[b][i];
    }
  }
}

}  // namespace

size_t decode_workspace_bytes(int64_t M, int32_t N, int32_t K, int32_t G, int32_t swiglu) {
  (void)K;
  const int64_t nt = swiglu ? (N / 2 + 127) / 128 : (N + kRows - 1) / kRows;
  const int64_t groups = G < M ? G : M;
  const int64_t tile_cap = (M / kMT + groups) * nt;
  const size_t cnt_bytes = ((static_cast<size_t>(tile_cap) * 4 + 255) / 256) * 256;
  const size_t part_bytes = static_cast<size_t>(device_sm_count()) * 2 * kMT * kRows * 4;
  return kWsHeaderBytes + cnt_bytes + part_bytes;
}

cudaError_t launch_decode_gemm(const GemmArgs &a, cudaStream_t stream) {
  const int64_t nt = a.swiglu ? (a.N / 2 + 127) / 128 : (a.N + kRows - 1) / kRows;
  const int64_t groups = a.G < a.M ? a.G : a.M;
  const int64_t tile_cap = (a.M / kMT + groups) * nt;
  const size_t cnt_bytes = ((static_cast<size_t>(tile_cap) * 4 + 255) / 256) * 256;
  char *ws = static_cast<char *>(a.workspace);
  WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
  int32_t *cnt = reinterpret_cast<int32_t *>(ws + kWsHeaderBytes);
  float *partials = reinterpret_cast<float *>(ws + kWsHeaderBytes + cnt_bytes);

  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t err = cudaFuncSetAttribute(decode_gemm_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    configured[dev] = true;
  }
  const int grid = device_sm_count();
  decode_gemm_kernel<<<grid, kThreads, kSmemBytes, stream>>>(
      a.x, a.w, a.absmax, a.sizes, a.expert_ids, a.G, a.M, a.N, a.K, a.E, a.swiglu, a.y, hdr, cnt,
      tile_cap, partials);
  return cudaGetLastError();
}

}  // namespace gnf4
