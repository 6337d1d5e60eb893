// prefill_gemm.cu -- prefill-regime grouped NF4 GEMM on the 5th-generation
// tensor cores (tcgen05, TMEM, TMA).
//
// Passage: "grouped-nf4-gemm -- single-launch W4A16 GEMM over fused NF4 MoE
// expert stacks", opening section (one launch for all active experts, LUT
// decode, blockwise fp32 absmax, fp32 accumulation, bf16 epilogue, no bf16
// weight copy in memory) and "The claim" (prefill: compute-bound M, a
// register-LUT M-tile mainloop). With ~1000 activation rows per expert the
// contraction is dense and bound by tensor-core throughput.
//
// Tile = 128 weight rows of one expert x 256 activation rows of one group,
// computed as D[weight row][activation row] = W . x^T (weights as the MMA's
// M side), K in stages of 64 (one absmax block).
//
// Roles (12 warps, one CTA per SM, persistent over tiles):
//   warp 0  TMA producer: x tile [256 rows x 64] bf16 -> shared memory ring
//           (4 stages, 128-byte swizzle, the canonical K-major operand layout).
//   warp 1  MMA issuer (one thread): tcgen05.mma kind::f16, A from TMEM, B
//           from shared memory, fp32 accumulator in TMEM (256 columns).
//   warp 2  allocates / frees the 512 TMEM columns.
//   warps 4-11  decoders + epilogue. Warp w owns TMEM lanes 32*(w%4).. (=
//           weight rows) and half of the stage's 64 K-elements. Each lane
//           loads its row's 16 packed bytes, decodes every byte with one
//           shared-memory load of the fp32 pair (NF4[hi], NF4[lo]) (table
//           replicated per lane: no bank conflicts), multiplies by the
//           block's absmax in fp32 (the exact fp32 weight), and splits it into
//           bf16 hi + bf16 lo (hi + lo = weight to 2^-18 relative). Both
//           halves go straight to TMEM with tcgen05.st: the decoded weights
//           never touch shared or global memory.
//   The MMA runs twice per K-step, on the hi and on the lo weights, into the
//   same accumulator, so the result is the fp32-exact-weight contraction
//   (a single 16-bit weight would miss the 1e-3*rms elementwise tolerance at
//   these output sizes). After the last stage the decoders read the
//   accumulator back (tcgen05.ld), round to bf16 and store y.
// Synchronisation: mbarriers per stage (x landed, weights decoded, stage
// free), accumulator full/empty; every wait is bounded (2 s), after which the
// kernel records GNF4_DEVERR_TIMEOUT, drains what it started and returns.
#include "launch.h"
#include "sm100.cuh"

namespace gnf4 {
namespace {

constexpr int kBM = 128;            // weight rows per tile (TMEM lanes, MMA M)
constexpr int kBN = 256;            // activation rows per tile (MMA N)
constexpr int kBK = 64;             // K per stage
constexpr int kStages = 4;
constexpr int kThreads = 384;       // 12 warps
constexpr int kDecodeWarp0 = 4;
constexpr int kDecodeThreads = 256; // warps 4..11
constexpr int kMaxG = GNF4_MAX_EXPERTS;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;     // accumulator: columns [0, 256)
constexpr uint32_t kACol = 256;     // stage s: hi at kACol + 64 s, lo at +32
constexpr int kXStageBytes = kBN * kBK * 2;   // 32 KB

// Shared memory layout (dynamic, 1024-aligned base).
constexpr int kXOff = 0;                                  // x ring (1024-aligned stages)
constexpr int kLutOff = kXOff + kStages * kXStageBytes;   // float2 [256][32]
constexpr int kLutBytes = 256 * 32 * 8;
constexpr int kTileStartOff = kLutOff + kLutBytes;        // int[kMaxG + 1]
constexpr int kRowOffOff = kTileStartOff + (kMaxG + 4) * 4;
constexpr int kGSizeOff = kRowOffOff + kMaxG * 4;
constexpr int kGExpOff = kGSizeOff + kMaxG * 4;
constexpr int kBarOff = kGExpOff + kMaxG * 4;             // mbarriers
constexpr int kNumBars = 3 * kStages + 3;
constexpr int kMiscOff = kBarOff + kNumBars * 8;          // int[8]
constexpr int kSmemBytes = kMiscOff + 8 * 4 + 1024;       // + alignment slack

// ------------------------------------------------------------------ PTX
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[tmem] . B[smem desc]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
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

// Shared-memory operand descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), leading offset unused (1), descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor: kind::f16, bf16 A and B (K-major), fp32 D, M=128, N=256.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
                            (static_cast<uint32_t>(kBM >> 4) << 24);

__device__ __forceinline__ uint4 ldg128_nc(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

struct TileInfo {
  int64_t row0;     // first activation row of the tile
  int32_t rows;     // valid activation rows (1..256)
  int32_t n0;       // first weight row (within the expert)
  int32_t e;        // expert
};

__device__ __forceinline__ TileInfo tile_info(int t, int G, int NJ, const int *tile_start,
                                              const int *row_off, const int *gsize,
                                              const int *gexp) {
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
  ti.n0 = j * kBM;
  ti.e = gexp[lo];
  return ti;
}

__global__ void __launch_bounds__(kThreads, 1)
    prefill_gemm_kernel(const __grid_constant__ CUtensorMap xmap, const uint8_t *__restrict__ w,
                        const float *__restrict__ absmax, const int32_t *__restrict__ sizes,
                        const int32_t *__restrict__ expert_ids, int32_t G, int64_t M, int32_t N,
                        int32_t K, int32_t E, uint16_t *__restrict__ y, WsHeader *hdr) {
  extern __shared__ char smem_raw[];
  char *smem = reinterpret_cast<char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~static_cast<uintptr_t>(1023));
  char *xs = smem + kXOff;
  int *tile_start = reinterpret_cast<int *>(smem + kTileStartOff);
  int *row_off = reinterpret_cast<int *>(smem + kRowOffOff);
  int *gsize = reinterpret_cast<int *>(smem + kGSizeOff);
  int *gexp = reinterpret_cast<int *>(smem + kGExpOff);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBarOff);
  uint64_t *x_full = bars;                  // [kStages] TMA landed
  uint64_t *a_full = bars + kStages;        // [kStages] weights decoded into TMEM
  uint64_t *st_free = bars + 2 * kStages;   // [kStages] MMA done reading the stage
  uint64_t *d_full = bars + 3 * kStages;    // accumulator complete
  uint64_t *d_empty = d_full + 1;           // accumulator read out
  uint64_t *drain = d_full + 2;             // final MMA drain
  int *misc = reinterpret_cast<int *>(smem + kMiscOff);
  volatile int *abort_flag = &misc[1];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();

  // ---- set-up: decode table, barriers, TMEM
  for (int i = tid; i < 256 * 32; i += kThreads) {
    const int b = i >> 5;
    reinterpret_cast<float2 *>(smem + kLutOff)[i] = make_float2(nf4_value(b >> 4), nf4_value(b & 15));
  }
  if (tid == 0) {
    misc[0] = 0;
    misc[1] = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&a_full[s], kDecodeThreads);
      mbar_init(&st_free[s], 1);
    }
    mbar_init(d_full, 1);
    mbar_init(d_empty, kDecodeThreads);
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tensormap(&xmap);
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&misc[4])),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }

  pdl_wait();   // inputs may come from the previous kernel on the stream

  // ---- group table (validated; same rules as the decode kernel)
  __shared__ int s_wsum[2][kThreads / 32];
  const int NJ = (N + kBM - 1) / kBM;
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[4]);
  const int errbits = misc[0];
  const int KB = K / kBK;
  const int tiles = tot_t;
  const int64_t row_bytes = K / 2;

  if (errbits == 0) {
    if (warp == 0) {
      // --------------------------------------------------------- TMA producer
      if (lane == 0) {
        uint32_t g = 0;   // stage ring counter
        for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
          const TileInfo ti = tile_info(t, G, NJ, tile_start, row_off, gsize, gexp);
          for (int kb = 0; kb < KB; ++kb, ++g) {
            const int s = g % kStages;
            const uint32_t ph = (g / kStages) & 1u;
            if (!wait_bar(&st_free[s], ph ^ 1u, abort_flag, hdr)) break;
            mbar_arrive_expect_tx(&x_full[s], kXStageBytes);
            tma_load_2d(xs + s * kXStageBytes, &xmap, kb * kBK, static_cast<int>(ti.row0), &x_full[s]);
          }
        }
        // drain: the last issued copies must land before the CTA exits
        for (uint32_t d = 0; d < kStages && d < g; ++d) {
          const uint32_t gg = g - 1 - d;
          drain_wait(&x_full[gg % kStages], (gg / kStages) & 1u);
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        uint32_t g = 0;
        uint32_t ntile = 0;
        for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x, ++ntile) {
          if (ntile > 0 && !wait_bar(d_empty, (ntile - 1) & 1u, abort_flag, hdr)) break;
          tc_fence_after();
          bool ok = true;
          for (int kb = 0; kb < KB; ++kb, ++g) {
            const int s = g % kStages;
            const uint32_t ph = (g / kStages) & 1u;
            if (!wait_bar(&x_full[s], ph, abort_flag, hdr) ||
                !wait_bar(&a_full[s], ph, abort_flag, hdr)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t xaddr = smem_u32(xs + s * kXStageBytes);
            const uint32_t a_hi = tmem + kACol + 64u * s, a_lo = a_hi + 32u;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t bdesc = sw128_desc(xaddr + kk * 32);
              mma_ts(tmem + kAccCol, a_hi + 8u * kk, bdesc, kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
              mma_ts(tmem + kAccCol, a_lo + 8u * kk, bdesc, kIdesc, 1u);
            }
            mma_commit(&st_free[s]);
          }
          if (!ok) break;
          mma_commit(d_full);
        }
        // drain every MMA this thread issued before TMEM is released
        mma_commit(drain);
        drain_wait(drain, 0);
      }
    } else if (warp >= kDecodeWarp0) {
      // ---------------------------------------------------- decode + epilogue
      const int dw = warp - kDecodeWarp0;
      const int quarter = warp & 3;          // TMEM lane quarter
      const int half = dw >> 2;              // K half of the stage / token half of the tile
      const int r = quarter * 32 + lane;     // weight row within the tile
      const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
      const char *lut = smem + kLutOff + lane * 8;
      uint32_t g = 0;
      uint32_t ntile = 0;
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x, ++ntile) {
        const TileInfo ti = tile_info(t, G, NJ, tile_start, row_off, gsize, gexp);
        const int n = ti.n0 + r;
        const bool rok = n < N;
        const int64_t wrow = static_cast<int64_t>(ti.e) * N + (rok ? n : 0);
        const uint8_t *wp = w + wrow * row_bytes + half * 16;
        const float *ap = absmax + wrow * KB;
        uint4 pk = rok ? ldg128_nc(wp) : make_uint4(0u, 0u, 0u, 0u);
        float am = rok ? __ldg(ap) : 0.0f;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % kStages;
          const uint32_t ph = (g / kStages) & 1u;
          // prefetch the next block's bytes before decoding this one
          uint4 pk_n = make_uint4(0u, 0u, 0u, 0u);
          float am_n = 0.0f;
          if (rok && kb + 1 < KB) {
            pk_n = ldg128_nc(wp + (kb + 1) * 32);
            am_n = __ldg(ap + kb + 1);
          }
          uint32_t hi[8 * 2], lo[8 * 2];
          const uint32_t words[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const uint32_t off = ((words[q] >> (8 * p)) & 0xFFu) * 256u;
              const float2 v = *reinterpret_cast<const float2 *>(lut + off);
              const float w0 = __fmul_rn(v.x, am), w1 = __fmul_rn(v.y, am);
              const __nv_bfloat162 h = __floats2bfloat162_rn(w0, w1);
              const uint32_t hb = *reinterpret_cast<const uint32_t *>(&h);
              const float h0 = __uint_as_float(hb << 16), h1 = __uint_as_float(hb & 0xFFFF0000u);
              const __nv_bfloat162 l = __floats2bfloat162_rn(w0 - h0, w1 - h1);
              hi[q * 4 + p] = hb;
              lo[q * 4 + p] = *reinterpret_cast<const uint32_t *>(&l);
            }
          }
          if (!warp_wait_bar(&st_free[s], ph ^ 1u, abort_flag, hdr)) { ok = false; break; }
          tc_fence_after();
          const uint32_t col = kACol + 64u * s + 16u * half;
          tmem_st16(tmem + lane_base + col, hi);
          tmem_st16(tmem + lane_base + col + 32u, lo);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&a_full[s]);
          pk = pk_n;
          am = am_n;
        }
        if (!ok) break;
        // ---- epilogue: accumulator -> bf16 y
        if (!warp_wait_bar(d_full, ntile & 1u, abort_flag, hdr)) break;
        tc_fence_after();
#pragma unroll 1
        for (int c0 = half * (kBN / 2); c0 < (half + 1) * (kBN / 2); c0 += 32) {
          uint32_t acc[32];
          tmem_ld32(tmem + lane_base + kAccCol + c0, acc);
          tmem_wait_ld();
          if (rok) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (c0 + c < ti.rows) {
                const __nv_bfloat16 b = __float2bfloat16_rn(__uint_as_float(acc[c]));
                y[(ti.row0 + c0 + c) * N + n] = *reinterpret_cast<const uint16_t *>(&b);
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(d_empty);
      }
    }
  } else if (blockIdx.x == 0 && tid == 0) {
    report_error(hdr, static_cast<uint32_t>(errbits), 0);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace

size_t prefill_workspace_bytes(int64_t M, int32_t N, int32_t K, int32_t G, int32_t swiglu) {
  (void)M; (void)N; (void)K; (void)G; (void)swiglu;
  return kWsHeaderBytes;
}

cudaError_t launch_prefill_gemm(const GemmArgs &a, cudaStream_t stream) {
  if (a.swiglu) return cudaErrorNotSupported;   // fused SwiGLU is decode-only for now
  CUtensorMap xmap;
  // activations as [M rows][K bf16], boxes of 256 rows x 64 elements
  if (!encode_tensor_map_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x,
                            static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M),
                            static_cast<uint64_t>(a.K) * 2, kBK, kBN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;

  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    cudaError_t err = cudaFuncSetAttribute(prefill_gemm_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  return launch_pdl(prefill_gemm_kernel, dim3(device_sm_count()), dim3(kThreads),
                    static_cast<size_t>(kSmemBytes), stream, xmap, a.w, a.absmax, a.sizes,
                    a.expert_ids, a.G, a.M, a.N, a.K, a.E, a.y,
                    static_cast<WsHeader *>(a.workspace));
}

}  // namespace gnf4
