// dgrad.cu -- the gradient of the grouped NF4 GEMM with respect to its
// activations: dx[m][k] = sum_n dy[m][n] * w[e][n][k], e the expert of row
// m's group, w = NF4[code] * absmax (one fp32 multiply, as the forward
// kernels and dequant_debug), summed in fp32 over n ascending, rounded once
// to bf16.
//
// Passage: "grouped-nf4-gemm" package page, header block ("Owns": the grouped
// packed GEMM and its dgrad); "Do not use this when" (the dgrad, like the
// GEMM, refuses tensors that are not on the device).
//
// A CUDA-core kernel for decode-sized problems: block (r, c) computes rows
// kDgradRows r .. +kDgradRows-1 of dx at columns 256 c + threadIdx.x. Each
// thread decodes the code of its column from the packed row of every n (two
// threads share a byte; a warp reads 16 contiguous bytes) and multiplies by
// dy[m][n], read by all threads of the block at once. Each block first checks
// the group metadata; on an error it writes nothing (the first block records
// the error bits).
#include "launch.h"

namespace gnf4 {
namespace {

constexpr int kDgradThreads = 256;
constexpr int kDgradRows = 4;

__global__ void __launch_bounds__(kDgradThreads)
    dgrad_kernel(const uint16_t *__restrict__ dy, const uint8_t *__restrict__ w,
                 const float *__restrict__ absmax, const int32_t *__restrict__ sizes,
                 const int32_t *__restrict__ expert_ids, int32_t G, int64_t M, int32_t N,
                 int32_t K, int32_t E, uint16_t *__restrict__ dx, WsHeader *hdr) {
  __shared__ int64_t s_start[GNF4_MAX_EXPERTS + 1];   // first row of group g
  __shared__ int s_bad;
  __shared__ float s_lut[16];   // the code table (a per-thread constant-memory
                                // index would serialise the warp)
  pdl_trigger();
  if (threadIdx.x < 16) s_lut[threadIdx.x] = nf4_value(threadIdx.x);
  pdl_wait();
  if (threadIdx.x == 0) {
    int bad = 0;
    int64_t off = 0;
    for (int g = 0; g < G; ++g) {
      const int sz = sizes[g];
      s_start[g] = off;
      if (sz < 0) bad |= GNF4_DEVERR_SIZES;
      if (sz > 0 && (expert_ids[g] < 0 || expert_ids[g] >= E)) bad |= GNF4_DEVERR_EXPERT;
      off += sz > 0 ? sz : 0;
    }
    s_start[G] = off;
    if (off != M) bad |= GNF4_DEVERR_SIZES;
    s_bad = bad;
    if (bad && blockIdx.x == 0 && blockIdx.y == 0) report_error(hdr, static_cast<uint32_t>(bad), 0);
  }
  __syncthreads();
  if (s_bad) return;
  const int k = blockIdx.y * kDgradThreads + threadIdx.x;
  const int64_t kb = K / 64;
  for (int r = 0; r < kDgradRows; ++r) {
    const int64_t m = static_cast<int64_t>(blockIdx.x) * kDgradRows + r;
    if (m >= M) break;
    // the group of row m: the last g with s_start[g] <= m (groups of size 0
    // share their start with the next group and are skipped by the search)
    int lo = 0, hi = G;   // s_start[lo] <= m < s_start[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_start[mid] <= m) lo = mid; else hi = mid;
    }
    const int e = expert_ids[lo];
    if (k >= K) continue;
    const uint8_t *wcol = w + static_cast<int64_t>(e) * N * (K / 2) + k / 2;
    const float *acol = absmax + static_cast<int64_t>(e) * N * kb + k / 64;
    const uint16_t *dyr = dy + m * N;
    const int shift = (k & 1) ? 0 : 4;   // even k: high nibble
    float acc = 0.0f;
    for (int n = 0; n < N; ++n) {
      const int code = (wcol[static_cast<int64_t>(n) * (K / 2)] >> shift) & 0xF;
      const float wv = __fmul_rn(s_lut[code], acol[static_cast<int64_t>(n) * kb]);
      const float g = __uint_as_float(static_cast<uint32_t>(dyr[n]) << 16);
      acc = fmaf(g, wv, acc);
    }
    const __nv_bfloat16 b = __float2bfloat16_rn(acc);
    dx[m * K + k] = *reinterpret_cast<const uint16_t *>(&b);
  }
}

}  // namespace

cudaError_t launch_grouped_dgrad(const uint16_t *dy, const uint8_t *w, const float *absmax,
                                 const int32_t *sizes, const int32_t *expert_ids, int32_t G,
                                 int64_t M, int32_t N, int32_t K, int32_t E, uint16_t *dx,
                                 WsHeader *hdr, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((M + kDgradRows - 1) / kDgradRows),
                  static_cast<unsigned>((K + kDgradThreads - 1) / kDgradThreads));
  return launch_pdl(dgrad_kernel, grid, dim3(kDgradThreads), 0, stream, dy, w, absmax, sizes,
                    expert_ids, G, M, N, K, E, dx, hdr);
}

}  // namespace gnf4
