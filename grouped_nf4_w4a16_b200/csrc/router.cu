// router.cu -- the steps on either side of the grouped GEMM: the router's
// top-k (gnf4_router_topk) before the token->expert sort, and the top-k
// weighted combine (gnf4_moe_combine) after the down projection.
//
// Passage: "grouped-nf4-gemm" package page, "Use this when" (the tail of
// small launches around the expert GEMMs in a batch-1 decode step, router
// softmax and top-k and the top-k combine among them, each to be folded into
// one launch) and its header block ("Owns": the decode glue kernels, combine
// among them); the README's opening section (the GEMM consumes
// (sizes, expert_ids) produced by the token->expert sort of the router's
// choices).
//
// router_topk: one warp per token. Each lane holds the logits of experts
// lane, lane + 32, ... in registers (E <= 1024); top_k rounds of a warp
// arg-max (larger logit first, equal logits by lower expert id; NaN ranks as
// -inf) pick the experts, then the softmax weights follow from the largest
// logit: over all E experts, or over the top_k selected ones.
//
// moe_combine: one block rebuilds the inverse of sorted_idx (slot -> row of
// y) in the workspace, then out[t][h] = bf16(sum_j w[t][j] * y[row][h]) in
// fp32, j ascending, one thread per 8 outputs (or per output where rows are
// not 16-byte multiples).
#include <climits>

#include "launch.h"

namespace gnf4 {
namespace {

constexpr int kRouterPerLane = GNF4_MAX_EXPERTS / 32;
constexpr int kRouterThreads = 256;

// (va, ia) ranks above (vb, ib)
__device__ __forceinline__ bool ranks_above(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__global__ void __launch_bounds__(kRouterThreads)
    router_topk_kernel(const float *__restrict__ logits, int64_t T, int32_t E, int32_t k,
                       int32_t renorm, int32_t *__restrict__ ids, float *__restrict__ weights) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kRouterThreads / 32);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (kRouterThreads / 32) + (threadIdx.x >> 5);
       t < T; t += nwarps) {
    const float *row = logits + t * E;
    float v[kRouterPerLane];
#pragma unroll
    for (int u = 0; u < kRouterPerLane; ++u) {
      const int e = lane + 32 * u;
      const float x = e < E ? __ldg(row + e) : -INFINITY;
      v[u] = x != x ? -INFINITY : x;   // NaN never ranks above a number
    }
    uint32_t taken = 0u;   // bit u: expert lane + 32 u already selected
    float sel_v = -INFINITY, vmax = -INFINITY;
    int sel_i = 0;         // lane j < k ends up holding the j-th selection
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = INT_MAX;
#pragma unroll
      for (int u = 0; u < kRouterPerLane; ++u) {
        const int e = lane + 32 * u;
        if (e < E && !((taken >> u) & 1u) && ranks_above(v[u], e, bv, bi)) {
          bv = v[u];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ranks_above(ov, oi, bv, bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      if (lane == j) {
        sel_v = bv;
        sel_i = bi;
      }
      if (j == 0) vmax = bv;
    }
    // softmax weights relative to the largest logit
    float part = 0.0f;
    if (renorm) {
      if (lane < k) part = expf(sel_v - vmax);
    } else {
#pragma unroll
      for (int u = 0; u < kRouterPerLane; ++u)
        if (lane + 32 * u < E) part += expf(v[u] - vmax);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane < k) {
      ids[t * k + lane] = sel_i;
      weights[t * k + lane] = expf(sel_v - vmax) / part;
    }
  }
}

// inv[s] = the row of y (position in sorted_idx) that holds slot s, -1 for
// slots left out; one block.
__global__ void __launch_bounds__(1024)
    combine_inverse_kernel(const int32_t *__restrict__ sorted_idx, int64_t S,
                           int32_t *__restrict__ inv, WsHeader *hdr) {
  pdl_trigger();
  pdl_wait();
  for (int64_t i = threadIdx.x; i < S; i += blockDim.x) inv[i] = -1;
  __syncthreads();
  for (int64_t i = threadIdx.x; i < S; i += blockDim.x) {
    const int32_t s = sorted_idx[i];
    if (s == -1) continue;
    if (s < 0 || s >= S) {
      report_error(hdr, GNF4_DEVERR_SLOT, static_cast<uint32_t>(i));
      continue;
    }
    inv[s] = static_cast<int32_t>(i);
  }
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__global__ void __launch_bounds__(256)
    combine_kernel(const uint16_t *__restrict__ y, const int32_t *__restrict__ inv,
                   const float *__restrict__ w, int64_t T, int32_t k, int32_t H, int32_t vec8,
                   uint16_t *__restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  if (vec8) {
    const int h8 = H / 8;
    for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < T * h8;
         q += stride) {
      const int64_t t = q / h8;
      const int c = static_cast<int>(q - t * h8);
      float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
      for (int j = 0; j < k; ++j) {
        const int32_t p = inv[t * k + j];
        if (p < 0) continue;
        const float wj = w[t * k + j];
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(y + static_cast<int64_t>(p) * H) + c);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = fmaf(wj, __uint_as_float(u[i] << 16), acc[2 * i]);
          acc[2 * i + 1] = fmaf(wj, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
        }
      }
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        o[i] = *reinterpret_cast<const uint32_t *>(&b);
      }
      reinterpret_cast<uint4 *>(out + t * H)[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  } else {
    for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < T * H;
         q += stride) {
      const int64_t t = q / H;
      const int h = static_cast<int>(q - t * H);
      float acc = 0.0f;
      for (int j = 0; j < k; ++j) {
        const int32_t p = inv[t * k + j];
        if (p < 0) continue;
        acc = fmaf(w[t * k + j], bf16_to_f32(y[static_cast<int64_t>(p) * H + h]), acc);
      }
      const __nv_bfloat16 b = __float2bfloat16_rn(acc);
      out[q] = *reinterpret_cast<const uint16_t *>(&b);
    }
  }
}

}  // namespace

size_t combine_workspace_bytes(int64_t S) {
  return kWsHeaderBytes + ((static_cast<size_t>(S) * 4 + 255) / 256) * 256;
}

cudaError_t launch_router_topk(const float *logits, int64_t T, int32_t E, int32_t k, int32_t renorm,
                               int32_t *ids, float *weights, cudaStream_t stream) {
  const int64_t want = (T + kRouterThreads / 32 - 1) / (kRouterThreads / 32);
  const int64_t cap = 8 * static_cast<int64_t>(device_sm_count());
  const int blocks = static_cast<int>(want < cap ? want : cap);
  return launch_pdl(router_topk_kernel, dim3(blocks), dim3(kRouterThreads), 0, stream, logits, T,
                    E, k, renorm, ids, weights);
}

cudaError_t launch_moe_combine(const uint16_t *y, const int32_t *sorted_idx, const float *w,
                               int64_t T, int32_t k, int32_t H, uint16_t *out, void *workspace,
                               cudaStream_t stream) {
  const int64_t S = T * k;
  WsHeader *hdr = static_cast<WsHeader *>(workspace);
  int32_t *inv = reinterpret_cast<int32_t *>(static_cast<char *>(workspace) + kWsHeaderBytes);
  cudaError_t err = launch_pdl(combine_inverse_kernel, dim3(1), dim3(1024), 0, stream, sorted_idx,
                               S, inv, hdr);
  if (err != cudaSuccess) return err;
  const int32_t vec8 = (H % 8 == 0 && (reinterpret_cast<uintptr_t>(y) & 15u) == 0 &&
                        (reinterpret_cast<uintptr_t>(out) & 15u) == 0)
                           ? 1
                           : 0;
  const int64_t work = vec8 ? T * (H / 8) : T * H;
  const int64_t want = (work + 255) / 256;
  const int64_t cap = 16 * static_cast<int64_t>(device_sm_count());
  const int blocks = static_cast<int>(want < 1 ? 1 : (want < cap ? want : cap));
  return launch_pdl(combine_kernel, dim3(blocks), dim3(256), 0, stream, y,
                    static_cast<const int32_t *>(inv), w, T, k, H, vec8, out);
}

}  // namespace gnf4
