// moe_align.cu -- stable counting sort of token->expert slots (one CTA).
//
// Passage: "grouped-nf4-gemm -- single-launch W4A16 GEMM over fused NF4 MoE
// expert stacks", opening section: (sizes, expert_ids) are supplied after the
// usual token->expert sort. The sort fixed here (gnf4.h documents it):
// groups = non-empty experts in ascending id, slots ascending within a group.
//
// Design: up to 32 slots, one warp (below); otherwise a single CTA (8 warps
// up to 4096 slots, else 32), everything in shared memory, one launch.
//   1. each warp owns a contiguous segment of the S = T*top_k slots and builds
//      its own per-expert histogram (shared-memory atomics);
//   2. per expert, an exclusive scan over the 32 warp histograms gives each
//      warp its starting rank inside the expert's group;
//   3. a block scan over experts gives each expert's first output position and
//      each non-empty expert its group index;
//   4. each warp walks its segment 32 slots at a time; lanes holding the same
//      expert find each other with __match_any_sync and take consecutive
//      positions in lane order, so the output is stable without atomics.
// The decode-regime problems this serves have at most a few thousand slots;
// the kernel is latency-bound (a few microseconds).
#include "launch.h"

namespace gnf4 {
namespace {

// NW warps; each warp owns a contiguous segment of the slots.
template <int NW>
__global__ void __launch_bounds__(NW * 32, 1)
    moe_align_kernel(const int32_t *__restrict__ topk, int32_t S, int32_t E,
                     int32_t *__restrict__ sorted_idx, int32_t *__restrict__ sizes,
                     int32_t *__restrict__ expert_ids, int32_t *__restrict__ num_groups,
                     WsHeader *hdr) {
  constexpr int NT = NW * 32;
  extern __shared__ int32_t sm[];
  int32_t *hist = sm;                 // [NW][E]
  int32_t *start = hist + NW * E;     // [E] first output position of each expert
  __shared__ int32_t warp_sum_v[NW];
  __shared__ int32_t warp_sum_f[NW];
  __shared__ int32_t s_valid, s_groups;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();
  for (int i = tid; i < NW * E; i += NT) hist[i] = 0;
  __syncthreads();
  pdl_wait();   // topk may come from the previous kernel on the stream

  const int seg = (S + NW - 1) / NW;
  const int beg = min(S, warp * seg), end = min(S, beg + seg);

  // 1. per-warp histograms
  for (int s = beg + lane; s < end; s += 32) {
    const int e = topk[s];
    if (e >= 0 && e < E) {
      atomicAdd(&hist[warp * E + e], 1);
    } else {
      report_error(hdr, GNF4_DEVERR_TOPK, static_cast<uint32_t>(s));
    }
  }
  __syncthreads();

  // 2. per expert: exclusive scan over the warps' histograms. Thread tid owns
  //    the contiguous experts [e0, e1); its local sums feed the block scan.
  const int per = (E + NT - 1) / NT;
  const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
  int my_v = 0, my_f = 0;
  for (int e = e0; e < e1; ++e) {
    int tot = 0;
    for (int w = 0; w < NW; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = tot;
      tot += c;
    }
    start[e] = tot;            // count for now; turned into a position below
    my_v += tot;
    my_f += tot > 0 ? 1 : 0;
  }

  // 3. block exclusive scans of counts (v) and non-empty flags (f) over experts
  int v = my_v, f = my_f;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, v, o);
    const int b = __shfl_up_sync(0xffffffffu, f, o);
    if (lane >= o) { v += a; f += b; }
  }
  if (lane == 31) { warp_sum_v[warp] = v; warp_sum_f[warp] = f; }
  __syncthreads();
  if (warp == 0) {
    const int a0 = lane < NW ? warp_sum_v[lane] : 0, b0 = lane < NW ? warp_sum_f[lane] : 0;
    int a = a0, b = b0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ua = __shfl_up_sync(0xffffffffu, a, o);
      const int ub = __shfl_up_sync(0xffffffffu, b, o);
      if (lane >= o) { a += ua; b += ub; }
    }
    if (lane < NW) { warp_sum_v[lane] = a - a0; warp_sum_f[lane] = b - b0; }
    if (lane == 31) { s_valid = a; s_groups = b; }
  }
  __syncthreads();
  {
    int pos = v - my_v + warp_sum_v[warp];
    int grp = f - my_f + warp_sum_f[warp];
    for (int e = e0; e < e1; ++e) {
      const int cnt = start[e];
      start[e] = pos;
      if (cnt > 0) { sizes[grp] = cnt; expert_ids[grp] = e; ++grp; }
      pos += cnt;
    }
  }
  __syncthreads();
  const int ngroups = s_groups;
  for (int g = ngroups + tid; g < E; g += NT) { sizes[g] = 0; expert_ids[g] = -1; }
  if (tid == 0) *num_groups = ngroups;

  // 4. stable scatter, 32 slots per warp step
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = beg; base < end; base += 32) {
    const int s = base + lane;
    const int e = (s < end) ? topk[s] : -1;
    const bool ok = (s < end) && e >= 0 && e < E;
    const int key = ok ? e : -1 - lane;   // invalid lanes never match each other
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    const int rank = __popc(peers & lt_mask);
    const int cur = ok ? hist[warp * E + e] : 0;
    __syncwarp();
    if (ok) {
      sorted_idx[start[e] + cur + rank] = s;
      if (rank == 0) hist[warp * E + e] = cur + __popc(peers);
    }
    __syncwarp();
  }
  // slots with an invalid id are left out; pad the tail of the permutation
  for (int i = s_valid + tid; i < S; i += NT) sorted_idx[i] = -1;
}

// S <= 32 (a decode step of a few tokens): one warp, slot s in lane s, no
// shared memory and no block barrier. A slot's position is the number of
// valid slots with a smaller expert id plus its rank among the slots of its
// own expert (lanes found with __match_any_sync); its expert's group index is
// the number of distinct smaller experts. Same output as the general kernel.
__global__ void __launch_bounds__(32, 1)
    moe_align_warp_kernel(const int32_t *__restrict__ topk, int32_t S, int32_t E,
                          int32_t *__restrict__ sorted_idx, int32_t *__restrict__ sizes,
                          int32_t *__restrict__ expert_ids, int32_t *__restrict__ num_groups,
                          WsHeader *hdr) {
  const int lane = threadIdx.x;
  pdl_trigger();
  pdl_wait();   // topk may come from the previous kernel on the stream
  const int e = lane < S ? topk[lane] : -1;
  const bool valid = lane < S && e >= 0 && e < E;
  if (lane < S && !valid) report_error(hdr, GNF4_DEVERR_TOPK, static_cast<uint32_t>(lane));
  const int key = valid ? e : -1 - lane;   // invalid lanes never match each other
  const unsigned peers = __match_any_sync(0xffffffffu, key);
  const unsigned lt_mask = (1u << lane) - 1u;
  const bool leader = valid && (peers & lt_mask) == 0u;   // lowest slot of its expert
  const unsigned vmask = __ballot_sync(0xffffffffu, valid);
  const unsigned lmask = __ballot_sync(0xffffffffu, leader);
  int before = 0, grp = 0;   // valid slots / distinct experts with a smaller id
  for (int j = 0; j < 32; ++j) {
    const int ej = __shfl_sync(0xffffffffu, key, j);
    if (((vmask >> j) & 1u) && ej < e) {
      ++before;
      grp += static_cast<int>((lmask >> j) & 1u);
    }
  }
  if (valid) sorted_idx[before + __popc(peers & lt_mask)] = lane;
  if (leader) {
    sizes[grp] = __popc(peers);
    expert_ids[grp] = e;
  }
  const int ngroups = __popc(lmask), nvalid = __popc(vmask);
  for (int g = ngroups + lane; g < E; g += 32) {
    sizes[g] = 0;
    expert_ids[g] = -1;
  }
  if (lane == 0) *num_groups = ngroups;
  // slots with an invalid id are left out; pad the tail of the permutation
  for (int i = nvalid + lane; i < S; i += 32) sorted_idx[i] = -1;
}

constexpr int kWarpSlots = 32;    // up to this many slots: the one-warp kernel
constexpr int kSmallWarps = 8;    // up to kSmallSlots slots
constexpr int kLargeWarps = 32;
constexpr int kSmallSlots = 4096;

}  // namespace

size_t moe_align_smem_bytes(int32_t E) {
  return static_cast<size_t>(kLargeWarps + 1) * static_cast<size_t>(E) * sizeof(int32_t);
}

cudaError_t launch_moe_align(const int32_t *topk, int32_t S, int32_t E, int32_t *sorted_idx,
                             int32_t *sizes, int32_t *expert_ids, int32_t *num_groups,
                             WsHeader *hdr, cudaStream_t stream) {
  // Opt in once per device to the largest table the kernels can need, so
  // that later calls (including ones under stream capture) set no attributes.
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    const int big = static_cast<int>(moe_align_smem_bytes(GNF4_MAX_EXPERTS));
    cudaError_t err = cudaFuncSetAttribute(moe_align_kernel<kSmallWarps>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, big);
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(moe_align_kernel<kLargeWarps>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, big);
    // Same shared-memory carveout as the GEMM kernels that follow, so the SM
    // need not be reconfigured between the launches of one MoE layer.
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(moe_align_kernel<kSmallWarps>,
                                 cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(moe_align_kernel<kLargeWarps>,
                                 cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  if (S <= kWarpSlots)
    return launch_pdl(moe_align_warp_kernel, dim3(1), dim3(32), 0, stream, topk, S, E, sorted_idx,
                      sizes, expert_ids, num_groups, hdr);
  if (S <= kSmallSlots) {
    const size_t smem = static_cast<size_t>(kSmallWarps + 1) * E * sizeof(int32_t);
    return launch_pdl(moe_align_kernel<kSmallWarps>, dim3(1), dim3(kSmallWarps * 32), smem, stream,
                      topk, S, E, sorted_idx, sizes, expert_ids, num_groups, hdr);
  }
  const size_t smem = static_cast<size_t>(kLargeWarps + 1) * E * sizeof(int32_t);
  return launch_pdl(moe_align_kernel<kLargeWarps>, dim3(1), dim3(kLargeWarps * 32), smem, stream,
                    topk, S, E, sorted_idx, sizes, expert_ids, num_groups, hdr);
}

}  // namespace gnf4
