// sm100.cuh -- sm_100a building blocks shared by the TMA-fed kernels:
// bounded mbarrier waits, 2-D tensor copies (TMA) into shared memory and the
// host-side tensor-map encoder.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace gnf4 {

// Every wait in these kernels gives up after this long, records
// GNF4_DEVERR_TIMEOUT and lets the kernel drain and return.
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr uint32_t kWaitHintNs = 100000;   // longest single suspension of a bounded wait

// Bytes of dynamic shared memory this CTA was launched with.
__device__ __forceinline__ uint32_t dynamic_smem_size() {
  uint32_t r;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

// Bounded wait; returns false (after flagging) if it ran out or another
// thread already flagged an abort.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         WsHeader *hdr) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  while (true) {
    // suspended rather than spinning: a waiting warp leaves the issue slots
    // of its scheduler to the warps that have work
    if (mbar_try_wait_sleep(bar, parity, kWaitHintNs)) return true;
    if (*abort_flag) return false;
    if (global_timer() - t0 > kTimeoutNs) {
      *abort_flag = 1;
      report_error(hdr, GNF4_DEVERR_TIMEOUT, blockIdx.x);
      return false;
    }
  }
}

// As wait_bar, with the time limit given (a kernel may shorten it on request).
__device__ __forceinline__ bool wait_bar_lim(uint64_t *bar, uint32_t parity,
                                             volatile int *abort_flag, WsHeader *hdr,
                                             uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  const uint32_t hint = limit_ns < kWaitHintNs ? static_cast<uint32_t>(limit_ns) : kWaitHintNs;
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, hint)) return true;
    if (*abort_flag) return false;
    if (global_timer() - t0 > limit_ns) {
      *abort_flag = 1;
      report_error(hdr, GNF4_DEVERR_TIMEOUT, blockIdx.x);
      return false;
    }
  }
}

// Warp-uniform bounded wait: lane 0 waits, every lane gets the same answer,
// so warp-collective instructions after it are never reached by part of a warp.
__device__ __forceinline__ bool warp_wait_bar(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag, WsHeader *hdr) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, abort_flag, hdr) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Bounded wait that ignores the abort flag: used only to let asynchronous
// work this thread started (copies, MMAs) finish before the CTA exits or
// frees what that work uses.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = global_timer();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer() - t0 > kTimeoutNs) return;
  }
}

// 2-D tiled tensor copy global -> shared memory, completion counted in bytes
// on `bar`. c0 is the innermost coordinate (its byte offset must be a
// multiple of 16, which every caller guarantees by construction).
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, int c0, int c1,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// 3-D tiled tensor copy (c0 innermost; same alignment rule).
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// 4-D tiled tensor copy (c0 innermost; same alignment rule).
__device__ __forceinline__ void tma_load_4d(void *smem_dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, int c3, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(smem_u32(bar))
      : "memory");
}

// 4-byte asynchronous copy global -> shared (src_bytes 0: writes zeros, reads nothing).
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}

// The mbarrier receives one arrival when this thread's earlier cp.async
// copies have landed (counted in the barrier's expected arrivals).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------ host side
// Encodes a tiled tensor map of rank 2 to 5: dims[0] is the contiguous
// dimension, pitches[i] the byte stride of dims[i + 1]. `promotion` is the
// L2 fetch size of each access (256 bytes unless a narrow box's neighbours
// would be evicted before they are used). Returns false if the driver
// refuses it.
bool encode_tensor_map(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *base,
                       const uint64_t *dims, const uint64_t *pitches, const uint32_t *box,
                       CUtensorMapSwizzle swizzle,
                       CUtensorMapL2promotion promotion = CU_TENSOR_MAP_L2_PROMOTION_L2_256B);

// 2-D row-major tensor [rows][cols] (row pitch in bytes).
inline bool encode_tensor_map_2d(
    CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t cols, uint64_t rows,
    uint64_t row_pitch_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle,
    CUtensorMapL2promotion promotion = CU_TENSOR_MAP_L2_PROMOTION_L2_256B) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t pitches[1] = {row_pitch_bytes};
  const uint32_t box[2] = {box_cols, box_rows};
  return encode_tensor_map(map, dtype, 2, base, dims, pitches, box, swizzle, promotion);
}

}  // namespace gnf4
