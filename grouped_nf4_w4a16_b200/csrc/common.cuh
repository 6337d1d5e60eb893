// common.cuh -- internal definitions shared by the libgnf4 kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/gnf4.h"

namespace gnf4 {

// The 16 NF4 code values (QLoRA / bitsandbytes table) as fp32 bit patterns.
// Index = 4-bit code. These are the fp32 encodings of the published decimal
// values (-1.0, -0.6961928009986877, ..., 0.7229568362236023, 1.0), stored as
// integers so that no decimal-to-binary conversion is involved at build time.
static __constant__ uint32_t kNf4Bits[16] = {
    0xBF800000u, 0xBF3239B1u, 0xBF066B30u, 0xBECA32A0u, 0xBE91A24Du, 0xBE3D353Fu,
    0xBDBA7871u, 0x00000000u, 0x3DA2FAFFu, 0x3E24CAE3u, 0x3E7C04DDu, 0x3EAD033Au,
    0x3EE1A4B8u, 0x3F1007ABu, 0x3F3913B3u, 0x3F800000u};

__device__ __forceinline__ float nf4_value(int code) { return __uint_as_float(kNf4Bits[code]); }

// Workspace header: the first 256 bytes of every workspace.
struct WsHeader {
  uint32_t error;       // GNF4_DEVERR_* bits, OR-ed by kernels
  uint32_t detail;      // first offending index (informational)
  uint32_t reserved[62];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

constexpr size_t kWsHeaderBytes = 256;

__device__ __forceinline__ void report_error(WsHeader *h, uint32_t bits, uint32_t detail) {
  if (h == nullptr) return;
  uint32_t old = atomicOr(&h->error, bits);
  if (old == 0) atomicExch(&h->detail, detail);
}

// Bounded mbarrier wait on the phase with parity `parity`. Returns false if
// the iteration limit ran out (the caller reports GNF4_DEVERR_TIMEOUT).
constexpr uint32_t kSpinLimit = 1u << 26;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

// As mbar_try_wait, but the thread may be suspended (issuing nothing) until
// the phase completes or about `hint_ns` nanoseconds pass.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
  }
  return false;
}

// Named barrier among `count` threads (multiple of 32) of this CTA.
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// 256-bit streaming load (32 bytes) that does not allocate in L1.
__device__ __forceinline__ void ldg256_stream(const void *p, uint32_t (&r)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}

__device__ __forceinline__ uint4 ldg128_stream(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }

// Programmatic dependent launch. Every kernel of the library is launched so
// that it may start while the previous kernel on the stream is still
// running; it then sets up what needs no input (shared-memory tables,
// barriers) and calls pdl_wait() before its first read or write of global
// memory: pdl_wait() returns once the previous kernel has finished and its
// writes are visible (at once when there is no such dependency).
// pdl_trigger() lets the next kernel on the stream start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace gnf4
