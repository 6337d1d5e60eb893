// lut_mma.cuh -- device helpers shared by the kernels that decode packed
// 4-bit codes through a per-lane replicated shared-memory table into fp16
// MMA fragments (mma.sync m16n8k16, fp32 accumulation): the grouped GEMM's
// decode-regime kernel and the grouped dgrad.
#pragma once

#include <cuda_fp16.h>

#include "sm100.cuh"

namespace gnf4 {

// ------------------------------------------------------------------ PTX

// Not volatile: the compiler may interleave independent accumulation chains.
__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A.B with a zero accumulator in.
__device__ __forceinline__ void mma_f16_z(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// prmt.b32 in its default mode: result byte i = byte (sel nibble i & 7) of
// {b, a} (the selectors used here never set bit 3 of a nibble).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Shared-memory loads at a 32-bit shared-window address. Volatile, so that
// they stay after the barrier wait (volatile asm too) that makes their data
// visible.
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

__device__ __forceinline__ float2 lds_f2(uint32_t a) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
  return v;
}

__device__ __forceinline__ uint4 lds_u4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}

// Table pairs of the 4 packed bytes of `word` (pair p: byte p) from this
// lane's slots: lutlane = shared address of the table (a multiple of 65536)
// + lane * 4, so one byte permute forms the whole address table + byte * 256
// + lane * 4; the remainder pair (PARTS == 2) sits 128 bytes on.
template <int PARTS>
__device__ __forceinline__ void decode_word(uint32_t lutlane, uint32_t word, uint32_t (&hi)[4],
                                            uint32_t (&lo)[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t a = prmt(word, lutlane, 0x7604u | (p << 4));
    if (PARTS == 2) {
      asm("ld.shared.b32 %0, [%2];\n\tld.shared.b32 %1, [%2+128];"
          : "=r"(hi[p]), "=r"(lo[p])
          : "r"(a));
    } else {
      asm("ld.shared.b32 %0, [%1];" : "=r"(hi[p]) : "r"(a));
      lo[p] = 0u;
    }
  }
}

// Bounded wait by every lane of the warp (no divergent branch); the lanes
// agree on the answer by vote.
__device__ __forceinline__ bool warp_wait_all(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag, WsHeader *hdr,
                                              uint64_t limit_ns) {
  return __all_sync(0xffffffffu, wait_bar_lim(bar, parity, abort_flag, hdr, limit_ns));
}

__device__ __forceinline__ bool warp_wait_one(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag, WsHeader *hdr,
                                              uint64_t limit_ns) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wait_bar_lim(bar, parity, abort_flag, hdr, limit_ns) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// One arrival on `bar` for the whole (converged) warp, by an elected lane.
__device__ __forceinline__ void mbar_arrive_elect(uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
      "@p mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

// 16-byte asynchronous copy global -> shared, bypassing L1 (src_bytes 0: zeros).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ uint32_t atomic_add_acq_rel(uint32_t *p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
               : "memory");
  return old;
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  const __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<const uint16_t *>(&b);
}

__device__ __forceinline__ uint32_t half_bits(float v) {
  const __half h = __float2half_rn(v);
  return static_cast<uint32_t>(*reinterpret_cast<const uint16_t *>(&h));
}

// hi[c]: fp16 bits of the NF4 code value (round to nearest even).
__device__ __forceinline__ uint32_t code_hi(int c) { return half_bits(nf4_value(c)); }

// lo[c]: fp16 bits of (NF4[c] - hi[c]) * 2^13 (round to nearest even). The
// remainder is exact in fp32 and at most 2^-12 in magnitude, so the scaled
// value stays below 2; hi + lo * 2^-13 is within 1e-7 relative of NF4[c].
__device__ __forceinline__ uint32_t code_lo(int c) {
  const __half h = __float2half_rn(nf4_value(c));
  return half_bits((nf4_value(c) - __half2float(h)) * 8192.0f);
}

// a / b and a % b for non-negative a, b > 0: 32-bit when both fit (a
// uniform branch; the 64-bit division is a long software sequence).
__device__ __forceinline__ int64_t div_fast(int64_t a, int64_t b) {
  if (((a | b) >> 32) == 0)
    return static_cast<int64_t>(static_cast<uint32_t>(a) / static_cast<uint32_t>(b));
  return a / b;
}

// Stream-K range arithmetic over W tile-stages and P CTAs: CTA b owns
// [range_lo(b), range_lo(b + 1)); cta_of(s) is the CTA that owns stage s.
// (64-bit products while W * P stays below 2^62, which covers every shape
// the host accepts by a wide margin; 128-bit otherwise)
__device__ __forceinline__ int64_t range_lo(int64_t W, int64_t P, int64_t b) {
  if (W < (int64_t{1} << 54)) return div_fast(W * b, P);
  return static_cast<int64_t>((static_cast<unsigned __int128>(W) * b) / P);
}
__device__ __forceinline__ int64_t cta_of(int64_t W, int64_t P, int64_t s) {
  if (W < (int64_t{1} << 54)) return div_fast((s + 1) * P - 1, W);
  return static_cast<int64_t>((static_cast<unsigned __int128>(s + 1) * P - 1) / W);
}


}  // namespace gnf4
