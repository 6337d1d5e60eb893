// dequant.cu -- gnf4_dequant_debug: materialise NF4[code] * absmax.
//
// Off the hot path: a debugging/parity aid, the analogue of the package's
// pure-torch reference decode ("grouped-nf4-gemm" package page, "Owns": pack
// and pure-torch reference operations). Each element is one IEEE fp32
// multiply (__fmul_rn); the bf16 output rounds that product once (RNE).
//
// One thread handles 16 packed bytes = 32 codes = half of one 64-element
// absmax block (K % 64 == 0, so a 16-byte chunk never straddles a row or a
// block). Grid-stride loop, 128-bit loads and stores.
#include "launch.h"

namespace gnf4 {
namespace {

template <bool kBf16>
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t *__restrict__ w,
                                                      const float *__restrict__ absmax,
                                                      int64_t nchunks, int32_t K,
                                                      void *__restrict__ out) {
  __shared__ float lut[16];
  pdl_trigger();
  if (threadIdx.x < 16) lut[threadIdx.x] = nf4_value(threadIdx.x);
  __syncthreads();
  pdl_wait();   // inputs may come from the previous kernel on the stream
  const int64_t chunks_per_row = K / 32;
  const int64_t blocks_per_row = K / 64;
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < nchunks;
       c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = c / chunks_per_row;
    const int64_t j = c - row * chunks_per_row;
    const uint4 packed = ldg128_stream(w + c * 16);
    const float a = absmax[row * blocks_per_row + j / 2];
    const uint32_t words[4] = {packed.x, packed.y, packed.z, packed.w};
    float v[32];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const uint32_t byte = (words[q] >> (8 * p)) & 0xFFu;
        v[8 * q + 2 * p] = __fmul_rn(lut[byte >> 4], a);        // even k: high nibble
        v[8 * q + 2 * p + 1] = __fmul_rn(lut[byte & 0xFu], a);  // odd k: low nibble
      }
    }
    const int64_t base = row * K + j * 32;
    if constexpr (kBf16) {
      uint4 *o = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + base);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t r[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * i + 2 * h], v[8 * i + 2 * h + 1]);
          r[h] = *reinterpret_cast<const uint32_t *>(&b2);
        }
        o[i] = make_uint4(r[0], r[1], r[2], r[3]);
      }
    } else {
      float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(out) + base);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
  }
}

}  // namespace

cudaError_t launch_dequant(const uint8_t *w, const float *absmax, int64_t rows, int32_t K,
                           int out_bf16, void *out, cudaStream_t stream) {
  const int64_t nchunks = rows * (K / 32);
  if (nchunks == 0) return cudaSuccess;
  const int threads = 256;
  int64_t want = (nchunks + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
  const int grid = static_cast<int>(want < cap ? want : cap);
  if (out_bf16)
    return launch_pdl(dequant_kernel<true>, dim3(grid), dim3(threads), 0, stream, w, absmax,
                      nchunks, K, out);
  return launch_pdl(dequant_kernel<false>, dim3(grid), dim3(threads), 0, stream, w, absmax,
                    nchunks, K, out);
}

}  // namespace gnf4
