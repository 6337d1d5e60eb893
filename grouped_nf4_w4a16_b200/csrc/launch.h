// launch.h -- internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstring>
#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

#include "common.cuh"

namespace gnf4 {

// Grouped GEMM problem as seen by the kernels (all pointers device memory).
struct GemmArgs {
  const uint16_t *x;        // bf16 [M][K] (nullptr when the rows are gathered)
  const uint8_t *w;         // [E][N][K/2]
  const float *absmax;      // [E][N][K/64] fp32 (NF4 with fp32 absmax; else nullptr)
  const void *scales;       // the block scales in their own encoding (== absmax for fp32)
  int32_t fmt = GNF4_FMT_NF4;           // gnf4_format
  int32_t scale_dtype = GNF4_SCALE_F32; // gnf4_scale_dtype
  int32_t epi = GNF4_EPI_NONE;          // gnf4_epilogue
  float alpha = 0.0f, limit = 0.0f;     // GNF4_EPI_SWIGLU_INTERLEAVED
  const uint16_t *hidden = nullptr;     // gather: [n_tokens][K]; row i = hidden[sorted_idx[i] / top_k]
  const int32_t *sorted_idx = nullptr;
  int64_t n_tokens = 0;
  int32_t top_k = 1;
  const int32_t *sizes;     // [G]
  const int32_t *expert_ids;// [G]
  int32_t G;
  int64_t M;
  int32_t N;
  int32_t K;
  int32_t E;
  int32_t swiglu;           // 0 / 1
  uint16_t *y;              // bf16 [M][N] or [M][N/2]
  void *workspace;
  size_t ws_bytes;
};

// ---- moe_align (moe_align.cu)
size_t moe_align_smem_bytes(int32_t E);
cudaError_t launch_moe_align(const int32_t *topk, int32_t S, int32_t E, int32_t *sorted_idx,
                             int32_t *sizes, int32_t *expert_ids, int32_t *num_groups,
                             WsHeader *hdr, cudaStream_t stream);

// ---- dequant_debug (dequant.cu)
cudaError_t launch_dequant(const uint8_t *w, const float *absmax, int64_t rows, int32_t K,
                           int out_bf16, void *out, cudaStream_t stream);

// ---- decode-regime grouped GEMM (decode_gemm.cu)
size_t decode_workspace_bytes(int64_t M, int32_t N, int32_t K, int32_t G, int32_t swiglu);
// Leading bytes of a decode workspace that must be zero before a launch
// (header and split-tile counters; the partial sums behind them need not be).
size_t decode_zero_prefix_bytes(int64_t M, int32_t N, int32_t G, int32_t swiglu);
cudaError_t launch_decode_gemm(const GemmArgs &a, cudaStream_t stream);

// ---- prefill-regime grouped GEMM (prefill_gemm.cu)
size_t prefill_workspace_bytes(int64_t M, int32_t N, int32_t K, int32_t G, int32_t swiglu);
// Whether the tensor-core kernel runs this combination of format, scales,
// epilogue and gather.
bool prefill_supports(const GemmArgs &a);
cudaError_t launch_prefill_gemm(const GemmArgs &a, cudaStream_t stream);

// ---- router top-k and weighted combine (router.cu)
size_t combine_workspace_bytes(int64_t S);
cudaError_t launch_router_topk(const float *logits, int64_t T, int32_t E, int32_t k, int32_t renorm,
                               int32_t *ids, float *weights, cudaStream_t stream);
cudaError_t launch_moe_combine(const uint16_t *y, const int32_t *sorted_idx, const float *w,
                               int64_t T, int32_t k, int32_t H, uint16_t *out, void *workspace,
                               cudaStream_t stream);

// ---- grouped dgrad (dgrad.cu)
size_t dgrad_workspace_bytes();
size_t dgrad_zero_prefix_bytes();
cudaError_t launch_grouped_dgrad(const uint16_t *dy, const uint8_t *w, const float *absmax,
                                 const int32_t *sizes, const int32_t *expert_ids, int32_t G,
                                 int64_t M, int32_t N, int32_t K, int32_t E, uint16_t *dx,
                                 WsHeader *hdr, cudaStream_t stream);

// ---- entry-point plumbing shared by gnf4_grouped_gemm and its no-allocation
// variant (api.cu): every host-side check except those of the workspace, in
// the order gnf4_grouped_gemm reports them, filling `out` (workspace unset)
// and the kernel to run (*use_out = GNF4_MODE_DECODE or GNF4_MODE_PREFILL;
// -1 with GNF4_OK when M == 0 and there is nothing to launch).
gnf4_status check_grouped_gemm(const uint16_t *x, const uint8_t *w, const float *absmax,
                               const int32_t *sizes, const int32_t *expert_ids, int32_t G,
                               int64_t M, int32_t N, int32_t K, int32_t E, int32_t blocksize,
                               int32_t epilogue, int32_t mode, uint16_t *y, GemmArgs *out,
                               int32_t *use_out);
gnf4_status launch_grouped_gemm(const GemmArgs &a, int32_t use, cudaStream_t s);
// The same for gnf4_grouped_gemm_ex's descriptor.
gnf4_status check_grouped_gemm_ex(const gnf4_gemm_desc *d, GemmArgs *out, int32_t *use_out);

// Number of SMs of the current device (cached per device).
int device_sm_count();

// Launches `kernel` on `stream` with programmatic stream serialization, so it
// may start before the previous kernel on the stream has finished (the
// kernel itself waits with pdl_wait() before touching global memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace gnf4
