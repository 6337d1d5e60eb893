// prefill_gemm.cu -- prefill-regime grouped NF4 GEMM (tensor cores).
// The tcgen05/TMEM kernel lands here; until then PREFILL mode is refused.
#include "launch.h"

namespace gnf4 {

size_t prefill_workspace_bytes(int64_t M, int32_t N, int32_t K, int32_t G, int32_t swiglu) {
  (void)M; (void)N; (void)K; (void)G; (void)swiglu;
  return 0;
}

cudaError_t launch_prefill_gemm(const GemmArgs &a, cudaStream_t stream) {
  (void)a; (void)stream;
  return cudaErrorNotSupported;
}

}  // namespace gnf4
