// noalloc.cu -- gnf4_grouped_gemm_noalloc: the decode grouped GEMM for callers
// that cannot allocate device memory.
//
// Some callers may not call cudaMalloc at all: a plugin running inside a host
// application that owns every byte of device memory through its own
// pre-planned pool, or a latency-critical path that cannot pay for the
// implicit synchronisation an allocation may bring. gnf4_grouped_gemm needs a
// caller-provided workspace (the status word the kernels report device-side
// errors in); this entry point instead uses a scratch array compiled into the
// library, so the caller passes only inputs and outputs.
//
// The array is reserved on every GPU that loads the library, for the life of
// the process. In host code its name only denotes a host-side stand-in, not a
// device address, so the address handed to the kernel is looked up once per
// device with cudaGetSymbolAddress (with that device current).
#include <mutex>

#include "launch.h"

namespace gnf4 {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GNF4_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_lock;
void *g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device, looked up on the
// first call for that device.
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> guard(g_scratch_lock);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace gnf4

using namespace gnf4;

extern "C" gnf4_status gnf4_grouped_gemm_noalloc(const uint16_t *x, const uint8_t *w,
                                                 const float *absmax, const int32_t *sizes,
                                                 const int32_t *expert_ids, int32_t G, int64_t M,
                                                 int32_t N, int32_t K, int32_t E,
                                                 int32_t blocksize, int32_t epilogue, uint16_t *y,
                                                 gnf4_stream_t stream) {
  // Every argument check of gnf4_grouped_gemm (decode mode) comes first, so a
  // refused call puts no work on the caller's stream.
  GemmArgs a;
  int32_t use = 0;
  const gnf4_status st = check_grouped_gemm(x, w, absmax, sizes, expert_ids, G, M, N, K, E,
                                            blocksize, epilogue, GNF4_MODE_DECODE, y, &a, &use);
  if (st != GNF4_OK || use < 0) return st;

  // the decode kernel's workspace must fit the scratch array
  const size_t need = decode_workspace_bytes(M, N, K, G, a.swiglu);
  if (need == 0 || need > GNF4_NOALLOC_SCRATCH_BYTES) return GNF4_ERR_SCRATCH_LIMIT;

  void *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return GNF4_ERR_CUDA;

  // The array still holds the previous call's contents: the part the kernel
  // needs at zero (status word, counters) is cleared on the caller's stream.
  const size_t clear = decode_zero_prefix_bytes(M, N, G, a.swiglu);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, clear, s) != cudaSuccess) return GNF4_ERR_CUDA;

  a.workspace = scratch;
  a.ws_bytes = GNF4_NOALLOC_SCRATCH_BYTES;
  return launch_grouped_gemm(a, GNF4_MODE_DECODE, s);
}
