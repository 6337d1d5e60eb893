// api.cu -- the extern "C" entry points of libgnf4 (see include/gnf4.h).
//
// Host-side argument checks (synchronous, before any launch), mode choice and
// kernel launches on the caller's stream. No allocation, no synchronisation
// (except gnf4_read_device_status), no host fallback: the package page
// "grouped-nf4-gemm" ("Do not use this when") states that nothing falls back
// silently on the CPU and host tensors are refused with an error.
#include <climits>
#include <cstring>

#include "launch.h"

namespace gnf4 {

int device_sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

namespace {

bool is_device_pointer(const void *p) {
  cudaPointerAttributes attr;
  std::memset(&attr, 0, sizeof(attr));
  const cudaError_t err = cudaPointerGetAttributes(&attr, p);
  if (err != cudaSuccess) {
    (void)cudaGetLastError();   // clear the sticky error of a bad query
    return false;
  }
  return attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

gnf4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? GNF4_OK : GNF4_ERR_CUDA; }

// Mean rows per possible group above which the tensor-core kernel is used.
constexpr int64_t kPrefillMeanRows = 64;

}  // namespace

gnf4_status check_grouped_gemm(const uint16_t *x, const uint8_t *w, const float *absmax,
                               const int32_t *sizes, const int32_t *expert_ids, int32_t G,
                               int64_t M, int32_t N, int32_t K, int32_t E, int32_t blocksize,
                               int32_t epilogue, int32_t mode, uint16_t *y, GemmArgs *out,
                               int32_t *use_out) {
  *use_out = -1;
  if (!x || !w || !absmax || !sizes || !expert_ids || !y) return GNF4_ERR_INVALID_ARGUMENT;
  if (M < 0 || N < 1 || K < 1 || E < 1 || G < 1) return GNF4_ERR_INVALID_ARGUMENT;
  if (epilogue != GNF4_EPI_NONE && epilogue != GNF4_EPI_SWIGLU) return GNF4_ERR_INVALID_ARGUMENT;
  if (mode != GNF4_MODE_AUTO && mode != GNF4_MODE_DECODE && mode != GNF4_MODE_PREFILL)
    return GNF4_ERR_INVALID_ARGUMENT;
  if (blocksize != GNF4_BLOCKSIZE || K % GNF4_BLOCKSIZE != 0) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (E > GNF4_MAX_EXPERTS || G > GNF4_MAX_EXPERTS) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (epilogue == GNF4_EPI_SWIGLU && (N % 2) != 0) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (M >= INT_MAX) return GNF4_ERR_UNSUPPORTED_SHAPE;
  // tensor-copy coordinates are 32-bit: every weight row index a copy can
  // start at (up to one expert plus one box past the stack) must fit
  if (static_cast<int64_t>(E) * N + N + 256 >= INT_MAX) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return GNF4_OK;   // nothing to launch (*use_out stays -1)
  if (!is_device_pointer(x) || !is_device_pointer(w) || !is_device_pointer(absmax) ||
      !is_device_pointer(sizes) || !is_device_pointer(expert_ids) || !is_device_pointer(y))
    return GNF4_ERR_HOST_POINTER;
  if (!aligned(x, 32) || !aligned(w, 32) || !aligned(y, 32) || !aligned(absmax, 4) ||
      !aligned(sizes, 4) || !aligned(expert_ids, 4))
    return GNF4_ERR_MISALIGNED;
  GemmArgs &a = *out;
  a.x = x; a.w = w; a.absmax = absmax; a.sizes = sizes; a.expert_ids = expert_ids;
  a.G = G; a.M = M; a.N = N; a.K = K; a.E = E; a.swiglu = (epilogue == GNF4_EPI_SWIGLU);
  a.y = y; a.workspace = nullptr; a.ws_bytes = 0;
  a.scales = absmax; a.epi = epilogue;
  const bool pf_ok = prefill_supports(a);
  int32_t use = mode;
  if (use == GNF4_MODE_AUTO) {
    const int64_t groups = G < E ? G : E;
    use = (M > kPrefillMeanRows * groups && pf_ok) ? GNF4_MODE_PREFILL : GNF4_MODE_DECODE;
  }
  if (use == GNF4_MODE_PREFILL && !pf_ok) return GNF4_ERR_UNSUPPORTED_SHAPE;
  *use_out = use;
  return GNF4_OK;
}

gnf4_status check_grouped_gemm_ex(const gnf4_gemm_desc *d, GemmArgs *out, int32_t *use_out) {
  *use_out = -1;
  if (!d) return GNF4_ERR_INVALID_ARGUMENT;
  if (d->struct_bytes != sizeof(gnf4_gemm_desc)) return GNF4_ERR_INVALID_ARGUMENT;
  const bool gather = d->x == nullptr;
  if (gather ? (!d->hidden || !d->sorted_idx) : (d->hidden != nullptr))
    return GNF4_ERR_INVALID_ARGUMENT;
  if (!d->w || !d->scales || !d->sizes || !d->expert_ids || !d->y) return GNF4_ERR_INVALID_ARGUMENT;
  if (d->M < 0 || d->N < 1 || d->K < 1 || d->E < 1 || d->G < 1) return GNF4_ERR_INVALID_ARGUMENT;
  if (d->format != GNF4_FMT_NF4 && d->format != GNF4_FMT_MXFP4) return GNF4_ERR_INVALID_ARGUMENT;
  if (d->format == GNF4_FMT_NF4 ? (d->scale_dtype != GNF4_SCALE_F32 &&
                                   d->scale_dtype != GNF4_SCALE_BF16)
                                : d->scale_dtype != GNF4_SCALE_E8M0)
    return GNF4_ERR_INVALID_ARGUMENT;
  if (d->epilogue != GNF4_EPI_NONE && d->epilogue != GNF4_EPI_SWIGLU &&
      d->epilogue != GNF4_EPI_SWIGLU_INTERLEAVED)
    return GNF4_ERR_INVALID_ARGUMENT;
  if (d->epilogue == GNF4_EPI_SWIGLU_INTERLEAVED &&
      !(d->swiglu_limit > 0.0f && d->swiglu_limit < 3.0e38f && d->swiglu_alpha == d->swiglu_alpha))
    return GNF4_ERR_INVALID_ARGUMENT;
  if (d->mode != GNF4_MODE_AUTO && d->mode != GNF4_MODE_DECODE && d->mode != GNF4_MODE_PREFILL)
    return GNF4_ERR_INVALID_ARGUMENT;
  if (gather && (d->top_k < 1 || d->n_tokens < 0)) return GNF4_ERR_INVALID_ARGUMENT;
  if (d->K % GNF4_BLOCKSIZE != 0) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (d->E > GNF4_MAX_EXPERTS || d->G > GNF4_MAX_EXPERTS) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (d->epilogue != GNF4_EPI_NONE && (d->N % 2) != 0) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (d->M >= INT_MAX) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (gather && d->n_tokens * static_cast<int64_t>(d->top_k) >= INT_MAX)
    return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<int64_t>(d->E) * d->N + d->N + 256 >= INT_MAX) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (d->M == 0) return GNF4_OK;
  const void *xs = gather ? static_cast<const void *>(d->hidden) : static_cast<const void *>(d->x);
  if (!is_device_pointer(xs) || !is_device_pointer(d->w) || !is_device_pointer(d->scales) ||
      !is_device_pointer(d->sizes) || !is_device_pointer(d->expert_ids) ||
      !is_device_pointer(d->y) || (gather && !is_device_pointer(d->sorted_idx)))
    return GNF4_ERR_HOST_POINTER;
  if (!aligned(xs, 32) || !aligned(d->w, 32) || !aligned(d->y, 32) || !aligned(d->scales, 4) ||
      !aligned(d->sizes, 4) || !aligned(d->expert_ids, 4) ||
      (gather && !aligned(d->sorted_idx, 4)))
    return GNF4_ERR_MISALIGNED;
  GemmArgs &a = *out;
  a.x = d->x; a.w = d->w;
  a.absmax = (d->format == GNF4_FMT_NF4 && d->scale_dtype == GNF4_SCALE_F32)
                 ? static_cast<const float *>(d->scales) : nullptr;
  a.scales = d->scales;
  a.fmt = d->format; a.scale_dtype = d->scale_dtype; a.epi = d->epilogue;
  a.alpha = d->swiglu_alpha; a.limit = d->swiglu_limit;
  a.hidden = gather ? d->hidden : nullptr;
  a.sorted_idx = gather ? d->sorted_idx : nullptr;
  a.n_tokens = gather ? d->n_tokens : 0;
  a.top_k = gather ? d->top_k : 1;
  a.sizes = d->sizes; a.expert_ids = d->expert_ids;
  a.G = d->G; a.M = d->M; a.N = d->N; a.K = d->K; a.E = d->E;
  a.swiglu = d->epilogue != GNF4_EPI_NONE;
  a.y = d->y; a.workspace = nullptr; a.ws_bytes = 0;
  const bool pf_ok = prefill_supports(a);
  int32_t use = d->mode;
  if (use == GNF4_MODE_AUTO) {
    const int64_t groups = d->G < d->E ? d->G : d->E;
    use = (d->M > kPrefillMeanRows * groups && pf_ok) ? GNF4_MODE_PREFILL : GNF4_MODE_DECODE;
  }
  if (use == GNF4_MODE_PREFILL && !pf_ok) return GNF4_ERR_UNSUPPORTED_SHAPE;
  *use_out = use;
  return GNF4_OK;
}

gnf4_status launch_grouped_gemm(const GemmArgs &a, int32_t use, cudaStream_t s) {
  const cudaError_t e =
      use == GNF4_MODE_PREFILL ? launch_prefill_gemm(a, s) : launch_decode_gemm(a, s);
  if (e == cudaErrorNotSupported) return GNF4_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(e);
}

}  // namespace gnf4

using namespace gnf4;

extern "C" {

int32_t gnf4_version(void) { return GNF4_VERSION; }

const char *gnf4_status_string(gnf4_status s) {
  switch (s) {
    case GNF4_OK: return "GNF4_OK";
    case GNF4_ERR_INVALID_ARGUMENT: return "GNF4_ERR_INVALID_ARGUMENT";
    case GNF4_ERR_HOST_POINTER: return "GNF4_ERR_HOST_POINTER (a pointer is not device memory; there is no host path)";
    case GNF4_ERR_UNSUPPORTED_SHAPE: return "GNF4_ERR_UNSUPPORTED_SHAPE";
    case GNF4_ERR_WORKSPACE_TOO_SMALL: return "GNF4_ERR_WORKSPACE_TOO_SMALL";
    case GNF4_ERR_CUDA: return "GNF4_ERR_CUDA";
    case GNF4_ERR_DEVICE_METADATA: return "GNF4_ERR_DEVICE_METADATA";
    case GNF4_ERR_TIMEOUT: return "GNF4_ERR_TIMEOUT";
    case GNF4_ERR_MISALIGNED: return "GNF4_ERR_MISALIGNED";
    case GNF4_ERR_SCRATCH_LIMIT:
      return "GNF4_ERR_SCRATCH_LIMIT (problem needs more than the fixed scratch of "
             "gnf4_grouped_gemm_noalloc; use gnf4_grouped_gemm with a workspace)";
  }
  return "GNF4_ERR_UNKNOWN";
}

size_t gnf4_workspace_bytes(int32_t op, int64_t M, int32_t N, int32_t K, int32_t E, int32_t G) {
  (void)E;
  if (op == GNF4_OP_MOE_ALIGN) return kWsHeaderBytes;
  if (op == GNF4_OP_MOE_COMBINE) return M < 0 ? 0 : combine_workspace_bytes(M);
  if (op == GNF4_OP_GROUPED_DGRAD) return dgrad_workspace_bytes();
  if (op != GNF4_OP_GROUPED_GEMM || M < 0 || N < 1 || K < 1 || G < 1) return 0;
  const size_t d = decode_workspace_bytes(M, N, K, G, 1);
  const size_t d2 = decode_workspace_bytes(M, N, K, G, 0);
  const size_t p = prefill_workspace_bytes(M, N, K, G, 0);
  const size_t p2 = prefill_workspace_bytes(M, N, K, G, 1);
  size_t r = d > d2 ? d : d2;
  if (p > r) r = p;
  if (p2 > r) r = p2;
  return r;
}

gnf4_status gnf4_moe_align(const int32_t *topk_ids, int64_t T, int32_t top_k, int32_t E,
                           int32_t *sorted_idx, int32_t *sizes, int32_t *expert_ids,
                           int32_t *num_groups, void *workspace, size_t ws_bytes,
                           gnf4_stream_t stream) {
  if (T < 0 || top_k < 1 || E < 1) return GNF4_ERR_INVALID_ARGUMENT;
  if ((T > 0 && (!topk_ids || !sorted_idx)) || !sizes || !expert_ids || !num_groups || !workspace)
    return GNF4_ERR_INVALID_ARGUMENT;
  if (E > GNF4_MAX_EXPERTS || T * static_cast<int64_t>(top_k) >= INT_MAX) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (ws_bytes < kWsHeaderBytes) return GNF4_ERR_WORKSPACE_TOO_SMALL;
  const bool need_ids = T > 0;
  if ((need_ids && (!is_device_pointer(topk_ids) || !is_device_pointer(sorted_idx))) ||
      !is_device_pointer(sizes) || !is_device_pointer(expert_ids) ||
      !is_device_pointer(num_groups) || !is_device_pointer(workspace))
    return GNF4_ERR_HOST_POINTER;
  if ((need_ids && (!aligned(topk_ids, 4) || !aligned(sorted_idx, 4))) || !aligned(sizes, 4) ||
      !aligned(expert_ids, 4) || !aligned(num_groups, 4) || !aligned(workspace, 16))
    return GNF4_ERR_MISALIGNED;
  const int32_t S = static_cast<int32_t>(T * top_k);
  return from_cuda(launch_moe_align(topk_ids, S, E, sorted_idx, sizes, expert_ids, num_groups,
                                    static_cast<WsHeader *>(workspace),
                                    reinterpret_cast<cudaStream_t>(stream)));
}

gnf4_status gnf4_grouped_gemm(const uint16_t *x, const uint8_t *w, const float *absmax,
                              const int32_t *sizes, const int32_t *expert_ids, int32_t G,
                              int64_t M, int32_t N, int32_t K, int32_t E, int32_t blocksize,
                              int32_t epilogue, int32_t mode, uint16_t *y, void *workspace,
                              size_t ws_bytes, gnf4_stream_t stream) {
  if (!workspace) return GNF4_ERR_INVALID_ARGUMENT;
  GemmArgs a;
  int32_t use = 0;
  const gnf4_status st = check_grouped_gemm(x, w, absmax, sizes, expert_ids, G, M, N, K, E,
                                            blocksize, epilogue, mode, y, &a, &use);
  if (st != GNF4_OK || use < 0) return st;
  if (!is_device_pointer(workspace)) return GNF4_ERR_HOST_POINTER;
  if (!aligned(workspace, 32)) return GNF4_ERR_MISALIGNED;
  a.workspace = workspace;
  a.ws_bytes = ws_bytes;
  // the workspace the chosen kernel needs (gnf4_workspace_bytes covers every mode)
  const size_t need = use == GNF4_MODE_PREFILL ? prefill_workspace_bytes(M, N, K, G, a.swiglu)
                                               : decode_workspace_bytes(M, N, K, G, a.swiglu);
  if (ws_bytes < need) return GNF4_ERR_WORKSPACE_TOO_SMALL;
  return launch_grouped_gemm(a, use, reinterpret_cast<cudaStream_t>(stream));
}

gnf4_status gnf4_grouped_gemm_ex(const gnf4_gemm_desc *desc, void *workspace, size_t ws_bytes,
                                 gnf4_stream_t stream) {
  if (!workspace) return GNF4_ERR_INVALID_ARGUMENT;
  GemmArgs a;
  int32_t use = 0;
  const gnf4_status st = check_grouped_gemm_ex(desc, &a, &use);
  if (st != GNF4_OK || use < 0) return st;
  if (!is_device_pointer(workspace)) return GNF4_ERR_HOST_POINTER;
  if (!aligned(workspace, 32)) return GNF4_ERR_MISALIGNED;
  a.workspace = workspace;
  a.ws_bytes = ws_bytes;
  const size_t need = use == GNF4_MODE_PREFILL
                          ? prefill_workspace_bytes(a.M, a.N, a.K, a.G, a.swiglu)
                          : decode_workspace_bytes(a.M, a.N, a.K, a.G, a.swiglu);
  if (ws_bytes < need) return GNF4_ERR_WORKSPACE_TOO_SMALL;
  return launch_grouped_gemm(a, use, reinterpret_cast<cudaStream_t>(stream));
}

gnf4_status gnf4_dequant_debug(const uint8_t *w, const float *absmax, int64_t rows, int32_t K,
                               int32_t blocksize, int32_t out_dtype, void *out,
                               gnf4_stream_t stream) {
  if (!w || !absmax || !out) return GNF4_ERR_INVALID_ARGUMENT;
  if (rows < 0 || K < 1) return GNF4_ERR_INVALID_ARGUMENT;
  if (out_dtype != GNF4_OUT_F32 && out_dtype != GNF4_OUT_BF16) return GNF4_ERR_INVALID_ARGUMENT;
  if (blocksize != GNF4_BLOCKSIZE || K % GNF4_BLOCKSIZE != 0) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return GNF4_OK;
  if (!is_device_pointer(w) || !is_device_pointer(absmax) || !is_device_pointer(out))
    return GNF4_ERR_HOST_POINTER;
  if (!aligned(w, 16) || !aligned(out, 16) || !aligned(absmax, 4)) return GNF4_ERR_MISALIGNED;
  return from_cuda(launch_dequant(w, absmax, rows, K, out_dtype == GNF4_OUT_BF16 ? 1 : 0, out,
                                  reinterpret_cast<cudaStream_t>(stream)));
}

gnf4_status gnf4_grouped_dgrad(const uint16_t *dy, const uint8_t *w, const float *absmax,
                               const int32_t *sizes, const int32_t *expert_ids, int32_t G,
                               int64_t M, int32_t N, int32_t K, int32_t E, int32_t blocksize,
                               uint16_t *dx, void *workspace, size_t ws_bytes,
                               gnf4_stream_t stream) {
  if (!dy || !w || !absmax || !sizes || !expert_ids || !dx || !workspace)
    return GNF4_ERR_INVALID_ARGUMENT;
  if (M < 0 || N < 1 || K < 1 || E < 1 || G < 1) return GNF4_ERR_INVALID_ARGUMENT;
  if (blocksize != GNF4_BLOCKSIZE || K % GNF4_BLOCKSIZE != 0) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (E > GNF4_MAX_EXPERTS || G > GNF4_MAX_EXPERTS || M >= INT_MAX) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (N % 8 != 0 || static_cast<int64_t>(E) * N + 256 >= INT_MAX) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (ws_bytes < dgrad_workspace_bytes()) return GNF4_ERR_WORKSPACE_TOO_SMALL;
  if (M == 0) return GNF4_OK;
  if (!is_device_pointer(dy) || !is_device_pointer(w) || !is_device_pointer(absmax) ||
      !is_device_pointer(sizes) || !is_device_pointer(expert_ids) || !is_device_pointer(dx) ||
      !is_device_pointer(workspace))
    return GNF4_ERR_HOST_POINTER;
  if (!aligned(dy, 16) || !aligned(w, 16) || !aligned(dx, 2) || !aligned(absmax, 4) ||
      !aligned(sizes, 4) || !aligned(expert_ids, 4) || !aligned(workspace, 16))
    return GNF4_ERR_MISALIGNED;
  return from_cuda(launch_grouped_dgrad(dy, w, absmax, sizes, expert_ids, G, M, N, K, E, dx,
                                        static_cast<WsHeader *>(workspace),
                                        reinterpret_cast<cudaStream_t>(stream)));
}

gnf4_status gnf4_router_topk(const float *logits, int64_t T, int32_t E, int32_t top_k,
                             int32_t renormalize, int32_t *topk_ids, float *topk_weights,
                             gnf4_stream_t stream) {
  if (T < 0 || E < 1 || top_k < 1) return GNF4_ERR_INVALID_ARGUMENT;
  if (renormalize != 0 && renormalize != 1) return GNF4_ERR_INVALID_ARGUMENT;
  if (E > GNF4_MAX_EXPERTS || top_k > GNF4_MAX_TOPK || top_k > E) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (T * static_cast<int64_t>(E) >= (static_cast<int64_t>(1) << 62)) return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return GNF4_OK;
  if (!logits || !topk_ids || !topk_weights) return GNF4_ERR_INVALID_ARGUMENT;
  if (!is_device_pointer(logits) || !is_device_pointer(topk_ids) || !is_device_pointer(topk_weights))
    return GNF4_ERR_HOST_POINTER;
  if (!aligned(logits, 4) || !aligned(topk_ids, 4) || !aligned(topk_weights, 4))
    return GNF4_ERR_MISALIGNED;
  return from_cuda(launch_router_topk(logits, T, E, top_k, renormalize, topk_ids, topk_weights,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

gnf4_status gnf4_moe_combine(const uint16_t *y, const int32_t *sorted_idx,
                             const float *topk_weights, int64_t T, int32_t top_k, int32_t H,
                             uint16_t *out, void *workspace, size_t ws_bytes,
                             gnf4_stream_t stream) {
  if (T < 0 || top_k < 1 || H < 1) return GNF4_ERR_INVALID_ARGUMENT;
  if (top_k > GNF4_MAX_TOPK || T * static_cast<int64_t>(top_k) >= INT_MAX)
    return GNF4_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return GNF4_OK;
  if (!y || !sorted_idx || !topk_weights || !out || !workspace) return GNF4_ERR_INVALID_ARGUMENT;
  if (ws_bytes < combine_workspace_bytes(T * top_k)) return GNF4_ERR_WORKSPACE_TOO_SMALL;
  if (!is_device_pointer(y) || !is_device_pointer(sorted_idx) || !is_device_pointer(topk_weights) ||
      !is_device_pointer(out) || !is_device_pointer(workspace))
    return GNF4_ERR_HOST_POINTER;
  if (!aligned(y, 2) || !aligned(out, 2) || !aligned(sorted_idx, 4) || !aligned(topk_weights, 4) ||
      !aligned(workspace, 16))
    return GNF4_ERR_MISALIGNED;
  return from_cuda(launch_moe_combine(y, sorted_idx, topk_weights, T, top_k, H, out, workspace,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

gnf4_status gnf4_read_device_status(void *workspace, int32_t clear, uint32_t *error_bits,
                                    gnf4_stream_t stream) {
  if (!workspace) return GNF4_ERR_INVALID_ARGUMENT;
  if (!is_device_pointer(workspace)) return GNF4_ERR_HOST_POINTER;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t h[2] = {0, 0};
  cudaError_t e = cudaMemcpyAsync(h, workspace, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && clear) {
    e = cudaMemsetAsync(workspace, 0, sizeof(h), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  }
  if (e != cudaSuccess) return GNF4_ERR_CUDA;
  if (error_bits) *error_bits = h[0];
  if (h[0] & (GNF4_DEVERR_SIZES | GNF4_DEVERR_EXPERT | GNF4_DEVERR_TOPK | GNF4_DEVERR_CAPACITY |
              GNF4_DEVERR_SLOT))
    return GNF4_ERR_DEVICE_METADATA;
  if (h[0] & GNF4_DEVERR_TIMEOUT) return GNF4_ERR_TIMEOUT;
  return GNF4_OK;
}

}  // extern "C"
