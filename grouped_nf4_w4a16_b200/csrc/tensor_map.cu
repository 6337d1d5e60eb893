// tensor_map.cu -- host-side encoding of the TMA tensor maps (driver entry
// point resolved through the runtime, so the library links no libcuda).
#include "sm100.cuh"

namespace gnf4 {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

bool encode_tensor_map(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *base,
                       const uint64_t *dims, const uint64_t *pitches, const uint32_t *box,
                       CUtensorMapSwizzle swizzle, CUtensorMapL2promotion promotion) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode_fn();
  if (encode == nullptr || rank < 2 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = static_cast<cuuint64_t>(dims[i]);
    b[i] = static_cast<cuuint32_t>(box[i]);
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = static_cast<cuuint64_t>(pitches[i]);
  const CUresult r = encode(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void *>(base), d,
                            st, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promotion,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace gnf4
