// tma.cu -- TMA tensor-map encoding through the driver entry point (no libcuda link).
#include <cudaTypedefs.h>

#include <mutex>

#include "llsa_internal.cuh"

namespace llsa {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

cudaError_t make_token_map_box(CUtensorMap* map, const void* base, int64_t rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if (((uintptr_t)base & 15u) != 0 || box_rows < 1 || box_rows > 256) return cudaErrorInvalidValue;
  cuuint64_t dims[2] = {64, (cuuint64_t)rows};
  cuuint64_t strides[1] = {64 * sizeof(__nv_bfloat16)};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_run_maps(RunMaps* maps, const void* base, int64_t rows) {
  for (int r = 0; r < kRunMax; ++r) {
    cudaError_t e = make_token_map_box(&maps->m[r], base, rows, 16 * (r + 1));
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace llsa
