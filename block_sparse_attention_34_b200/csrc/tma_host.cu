// Host-side TMA tensor-map encoding for the row-gather loads of the sm_100a
// kernels.  The driver's cuTensorMapEncodeTiled is reached through the
// runtime's driver entry-point query, so the library needs no link-time
// dependency on libcuda.
#include <cudaTypedefs.h>

#include <mutex>

#include "sm100.cuh"

namespace paro {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

bool encode_gather_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       int elem_bytes, uint32_t box_cols) {
  return encode_tile_map(map, base, rows, cols, elem_bytes, box_cols, 1);
}

bool encode_tile_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                     int elem_bytes, uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  if (box_cols * (uint32_t)elem_bytes != 128u || box_rows < 1 || box_rows > 256) return false;
  if (rows == 0 || rows > 0xFFFFFFFFull || (reinterpret_cast<uintptr_t>(base) & 15u) != 0)
    return false;
  const CUtensorMapDataType dt =
      elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (cuuint64_t)elem_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace paro
