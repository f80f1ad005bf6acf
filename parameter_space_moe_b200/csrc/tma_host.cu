// Host-side encoding of TMA tensor maps through the driver entry point (no link-time libcuda).
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_common.cuh"

namespace swimba {

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

bool encode_tmap_2d(CUtensorMap* map, const void* base, int dtype, uint64_t cols, uint64_t rows, uint64_t pitch_bytes,
                    uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const CUtensorMapDataType t = dtype == SWIMBA_BF16  ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                : dtype == SWIMBA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                      : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(map, t, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_3d_slot(CUtensorMap* map, const void* base, int dtype, uint64_t cols, uint64_t slots, uint64_t rows,
                         uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const CUtensorMapDataType t = dtype == SWIMBA_BF16  ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                : dtype == SWIMBA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                      : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const uint64_t eb = dtype == SWIMBA_F32 ? 4 : 2;
  cuuint64_t dims[3] = {cols, slots, rows};
  cuuint64_t strides[2] = {cols * eb, slots * cols * eb};
  cuuint32_t box[3] = {box_cols, 1, box_rows};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, t, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace swimba
