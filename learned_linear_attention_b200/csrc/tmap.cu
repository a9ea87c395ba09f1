// tmap.cu -- host-side TMA tensor-map encoding through the driver entry
// point (no link-time dependency on libcuda).
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"

namespace ttt {

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

static void load_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

int make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                      uint64_t batch, uint64_t row_stride, uint64_t batch_stride,
                      uint32_t box_inner, uint32_t box_rows) {
  std::call_once(g_encode_once, load_encode);
  if (g_encode == nullptr) return -1;
  // a map over no buffer would let a TMA load read address 0: refuse it
  if (base == nullptr) return -1;
  if (rows == 0) rows = 1;
  if (batch == 0) batch = 1;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {row_stride, batch_stride};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

int make_tmap_bf16_3d_sw(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                         uint64_t batch, uint64_t row_stride, uint64_t batch_stride,
                         uint32_t box_inner, uint32_t box_rows, int swizzle_bytes) {
  std::call_once(g_encode_once, load_encode);
  if (g_encode == nullptr) return -1;
  if (base == nullptr) return -1;
  CUtensorMapSwizzle sw;
  switch (swizzle_bytes) {
    case 0: sw = CU_TENSOR_MAP_SWIZZLE_NONE; break;
    case 32: sw = CU_TENSOR_MAP_SWIZZLE_32B; break;
    case 64: sw = CU_TENSOR_MAP_SWIZZLE_64B; break;
    case 128: sw = CU_TENSOR_MAP_SWIZZLE_128B; break;
    default: return -1;
  }
  if (rows == 0) rows = 1;
  if (batch == 0) batch = 1;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {row_stride, batch_stride};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

int make_tmap_bf16_blocked(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                           uint64_t batch, uint64_t row_stride, uint64_t batch_stride,
                           uint32_t box_rows, uint32_t box_blocks) {
  std::call_once(g_encode_once, load_encode);
  if (g_encode == nullptr) return -1;
  if (base == nullptr || inner % 64 != 0) return -1;
  if (rows == 0) rows = 1;
  if (batch == 0) batch = 1;
  cuuint64_t dims[4] = {64, rows, inner / 64, batch};
  cuuint64_t strides[3] = {row_stride, 128, batch_stride};
  cuuint32_t box[4] = {64, box_rows, box_blocks, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

}  // namespace ttt
