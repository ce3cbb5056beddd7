// Host helpers of the tensor-core attention passes: TMA descriptors and the configurations
// the tcgen05 kernels cover (bf16, head_dim 128, KV block 64).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "sas_common.cuh"
#include "sas_kernels.h"

namespace sas {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 3-D bf16 map over [n2][n1][n0] (n0 contiguous) with a (b0, b1, b2) box, 128B swizzle.
bool make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t n0, uint64_t n1, uint64_t n2,
                       uint32_t b0, uint32_t b1, uint32_t b2) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {n0, n1, n2};
  cuuint64_t strides[2] = {n0 * 2, n0 * n1 * 2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 map over a row-major [n1 rows][n0 columns] matrix with rows `row_bytes` apart and a
// (b0 columns, b1 rows) box, 128B swizzle.
bool make_tmap_bf16_2d(CUtensorMap* m, const void* base, uint64_t n0, uint64_t n1,
                       uint64_t row_bytes, uint32_t b0, uint32_t b1) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {n0, n1};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {b0, b1};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D fp32 map over [n2][n1][n0] (n0 contiguous) with a (b0, b1, b2) box, no swizzle (the
// shared box is dense: b0 * 4 bytes per row).
bool make_tmap_f32_3d(CUtensorMap* m, const void* base, uint64_t n0, uint64_t n1, uint64_t n2,
                      uint32_t b0, uint32_t b1, uint32_t b2) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {n0, n1, n2};
  cuuint64_t strides[2] = {n0 * 4, n0 * n1 * 4};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 map of rank 2..5 over a contiguous array (dims[0] contiguous) with the given box, 128B
// swizzle (box[0] * 4 must be 128 bytes).
bool make_tmap_f32_sw128(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                         const uint32_t* box) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn || rank < 2 || rank > 5) return false;
  cuuint64_t d[5], str[4];
  cuuint32_t bx[5], estr[5];
  uint64_t stride = 4;
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    estr[i] = 1;
    if (i > 0) str[i - 1] = stride;
    stride *= dims[i];
  }
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, rank, const_cast<void*>(base), d, str, bx, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tma_available() { return encode_fn() != nullptr; }

// Tokens per 128-row tile: Mq tokens x G heads <= 128 (G = 5: 25 tokens, 125 rows).
int tc_rows_per_tile(int G) { return G == 5 ? 25 : 128 / G; }

bool attn_tc_supported(const sas_problem& p) {
  const int G = p.num_q_heads / p.num_kv_heads;
  return p.dtype == SAS_BF16 && p.head_dim == 128 && p.block == 64 &&
         (G == 1 || G == 2 || G == 4 || G == 5 || G == 8) && encode_fn() != nullptr;
}

}  // namespace sas
