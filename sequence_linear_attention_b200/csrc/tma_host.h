// Host-side TMA descriptor encoding for the token tensors [B, N, H, d] (bf16)
// and the fp32 state arrays.
// cuTensorMapEncodeTiled is fetched from the driver through the runtime, so the
// library does not link against libcuda directly.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <climits>

namespace lasp {

inline PFN_cuTensorMapEncodeTiled_v12000 tmap_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// A 4-D view (d, H, N, B) of a [B, N, H, d] bf16 tensor; one box is 64
// features x 1 head x `rows` tokens x 1 batch, stored in shared memory as
// `rows` lines of 128 bytes with the 128-byte swizzle. Rows past N read as 0
// and are dropped on store.
inline bool make_token_map(CUtensorMap* map, const void* base, int B, int H, int64_t N, int d, int rows) {
  auto fn = tmap_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)N * H * d * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A 2-D view (d, rows) of an fp32 state array [..., d, d] (rows = number of
// states x d); one box is 32 columns x box_rows rows, stored in shared memory
// as lines of 128 bytes with the 128-byte swizzle (a d = 128 state is 4 boxes
// of 128 rows).
inline bool make_state_map(CUtensorMap* map, const float* base, int64_t nstates, int d, int box_rows = 128) {
  auto fn = tmap_encode_fn();
  const int64_t rows = nstates * d;
  if (fn == nullptr || rows <= 0 || rows > (int64_t)INT32_MAX) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 4};
  cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A 4-D view (d, H, N, B) of a [B, N, H, d] fp32 tensor (the log-gates of
// the gated form); one box is 32 features x 1 head x `rows` tokens x 1 batch,
// stored as `rows` lines of 128 bytes with the 128-byte swizzle (16-byte chunk
// c of line t lands at chunk c ^ (t % 8)).
inline bool make_gate_map(CUtensorMap* map, const float* base, int B, int H, int64_t N, int d, int rows) {
  auto fn = tmap_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 4, (cuuint64_t)H * d * 4, (cuuint64_t)N * H * d * 4};
  cuuint32_t box[4] = {32, 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace lasp
