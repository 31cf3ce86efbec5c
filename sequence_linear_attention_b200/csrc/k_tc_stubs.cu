// Placeholder definitions used until the tensor-core kernels are enabled.
#include "kernels.h"
#include "tc_kernels.h"

namespace lasp {

cudaError_t tc_chunk_states(const void* a, const void* b, const float* decay, float* M, int B, int H, int64_t N,
                            int d, int C, int kind, cudaStream_t st) {
  return simt_chunk_states(a, b, decay, M, B, H, N, d, C, kind, 1, st);
}
bool tc_out_ok(int, int, int64_t) { return false; }
cudaError_t tc_chunk_out(const void*, const void*, const void*, const float*, const float*, void*, int, int, int64_t,
                         int, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
bool tc_bwd_ok(int, int, int64_t) { return false; }
cudaError_t tc_chunk_bwd(const void*, const void*, const void*, const void*, const float*, const float*,
                         const float*, void*, void*, void*, int, int, int64_t, int, int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace lasp
