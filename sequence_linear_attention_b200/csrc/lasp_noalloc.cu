// lasp_bwd_noalloc: the backward pass for callers that cannot allocate device
// memory. lasp_bwd needs a caller-provided fp32 workspace for the gradient
// states R (B * N/C * H * d * d floats); this variant keeps R in a fixed array
// compiled into the library instead, so the caller passes only its inputs and
// outputs. Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "kernels.h"
#include "lasp_common.cuh"
#include "tc_kernels.h"

namespace lasp {
namespace noalloc_detail {

// 32 MiB of gradient-state workspace, resident on every GPU that loads the
// library until the process exits. Enough for B * (N / C) * H <= 512 states
// of d = 128.
constexpr size_t kScratchBytes = (size_t)32 << 20;
static_assert(kScratchBytes == (size_t)LASP_NOALLOC_SCRATCH_BYTES,
              "the workspace size must equal the limit the header publishes");
static __device__ __align__(256) float g_bwd_scratch[kScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_bwd_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
int scratch_for_current_device(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LASP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr) return LASP_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return LASP_OK;
}

}  // namespace noalloc_detail
}  // namespace lasp

extern "C" int lasp_bwd_noalloc(const void* q, const void* k, const void* v, const float* decay, const void* dout,
                                void* dq, void* dk, void* dv, int B, int H, int64_t N, int d, int C, int dtype,
                                const float* state_cache, const float* dstate_in, float* dinit_state,
                                void* stream) {
  using namespace lasp;
  using namespace lasp::api_detail;
  int s = check_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (N == 0) return LASP_OK;
  if ((s = check_ptrs({q, k, v, dout, dq, dk, dv, state_cache}, {decay, dstate_in, dinit_state}))) return s;
  const int T = (int)(N / C);
  const size_t need = (size_t)B * T * H * d * d * sizeof(float);
  if (need > noalloc_detail::kScratchBytes) return LASP_ERR_UNSUPPORTED;
  float* R = nullptr;
  if ((s = noalloc_detail::scratch_for_current_device(&R))) return s;
  cudaStream_t st = (cudaStream_t)stream;
  // the same steps as lasp_bwd, with the workspace in the fixed array; every
  // element of R that is read is written first, so nothing is cleared
  if (tc_bwd_walk_ok(dtype, d, C, N)) {
    const int G = walk_segment_tokens(N, C);
    const int stride = G / C;
    if ((s = cuda_status(tc_chunk_states_slots(q, dout, decay, R, B, H, N, d, G, 1, T, stride, stride - 1, st))))
      return s;
    if ((s = cuda_status(launch_state_scan_slots(R, R, decay, dstate_in, dinit_state, B, (int)(N / G), H, d, G, 1, T,
                                                 stride, stride - 1, st))))
      return s;
    return cuda_status(tc_bwd_walk(q, k, v, dout, decay, state_cache, R, dq, dk, dv, B, H, N, d, C, G,
                                   num_sms_current_device(), st));
  }
  if ((s = chunk_states_impl(q, dout, decay, R, B, H, N, d, C, dtype, 1, st))) return s;
  if ((s = cuda_status(launch_state_scan(R, R, decay, dstate_in, dinit_state, B, T, H, d, C, 1, st)))) return s;
  return chunk_grads_impl(q, k, v, dout, decay, state_cache, R, dq, dk, dv, B, H, N, d, C, dtype, st);
}
