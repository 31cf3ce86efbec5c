// C ABI of the softmax-attention layers of a hybrid model (include/lasp.h,
// "Softmax attention"): LASP-2 review page, "Summary" (LASP-2H applies the
// AllGather pattern to standard attention, gathering K_t and V_t). Host-side
// validation and dispatch; nothing here allocates.
#include <math.h>

#include "kernels.h"
#include "lasp_common.cuh"
#include "tc_kernels.h"

namespace lasp {
namespace softmax_api_detail {

using namespace api_detail;

int check_softmax(int B, int H, int64_t Nq, int64_t Nk, int64_t q_offset, int d, float scale, int dtype) {
  if (dtype != LASP_F32 && dtype != LASP_BF16) return LASP_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Nq < 0 || Nk < 0 || q_offset < 0) return LASP_ERR_INVALID_ARG;
  if (q_offset + Nq > Nk) return LASP_ERR_INVALID_ARG;  // a query's own key must exist
  if (!(scale > 0.f) || !isfinite(scale)) return LASP_ERR_INVALID_ARG;
  if (B > 65535 || H > 65535 || Nk > INT32_MAX) return LASP_ERR_UNSUPPORTED;
  if (!tc_softmax_ok(dtype, d)) return LASP_ERR_UNSUPPORTED;
  return LASP_OK;
}

}  // namespace softmax_api_detail
}  // namespace lasp

using namespace lasp;
using namespace lasp::api_detail;
using namespace lasp::softmax_api_detail;

extern "C" {

int lasp_softmax_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int64_t Nq,
                     int64_t Nk, int64_t q_offset, int d, float scale, int dtype, void* stream) {
  int s = check_softmax(B, H, Nq, Nk, q_offset, d, scale, dtype);
  if (s) return s;
  if (Nq == 0) return LASP_OK;
  if ((s = check_ptrs({q, k, v, o, lse}, {}))) return s;
  cudaStream_t st = (cudaStream_t)stream;
  return cuda_status(traced(K_SOFTMAX_FWD, st, [&] {
    return tc_softmax_fwd(q, k, v, o, lse, B, H, Nq, Nk, q_offset, scale, st);
  }));
}

int lasp_softmax_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, float* delta, int B, int H, int64_t Nq, int64_t Nk,
                     int64_t q_offset, int d, float scale, int dtype, void* stream) {
  int s = check_softmax(B, H, Nq, Nk, q_offset, d, scale, dtype);
  if (s) return s;
  if ((s = check_ptrs({k, v, dk, dv}, {q, o, lse, dout, dq, delta}))) return s;
  if (Nq > 0 && (s = check_ptrs({q, o, lse, dout, dq, delta}, {}))) return s;
  if (Nk == 0) return LASP_OK;
  cudaStream_t st = (cudaStream_t)stream;
  if (Nq == 0) {  // no query: every key's gradient is zero (bf16 zero is all-zero bytes)
    const size_t bytes = (size_t)B * Nk * H * d * 2;
    if ((s = cuda_status(cudaMemsetAsync(dk, 0, bytes, st)))) return s;
    return cuda_status(cudaMemsetAsync(dv, 0, bytes, st));
  }
  if ((s = cuda_status(traced(K_SOFTMAX_DELTA, st, [&] { return tc_softmax_delta(o, dout, delta, B, H, Nq, st); }))))
    return s;
  // every key tile is written (zeros where no query reaches it)
  if ((s = cuda_status(traced(K_SOFTMAX_DKDV, st, [&] {
         return tc_softmax_dkdv(q, k, v, lse, dout, dk, dv, delta, B, H, Nq, Nk, q_offset, scale, st);
       }))))
    return s;
  return cuda_status(traced(K_SOFTMAX_DQ, st, [&] {
    return tc_softmax_dq(q, k, v, lse, dout, dq, delta, B, H, Nq, Nk, q_offset, scale, st);
  }));
}

}  // extern "C"
