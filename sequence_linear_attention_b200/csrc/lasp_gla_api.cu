// C ABI of the gated form (include/lasp.h, "Gated form"): a decay per token
// and key feature, LASP Appendix A.4, Eq. 24 with the GLA / GateLoop row of
// Table 5. Host-side validation and dispatch; nothing here allocates.
//
// The state cache of lasp_gla_fwd holds B x T x H chunk slots of fp32 d x d
// states, then B x T x H slots of d log-gate totals, then as many again for
// segment totals: B*T*H*d*(d+2) floats. The CUDA-core path fills every
// chunk's slot (P_c, gsum_c). The tensor-core path walks segments of about
// 1024 tokens: their states and log-gate totals (the segment state kernel) go
// to the slots of each segment's first chunk, the scan over
// segments turns them into the states entering the segments, and the walk
// carries the state through each segment's tiles, leaving in the slot of every
// tile's first chunk the bf16 operand tile of diag(e^{r}) P (r the tile's
// middle-row log-gate sums) that the backward loads back as is. The backward
// takes the same segments: their gradient states go to the workspace slot of
// each segment's last chunk, the scan over segments (with the forward's
// segment totals) turns them into the states entering the segments from the
// right, and the gradient kernel walks each segment's tiles backward, forming
// every other tile's entering state on the way (in the slot of the segment's
// first chunk).
//
// The tensor-core kernels factor the intra-tile gate products around each
// tile's middle row, which holds while the log-gates of each half-tile span
// at most 80 (natural log). The forward's segment-state kernel checks every
// tile and sets a flag word that follows the state arrays in the cache. A call
// with such a tile then runs, in place of the tensor-core output kernel, the
// exact CUDA-core sequence (per-chunk states, scan, output), and its backward,
// reading the same flag, runs the CUDA-core backward; the kernels of the
// sequence not taken return at once. No host synchronisation decides this.
#include "kernels.h"
#include "lasp_common.cuh"
#include "tc_kernels.h"

namespace lasp {
namespace gla_api_detail {

using namespace api_detail;

int check_gla_sizes(int B, int H, int64_t N, int d, int C, int dtype) {
  int s = check_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (C > 128) return LASP_ERR_UNSUPPORTED;  // a chunk's cumulative gates stay in shared memory
  return LASP_OK;
}

int states_impl(const void* x, const void* y, const float* g, float* M, float* gsum, int B, int H, int64_t N, int d,
                int C, int dtype, int kind, cudaStream_t st) {
  if (C == 128 && tc_gla_ok(dtype, d, C, N))
    return cuda_status(traced(K_GLA_STATES_TC, st, [&] {
      return tc_gla_chunk_states(x, y, g, M, gsum, nullptr, B, H, N, kind, N / C, 1, 0, 1, 1, st);
    }));
  return cuda_status(traced(K_GLA_STATES, st, [&] {
    return gla_simt_chunk_states(x, y, g, M, gsum, B, H, N, d, C, kind, dtype, st);
  }));
}

// T scan elements in every stride-th slot (from offset) of t_slots slots; the
// log-gate totals of element c in slot c * stride + goffset
int scan_impl(const float* M, float* P, const float* gsum, const float* init, float* total, int B, int T, int H,
              int d, int reverse, int64_t t_slots, int stride, int offset, int goffset, cudaStream_t st,
              RunIf run = {}, int id = K_GLA_SCAN) {
  return cuda_status(traced(id, st, [&] {
    return launch_gla_scan(M, P, gsum, init, total, B, T, H, d, reverse, t_slots, stride, offset, goffset, st,
                           run);
  }));
}

// the cache's flag word: after the states and the two log-gate total arrays
constexpr int64_t kFlagFloats = 4;
int64_t cache_state_floats(int B, int H, int64_t N, int d, int C) { return (int64_t)B * (N / C) * H * d * (d + 2); }

}  // namespace gla_api_detail
}  // namespace lasp

using namespace lasp;
using namespace lasp::api_detail;
using namespace lasp::gla_api_detail;

extern "C" {

int64_t lasp_gla_cache_floats(int B, int H, int64_t N, int d, int C) {
  if (check_gla_sizes(B, H, N, d, C, LASP_F32)) return -1;
  return cache_state_floats(B, H, N, d, C) + kFlagFloats;
}

int lasp_gla_chunk_states(const void* x, const void* y, const float* g, float* M, float* gsum, int B, int H,
                          int64_t N, int d, int C, int dtype, int kind, void* stream) {
  int s = check_gla_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (kind != 0 && kind != 1) return LASP_ERR_INVALID_ARG;
  if (N == 0) return LASP_OK;
  if ((s = check_ptrs({x, y, g, M}, {gsum}))) return s;
  return states_impl(x, y, g, M, gsum, B, H, N, d, C, dtype, kind, (cudaStream_t)stream);
}

int lasp_gla_state_prefix(const float* M, float* Mprefix, const float* gsum, const float* init, float* total, int B,
                          int T, int H, int d, int reverse, void* stream) {
  if (B < 1 || H < 1 || T < 0 || (reverse != 0 && reverse != 1)) return LASP_ERR_INVALID_ARG;
  if (d != 32 && d != 64 && d != 128) return LASP_ERR_UNSUPPORTED;
  int s;
  if (T > 0) {
    if ((s = check_ptrs({M, Mprefix, gsum}, {init, total}))) return s;
  } else {
    if ((s = check_ptrs({}, {init, total}))) return s;
    if (total == nullptr) return LASP_OK;
  }
  return scan_impl(M, Mprefix, gsum, init, total, B, T, H, d, reverse, T, 1, 0, 0, (cudaStream_t)stream);
}

int lasp_gla_fwd(const void* q, const void* k, const void* v, const float* g, void* o, int B, int H, int64_t N, int d,
                 int C, int dtype, float* state_cache, const float* init_state, void* stream) {
  int s = check_gla_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (N == 0) return LASP_OK;
  if ((s = check_ptrs({q, k, v, g, o, state_cache}, {init_state}))) return s;
  cudaStream_t st = (cudaStream_t)stream;
  const int T = (int)(N / C);
  float* gsum = state_cache + (int64_t)B * T * H * d * d;
  if (tc_gla_ok(dtype, d, C, N)) {
    // segments of S 128-token tiles: their states and log-gate totals into the
    // slots of each segment's first chunk (the tiles' own totals into their
    // slots, for the backward), the prefix over segments in place, then the
    // walk through each segment's tiles
    const int stride = 128 / C;
    const int S = walk_segment_tokens(N, 128) / 128;
    const int nseg = (int)(N / 128) / S;
    float* gseg = gsum + (int64_t)B * T * H * d;
    int* flag = reinterpret_cast<int*>(state_cache + cache_state_floats(B, H, N, d, C));
    if ((s = cuda_status(cudaMemsetAsync(flag, 0, sizeof(int), st)))) return s;
    if ((s = cuda_status(traced(K_GLA_SEG_STATES, st, [&] {
           return tc_gla_chunk_states(k, v, g, state_cache, gseg, nullptr, B, H, N, 0, T, S * stride, 0, S, stride, st,
                                      flag);
         }))))
      return s;
    if ((s = cuda_status(traced(K_GLA_SEG_SCAN, st, [&] {
           return launch_gla_scan(state_cache, state_cache, gseg, init_state, nullptr, B, nseg, H, d, 0, T, S * stride,
                                  0, 0, st);
         }))))
      return s;
    const RunIf tc{flag, 0}, exact{flag, 1};
    if ((s = cuda_status(traced(K_GLA_OUT_TC, st, [&] {
           return tc_gla_chunk_out(q, k, v, g, state_cache, o, B, H, N, T, stride, S, st, tc);
         }))))
      return s;
    // the exact sequence, which runs only when the flag is set
    if ((s = cuda_status(traced(K_GLA_EXACT_STATES, st, [&] {
           return gla_simt_chunk_states(k, v, g, state_cache, gsum, B, H, N, d, C, 0, dtype, st, exact);
         }))))
      return s;
    if ((s = scan_impl(state_cache, state_cache, gsum, init_state, nullptr, B, T, H, d, 0, T, 1, 0, 0, st, exact,
                       K_GLA_EXACT_SCAN)))
      return s;
    return cuda_status(traced(K_GLA_EXACT_OUT, st, [&] {
      return gla_simt_chunk_out(q, k, v, g, state_cache, o, B, H, N, d, C, dtype, st, exact);
    }));
  }
  // 1. chunk states M_c and log-gate totals; 2. exclusive prefix in place -> P_c; 3. output
  if ((s = states_impl(k, v, g, state_cache, gsum, B, H, N, d, C, dtype, 0, st))) return s;
  if ((s = scan_impl(state_cache, state_cache, gsum, init_state, nullptr, B, T, H, d, 0, T, 1, 0, 0, st))) return s;
  return cuda_status(traced(K_GLA_OUT, st, [&] {
    return gla_simt_chunk_out(q, k, v, g, state_cache, o, B, H, N, d, C, dtype, st);
  }));
}

int lasp_gla_bwd(const void* q, const void* k, const void* v, const float* g, const void* dout, void* dq, void* dk,
                 void* dv, float* dg, int B, int H, int64_t N, int d, int C, int dtype, const float* state_cache,
                 float* dstate_ws, const float* dstate_in, float* dinit_state, void* stream) {
  int s = check_gla_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (N == 0) return LASP_OK;
  if ((s = check_ptrs({q, k, v, g, dout, dq, dk, dv, dg, state_cache, dstate_ws}, {dstate_in, dinit_state})))
    return s;
  cudaStream_t st = (cudaStream_t)stream;
  const int T = (int)(N / C);
  const float* gsum = state_cache + (int64_t)B * T * H * d * d;
  if (tc_gla_ok(dtype, d, C, N)) {
    // the forward's segments of S 128-token tiles: gradient states into the
    // slots of each segment's last chunk, the suffix over segments in place
    // (the segments' log-gate totals sit in the cache's third array, in the
    // slots of their first chunks), then the gradients, walking each segment
    const int stride = 128 / C;
    const int S = walk_segment_tokens(N, 128) / 128;
    const int nseg = (int)(N / 128) / S;
    const float* gseg = gsum + (int64_t)B * T * H * d;
    // the forward's choice, in the cache's flag word
    const int* flag = reinterpret_cast<const int*>(state_cache + cache_state_floats(B, H, N, d, C));
    const RunIf tc{flag, 0}, exact{flag, 1};
    if ((s = cuda_status(traced(K_GLA_SEG_STATES, st, [&] {
           return tc_gla_chunk_states(q, dout, g, dstate_ws, nullptr, nullptr, B, H, N, 1, T, S * stride,
                                      S * stride - 1, S, stride, st, nullptr, tc);
         }))))
      return s;
    if ((s = scan_impl(dstate_ws, dstate_ws, gseg, dstate_in, dinit_state, B, nseg, H, d, 1, T, S * stride,
                       S * stride - 1, 0, st, tc, K_GLA_SEG_SCAN)))
      return s;
    if ((s = cuda_status(traced(K_GLA_BWD_TC, st, [&] {
           return tc_gla_chunk_bwd(q, k, v, dout, g, state_cache, dstate_ws, dq, dk, dv, dg, B, H, N, T, stride, S, st,
                                   tc);
         }))))
      return s;
    // the exact sequence, which runs only when the forward took it
    if ((s = cuda_status(traced(K_GLA_EXACT_STATES, st, [&] {
           return gla_simt_chunk_states(q, dout, g, dstate_ws, nullptr, B, H, N, d, C, 1, dtype, st, exact);
         }))))
      return s;
    if ((s = scan_impl(dstate_ws, dstate_ws, gsum, dstate_in, dinit_state, B, T, H, d, 1, T, 1, 0, 0, st, exact,
                       K_GLA_EXACT_SCAN)))
      return s;
    return cuda_status(traced(K_GLA_EXACT_BWD, st, [&] {
      return gla_simt_chunk_bwd(q, k, v, dout, g, state_cache, dstate_ws, dq, dk, dv, dg, B, H, N, d, C, dtype, st,
                                exact);
    }));
  }
  // 1. gradient chunk states dM_c; 2. exclusive suffix in place -> R_c (and
  // dinit); 3. dQ, dK, dV and the log-gate gradient
  if ((s = states_impl(q, dout, g, dstate_ws, nullptr, B, H, N, d, C, dtype, 1, st))) return s;
  if ((s = scan_impl(dstate_ws, dstate_ws, gsum, dstate_in, dinit_state, B, T, H, d, 1, T, 1, 0, 0, st))) return s;
  return cuda_status(traced(K_GLA_BWD, st, [&] {
    return gla_simt_chunk_bwd(q, k, v, dout, g, state_cache, dstate_ws, dq, dk, dv, dg, B, H, N, d, C, dtype, st);
  }));
}

}  // extern "C"
