// C ABI of include/lasp.h: host-side validation and dispatch to the kernels.
// Nothing here allocates memory; every launch goes to the caller's stream.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <vector>

#include "kernels.h"
#include "lasp_common.cuh"
#include "sm100.cuh"
#include "tc_kernels.h"

namespace lasp {

namespace api_detail {

// ---------------------------------------------------------------- tracing
// Kernel identities reported by lasp_trace_read / lasp_kernel_name.
enum KernelId : int {
  K_STATES_TC = 1,      // per-chunk states, tensor cores
  K_STATES_SIMT = 2,    // per-chunk states, CUDA cores
  K_SCAN = 3,           // per-chunk prefix / suffix
  K_OUT_TC = 4,         // output, one tile per CTA
  K_OUT_SIMT = 5,
  K_BWD_TC = 6,         // dQ/dK/dV, one tile per CTA
  K_BWD_SIMT = 7,
  K_FWD_WALK = 8,       // output walk over segments
  K_BWD_WALK = 9,       // dQ/dK/dV walk over segments
  K_SEG_STATES = 10,    // segment states (tensor cores)
  K_SEG_SCAN = 11,      // prefix / suffix over segments
  K_PROBE = 12,
  K_BIDIR_TOTAL = 13,   // bidirectional: sum of the segment states
  K_BIDIR_APPLY = 14,   // bidirectional: token tiles times the total state
  K_GLA_STATES = 15,    // gated form: per-chunk states and log-gate totals
  K_GLA_SCAN = 16,      // gated form: prefix / suffix with a diagonal decay
  K_GLA_OUT = 17,       // gated form: output
  K_GLA_BWD = 18,       // gated form: dQ/dK/dV and the log-gate gradient
  K_GLA_STATES_TC = 19,  // gated form on the tensor cores: states
  K_GLA_OUT_TC = 20,     // gated form on the tensor cores: output
  K_GLA_BWD_TC = 21,     // gated form on the tensor cores: gradients
  K_STATE_TOTAL = 22,    // decayed total of a sequence's states (the LASP-2 shard state)
  K_GLA_SEG_STATES = 23,  // gated form on the tensor cores: segment states (both directions)
  K_GLA_SEG_SCAN = 24,    // gated form: prefix / suffix over segments
  // gated form, the exact CUDA-core sequence a tensor-core call switches to
  // on the device when a tile's log-gates leave the factorized form's range
  // (the kernels return at once otherwise)
  K_GLA_EXACT_STATES = 25,
  K_GLA_EXACT_SCAN = 26,
  K_GLA_EXACT_OUT = 27,
  K_GLA_EXACT_BWD = 28,
  K_SOFTMAX_FWD = 29,    // softmax attention (hybrid layers): forward
  K_SOFTMAX_DELTA = 30,  // softmax attention: rowsum(do . o)
  K_SOFTMAX_DKDV = 31,   // softmax attention: dK, dV per key tile
  K_SOFTMAX_DQ = 32,     // softmax attention: dQ per query tile
  K_COUNT
};

struct Trace {
  std::mutex mu;
  std::vector<cudaEvent_t> ev;
  std::vector<int> ids;
  int n = 0;
  int cap = 0;
};
Trace g_trace;

// Runs `launch`; while tracing is on, brackets it with two events on `st`.
template <class F>
cudaError_t traced(int id, cudaStream_t st, F&& launch) {
  if (g_trace.cap == 0) return launch();
  std::lock_guard<std::mutex> lock(g_trace.mu);
  if (g_trace.n >= g_trace.cap) return launch();
  cudaEventRecord(g_trace.ev[2 * g_trace.n], st);
  cudaError_t e = launch();
  cudaEventRecord(g_trace.ev[2 * g_trace.n + 1], st);
  g_trace.ids[g_trace.n++] = id;
  return e;
}

__global__ void wait_probe_kernel() {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
    // Nothing arrives on the barrier: the wait can only end by its limit.
    sm100::mbar_wait(&bar, 0, SITE_PROBE);
  }
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int check_ptrs(std::initializer_list<const void*> required, std::initializer_list<const void*> optional) {
  for (const void* p : required) {
    if (p == nullptr) return LASP_ERR_INVALID_ARG;
    if (!aligned16(p)) return LASP_ERR_MISALIGNED;
  }
  for (const void* p : optional)
    if (p != nullptr && !aligned16(p)) return LASP_ERR_MISALIGNED;
  return LASP_OK;
}

inline int check_sizes(int B, int H, int64_t N, int d, int64_t C, int dtype) {
  if (dtype != LASP_F32 && dtype != LASP_BF16) return LASP_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 0 || C < 1) return LASP_ERR_INVALID_ARG;
  if (B > 65535 || H > 65535) return LASP_ERR_UNSUPPORTED;  // grid y / z limits
  if (d != 32 && d != 64 && d != 128) return LASP_ERR_UNSUPPORTED;
  if (N % C != 0) return LASP_ERR_INVALID_ARG;
  if (N / C > INT32_MAX) return LASP_ERR_UNSUPPORTED;
  return LASP_OK;
}

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? LASP_OK : LASP_ERR_CUDA; }

int chunk_states_impl(const void* a, const void* b, const float* decay, float* M, int B, int H, int64_t N, int d,
                      int C, int dtype, int kind, cudaStream_t st) {
  if (tc_states_ok(dtype, d, C))
    return cuda_status(traced(K_STATES_TC, st, [&] { return tc_chunk_states(a, b, decay, M, B, H, N, d, C, kind, st); }));
  return cuda_status(
      traced(K_STATES_SIMT, st, [&] { return simt_chunk_states(a, b, decay, M, B, H, N, d, C, kind, dtype, st); }));
}

int scan_impl(int id, const float* M, float* P, const float* decay, const float* init, float* total, int B, int T,
              int H, int d, int64_t C, int reverse, cudaStream_t st) {
  return cuda_status(
      traced(id, st, [&] { return launch_state_scan(M, P, decay, init, total, B, T, H, d, C, reverse, st); }));
}

int num_sms_current_device() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

int chunk_out_impl(const void* q, const void* k, const void* v, const float* decay, const float* P, void* o, int B,
                   int H, int64_t N, int d, int C, int dtype, cudaStream_t st) {
  if (tc_out_ok(dtype, d, C))
    return cuda_status(traced(K_OUT_TC, st, [&] { return tc_chunk_out(q, k, v, decay, P, o, B, H, N, d, C, st); }));
  return cuda_status(
      traced(K_OUT_SIMT, st, [&] { return simt_chunk_out(q, k, v, decay, P, o, B, H, N, d, C, dtype, st); }));
}

int chunk_grads_impl(const void* q, const void* k, const void* v, const void* dout, const float* decay,
                     const float* P, const float* R, void* dq, void* dk, void* dv, int B, int H, int64_t N, int d,
                     int C, int dtype, cudaStream_t st) {
  if (tc_bwd_ok(dtype, d, C))
    return cuda_status(
        traced(K_BWD_TC, st, [&] { return tc_chunk_bwd(q, k, v, dout, decay, P, R, dq, dk, dv, B, H, N, d, C, st); }));
  return cuda_status(traced(
      K_BWD_SIMT, st, [&] { return simt_chunk_bwd(q, k, v, dout, decay, P, R, dq, dk, dv, B, H, N, d, C, dtype, st); }));
}

// lasp_fwd in two parts. States: the chunk (or, on the walk path, segment)
// states into the cache and, if total is non-NULL, their decayed total with a
// zero start. Finish: the prefix from init and the output.
// bh0, nbh (walk path only): the (b, h) pairs bh0 .. bh0 + nbh - 1; nbh < 0: all.
int fwd_states_impl(const void* k, const void* v, const float* decay, int B, int H, int64_t N, int d, int C,
                    int dtype, float* state_cache, float* total, cudaStream_t st, int64_t bh0 = 0,
                    int64_t nbh = -1) {
  const int T = (int)(N / C);
  int s;
  if (tc_fwd_walk_ok(dtype, d, C, N)) {
    // segments of G tokens: their states go to the slots of their first chunks
    const int G = walk_segment_tokens(N, C);
    const int stride = G / C;
    if ((s = cuda_status(traced(K_SEG_STATES, st, [&] {
           return tc_chunk_states_slots(k, v, decay, state_cache, B, H, N, d, G, 0, T, stride, 0, st, bh0, nbh);
         }))))
      return s;
    if (!total) return LASP_OK;
    return cuda_status(traced(K_STATE_TOTAL, st, [&] {
      return launch_state_scan_slots(state_cache, nullptr, decay, nullptr, total, B, (int)(N / G), H, d, G, 0, T,
                                     stride, 0, st, bh0, nbh);
    }));
  }
  if ((s = chunk_states_impl(k, v, decay, state_cache, B, H, N, d, C, dtype, 0, st))) return s;
  return total ? scan_impl(K_STATE_TOTAL, state_cache, nullptr, decay, nullptr, total, B, T, H, d, C, 0, st) : LASP_OK;
}

int fwd_finish_impl(const void* q, const void* k, const void* v, const float* decay, void* o, int B, int H, int64_t N,
                    int d, int C, int dtype, float* state_cache, const float* init_state, cudaStream_t st,
                    int64_t bh0 = 0, int64_t nbh = -1) {
  const int T = (int)(N / C);
  int s;
  if (tc_fwd_walk_ok(dtype, d, C, N)) {
    // the exclusive prefix over segments turns their states into P of their
    // first chunks, and the walk carries the state through each segment,
    // filling the other slots
    const int G = walk_segment_tokens(N, C);
    const int stride = G / C;
    if ((s = cuda_status(traced(K_SEG_SCAN, st, [&] {
           return launch_state_scan_slots(state_cache, state_cache, decay, init_state, nullptr, B, (int)(N / G), H, d,
                                          G, 0, T, stride, 0, st, bh0, nbh);
         }))))
      return s;
    const int sms = num_sms_current_device();
    return cuda_status(traced(K_FWD_WALK, st, [&] {
      return tc_fwd_walk(q, k, v, decay, state_cache, o, B, H, N, d, C, G, sms, st, bh0, nbh);
    }));
  }
  // exclusive prefix in place -> P_c; then the output
  if ((s = scan_impl(K_SCAN, state_cache, state_cache, decay, init_state, nullptr, B, T, H, d, C, 0, st))) return s;
  return chunk_out_impl(q, k, v, decay, state_cache, o, B, H, N, d, C, dtype, st);
}

// lasp_bwd in two parts. States: the gradient chunk (or segment) states into
// the workspace and, if total is non-NULL, their decayed total with nothing
// entering from after the sequence. Finish: the suffix from dstate_in (and
// dinit) and dQ, dK, dV.
int bwd_states_impl(const void* q, const void* dout, const float* decay, int B, int H, int64_t N, int d, int C,
                    int dtype, float* dstate_ws, float* total, cudaStream_t st, int64_t bh0 = 0, int64_t nbh = -1) {
  const int T = (int)(N / C);
  int s;
  if (tc_bwd_walk_ok(dtype, d, C, N)) {
    // segments of G tokens: their gradient states go to the slots of their last chunks
    const int G = walk_segment_tokens(N, C);
    const int stride = G / C;
    if ((s = cuda_status(traced(K_SEG_STATES, st, [&] {
           return tc_chunk_states_slots(q, dout, decay, dstate_ws, B, H, N, d, G, 1, T, stride, stride - 1, st, bh0,
                                        nbh);
         }))))
      return s;
    if (!total) return LASP_OK;
    return cuda_status(traced(K_STATE_TOTAL, st, [&] {
      return launch_state_scan_slots(dstate_ws, nullptr, decay, nullptr, total, B, (int)(N / G), H, d, G, 1, T,
                                     stride, stride - 1, st, bh0, nbh);
    }));
  }
  if ((s = chunk_states_impl(q, dout, decay, dstate_ws, B, H, N, d, C, dtype, 1, st))) return s;
  return total ? scan_impl(K_STATE_TOTAL, dstate_ws, nullptr, decay, nullptr, total, B, T, H, d, C, 1, st) : LASP_OK;
}

int bwd_finish_impl(const void* q, const void* k, const void* v, const float* decay, const void* dout, void* dq,
                    void* dk, void* dv, int B, int H, int64_t N, int d, int C, int dtype, const float* state_cache,
                    float* dstate_ws, const float* dstate_in, float* dinit_state, cudaStream_t st,
                    int64_t bh0 = 0, int64_t nbh = -1) {
  const int T = (int)(N / C);
  int s;
  if (tc_bwd_walk_ok(dtype, d, C, N)) {
    // the exclusive suffix over segments turns their gradient states into R of
    // their last chunks (and gives dinit), and the walk carries R backward
    // through each segment
    const int G = walk_segment_tokens(N, C);
    const int stride = G / C;
    if ((s = cuda_status(traced(K_SEG_SCAN, st, [&] {
           return launch_state_scan_slots(dstate_ws, dstate_ws, decay, dstate_in, dinit_state, B, (int)(N / G), H, d,
                                          G, 1, T, stride, stride - 1, st, bh0, nbh);
         }))))
      return s;
    const int sms = num_sms_current_device();
    return cuda_status(traced(K_BWD_WALK, st, [&] {
      return tc_bwd_walk(q, k, v, dout, decay, state_cache, dstate_ws, dq, dk, dv, B, H, N, d, C, G, sms, st, bh0,
                         nbh);
    }));
  }
  // exclusive suffix in place -> R_c (and dinit); then dQ, dK, dV
  if ((s = scan_impl(K_SCAN, dstate_ws, dstate_ws, decay, dstate_in, dinit_state, B, T, H, d, C, 1, st))) return s;
  return chunk_grads_impl(q, k, v, dout, decay, state_cache, dstate_ws, dq, dk, dv, B, H, N, d, C, dtype, st);
}


}  // namespace api_detail
}  // namespace lasp

using namespace lasp;
using namespace lasp::api_detail;

extern "C" {

int lasp_version(void) { return 100; }

const char* lasp_status_string(int status) {
  switch (status) {
    case LASP_OK: return "LASP_OK";
    case LASP_ERR_INVALID_ARG: return "LASP_ERR_INVALID_ARG";
    case LASP_ERR_UNSUPPORTED: return "LASP_ERR_UNSUPPORTED";
    case LASP_ERR_MISALIGNED: return "LASP_ERR_MISALIGNED";
    case LASP_ERR_CUDA: return "LASP_ERR_CUDA";
    case LASP_ERR_TIMEOUT: return "LASP_ERR_TIMEOUT";
    default: return "LASP_ERR_UNKNOWN";
  }
}

int lasp_chunk_states(const void* q, const void* k, const void* v, const float* decay, float* M, int B, int H,
                      int64_t N, int d, int C, int dtype, void* stream) {
  (void)q;
  int s = check_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (N == 0) return LASP_OK;
  if ((s = check_ptrs({k, v, M}, {decay}))) return s;
  return chunk_states_impl(k, v, decay, M, B, H, N, d, C, dtype, 0, (cudaStream_t)stream);
}

int lasp_chunk_dstates(const void* q, const void* dout, const float* decay, float* dM, int B, int H, int64_t N,
                       int d, int C, int dtype, void* stream) {
  int s = check_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (N == 0) return LASP_OK;
  if ((s = check_ptrs({q, dout, dM}, {decay}))) return s;
  return chunk_states_impl(q, dout, decay, dM, B, H, N, d, C, dtype, 1, (cudaStream_t)stream);
}

int lasp_state_prefix(const float* M, float* Mprefix, const float* decay, const float* init, float* total, int B,
                      int T, int H, int d, int64_t C, int reverse, void* stream) {
  if (B < 1 || H < 1 || T < 0 || C < 1 || (reverse != 0 && reverse != 1)) return LASP_ERR_INVALID_ARG;
  if (d != 32 && d != 64 && d != 128) return LASP_ERR_UNSUPPORTED;
  if (C > (int64_t)1 << 24) return LASP_ERR_UNSUPPORTED;  // lambda^C exponent kept exact in fp32
  if (T > 0) {
    int s = check_ptrs({M, Mprefix}, {decay, init, total});
    if (s) return s;
  } else {
    int s = check_ptrs({}, {decay, init, total});
    if (s) return s;
    if (total == nullptr) return LASP_OK;
  }
  return scan_impl(K_SCAN, M, Mprefix, decay, init, total, B, T, H, d, C, reverse, (cudaStream_t)stream);
}

int lasp_fwd_states(const void* k, const void* v, const float* decay, int B, int H, int64_t N, int d, int C,
                    int dtype, float* state_cache, float* total, void* stream) {
  int s = check_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (N == 0) {
    if ((s = check_ptrs({}, {decay, total}))) return s;
    return total ? scan_impl(K_STATE_TOTAL, nullptr, nullptr, decay, nullptr, total, B, 0, H, d, C, 0,
                             (cudaStream_t)stream)
                 : LASP_OK;
  }
  if ((s = check_ptrs({k, v, state_cache}, {decay, total}))) return s;
  return fwd_states_impl(k, v, decay, B, H, N, d, C, dtype, state_cache, total, (cudaStream_t)stream);
}

int lasp_fwd_finish(const void* q, const void* k, const void* v, const float* decay, void* o, int B, int H,
                    int64_t N, int d, int C, int dtype, float* state_cache, const float* init_state, void* stream) {
  int s = check_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (N == 0) return LASP_OK;
  if ((s = check_ptrs({q, k, v, o, state_cache}, {decay, init_state}))) return s;
  return fwd_finish_impl(q, k, v, decay, o, B, H, N, d, C, dtype, state_cache, init_state, (cudaStream_t)stream);
}

int lasp_parts_ok(int64_t N, int C, int d, int dtype) {
  return N > 0 && C >= 1 && N % C == 0 && tc_fwd_walk_ok(dtype, d, C, N) && tc_bwd_walk_ok(dtype, d, C, N) ? 1 : 0;
}

}  // extern "C"

namespace lasp {
namespace api_detail {

// The (b, h) pairs of part `part` of `nparts`: bh0 .. bh0 + nbh - 1 (b-major),
// after the same size checks as the whole call; nparts > 1 only where both
// walks run (lasp_parts_ok).
int part_range(int B, int H, int64_t N, int d, int C, int dtype, int part, int nparts, int64_t* bh0, int64_t* nbh) {
  int s = check_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  const int64_t bh = (int64_t)B * H;
  if (nparts < 1 || part < 0 || part >= nparts || nparts > bh) return LASP_ERR_INVALID_ARG;
  if (nparts > 1 && !lasp_parts_ok(N, C, d, dtype)) return LASP_ERR_UNSUPPORTED;
  *bh0 = bh * part / nparts;
  *nbh = bh * (part + 1) / nparts - *bh0;
  return LASP_OK;
}

}  // namespace api_detail
}  // namespace lasp

extern "C" {

int lasp_fwd_states_part(const void* k, const void* v, const float* decay, int B, int H, int64_t N, int d, int C,
                         int dtype, float* state_cache, float* total, int part, int nparts, void* stream) {
  int64_t bh0 = 0, nbh = 0;
  int s = part_range(B, H, N, d, C, dtype, part, nparts, &bh0, &nbh);
  if (s) return s;
  if (nparts == 1) return lasp_fwd_states(k, v, decay, B, H, N, d, C, dtype, state_cache, total, stream);
  if ((s = check_ptrs({k, v, state_cache}, {decay, total}))) return s;
  return fwd_states_impl(k, v, decay, B, H, N, d, C, dtype, state_cache, total, (cudaStream_t)stream, bh0, nbh);
}

int lasp_fwd_finish_part(const void* q, const void* k, const void* v, const float* decay, void* o, int B, int H,
                         int64_t N, int d, int C, int dtype, float* state_cache, const float* init_state, int part,
                         int nparts, void* stream) {
  int64_t bh0 = 0, nbh = 0;
  int s = part_range(B, H, N, d, C, dtype, part, nparts, &bh0, &nbh);
  if (s) return s;
  if (nparts == 1) return lasp_fwd_finish(q, k, v, decay, o, B, H, N, d, C, dtype, state_cache, init_state, stream);
  if ((s = check_ptrs({q, k, v, o, state_cache}, {decay, init_state}))) return s;
  return fwd_finish_impl(q, k, v, decay, o, B, H, N, d, C, dtype, state_cache, init_state, (cudaStream_t)stream,
                         bh0, nbh);
}

int lasp_bwd_states_part(const void* q, const void* dout, const float* decay, int B, int H, int64_t N, int d, int C,
                         int dtype, float* dstate_ws, float* total, int part, int nparts, void* stream) {
  int64_t bh0 = 0, nbh = 0;
  int s = part_range(B, H, N, d, C, dtype, part, nparts, &bh0, &nbh);
  if (s) return s;
  if (nparts == 1) return lasp_bwd_states(q, dout, decay, B, H, N, d, C, dtype, dstate_ws, total, stream);
  if ((s = check_ptrs({q, dout, dstate_ws}, {decay, total}))) return s;
  return bwd_states_impl(q, dout, decay, B, H, N, d, C, dtype, dstate_ws, total, (cudaStream_t)stream, bh0, nbh);
}

int lasp_bwd_finish_part(const void* q, const void* k, const void* v, const float* decay, const void* dout, void* dq,
                         void* dk, void* dv, int B, int H, int64_t N, int d, int C, int dtype,
                         const float* state_cache, float* dstate_ws, const float* dstate_in, float* dinit_state,
                         int part, int nparts, void* stream) {
  int64_t bh0 = 0, nbh = 0;
  int s = part_range(B, H, N, d, C, dtype, part, nparts, &bh0, &nbh);
  if (s) return s;
  if (nparts == 1)
    return lasp_bwd_finish(q, k, v, decay, dout, dq, dk, dv, B, H, N, d, C, dtype, state_cache, dstate_ws, dstate_in,
                           dinit_state, stream);
  if ((s = check_ptrs({q, k, v, dout, dq, dk, dv, state_cache, dstate_ws}, {decay, dstate_in, dinit_state})))
    return s;
  return bwd_finish_impl(q, k, v, decay, dout, dq, dk, dv, B, H, N, d, C, dtype, state_cache, dstate_ws, dstate_in,
                         dinit_state, (cudaStream_t)stream, bh0, nbh);
}

int lasp_fwd(const void* q, const void* k, const void* v, const float* decay, void* o, int B, int H, int64_t N,
             int d, int C, int dtype, float* state_cache, const float* init_state, void* stream) {
  int s = check_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (N == 0) return LASP_OK;
  if ((s = check_ptrs({q, k, v, o, state_cache}, {decay, init_state}))) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if ((s = fwd_states_impl(k, v, decay, B, H, N, d, C, dtype, state_cache, nullptr, st))) return s;
  return fwd_finish_impl(q, k, v, decay, o, B, H, N, d, C, dtype, state_cache, init_state, st);
}

int lasp_chunk_out(const void* q, const void* k, const void* v, const float* decay, const float* P, void* o, int B,
                   int H, int64_t N, int d, int C, int dtype, void* stream) {
  int s = check_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (N == 0) return LASP_OK;
  if ((s = check_ptrs({q, k, v, P, o}, {decay}))) return s;
  return chunk_out_impl(q, k, v, decay, P, o, B, H, N, d, C, dtype, (cudaStream_t)stream);
}

int lasp_chunk_grads(const void* q, const void* k, const void* v, const void* dout, const float* decay,
                     const float* P, const float* R, void* dq, void* dk, void* dv, int B, int H, int64_t N, int d,
                     int C, int dtype, void* stream) {
  int s = check_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (N == 0) return LASP_OK;
  if ((s = check_ptrs({q, k, v, dout, P, R, dq, dk, dv}, {decay}))) return s;
  return chunk_grads_impl(q, k, v, dout, decay, P, R, dq, dk, dv, B, H, N, d, C, dtype, (cudaStream_t)stream);
}

int lasp_bwd_states(const void* q, const void* dout, const float* decay, int B, int H, int64_t N, int d, int C,
                    int dtype, float* dstate_ws, float* total, void* stream) {
  int s = check_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (N == 0) {
    if ((s = check_ptrs({}, {decay, total}))) return s;
    return total ? scan_impl(K_STATE_TOTAL, nullptr, nullptr, decay, nullptr, total, B, 0, H, d, C, 1,
                             (cudaStream_t)stream)
                 : LASP_OK;
  }
  if ((s = check_ptrs({q, dout, dstate_ws}, {decay, total}))) return s;
  return bwd_states_impl(q, dout, decay, B, H, N, d, C, dtype, dstate_ws, total, (cudaStream_t)stream);
}

int lasp_bwd_finish(const void* q, const void* k, const void* v, const float* decay, const void* dout, void* dq,
                    void* dk, void* dv, int B, int H, int64_t N, int d, int C, int dtype, const float* state_cache,
                    float* dstate_ws, const float* dstate_in, float* dinit_state, void* stream) {
  int s = check_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (N == 0) return LASP_OK;
  if ((s = check_ptrs({q, k, v, dout, dq, dk, dv, state_cache, dstate_ws}, {decay, dstate_in, dinit_state})))
    return s;
  return bwd_finish_impl(q, k, v, decay, dout, dq, dk, dv, B, H, N, d, C, dtype, state_cache, dstate_ws, dstate_in,
                         dinit_state, (cudaStream_t)stream);
}

int lasp_bwd(const void* q, const void* k, const void* v, const float* decay, const void* dout, void* dq, void* dk,
             void* dv, int B, int H, int64_t N, int d, int C, int dtype, const float* state_cache, float* dstate_ws,
             const float* init_state, const float* dstate_in, float* dinit_state, void* stream) {
  (void)init_state;
  int s = check_sizes(B, H, N, d, C, dtype);
  if (s) return s;
  if (N == 0) return LASP_OK;
  if ((s = check_ptrs({q, k, v, dout, dq, dk, dv, state_cache, dstate_ws}, {decay, init_state, dstate_in, dinit_state})))
    return s;
  cudaStream_t st = (cudaStream_t)stream;
  if ((s = bwd_states_impl(q, dout, decay, B, H, N, d, C, dtype, dstate_ws, nullptr, st))) return s;
  return bwd_finish_impl(q, k, v, decay, dout, dq, dk, dv, B, H, N, d, C, dtype, state_cache, dstate_ws, dstate_in,
                         dinit_state, st);
}

int lasp_check_device_status(void* stream, int* site) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return LASP_ERR_CUDA;
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, g_device_status, sizeof(word)) != cudaSuccess) return LASP_ERR_CUDA;
  if (word != 0 && cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return LASP_ERR_CUDA;
  if (site) *site = (int)(word & 0xFFFFu);
  return (int)(word >> 16);
}

int lasp_trace_enable(int capacity) {
  if (capacity < 0) return LASP_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_trace.mu);
  for (cudaEvent_t e : g_trace.ev) cudaEventDestroy(e);
  g_trace.ev.clear();
  g_trace.ids.assign(capacity, 0);
  g_trace.n = 0;
  g_trace.cap = 0;
  for (int i = 0; i < 2 * capacity; ++i) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) {
      for (cudaEvent_t x : g_trace.ev) cudaEventDestroy(x);
      g_trace.ev.clear();
      return LASP_ERR_CUDA;
    }
    g_trace.ev.push_back(e);
  }
  g_trace.cap = capacity;
  return LASP_OK;
}

int lasp_trace_read(int* kernel_ids, float* ms, int capacity) {
  if (capacity < 0 || (capacity > 0 && (kernel_ids == nullptr || ms == nullptr))) return -LASP_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_trace.mu);
  const int n = g_trace.n < capacity ? g_trace.n : capacity;
  for (int i = 0; i < n; ++i) {
    if (cudaEventSynchronize(g_trace.ev[2 * i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms[i], g_trace.ev[2 * i], g_trace.ev[2 * i + 1]) != cudaSuccess)
      return -LASP_ERR_CUDA;
    kernel_ids[i] = g_trace.ids[i];
  }
  g_trace.n = 0;
  return n;
}

const char* lasp_kernel_name(int id) {
  switch (id) {
    case K_STATES_TC: return "chunk_states_tc";
    case K_STATES_SIMT: return "chunk_states_simt";
    case K_SCAN: return "state_scan";
    case K_OUT_TC: return "chunk_out_tc";
    case K_OUT_SIMT: return "chunk_out_simt";
    case K_BWD_TC: return "chunk_bwd_tc";
    case K_BWD_SIMT: return "chunk_bwd_simt";
    case K_FWD_WALK: return "fwd_walk_tc";
    case K_BWD_WALK: return "bwd_walk_tc";
    case K_SEG_STATES: return "segment_states_tc";
    case K_SEG_SCAN: return "segment_scan";
    case K_PROBE: return "wait_probe";
    case K_BIDIR_TOTAL: return "bidir_total";
    case K_BIDIR_APPLY: return "bidir_apply_tc";
    case K_GLA_STATES: return "gla_states_simt";
    case K_GLA_SCAN: return "gla_scan";
    case K_GLA_OUT: return "gla_out_simt";
    case K_GLA_BWD: return "gla_bwd_simt";
    case K_GLA_STATES_TC: return "gla_states_tc";
    case K_GLA_OUT_TC: return "gla_out_tc";
    case K_GLA_BWD_TC: return "gla_bwd_tc";
    case K_STATE_TOTAL: return "state_total";
    case K_GLA_SEG_STATES: return "gla_segment_states_tc";
    case K_GLA_SEG_SCAN: return "gla_segment_scan";
    case K_GLA_EXACT_STATES: return "gla_states_exact";
    case K_GLA_EXACT_SCAN: return "gla_scan_exact";
    case K_GLA_EXACT_OUT: return "gla_out_exact";
    case K_GLA_EXACT_BWD: return "gla_bwd_exact";
    case K_SOFTMAX_FWD: return "softmax_fwd_tc";
    case K_SOFTMAX_DELTA: return "softmax_delta";
    case K_SOFTMAX_DKDV: return "softmax_dkdv_tc";
    case K_SOFTMAX_DQ: return "softmax_dq_tc";
    default: return "unknown";
  }
}

int lasp_segment_tokens(int64_t N, int C, int d, int dtype) {
  if (N <= 0 || C < 1 || N % C != 0) return 0;
  return tc_fwd_walk_ok(dtype, d, C, N) ? walk_segment_tokens(N, C) : C;
}

int lasp_set_wait_limit_ns(uint64_t limit_ns) {
  unsigned long long v = limit_ns;
  return cuda_status(cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)));
}

int lasp_wait_probe(void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  return cuda_status(traced(K_PROBE, st, [&] {
    wait_probe_kernel<<<1, 32, 0, st>>>();
    return cudaGetLastError();
  }));
}

}  // extern "C"

// ------------------------------------------------ bidirectional (unmasked) form
namespace {
int64_t bidir_segments(int64_t N) { return N / walk_segment_tokens(N, 128); }
}  // namespace

int64_t lasp_bidir_workspace_floats(int B, int H, int64_t N, int d, int dtype) {
  using namespace lasp;
  if (lasp::api_detail::check_sizes(B, H, N, d, 1, dtype) || N == 0 || !tc_bidir_ok(dtype, d, N)) return 0;
  const int64_t s = (int64_t)d * d;
  return ((int64_t)B * bidir_segments(N) * H + (int64_t)B * H) * s + (int64_t)B * H * s / 2;
}

int64_t lasp_bidir_state_offset(int B, int H, int64_t N, int d, int dtype) {
  using namespace lasp;
  if (lasp::api_detail::check_sizes(B, H, N, d, 1, dtype) || N == 0 || !tc_bidir_ok(dtype, d, N)) return -1;
  return (int64_t)B * bidir_segments(N) * H * d * d;
}

namespace {
// segment states of (a, b) with lambda = 1 into ws, then their sum (fp32 and
// the bf16 operand tile) behind them
int bidir_total_state(const void* a, const void* b, int kind, float* ws, int B, int H, int64_t N, int d,
                      cudaStream_t st) {
  using namespace lasp;
  using namespace lasp::api_detail;
  const int G = walk_segment_tokens(N, 128);
  const int nseg = (int)(N / G);
  const int64_t off = (int64_t)B * nseg * H * d * d;
  int s;
  if ((s = cuda_status(traced(K_SEG_STATES, st, [&] {
         return tc_chunk_states_slots(a, b, nullptr, ws, B, H, N, d, G, kind, nseg, 1, 0, st);
       }))))
    return s;
  return cuda_status(traced(K_BIDIR_TOTAL, st, [&] {
    return bidir_total(ws, ws + off, ws + off + (int64_t)B * H * d * d, B, H, nseg, st);
  }));
}
}  // namespace

int lasp_bidir_fwd(const void* q, const void* k, const void* v, void* o, int B, int H, int64_t N, int d, int dtype,
                   float* ws, void* stream) {
  using namespace lasp;
  using namespace lasp::api_detail;
  int s = check_sizes(B, H, N, d, 1, dtype);
  if (s) return s;
  if (N == 0) return LASP_OK;
  if (!tc_bidir_ok(dtype, d, N)) return LASP_ERR_UNSUPPORTED;
  if ((s = check_ptrs({q, k, v, o, ws}, {}))) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if ((s = bidir_total_state(k, v, 0, ws, B, H, N, d, st))) return s;
  const float* tiles = ws + lasp_bidir_state_offset(B, H, N, d, dtype) + (int64_t)B * H * d * d;
  const int sms = num_sms_current_device();
  return cuda_status(traced(K_BIDIR_APPLY, st, [&] { return tc_bidir_apply(q, tiles, o, B, H, N, d, 0, sms, st); }));
}

int lasp_bidir_bwd(const void* q, const void* k, const void* v, const void* dout, void* dq, void* dk, void* dv, int B,
                   int H, int64_t N, int d, int dtype, const float* ws, float* dws, void* stream) {
  using namespace lasp;
  using namespace lasp::api_detail;
  int s = check_sizes(B, H, N, d, 1, dtype);
  if (s) return s;
  if (N == 0) return LASP_OK;
  if (!tc_bidir_ok(dtype, d, N)) return LASP_ERR_UNSUPPORTED;
  if ((s = check_ptrs({q, k, v, dout, dq, dk, dv, ws, dws}, {}))) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if ((s = bidir_total_state(q, dout, 1, dws, B, H, N, d, st))) return s;
  const int64_t toff = lasp_bidir_state_offset(B, H, N, d, dtype) + (int64_t)B * H * d * d;
  const float* m_tiles = ws + toff;
  const float* dm_tiles = dws + toff;
  const int sms = num_sms_current_device();
  // dQ = dO M^T, dK = V dM^T, dV = K dM
  if ((s = cuda_status(traced(K_BIDIR_APPLY, st, [&] { return tc_bidir_apply(dout, m_tiles, dq, B, H, N, d, 1, sms, st); }))))
    return s;
  if ((s = cuda_status(traced(K_BIDIR_APPLY, st, [&] { return tc_bidir_apply(v, dm_tiles, dk, B, H, N, d, 1, sms, st); }))))
    return s;
  return cuda_status(traced(K_BIDIR_APPLY, st, [&] { return tc_bidir_apply(k, dm_tiles, dv, B, H, N, d, 0, sms, st); }));
}
