// Internal launchers behind the C ABI of include/lasp.h. Each returns the
// cudaError_t of its launch; arguments are already validated by lasp_api.cu.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace lasp {

// A launch whose work depends on a word an earlier kernel of the same call
// wrote on the device: the kernel runs when flag is NULL or when (*flag != 0)
// equals want, and returns at once otherwise. This lets a call choose between
// two kernel sequences on the device, with no host synchronisation.
struct RunIf {
  const int* flag = nullptr;
  int want = 0;
};

// Blocks for a kernel that loops over `items` work items with a grid stride:
// one block per item, except for a launch that runs only when the flag is set
// (want = 1: the gated form's exact fallback, which usually returns at once),
// which gets two per SM, so that skipping costs little.
inline int64_t grid_for(int64_t items, RunIf run) {
  if (run.flag == nullptr || run.want == 0) return items;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return items < 2 * (int64_t)sms ? items : 2 * (int64_t)sms;
}

// Exclusive decayed scan over chunk states (k_state_scan.cu).
cudaError_t launch_state_scan(const float* M, float* P, const float* decay, const float* init, float* total,
                              int B, int T, int H, int d, int64_t C, int reverse, cudaStream_t st);

// The same scan over every slot_stride-th state of an array of t_slots states,
// starting at slot slot_offset (segment states stored inside a chunk array).
// bh0, nbh: only the (b, h) pairs bh0 .. bh0 + nbh - 1 (b-major; nbh < 0: all);
// init and total stay [B, H, d, d] arrays.
cudaError_t launch_state_scan_slots(const float* M, float* P, const float* decay, const float* init, float* total,
                                    int B, int T, int H, int d, int64_t C, int reverse, int64_t t_slots,
                                    int slot_stride, int slot_offset, cudaStream_t st, int64_t bh0 = 0,
                                    int64_t nbh = -1);

// CUDA-core kernels, any d in {32, 64, 128} and any C (k_simt.cu).
// kind 0: M_c = sum lambda^{C-1-t} a_t^T b_t ; kind 1: sum lambda^{t+1} a_t^T b_t.
cudaError_t simt_chunk_states(const void* a, const void* b, const float* decay, float* M, int B, int H,
                              int64_t N, int d, int C, int kind, int dtype, cudaStream_t st);
cudaError_t simt_chunk_out(const void* q, const void* k, const void* v, const float* decay, const float* P,
                           void* o, int B, int H, int64_t N, int d, int C, int dtype, cudaStream_t st);
cudaError_t simt_chunk_bwd(const void* q, const void* k, const void* v, const void* dout, const float* decay,
                           const float* P, const float* Rs, void* dq, void* dk, void* dv, int B, int H,
                           int64_t N, int d, int C, int dtype, cudaStream_t st);

// Gated form (k_gla_simt.cu, k_state_scan.cu): a decay per token and key
// feature; g is the log-gate [B, N, H, d] (float32), gsum the chunk totals
// [B, T, H, d]. kind 0: M_c = sum_t diag(e^{b_end - b_t}) k_t^T v_t (and
// gsum if non-null); kind 1: dM_c = sum_t diag(e^{b_t}) q_t^T do_t.
cudaError_t gla_simt_chunk_states(const void* x, const void* y, const float* g, float* M, float* gsum, int B, int H,
                                  int64_t N, int d, int C, int kind, int dtype, cudaStream_t st, RunIf run = {});
// The gated scan over T elements held in every slot_stride-th slot (from
// slot_offset) of an array of t_slots states; element c's log-gate totals in
// slot c * slot_stride + gsum_offset of gsum.
cudaError_t launch_gla_scan(const float* M, float* P, const float* gsum, const float* init, float* total, int B,
                            int T, int H, int d, int reverse, int64_t t_slots, int slot_stride, int slot_offset,
                            int gsum_offset, cudaStream_t st, RunIf run = {});
cudaError_t gla_simt_chunk_out(const void* q, const void* k, const void* v, const float* g, const float* P, void* o,
                               int B, int H, int64_t N, int d, int C, int dtype, cudaStream_t st, RunIf run = {});
cudaError_t gla_simt_chunk_bwd(const void* q, const void* k, const void* v, const void* dout, const float* g,
                               const float* P, const float* Rs, void* dq, void* dk, void* dv, float* dg, int B, int H,
                               int64_t N, int d, int C, int dtype, cudaStream_t st, RunIf run = {});

// One CTA waiting on a barrier nothing completes; ends by the wait limit.
cudaError_t launch_wait_probe(cudaStream_t st);

}  // namespace lasp
