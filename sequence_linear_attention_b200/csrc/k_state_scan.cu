// Exclusive decayed scan over per-chunk d x d states (LASP-2: prefix sum of
// the gathered M_t in the forward pass, suffix sum of dM_t in the backward
// pass; LASP Eq. 10 and Eq. 20 give the per-chunk decay lambda^C).
//
//   forward:  P_0 = init,     P_c = g P_{c-1} + M_{c-1},  g = lambda^C
//   reverse:  R_{T-1} = init, R_c = g R_{c+1} + M_{c+1}
//
// The gated form (LASP Appendix A.4, Eq. 24 with the GLA row of Table 5)
// replaces the scalar g by a diagonal: the step through chunk c scales row i
// by exp(gsum_c[i]), gsum_c being the chunk's total log-gate (kGated).
//
// The scan is pure HBM traffic: every state element is read once and written
// once. One thread owns one float4 of the d*d state of one (b, h) and walks the
// chunks in order; the loads of a group of kUnroll chunks do not depend on the
// recurrence, so they are issued one group ahead of the FMAs and stores,
// keeping up to 2 * kUnroll * 16 bytes in flight per thread. Consecutive threads own consecutive
// float4s of one state, so every warp access is a fully coalesced 512-byte run.
// M and P may be the same array: each element is loaded before it is stored,
// by the same thread. With P = NULL only the total is written (the LASP-2
// shard state): the states are then read with plain loads, so that a step that
// scans them again soon after finds them in L2.
#include "kernels.h"
#include "lasp_common.cuh"

namespace lasp {
namespace scan_detail {

constexpr int kUnroll = 8;
constexpr int kThreads = 64;  // small blocks spread the work evenly over the SMs

// store that asks L2 to keep the line (the walk reads P next)
__device__ __forceinline__ void st_keep(float4* p, float4 v, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w), "l"(policy)
               : "memory");
}

__device__ __forceinline__ float4 fma4(float g, float4 a, float4 m) {
  return make_float4(fmaf(g, a.x, m.x), fmaf(g, a.y, m.y), fmaf(g, a.z, m.z), fmaf(g, a.w, m.w));
}

constexpr float kLog2e = 1.4426950408889634f;

// gsum (kGated only): [B, t_slots, H, d] log-gate totals, scan element c's at
// slot c * slot_stride + gsum_offset
template <bool kGated>
__global__ void __launch_bounds__(kThreads) state_scan_kernel(const float4* M, float4* P, const float* decay,
                                                              const float* __restrict__ gsum,
                                                              const float4* __restrict__ init,
                                                              float4* __restrict__ total, int H, int T,
                                                              int d, int dd4, int64_t n_threads, float Cf,
                                                              int reverse, int64_t t_slots, int slot_stride,
                                                              int slot_offset, int gsum_offset, RunIf run_if,
                                                              int64_t idx0) {
  if (!runs(run_if)) return;
  // thread idx of idx0 .. idx0 + n_threads - 1 of the whole (b, h, float4) space
  const int64_t idx = idx0 + (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (idx >= idx0 + n_threads) return;
  const int e = (int)(idx % dd4);
  const int h = (int)((idx / dd4) % H);
  const int64_t b = idx / ((int64_t)dd4 * H);
  const float g = kGated ? 1.f : decay_pow(log2f(load_decay(decay, h)), Cf);
  uint64_t keep;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(keep));
  const int64_t bh = b * H + h;
  float4 acc = init ? init[bh * dd4 + e] : make_float4(0.f, 0.f, 0.f, 0.f);
  // scan element c lives in slot c * slot_stride + slot_offset of an array of t_slots states
  const int64_t cstride = (int64_t)slot_stride * H * dd4;  // float4s between element c and c+1
  const int64_t base = ((b * t_slots + slot_offset) * H + h) * (int64_t)dd4 + e;
  const int64_t step = reverse ? -cstride : cstride;
  int64_t off = reverse ? base + (int64_t)(T - 1) * cstride : base;
  // the log-gate total of this thread's state row in scan element c
  const int64_t gstride = (int64_t)slot_stride * H * d;
  const int64_t gstep = reverse ? -gstride : gstride;
  int64_t goff = ((b * t_slots + gsum_offset) * H + h) * (int64_t)d + (4 * e) / d;
  if (reverse) goff += (int64_t)(T - 1) * gstride;
  // software pipeline: the loads of group g + 1 are issued before group g is
  // scanned and stored, so a group's worth of loads is always in flight
  const int ngroups = T / kUnroll;
  const bool write = P != nullptr;
  auto ld = [&](int64_t i) { return write ? __ldcs(M + i) : __ldg(M + i); };
  float4 cur[kUnroll];
  float gc[kUnroll];
  if (ngroups > 0) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      cur[u] = ld(off + u * step);
      if (kGated) gc[u] = gsum[goff + u * gstep];
    }
  }
  for (int gi = 0; gi < ngroups; ++gi) {
    const bool more = gi + 1 < ngroups;
    float4 nxt[kUnroll];
    float gn[kUnroll];
    if (more) {
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        nxt[u] = ld(off + (kUnroll + u) * step);
        if (kGated) gn[u] = gsum[goff + (kUnroll + u) * gstep];
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (write) st_keep(P + off + u * step, acc, keep);
      acc = fma4(kGated ? exp2f(gc[u] * kLog2e) : g, acc, cur[u]);
    }
    off += kUnroll * step;
    goff += kUnroll * gstep;
    if (more) {
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        cur[u] = nxt[u];
        if (kGated) gc[u] = gn[u];
      }
    }
  }
  int n = ngroups * kUnroll;
  for (; n < T; ++n) {
    float4 m = ld(off);
    if (write) st_keep(P + off, acc, keep);
    acc = fma4(kGated ? exp2f(gsum[goff] * kLog2e) : g, acc, m);
    off += step;
    goff += gstep;
  }
  if (total) total[bh * dd4 + e] = acc;
}

}  // namespace scan_detail

cudaError_t launch_state_scan_slots(const float* M, float* P, const float* decay, const float* init, float* total,
                                    int B, int T, int H, int d, int64_t C, int reverse, int64_t t_slots,
                                    int slot_stride, int slot_offset, cudaStream_t st, int64_t bh0, int64_t nbh) {
  const int dd4 = d * d / 4;
  if (nbh < 0) nbh = (int64_t)B * H;
  const int64_t n_threads = nbh * dd4;
  if (n_threads == 0) return cudaSuccess;
  const int64_t blocks = (n_threads + scan_detail::kThreads - 1) / scan_detail::kThreads;
  scan_detail::state_scan_kernel<false><<<(unsigned)blocks, scan_detail::kThreads, 0, st>>>(
      (const float4*)M, (float4*)P, decay, nullptr, (const float4*)init, (float4*)total, H, T, d, dd4,
      n_threads, (float)C, reverse, t_slots, slot_stride, slot_offset, 0, RunIf{}, bh0 * dd4);
  return cudaGetLastError();
}

cudaError_t launch_gla_scan(const float* M, float* P, const float* gsum, const float* init, float* total, int B,
                            int T, int H, int d, int reverse, int64_t t_slots, int slot_stride, int slot_offset,
                            int gsum_offset, cudaStream_t st, RunIf run) {
  const int dd4 = d * d / 4;
  const int64_t n_threads = (int64_t)B * H * dd4;
  // one thread per element: a launch that returns at once still has the full grid
  const int64_t blocks = (n_threads + scan_detail::kThreads - 1) / scan_detail::kThreads;
  scan_detail::state_scan_kernel<true><<<(unsigned)blocks, scan_detail::kThreads, 0, st>>>(
      (const float4*)M, (float4*)P, nullptr, gsum, (const float4*)init, (float4*)total, H, T, d, dd4, n_threads,
      1.f, reverse, t_slots, slot_stride, slot_offset, gsum_offset, run, 0);
  return cudaGetLastError();
}

cudaError_t launch_state_scan(const float* M, float* P, const float* decay, const float* init, float* total,
                              int B, int T, int H, int d, int64_t C, int reverse, cudaStream_t st) {
  return launch_state_scan_slots(M, P, decay, init, total, B, T, H, d, C, reverse, T, 1, 0, st);
}

}  // namespace lasp
