// CUDA-core kernels of the gated form: a decay per token and key feature.
// Page "Linear Attention Sequence Parallelism" (LASP), Appendix A.4, Eq. 24
// (m_t = o_t m_{t-1} + e_t i_t^T) with the GLA / GateLoop row of Table 5
// (oscillation g_t 1^T): per batch b and head h,
//     S_s = diag(exp(g_s)) S_{s-1} + k_s^T v_s,    o_s = q_s S_s,
// g_s[i] being the natural log of the gate of key feature i.
//
// Chunked form (0-based; chunk c holds tokens cC .. cC+C-1). Inside a chunk
// b_t[i] = sum_{r<=t} g_{cC+r}[i] (inclusive, from the chunk start) and
// b_end = b_{C-1}, the chunk's total log-gate ("gsum"):
//   states, kind 0:  M_c[i][j]  = sum_t e^{b_end[i]-b_t[i]} k_t[i] v_t[j]
//   states, kind 1:  dM_c[i][j] = sum_t e^{b_t[i]} q_t[i] do_t[j]
//   output:  o_t = (q_t . e^{b_t}) P_c + sum_{s<=t} A_ts v_s,
//            A_ts = sum_i q_t[i] k_s[i] e^{b_t[i]-b_s[i]}
//   gradients, given P_c (entering) and R_c (gradient of the state leaving):
//     dq_t = e^{b_t} . (do_t P_c^T) + sum_{s<=t} (do_t . v_s) k_s . e^{b_t-b_s}
//     dk_s = sum_{t>=s} (do_t . v_s) q_t . e^{b_t-b_s} + e^{b_end-b_s} . (v_s R_c^T)
//     dv_s = sum_{t>=s} A_ts do_t + (k_s . e^{b_end-b_s}) R_c
//     dg_s = sum_{t>=s} (q_t . dq'_t - k_t . dk'_t) + sum_{t<s} k_t . dk^inter_t
//            + e^{b_end} . rowsum(R_c . P_c)                          (t in the chunk)
//   with dq' = dq minus its s = t term (do_t . v_t) k_t, and dk' = dk minus its
//   t = s term (do_s . v_s) q_s and minus its inter term dk^inter_s =
//   e^{b_end-b_s} . (v_s R_c^T).
// The log-gate gradient follows from the output depending on the gates only
// through q_t e^{b_t}, k_s e^{-b_s} and the leaving state's e^{b_end}: summed
// over t >= s, q_t . dq_t - k_t . dk_t plus rowsum(R_c . S_end) (S_end the state
// leaving the chunk) is dg_s. The arrangement above is the same sum with the
// two exactly cancelling parts left out (the s = t pair of every token, and
// the t >= s part of sum_t k_t . dk^inter_t, which rowsum(R_c . S_end) adds
// back), so that every remaining term carries the gates between its two ends:
// with strong gates dg is then tiny and still accurate to its own size.
//
// Every gate factor is exp2 of a difference of cumulative log-gates taken per
// element, so none overflows: for gates in (0, 1] each factor is at most 1.
// One CTA per (chunk, head, batch); the chunk's cumulative log-gates (times
// log2 e) sit in shared memory.
#include "kernels.h"
#include "lasp_common.cuh"

namespace lasp {
namespace gla_simt_detail {

constexpr int kWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T>
__device__ __forceinline__ const T* row_ptr(const T* x, int b, int64_t n, int h, int H, int64_t N, int D) {
  return x + (((int64_t)b * N + n) * H + h) * D;
}

// cb[t * D + i] = log2(e) * b_t[i] for the chunk's tokens, and gsum[i] =
// b_end[i] if gsum is given. One thread per feature walks the tokens (the
// loads of a warp are consecutive features of one token). All threads call it.
template <int D>
__device__ __forceinline__ void cumulative_gates(const float* __restrict__ g, float* cb, float* gsum, int b,
                                                 int64_t c, int h, int H, int64_t N, int C) {
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    const float* gp = g + (((int64_t)b * N + c * C) * H + h) * D + i;
    float acc = 0.f;
    for (int t = 0; t < C; ++t) {
      acc += gp[(int64_t)t * H * D];
      cb[t * D + i] = acc * kLog2e;
    }
    if (gsum) gsum[i] = acc;
  }
  __syncthreads();
}

template <typename T, int D>
__global__ void __launch_bounds__(256) gla_states_simt(const T* __restrict__ x, const T* __restrict__ y,
                                                       const float* __restrict__ g, float* __restrict__ M,
                                                       float* __restrict__ gsum, int B, int H, int64_t N, int C,
                                                       int kind, RunIf run_if) {
  if (!runs(run_if)) return;
  constexpr int TB = 32;
  constexpr int R = D * D / 256;
  extern __shared__ float smem[];
  float* cb = smem;       // [C][D]
  float* xs = cb + C * D;  // [TB][D], gate-weighted x
  float* ys = xs + TB * D;  // [TB][D]
  const int64_t nchunks = N / C;
  const int64_t items = nchunks * H * (int64_t)B;
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
  const int c = (int)(item % nchunks), h = (int)((item / nchunks) % H), b = (int)(item / (nchunks * H));
  const int64_t slot = ((int64_t)b * nchunks + c) * H + h;
  cumulative_gates<D>(g, cb, gsum ? gsum + slot * D : nullptr, b, c, h, H, N, C);
  const float* cend = cb + (C - 1) * D;
  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.f;
  for (int t0 = 0; t0 < C; t0 += TB) {
    for (int e = threadIdx.x; e < TB * D; e += blockDim.x) {
      const int t = e / D, f = e % D;
      float va = 0.f, vb = 0.f;
      if (t0 + t < C) {
        const int64_t n = (int64_t)c * C + t0 + t;
        const float lg = cb[(t0 + t) * D + f];
        const float w = kind == 0 ? exp2f(cend[f] - lg) : exp2f(lg);
        va = w * Elem<T>::load(row_ptr(x, b, n, h, H, N, D) + f);
        vb = Elem<T>::load(row_ptr(y, b, n, h, H, N, D) + f);
      }
      xs[t * D + f] = va;
      ys[t * D + f] = vb;
    }
    __syncthreads();
    const int tn = min(TB, C - t0);
    for (int t = 0; t < tn; ++t) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int e = threadIdx.x + 256 * r;
        acc[r] = fmaf(xs[t * D + e / D], ys[t * D + e % D], acc[r]);
      }
    }
    __syncthreads();
  }
  float* out = M + slot * D * D;
#pragma unroll
  for (int r = 0; r < R; ++r) out[threadIdx.x + 256 * r] = acc[r];
  __syncthreads();  // the next item rewrites the shared arrays
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) gla_out_simt(const T* __restrict__ q, const T* __restrict__ k,
                                                            const T* __restrict__ v, const float* __restrict__ g,
                                                            const float* __restrict__ P, T* __restrict__ o, int B,
                                                            int H, int64_t N, int C, RunIf run_if) {
  if (!runs(run_if)) return;
  constexpr int R = D / 32;
  extern __shared__ float cb[];  // [C][D]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nchunks = N / C;
  const int64_t items = nchunks * H * (int64_t)B;
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
  const int c = (int)(item % nchunks), h = (int)((item / nchunks) % H), b = (int)(item / (nchunks * H));
  cumulative_gates<D>(g, cb, nullptr, b, c, h, H, N, C);
  const float* Pc = P + (((int64_t)b * nchunks + c) * H + h) * D * D;
  for (int i = warp; i < C; i += kWarps) {
    const int64_t ni = (int64_t)c * C + i;
    const T* qi = row_ptr(q, b, ni, h, H, N, D);
    float qr[R], ci[R], acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      qr[r] = Elem<T>::load(qi + lane + 32 * r);
      ci[r] = cb[i * D + lane + 32 * r];
      acc[r] = 0.f;
    }
    for (int j = 0; j <= i; ++j) {
      const int64_t nj = (int64_t)c * C + j;
      const T* kj = row_ptr(k, b, nj, h, H, N, D);
      const T* vj = row_ptr(v, b, nj, h, H, N, D);
      float s = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int f = lane + 32 * r;
        s = fmaf(qr[r] * exp2f(ci[r] - cb[j * D + f]), Elem<T>::load(kj + f), s);
      }
      s = warp_sum(s);
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = fmaf(s, Elem<T>::load(vj + lane + 32 * r), acc[r]);
    }
    float qe[R];
#pragma unroll
    for (int r = 0; r < R; ++r) qe[r] = qr[r] * exp2f(ci[r]);
    for (int m = 0; m < D; ++m) {
      const float qm = __shfl_sync(0xffffffffu, qe[m / 32], m % 32);
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = fmaf(qm, Pc[m * D + lane + 32 * r], acc[r]);
    }
    T* oi = o + (((int64_t)b * N + ni) * H + h) * D;
#pragma unroll
    for (int r = 0; r < R; ++r) Elem<T>::store(oi + lane + 32 * r, acc[r]);
  }
  __syncthreads();  // the next item rewrites the cumulative gates
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) gla_bwd_simt(const T* __restrict__ q, const T* __restrict__ k,
                                                            const T* __restrict__ v, const T* __restrict__ dout,
                                                            const float* __restrict__ g, const float* __restrict__ P,
                                                            const float* __restrict__ Rs, T* __restrict__ dq,
                                                            T* __restrict__ dk, T* __restrict__ dv,
                                                            float* __restrict__ dg, int B, int H, int64_t N, int C,
                                                            RunIf run_if) {
  if (!runs(run_if)) return;
  constexpr int R = D / 32;
  extern __shared__ float smem[];
  float* cb = smem;          // [C][D] cumulative log-gates (times log2 e)
  float* dB = cb + C * D;    // [C][D] q . dq' - k . dk' of each token
  float* kdi = dB + C * D;   // [C][D] k . dk^inter of each token
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nchunks = N / C;
  const int64_t items = nchunks * H * (int64_t)B;
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
  const int c = (int)(item % nchunks), h = (int)((item / nchunks) % H), b = (int)(item / (nchunks * H));
  cumulative_gates<D>(g, cb, nullptr, b, c, h, H, N, C);
  const float* cend = cb + (C - 1) * D;
  const float* Pc = P + (((int64_t)b * nchunks + c) * H + h) * D * D;
  const float* Rc = Rs + (((int64_t)b * nchunks + c) * H + h) * D * D;
  for (int i = warp; i < C; i += kWarps) {
    const int64_t ni = (int64_t)c * C + i;
    float qi[R], ki[R], vi[R], doi[R], ci[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int f = lane + 32 * r;
      qi[r] = Elem<T>::load(row_ptr(q, b, ni, h, H, N, D) + f);
      ki[r] = Elem<T>::load(row_ptr(k, b, ni, h, H, N, D) + f);
      vi[r] = Elem<T>::load(row_ptr(v, b, ni, h, H, N, D) + f);
      doi[r] = Elem<T>::load(row_ptr(dout, b, ni, h, H, N, D) + f);
      ci[r] = cb[i * D + f];
    }
    float gq[R], gk[R], gv[R];  // dq', dk' (no s = t term, no inter term in dk) and dv
#pragma unroll
    for (int r = 0; r < R; ++r) gq[r] = gk[r] = gv[r] = 0.f;
    // dq: keys s < i
    for (int j = 0; j < i; ++j) {
      const int64_t nj = (int64_t)c * C + j;
      const T* kj = row_ptr(k, b, nj, h, H, N, D);
      const T* vj = row_ptr(v, b, nj, h, H, N, D);
      float s = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) s = fmaf(doi[r], Elem<T>::load(vj + lane + 32 * r), s);
      s = warp_sum(s);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int f = lane + 32 * r;
        gq[r] = fmaf(s * exp2f(ci[r] - cb[j * D + f]), Elem<T>::load(kj + f), gq[r]);
      }
    }
    // the s = t pair: dq += (do_i . v_i) k_i, dk += (do_i . v_i) q_i, dv += (q_i . k_i) do_i
    float sd = 0.f, ad = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      sd = fmaf(doi[r], vi[r], sd);
      ad = fmaf(qi[r], ki[r], ad);
    }
    sd = warp_sum(sd);
    ad = warp_sum(ad);
#pragma unroll
    for (int r = 0; r < R; ++r) gv[r] = ad * doi[r];
    // dk, dv: queries t > i
    for (int t = i + 1; t < C; ++t) {
      const int64_t nt = (int64_t)c * C + t;
      const T* qt = row_ptr(q, b, nt, h, H, N, D);
      const T* dot = row_ptr(dout, b, nt, h, H, N, D);
      float sb = 0.f, sc = 0.f;
      float qw[R], dtr[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int f = lane + 32 * r;
        qw[r] = Elem<T>::load(qt + f) * exp2f(cb[t * D + f] - ci[r]);  // q_t e^{b_t - b_i}
        dtr[r] = Elem<T>::load(dot + f);
        sb = fmaf(dtr[r], vi[r], sb);
        sc = fmaf(qw[r], ki[r], sc);
      }
      sb = warp_sum(sb);  // do_t . v_i
      sc = warp_sum(sc);  // A_ti
#pragma unroll
      for (int r = 0; r < R; ++r) {
        gk[r] = fmaf(sb, qw[r], gk[r]);
        gv[r] = fmaf(sc, dtr[r], gv[r]);
      }
    }
    // inter terms: dq += e^{b_i} (P do_i); dk^inter = e^{b_end - b_i} (R v_i);
    // dv += R^T (k_i e^{b_end - b_i})
    float eq[R], ek[R], iv[R], gki[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      eq[r] = exp2f(ci[r]);
      ek[r] = exp2f(cend[lane + 32 * r] - ci[r]);
      iv[r] = 0.f;
      gki[r] = 0.f;
    }
    for (int m = 0; m < D; ++m) {
      float pq = 0.f, rk = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        pq = fmaf(Pc[m * D + lane + 32 * r], doi[r], pq);
        rk = fmaf(Rc[m * D + lane + 32 * r], vi[r], rk);
      }
      pq = warp_sum(pq);
      rk = warp_sum(rk);
      const float km = __shfl_sync(0xffffffffu, ki[m / 32] * ek[m / 32], m % 32);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (m / 32 == r && m % 32 == lane) {
          gq[r] = fmaf(eq[r], pq, gq[r]);
          gki[r] = ek[r] * rk;
        }
        iv[r] = fmaf(km, Rc[m * D + lane + 32 * r], iv[r]);
      }
    }
    const int64_t off = (((int64_t)b * N + ni) * H + h) * D;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int f = lane + 32 * r;
      Elem<T>::store(dq + off + f, fmaf(sd, ki[r], gq[r]));
      Elem<T>::store(dk + off + f, fmaf(sd, qi[r], gk[r]) + gki[r]);
      Elem<T>::store(dv + off + f, gv[r] + iv[r]);
      dB[i * D + f] = qi[r] * gq[r] - ki[r] * gk[r];
      kdi[i * D + f] = ki[r] * gki[r];
    }
  }
  __syncthreads();
  // dg, one thread per feature: the suffix of dB, the exclusive prefix of
  // k . dk^inter, and e^{b_end} <R_c, P_c> of the feature's row
  for (int f = threadIdx.x; f < D; f += blockDim.x) {
    float rp = 0.f;
    for (int j = 0; j < D; ++j) rp = fmaf(Rc[f * D + j], Pc[f * D + j], rp);
    const float bnd = exp2f(cend[f]) * rp;
    float pre = 0.f;
    for (int t = 0; t < C; ++t) {  // dB[t] <- sum_{t' < t} k . dk^inter
      const float x = kdi[t * D + f];
      kdi[t * D + f] = pre;
      pre += x;
    }
    float run = 0.f;
    for (int t = C - 1; t >= 0; --t) {
      run += dB[t * D + f];
      dg[(((int64_t)b * N + (int64_t)c * C + t) * H + h) * D + f] = run + kdi[t * D + f] + bnd;
    }
  }
  __syncthreads();  // the next item rewrites the shared arrays
  }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename T, int D>
cudaError_t launch_states_d(const void* x, const void* y, const float* g, float* M, float* gsum, int B, int H,
                            int64_t N, int C, int kind, cudaStream_t st, RunIf run) {
  const size_t smem = (size_t)(C + 64) * D * sizeof(float);
  cudaError_t e = set_smem(gla_states_simt<T, D>, smem);
  if (e != cudaSuccess) return e;
  gla_states_simt<T, D><<<(unsigned)grid_for(N / C * H * B, run), 256, smem, st>>>((const T*)x, (const T*)y, g, M, gsum, B, H,
                                                                          N, C, kind, run);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_out_d(const void* q, const void* k, const void* v, const float* g, const float* P, void* o,
                         int B, int H, int64_t N, int C, cudaStream_t st, RunIf run) {
  const size_t smem = (size_t)C * D * sizeof(float);
  cudaError_t e = set_smem(gla_out_simt<T, D>, smem);
  if (e != cudaSuccess) return e;
  gla_out_simt<T, D><<<(unsigned)grid_for(N / C * H * B, run), kWarps * 32, smem, st>>>(
      (const T*)q, (const T*)k, (const T*)v, g, P, (T*)o, B, H, N, C, run);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_bwd_d(const void* q, const void* k, const void* v, const void* dout, const float* g,
                         const float* P, const float* Rs, void* dq, void* dk, void* dv, float* dg, int B, int H,
                         int64_t N, int C, cudaStream_t st, RunIf run) {
  const size_t smem = (size_t)3 * C * D * sizeof(float);
  cudaError_t e = set_smem(gla_bwd_simt<T, D>, smem);
  if (e != cudaSuccess) return e;
  gla_bwd_simt<T, D><<<(unsigned)grid_for(N / C * H * B, run), kWarps * 32, smem, st>>>(
      (const T*)q, (const T*)k, (const T*)v, (const T*)dout, g, P, Rs, (T*)dq, (T*)dk, (T*)dv, dg, B, H, N, C, run);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_states(const void* x, const void* y, const float* g, float* M, float* gsum, int B, int H,
                          int64_t N, int d, int C, int kind, cudaStream_t st, RunIf run) {
  switch (d) {
    case 32: return launch_states_d<T, 32>(x, y, g, M, gsum, B, H, N, C, kind, st, run);
    case 64: return launch_states_d<T, 64>(x, y, g, M, gsum, B, H, N, C, kind, st, run);
    default: return launch_states_d<T, 128>(x, y, g, M, gsum, B, H, N, C, kind, st, run);
  }
}

template <typename T>
cudaError_t launch_out(const void* q, const void* k, const void* v, const float* g, const float* P, void* o, int B,
                       int H, int64_t N, int d, int C, cudaStream_t st, RunIf run) {
  switch (d) {
    case 32: return launch_out_d<T, 32>(q, k, v, g, P, o, B, H, N, C, st, run);
    case 64: return launch_out_d<T, 64>(q, k, v, g, P, o, B, H, N, C, st, run);
    default: return launch_out_d<T, 128>(q, k, v, g, P, o, B, H, N, C, st, run);
  }
}

template <typename T>
cudaError_t launch_bwd(const void* q, const void* k, const void* v, const void* dout, const float* g,
                       const float* P, const float* Rs, void* dq, void* dk, void* dv, float* dg, int B, int H,
                       int64_t N, int d, int C, cudaStream_t st, RunIf run) {
  switch (d) {
    case 32: return launch_bwd_d<T, 32>(q, k, v, dout, g, P, Rs, dq, dk, dv, dg, B, H, N, C, st, run);
    case 64: return launch_bwd_d<T, 64>(q, k, v, dout, g, P, Rs, dq, dk, dv, dg, B, H, N, C, st, run);
    default: return launch_bwd_d<T, 128>(q, k, v, dout, g, P, Rs, dq, dk, dv, dg, B, H, N, C, st, run);
  }
}

}  // namespace gla_simt_detail

cudaError_t gla_simt_chunk_states(const void* x, const void* y, const float* g, float* M, float* gsum, int B, int H,
                                  int64_t N, int d, int C, int kind, int dtype, cudaStream_t st, RunIf run) {
  using namespace gla_simt_detail;
  return dtype == LASP_F32 ? launch_states<float>(x, y, g, M, gsum, B, H, N, d, C, kind, st, run)
                           : launch_states<__nv_bfloat16>(x, y, g, M, gsum, B, H, N, d, C, kind, st, run);
}

cudaError_t gla_simt_chunk_out(const void* q, const void* k, const void* v, const float* g, const float* P, void* o,
                               int B, int H, int64_t N, int d, int C, int dtype, cudaStream_t st, RunIf run) {
  using namespace gla_simt_detail;
  return dtype == LASP_F32 ? launch_out<float>(q, k, v, g, P, o, B, H, N, d, C, st, run)
                           : launch_out<__nv_bfloat16>(q, k, v, g, P, o, B, H, N, d, C, st, run);
}

cudaError_t gla_simt_chunk_bwd(const void* q, const void* k, const void* v, const void* dout, const float* g,
                               const float* P, const float* Rs, void* dq, void* dk, void* dv, float* dg, int B, int H,
                               int64_t N, int d, int C, int dtype, cudaStream_t st, RunIf run) {
  using namespace gla_simt_detail;
  return dtype == LASP_F32 ? launch_bwd<float>(q, k, v, dout, g, P, Rs, dq, dk, dv, dg, B, H, N, d, C, st, run)
                           : launch_bwd<__nv_bfloat16>(q, k, v, dout, g, P, Rs, dq, dk, dv, dg, B, H, N, d, C, st,
                                                       run);
}

}  // namespace lasp
