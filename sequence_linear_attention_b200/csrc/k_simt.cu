// CUDA-core (FFMA) kernels for the chunked forward and backward passes.
//
// These evaluate the chunk equations of the LASP page (v3, section 3.2) with
// fp32 arithmetic and no tensor cores: the fp32 path needs true fp32 products
// (a TF32 tensor-core product would not meet a 1e-4 relative bound), and they
// also serve every size the tensor-core kernels do not take (d = 32, or C not
// a multiple of 16). One CTA per (chunk, head, batch); inside it, one warp per
// token row, features spread over the 32 lanes.
#include "kernels.h"
#include "lasp_common.cuh"

namespace lasp {
namespace simt_detail {

constexpr int kWarps = 4;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T>
__device__ __forceinline__ const T* row_ptr(const T* x, int b, int64_t n, int h, int H, int64_t N, int D) {
  return x + (((int64_t)b * N + n) * H + h) * D;
}

// Chunk states (LASP Eq. 10 with KV_{t-1} = 0, and Eq. 20's (Lambda Q_t)^T dO_t):
//   M_c[i][j] = sum_t w_t a_t[i] b_t[j],  w_t = lambda^{C-1-t} (kind 0) or lambda^{t+1} (kind 1).
template <typename T, int D>
__global__ void __launch_bounds__(256) chunk_states_simt(const T* __restrict__ a, const T* __restrict__ bsrc,
                                                         const float* decay, float* __restrict__ M,
                                                         int H, int64_t N, int C, int kind) {
  constexpr int TB = 32;
  constexpr int R = D * D / 256;
  __shared__ float as[TB][D];
  __shared__ float bs[TB][D];
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t nchunks = N / C;
  const float l2 = log2f(load_decay(decay, h));
  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.f;
  for (int t0 = 0; t0 < C; t0 += TB) {
    for (int e = threadIdx.x; e < TB * D; e += blockDim.x) {
      int t = e / D, f = e % D;
      float va = 0.f, vb = 0.f;
      if (t0 + t < C) {
        int64_t n = (int64_t)c * C + t0 + t;
        float w = kind == 0 ? decay_pow(l2, (float)(C - 1 - (t0 + t))) : decay_pow(l2, (float)(t0 + t + 1));
        va = w * Elem<T>::load(row_ptr(a, b, n, h, H, N, D) + f);
        vb = Elem<T>::load(row_ptr(bsrc, b, n, h, H, N, D) + f);
      }
      as[t][f] = va;
      bs[t][f] = vb;
    }
    __syncthreads();
    const int tn = min(TB, C - t0);
    for (int t = 0; t < tn; ++t) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        int e = threadIdx.x + 256 * r;
        acc[r] = fmaf(as[t][e / D], bs[t][e % D], acc[r]);
      }
    }
    __syncthreads();
  }
  float* out = M + (((int64_t)b * nchunks + c) * H + h) * D * D;
#pragma unroll
  for (int r = 0; r < R; ++r) out[threadIdx.x + 256 * r] = acc[r];
}

// Forward output for one chunk (LASP Eq. 7, 9, 11; Algorithm 2 steps 9, 14, 15):
//   o_i = sum_{j<=i} lambda^{i-j} (q_i . k_j) v_j + lambda^{i+1} q_i P_c.
template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) chunk_out_simt(const T* __restrict__ q, const T* __restrict__ k,
                                                              const T* __restrict__ v, const float* decay,
                                                              const float* __restrict__ P, T* __restrict__ o,
                                                              int H, int64_t N, int C) {
  constexpr int R = D / 32;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nchunks = N / C;
  const float l2 = log2f(load_decay(decay, h));
  const float* Pc = P + (((int64_t)b * nchunks + c) * H + h) * D * D;
  for (int i = warp; i < C; i += kWarps) {
    const int64_t ni = (int64_t)c * C + i;
    const T* qi = row_ptr(q, b, ni, h, H, N, D);
    float qr[R], acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      qr[r] = Elem<T>::load(qi + lane + 32 * r);
      acc[r] = 0.f;
    }
    for (int j = 0; j <= i; ++j) {
      const int64_t nj = (int64_t)c * C + j;
      const T* kj = row_ptr(k, b, nj, h, H, N, D);
      const T* vj = row_ptr(v, b, nj, h, H, N, D);
      float s = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) s = fmaf(qr[r], Elem<T>::load(kj + lane + 32 * r), s);
      s = warp_sum(s) * decay_pow(l2, (float)(i - j));
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = fmaf(s, Elem<T>::load(vj + lane + 32 * r), acc[r]);
    }
    float inter[R];
#pragma unroll
    for (int r = 0; r < R; ++r) inter[r] = 0.f;
    for (int m = 0; m < D; ++m) {
      float qm = __shfl_sync(0xffffffffu, qr[m / 32], m % 32);
#pragma unroll
      for (int r = 0; r < R; ++r) inter[r] = fmaf(qm, Pc[m * D + lane + 32 * r], inter[r]);
    }
    const float wi = decay_pow(l2, (float)(i + 1));
    T* oi = o + ((((int64_t)b * N + ni) * H + h) * D);
#pragma unroll
    for (int r = 0; r < R; ++r) Elem<T>::store(oi + lane + 32 * r, fmaf(wi, inter[r], acc[r]));
  }
}

// Backward for one chunk (LASP Eq. 14, 16, 17, 19, 22, 23; Algorithm 3):
//   dq_i = sum_{j<=i} lambda^{i-j} (do_i . v_j) k_j + lambda^{i+1} do_i P_c^T
//   dk_i = sum_{t>=i} lambda^{t-i} (do_t . v_i) q_t + lambda^{C-1-i} v_i R_c^T
//   dv_i = sum_{t>=i} lambda^{t-i} (q_t . k_i) do_t + lambda^{C-1-i} k_i R_c
template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) chunk_bwd_simt(const T* __restrict__ q, const T* __restrict__ k,
                                                              const T* __restrict__ v, const T* __restrict__ dout,
                                                              const float* decay, const float* __restrict__ P,
                                                              const float* __restrict__ Rs, T* __restrict__ dq,
                                                              T* __restrict__ dk, T* __restrict__ dv,
                                                              int H, int64_t N, int C) {
  constexpr int R = D / 32;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nchunks = N / C;
  const float l2 = log2f(load_decay(decay, h));
  const float* Pc = P + (((int64_t)b * nchunks + c) * H + h) * D * D;
  const float* Rc = Rs + (((int64_t)b * nchunks + c) * H + h) * D * D;
  for (int i = warp; i < C; i += kWarps) {
    const int64_t ni = (int64_t)c * C + i;
    float qi[R], ki[R], vi[R], doi[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      int f = lane + 32 * r;
      qi[r] = Elem<T>::load(row_ptr(q, b, ni, h, H, N, D) + f);
      ki[r] = Elem<T>::load(row_ptr(k, b, ni, h, H, N, D) + f);
      vi[r] = Elem<T>::load(row_ptr(v, b, ni, h, H, N, D) + f);
      doi[r] = Elem<T>::load(row_ptr(dout, b, ni, h, H, N, D) + f);
    }
    float gq[R], gk[R], gv[R];
#pragma unroll
    for (int r = 0; r < R; ++r) gq[r] = gk[r] = gv[r] = 0.f;
    // dq: keys j <= i
    for (int j = 0; j <= i; ++j) {
      const int64_t nj = (int64_t)c * C + j;
      const T* kj = row_ptr(k, b, nj, h, H, N, D);
      const T* vj = row_ptr(v, b, nj, h, H, N, D);
      float s = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) s = fmaf(doi[r], Elem<T>::load(vj + lane + 32 * r), s);
      s = warp_sum(s) * decay_pow(l2, (float)(i - j));
#pragma unroll
      for (int r = 0; r < R; ++r) gq[r] = fmaf(s, Elem<T>::load(kj + lane + 32 * r), gq[r]);
    }
    // dk, dv: queries t >= i
    for (int t = i; t < C; ++t) {
      const int64_t nt = (int64_t)c * C + t;
      const T* qt = row_ptr(q, b, nt, h, H, N, D);
      const T* dot = row_ptr(dout, b, nt, h, H, N, D);
      float sb = 0.f, sc = 0.f;
      float qtr[R], dtr[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        qtr[r] = Elem<T>::load(qt + lane + 32 * r);
        dtr[r] = Elem<T>::load(dot + lane + 32 * r);
        sb = fmaf(dtr[r], vi[r], sb);
        sc = fmaf(qtr[r], ki[r], sc);
      }
      const float w = decay_pow(l2, (float)(t - i));
      sb = warp_sum(sb) * w;
      sc = warp_sum(sc) * w;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        gk[r] = fmaf(sb, qtr[r], gk[r]);
        gv[r] = fmaf(sc, dtr[r], gv[r]);
      }
    }
    // inter terms: dq += lambda^{i+1} P do_i ; dk += lambda^{C-1-i} R v_i ; dv += lambda^{C-1-i} R^T k_i
    const float wq = decay_pow(l2, (float)(i + 1));
    const float wk = decay_pow(l2, (float)(C - 1 - i));
    float iv[R];
#pragma unroll
    for (int r = 0; r < R; ++r) iv[r] = 0.f;
    for (int m = 0; m < D; ++m) {
      float pq = 0.f, rk = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        pq = fmaf(Pc[m * D + lane + 32 * r], doi[r], pq);
        rk = fmaf(Rc[m * D + lane + 32 * r], vi[r], rk);
      }
      pq = warp_sum(pq);
      rk = warp_sum(rk);
      float km = __shfl_sync(0xffffffffu, ki[m / 32], m % 32);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (m / 32 == r && m % 32 == lane) {
          gq[r] = fmaf(wq, pq, gq[r]);
          gk[r] = fmaf(wk, rk, gk[r]);
        }
        iv[r] = fmaf(km, Rc[m * D + lane + 32 * r], iv[r]);
      }
    }
    const int64_t off = (((int64_t)b * N + ni) * H + h) * D;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      int f = lane + 32 * r;
      Elem<T>::store(dq + off + f, gq[r]);
      Elem<T>::store(dk + off + f, gk[r]);
      Elem<T>::store(dv + off + f, fmaf(wk, iv[r], gv[r]));
    }
  }
}

template <typename T>
cudaError_t launch_states(const void* a, const void* b, const float* decay, float* M, int B, int H,
                          int64_t N, int d, int C, int kind, cudaStream_t st) {
  dim3 grid((unsigned)(N / C), H, B);
  const T* pa = (const T*)a;
  const T* pb = (const T*)b;
  switch (d) {
    case 32: chunk_states_simt<T, 32><<<grid, 256, 0, st>>>(pa, pb, decay, M, H, N, C, kind); break;
    case 64: chunk_states_simt<T, 64><<<grid, 256, 0, st>>>(pa, pb, decay, M, H, N, C, kind); break;
    default: chunk_states_simt<T, 128><<<grid, 256, 0, st>>>(pa, pb, decay, M, H, N, C, kind); break;
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_out(const void* q, const void* k, const void* v, const float* decay, const float* P,
                       void* o, int B, int H, int64_t N, int d, int C, cudaStream_t st) {
  dim3 grid((unsigned)(N / C), H, B);
  const T *pq = (const T*)q, *pk = (const T*)k, *pv = (const T*)v;
  T* po = (T*)o;
  switch (d) {
    case 32: chunk_out_simt<T, 32><<<grid, kWarps * 32, 0, st>>>(pq, pk, pv, decay, P, po, H, N, C); break;
    case 64: chunk_out_simt<T, 64><<<grid, kWarps * 32, 0, st>>>(pq, pk, pv, decay, P, po, H, N, C); break;
    default: chunk_out_simt<T, 128><<<grid, kWarps * 32, 0, st>>>(pq, pk, pv, decay, P, po, H, N, C); break;
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_bwd(const void* q, const void* k, const void* v, const void* dout, const float* decay,
                       const float* P, const float* Rs, void* dq, void* dk, void* dv, int B, int H,
                       int64_t N, int d, int C, cudaStream_t st) {
  dim3 grid((unsigned)(N / C), H, B);
  const T *pq = (const T*)q, *pk = (const T*)k, *pv = (const T*)v, *pd = (const T*)dout;
  T *gq = (T*)dq, *gk = (T*)dk, *gv = (T*)dv;
  switch (d) {
    case 32: chunk_bwd_simt<T, 32><<<grid, kWarps * 32, 0, st>>>(pq, pk, pv, pd, decay, P, Rs, gq, gk, gv, H, N, C); break;
    case 64: chunk_bwd_simt<T, 64><<<grid, kWarps * 32, 0, st>>>(pq, pk, pv, pd, decay, P, Rs, gq, gk, gv, H, N, C); break;
    default: chunk_bwd_simt<T, 128><<<grid, kWarps * 32, 0, st>>>(pq, pk, pv, pd, decay, P, Rs, gq, gk, gv, H, N, C); break;
  }
  return cudaGetLastError();
}

}  // namespace simt_detail

cudaError_t simt_chunk_states(const void* a, const void* b, const float* decay, float* M, int B, int H,
                              int64_t N, int d, int C, int kind, int dtype, cudaStream_t st) {
  return dtype == LASP_F32 ? simt_detail::launch_states<float>(a, b, decay, M, B, H, N, d, C, kind, st)
                           : simt_detail::launch_states<__nv_bfloat16>(a, b, decay, M, B, H, N, d, C, kind, st);
}

cudaError_t simt_chunk_out(const void* q, const void* k, const void* v, const float* decay, const float* P,
                           void* o, int B, int H, int64_t N, int d, int C, int dtype, cudaStream_t st) {
  return dtype == LASP_F32 ? simt_detail::launch_out<float>(q, k, v, decay, P, o, B, H, N, d, C, st)
                           : simt_detail::launch_out<__nv_bfloat16>(q, k, v, decay, P, o, B, H, N, d, C, st);
}

cudaError_t simt_chunk_bwd(const void* q, const void* k, const void* v, const void* dout, const float* decay,
                           const float* P, const float* Rs, void* dq, void* dk, void* dv, int B, int H,
                           int64_t N, int d, int C, int dtype, cudaStream_t st) {
  return dtype == LASP_F32
             ? simt_detail::launch_bwd<float>(q, k, v, dout, decay, P, Rs, dq, dk, dv, B, H, N, d, C, st)
             : simt_detail::launch_bwd<__nv_bfloat16>(q, k, v, dout, decay, P, Rs, dq, dk, dv, B, H, N, d, C, st);
}

}  // namespace lasp
