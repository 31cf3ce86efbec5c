// Tensor-core kernels of the gated form (a decay per token and key feature;
// LASP Appendix A.4, Eq. 24 with the GLA / GateLoop row of Table 5), bf16,
// d = 128, one 128-token chunk per CTA. The chunk equations are those of
// k_gla_simt.cu (b_t = inclusive cumulative log-gate from the chunk start,
// b_end its last row).
//
// The intra-chunk products need the factor e^{b_t[i] - b_s[i]} inside a
// contraction over i, which a single MMA can carry only if it splits into a
// row factor and a column factor. With r = b_{63}, the middle row, as the
// reference of each feature:
//   Q^ = q . e^{b - r},  K^ = k . e^{r - b}   (bf16 operands, formed in place)
//   A  = Q^ K^^T         (A_ts = sum_i q_t[i] k_s[i] e^{b_t[i] - b_s[i]})
// and the inter terms take diagonal scalings of the states:
//   o   = (A . causal) V + Q^ P',                 P' = diag(e^{r}) P_c
//   dq  = E . ((dA . strict) K^ + dO P'^T) + (do_t . v_t) k_t,       E = e^{b - r}
//   dk  = E^-1 . ((dA . strict)^T Q^ + V R'^T) + (do_s . v_s) q_s,  R' = diag(e^{b_end - r}) R_c
//   dv  = (A . causal)^T dO + K^ R'
// (dA = dO V^T; "strict" leaves out the diagonal, whose pair is added in
// fp32 so that the log-gate gradient can leave it out, see k_gla_simt.cu.)
// Every factor of Q^ and K^ is at most e^{|b_t - r|}; the form is exact as
// long as that stays inside the bf16 / fp32 range, i.e. the log-gates of each
// half of the chunk sum to at least -kMaxSpan. Each CTA checks this for its
// chunk and records LASP_ERR_INVALID_ARG (site SITE_GATE_RANGE) if not; the
// CUDA-core kernels have no such limit.
//
// Thread layout (256 threads): warp w owns tile rows / TMEM lanes 32*(w%4)..
// and the column half w/4 of every row-wise step. A row's cumulative log-gates
// come from a warp-shuffle scan of the loaded gates down the rows (no gate
// tile in shared memory).
#include "kernels.h"
#include "lasp_common.cuh"
#include "sm100.cuh"
#include "tc_kernels.h"
#include "tma_host.h"

namespace lasp {
namespace tc_gla_detail {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr uint32_t kTileBytes = kTile * kD * 2;
constexpr uint32_t kBox = kTileBytes / 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kMaxSpan = 80.f;  // largest |b_t - r| (natural log) the factorized form takes
constexpr uint32_t kBarAll = 1;   // named barrier over all 256 threads

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t x) {
  return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&x));
}
__device__ __forceinline__ uint4* tile16(uint8_t* tile, int row, int col) {
  return reinterpret_cast<uint4*>(tile + (col >> 6) * kBox + sw128_offset(row, (col & 63) >> 3));
}
__device__ __forceinline__ uint64_t kmaj(uint32_t tile, int kk) {
  return sw128_desc(tile + (kk >> 2) * kBox + (kk & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t mnmaj(uint32_t tile, int kk) { return sw128_desc(tile + kk * 2048, kBox, 1024); }

// Multiplies the 64 bf16 entries of row `row`, columns half*64.., of a tile by
// exp2(sgn * x[u]) (x in log2 units), in place.
__device__ __forceinline__ void scale_row_half(uint8_t* tile, int row, int half, const float (&x)[64], float sgn) {
#pragma unroll
  for (int c8 = 0; c8 < 8; ++c8) {
    uint4* p = tile16(tile, row, half * 64 + c8 * 8);
    uint4 w = *p;
    uint32_t* e = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = unpack_bf16(e[u]);
      e[u] = pack_bf16(f.x * exp2f(sgn * x[c8 * 8 + 2 * u]), f.y * exp2f(sgn * x[c8 * 8 + 2 * u + 1]));
    }
    *p = w;
  }
}

// Inclusive cumulative log-gates (natural log) of row t over the 64 columns of
// `half`: b[u] = sum_{r<=t} g_r[half*64 + u]. g_chunk points at the chunk's
// first token, rows row_stride floats apart. A shuffle scan down the warp's 32
// rows, then the totals of the warps above through `tot` ([8][64] floats).
// All 256 threads call it (it contains a barrier).
__device__ __forceinline__ void row_cumgates(const float* __restrict__ g_chunk, int64_t row_stride, int t, int half,
                                             int warp, int lane, float (&b)[64], float* tot) {
  const float4* gp = reinterpret_cast<const float4*>(g_chunk + (int64_t)t * row_stride + half * 64);
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const float4 x = __ldcs(gp + u);
    b[4 * u] = x.x;
    b[4 * u + 1] = x.y;
    b[4 * u + 2] = x.z;
    b[4 * u + 3] = x.w;
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int u = 0; u < 64; ++u) {
      const float y = __shfl_up_sync(0xffffffffu, b[u], o);
      if (lane >= o) b[u] += y;
    }
  }
  if (lane == 31) {
#pragma unroll
    for (int u = 0; u < 64; ++u) tot[warp * 64 + u] = b[u];
  }
  named_sync(kBarAll, kThreads);
  const int wq = warp & 3;
  for (int w2 = 0; w2 < wq; ++w2) {
#pragma unroll
    for (int u = 0; u < 64; ++u) b[u] += tot[(w2 + 4 * half) * 64 + u];
  }
}

// Publishes row `src_row`'s b (all 128 features) into dst[128] (natural log).
__device__ __forceinline__ void publish_row(int t, int src_row, int half, const float (&b)[64], float* dst) {
  if (t == src_row) {
#pragma unroll
    for (int u = 0; u < 64; ++u) dst[half * 64 + u] = b[u];
  }
}

// fp32 d x d state rows (global) -> bf16 operand tile, row m scaled by
// exp2(scale_log2[m]). Warp w converts rows w, w + 8, ...; lane covers 4 columns.
__device__ __forceinline__ void load_scaled_state(uint8_t* tile, const float* __restrict__ src,
                                                  const float* scale_log2, int warp, int lane) {
  const float4* p = reinterpret_cast<const float4*>(src);
  float4 x[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) x[u] = __ldcs(p + (warp + 8 * u) * (kD / 4) + lane);
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int m = warp + 8 * u;
    const float w = exp2f(scale_log2[m]);
    const int col = lane * 4;
    const uint32_t off = (col >> 6) * kBox + sw128_offset(m, (col & 63) >> 3) + (col & 7) * 2;
    *reinterpret_cast<uint2*>(tile + off) = make_uint2(pack_bf16(x[u].x * w, x[u].y * w), pack_bf16(x[u].z * w, x[u].w * w));
  }
}

// ---------------------------------------------------------------- states
struct SmemStates {
  uint64_t load, mma;
  uint32_t tmem_base;
  int abort;
  float tot[8 * 64];
  float bend[kD];
};

// kind 0: M_c = (k . e^{b_end - b})^T v, gsum_c = b_end; kind 1: dM_c = (q . e^{b})^T do.
// x, y: the two token operands ((k, v) or (q, do)); the gate factor goes on x.
__global__ void __launch_bounds__(kThreads, 2) gla_states_tc(const __grid_constant__ CUtensorMap map_x,
                                                             const __grid_constant__ CUtensorMap map_y,
                                                             const float* __restrict__ g, float* __restrict__ M,
                                                             float* __restrict__ gsum, int H, int64_t N, int kind) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sX = base;
  uint8_t* sY = base + kTileBytes;
  SmemStates* s = reinterpret_cast<SmemStates*>(base + 2 * kTileBytes);
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = (warp & 3) * 32 + lane, half = warp >> 2;
  const int64_t row0 = (int64_t)c * kTile;
  const int64_t T = N / kTile;
  if (tid == 0) {
    prefetch_tmap(&map_x);
    prefetch_tmap(&map_y);
    mbar_init(&s->load, 1);
    mbar_init(&s->mma, 1);
    s->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s->tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s->tmem_base;
  if (tid == 0) {
    mbar_arrive_expect_tx(&s->load, 2 * kTileBytes);
    tma_load_4d(sX, &map_x, &s->load, 0, h, (int)row0, b);
    tma_load_4d(sX + kBox, &map_x, &s->load, 64, h, (int)row0, b);
    tma_load_4d(sY, &map_y, &s->load, 0, h, (int)row0, b);
    tma_load_4d(sY + kBox, &map_y, &s->load, 64, h, (int)row0, b);
  }
  float bl[64];
  row_cumgates(g + ((int64_t)b * N + row0) * H * kD + (int64_t)h * kD, (int64_t)H * kD, t, half, warp, lane, bl,
               s->tot);
  publish_row(t, kTile - 1, half, bl, s->bend);
  named_sync(kBarAll, kThreads);
  // the gate factor of row t: e^{b_end - b_t} (kind 0) or e^{b_t} (kind 1), in log2 units
#pragma unroll
  for (int u = 0; u < 64; ++u) bl[u] = (kind == 0 ? s->bend[half * 64 + u] - bl[u] : bl[u]) * kLog2e;
  if (!mbar_wait(&s->load, 0, SITE_STATES_TMA)) s->abort = 1;
  scale_row_half(sX, t, half, bl, 1.f);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (s->abort) goto cleanup;
  if (tid == 0) {
    tc_fence_after();
    constexpr uint32_t id_nn = idesc_bf16(128, 128, 1, 1);
    const uint32_t aX = smem_u32(sX), aY = smem_u32(sY);
    for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem, mnmaj(aX, kk), mnmaj(aY, kk), id_nn, kk != 0);
    mma_commit(&s->mma);
  }
  if (kind == 0 && gsum != nullptr && tid < kD) gsum[((b * T + c) * H + h) * kD + tid] = s->bend[tid];
  if (mbar_wait(&s->mma, 0, SITE_STATES_MMA)) {
    tc_fence_after();
    // row i of M (TMEM lane i), columns half*64..
    const int i = t;
    float* out = M + (((b * T + c) * H + h) * kD + i) * kD + half * 64;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
      uint32_t r[32];
      tmem_ld32(lane_base + half * 64 + c2 * 32, r);
      tmem_ld_wait();
#pragma unroll
      for (int u = 0; u < 8; ++u)
        __stcs(reinterpret_cast<float4*>(out + c2 * 32) + u,
               make_float4(__uint_as_float(r[4 * u]), __uint_as_float(r[4 * u + 1]), __uint_as_float(r[4 * u + 2]),
                           __uint_as_float(r[4 * u + 3])));
    }
  } else {
    s->abort = 1;
  }
cleanup:
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

// ---------------------------------------------------------------- output
struct SmemOut {
  uint64_t load, mma1, mma2;
  uint32_t tmem_base;
  int abort;
  float tot[8 * 64];
  float r[kD];       // b at the middle row (natural log)
  float rl2[kD];     // the same, times log2 e
};

__global__ void __launch_bounds__(kThreads, 1) gla_out_tc(const __grid_constant__ CUtensorMap map_q,
                                                          const __grid_constant__ CUtensorMap map_k,
                                                          const __grid_constant__ CUtensorMap map_v,
                                                          const __grid_constant__ CUtensorMap map_o,
                                                          const float* __restrict__ g, const float* __restrict__ P,
                                                          int H, int64_t N) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = base;                   // Q^
  uint8_t* sK = base + 1 * kTileBytes;  // K^
  uint8_t* sV = base + 2 * kTileBytes;
  uint8_t* sX = base + 3 * kTileBytes;  // P'
  uint8_t* sA = base + 4 * kTileBytes;  // A . causal, then O out
  SmemOut* s = reinterpret_cast<SmemOut*>(base + 5 * kTileBytes);
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = (warp & 3) * 32 + lane, half = warp >> 2;
  const int64_t row0 = (int64_t)c * kTile;
  const int64_t T = N / kTile;
  if (tid == 0) {
    prefetch_tmap(&map_q);
    prefetch_tmap(&map_k);
    prefetch_tmap(&map_v);
    prefetch_tmap(&map_o);
    mbar_init(&s->load, 1);
    mbar_init(&s->mma1, 1);
    mbar_init(&s->mma2, 1);
    s->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s->tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s->tmem_base;
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  const uint32_t T0 = 0, T1 = 128;
  if (tid == 0) {
    mbar_arrive_expect_tx(&s->load, 3 * kTileBytes);
    tma_load_4d(sQ, &map_q, &s->load, 0, h, (int)row0, b);
    tma_load_4d(sQ + kBox, &map_q, &s->load, 64, h, (int)row0, b);
    tma_load_4d(sK, &map_k, &s->load, 0, h, (int)row0, b);
    tma_load_4d(sK + kBox, &map_k, &s->load, 64, h, (int)row0, b);
    tma_load_4d(sV, &map_v, &s->load, 0, h, (int)row0, b);
    tma_load_4d(sV + kBox, &map_v, &s->load, 64, h, (int)row0, b);
  }
  float bl[64];
  row_cumgates(g + ((int64_t)b * N + row0) * H * kD + (int64_t)h * kD, (int64_t)H * kD, t, half, warp, lane, bl,
               s->tot);
  publish_row(t, kTile / 2 - 1, half, bl, s->r);
  named_sync(kBarAll, kThreads);
  {
    bool ok = true;
#pragma unroll
    for (int u = 0; u < 64; ++u) {
      const float x = bl[u] - s->r[half * 64 + u];
      ok = ok && fabsf(x) <= kMaxSpan;
      bl[u] = x * kLog2e;  // log2 E
    }
    if (!ok) record_error(LASP_ERR_INVALID_ARG, SITE_GATE_RANGE);
  }
  if (tid < kD) s->rl2[tid] = s->r[tid] * kLog2e;
  named_sync(kBarAll, kThreads);
  // P' = diag(e^{r}) P_c into X (the global loads overlap the TMA loads)
  load_scaled_state(sX, P + ((b * T + c) * H + h) * (int64_t)kD * kD, s->rl2, warp, lane);
  if (!mbar_wait(&s->load, 0, SITE_OUT_TMA)) s->abort = 1;
  scale_row_half(sQ, t, half, bl, 1.f);   // Q^ = q . E
  scale_row_half(sK, t, half, bl, -1.f);  // K^ = k / E
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (s->abort) goto cleanup;
  {
    const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aX = smem_u32(sX), aA = smem_u32(sA);
    constexpr uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t id_kn = idesc_bf16(128, 128, 0, 1);
    if (tid == 0) {
      tc_fence_after();
      for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T0, kmaj(aQ, kk), kmaj(aK, kk), id_kk, kk != 0);
      mma_commit(&s->mma1);
      // the inter term does not wait for the mask
      for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T1, kmaj(aQ, kk), mnmaj(aX, kk), id_kn, kk != 0);
    }
    // A . causal -> sA (row t, column half)
    if (mbar_wait(&s->mma1, 0, SITE_OUT_MMA)) {
      tc_fence_after();
#pragma unroll 1
      for (int c2 = 0; c2 < 2; ++c2) {
        const int col0 = half * 64 + c2 * 32;
        uint32_t r[32];
        tmem_ld32(lane_base + T0 + col0, r);
        tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          float f[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) f[u] = col0 + q4 * 8 + u <= t ? __uint_as_float(r[q4 * 8 + u]) : 0.f;
          *tile16(sA, t, col0 + q4 * 8) = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]),
                                                     pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
        }
      }
    } else {
      s->abort = 1;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (s->abort) goto cleanup;
    if (tid == 0) {
      tc_fence_after();
      for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + T1, kmaj(aA, kk), mnmaj(aV, kk), id_kn, 1);
      mma_commit(&s->mma2);
    }
    // O -> sA (free once the MMA has read it) -> TMA store
    if (mbar_wait(&s->mma2, 0, SITE_OUT_MMA)) {
      tc_fence_after();
#pragma unroll 1
      for (int c2 = 0; c2 < 2; ++c2) {
        const int col0 = half * 64 + c2 * 32;
        uint32_t r[32];
        tmem_ld32(lane_base + T1 + col0, r);
        tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          *tile16(sA, t, col0 + q4 * 8) =
              make_uint4(pack_bf16(__uint_as_float(r[q4 * 8]), __uint_as_float(r[q4 * 8 + 1])),
                         pack_bf16(__uint_as_float(r[q4 * 8 + 2]), __uint_as_float(r[q4 * 8 + 3])),
                         pack_bf16(__uint_as_float(r[q4 * 8 + 4]), __uint_as_float(r[q4 * 8 + 5])),
                         pack_bf16(__uint_as_float(r[q4 * 8 + 6]), __uint_as_float(r[q4 * 8 + 7])));
      }
      fence_async_smem();
    } else {
      s->abort = 1;
    }
    __syncthreads();
    if (tid == 0 && !s->abort) {
      tma_store_4d(&map_o, sA, 0, h, (int)row0, b);
      tma_store_4d(&map_o, sA + kBox, 64, h, (int)row0, b);
      tma_store_commit();
      tma_store_wait_read0();
    }
  }
cleanup:
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace tc_gla_detail

bool tc_gla_ok(int dtype, int d, int64_t C) {
  return dtype == LASP_BF16 && d == tc_gla_detail::kD && C == tc_gla_detail::kTile;
}

cudaError_t tc_gla_chunk_states(const void* x, const void* y, const float* g, float* M, float* gsum, int B, int H,
                                int64_t N, int kind, cudaStream_t st) {
  using namespace tc_gla_detail;
  CUtensorMap mx, my;
  if (!make_token_map(&mx, x, B, H, N, kD, kTile) || !make_token_map(&my, y, B, H, N, kD, kTile))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + 2 * (size_t)kTileBytes + sizeof(SmemStates);
  cudaError_t e = cudaFuncSetAttribute(gla_states_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  gla_states_tc<<<dim3((unsigned)(N / kTile), H, B), kThreads, smem, st>>>(mx, my, g, M, gsum, H, N, kind);
  return cudaGetLastError();
}

cudaError_t tc_gla_chunk_out(const void* q, const void* k, const void* v, const float* g, const float* P, void* o,
                             int B, int H, int64_t N, cudaStream_t st) {
  using namespace tc_gla_detail;
  CUtensorMap mq, mk, mv, mo;
  if (!make_token_map(&mq, q, B, H, N, kD, kTile) || !make_token_map(&mk, k, B, H, N, kD, kTile) ||
      !make_token_map(&mv, v, B, H, N, kD, kTile) || !make_token_map(&mo, o, B, H, N, kD, kTile))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + 5 * (size_t)kTileBytes + sizeof(SmemOut);
  cudaError_t e = cudaFuncSetAttribute(gla_out_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  gla_out_tc<<<dim3((unsigned)(N / kTile), H, B), kThreads, smem, st>>>(mq, mk, mv, mo, g, P, H, N);
  return cudaGetLastError();
}

}  // namespace lasp
