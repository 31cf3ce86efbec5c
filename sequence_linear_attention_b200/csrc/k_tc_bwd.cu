// Backward pass of one 128-token tile on the 5th-generation tensor cores
// (LASP Eq. 14, 16, 17, 19, 22, 23; Algorithm 3 steps 7-17), bf16, d = 128, 64 or 32:
//   dP = (dO V^T) . Mask,  S = (Q K^T) . Mask,   Mask_ij = lambda^{i-j} (j <= i)
//   dQ = dP K   + diag(lambda^{i+1})    dO P^T
//   dK = dP^T Q + diag(lambda^{e-j})    V  R^T
//   dV = S^T dO + diag(lambda^{e-j})    K  R
// where P is the state entering the tile (cached P of its first chunk), R the
// gradient state entering it from the right (R of its last chunk) and e the
// tile's last row. A tile spans 128/C chunks when C < 128; the masked products
// over the whole tile regroup the per-chunk intra and inter terms (LASP Eq. 8,
// 15, 18, 21).
//
// One CTA per (tile, head, batch), 256 threads; in every epilogue warp w owns
// the TMEM lanes (rows) 32*(w%4).. and the column half w/4. Shared memory holds
// seven 32 KB bf16 tiles: Q, K, V, dO (TMA, 128-byte swizzle), X (P, later R,
// converted from fp32), dP' and S'. R arrives at the start by one bulk copy
// into the dP'/S' space (64 KB of fp32, idle until epilogue 1) and moves to
// registers before epilogue 1, so no global load waits in mid-kernel. Each
// stored tile serves both as a K-major and as an MN-major operand, so no
// transposed copy is made: dP' [i][j] is the K-major A of dP' K and the
// MN-major A of dP'^T Q, and so on. The 512 TMEM columns hold four 128-column
// fp32 accumulators, reused across three MMA phases:
//   phase 1:  T0 = dO V^T, T1 = Q K^T, T2 = dO P^T          -> epilogue 1 (masks)
//   phase 2:  T3 = dP' K                                     -> epilogue 2 (dQ)
//   phase 3:  T0 = dP'^T Q, T1 = S'^T dO, T2 = V R^T, T3 = K R -> epilogue 3 (dK, dV)
// The decay factors of the inter terms are applied in fp32 in the epilogues.
// With d = 64 or 32 the tiles keep their 128 features: the second 64-feature
// box of Q, K, V and dO is zero in shared memory instead of loaded (for d = 32
// the first box's upper 32 features read as zeros: they lie past the tensor's
// feature extent), P and R fill the top-left d x d block of X, the feature
// reductions stop at d and only the first d columns of dQ, dK and dV are
// stored.
#include "kernels.h"
#include "lasp_common.cuh"
#include "sm100.cuh"
#include "tc_kernels.h"
#include "tma_host.h"

namespace lasp {
namespace tc_bwd_detail {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerWarp = 128 / kWarps;
constexpr uint32_t kTileBytes = kTile * kD * 2;
constexpr uint32_t kBox = kTileBytes / 2;
constexpr uint32_t kTmemCols = 512;

struct Smem {
  uint64_t load, rload, mma1a, mma1b, mma2, mma3;
  uint32_t tmem_base;
  int abort;
  float pw[kTile];
};



// Row r of a d x d fp32 state [m][e], float4 `lane` (columns 4*lane..4*lane+3),
// written as bf16 into the operand tile (row m, column e).
__device__ __forceinline__ void put_state_row(uint8_t* tile, int r, int lane, float4 x) {
  const int col = lane * 4;
  const uint32_t off = (col >> 6) * kBox + sw128_offset(r, (col & 63) >> 3) + (col & 7) * 2;
  *reinterpret_cast<uint2*>(tile + off) = make_uint2(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w));
}

// fp32 d x d state in global memory -> bf16 tile (zero outside d x d). Warp w
// converts rows w, w + 8, ...; all of its loads are in flight together.
__device__ __forceinline__ void load_state_tile(uint8_t* tile, const float* src, int d, int warp, int lane) {
  const float4* p = reinterpret_cast<const float4*>(src);
  float4 x[kRowsPerWarp];
#pragma unroll
  for (int u = 0; u < kRowsPerWarp; ++u) {
    const int r = warp + kWarps * u;
    x[u] = r < d && 4 * lane < d ? __ldcs(p + r * (d / 4) + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int u = 0; u < kRowsPerWarp; ++u) put_state_row(tile, warp + kWarps * u, lane, x[u]);
}


__global__ void __launch_bounds__(kThreads, 1) chunk_bwd_tc(const __grid_constant__ CUtensorMap map_q,
                                                             const __grid_constant__ CUtensorMap map_k,
                                                             const __grid_constant__ CUtensorMap map_v,
                                                             const __grid_constant__ CUtensorMap map_do,
                                                             const __grid_constant__ CUtensorMap map_dk,
                                                             const __grid_constant__ CUtensorMap map_dv,
                                                             const float* decay, const float* __restrict__ P,
                                                             const float* __restrict__ R,
                                                             __nv_bfloat16* __restrict__ dq, int H, int d,
                                                             int64_t N, int T, int C) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = base;
  uint8_t* sK = base + 1 * kTileBytes;
  uint8_t* sV = base + 2 * kTileBytes;
  uint8_t* sD = base + 3 * kTileBytes;
  uint8_t* sX = base + 4 * kTileBytes;  // P, then R
  uint8_t* sA = base + 5 * kTileBytes;  // dP', later dK out
  uint8_t* sB = base + 6 * kTileBytes;  // S',  later dV out
  Smem* s = reinterpret_cast<Smem*>(base + 7 * kTileBytes);

  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = tile * kTile;
  const int last = (int)min((int64_t)kTile, N - row0) - 1;  // last valid row of the tile
  const float lam = load_decay(decay, h);
  const float l2 = log2f(lam);
  const int nbox = d > 64 ? 2 : 1;  // 64-feature boxes loaded per tile

  if (nbox == 1) {
    // the second box of Q, K, V and dO stays zero
    for (int t = 0; t < 4; ++t) {
      uint4* z = reinterpret_cast<uint4*>(base + t * kTileBytes + kBox);
      for (uint32_t q = tid; q < kBox / 16; q += kThreads) z[q] = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
  }
  if (tid == 0) {
    prefetch_tmap(&map_q);
    prefetch_tmap(&map_k);
    prefetch_tmap(&map_v);
    prefetch_tmap(&map_do);
    mbar_init(&s->load, 1);
    mbar_init(&s->rload, 1);
    mbar_init(&s->mma1a, 1);
    mbar_init(&s->mma1b, 1);
    mbar_init(&s->mma2, 1);
    mbar_init(&s->mma3, 1);
    s->abort = 0;
    fence_mbar_init();
  }
  if (tid < kTile) s->pw[tid] = decay_pow(l2, (float)tid);
  if (warp == 0) {
    tmem_alloc(&s->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s->tmem_base;
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  const int half = warp >> 2;  // column half of every epilogue
  const uint32_t T0 = 0, T1 = 128, T2 = 256, T3 = 384;

  if (tid == 0) {
    mbar_arrive_expect_tx(&s->load, 4 * nbox * kBox);
    tma_load_4d(sQ, &map_q, &s->load, 0, h, row0, b);
    tma_load_4d(sK, &map_k, &s->load, 0, h, row0, b);
    tma_load_4d(sV, &map_v, &s->load, 0, h, row0, b);
    tma_load_4d(sD, &map_do, &s->load, 0, h, row0, b);
    if (nbox == 2) {
      tma_load_4d(sQ + kBox, &map_q, &s->load, 64, h, row0, b);
      tma_load_4d(sK + kBox, &map_k, &s->load, 64, h, row0, b);
      tma_load_4d(sV + kBox, &map_v, &s->load, 64, h, row0, b);
      tma_load_4d(sD + kBox, &map_do, &s->load, 64, h, row0, b);
    }
  }
  const int c_first = row0 / C, c_last = (row0 + last) / C;
  if (tid == 32) {
    // R of the tile's last chunk, fp32 [d][d], into the (still unused) dP'/S'
    // space, in copies of at most 16 KB
    const float* Rc = R + ((((int64_t)b * T + c_last) * H + h) * d) * d;
    const uint32_t rbytes = d * d * 4, pb = rbytes < 16384 ? rbytes : 16384;
    mbar_arrive_expect_tx(&s->rload, rbytes);
    for (uint32_t part = 0; part < rbytes / pb; ++part)
      bulk_load(sA + part * pb, Rc + part * (pb / 4), pb, &s->rload);
  }
  load_state_tile(sX, P + ((((int64_t)b * T + c_first) * H + h) * d) * d, d, warp, lane);
  fence_async_smem();
  __syncthreads();

  constexpr uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t id_kn = idesc_bf16(128, 128, 0, 1);
  constexpr uint32_t id_nn = idesc_bf16(128, 128, 1, 1);
  const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aD = smem_u32(sD);
  const uint32_t aX = smem_u32(sX), aA = smem_u32(sA), aB = smem_u32(sB);

  // ---- phase 1: dP = dO V^T, S = Q K^T, dQ_inter = dO P^T
  if (tid == 0) {
    if (mbar_wait(&s->load, 0, SITE_BWD_TMA)) {
      tc_fence_after();
      for (int kk = 0; kk < d / 16; ++kk) mma_bf16(tmem + T0, kmaj(aD, kk), kmaj(aV, kk), id_kk, kk != 0);
      for (int kk = 0; kk < d / 16; ++kk) mma_bf16(tmem + T1, kmaj(aQ, kk), kmaj(aK, kk), id_kk, kk != 0);
      mma_commit(&s->mma1a);
      for (int kk = 0; kk < d / 16; ++kk) mma_bf16(tmem + T2, kmaj(aD, kk), kmaj(aX, kk), id_kk, kk != 0);
      mma_commit(&s->mma1b);
    } else {
      s->abort = 1;
    }
  }

  // ---- R (fp32, in the dP'/S' space) -> registers; that space is then free
  float4 rreg[kRowsPerWarp];
  if (mbar_wait(&s->rload, 0, SITE_BWD_TMA)) {
    const float4* rs4 = reinterpret_cast<const float4*>(sA);
#pragma unroll
    for (int u = 0; u < kRowsPerWarp; ++u) {
      const int r = warp + kWarps * u;
      rreg[u] = r < d && 4 * lane < d ? rs4[r * (d / 4) + lane] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else {
    s->abort = 1;
  }
  __syncthreads();

  // ---- epilogue 1: masks, dP' -> sA, S' -> sB (row i, column half `half`)
  const int i = (warp & 3) * 32 + lane;
  if (mbar_wait(&s->mma1a, 0, SITE_BWD_MMA)) {
    tc_fence_after();
#pragma unroll 1
    for (int cc = 2 * half; cc < 2 * half + 2; ++cc) {
      uint32_t rp[32], rs[32];
      tmem_ld32(lane_base + T0 + cc * 32, rp);
      tmem_ld32(lane_base + T1 + cc * 32, rs);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float fp[8], fs[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = cc * 32 + q * 8 + u;
          const float w = j <= i ? s->pw[i - j] : 0.f;
          fp[u] = __uint_as_float(rp[q * 8 + u]) * w;
          fs[u] = __uint_as_float(rs[q * 8 + u]) * w;
        }
        st_tile16(sA, i, cc * 32 + q * 8,
                  make_uint4(pack_bf16(fp[0], fp[1]), pack_bf16(fp[2], fp[3]), pack_bf16(fp[4], fp[5]),
                             pack_bf16(fp[6], fp[7])));
        st_tile16(sB, i, cc * 32 + q * 8,
                  make_uint4(pack_bf16(fs[0], fs[1]), pack_bf16(fs[2], fs[3]), pack_bf16(fs[4], fs[5]),
                             pack_bf16(fs[6], fs[7])));
      }
    }
  } else {
    s->abort = 1;
  }
  // X is free once dQ_inter has read P: R (bf16) replaces it
  if (mbar_wait(&s->mma1b, 0, SITE_BWD_MMA)) {
#pragma unroll
    for (int u = 0; u < kRowsPerWarp; ++u) put_state_row(sX, warp + kWarps * u, lane, rreg[u]);
  } else {
    s->abort = 1;
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (s->abort) goto cleanup;

  // ---- phase 2: dQ_intra = dP' K   (A = dP' K-major over j, B = K MN-major: rows j)
  if (tid == 0) {
    tc_fence_after();
    for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + T3, kmaj(aA, kk), mnmaj(aK, kk), id_kn, kk != 0);
    mma_commit(&s->mma2);
  }
  // ---- epilogue 2: dQ = T3 + lambda^{i+1} T2, stored straight to global
  if (!s->abort && mbar_wait(&s->mma2, 0, SITE_BWD_MMA)) {
    tc_fence_after();
    const float wi = decay_pow(l2, (float)(i + 1));
    const bool valid = i <= last;
    __nv_bfloat16* out = dq + (((int64_t)b * N + row0 + i) * H + h) * d;
#pragma unroll 1
    for (int cc = 2 * half; cc < 2 * half + 2 && cc * 32 < d; ++cc) {
      uint32_t ra[32], re[32];
      tmem_ld32(lane_base + T3 + cc * 32, ra);
      tmem_ld32(lane_base + T2 + cc * 32, re);
      tmem_ld_wait();
      if (valid) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float o[8];
#pragma unroll
          for (int u = 0; u < 8; ++u)
            o[u] = fmaf(wi, __uint_as_float(re[q * 8 + u]), __uint_as_float(ra[q * 8 + u]));
          *reinterpret_cast<uint4*>(out + cc * 32 + q * 8) =
              make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]), pack_bf16(o[6], o[7]));
        }
      }
    }
  } else {
    s->abort = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (s->abort) goto cleanup;

  // ---- phase 3: dK = dP'^T Q + ., dV = S'^T dO + ., inter terms V R^T and K R
  if (tid == 0) {
    tc_fence_after();
    for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + T0, mnmaj(aA, kk), mnmaj(aQ, kk), id_nn, kk != 0);
    for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + T1, mnmaj(aB, kk), mnmaj(aD, kk), id_nn, kk != 0);
    for (int kk = 0; kk < d / 16; ++kk) mma_bf16(tmem + T2, kmaj(aV, kk), kmaj(aX, kk), id_kk, kk != 0);
    for (int kk = 0; kk < d / 16; ++kk) mma_bf16(tmem + T3, kmaj(aK, kk), mnmaj(aX, kk), id_kn, kk != 0);
    mma_commit(&s->mma3);
  }

  // ---- epilogue 3: row j, column half `half`; dK -> sA, dV -> sB, then TMA stores
  if (mbar_wait(&s->mma3, 0, SITE_BWD_MMA)) {
    tc_fence_after();
    const int j = i;
    const float wj = j <= last ? decay_pow(l2, (float)(last - j)) : 0.f;
#pragma unroll 1
    for (int cc = 2 * half; cc < 2 * half + 2; ++cc) {
      uint32_t ka[32], ke[32];
      tmem_ld32(lane_base + T0 + cc * 32, ka);
      tmem_ld32(lane_base + T2 + cc * 32, ke);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float o[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) o[u] = fmaf(wj, __uint_as_float(ke[q * 8 + u]), __uint_as_float(ka[q * 8 + u]));
        st_tile16(sA, j, cc * 32 + q * 8,
                  make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]), pack_bf16(o[6], o[7])));
      }
      tmem_ld32(lane_base + T1 + cc * 32, ka);
      tmem_ld32(lane_base + T3 + cc * 32, ke);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float o[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) o[u] = fmaf(wj, __uint_as_float(ke[q * 8 + u]), __uint_as_float(ka[q * 8 + u]));
        st_tile16(sB, j, cc * 32 + q * 8,
                  make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]), pack_bf16(o[6], o[7])));
      }
    }
    fence_async_smem();
  } else {
    s->abort = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && !s->abort) {
    tma_store_4d(&map_dk, sA, 0, h, row0, b);
    tma_store_4d(&map_dv, sB, 0, h, row0, b);
    if (nbox == 2) {
      tma_store_4d(&map_dk, sA + kBox, 64, h, row0, b);
      tma_store_4d(&map_dv, sB + kBox, 64, h, row0, b);
    }
    tma_store_commit();
    tma_store_wait_read0();
  }

cleanup:
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc_bwd_detail

bool tc_bwd_ok(int dtype, int d, int64_t C) {
  return dtype == LASP_BF16 && (d == 32 || d == 64 || d == tc_bwd_detail::kD) && C <= tc_bwd_detail::kTile && tc_bwd_detail::kTile % C == 0 &&
         C % 16 == 0;
}

cudaError_t tc_chunk_bwd(const void* q, const void* k, const void* v, const void* dout, const float* decay,
                         const float* P, const float* Rs, void* dq, void* dk, void* dv, int B, int H, int64_t N, int d,
                         int C, cudaStream_t st) {
  using namespace tc_bwd_detail;
  CUtensorMap mq, mk, mv, mdo, mdk, mdv;
  if (!make_token_map(&mq, q, B, H, N, d, kTile) || !make_token_map(&mk, k, B, H, N, d, kTile) ||
      !make_token_map(&mv, v, B, H, N, d, kTile) || !make_token_map(&mdo, dout, B, H, N, d, kTile) ||
      !make_token_map(&mdk, dk, B, H, N, d, kTile) || !make_token_map(&mdv, dv, B, H, N, d, kTile))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + 7 * (size_t)kTileBytes + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(chunk_bwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned tiles = (unsigned)((N + kTile - 1) / kTile);
  dim3 grid(tiles, H, B);
  chunk_bwd_tc<<<grid, kThreads, smem, st>>>(mq, mk, mv, mdo, mdk, mdv, decay, P, Rs, (__nv_bfloat16*)dq, H, d, N,
                                             (int)(N / C), C);
  return cudaGetLastError();
}

}  // namespace lasp
