// Forward output on the 5th-generation tensor cores (LASP Eq. 7, 9, 11;
// Algorithm 2 steps 9, 14, 15), for bf16 inputs with d = 128, 64 or 32:
//   O = [(Q K^T) . Mask] V + Lambda Q P,  Mask_ij = lambda^{i-j} (j <= i), Lambda = diag(lambda^{i+1}),
// over a tile of 128 tokens that starts at a chunk boundary; P is the state
// entering the tile (the cached P_c of its first chunk). When C < 128 a tile
// spans 128/C chunks: the masked product over the whole tile is the same sum
// as the per-chunk intra terms plus the inter terms of the chunks inside it
// (LASP Eq. 8 regrouped), so only the first chunk's P is read.
//
// One CTA per (tile, head, batch), 256 threads. In the epilogues warp w reads
// TMEM lanes 32*(w%4).. (the rows it may access) and the column half w/4, so
// the two warpgroups share every epilogue.
//  1. thread 0: TMA loads Q, K, V (128 x 128 bf16, two 64-feature boxes each,
//     128-byte swizzle); all threads: P (fp32, 64 KB) -> bf16 into shared
//     memory as an MN-major operand.
//  2. thread 0: S = Q K^T (TMEM cols 0..127), O_inter = Q P (cols 256..383).
//  3. all: S -> S' = Mask . S in fp32, bf16 into the K tile (K is dead).
//  4. thread 0: O_intra = S' V (cols 128..255).
//  5. all: O = O_intra + lambda^{i+1} O_inter in fp32, bf16 into the Q tile,
//     then one TMA store of the 128 x 128 tile (rows past N are dropped).
// With d = 64 or 32 the tiles keep their 128 features: the second 64-feature
// box of Q, K and V is zero in shared memory instead of loaded (for d = 32 the
// first box's upper 32 features read as zeros: they lie past the tensor's
// feature extent), P fills the top-left d x d block of its tile, the feature
// reductions stop at d and only the first box of the output is stored (its
// columns past d are dropped).
#include "kernels.h"
#include "lasp_common.cuh"
#include "sm100.cuh"
#include "tc_kernels.h"
#include "tma_host.h"

namespace lasp {
namespace tc_out_detail {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr uint32_t kTileBytes = kTile * kD * 2;  // 32 KB: two 16 KB boxes
constexpr uint32_t kBox = kTileBytes / 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColIntra = 128, kColInter = 256;

struct Smem {
  uint64_t load, s_done, o_done;
  uint32_t tmem_base;
  int abort;
  float pw[kTile];  // lambda^n, n = 0..127
};

// Writes 8 consecutive bf16 (16 bytes) of row `row`, starting at column
// `col` (a multiple of 8), into a 128 x 128 tile stored as two 64-column,
// 128-byte-swizzled boxes.


__global__ void __launch_bounds__(kThreads, 1) chunk_out_tc(const __grid_constant__ CUtensorMap map_q,
                                                             const __grid_constant__ CUtensorMap map_k,
                                                             const __grid_constant__ CUtensorMap map_v,
                                                             const __grid_constant__ CUtensorMap map_o,
                                                             const float* decay, const float* __restrict__ P,
                                                             int H, int d, int T, int C) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = base;                    // Q, later the output tile
  uint8_t* sK = base + kTileBytes;       // K, later S'
  uint8_t* sV = base + 2 * kTileBytes;
  uint8_t* sP = base + 3 * kTileBytes;   // P in bf16, MN-major (rows = key feature)
  Smem* s = reinterpret_cast<Smem*>(base + 4 * kTileBytes);

  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = tile * kTile;
  const float lam = load_decay(decay, h);
  const float l2 = log2f(lam);
  const int nbox = d > 64 ? 2 : 1;  // 64-feature boxes loaded per tile

  if (nbox == 1) {
    // the second box of Q, K and V stays zero
    for (int t = 0; t < 3; ++t) {
      uint4* z = reinterpret_cast<uint4*>(base + t * kTileBytes + kBox);
      for (uint32_t q = tid; q < kBox / 16; q += kThreads) z[q] = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
  }
  if (tid == 0) {
    prefetch_tmap(&map_q);
    prefetch_tmap(&map_k);
    prefetch_tmap(&map_v);
    prefetch_tmap(&map_o);
    mbar_init(&s->load, 1);
    mbar_init(&s->s_done, 1);
    mbar_init(&s->o_done, 1);
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

  if (tid == 0) {
    mbar_arrive_expect_tx(&s->load, 3 * nbox * kBox);
    tma_load_4d(sQ, &map_q, &s->load, 0, h, row0, b);
    tma_load_4d(sK, &map_k, &s->load, 0, h, row0, b);
    tma_load_4d(sV, &map_v, &s->load, 0, h, row0, b);
    if (nbox == 2) {
      tma_load_4d(sQ + kBox, &map_q, &s->load, 64, h, row0, b);
      tma_load_4d(sK + kBox, &map_k, &s->load, 64, h, row0, b);
      tma_load_4d(sV + kBox, &map_v, &s->load, 64, h, row0, b);
    }
  }

  // P of the tile's first chunk, fp32 [k][v] -> bf16 operand tile (row k,
  // column v; zero outside d x d)
  {
    const int c0 = row0 / C;
    const float4* Pc = reinterpret_cast<const float4*>(P + ((((int64_t)b * T + c0) * H + h) * d) * d);
    // warp w converts rows w, w + 8, ...: all 16 of its loads are in flight together
    constexpr int kWarps = kThreads / 32, kRows = kD / kWarps;
    const int col = lane * 4;
    {
      float4 x[kRows];
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const int r = warp + kWarps * u;
        x[u] = r < d && col < d ? __ldcs(Pc + r * (d / 4) + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const int r = warp + kWarps * u;
        const uint32_t off = (col >> 6) * kBox + sw128_offset(r, (col & 63) >> 3) + (col & 7) * 2;
        *reinterpret_cast<uint2*>(sP + off) = make_uint2(pack_bf16(x[u].x, x[u].y), pack_bf16(x[u].z, x[u].w));
      }
    }
    fence_async_smem();
  }
  __syncthreads();

  constexpr uint32_t idesc_kk = idesc_bf16(128, 128, 0, 0);  // A K-major, B K-major
  constexpr uint32_t idesc_kn = idesc_bf16(128, 128, 0, 1);  // A K-major, B MN-major
  if (tid == 0) {
    if (mbar_wait(&s->load, 0, SITE_OUT_TMA)) {
      tc_fence_after();
      const uint32_t q0 = smem_u32(sQ), k0 = smem_u32(sK), p0 = smem_u32(sP);
      // S = Q K^T : K index = feature (16 per MMA), both operands K-major
      for (int kk = 0; kk < d / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
        mma_bf16(tmem + kColS, sw128_desc(q0 + off, 16, 1024), sw128_desc(k0 + off, 16, 1024), idesc_kk, kk != 0);
      }
      mma_commit(&s->s_done);
      // O_inter = Q P : K index = key feature; P rows are key features (MN-major B)
      for (int kk = 0; kk < d / 16; ++kk) {
        const uint32_t aoff = (kk >> 2) * kBox + (kk & 3) * 32;
        mma_bf16(tmem + kColInter, sw128_desc(q0 + aoff, 16, 1024), sw128_desc(p0 + kk * 2048, kBox, 1024),
                 idesc_kn, kk != 0);
      }
    } else {
      s->abort = 1;
    }
  }

  // S' = Mask . S, written over the K tile as a K-major A operand; this thread
  // owns row i and the column half `half`
  const int i = (warp & 3) * 32 + lane, half = warp >> 2;
  bool ok = mbar_wait(&s->s_done, 0, SITE_OUT_MMA);
  tc_fence_after();
  if (ok) {
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
#pragma unroll 1
    for (int cc = 2 * half; cc < 2 * half + 2; ++cc) {
      uint32_t r[32];
      tmem_ld32(lane_base + kColS + cc * 32, r);
      tmem_ld_wait();
      float w[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const int j = cc * 32 + q;
        w[q] = j <= i ? __uint_as_float(r[q]) * s->pw[i - j] : 0.f;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        st_tile16(sK, i, cc * 32 + q * 8,
                  make_uint4(pack_bf16(w[8 * q], w[8 * q + 1]), pack_bf16(w[8 * q + 2], w[8 * q + 3]),
                             pack_bf16(w[8 * q + 4], w[8 * q + 5]), pack_bf16(w[8 * q + 6], w[8 * q + 7])));
    }
    fence_async_smem();
  } else {
    s->abort = 1;
  }
  tc_fence_before();
  __syncthreads();

  if (tid == 0 && !s->abort) {
    tc_fence_after();
    const uint32_t a0 = smem_u32(sK), v0 = smem_u32(sV);
    // O_intra = S' V : K index = key token j; V rows are tokens (MN-major B)
    for (int kk = 0; kk < kTile / 16; ++kk) {
      const uint32_t aoff = (kk >> 2) * kBox + (kk & 3) * 32;
      mma_bf16(tmem + kColIntra, sw128_desc(a0 + aoff, 16, 1024), sw128_desc(v0 + kk * 2048, kBox, 1024),
               idesc_kn, kk != 0);
    }
    mma_commit(&s->o_done);  // covers the O_inter MMAs issued earlier too
  }

  ok = !s->abort && mbar_wait(&s->o_done, 0, SITE_OUT_MMA);
  tc_fence_after();
  if (ok) {
    const float wi = decay_pow(l2, (float)(i + 1));
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
#pragma unroll 1
    for (int cc = 2 * half; cc < 2 * half + 2; ++cc) {
      uint32_t a[32], e[32];
      tmem_ld32(lane_base + kColIntra + cc * 32, a);
      tmem_ld32(lane_base + kColInter + cc * 32, e);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float o[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) o[u] = fmaf(wi, __uint_as_float(e[8 * q + u]), __uint_as_float(a[8 * q + u]));
        st_tile16(sQ, i, cc * 32 + q * 8,
                  make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]),
                             pack_bf16(o[6], o[7])));
      }
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && ok) {
    tma_store_4d(&map_o, sQ, 0, h, row0, b);
    if (nbox == 2) tma_store_4d(&map_o, sQ + kBox, 64, h, row0, b);
    tma_store_commit();
    tma_store_wait_read0();
  }
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc_out_detail

bool tc_out_ok(int dtype, int d, int64_t C) {
  return dtype == LASP_BF16 && (d == 32 || d == 64 || d == tc_out_detail::kD) && C <= tc_out_detail::kTile && tc_out_detail::kTile % C == 0 &&
         C % 16 == 0;
}

cudaError_t tc_chunk_out(const void* q, const void* k, const void* v, const float* decay, const float* P, void* o,
                         int B, int H, int64_t N, int d, int C, cudaStream_t st) {
  using namespace tc_out_detail;
  CUtensorMap mq, mk, mv, mo;
  if (!make_token_map(&mq, q, B, H, N, d, kTile) || !make_token_map(&mk, k, B, H, N, d, kTile) ||
      !make_token_map(&mv, v, B, H, N, d, kTile) || !make_token_map(&mo, o, B, H, N, d, kTile))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + 4 * (size_t)kTileBytes + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(chunk_out_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned tiles = (unsigned)((N + kTile - 1) / kTile);
  dim3 grid(tiles, H, B);
  chunk_out_tc<<<grid, kThreads, smem, st>>>(mq, mk, mv, mo, decay, P, H, d, (int)(N / C), C);
  return cudaGetLastError();
}

}  // namespace lasp
