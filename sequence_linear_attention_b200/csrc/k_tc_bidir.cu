// Bidirectional (unmasked) linear attention on one GPU: LASP Eq. 3 as the
// right product O = Q (K^T V) without Norm, which the LASP-2 review page
// ("Summary") describes as the unmasked variant: every chunk's state M_t is
// gathered, M_{1:T} = sum_t M_t, and each chunk computes Q_t M_{1:T}; the
// backward pass does the same with dM = sum_t Q_t^T dO_t, then
//   dQ = dO M^T,   dK = V dM^T,   dV = K dM.
// bf16, d = 128, N a multiple of 128.
//
// Three kernels: the segment-state kernel (k_tc_states.cu, lambda = 1) writes
// one d x d state per segment; bidir_total sums a (b, h)'s segment states in
// a fixed order into the fp32 total and its bf16 operand tile; bidir_apply_tc
// streams 128-token tiles X of one token tensor through Y = X S with S the
// total's tile (used as S or as S^T), one tcgen05.mma group per tile.
#include <algorithm>

#include "kernels.h"
#include "lasp_common.cuh"
#include "sm100.cuh"
#include "tc_kernels.h"
#include "tma_host.h"

namespace lasp {
namespace tc_bidir_detail {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTile = 128;
constexpr uint32_t kTileBytes = kTile * kD * 2;  // 32 KB: two 64-feature boxes
constexpr uint32_t kBox = kTileBytes / 2;

// ------------------------------------------------------------------ totals
// total = sum over the nseg segment states of (b, h), written as fp32 and as
// the bf16 operand tile (two 64-column boxes of 128 rows, 128-byte swizzled:
// element (r, c) sits in box c / 64, row r, 16-byte chunk ((c % 64) / 8) ^
// (r % 8)). A block takes 32 float4s of the state; its four warps sum a
// quarter of the segments each (eight loads in flight per thread), and the
// four partial sums are added in a fixed order, so the result does not depend
// on timing.
constexpr int kTotalThreads = 128;
constexpr int kTotalCols = 32;  // float4s of the state per block

__global__ void __launch_bounds__(kTotalThreads) bidir_total(const float4* __restrict__ seg, float4* __restrict__ total,
                                                            uint8_t* __restrict__ tiles, int H, int nseg) {
  __shared__ float4 part[kTotalThreads / kTotalCols][kTotalCols];
  const int bh = blockIdx.y;  // b * H + h
  const int b = bh / H, h = bh % H;
  const int col = threadIdx.x % kTotalCols, grp = threadIdx.x / kTotalCols;
  const int e4 = blockIdx.x * kTotalCols + col;  // float4 index in the state
  constexpr int kPer = kD * kD / 4;
  constexpr int kGroups = kTotalThreads / kTotalCols;
  const int64_t step = (int64_t)H * kPer;  // float4s from one segment slot to the next
  const float4* p = seg + ((int64_t)b * nseg * H + h) * kPer + e4;
  const int per = (nseg + kGroups - 1) / kGroups;
  const int g0 = grp * per, g1 = g0 + per < nseg ? g0 + per : nseg;
  float4 a[8] = {};
  int g = g0;
  for (; g + 8 <= g1; g += 8) {
    float4 x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = __ldcs(p + (g + u) * step);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      a[u].x += x[u].x;
      a[u].y += x[u].y;
      a[u].z += x[u].z;
      a[u].w += x[u].w;
    }
  }
  for (; g < g1; ++g) {
    const float4 x = __ldcs(p + g * step);
    a[0].x += x.x;
    a[0].y += x.y;
    a[0].z += x.z;
    a[0].w += x.w;
  }
  float4 s;
  s.x = ((a[0].x + a[1].x) + (a[2].x + a[3].x)) + ((a[4].x + a[5].x) + (a[6].x + a[7].x));
  s.y = ((a[0].y + a[1].y) + (a[2].y + a[3].y)) + ((a[4].y + a[5].y) + (a[6].y + a[7].y));
  s.z = ((a[0].z + a[1].z) + (a[2].z + a[3].z)) + ((a[4].z + a[5].z) + (a[6].z + a[7].z));
  s.w = ((a[0].w + a[1].w) + (a[2].w + a[3].w)) + ((a[4].w + a[5].w) + (a[6].w + a[7].w));
  part[grp][col] = s;
  __syncthreads();
  if (grp != 0) return;
#pragma unroll
  for (int q = 1; q < kGroups; ++q) {
    s.x += part[q][col].x;
    s.y += part[q][col].y;
    s.z += part[q][col].z;
    s.w += part[q][col].w;
  }
  total[(int64_t)bh * kPer + e4] = s;
  const int r = (e4 * 4) / kD, c = (e4 * 4) % kD;
  const int cb = c & 63;
  uint8_t* t = tiles + (int64_t)bh * kTileBytes + (c >> 6) * kBox + r * 128 + ((((cb >> 3) ^ (r & 7))) << 4) +
               (cb & 7) * 2;
  __nv_bfloat162 lo = __floats2bfloat162_rn(s.x, s.y), hi = __floats2bfloat162_rn(s.z, s.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(t) = u;
}

// ------------------------------------------------------------------- apply
// warp 0: TMA (token tiles into a ring of three slots, the (b, h)'s state tile
// into one of two buffers), warp 1: MMA (two TMEM accumulators), warps 2-9:
// epilogue (TMEM -> bf16 -> one of two staging tiles -> TMA store).
constexpr int kThreads = 320;
constexpr int kEpiThreads = 256;
constexpr int kSlots = 3;
constexpr uint32_t kEpiBar = 1;
constexpr uint32_t kTmemCols = 256;

struct Smem {
  uint64_t full[kSlots], empty[kSlots];
  uint64_t s_full[2], s_empty[2];
  uint64_t acc_full[2], acc_empty[2];
  uint32_t tmem_base;
  int abort;
};


// Y[b, tile rows, h, :] = X[b, tile rows, h, :] S_bh, S_bh the bf16 operand
// tile of (b, h) used as stored (b_kmajor = 0: Y = X S) or transposed
// (b_kmajor = 1: Y = X S^T). CTA c takes the tiles c*R .. c*R + R - 1 of the
// (b, h, tile) order, so its state tile changes at most a few times.
__global__ void __launch_bounds__(kThreads, 1) bidir_apply_tc(const __grid_constant__ CUtensorMap map_x,
                                                             const __grid_constant__ CUtensorMap map_y,
                                                             const uint8_t* __restrict__ stiles, int H, int ntiles,
                                                             int64_t nitems, int64_t per_cta, int b_kmajor) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* xs = base;                                // kSlots token tiles
  uint8_t* ss = base + kSlots * kTileBytes;          // two state tiles
  uint8_t* ys = base + (kSlots + 2) * kTileBytes;    // two staging tiles
  Smem* s = reinterpret_cast<Smem*>(base + (kSlots + 4) * kTileBytes);
  const volatile int* abort_flag = &s->abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t first = (int64_t)blockIdx.x * per_cta;
  const int64_t last = first + per_cta < nitems ? first + per_cta : nitems;  // exclusive
  const int64_t n = last > first ? last - first : 0;

  if (tid == 0) {
    prefetch_tmap(&map_x);
    prefetch_tmap(&map_y);
    for (int q = 0; q < kSlots; ++q) {
      mbar_init(&s->full[q], 1);
      mbar_init(&s->empty[q], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&s->s_full[q], 1);
      mbar_init(&s->s_empty[q], 1);
      mbar_init(&s->acc_full[q], 1);
      mbar_init(&s->acc_empty[q], kEpiThreads);
    }
    s->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&s->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int64_t prev_bh = -1;
      uint32_t nstate = 0;  // state tiles loaded so far
      for (int64_t g = 0; g < n; ++g) {
        const int64_t w = first + g;
        const int64_t bh = w / ntiles;
        const int t = (int)(w % ntiles);
        if (bh != prev_bh) {
          const uint32_t sb = nstate & 1u;
          if (nstate >= 2 && !mbar_wait_or_abort(&s->s_empty[sb], ((nstate >> 1) - 1) & 1u, SITE_OUT_MMA, abort_flag)) {
            s->abort = 1;
            break;
          }
          mbar_arrive_expect_tx(&s->s_full[sb], kTileBytes);
          bulk_load(ss + sb * kTileBytes, stiles + bh * kTileBytes, kTileBytes, &s->s_full[sb]);
          ++nstate;
          prev_bh = bh;
        }
        const int slot = (int)(g % kSlots);
        const int64_t u = g / kSlots;
        if (u > 0 && !mbar_wait_or_abort(&s->empty[slot], (uint32_t)((u - 1) & 1), SITE_OUT_MMA, abort_flag)) {
          s->abort = 1;
          break;
        }
        const int b = (int)(bh / H), h = (int)(bh % H);
        uint8_t* x = xs + slot * kTileBytes;
        mbar_arrive_expect_tx(&s->full[slot], kTileBytes);
        tma_load_4d(x, &map_x, &s->full[slot], 0, h, t * kTile, b);
        tma_load_4d(x + kBox, &map_x, &s->full[slot], 64, h, t * kTile, b);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, 128, 0, b_kmajor ? 0 : 1);
      int64_t prev_bh = -1;
      uint32_t nstate = 0;
      bool ok = true;
      for (int64_t g = 0; g < n && ok; ++g) {
        const int64_t bh = (first + g) / ntiles;
        if (bh != prev_bh) {
          // all MMAs so far were the last readers of the other state buffer
          if (nstate >= 1) mma_commit(&s->s_empty[(nstate - 1) & 1u]);
          const uint32_t sb = nstate & 1u;
          if (!(ok = mbar_wait_or_abort(&s->s_full[sb], (nstate >> 1) & 1u, SITE_OUT_TMA, abort_flag))) break;
          ++nstate;
          prev_bh = bh;
        }
        const int slot = (int)(g % kSlots);
        const int acc = (int)(g & 1);
        if (!(ok = mbar_wait_or_abort(&s->full[slot], (uint32_t)((g / kSlots) & 1), SITE_OUT_TMA, abort_flag))) break;
        if (g >= 2 && !(ok = mbar_wait_or_abort(&s->acc_empty[acc], (uint32_t)(((g >> 1) - 1) & 1), SITE_OUT_MMA,
                                                abort_flag)))
          break;
        tc_fence_after();
        const uint32_t ax = smem_u32(xs + slot * kTileBytes);
        const uint32_t as = smem_u32(ss + ((nstate - 1) & 1u) * kTileBytes);
        for (int kk = 0; kk < kD / 16; ++kk)
          mma_bf16(tmem + acc * 128, kmaj(ax, kk), b_kmajor ? kmaj(as, kk) : mnmaj(as, kk), idesc, kk != 0);
        mma_commit(&s->empty[slot]);
        mma_commit(&s->acc_full[acc]);
      }
      if (!ok) s->abort = 1;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;               // TMEM lanes 32*quad..
    const int half = (warp - 2) >> 2;        // column half
    const int row = quad * 32 + lane;
    const bool leader = tid == 64;           // issues the stores of the staging tiles
    bool bad = false;
    for (int64_t g = 0; g < n; ++g) {
      const int acc = (int)(g & 1);
      if (!bad && !mbar_wait_or_abort(&s->acc_full[acc], (uint32_t)((g >> 1) & 1), SITE_OUT_MMA, abort_flag)) {
        bad = true;
        s->abort = 1;
      }
      tc_fence_after();
      uint32_t r0[32], r1[32];
      const uint32_t tb = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)acc * 128 + half * 64;
      tmem_ld32(tb, r0);
      tmem_ld32(tb + 32, r1);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&s->acc_empty[acc]);
      uint32_t p[32];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        p[q] = pack_bf16(__uint_as_float(r0[2 * q]), __uint_as_float(r0[2 * q + 1]));
        p[16 + q] = pack_bf16(__uint_as_float(r1[2 * q]), __uint_as_float(r1[2 * q + 1]));
      }
      // the staging tile is free once the store issued two tiles ago has read it
      uint8_t* y = ys + (g & 1) * kTileBytes;
      if (leader) tma_store_wait_read1();
      named_sync(kEpiBar, kEpiThreads);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        st_tile16(y, row, half * 64 + q * 8, make_uint4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]));
      fence_async_smem();
      named_sync(kEpiBar, kEpiThreads);
      if (leader) {
        const int64_t w = first + g;
        const int64_t bh = w / ntiles;
        const int t = (int)(w % ntiles);
        tma_store_4d(&map_y, y, 0, (int)(bh % H), t * kTile, (int)(bh / H));
        tma_store_4d(&map_y, y + kBox, 64, (int)(bh % H), t * kTile, (int)(bh / H));
        tma_store_commit();
      }
    }
    if (leader) tma_store_wait0();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc_bidir_detail

bool tc_bidir_ok(int dtype, int d, int64_t N) {
  return dtype == LASP_BF16 && d == tc_bidir_detail::kD && N % tc_bidir_detail::kTile == 0;
}

cudaError_t bidir_total(const float* seg, float* total, void* tiles, int B, int H, int nseg, cudaStream_t st) {
  using namespace tc_bidir_detail;
  dim3 grid(kD * kD / 4 / kTotalCols, (unsigned)(B * H));
  bidir_total<<<grid, kTotalThreads, 0, st>>>(reinterpret_cast<const float4*>(seg), reinterpret_cast<float4*>(total),
                                             static_cast<uint8_t*>(tiles), H, nseg);
  return cudaGetLastError();
}

cudaError_t tc_bidir_apply(const void* x, const void* stiles, void* y, int B, int H, int64_t N, int d, int b_kmajor,
                           int num_sms, cudaStream_t st) {
  using namespace tc_bidir_detail;
  CUtensorMap mx, my;
  if (!make_token_map(&mx, x, B, H, N, d, kTile) || !make_token_map(&my, y, B, H, N, d, kTile))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + (kSlots + 4) * (size_t)kTileBytes + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(bidir_apply_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int ntiles = (int)(N / kTile);
  const int64_t nitems = (int64_t)B * H * ntiles;
  const int64_t grid = std::min<int64_t>(nitems, num_sms);
  const int64_t per_cta = (nitems + grid - 1) / grid;
  bidir_apply_tc<<<(unsigned)grid, kThreads, smem, st>>>(mx, my, static_cast<const uint8_t*>(stiles), H, ntiles,
                                                         nitems, per_cta, b_kmajor);
  return cudaGetLastError();
}

}  // namespace lasp
