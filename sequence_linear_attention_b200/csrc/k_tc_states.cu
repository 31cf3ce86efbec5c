// Chunk states on the 5th-generation tensor cores (LASP Eq. 10 with
// KV_{t-1} = 0, and the gradient state of Eq. 20):
//   M_c = (diag(w) A_c)^T B_c,   A_c, B_c = C x d token tiles of chunk c,
//   w_t = lambda^{C-1-t} (kind 0, (A, B) = (K, V)) or lambda^{t+1} (kind 1, (Q, dO)).
//
// One CTA per (chunk, head, batch), 256 threads. The chunk is consumed in
// stages of KB tokens (KB = 128, or the largest of 64/32/16 dividing C). Per
// stage: TMA brings A and B (KB rows x 128 features, two 64-feature boxes each,
// 128-byte swizzle) into a shared-memory slot; when lambda != 1 the four warps
// scale the rows of A by w_t in place (bf16); one thread issues KB/16
// tcgen05.mma (M = N = 128 features, K = 16 tokens) that accumulate M_c in
// TMEM. Both operands are MN-major: the tiles arrive token-major with features
// contiguous, which is exactly A^T and B with the reduced (token) index as the
// slow one. Up to three slots keep two stages' loads in flight under the
// current stage's scaling and MMAs. The epilogue reads the 128 x 128 fp32
// accumulator from TMEM (warp w: rows 32*(w%4).., column half w/4) and writes
// the state row by row.
#include <algorithm>

#include "kernels.h"
#include "lasp_common.cuh"
#include "sm100.cuh"
#include "tc_kernels.h"
#include "tma_host.h"

namespace lasp {
namespace tc_states_detail {

using namespace sm100;

constexpr int kD = 128;           // head dimension handled here
constexpr int kThreads = 256;
constexpr int kMaxSlots = 3;
constexpr uint32_t kTmemCols = 128;  // one 128 x 128 fp32 accumulator

struct Smem {
  uint64_t full[kMaxSlots];
  uint64_t empty[kMaxSlots];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ uint32_t bf16x2_scale(uint32_t x, float w) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&x);
  float2 f = __bfloat1622float2(h);
  __nv_bfloat162 r = __floats2bfloat162_rn(f.x * w, f.y * w);
  return *reinterpret_cast<uint32_t*>(&r);
}

// Issues the four TMA boxes of one stage (A and B, two 64-feature boxes each)
// into `slot`.
__device__ __forceinline__ void issue_stage(uint8_t* tiles, uint32_t tile_bytes, Smem* s, const CUtensorMap* map_a,
                                            const CUtensorMap* map_b, int slot, int row, int h, int b) {
  uint8_t* a = tiles + (size_t)slot * 2 * tile_bytes;
  uint8_t* bb = a + tile_bytes;
  mbar_arrive_expect_tx(&s->full[slot], 2 * tile_bytes);
  tma_load_4d(a, map_a, &s->full[slot], 0, h, row, b);
  tma_load_4d(a + tile_bytes / 2, map_a, &s->full[slot], 64, h, row, b);
  tma_load_4d(bb, map_b, &s->full[slot], 0, h, row, b);
  tma_load_4d(bb + tile_bytes / 2, map_b, &s->full[slot], 64, h, row, b);
}

__global__ void __launch_bounds__(kThreads, 1) chunk_states_tc(const __grid_constant__ CUtensorMap map_a,
                                                            const __grid_constant__ CUtensorMap map_b,
                                                            const float* decay, float* __restrict__ M, int H,
                                                            int C, int KB, int kind, int64_t t_out,
                                                            int slot_stride, int slot_offset) {
  extern __shared__ uint8_t smem_raw[];
  // tiles need 1024-byte alignment for the 128-byte swizzle atoms
  uint8_t* tiles = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int nstages = C / KB;
  const int nslots = nstages < kMaxSlots ? nstages : kMaxSlots;
  const uint32_t tile_bytes = (uint32_t)KB * 256;  // KB rows x 128 features x bf16
  Smem* s = reinterpret_cast<Smem*>(tiles + nslots * 2 * tile_bytes);

  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float lam = load_decay(decay, h);
  const float l2 = log2f(lam);
  const bool scale = lam != 1.0f;

  if (tid == 0) {
    prefetch_tmap(&map_a);
    prefetch_tmap(&map_b);
    for (int q = 0; q < kMaxSlots; ++q) {
      mbar_init(&s->full[q], 1);
      mbar_init(&s->empty[q], 1);
    }
    mbar_init(&s->done, 1);
    s->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s->tmem_base;

  if (tid == 0) {
    for (int k = 0; k < nslots; ++k) issue_stage(tiles, tile_bytes, s, &map_a, &map_b, k, c * C + k * KB, h, b);
  }

  constexpr uint32_t idesc = idesc_bf16(128, 128, 1, 1);
  for (int k = 0; k < nstages; ++k) {
    const int slot = k % nslots;
    const uint32_t par = (uint32_t)(k / nslots) & 1u;
    if (!mbar_wait(&s->full[slot], par, SITE_STATES_TMA)) s->abort = 1;
    if (scale) {
      // scale row r of A by w_{k*KB + r}; the row of a 16-byte chunk is its
      // byte offset / 128 in either 64-feature box, whatever the swizzle
      uint4* a = reinterpret_cast<uint4*>(tiles + (size_t)slot * 2 * tile_bytes);
      const int nchunks = KB * 16;
      for (int g = tid; g < nchunks; g += kThreads) {
        const int r = (g % (KB * 8)) / 8;
        const int t = k * KB + r;
        const float w = kind == 0 ? decay_pow(l2, (float)(C - 1 - t)) : decay_pow(l2, (float)(t + 1));
        uint4 x = a[g];
        x.x = bf16x2_scale(x.x, w);
        x.y = bf16x2_scale(x.y, w);
        x.z = bf16x2_scale(x.z, w);
        x.w = bf16x2_scale(x.w, w);
        a[g] = x;
      }
      fence_async_smem();
    }
    __syncthreads();
    if (s->abort) break;
    if (tid == 0) {
      tc_fence_after();
      const uint32_t a0 = smem_u32(tiles + (size_t)slot * 2 * tile_bytes), b0 = a0 + tile_bytes;
      for (int j = 0; j < KB / 16; ++j) {
        const uint64_t ad = sw128_desc(a0 + j * 2048, KB * 128, 1024);
        const uint64_t bd = sw128_desc(b0 + j * 2048, KB * 128, 1024);
        mma_bf16(tmem, ad, bd, idesc, (k | j) != 0);
      }
      mma_commit(k + 1 < nstages ? &s->empty[slot] : &s->done);
      // refill the slot of the previous stage (its MMAs were issued one stage
      // ago), keeping nslots - 1 stages in flight while this one is consumed
      const int kr = k - 1 + nslots;
      if (k >= 1 && kr < nstages) {
        const int pslot = (k - 1) % nslots;
        if (mbar_wait(&s->empty[pslot], (uint32_t)((k - 1) / nslots) & 1u, SITE_STATES_MMA))
          issue_stage(tiles, tile_bytes, s, &map_a, &map_b, pslot, c * C + kr * KB, h, b);
        else
          s->abort = 1;
      }
    }
  }
  __syncthreads();
  const bool ok = !s->abort && mbar_wait(&s->done, 0, SITE_STATES_MMA);
  tc_fence_after();
  if (ok) {
    // warp w reads TMEM lanes (rows) 32*(w%4).. and the column half w/4
    const int row = (warp & 3) * 32 + lane, half = warp >> 2;
    // chunk c's state goes to slot c * slot_stride + slot_offset of an array with t_out slots
    const int64_t slot = (int64_t)c * slot_stride + slot_offset;
    float* out = M + ((((int64_t)b * t_out + slot) * H + h) * kD + row) * kD;
#pragma unroll 1
    for (int cc = 2 * half; cc < 2 * half + 2; ++cc) {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + cc * 32, r);
      tmem_ld_wait();
      float4* o4 = reinterpret_cast<float4*>(out + cc * 32);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        o4[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]), __uint_as_float(r[4 * q + 2]),
                            __uint_as_float(r[4 * q + 3]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

inline int stage_rows(int C) {
  for (int kb : {128, 64, 32, 16})
    if (C % kb == 0) return kb;
  return 0;
}

}  // namespace tc_states_detail

bool tc_states_ok(int dtype, int d, int64_t C) {
  return dtype == LASP_BF16 && d == tc_states_detail::kD && C % 16 == 0;
}

cudaError_t tc_chunk_states_slots(const void* a, const void* bm, const float* decay, float* M, int B, int H,
                                  int64_t N, int d, int C, int kind, int64_t t_out, int slot_stride, int slot_offset,
                                  cudaStream_t st) {
  using namespace tc_states_detail;
  const int KB = stage_rows(C);
  CUtensorMap ma, mb;
  if (!make_token_map(&ma, a, B, H, N, d, KB) || !make_token_map(&mb, bm, B, H, N, d, KB))
    return cudaErrorInvalidValue;
  const int nslots = std::min(C / KB, kMaxSlots);
  const size_t smem = 1024 + (size_t)nslots * 2 * KB * 256 + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(chunk_states_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(N / C), H, B);
  chunk_states_tc<<<grid, kThreads, smem, st>>>(ma, mb, decay, M, H, C, KB, kind, t_out, slot_stride, slot_offset);
  return cudaGetLastError();
}

cudaError_t tc_chunk_states(const void* a, const void* bm, const float* decay, float* M, int B, int H, int64_t N,
                            int d, int C, int kind, cudaStream_t st) {
  return tc_chunk_states_slots(a, bm, decay, M, B, H, N, d, C, kind, N / C, 1, 0, st);
}

}  // namespace lasp
