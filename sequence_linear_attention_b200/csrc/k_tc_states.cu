// Chunk states on the 5th-generation tensor cores (LASP Eq. 10 with
// KV_{t-1} = 0, and the gradient state of Eq. 20):
//   M_c = (diag(w) A_c)^T B_c,   A_c, B_c = C x d token tiles of chunk c,
//   w_t = lambda^{C-1-t} (kind 0, (A, B) = (K, V)) or lambda^{t+1} (kind 1, (Q, dO)).
//
// Persistent CTAs (one per SM, 256 threads) take the (chunk, head, batch)
// items in turn. A chunk is consumed in stages of KB tokens (KB = 128, or the
// largest of 64/32/16 dividing C), and the stages of all of a CTA's chunks
// form one stream. Per
// stage: TMA brings A and B (KB rows x 128 features, two 64-feature boxes each,
// 128-byte swizzle) into a shared-memory slot; when lambda != 1 the four warps
// scale the rows of A by w_t in place (bf16); one thread issues KB/16
// tcgen05.mma (M = N = 128 features, K = 16 tokens) that accumulate M_c in
// TMEM. Both operands are MN-major: the tiles arrive token-major with features
// contiguous, which is exactly A^T and B with the reduced (token) index as the
// slow one. Up to six slots (192 KB) keep all but one stage's loads in flight
// under the current stage's scaling and MMAs (thread 32 issues the loads,
// thread 0 the MMAs). The epilogue reads the 128 x 128 fp32
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
constexpr int kMaxSlots = 6;
constexpr size_t kStageBudget = 192 * 1024;  // shared memory for the stage slots
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

// Work item n of this CTA (chunk index c, head h, batch b).
struct Work {
  int c, h, b;
};
__device__ __forceinline__ Work work_of(int64_t n, int T, int H) {
  const int64_t w = blockIdx.x + n * gridDim.x;
  Work r;
  r.c = (int)(w % T);
  r.h = (int)((w / T) % H);
  r.b = (int)(w / ((int64_t)T * H));
  return r;
}

// Persistent: each CTA takes chunks blockIdx.x, blockIdx.x + gridDim.x, ...
// and consumes their stages as one stream, so the next chunk's loads are in
// flight during the current chunk's epilogue.
__global__ void __launch_bounds__(kThreads, 1) chunk_states_tc(const __grid_constant__ CUtensorMap map_a,
                                                            const __grid_constant__ CUtensorMap map_b,
                                                            const float* decay, float* __restrict__ M, int H,
                                                            int C, int KB, int nslots, int kind, int T,
                                                            int64_t nitems, int64_t t_out, int slot_stride,
                                                            int slot_offset) {
  extern __shared__ uint8_t smem_raw[];
  // tiles need 1024-byte alignment for the 128-byte swizzle atoms
  uint8_t* tiles = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int nstages = C / KB;
  const uint32_t tile_bytes = (uint32_t)KB * 256;  // KB rows x 128 features x bf16
  Smem* s = reinterpret_cast<Smem*>(tiles + nslots * 2 * tile_bytes);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kProducer = 32;  // issues the TMA loads; thread 0 issues the MMAs
  const int64_t my_items = nitems > blockIdx.x ? (nitems - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int64_t nstream = my_items * nstages;  // stages this CTA consumes

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

  auto issue = [&](int64_t g) {
    const Work wk = work_of(g / nstages, T, H);
    const int k = (int)(g % nstages);
    issue_stage(tiles, tile_bytes, s, &map_a, &map_b, (int)(g % nslots), wk.c * C + k * KB, wk.h, wk.b);
  };
  if (tid == kProducer)
    for (int64_t g = 0; g < nslots && g < nstream; ++g) issue(g);

  constexpr uint32_t idesc = idesc_bf16(128, 128, 1, 1);
  Work wk{0, 0, 0};
  float lam = 1.f, l2 = 0.f;
  for (int64_t g = 0; g < nstream; ++g) {
    const int slot = (int)(g % nslots);
    const uint32_t par = (uint32_t)((g / nslots) & 1);
    const int k = (int)(g % nstages);
    const int64_t n = g / nstages;
    if (k == 0) {  // a new chunk: its coordinates and decay
      wk = work_of(n, T, H);
      lam = load_decay(decay, wk.h);
      l2 = log2f(lam);
    }
    if (!mbar_wait(&s->full[slot], par, SITE_STATES_TMA)) s->abort = 1;
    if (lam != 1.0f) {
      // scale row r of A by w_{k*KB + r}; the row of a 16-byte chunk is its
      // byte offset / 128 in either 64-feature box, whatever the swizzle
      uint4* a = reinterpret_cast<uint4*>(tiles + (size_t)slot * 2 * tile_bytes);
      const int nchunks = KB * 16;
      for (int q = tid; q < nchunks; q += kThreads) {
        const int r = (q % (KB * 8)) / 8;
        const int t = k * KB + r;
        const float w = kind == 0 ? decay_pow(l2, (float)(C - 1 - t)) : decay_pow(l2, (float)(t + 1));
        uint4 x = a[q];
        x.x = bf16x2_scale(x.x, w);
        x.y = bf16x2_scale(x.y, w);
        x.z = bf16x2_scale(x.z, w);
        x.w = bf16x2_scale(x.w, w);
        a[q] = x;
      }
      fence_async_smem();
    }
    tc_fence_before();
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
      mma_commit(&s->empty[slot]);
      if (k == nstages - 1) mma_commit(&s->done);
    }
    if (tid == kProducer && g >= 1 && g - 1 + nslots < nstream) {
      // refill the slot of the previous stage (its MMAs were issued one step
      // ago), keeping nslots - 1 stages in flight while this one is consumed
      const int64_t gp = g - 1;
      if (mbar_wait(&s->empty[gp % nslots], (uint32_t)((gp / nslots) & 1), SITE_STATES_MMA)) issue(gp + nslots);
      else s->abort = 1;
    }
    if (k == nstages - 1) {
      // epilogue of this chunk: warp w reads TMEM lanes (rows) 32*(w%4).. and the
      // column half w/4; the state goes to slot c * slot_stride + slot_offset
      if (mbar_wait(&s->done, (uint32_t)(n & 1), SITE_STATES_MMA)) {
        tc_fence_after();
        const int row = (warp & 3) * 32 + lane, half = warp >> 2;
        const int64_t oslot = (int64_t)wk.c * slot_stride + slot_offset;
        float* out = M + ((((int64_t)wk.b * t_out + oslot) * H + wk.h) * kD + row) * kD;
        uint32_t r0[32], r1[32];
        tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (2 * half) * 32, r0);
        tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (2 * half + 1) * 32, r1);
        tmem_ld_wait();
        float4* o0 = reinterpret_cast<float4*>(out + (2 * half) * 32);
        float4* o1 = reinterpret_cast<float4*>(out + (2 * half + 1) * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          __stcs(o0 + q, make_float4(__uint_as_float(r0[4 * q]), __uint_as_float(r0[4 * q + 1]),
                                     __uint_as_float(r0[4 * q + 2]), __uint_as_float(r0[4 * q + 3])));
          __stcs(o1 + q, make_float4(__uint_as_float(r1[4 * q]), __uint_as_float(r1[4 * q + 1]),
                                     __uint_as_float(r1[4 * q + 2]), __uint_as_float(r1[4 * q + 3])));
        }
      } else {
        s->abort = 1;
      }
      // the next chunk's first MMA overwrites the accumulator
      tc_fence_before();
      __syncthreads();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// Stage rows: the largest of 128/64/32/16 dividing C.
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
  const int nslots = (int)std::min<size_t>(kMaxSlots, kStageBudget / ((size_t)2 * KB * 256));
  const size_t smem = 1024 + (size_t)nslots * 2 * KB * 256 + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(chunk_states_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int T = (int)(N / C);
  const int64_t nitems = (int64_t)B * H * T;
  const unsigned grid = (unsigned)std::min<int64_t>(nitems, sms);
  chunk_states_tc<<<grid, kThreads, smem, st>>>(ma, mb, decay, M, H, C, KB, nslots, kind, T, nitems, t_out,
                                               slot_stride, slot_offset);
  return cudaGetLastError();
}

cudaError_t tc_chunk_states(const void* a, const void* bm, const float* decay, float* M, int B, int H, int64_t N,
                            int d, int C, int kind, cudaStream_t st) {
  return tc_chunk_states_slots(a, bm, decay, M, B, H, N, d, C, kind, N / C, 1, 0, st);
}

}  // namespace lasp
