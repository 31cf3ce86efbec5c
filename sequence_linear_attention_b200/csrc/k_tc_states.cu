// Chunk states on the 5th-generation tensor cores (LASP Eq. 10 with
// KV_{t-1} = 0, and the gradient state of Eq. 20):
//   M_c = (diag(w) A_c)^T B_c,   A_c, B_c = C x d token tiles of chunk c,
//   w_t = lambda^{C-1-t} (kind 0, (A, B) = (K, V)) or lambda^{t+1} (kind 1, (Q, dO)).
//
// Persistent, warp-specialized CTAs (one per SM) take the (chunk, head,
// batch) items in turn. A chunk is consumed in stages of KB tokens (KB = 128,
// or the largest of 64/32/16 dividing C); the stages of all of a CTA's chunks
// form one stream through up to six shared-memory slots (192 KB). Per stage:
// warp 1 brings A and B by TMA (KB rows x 128 features, two 64-feature boxes
// each, 128-byte swizzle; with d <= 64 only the first box is loaded (for d =
// 32 its upper 32 features read as zeros) and the second stays zero, so the
// MMA shape does not change); when lambda != 1 the eight worker warps scale the
// rows of A by w_t in place (bf16, one thread per 128-byte row); warp 0 issues
// KB/16 tcgen05.mma (M = N = 128 features, K = 16 tokens) accumulating M_c in
// TMEM. Both operands are MN-major: the tiles arrive token-major with features
// contiguous, which is exactly A^T and B with the reduced (token) index as the
// slow one. Two TMEM accumulators alternate between chunks; the workers read a
// finished one (warp w: TMEM lanes 32*(w%4).., one column half) and store it by
// TMA in 32 x 32 blocks staged in shared memory, while the next chunk
// accumulates. Only the d x d block of each accumulator is stored.
#include <algorithm>

#include "kernels.h"
#include "lasp_common.cuh"
#include "sm100.cuh"
#include "tc_kernels.h"
#include "tma_host.h"

namespace lasp {
namespace tc_states_detail {

using namespace sm100;

constexpr int kD = 128;              // features per tile (d = 64 fills the first half)
constexpr int kThreads = 320;        // warp 0: MMA, warp 1: TMA, warps 2-9: scaling and epilogue
constexpr int kWorkers = 256;
constexpr uint32_t kStageOutBytes = 32 * 128;  // per worker warp: a 32 x 32 fp32 block of the state
constexpr int kMaxSlots = 6;
constexpr size_t kStageBudget = 192 * 1024;  // shared memory for the stage slots
constexpr uint32_t kTmemCols = 256;  // two 128 x 128 fp32 accumulators

__device__ __forceinline__ bool aborted(const int* flag) { return *(volatile const int*)flag != 0; }

struct Smem {
  uint64_t full[kMaxSlots];    // TMA bytes of a stage have landed
  uint64_t scaled[kMaxSlots];  // the workers have scaled a stage's A rows
  uint64_t empty[kMaxSlots];   // the MMAs reading a stage have completed
  uint64_t acc_full[2];        // an accumulator holds a finished state
  uint64_t acc_empty[2];       // the workers have read an accumulator out
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ uint32_t bf16x2_scale(uint32_t x, float w) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&x);
  float2 f = __bfloat1622float2(h);
  __nv_bfloat162 r = __floats2bfloat162_rn(f.x * w, f.y * w);
  return *reinterpret_cast<uint32_t*>(&r);
}

// Work item n of this CTA (chunk index c, head h, batch b).
struct Work {
  int c, h, b;
};
__device__ __forceinline__ Work work_of(int64_t n, int T, int H, int64_t item0) {
  const int64_t w = item0 + blockIdx.x + n * gridDim.x;
  Work r;
  r.c = (int)(w % T);
  r.h = (int)((w / T) % H);
  r.b = (int)(w / ((int64_t)T * H));
  return r;
}

// Persistent and warp-specialized: each CTA takes chunks blockIdx.x,
// blockIdx.x + gridDim.x, ... and their KB-token stages form one stream that
// flows through nslots shared-memory slots: warp 1 loads a stage, the four
// worker warps scale its A rows by the decay weights, warp 0 issues its MMAs
// into one of two TMEM accumulators; when a chunk's last stage is done the
// workers read that accumulator out while the next chunk accumulates in the
// other one. Hand-offs are mbarriers; no CTA-wide barrier in the stream.
__global__ void __launch_bounds__(kThreads, 1) chunk_states_tc(const __grid_constant__ CUtensorMap map_a,
                                                            const __grid_constant__ CUtensorMap map_b,
                                                            const __grid_constant__ CUtensorMap map_m,
                                                            const float* decay, int H, int d,
                                                            int C, int KB, int nslots, int kind, int T,
                                                            int64_t nitems, int64_t t_out, int slot_stride,
                                                            int slot_offset, int64_t item0) {
  extern __shared__ uint8_t smem_raw[];
  // tiles need 1024-byte alignment for the 128-byte swizzle atoms
  uint8_t* tiles = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int nstages = C / KB;
  const uint32_t tile_bytes = (uint32_t)KB * 256;  // KB rows x 128 features x bf16
  uint8_t* out_stage = tiles + nslots * 2 * tile_bytes;  // kStageOutBytes per worker warp
  Smem* s = reinterpret_cast<Smem*>(out_stage + (kWorkers / 32) * kStageOutBytes);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t my_items = nitems > blockIdx.x ? (nitems - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int64_t nstream = my_items * nstages;
  const int nbox = d > 64 ? 2 : 1;  // 64-feature boxes loaded per tile

  if (nbox == 1) {
    // the second box of every A and B tile stays zero for the whole kernel
    for (int s2 = 0; s2 < 2 * nslots; ++s2) {
      uint4* z = reinterpret_cast<uint4*>(tiles + (size_t)s2 * tile_bytes + tile_bytes / 2);
      for (uint32_t q = threadIdx.x; q < tile_bytes / 32; q += kThreads) z[q] = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
  }

  if (tid == 0) {
    prefetch_tmap(&map_a);
    prefetch_tmap(&map_b);
    prefetch_tmap(&map_m);
    for (int q = 0; q < kMaxSlots; ++q) {
      mbar_init(&s->full[q], 1);
      mbar_init(&s->scaled[q], kWorkers);
      mbar_init(&s->empty[q], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&s->acc_full[q], 1);
      mbar_init(&s->acc_empty[q], kWorkers);
    }
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

  if (warp == 1) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      // the token tiles stream through once; the states written below stay in
      // L2 for the scan that reads them next
      const uint64_t stream_policy = l2_evict_first();
      for (int64_t g = 0; g < nstream && !aborted(&s->abort); ++g) {
        const int slot = (int)(g % nslots);
        const int64_t u = g / nslots;
        if (u > 0 && !mbar_wait(&s->empty[slot], (uint32_t)((u - 1) & 1), SITE_STATES_MMA)) {
          s->abort = 1;
          break;
        }
        const Work wk = work_of(g / nstages, T, H, item0);
        const int row = wk.c * C + (int)(g % nstages) * KB;
        uint8_t* a = tiles + (size_t)slot * 2 * tile_bytes;
        uint8_t* bb = a + tile_bytes;
        mbar_arrive_expect_tx(&s->full[slot], nbox * tile_bytes);
        tma_load_4d_hint(a, &map_a, &s->full[slot], 0, wk.h, row, wk.b, stream_policy);
        tma_load_4d_hint(bb, &map_b, &s->full[slot], 0, wk.h, row, wk.b, stream_policy);
        if (nbox == 2) {
          tma_load_4d_hint(a + tile_bytes / 2, &map_a, &s->full[slot], 64, wk.h, row, wk.b, stream_policy);
          tma_load_4d_hint(bb + tile_bytes / 2, &map_b, &s->full[slot], 64, wk.h, row, wk.b, stream_policy);
        }
      }
    }
  } else if (warp == 0) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, 128, 1, 1);
      for (int64_t g = 0; g < nstream && !aborted(&s->abort); ++g) {
        const int slot = (int)(g % nslots);
        const int64_t u = g / nslots;
        const int k = (int)(g % nstages);
        const int64_t n = g / nstages;
        const int acc = (int)(n & 1);
        if (!mbar_wait(&s->scaled[slot], (uint32_t)(u & 1), SITE_STATES_TMA)) {
          s->abort = 1;
          break;
        }
        if (k == 0 && n >= 2 && !mbar_wait(&s->acc_empty[acc], (uint32_t)(((n >> 1) - 1) & 1), SITE_STATES_MMA)) {
          s->abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(tiles + (size_t)slot * 2 * tile_bytes), b0 = a0 + tile_bytes;
        const uint32_t d = tmem + (uint32_t)acc * 128;
        for (int j = 0; j < KB / 16; ++j) {
          const uint64_t ad = sw128_desc(a0 + j * 2048, KB * 128, 1024);
          const uint64_t bd = sw128_desc(b0 + j * 2048, KB * 128, 1024);
          mma_bf16(d, ad, bd, idesc, (k | j) != 0);
        }
        mma_commit(&s->empty[slot]);
        if (k == nstages - 1) mma_commit(&s->acc_full[acc]);
      }
    }
  } else {
    // ------------------------------------------------- workers (warps 2-9)
    const int wt = tid - 64;              // 0..255
    const int quad = warp & 3;            // the TMEM lanes this warp may read
    const int colhalf = (warp - 2) >> 2;  // and the half of the columns it writes out
    uint8_t* stage_out = out_stage + (warp - 2) * kStageOutBytes;
    Work wk{0, 0, 0};
    float lam = 1.f, l2 = 0.f;
    for (int64_t g = 0; g < nstream; ++g) {
      const int slot = (int)(g % nslots);
      const int64_t u = g / nslots;
      const int k = (int)(g % nstages);
      const int64_t n = g / nstages;
      if (k == 0) {
        wk = work_of(n, T, H, item0);
        lam = load_decay(decay, wk.h);
        l2 = log2f(lam);
      }
      if (!mbar_wait(&s->full[slot], (uint32_t)(u & 1), SITE_STATES_TMA)) {
        s->abort = 1;
        break;
      }
      if (lam != 1.0f) {
        // scale row r of A by w_{k*KB + r}: one thread per row of a 64-feature
        // box (8 chunks of 16 bytes, chunk c of row r stored at position
        // c ^ (r & 7), so the eight rows of a quarter-warp hit different banks)
        uint8_t* a = tiles + (size_t)slot * 2 * tile_bytes;
        for (int q = wt; q < nbox * KB; q += kWorkers) {
          const int r = q % KB;
          const int t = k * KB + r;
          const float w = kind == 0 ? decay_pow(l2, (float)(C - 1 - t)) : decay_pow(l2, (float)(t + 1));
          uint8_t* line = a + (q / KB) * (tile_bytes / 2) + r * 128;
          uint4 x[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) x[c] = *reinterpret_cast<const uint4*>(line + ((c ^ (r & 7)) << 4));
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            x[c].x = bf16x2_scale(x[c].x, w);
            x[c].y = bf16x2_scale(x[c].y, w);
            x[c].z = bf16x2_scale(x[c].z, w);
            x[c].w = bf16x2_scale(x[c].w, w);
            *reinterpret_cast<uint4*>(line + ((c ^ (r & 7)) << 4)) = x[c];
          }
        }
        fence_async_smem();
      }
      mbar_arrive(&s->scaled[slot]);
      if (k == nstages - 1) {
        // the chunk's state: accumulator n & 1 -> slot c * slot_stride + slot_offset,
        // as 32 x 32 blocks staged in shared memory and stored by TMA
        const int acc = (int)(n & 1);
        if (!mbar_wait(&s->acc_full[acc], (uint32_t)((n >> 1) & 1), SITE_STATES_MMA)) {
          s->abort = 1;
          break;
        }
        tc_fence_after();
        const int64_t oslot = (int64_t)wk.c * slot_stride + slot_offset;
        const int y = (int)((((int64_t)wk.b * t_out + oslot) * H + wk.h) * d + quad * 32);
        // this warp's 32 rows x 64 columns of the accumulator, if inside d x d
        const bool mine = quad * 32 < d && colhalf * 64 < d;
        const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)acc * 128;
        uint32_t r0[32], r1[32];
        tmem_ld32(tbase + (2 * colhalf) * 32, r0);
        tmem_ld32(tbase + (2 * colhalf + 1) * 32, r1);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s->acc_empty[acc]);
#pragma unroll
        for (int cb = 0; cb < 2 && mine && (2 * colhalf + cb) * 32 < d; ++cb) {
          // the staging block is free once this warp's previous store has read it
          if (lane == 0) tma_store_wait_read0();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t* v = cb == 0 ? r0 + 4 * c : r1 + 4 * c;
            *reinterpret_cast<uint4*>(stage_out + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                make_uint4(v[0], v[1], v[2], v[3]);
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d_hint(&map_m, stage_out, (2 * colhalf + cb) * 32, y, l2_evict_last());
            tma_store_commit();
          }
        }
      }
    }
    if (lane == 0) tma_store_wait0();
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
  return dtype == LASP_BF16 && (d == 32 || d == 64 || d == tc_states_detail::kD) && C % 16 == 0;
}

cudaError_t tc_chunk_states_slots(const void* a, const void* bm, const float* decay, float* M, int B, int H,
                                  int64_t N, int d, int C, int kind, int64_t t_out, int slot_stride, int slot_offset,
                                  cudaStream_t st, int64_t bh0, int64_t nbh) {
  using namespace tc_states_detail;
  const int KB = stage_rows(C);
  CUtensorMap ma, mb, mm;
  if (!make_token_map(&ma, a, B, H, N, d, KB) || !make_token_map(&mb, bm, B, H, N, d, KB) ||
      !make_state_map(&mm, M, (int64_t)B * t_out * H, d, 32))
    return cudaErrorInvalidValue;
  const int nslots = (int)std::min<size_t>(kMaxSlots, kStageBudget / ((size_t)2 * KB * 256));
  const size_t smem = 1024 + (size_t)nslots * 2 * KB * 256 + (kWorkers / 32) * kStageOutBytes + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(chunk_states_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int T = (int)(N / C);
  if (nbh < 0) nbh = (int64_t)B * H;  // (b, h) pairs bh0 .. bh0 + nbh - 1, in b-major order
  const int64_t nitems = nbh * T;
  if (nitems == 0) return cudaSuccess;
  const unsigned grid = (unsigned)std::min<int64_t>(nitems, sms);
  chunk_states_tc<<<grid, kThreads, smem, st>>>(ma, mb, mm, decay, H, d, C, KB, nslots, kind, T, nitems, t_out,
                                               slot_stride, slot_offset, bh0 * T);
  return cudaGetLastError();
}

cudaError_t tc_chunk_states(const void* a, const void* bm, const float* decay, float* M, int B, int H, int64_t N,
                            int d, int C, int kind, cudaStream_t st) {
  return tc_chunk_states_slots(a, bm, decay, M, B, H, N, d, C, kind, N / C, 1, 0, st);
}

}  // namespace lasp
