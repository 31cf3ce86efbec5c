// Forward pass over segments, with the running state kept on chip: the
// LASP-2 decomposition applied inside one GPU (LASP-2 review, "The reading":
// per-chunk states, a prefix over them, then a local pass), with the local
// pass done like LASP's own recurrence over chunks (LASP Algorithm 2 steps
// 11-18: O_inter from KV_{t-1}, then KV_t = lambda^C KV_{t-1} + (lambda^C
// Lambda^-1 K_t)^T V_t), bf16, d = 128.
//
// The sequence is cut into segments of G tokens (a multiple of C and of the
// 128-token tile). Before this kernel, the segment states and an exclusive
// prefix over them put P of each segment's first chunk into the state cache.
// Here one persistent CTA (256 threads) takes segments in turn and walks their
// 128-token tiles in order, holding the state P (fp32) in TMEM:
//
//   MMA 1:  S = Q K^T (TMEM S),  O_inter = Q P_bf16 (TMEM I)
//   epi A:  S' = Mask . S -> bf16 over Q;  K~ = diag(lambda^{127-j}) K in place;
//           P <- lambda^128 P in TMEM (and, for C > 128, P -> fp32 cache at chunk starts)
//   MMA 2:  O_intra = S' V (TMEM O);  P += K~^T V (TMEM P)
//   epi B:  O = O_intra + lambda^{i+1} O_inter -> bf16 over K~ -> TMA store;
//           P -> bf16 operand for the next tile
//
// With C = 128 each tile starts a chunk, and the bf16 operand tile of the
// entering state (already in shared memory for O_inter) goes to the chunk's
// cache slot by one bulk copy; the backward walk loads it back as is. Two sets
// of Q/K/V buffers alternate: while a tile is computed, the next tile's loads
// (possibly of the next segment) are in flight. In every epilogue
// warp w owns TMEM lanes (rows) 32*(w%4).. and the column half w/4.
#include <algorithm>

#include "kernels.h"
#include "lasp_common.cuh"
#include "sm100.cuh"
#include "tc_kernels.h"
#include "tma_host.h"

namespace lasp {
namespace tc_fwd_walk_detail {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr uint32_t kTileBytes = kTile * kD * 2;
constexpr uint32_t kBox = kTileBytes / 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t TS = 0, TI = 128, TO = 256, TP = 384;

struct Smem {
  uint64_t load[2];
  uint64_t mma1, mma2a, mma2;
  uint64_t ld_state;
  uint32_t tmem_base;
  int abort;
  float pw[kTile];
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t x, float w) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&x);
  float2 f = __bfloat1622float2(h);
  return pack_bf16(f.x * w, f.y * w);
}
__device__ __forceinline__ void st_tile16(uint8_t* tile, int row, int col, uint4 v) {
  *reinterpret_cast<uint4*>(tile + (col >> 6) * kBox + sw128_offset(row, (col & 63) >> 3)) = v;
}
__device__ __forceinline__ uint64_t kmaj(uint32_t tile, int kk) {
  return sw128_desc(tile + (kk >> 2) * kBox + (kk & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t mnmaj(uint32_t tile, int kk) { return sw128_desc(tile + kk * 2048, kBox, 1024); }

// 32 fp32 values of row `row` (columns col..col+31) -> bf16 into a tile.
__device__ __forceinline__ void st_row32_bf16(uint8_t* tile, int row, int col, const float* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    st_tile16(tile, row, col + q * 8,
              make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                         pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7])));
}

struct Item {
  int b, h, seg;
};
__device__ __forceinline__ Item item_of(int64_t w, int H, int nseg) {
  Item it;
  it.seg = (int)(w % nseg);
  it.h = (int)((w / nseg) % H);
  it.b = (int)(w / ((int64_t)nseg * H));
  return it;
}

__global__ void __launch_bounds__(kThreads, 1) fwd_walk_tc(const __grid_constant__ CUtensorMap map_q,
                                                            const __grid_constant__ CUtensorMap map_k,
                                                            const __grid_constant__ CUtensorMap map_v,
                                                            const __grid_constant__ CUtensorMap map_o,
                                                            const __grid_constant__ CUtensorMap map_state,
                                                            const float* decay, float* __restrict__ P, int H,
                                                            int T, int C, int G, int nseg, int64_t nitems,
                                                            int cache_bf16) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sP = base + 6 * kTileBytes;
  Smem* s = reinterpret_cast<Smem*>(base + 7 * kTileBytes);
  auto bufQ = [&](int set) { return base + set * 3 * kTileBytes; };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i = (warp & 3) * 32 + lane;  // the row this thread owns in every epilogue
  const int half = warp >> 2;            // and the column half
  const int tiles = G / kTile;

  if (tid == 0) {
    prefetch_tmap(&map_q);
    prefetch_tmap(&map_k);
    prefetch_tmap(&map_v);
    prefetch_tmap(&map_o);
    mbar_init(&s->load[0], 1);
    mbar_init(&s->load[1], 1);
    mbar_init(&s->mma1, 1);
    mbar_init(&s->mma2a, 1);
    mbar_init(&s->mma2, 1);
    mbar_init(&s->ld_state, 1);
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
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);

  // loads of one tile (Q, K, V: two 64-feature boxes each) into buffer set `set`
  auto issue_loads = [&](int set, const Item& it, int t) {
    uint8_t* q = bufQ(set);
    const int row = it.seg * G + t * kTile;
    mbar_arrive_expect_tx(&s->load[set], 3 * kTileBytes);
    tma_load_4d(q, &map_q, &s->load[set], 0, it.h, row, it.b);
    tma_load_4d(q + kBox, &map_q, &s->load[set], 64, it.h, row, it.b);
    tma_load_4d(q + kTileBytes, &map_k, &s->load[set], 0, it.h, row, it.b);
    tma_load_4d(q + kTileBytes + kBox, &map_k, &s->load[set], 64, it.h, row, it.b);
    tma_load_4d(q + 2 * kTileBytes, &map_v, &s->load[set], 0, it.h, row, it.b);
    tma_load_4d(q + 2 * kTileBytes + kBox, &map_v, &s->load[set], 64, it.h, row, it.b);
  };

  // the fp32 state entering a segment (the slot of its first chunk) as four
  // 32-column boxes: boxes 0, 1 into the K buffer of `set`, boxes 2, 3 into its
  // V buffer, both free at that point
  auto issue_state_load = [&](int set, const Item& it) {
    const int64_t slot = ((int64_t)it.seg * G) / C;
    const int y = (int)((((int64_t)it.b * T + slot) * H + it.h) * kD);
    mbar_arrive_expect_tx(&s->ld_state, kD * kD * 4);
#pragma unroll
    for (int bx = 0; bx < 4; ++bx)
      tma_load_2d(bufQ(set) + (1 + (bx >> 1)) * kTileBytes + (bx & 1) * kBox, &map_state, &s->ld_state, 32 * bx, y);
  };

  // thread 32 issues every TMA load and bulk copy (and waits for the stores it
  // issued); thread 0 issues the MMAs
  constexpr int kProducer = 32;
  if (tid == kProducer && (int64_t)blockIdx.x < nitems) {
    prefetch_tmap(&map_state);
    const Item first = item_of(blockIdx.x, H, nseg);
    issue_loads(0, first, 0);
    issue_state_load(1, first);
  }

  constexpr uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t id_kn = idesc_bf16(128, 128, 0, 1);
  constexpr uint32_t id_nn = idesc_bf16(128, 128, 1, 1);
  uint32_t it = 0;  // tiles processed by this CTA
  uint32_t nseg_done = 0;  // segments started by this CTA
  bool stop = false;

  for (int64_t w = blockIdx.x; w < nitems && !stop; w += gridDim.x) {
    const Item item = item_of(w, H, nseg);
    const float lam = load_decay(decay, item.h);
    const float l2 = log2f(lam);
    const bool scale = lam != 1.0f;
    const float g_tile = decay_pow(l2, (float)kTile);
    if (tid < kTile) s->pw[tid] = decay_pow(l2, (float)tid);

    // entering state of the segment, loaded by TMA into the buffer set the
    // previous tile used (see issue_state_load): TMEM P and bf16 operand. Row i
    // of a swizzled box has its 16-byte chunk c at position c ^ (i & 7), so the
    // eight rows of a quarter-warp read different banks.
    if (mbar_wait(&s->ld_state, nseg_done & 1u, SITE_OUT_TMA)) {
      const uint8_t* src = bufQ((it & 1) ^ 1) + (1 + half) * kTileBytes;
      float v[64];
#pragma unroll
      for (int bb = 0; bb < 2; ++bb)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float4 x = *reinterpret_cast<const float4*>(src + bb * kBox + sw128_offset(i, c));
          v[bb * 32 + 4 * c] = x.x;
          v[bb * 32 + 4 * c + 1] = x.y;
          v[bb * 32 + 4 * c + 2] = x.z;
          v[bb * 32 + 4 * c + 3] = x.w;
        }
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t r[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(v[c2 * 32 + q]);
        tmem_st32(lane_base + TP + half * 64 + c2 * 32, r);
        st_row32_bf16(sP, i, half * 64 + c2 * 32, v + c2 * 32);
      }
      tmem_st_wait();
      fence_async_smem();
    } else {
      s->abort = 1;
    }
    ++nseg_done;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (s->abort) break;

    for (int t = 0; t < tiles; ++t, ++it) {
      const int set = it & 1;
      uint8_t* sQ = bufQ(set);
      uint8_t* sK = sQ + kTileBytes;
      uint8_t* sV = sQ + 2 * kTileBytes;
      const int row0 = item.seg * G + t * kTile;

      if (tid == kProducer) {
        // prefetch the next tile of this CTA's stream into the other set; its K
        // buffer is the source of the previous tile's output store
        Item nx = item;
        int nt = t + 1;
        bool has_next = true;
        if (nt == tiles) {
          nt = 0;
          has_next = w + gridDim.x < nitems;
          if (has_next) nx = item_of(w + gridDim.x, H, nseg);
        }
        if (has_next) {
          tma_store_wait_read0();
          issue_loads(set ^ 1, nx, nt);
        }
        if (t == (tiles > 1 ? tiles - 2 : 0) && w + gridDim.x < nitems) {
          // the next segment's entering state is read by all threads at the
          // segment switch; bring it into L2 while this segment's last tiles run
          const Item ns = item_of(w + gridDim.x, H, nseg);
          const int64_t slot = ((int64_t)ns.seg * G) / C;
          const float* src = P + (((int64_t)ns.b * T + slot) * H + ns.h) * kD * kD;
          bulk_prefetch_l2(src, kD * kD * sizeof(float));
        }
        if (cache_bf16) {
          // the bf16 operand tile of the state entering this chunk, as it sits
          // in shared memory, is the cache entry the backward pass loads back
          uint8_t* slot = reinterpret_cast<uint8_t*>(P + (((int64_t)item.b * T + row0 / C) * H + item.h) * kD * kD);
          bulk_store(slot, sP, kTileBytes);
          tma_store_commit();
        }
      }
      if (tid == 0) {
        // MMA 1: S = Q K^T, O_inter = Q P
        if (mbar_wait(&s->load[set], (it >> 1) & 1u, SITE_OUT_TMA)) {
          tc_fence_after();
          const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aP = smem_u32(sP);
          for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + TS, kmaj(aQ, kk), kmaj(aK, kk), id_kk, kk != 0);
          for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + TI, kmaj(aQ, kk), mnmaj(aP, kk), id_kn, kk != 0);
          mma_commit(&s->mma1);
        } else {
          s->abort = 1;
        }
      }

      // ---- epilogue A1: S' = Mask . S into the Q buffer (Q has been read by
      // both MMAs); the 32 x 32 blocks above the diagonal are zeros
      if (mbar_wait(&s->mma1, it & 1u, SITE_OUT_MMA)) {
        tc_fence_after();
#pragma unroll 1
        for (int cc = 2 * half; cc < 2 * half + 2; ++cc) {
          if (cc > (warp & 3)) {
#pragma unroll
            for (int q = 0; q < 4; ++q) st_tile16(sQ, i, cc * 32 + q * 8, make_uint4(0u, 0u, 0u, 0u));
            continue;
          }
          uint32_t r[32];
          tmem_ld32(lane_base + TS + cc * 32, r);
          tmem_ld_wait();
          float w32[32];
          if (cc < (warp & 3)) {
#pragma unroll
            for (int q = 0; q < 32; ++q) w32[q] = __uint_as_float(r[q]) * s->pw[i - cc * 32 - q];
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const int j = cc * 32 + q;
              w32[q] = j <= i ? __uint_as_float(r[q]) * s->pw[i - j] : 0.f;
            }
          }
          st_row32_bf16(sQ, i, cc * 32, w32);
        }
        fence_async_smem();
      } else {
        s->abort = 1;
      }
      tc_fence_before();
      __syncthreads();
      if (s->abort) {
        stop = true;
        break;
      }
      // ---- MMA 2a: O_intra = S' V (runs under epilogue A2)
      if (tid == 0) {
        tc_fence_after();
        const uint32_t aS = smem_u32(sQ), aV = smem_u32(sV);
        for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + TO, kmaj(aS, kk), mnmaj(aV, kk), id_kn, kk != 0);
        mma_commit(&s->mma2a);
      }

      // ---- epilogue A2: K~ = diag(lambda^{127-j}) K in place (K has been read
      // by the S MMA); the state entering this tile into the cache at chunk
      // starts (C > 128), then pre-scaled by lambda^128
      if (scale) {
        uint4* k4 = reinterpret_cast<uint4*>(sK);
#pragma unroll 2
        for (int g = tid; g < kTile * 16; g += kThreads) {
          const int r = (g & (kTile * 8 - 1)) >> 3;  // row of this 16-byte chunk in its box
          const float wk = s->pw[kTile - 1 - r];
          uint4 x = k4[g];
          x.x = scale_bf16x2(x.x, wk);
          x.y = scale_bf16x2(x.y, wk);
          x.z = scale_bf16x2(x.z, wk);
          x.w = scale_bf16x2(x.w, wk);
          k4[g] = x;
        }
      }
      {
        const bool write_cache = !cache_bf16 && t > 0 && (t * kTile) % C == 0;
        if (write_cache || scale) {
          float* dst = P + ((((int64_t)item.b * T + row0 / C) * H + item.h) * kD + i) * kD + half * 64;
          uint32_t r[2][32];
          tmem_ld32(lane_base + TP + half * 64, r[0]);
          tmem_ld32(lane_base + TP + half * 64 + 32, r[1]);
          tmem_ld_wait();
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            if (write_cache) {
              float4* d4 = reinterpret_cast<float4*>(dst + c2 * 32);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                __stcs(d4 + q, make_float4(__uint_as_float(r[c2][4 * q]), __uint_as_float(r[c2][4 * q + 1]),
                                           __uint_as_float(r[c2][4 * q + 2]), __uint_as_float(r[c2][4 * q + 3])));
            }
            if (scale) {
#pragma unroll
              for (int q = 0; q < 32; ++q) r[c2][q] = __float_as_uint(__uint_as_float(r[c2][q]) * g_tile);
              tmem_st32(lane_base + TP + half * 64 + c2 * 32, r[c2]);
            }
          }
          tmem_st_wait();
        }
      }
      fence_async_smem();
      if (tid == kProducer && cache_bf16) tma_store_wait_read0();  // epilogue B rewrites sP
      tc_fence_before();
      __syncthreads();
      // ---- MMA 2b: P += K~^T V (runs under epilogue B1)
      if (tid == 0) {
        tc_fence_after();
        const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
        for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + TP, mnmaj(aK, kk), mnmaj(aV, kk), id_nn, 1);
        mma_commit(&s->mma2);
      }

      // ---- epilogue B1: O = O_intra + lambda^{i+1} O_inter -> bf16 over S'
      // (which MMA 2a has read), for the TMA store
      if (mbar_wait(&s->mma2a, it & 1u, SITE_OUT_MMA)) {
        tc_fence_after();
        const float wi = decay_pow(l2, (float)(i + 1));
        uint32_t a0[32], e0[32], a1[32], e1[32];
        tmem_ld32(lane_base + TO + (2 * half) * 32, a0);
        tmem_ld32(lane_base + TI + (2 * half) * 32, e0);
        tmem_ld32(lane_base + TO + (2 * half + 1) * 32, a1);
        tmem_ld32(lane_base + TI + (2 * half + 1) * 32, e1);
        tmem_ld_wait();
        float o[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) o[q] = fmaf(wi, __uint_as_float(e0[q]), __uint_as_float(a0[q]));
        st_row32_bf16(sQ, i, 2 * half * 32, o);
#pragma unroll
        for (int q = 0; q < 32; ++q) o[q] = fmaf(wi, __uint_as_float(e1[q]), __uint_as_float(a1[q]));
        st_row32_bf16(sQ, i, (2 * half + 1) * 32, o);
      } else {
        s->abort = 1;
      }
      // ---- epilogue B2: P -> bf16 operand for the next tile
      if (mbar_wait(&s->mma2, it & 1u, SITE_OUT_MMA)) {
        tc_fence_after();
        // MMA 2b has read this set's K~ and V buffers: the next segment's
        // entering state goes there
        if (tid == kProducer && t == tiles - 1 && w + gridDim.x < nitems)
          issue_state_load(set, item_of(w + gridDim.x, H, nseg));
        uint32_t r0[32], r1[32];
        tmem_ld32(lane_base + TP + (2 * half) * 32, r0);
        tmem_ld32(lane_base + TP + (2 * half + 1) * 32, r1);
        tmem_ld_wait();
        float p[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) p[q] = __uint_as_float(r0[q]);
        st_row32_bf16(sP, i, 2 * half * 32, p);
#pragma unroll
        for (int q = 0; q < 32; ++q) p[q] = __uint_as_float(r1[q]);
        st_row32_bf16(sP, i, (2 * half + 1) * 32, p);
      } else {
        s->abort = 1;
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      if (s->abort) {
        stop = true;
        break;
      }
      if (tid == kProducer) {
        tma_store_4d(&map_o, sQ, 0, item.h, row0, item.b);
        tma_store_4d(&map_o, sQ + kBox, 64, item.h, row0, item.b);
        tma_store_commit();
      }
    }
  }
  if (tid == kProducer) tma_store_wait0();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc_fwd_walk_detail

bool tc_fwd_walk_ok(int dtype, int d, int64_t C) {
  return dtype == LASP_BF16 && d == tc_fwd_walk_detail::kD && C % tc_fwd_walk_detail::kTile == 0;
}

int walk_segment_tokens(int64_t N, int C) {
  // about 1024 tokens per segment: enough tiles per walk to hide the segment's
  // first load, enough segments to spread over the SMs
  int m = C >= 1024 ? 1 : 1024 / C;
  while (m > 1 && N % ((int64_t)C * m) != 0) --m;
  return C * m;
}

cudaError_t tc_fwd_walk(const void* q, const void* k, const void* v, const float* decay, float* P, void* o, int B,
                        int H, int64_t N, int d, int C, int G, int num_sms, cudaStream_t st) {
  using namespace tc_fwd_walk_detail;
  CUtensorMap mq, mk, mv, mo, mp;
  if (!make_token_map(&mq, q, B, H, N, d, kTile) || !make_token_map(&mk, k, B, H, N, d, kTile) ||
      !make_token_map(&mv, v, B, H, N, d, kTile) || !make_token_map(&mo, o, B, H, N, d, kTile) ||
      !make_state_map(&mp, P, (int64_t)B * (N / C) * H, d))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + 7 * (size_t)kTileBytes + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(fwd_walk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int nseg = (int)(N / G);
  const int64_t nitems = (int64_t)B * H * nseg;
  const unsigned grid = (unsigned)std::min<int64_t>(nitems, num_sms);
  // with C = 128 the backward walk reads the cache: it gets each chunk's state
  // as the bf16 operand tile; otherwise the cache holds fp32 states
  const int cache_bf16 = C == kTile ? 1 : 0;
  fwd_walk_tc<<<grid, kThreads, smem, st>>>(mq, mk, mv, mo, mp, decay, P, H, (int)(N / C), C, G, nseg, nitems,
                                           cache_bf16);
  return cudaGetLastError();
}

}  // namespace lasp
