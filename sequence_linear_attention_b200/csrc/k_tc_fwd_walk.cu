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
// Here one persistent CTA per SM takes segments in turn and walks their
// 128-token tiles in order, holding the state P (fp32) in TMEM. One warp issues
// the MMAs, one the TMA loads and stores, eight run the epilogues; they hand
// work to each other through mbarriers. Per tile:
//
//   MMA 1:  S = Q K^T (TMEM S)  | O_inter = Q P_bf16 (TMEM I)
//   epi A1: S' = Mask . S -> bf16 over Q (once both parts of MMA 1 have read Q)
//   MMA 2a: O_intra = S' V (TMEM O), under
//   epi A2: K~ = diag(lambda^{127-j}) K in place; P <- lambda^128 P in TMEM (and,
//           for C > 256, P -> fp32 cache at chunk starts)
//   MMA 2b: P += K~^T V (TMEM P), under
//   epi B1: O = O_intra + lambda^{i+1} O_inter -> bf16 over S' -> TMA store
//   epi B2: P -> bf16 operand for the next tile
//
// With C = 128 each tile starts a chunk, and the bf16 operand tile of the
// entering state (already in shared memory for O_inter) goes to the chunk's
// cache slot by one bulk copy; the backward walk loads it back as is. Shorter
// chunks use the slot of the tile's first chunk; C = 256 puts the two tiles of
// a chunk in the two halves of its slot. Two sets
// of Q/K/V buffers alternate: while a tile is computed, the next tile's loads
// (possibly of the next segment) are in flight; a segment's fp32 entering state
// is loaded by TMA into the K and V buffers of the set the previous tile used.
// In every epilogue warp w owns TMEM lanes (rows) 32*(w%4).. and the column
// half w/4.
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
// warps 0-7 run the epilogues (warp w owns TMEM lanes 32*(w%4).. and column
// half w/4), warp 8 issues the MMAs, warp 9 the TMA loads and stores
constexpr int kEpiThreads = 256;
constexpr int kMmaWarp = 8;
constexpr int kProducerWarp = 9;
constexpr int kThreads = 320;
constexpr uint32_t kEpiBar = 1;  // named barrier of the epilogue warps
constexpr uint32_t kTileBytes = kTile * kD * 2;
constexpr uint32_t kBox = kTileBytes / 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t TS = 0, TI = 128, TO = 256, TP = 384;

struct Smem {
  uint64_t load[2], ld_state;            // TMA -> MMA warp / epilogue
  uint64_t mma1a, mma1, mma2a, mma2[2];  // MMA commits -> epilogue / producer (mma2 per buffer set)
  uint64_t e_a1, e_a2, e_b1[2], e_b2;    // epilogue -> MMA warp / producer (256 arrivals; e_b1 per set)
  uint64_t state_read;                   // epilogue -> producer: the entering state has been read
  uint64_t sp_free;                      // producer -> epilogue: P's operand tile is in the cache
  uint32_t tmem_base;
  int abort;
  float pw[kTile];
};

__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t x, float w) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&x);
  float2 f = __bfloat1622float2(h);
  return pack_bf16(f.x * w, f.y * w);
}

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
                                                            int cache_bf16, int64_t item0) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sP = base + 6 * kTileBytes;
  Smem* s = reinterpret_cast<Smem*>(base + 7 * kTileBytes);
  auto bufQ = [&](int set) { return base + set * 3 * kTileBytes; };
  const volatile int* abort_flag = &s->abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tiles = G / kTile;

  if (tid == 0) {
    prefetch_tmap(&map_q);
    prefetch_tmap(&map_k);
    prefetch_tmap(&map_v);
    prefetch_tmap(&map_o);
    prefetch_tmap(&map_state);
    mbar_init(&s->load[0], 1);
    mbar_init(&s->load[1], 1);
    mbar_init(&s->ld_state, 1);
    mbar_init(&s->mma1a, 1);
    mbar_init(&s->mma1, 1);
    mbar_init(&s->mma2a, 1);
    mbar_init(&s->mma2[0], 1);
    mbar_init(&s->mma2[1], 1);
    mbar_init(&s->e_a1, kEpiThreads);
    mbar_init(&s->e_a2, kEpiThreads);
    mbar_init(&s->e_b1[0], kEpiThreads);
    mbar_init(&s->e_b1[1], kEpiThreads);
    mbar_init(&s->e_b2, kEpiThreads);
    mbar_init(&s->state_read, kEpiThreads);
    mbar_init(&s->sp_free, 1);
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

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
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
      // 32-column boxes: boxes 0, 1 into the K buffer of `set`, boxes 2, 3 into
      // its V buffer
      auto issue_state_load = [&](int set, const Item& it) {
        const int64_t slot = ((int64_t)it.seg * G) / C;
        const int y = (int)((((int64_t)it.b * T + slot) * H + it.h) * kD);
        mbar_arrive_expect_tx(&s->ld_state, kD * kD * 4);
#pragma unroll
        for (int bx = 0; bx < 4; ++bx)
          tma_load_2d(bufQ(set) + (1 + (bx >> 1)) * kTileBytes + (bx & 1) * kBox, &map_state, &s->ld_state, 32 * bx,
                      y);
      };
      auto store_o = [&](int set, const Item& it, int row0) {
        tma_store_4d(&map_o, bufQ(set), 0, it.h, row0, it.b);
        tma_store_4d(&map_o, bufQ(set) + kBox, 64, it.h, row0, it.b);
        tma_store_commit();
      };

      if ((int64_t)blockIdx.x < nitems) {
        const Item first = item_of(item0 + blockIdx.x, H, nseg);
        issue_loads(0, first, 0);
        issue_state_load(1, first);
      }
      uint32_t it = 0, nsg = 0;
      Item prev{0, 0, 0};
      int prev_row = 0;
      bool ok = true;
      for (int64_t w = blockIdx.x; w < nitems && ok; w += gridDim.x) {
        const Item item = item_of(item0 + w, H, nseg);
        for (int t = 0; t < tiles && ok; ++t, ++it) {
          const int set = it & 1;
          const uint32_t par = it & 1u;
          const int row0 = item.seg * G + t * kTile;
          // the previous tile's O (staged over its S') goes out; once it has
          // been read, MMA 2 of that tile is done and (at a segment start) the
          // entering state has been read, its buffer set takes the next tile
          // (barriers kept per buffer set never run two phases ahead of a waiter:
          // their next phase needs the loads this thread issues after the wait)
          const uint32_t ppar = ((it - 1) >> 1) & 1u;  // phase of the previous tile's set
          if (it > 0) {
            if (!(ok = mbar_wait_or_abort(&s->e_b1[set ^ 1], ppar, SITE_OUT_TMA, abort_flag))) break;
            store_o(set ^ 1, prev, prev_row);
          }
          if (t == 0 && !(ok = mbar_wait_or_abort(&s->state_read, nsg & 1u, SITE_OUT_TMA, abort_flag))) break;
          if (t == 0) ++nsg;
          Item nx = item;
          int nt = t + 1;
          bool has_next = true;
          if (nt == tiles) {
            nt = 0;
            has_next = w + gridDim.x < nitems;
            if (has_next) nx = item_of(item0 + w + gridDim.x, H, nseg);
          }
          if (has_next) {
            if (it > 0 && !(ok = mbar_wait_or_abort(&s->mma2[set ^ 1], ppar, SITE_OUT_MMA, abort_flag))) break;
            tma_store_wait_read0();
            issue_loads(set ^ 1, nx, nt);
          }
          if (t == (tiles > 1 ? tiles - 2 : 0) && w + gridDim.x < nitems) {
            // the next segment's entering state, into L2 while this segment's
            // last tiles run
            const Item ns = item_of(item0 + w + gridDim.x, H, nseg);
            const int64_t slot = ((int64_t)ns.seg * G) / C;
            bulk_prefetch_l2(P + (((int64_t)ns.b * T + slot) * H + ns.h) * kD * kD, kD * kD * sizeof(float));
          }
          // the bf16 operand tile of the state entering this tile, as it sits in
          // shared memory, is the cache entry the backward pass loads back
          if (!(ok = mbar_wait_or_abort(&s->e_b2, par, SITE_OUT_TMA, abort_flag))) break;
          if (cache_bf16) {
            // in the slot of the tile's first chunk; with C = 256 one 64 KB slot
            // holds the tiles of both halves of its chunk
            const int half_of_chunk = C > kTile ? (row0 / kTile) % (C / kTile) : 0;
            uint8_t* slot = reinterpret_cast<uint8_t*>(P + (((int64_t)item.b * T + row0 / C) * H + item.h) * kD * kD) +
                            (size_t)half_of_chunk * kTileBytes;
            bulk_store(slot, sP, kTileBytes);
            tma_store_commit();
            tma_store_wait_read0();
          }
          mbar_arrive(&s->sp_free);
          // at the segment's last tile, once MMA 2 has read K~ and V, the next
          // segment's entering state goes there
          if (t == tiles - 1 && w + gridDim.x < nitems) {
            if (!(ok = mbar_wait_or_abort(&s->mma2[set], (it >> 1) & 1u, SITE_OUT_MMA, abort_flag))) break;
            issue_state_load(set, item_of(item0 + w + gridDim.x, H, nseg));
          }
          prev = item;
          prev_row = row0;
        }
      }
      if (ok && it > 0 && mbar_wait_or_abort(&s->e_b1[(it - 1) & 1], ((it - 1) >> 1) & 1u, SITE_OUT_TMA, abort_flag))
        store_o((it - 1) & 1, prev, prev_row);
      if (!ok) s->abort = 1;
      tma_store_wait0();
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t id_kn = idesc_bf16(128, 128, 0, 1);
      constexpr uint32_t id_nn = idesc_bf16(128, 128, 1, 1);
      const uint32_t aP = smem_u32(sP);
      uint32_t it = 0;
      bool ok = true;
      for (int64_t w = blockIdx.x; w < nitems && ok; w += gridDim.x) {
        for (int t = 0; t < tiles; ++t, ++it) {
          const int set = it & 1;
          const uint32_t par = it & 1u;
          const uint32_t aQ = smem_u32(bufQ(set)), aK = aQ + kTileBytes, aV = aQ + 2 * kTileBytes;
          // ---- MMA 1a: S = Q K^T (TMEM S was read by the previous epilogue A1)
          if (!(ok = mbar_wait_or_abort(&s->load[set], (it >> 1) & 1u, SITE_OUT_TMA, abort_flag))) break;
          tc_fence_after();
          for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + TS, kmaj(aQ, kk), kmaj(aK, kk), id_kk, kk != 0);
          mma_commit(&s->mma1a);
          // ---- MMA 1b: O_inter = Q P, once P is in shared memory and the
          // previous epilogue B1 has read TMEM I and O
          ok = (it == 0 || mbar_wait_or_abort(&s->e_b1[set ^ 1], ((it - 1) >> 1) & 1u, SITE_OUT_MMA, abort_flag)) &&
               mbar_wait_or_abort(&s->e_b2, par, SITE_OUT_MMA, abort_flag);
          if (!ok) break;
          tc_fence_after();
          for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + TI, kmaj(aQ, kk), mnmaj(aP, kk), id_kn, kk != 0);
          mma_commit(&s->mma1);
          // ---- MMA 2a: O_intra = S' V
          if (!(ok = mbar_wait_or_abort(&s->e_a1, par, SITE_OUT_MMA, abort_flag))) break;
          tc_fence_after();
          for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + TO, kmaj(aQ, kk), mnmaj(aV, kk), id_kn, kk != 0);
          mma_commit(&s->mma2a);
          // ---- MMA 2b: P += K~^T V (TMEM P pre-scaled by lambda^128 in epilogue A2)
          if (!(ok = mbar_wait_or_abort(&s->e_a2, par, SITE_OUT_MMA, abort_flag))) break;
          tc_fence_after();
          for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + TP, mnmaj(aK, kk), mnmaj(aV, kk), id_nn, 1);
          mma_commit(&s->mma2[set]);
        }
      }
      if (!ok) s->abort = 1;
    }
  } else {
    // ------------------------------------------------------------ epilogues
    const int i = (warp & 3) * 32 + lane;  // the row this thread owns
    const int half = warp >> 2;            // and the column half
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    bool bad = false;
    // a failed wait stops the other roles too; this thread runs on (on
    // whatever data) to the next point where all epilogue warps agree to stop
    auto wait = [&](uint64_t* bar, uint32_t parity, unsigned int site) {
      if (!bad && !mbar_wait_or_abort(bar, parity, site, abort_flag)) {
        bad = true;
        s->abort = 1;
      }
    };
    uint32_t it = 0, nsg = 0;
    for (int64_t w = blockIdx.x; w < nitems; w += gridDim.x) {
      if (named_sync_or(kEpiBar, kEpiThreads, bad)) break;  // every epilogue thread is past the last segment
      const Item item = item_of(item0 + w, H, nseg);
      const float lam = load_decay(decay, item.h);
      const float l2 = log2f(lam);
      const bool scale = lam != 1.0f;
      const float g_tile = decay_pow(l2, (float)kTile);
      if (tid < kTile) s->pw[tid] = decay_pow(l2, (float)tid);

      // entering state of the segment, loaded by TMA into the K and V buffers
      // of the set the previous tile used: TMEM P and the bf16 operand. Row i
      // of a swizzled box has its 16-byte chunk c at position c ^ (i & 7), so
      // the eight rows of a quarter-warp read different banks.
      wait(&s->ld_state, nsg & 1u, SITE_OUT_TMA);
      ++nsg;
      {
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
        tc_fence_after();
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          uint32_t r[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(v[c2 * 32 + q]);
          tmem_st32(lane_base + TP + half * 64 + c2 * 32, r);
          st_row32_bf16(sP, i, half * 64 + c2 * 32, v + c2 * 32);
        }
        tmem_st_wait();
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&s->state_read);
      mbar_arrive(&s->e_b2);  // P of the segment's first tile is in place
      named_sync(kEpiBar, kEpiThreads);  // the decay table is written

      for (int t = 0; t < tiles; ++t, ++it) {
        const int set = it & 1;
        const uint32_t par = it & 1u;
        uint8_t* sQ = bufQ(set);
        uint8_t* sK = sQ + kTileBytes;

        // ---- epilogue A1: S' = Mask . S over Q once both MMA 1 parts have read
        // Q; the 32 x 32 blocks above the diagonal are zeros
        wait(&s->mma1a, par, SITE_OUT_MMA);
        tc_fence_after();
        uint32_t ps[2][16];  // bf16 pairs of S'
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          const int cc = 2 * half + c2;
          if (cc > (warp & 3)) {
#pragma unroll
            for (int q = 0; q < 16; ++q) ps[c2][q] = 0u;
            continue;
          }
          uint32_t r[32];
          tmem_ld32(lane_base + TS + cc * 32, r);
          tmem_ld_wait();
          if (cc < (warp & 3)) {
            // below the diagonal (every j < i): lambda^{i-j} from the smallest
            // power up, one multiplication by lambda per column
            float wgt = s->pw[i - cc * 32 - 31];
#pragma unroll
            for (int q = 15; q >= 0; --q) {
              const float hi = __uint_as_float(r[2 * q + 1]) * wgt;
              wgt *= lam;
              const float lo = __uint_as_float(r[2 * q]) * wgt;
              wgt *= lam;
              ps[c2][q] = pack_bf16(lo, hi);
            }
          } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int j = cc * 32 + 2 * q;
              ps[c2][q] = pack_bf16(j <= i ? __uint_as_float(r[2 * q]) * s->pw[i - j] : 0.f,
                                    j + 1 <= i ? __uint_as_float(r[2 * q + 1]) * s->pw[i - j - 1] : 0.f);
            }
          }
        }
        tc_fence_before();
        wait(&s->mma1, par, SITE_OUT_MMA);
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_tile16(sQ, i, (2 * half + c2) * 32 + q * 8,
                      make_uint4(ps[c2][4 * q], ps[c2][4 * q + 1], ps[c2][4 * q + 2], ps[c2][4 * q + 3]));
        fence_async_smem();
        mbar_arrive(&s->e_a1);

        // ---- epilogue A2 (under MMA 2a): K~ = diag(lambda^{127-j}) K in place;
        // the state entering this tile into the cache at chunk starts (C > 128),
        // then pre-scaled by lambda^128
        if (scale) {
          uint4* k4 = reinterpret_cast<uint4*>(sK);
#pragma unroll 2
          for (int g = tid; g < kTile * 16; g += kEpiThreads) {
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
          const int row0 = item.seg * G + t * kTile;
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
        tc_fence_before();
        mbar_arrive(&s->e_a2);

        // ---- epilogue B1 (under MMA 2b): O = O_intra + lambda^{i+1} O_inter ->
        // bf16 over S' (which MMA 2a has read), stored by the TMA warp
        wait(&s->mma2a, par, SITE_OUT_MMA);
        tc_fence_after();
        {
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
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&s->e_b1[set]);

        // ---- epilogue B2: P -> bf16 operand for the next tile (the segment's
        // last tile leaves that to the next segment's entering state)
        wait(&s->mma2[set], (it >> 1) & 1u, SITE_OUT_MMA);
        tc_fence_after();
        wait(&s->sp_free, par, SITE_OUT_TMA);  // this tile's P has been copied to the cache
        if (t < tiles - 1) {
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
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(&s->e_b2);
        }
      }
    }
    if (named_sync_or(kEpiBar, kEpiThreads, bad) && tid == 0) s->abort = 1;
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc_fwd_walk_detail

bool tc_fwd_walk_ok(int dtype, int d, int64_t C, int64_t N) {
  // 128-token tiles: chunks that divide a tile or are made of whole tiles
  using tc_fwd_walk_detail::kTile;
  if (dtype != LASP_BF16 || d != tc_fwd_walk_detail::kD || C < 1) return false;
  const int64_t unit = C > kTile ? C : kTile;
  return (C % kTile == 0 || kTile % C == 0) && N % unit == 0;
}

int walk_segment_tokens(int64_t N, int C) {
  // about 1024 tokens per segment (a multiple of the tile and of the chunk):
  // enough tiles per walk to hide the segment's first load, enough segments to
  // spread over the SMs
  const int unit = C > tc_fwd_walk_detail::kTile ? C : tc_fwd_walk_detail::kTile;
  int m = unit >= 1024 ? 1 : 1024 / unit;
  while (m > 1 && N % ((int64_t)unit * m) != 0) --m;
  return unit * m;
}

cudaError_t tc_fwd_walk(const void* q, const void* k, const void* v, const float* decay, float* P, void* o, int B,
                        int H, int64_t N, int d, int C, int G, int num_sms, cudaStream_t st, int64_t bh0,
                        int64_t nbh) {
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
  // the segments of (b, h) pairs bh0 .. bh0 + nbh - 1 (items in b, h, segment order)
  if (nbh < 0) nbh = (int64_t)B * H;
  const int64_t nitems = nbh * nseg;
  if (nitems == 0) return cudaSuccess;
  const unsigned grid = (unsigned)std::min<int64_t>(nitems, num_sms);
  // with chunks that divide the tile, or of two tiles, the backward walk reads
  // the cache: it gets each tile's entering state as the bf16 operand tile (in
  // the slot of the tile's first chunk, two tiles to a slot when C = 256); with
  // longer chunks the cache holds fp32 states
  const int cache_bf16 = (C <= kTile || C == 2 * kTile) ? 1 : 0;
  fwd_walk_tc<<<grid, kThreads, smem, st>>>(mq, mk, mv, mo, mp, decay, P, H, (int)(N / C), C, G, nseg, nitems,
                                           cache_bf16, bh0 * nseg);
  return cudaGetLastError();
}

}  // namespace lasp
