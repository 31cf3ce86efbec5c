// Backward pass over segments with the gradient state kept on chip: the
// mirror of the forward walk (LASP Algorithm 3 steps 12-20, dKV_t =
// lambda^C dKV_{t+1} + (Lambda Q_t)^T dO_t, walked from the last chunk to the
// first; LASP-2 review, "Core claim": suffix over the gradient states),
// bf16, d = 128, chunk C = 128 = one tile.
//
// Before this kernel, the segment gradient states and an exclusive suffix
// over them put, in the R slot of each segment's last chunk, the gradient
// state entering that chunk from the tokens after the segment. One persistent
// CTA per SM takes segments in turn and walks their chunks backward, holding R
// (fp32) in TMEM; P of each chunk comes from the forward walk's cache as a
// ready bf16 operand tile. Per chunk c (LASP Eq. 14-23), with the MMAs issued
// by one warp and the epilogues run by eight others:
//
//   MMA 1:  T0 = dO V^T,  T1 = Q K^T  | T2 = dO P^T
//   epi 1:  dP' = Mask . T0 -> A,  S' = Mask . T1 -> B
//   MMA 2:  T0 = dP' K                 | T1 = S'^T dO
//   epi 2:  (under MMA 2) V <- diag(lambda^{127-j}) V;  R -> bf16 X (replacing
//           P), R <- lambda^128 R in TMEM;  dQ = T0 + lambda^{i+1} T2 -> over S'
//           (TMA store)
//   MMA 3:  T0 = V~ R^T,  T2 = K R    | T0 += dP'^T Q (dK)
//   epi 3:  (under MMA 3) dO <- diag(lambda^{j+1}) dO;
//   MMA 4:  R += Q^T dO~               (the state for chunk c - 1)
//   epi 3:  dK = T0, dV = T1 + lambda^{127-j} T2 -> over Q and dO~ (TMA stores)
//
// A bar marks a commit the epilogue can start on while the rest runs.
//
// The decay of the dK inter term rides on the bf16 operand V~ so both dK terms
// share an accumulator (TMEM has no fifth block); the dQ and dV inter terms
// keep fp32 row scalings. Two pairs of tile buffers trade roles from chunk to
// chunk: one holds the chunk's Q and dO and then its outgoing dK and dV, the
// other its dP' and S' (and dQ) and then the next chunk's Q and dO, which are
// loaded as soon as dQ has left and dP'^T Q is done, followed by P's cache
// tile; the next K and V go in once the first part of MMA 3 is done. R is not
// stored per chunk: only the segment-level slots of the workspace are used. In every epilogue warp w owns TMEM lanes
// (rows) 32*(w%4).. and the column half w/4.
#include <algorithm>

#include "kernels.h"
#include "lasp_common.cuh"
#include "sm100.cuh"
#include "tc_kernels.h"
#include "tma_host.h"

namespace lasp {
namespace tc_bwd_walk_detail {

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
constexpr uint32_t T0 = 0, T1 = 128, T2 = 256, TR = 384;

struct Smem {
  uint64_t ld_kv, ld_qd, ld_p, ld_r;  // TMA -> MMA warp / epilogue
  uint64_t c1, c1b, c2, c2b, c3a, c3, c4;  // MMA commits -> epilogue / producer
  uint64_t e1, e2, e3a, e0;  // epilogue -> MMA warp (256 arrivals each)
  uint64_t e2q;              // epilogue -> producer: dQ staged (256 arrivals)
  uint64_t staged;           // epilogue -> producer: dK, dV staged (256 arrivals)
  uint64_t free_a, free_b;   // producer -> epilogue: the previous dK / dV stores have read the buffer
  uint32_t tmem_base;
  int abort;
  float pw[kTile];
};

__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t x, float w) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&x);
  float2 f = __bfloat1622float2(h);
  return pack_bf16(f.x * w, f.y * w);
}
__device__ __forceinline__ void st_row32_bf16(uint8_t* tile, int row, int col, const float* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    st_tile16(tile, row, col + q * 8,
              make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                         pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7])));
}

// Scales row r of a 128 x 128 bf16 tile by w[r] (w indexed through `pw` with
// `flip`: w = pw[flip ? 127 - r : r] * post), in place; all threads.
__device__ __forceinline__ void scale_rows(uint8_t* tile, const float* pw, bool flip, float post, int tid) {
  uint4* t4 = reinterpret_cast<uint4*>(tile);
#pragma unroll 2
  for (int g = tid; g < kTile * 16; g += kEpiThreads) {
    const int r = (g & (kTile * 8 - 1)) >> 3;
    const float w = pw[flip ? kTile - 1 - r : r] * post;
    uint4 x = t4[g];
    x.x = scale_bf16x2(x.x, w);
    x.y = scale_bf16x2(x.y, w);
    x.z = scale_bf16x2(x.z, w);
    x.w = scale_bf16x2(x.w, w);
    t4[g] = x;
  }
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

__global__ void __launch_bounds__(kThreads, 1) bwd_walk_tc(
    const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_do,
    const __grid_constant__ CUtensorMap map_dq, const __grid_constant__ CUtensorMap map_dk,
    const __grid_constant__ CUtensorMap map_dv,
    const __grid_constant__ CUtensorMap map_state, const float* decay, const float* __restrict__ P,
    float* __restrict__ R, int H, int64_t N, int T, int C, int G, int nseg,
    int64_t nitems, int64_t item0) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sK = base + 1 * kTileBytes;
  uint8_t* sV = base + 2 * kTileBytes;
  uint8_t* sX = base + 4 * kTileBytes;  // P, then R (bf16)
  // two buffer pairs trade roles from chunk to chunk: one holds the chunk's Q
  // and dO (and, once MMA 4 has read them, its dK and dV on their way out), the
  // other dP' and S' (and, once MMA 3 has read those, the next chunk's Q and dO)
  // (pair 0: buffers 0 and 3; pair 1: buffers 5 and 6)
  auto pair = [&](uint32_t p, int m) { return base + (p ? 5 + m : 3 * m) * kTileBytes; };
  Smem* s = reinterpret_cast<Smem*>(base + 7 * kTileBytes);
  const volatile int* abort_flag = &s->abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tiles = G / kTile;

  if (tid == 0) {
    prefetch_tmap(&map_q);
    prefetch_tmap(&map_k);
    prefetch_tmap(&map_v);
    prefetch_tmap(&map_do);
    prefetch_tmap(&map_state);
    mbar_init(&s->ld_kv, 1);
    mbar_init(&s->ld_qd, 1);
    mbar_init(&s->ld_p, 1);
    mbar_init(&s->ld_r, 1);
    mbar_init(&s->c1, 1);
    mbar_init(&s->c1b, 1);
    mbar_init(&s->c2, 1);
    mbar_init(&s->c2b, 1);
    mbar_init(&s->c3a, 1);
    mbar_init(&s->c3, 1);
    mbar_init(&s->c4, 1);
    mbar_init(&s->e1, kEpiThreads);
    mbar_init(&s->e2, kEpiThreads);
    mbar_init(&s->e2q, kEpiThreads);
    mbar_init(&s->e3a, kEpiThreads);
    mbar_init(&s->e0, kEpiThreads);
    mbar_init(&s->staged, kEpiThreads);
    mbar_init(&s->free_a, 1);
    mbar_init(&s->free_b, 1);
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
      // the forward's cached bf16 tile of the state entering the tile at row
      // `row` of the sequence: in the slot of the tile's first chunk, the
      // second half of that slot for the second tile of a 256-token chunk
      auto ptile = [&](const Item& it, int64_t row) {
        const int half_of_chunk = C > kTile ? (int)((row / kTile) % (C / kTile)) : 0;
        return reinterpret_cast<const uint8_t*>(P + (((int64_t)it.b * T + row / C) * H + it.h) * kD * kD) +
               (size_t)half_of_chunk * kTileBytes;
      };
      auto load_kv = [&](const Item& it, int t) {
        const int row = it.seg * G + t * kTile;
        mbar_arrive_expect_tx(&s->ld_kv, 2 * kTileBytes);
        tma_load_4d(sK, &map_k, &s->ld_kv, 0, it.h, row, it.b);
        tma_load_4d(sK + kBox, &map_k, &s->ld_kv, 64, it.h, row, it.b);
        tma_load_4d(sV, &map_v, &s->ld_kv, 0, it.h, row, it.b);
        tma_load_4d(sV + kBox, &map_v, &s->ld_kv, 64, it.h, row, it.b);
      };
      auto load_qd = [&](const Item& it, int t, uint32_t p) {
        const int row = it.seg * G + t * kTile;
        uint8_t* q = pair(p, 0);
        uint8_t* d = pair(p, 1);
        mbar_arrive_expect_tx(&s->ld_qd, 2 * kTileBytes);
        tma_load_4d(q, &map_q, &s->ld_qd, 0, it.h, row, it.b);
        tma_load_4d(q + kBox, &map_q, &s->ld_qd, 64, it.h, row, it.b);
        tma_load_4d(d, &map_do, &s->ld_qd, 0, it.h, row, it.b);
        tma_load_4d(d + kBox, &map_do, &s->ld_qd, 64, it.h, row, it.b);
      };
      // P of a chunk: the forward walk stored it in the chunk's cache slot as the
      // bf16 operand tile (128-byte swizzled), so it is copied into X as is
      auto load_p = [&](const Item& it, int t) {
        mbar_arrive_expect_tx(&s->ld_p, kTileBytes);
        bulk_load(sX, ptile(it, (int64_t)it.seg * G + (int64_t)t * kTile), kTileBytes, &s->ld_p);
      };
      // one bulk group per tensor, so that the dK buffer frees up first
      auto store_tile = [&](const CUtensorMap* map, const uint8_t* src, const Item& it, int row0) {
        tma_store_4d(map, src, 0, it.h, row0, it.b);
        tma_store_4d(map, src + kBox, 64, it.h, row0, it.b);
        tma_store_commit();
      };

      if ((int64_t)blockIdx.x < nitems) {
        const Item first = item_of(item0 + blockIdx.x, H, nseg);
        load_kv(first, tiles - 1);
        load_qd(first, tiles - 1, 0);
        load_p(first, tiles - 1);
      }
      uint32_t it = 0;
      Item prev{0, 0, 0};
      int prev_row = 0;
      bool ok = true;
      for (int64_t w = blockIdx.x; w < nitems && ok; w += gridDim.x) {
        const Item item = item_of(item0 + w, H, nseg);
        for (int t = tiles - 1; t >= 0 && ok; --t, ++it) {
          const uint32_t par = it & 1u;
          const int row0 = item.seg * G + t * kTile;
          // the previous chunk's dK and dV, staged over its Q and dO~, go out;
          // once they have been read, that pair is this chunk's dP'/S' pair
          if (it > 0) {
            if (!(ok = mbar_wait_or_abort(&s->staged, (it - 1) & 1u, SITE_BWD_TMA, abort_flag))) break;
            store_tile(&map_dk, pair(par ^ 1u, 0), prev, prev_row);
            store_tile(&map_dv, pair(par ^ 1u, 1), prev, prev_row);
            tma_store_wait_read1();
            mbar_arrive(&s->free_a);
          }
          tma_store_wait_read0();
          if (t == tiles - 1) {
            // R entering the segment's last chunk, as four 32-column fp32 boxes
            // into the dP'/S' pair; epilogue 1 moves it into TMEM
            const int64_t slot = (int64_t)(item.seg + 1) * (G / C) - 1;  // the segment's last chunk
            const int y = (int)((((int64_t)item.b * T + slot) * H + item.h) * kD);
            mbar_arrive_expect_tx(&s->ld_r, kD * kD * 4);
#pragma unroll
            for (int bx = 0; bx < 4; ++bx)
              tma_load_2d(pair(par ^ 1u, bx >> 1) + (bx & 1) * kBox, &map_state, &s->ld_r, 32 * bx, y);
          }
          if (it == 0) mbar_arrive(&s->free_a);
          mbar_arrive(&s->free_b);

          // the next chunk of this CTA's stream
          Item nx = item;
          int nt = t - 1;
          bool has_next = true;
          if (nt < 0) {
            has_next = w + gridDim.x < nitems;
            if (has_next) {
              nx = item_of(item0 + w + gridDim.x, H, nseg);
              nt = tiles - 1;
            }
          }
          if (has_next) {
            // into L2 now, so that the loads issued once this chunk's MMAs have
            // freed their buffers are short
            const int nrow = nx.seg * G + nt * kTile;
            tma_prefetch_4d(&map_q, 0, nx.h, nrow, nx.b);
            tma_prefetch_4d(&map_q, 64, nx.h, nrow, nx.b);
            tma_prefetch_4d(&map_do, 0, nx.h, nrow, nx.b);
            tma_prefetch_4d(&map_do, 64, nx.h, nrow, nx.b);
            tma_prefetch_4d(&map_k, 0, nx.h, nrow, nx.b);
            tma_prefetch_4d(&map_k, 64, nx.h, nrow, nx.b);
            tma_prefetch_4d(&map_v, 0, nx.h, nrow, nx.b);
            tma_prefetch_4d(&map_v, 64, nx.h, nrow, nx.b);
            bulk_prefetch_l2(ptile(nx, nrow), kTileBytes);
          }
          if (t == (tiles > 1 ? 1 : 0) && w + gridDim.x < nitems) {
            // and the next segment's entering R, read at the segment switch
            const Item ns = item_of(item0 + w + gridDim.x, H, nseg);
            const int64_t slot = (int64_t)(ns.seg + 1) * (G / C) - 1;
            bulk_prefetch_l2(R + (((int64_t)ns.b * T + slot) * H + ns.h) * kD * kD, kD * kD * sizeof(float));
          }
          // dQ, staged over S' (which MMA 2 has read), goes out
          if (!(ok = mbar_wait_or_abort(&s->e2q, par, SITE_BWD_TMA, abort_flag))) break;
          store_tile(&map_dq, pair(par ^ 1u, 1), item, row0);
          // K, V and X are free once the first part of MMA 3 is done; the next
          // Q and dO go into the dP'/S' pair once dP'^T Q has read dP' and dQ
          // has left
          if (!(ok = mbar_wait_or_abort(&s->c3a, par, SITE_BWD_MMA, abort_flag))) break;
          if (has_next) {
            load_kv(nx, nt);
          }
          if (!(ok = mbar_wait_or_abort(&s->c3, par, SITE_BWD_MMA, abort_flag))) break;
          tma_store_wait_read0();
          if (has_next) {
            load_qd(nx, nt, par ^ 1u);
            load_p(nx, nt);  // last: only the third GEMM of MMA 1 reads it
          }
          prev = item;
          prev_row = row0;
        }
      }
      if (ok && it > 0 && mbar_wait_or_abort(&s->staged, (it - 1) & 1u, SITE_BWD_TMA, abort_flag)) {
        store_tile(&map_dk, pair((it - 1) & 1u, 0), prev, prev_row);
        store_tile(&map_dv, pair((it - 1) & 1u, 1), prev, prev_row);
      }
      if (!ok) s->abort = 1;
      tma_store_wait0();
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t id_kn = idesc_bf16(128, 128, 0, 1);
      constexpr uint32_t id_nn = idesc_bf16(128, 128, 1, 1);
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aX = smem_u32(sX);
      uint32_t it = 0;
      bool ok = true;
      for (int64_t w = blockIdx.x; w < nitems && ok; w += gridDim.x) {
        for (int t = tiles - 1; t >= 0; --t, ++it) {
          const uint32_t par = it & 1u;
          const uint32_t aQ = smem_u32(pair(par, 0)), aD = smem_u32(pair(par, 1));
          const uint32_t aA = smem_u32(pair(par ^ 1u, 0)), aB = smem_u32(pair(par ^ 1u, 1));
          // MMA 1 needs this chunk's loads, and TMEM 0-2 drained by the previous epilogue 3
          ok = mbar_wait_or_abort(&s->ld_kv, par, SITE_BWD_TMA, abort_flag) &&
               mbar_wait_or_abort(&s->ld_qd, par, SITE_BWD_TMA, abort_flag) &&
               (it == 0 || mbar_wait_or_abort(&s->e0, (it - 1) & 1u, SITE_BWD_MMA, abort_flag));
          if (!ok) break;
          tc_fence_after();
          // ---- MMA 1: T0 = dO V^T, T1 = Q K^T | T2 = dO P^T (P's tile is loaded last)
          for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T0, kmaj(aD, kk), kmaj(aV, kk), id_kk, kk != 0);
          for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T1, kmaj(aQ, kk), kmaj(aK, kk), id_kk, kk != 0);
          mma_commit(&s->c1);
          if (!(ok = mbar_wait_or_abort(&s->ld_p, par, SITE_BWD_TMA, abort_flag))) break;
          tc_fence_after();
          for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T2, kmaj(aD, kk), kmaj(aX, kk), id_kk, kk != 0);
          mma_commit(&s->c1b);
          // ---- MMA 2: T0 = dP' K | T1 = S'^T dO
          if (!(ok = mbar_wait_or_abort(&s->e1, par, SITE_BWD_MMA, abort_flag))) break;
          tc_fence_after();
          for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + T0, kmaj(aA, kk), mnmaj(aK, kk), id_kn, kk != 0);
          mma_commit(&s->c2);
          for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + T1, mnmaj(aB, kk), mnmaj(aD, kk), id_nn, kk != 0);
          mma_commit(&s->c2b);
          // ---- MMA 3: T0 = V~ R^T, T2 = K R | T0 += dP'^T Q
          if (!(ok = mbar_wait_or_abort(&s->e2, par, SITE_BWD_MMA, abort_flag))) break;
          tc_fence_after();
          for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T0, kmaj(aV, kk), kmaj(aX, kk), id_kk, kk != 0);
          for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T2, kmaj(aK, kk), mnmaj(aX, kk), id_kn, kk != 0);
          mma_commit(&s->c3a);
          for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + T0, mnmaj(aA, kk), mnmaj(aQ, kk), id_nn, 1);
          mma_commit(&s->c3);
          // ---- MMA 4: R += Q^T dO~ (TMEM R was pre-scaled by lambda^128 in epilogue 1)
          if (!(ok = mbar_wait_or_abort(&s->e3a, par, SITE_BWD_MMA, abort_flag))) break;
          tc_fence_after();
          for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + TR, mnmaj(aQ, kk), mnmaj(aD, kk), id_nn, 1);
          mma_commit(&s->c4);
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
    uint32_t it = 0;
    uint32_t nseg_done = 0;  // segments started by this CTA
    for (int64_t w = blockIdx.x; w < nitems; w += gridDim.x) {
      if (named_sync_or(kEpiBar, kEpiThreads, bad)) break;  // every epilogue thread is past the last segment
      const Item item = item_of(item0 + w, H, nseg);
      const float lam = load_decay(decay, item.h);
      const float l2 = log2f(lam);
      const bool scale = lam != 1.0f;
      const float g_tile = decay_pow(l2, (float)kTile);
      if (tid < kTile) s->pw[tid] = decay_pow(l2, (float)tid);
      named_sync(kEpiBar, kEpiThreads);

      for (int t = tiles - 1; t >= 0; --t, ++it) {
        const uint32_t par = it & 1u;
        uint8_t* sQ = pair(par, 0);       // Q, then dK out
        uint8_t* sD = pair(par, 1);       // dO, then dV out
        uint8_t* sA = pair(par ^ 1u, 0);  // dP'
        uint8_t* sB = pair(par ^ 1u, 1);  // S'

        // ---- epilogue 1
        if (t == tiles - 1) {
          // the segment's entering R: dP'/S' pair -> TMEM R, once the previous
          // chunk's MMA 4 is done with TMEM R. Row i of a swizzled box has its
          // 16-byte chunk c at position c ^ (i & 7), so the eight rows of a
          // quarter-warp read different banks.
          wait(&s->ld_r, nseg_done & 1u, SITE_BWD_TMA);
          if (it > 0) wait(&s->c4, (it - 1) & 1u, SITE_BWD_MMA);
          tc_fence_after();
          const uint8_t* src = pair(par ^ 1u, half);
          uint32_t r[2][32];
#pragma unroll
          for (int bb = 0; bb < 2; ++bb)
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 x = *reinterpret_cast<const uint4*>(src + bb * kBox + sw128_offset(i, c));
              r[bb][4 * c] = x.x;
              r[bb][4 * c + 1] = x.y;
              r[bb][4 * c + 2] = x.z;
              r[bb][4 * c + 3] = x.w;
            }
          tmem_st32(lane_base + TR + half * 64, r[0]);
          tmem_st32(lane_base + TR + half * 64 + 32, r[1]);
          tmem_st_wait();
          ++nseg_done;
          named_sync(kEpiBar, kEpiThreads);  // all of R is read before the pair is rewritten
        }
        // dP' = Mask . T0 and S' = Mask . T1 into the buffers the previous
        // chunk's dK and dV stores have left
        wait(&s->free_a, par, SITE_BWD_TMA);
        wait(&s->free_b, par, SITE_BWD_TMA);
        wait(&s->c1, par, SITE_BWD_MMA);
        tc_fence_after();
#pragma unroll 1
        for (int cc = 2 * half; cc < 2 * half + 2; ++cc) {
          if (cc > (warp & 3)) {
            // the 32 x 32 block lies above the diagonal of this warp's rows
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              st_tile16(sA, i, cc * 32 + q * 8, make_uint4(0u, 0u, 0u, 0u));
              st_tile16(sB, i, cc * 32 + q * 8, make_uint4(0u, 0u, 0u, 0u));
            }
            continue;
          }
          uint32_t rp[32], rs[32];
          tmem_ld32(lane_base + T0 + cc * 32, rp);
          tmem_ld32(lane_base + T1 + cc * 32, rs);
          tmem_ld_wait();
          float fp[32], fs[32];
          if (cc < (warp & 3)) {
            // below the diagonal (every j < i): lambda^{i-j} from the smallest
            // power up, one multiplication by lambda per column
            float wgt = s->pw[i - cc * 32 - 31];
#pragma unroll
            for (int q = 31; q >= 0; --q) {
              fp[q] = __uint_as_float(rp[q]) * wgt;
              fs[q] = __uint_as_float(rs[q]) * wgt;
              wgt *= lam;
            }
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const int j = cc * 32 + q;
              const float wgt = j <= i ? s->pw[i - j] : 0.f;
              fp[q] = __uint_as_float(rp[q]) * wgt;
              fs[q] = __uint_as_float(rs[q]) * wgt;
            }
          }
          st_row32_bf16(sA, i, cc * 32, fp);
          st_row32_bf16(sB, i, cc * 32, fs);
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&s->e1);

        // while MMA 2 runs: V~ = diag(lambda^{127-j}) V (MMA 1 has read V), and R
        // of this chunk -> bf16 X (once dO P^T has read P), pre-scaled by
        // lambda^128 for MMA 4
        if (scale) scale_rows(sV, s->pw, true, 1.f, tid);
        wait(&s->c1b, par, SITE_BWD_MMA);
        tc_fence_after();
        {
          uint32_t r[2][32];
          tmem_ld32(lane_base + TR + half * 64, r[0]);
          tmem_ld32(lane_base + TR + half * 64 + 32, r[1]);
          tmem_ld_wait();
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            float f[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) f[q] = __uint_as_float(r[c2][q]);
            st_row32_bf16(sX, i, half * 64 + c2 * 32, f);
            if (scale) {
#pragma unroll
              for (int q = 0; q < 32; ++q) r[c2][q] = __float_as_uint(f[q] * g_tile);
              tmem_st32(lane_base + TR + half * 64 + c2 * 32, r[c2]);
            }
          }
        }
        tmem_st_wait();

        // ---- epilogue 2: dQ = T0 + lambda^{i+1} T2, staged over S' once
        // S'^T dO has read it (the TMA warp stores it)
        wait(&s->c2, par, SITE_BWD_MMA);
        tc_fence_after();
        {
          const float wi = decay_pow(l2, (float)(i + 1));
          uint32_t pq[2][16];
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            uint32_t ra[32], re[32];
            tmem_ld32(lane_base + T0 + (2 * half + c2) * 32, ra);
            tmem_ld32(lane_base + T2 + (2 * half + c2) * 32, re);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 16; ++q)
              pq[c2][q] = pack_bf16(fmaf(wi, __uint_as_float(re[2 * q]), __uint_as_float(ra[2 * q])),
                                    fmaf(wi, __uint_as_float(re[2 * q + 1]), __uint_as_float(ra[2 * q + 1])));
          }
          // TMEM 0 and 2 are read and X holds R: MMA 3 may start
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(&s->e2);
          wait(&s->c2b, par, SITE_BWD_MMA);
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
            for (int q = 0; q < 4; ++q)
              st_tile16(sB, i, (2 * half + c2) * 32 + q * 8,
                        make_uint4(pq[c2][4 * q], pq[c2][4 * q + 1], pq[c2][4 * q + 2], pq[c2][4 * q + 3]));
        }
        fence_async_smem();
        mbar_arrive(&s->e2q);

        // ---- epilogue 3a: dO~ = diag(lambda^{j+1}) dO (S'^T dO has read dO), while MMA 3 runs
        if (scale) {
          scale_rows(sD, s->pw, false, lam, tid);  // lambda^{j+1} = pw[j] * lambda
          fence_async_smem();
        }
        mbar_arrive(&s->e3a);

        // ---- epilogue 3b: dK = T0, dV = T1 + lambda^{127-j} T2, staged over
        // Q and dO~ once MMA 4 has read them
        wait(&s->c3, par, SITE_BWD_MMA);
        tc_fence_after();
        {
          const float wj = decay_pow(l2, (float)(kTile - 1 - i));  // dV inter decay of row j = i
          uint32_t pk[2][16], pv[2][16];  // bf16 pairs of dK and dV, held until MMA 4 is done
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            uint32_t ka[32], va[32], ve[32];
            tmem_ld32(lane_base + T0 + (2 * half + c2) * 32, ka);
            tmem_ld32(lane_base + T1 + (2 * half + c2) * 32, va);
            tmem_ld32(lane_base + T2 + (2 * half + c2) * 32, ve);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              pk[c2][q] = pack_bf16(__uint_as_float(ka[2 * q]), __uint_as_float(ka[2 * q + 1]));
              pv[c2][q] = pack_bf16(fmaf(wj, __uint_as_float(ve[2 * q]), __uint_as_float(va[2 * q])),
                                    fmaf(wj, __uint_as_float(ve[2 * q + 1]), __uint_as_float(va[2 * q + 1])));
            }
          }
          tc_fence_before();
          mbar_arrive(&s->e0);  // TMEM 0-2 are free for the next chunk's MMA 1
          wait(&s->c4, par, SITE_BWD_MMA);
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int col = (2 * half + c2) * 32 + q * 8;
              st_tile16(sQ, i, col, make_uint4(pk[c2][4 * q], pk[c2][4 * q + 1], pk[c2][4 * q + 2], pk[c2][4 * q + 3]));
              st_tile16(sD, i, col, make_uint4(pv[c2][4 * q], pv[c2][4 * q + 1], pv[c2][4 * q + 2], pv[c2][4 * q + 3]));
            }
        }
        fence_async_smem();
        mbar_arrive(&s->staged);
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

}  // namespace tc_bwd_walk_detail

bool tc_bwd_walk_ok(int dtype, int d, int64_t C, int64_t N) {
  // chunks that divide the 128-token tile, or of two tiles: the forward walk
  // leaves the bf16 operand tile of each tile's entering state in the slot of
  // its first chunk (C = 256: the two tiles of a chunk in the two halves of its
  // 64 KB slot)
  using tc_bwd_walk_detail::kTile;
  if (dtype != LASP_BF16 || d != tc_bwd_walk_detail::kD || C < 1) return false;
  if (C == 2 * kTile) return N % C == 0;
  return C <= kTile && kTile % C == 0 && N % kTile == 0;
}

cudaError_t tc_bwd_walk(const void* q, const void* k, const void* v, const void* dout, const float* decay,
                        const float* P, float* R, void* dq, void* dk, void* dv, int B, int H, int64_t N, int d, int C,
                        int G, int num_sms, cudaStream_t st, int64_t bh0, int64_t nbh) {
  using namespace tc_bwd_walk_detail;
  CUtensorMap mq, mk, mv, mdo, mdq, mdk, mdv, mr;
  if (!make_token_map(&mq, q, B, H, N, d, kTile) || !make_token_map(&mk, k, B, H, N, d, kTile) ||
      !make_token_map(&mv, v, B, H, N, d, kTile) || !make_token_map(&mdo, dout, B, H, N, d, kTile) ||
      !make_token_map(&mdq, dq, B, H, N, d, kTile) || !make_token_map(&mdk, dk, B, H, N, d, kTile) ||
      !make_token_map(&mdv, dv, B, H, N, d, kTile) ||
      !make_state_map(&mr, R, (int64_t)B * (N / C) * H, d))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + 7 * (size_t)kTileBytes + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(bwd_walk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int nseg = (int)(N / G);
  // the segments of (b, h) pairs bh0 .. bh0 + nbh - 1 (items in b, h, segment order)
  if (nbh < 0) nbh = (int64_t)B * H;
  const int64_t nitems = nbh * nseg;
  if (nitems == 0) return cudaSuccess;
  const unsigned grid = (unsigned)std::min<int64_t>(nitems, num_sms);
  bwd_walk_tc<<<grid, kThreads, smem, st>>>(mq, mk, mv, mdo, mdq, mdk, mdv, mr, decay, P, R, H, N, (int)(N / C), C, G,
                                            nseg, nitems, bh0 * nseg);
  return cudaGetLastError();
}

}  // namespace lasp
