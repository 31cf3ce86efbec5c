// Tensor-core kernels of the gated form (a decay per token and key feature;
// LASP Appendix A.4, Eq. 24 with the GLA / GateLoop row of Table 5), bf16,
// d = 128, over 128-token tiles. A tile spans 128/C chunks (C dividing 128);
// its masked products regroup the per-chunk intra and inter terms, so it
// follows the chunk equations of k_gla_simt.cu with the tile as the chunk
// (b_t = inclusive cumulative log-gate from the tile start, b_end its last
// row), the states being needed at tile boundaries only. The forward works on
// segments of tiles: the state kernel sums each segment's tiles into one
// state, and the output kernel walks each segment's tiles with the state in
// TMEM. The backward works on the same segments: one gradient state per
// segment, and a walk back through each segment's tiles that forms every
// tile's entering gradient state from the one after it.
//
// The intra-tile products need the factor e^{b_t[i] - b_s[i]} inside a
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
// half of the tile sum to at least -kMaxSpan. Each CTA checks this for its
// tile and records LASP_ERR_INVALID_ARG (site SITE_GATE_RANGE) if not; the
// CUDA-core kernels have no such limit.
//
// Thread layout (256 threads; 512 in the gradient kernel): warp w owns tile
// rows / TMEM lanes 32*(w%4).. and the column half (quarter) w/4 of every
// row-wise step. The cumulative log-gates:
// the state kernel sums them by 16-row groups (a warp per group, float4 loads)
// and scales its operand in place; the output and backward kernels load the
// gate tile by TMA and walk it in shared memory (a feature and half the rows
// per thread) before the row-wise steps read it.
#include <algorithm>

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
// the state kernel's bound on a half-tile's sum of |log-gate|: a little under
// kMaxSpan, so that no rounding of the two different sums lets a tile past it
// that the output and backward kernels would then reject
constexpr float kSpanCheck = kMaxSpan - 1.f;
constexpr uint32_t kBarAll = 1;   // named barrier over all threads of the CTA

// 2^x by the hardware's approximate exponential (relative error near 2^-22;
// results below 2^-126 flush to zero). Every exponent here is a difference of
// log-gate sums within the factorized range, or a gate factor at most 1.
__device__ __forceinline__ float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Orders this thread's generic-proxy writes to global memory before later
// async-proxy (bulk copy) reads of them.
__device__ __forceinline__ void fence_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }


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
      e[u] = pack_bf16(f.x * ex2a(sgn * x[c8 * 8 + 2 * u]), f.y * ex2a(sgn * x[c8 * 8 + 2 * u + 1]));
    }
    *p = w;
  }
}

// Element (t, i) of a [128][128] fp32 tile as the gate map's TMA loads lay it
// out: four 32-feature blocks of 128 lines of 128 bytes, 16-byte chunk c of
// line t at chunk c ^ (t % 8). A warp walking 32 features of one line and a
// warp reading float4s of 32 different lines both touch every bank once.
__device__ __forceinline__ int gate_slot(int t, int i) {
  return (i >> 5) * (kTile * 32) + t * 32 + 4 * (((i & 31) >> 2) ^ (t & 7)) + (i & 3);
}

// Feature i = tid % 128 over the rows of half tid / 128 of the tile (both
// halves at once, all 256 threads): the log-gates become sums from the half's
// first row, in place. Rows 0-63 then hold b_t; rows 64-127 hold b_t - r with
// r = b_63, the middle row. r goes to r[], the second half's total b_end - r
// to dend[].
__device__ __forceinline__ void walk_tile(float* bt, int tid, float* r, float* dend) {
  const int i = tid & (kD - 1), t1 = (tid >> 7) * (kTile / 2);
  float acc = 0.f;
#pragma unroll 1
  for (int t0 = t1; t0 < t1 + kTile / 2; t0 += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = bt[gate_slot(t0 + u, i)];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      acc += v[u];
      bt[gate_slot(t0 + u, i)] = acc;
    }
  }
  (t1 == 0 ? r : dend)[i] = acc;
}

// The 64 values of row t, columns half*64.., of such a tile.
__device__ __forceinline__ void read_gate_row(const float* bt, int t, int half, float (&b)[64]) {
#pragma unroll
  for (int cb = 0; cb < 2; ++cb)
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 v =
          *reinterpret_cast<const float4*>(bt + (2 * half + cb) * (kTile * 32) + t * 32 + 4 * (q ^ (t & 7)));
      b[cb * 32 + 4 * q] = v.x;
      b[cb * 32 + 4 * q + 1] = v.y;
      b[cb * 32 + 4 * q + 2] = v.z;
      b[cb * 32 + 4 * q + 3] = v.w;
    }
}

// Four TMA loads of the tile's log-gates (fp32, 64 KB) into the gate tile.
__device__ __forceinline__ void load_gate_tile(float* bt, const CUtensorMap* map_g, uint64_t* bar, int h, int row0,
                                               int b) {
  mbar_arrive_expect_tx(bar, kTile * kD * 4);
#pragma unroll
  for (int cb = 0; cb < 4; ++cb) tma_load_4d(bt + cb * (kTile * 32), map_g, bar, cb * 32, h, row0, b);
}

// ---------------------------------------------------------------- states
struct SmemStates {
  uint64_t load, mma;
  uint32_t tmem_base;
  int abort;
  alignas(16) float grp[8][kD];  // the log-gates of each feature summed over each 16-row group (float4 access)
  alignas(16) float grp_abs[8][kD];  // the same sums of |log-gate| (the span check)
};

// kind 0: M_c = (k . e^{b_end - b})^T v and gsum_c = b_end; kind 1: dM_c =
// (q . e^{b})^T do. x, y: the two token operands ((k, v) or (q, do)); the gate
// factor goes on x, scaled in place. Warp w takes rows 16w..16w+15, lane l
// features 4l..4l+3 (one 512-byte float4 row per warp-wide load): it sums its
// group's log-gates, the eight groups' sums give each group's offset, and a
// second pass over the loaded values (down for kind 1, up for kind 0:
// e^{b_end - b_t} = e^{sum_{r>t} g_r}) scales the tile.
//
// A CTA takes `tiles` consecutive tiles (a segment of the sequence, one state
// for all of them): kind 0 from the last tile to the first, kind 1 from the
// first to the last, each thread carrying the log-gate sum of its features
// over the tiles already done. That sum joins every factor of the next tile,
// so the tiles' products add up in one TMEM accumulator with no rescaling;
// every factor stays at most 1 for log-gates <= 0. gsum (kind 0, may be NULL)
// receives the item's total log-gate in the item's slot; gsum_tile (may be
// NULL) every tile's own total in the slot of tile c, c * tstride.
// kOne: one tile per CTA (tiles = 1 at compile time).
template <bool kOne>
__global__ void __launch_bounds__(kThreads, 2) gla_states_tc(const __grid_constant__ CUtensorMap map_x,
                                                             const __grid_constant__ CUtensorMap map_y,
                                                             const float* __restrict__ g, float* __restrict__ M,
                                                             float* __restrict__ gsum, float* __restrict__ gsum_tile,
                                                             int H, int64_t N, int kind, int64_t t_slots, int stride,
                                                             int offset, int tiles_arg, int tstride,
                                                             int* __restrict__ span_flag, RunIf run_if) {
  if (!runs(run_if)) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sX = base;
  uint8_t* sY = base + kTileBytes;
  SmemStates* s = reinterpret_cast<SmemStates*>(base + 2 * kTileBytes);
  const int tiles = kOne ? 1 : tiles_arg;
  const int item = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t sl = (int64_t)b * t_slots + (int64_t)item * stride + offset;  // the state slot of this item
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
  const int f0 = lane * 4;  // features f0..f0+3
  float4 off = make_float4(0.f, 0.f, 0.f, 0.f);  // log-gate sum of the tiles already done
  for (int j = 0; j < tiles; ++j) {
    const int64_t tile = (int64_t)item * tiles + (kind == 0 ? tiles - 1 - j : j);
    const int64_t row0 = tile * kTile;
    const uint32_t par = (uint32_t)j & 1u;
    if (tid == 0) {
      // the previous tile's MMA has read sX and sY (waited below)
      mbar_arrive_expect_tx(&s->load, 2 * kTileBytes);
      tma_load_4d(sX, &map_x, &s->load, 0, h, (int)row0, b);
      tma_load_4d(sX + kBox, &map_x, &s->load, 64, h, (int)row0, b);
      tma_load_4d(sY, &map_y, &s->load, 0, h, (int)row0, b);
      tma_load_4d(sY + kBox, &map_y, &s->load, 64, h, (int)row0, b);
    }
    const int64_t rs = (int64_t)H * kD;
    const float4* gp =
        reinterpret_cast<const float4*>(g + ((int64_t)b * N + row0 + warp * 16) * rs + (int64_t)h * kD + f0);
    float4 gv[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) gv[u] = __ldg(gp + (int64_t)u * (rs / 4));
    float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      tot.x += gv[u].x;
      tot.y += gv[u].y;
      tot.z += gv[u].z;
      tot.w += gv[u].w;
    }
    *reinterpret_cast<float4*>(&s->grp[warp][f0]) = tot;
    if (span_flag != nullptr) {
      float4 ab = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        ab.x += fabsf(gv[u].x);
        ab.y += fabsf(gv[u].y);
        ab.z += fabsf(gv[u].z);
        ab.w += fabsf(gv[u].w);
      }
      *reinterpret_cast<float4*>(&s->grp_abs[warp][f0]) = ab;
    }
    const bool ok = mbar_wait(&s->load, par, SITE_STATES_TMA);
    if (!ok) s->abort = 1;
    __syncthreads();
    // the part of the exponent from the other groups (kind 1 sums down from
    // row 0, kind 0 up from the last row) and from the tiles already done;
    // the tile's own total joins `off` for the next tile
    float4 acc = off, all = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int w2 = 0; w2 < 8; ++w2) {
      const float4 x = *reinterpret_cast<const float4*>(&s->grp[w2][f0]);
      all.x += x.x;
      all.y += x.y;
      all.z += x.z;
      all.w += x.w;
      if (kind == 0 ? w2 > warp : w2 < warp) {
        acc.x += x.x;
        acc.y += x.y;
        acc.z += x.z;
        acc.w += x.w;
      }
    }
    off.x += all.x;
    off.y += all.y;
    off.z += all.z;
    off.w += all.w;
    if (span_flag != nullptr && warp < 2) {
      // warp 0 the tile's first half, warp 1 its second: the sum of |g| over
      // a half bounds every |b_t - r| of that half in the factorized form of
      // the output and backward kernels (r = b at the middle row)
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int w2 = 4 * warp; w2 < 4 * warp + 4; ++w2) {
        const float4 x = *reinterpret_cast<const float4*>(&s->grp_abs[w2][f0]);
        a.x += x.x;
        a.y += x.y;
        a.z += x.z;
        a.w += x.w;
      }
      if (!(fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w)) <= kSpanCheck)) *span_flag = 1;
    }
    if (gsum_tile != nullptr && warp == 0)
      *reinterpret_cast<float4*>(gsum_tile + (((int64_t)b * t_slots + tile * tstride) * H + h) * kD + f0) = all;
    uint8_t* colp = sX + (f0 >> 6) * kBox + (f0 & 7) * 2;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      const int u = kind == 0 ? 15 - n : n;
      if (kind != 0) {
        acc.x += gv[u].x;
        acc.y += gv[u].y;
        acc.z += gv[u].z;
        acc.w += gv[u].w;
      }
      uint2* e = reinterpret_cast<uint2*>(colp + sw128_offset(warp * 16 + u, (f0 & 63) >> 3));
      if (ok) {
        uint2 w = *e;
        const float2 a = unpack_bf16(w.x), c2 = unpack_bf16(w.y);
        w.x = pack_bf16(a.x * ex2a(acc.x * kLog2e), a.y * ex2a(acc.y * kLog2e));
        w.y = pack_bf16(c2.x * ex2a(acc.z * kLog2e), c2.y * ex2a(acc.w * kLog2e));
        *e = w;
      }
      if (kind == 0) {
        acc.x += gv[u].x;
        acc.y += gv[u].y;
        acc.z += gv[u].z;
        acc.w += gv[u].w;
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();  // every thread has read grp and scaled its rows
    if (s->abort) goto cleanup;
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id_nn = idesc_bf16(128, 128, 1, 1);
      const uint32_t aX = smem_u32(sX), aY = smem_u32(sY);
      for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem, mnmaj(aX, kk), mnmaj(aY, kk), id_nn, kk != 0 || j > 0);
      mma_commit(&s->mma);
    }
    if (j + 1 < tiles) {
      // the MMA has read sX and sY before the next tile's loads go there
      if (!mbar_wait(&s->mma, par, SITE_STATES_MMA)) s->abort = 1;
      __syncthreads();
      if (s->abort) goto cleanup;
    }
  }
  // the item's total log-gate (kind 0): every warp holds it; warp 0 writes it
  if (kind == 0 && gsum != nullptr && warp == 0)
    *reinterpret_cast<float4*>(gsum + (sl * H + h) * kD + f0) = off;
  if (mbar_wait(&s->mma, (uint32_t)(tiles - 1) & 1u, SITE_STATES_MMA)) {
    tc_fence_after();
    // row i of M (TMEM lane i), columns half*64..
    const int i = (warp & 3) * 32 + lane, half = warp >> 2;
    float* out = M + ((sl * H + h) * kD + i) * kD + half * 64;
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

// Phase 0 of the output and backward kernels: once the gate tile has landed
// (barrier gbar, phase of the given parity), its walk (b at the middle row into r[], b_end - r into
// dend[]), then, for row t and column half `half` of every thread, the range
// check and x = (b_t - r) log2 e, returned in x[].
// Returns whether this thread's wait for the gate tile succeeded.
__device__ __forceinline__ bool gate_rows(float* bt, uint64_t* gbar, uint32_t parity, int* abort, unsigned int site,
                                          float* r, float* dend, int tid, int t, int half, float (&x)[64]) {
  const bool landed = mbar_wait(gbar, parity, site);
  if (!landed) *abort = 1;
  walk_tile(bt, tid, r, dend);
  named_sync(kBarAll, kThreads);
  read_gate_row(bt, t, half, x);
  const bool first = t < kTile / 2;  // rows of the second half already hold b_t - r
  bool ok = true;
#pragma unroll
  for (int u = 0; u < 64; ++u) {
    const float y = first ? x[u] - r[half * 64 + u] : x[u];
    ok = ok && fabsf(y) <= kMaxSpan;
    x[u] = y * kLog2e;
  }
  if (!ok) record_error(LASP_ERR_INVALID_ARG, SITE_GATE_RANGE);
  return landed;
}

// ---------------------------------------------------------------- output
// One persistent CTA per SM walks segments of `tiles` tiles (tiles = 1: every
// tile on its own, its entering state from the cache). At a segment's first
// tile the state P entering the segment arrives from the cache slot by TMA.
// Each tile then forms P' = diag(e^{r}) P, the bf16 operand of the inter term
// (also stored in the tile's cache slot for the backward) and, inside a
// segment, the fp32 accumulator in TMEM onto which the last MMA adds K^^T V.
// The next tile multiplies that accumulator by e^{b_end - r} of this tile,
// which gives its entering state. TMEM: T0 = Q^K^^T, T1 = the output,
// TP = the state.
struct SmemOut {
  uint64_t gload, load, ldp, mma1, mma2;
  uint32_t tmem_base;
  int abort;
  float r[kD], dend[kD];
};

__global__ void __launch_bounds__(kThreads, 1) gla_out_tc(const __grid_constant__ CUtensorMap map_q,
                                                          const __grid_constant__ CUtensorMap map_k,
                                                          const __grid_constant__ CUtensorMap map_v,
                                                          const __grid_constant__ CUtensorMap map_o,
                                                          const __grid_constant__ CUtensorMap map_g,
                                                          const __grid_constant__ CUtensorMap map_p,
                                                          float* __restrict__ P, int H, int64_t N,
                                                          int64_t t_slots, int stride, int ntx, int tiles,
                                                          int64_t nseg, RunIf run_if) {
  if (!runs(run_if)) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = base;                   // Q^
  uint8_t* sK = base + 1 * kTileBytes;  // K^
  uint8_t* sV = base + 2 * kTileBytes;
  uint8_t* sX = base + 3 * kTileBytes;  // P'
  uint8_t* sA = base + 4 * kTileBytes;  // A . causal, then O out
  float* bt = reinterpret_cast<float*>(base + 5 * kTileBytes);  // gate tile, 64 KB (then a segment's P)
  SmemOut* s = reinterpret_cast<SmemOut*>(base + 7 * kTileBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = (warp & 3) * 32 + lane, half = warp >> 2;
  const int spq = ntx / tiles;  // segments per sequence
  // segment sg: tiles cs * tiles .. of head h of sequence b, in launch order
  auto seg_of = [&](int64_t sg, int& cs, int& h, int& b) {
    cs = (int)(sg % spq);
    h = (int)((sg / spq) % H);
    b = (int)(sg / ((int64_t)spq * H));
  };
  // the cache slot of tile c (the slot of its first chunk)
  auto slot_of = [&](int c, int h, int b) { return ((int64_t)b * t_slots + (int64_t)c * stride) * H + h; };
  auto load_tokens = [&](int h, int row, int b) {
    mbar_arrive_expect_tx(&s->load, 3 * kTileBytes);
    tma_load_4d(sQ, &map_q, &s->load, 0, h, row, b);
    tma_load_4d(sQ + kBox, &map_q, &s->load, 64, h, row, b);
    tma_load_4d(sK, &map_k, &s->load, 0, h, row, b);
    tma_load_4d(sK + kBox, &map_k, &s->load, 64, h, row, b);
    tma_load_4d(sV, &map_v, &s->load, 0, h, row, b);
    tma_load_4d(sV + kBox, &map_v, &s->load, 64, h, row, b);
  };
  if (tid == 0) {
    prefetch_tmap(&map_q);
    prefetch_tmap(&map_k);
    prefetch_tmap(&map_v);
    prefetch_tmap(&map_o);
    prefetch_tmap(&map_g);
    prefetch_tmap(&map_p);
    mbar_init(&s->gload, 1);
    mbar_init(&s->load, 1);
    mbar_init(&s->ldp, 1);
    mbar_init(&s->mma1, 1);
    mbar_init(&s->mma2, 1);
    s->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s->tmem_base;
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  const uint32_t T0 = 0, T1 = 128, TP = 256;
  if (tid == 0 && (int64_t)blockIdx.x < nseg) {
    // the first tile's loads; a later tile's are issued during the tile before
    int cs, h, b;
    seg_of(blockIdx.x, cs, h, b);
    load_gate_tile(bt, &map_g, &s->gload, h, cs * tiles * kTile, b);
    bulk_prefetch_l2(P + slot_of(cs * tiles, h, b) * kD * kD, kD * kD * 4);  // loaded after the gate walk
    load_tokens(h, cs * tiles * kTile, b);
  }
  uint32_t ph = 0;            // parity of the per-tile barriers' phase for this CTA's current tile
  uint32_t pph = 0;           // parity of the P barrier (once per segment)
  // thread 0: the phase parity of a gate-tile / token-tile load in flight
  // (this tile's until its wait succeeds, then the next tile's once issued),
  // or -1; cleanup waits for it once more, so no load lands after the exit
  int gate_out = (tid == 0 && (int64_t)blockIdx.x < nseg) ? 0 : -1;
  int tok_out = gate_out;
  bool p_ahead = false;       // thread 0: P's load into the gate tile's space is in flight
  float dprev = 0.f;          // b_end - r of state row t in the tile before (inside a segment)
  for (int64_t sg = blockIdx.x; sg < nseg; sg += gridDim.x) {
  for (int j = 0; j < tiles; ++j, ph ^= 1u) {
  int cs, h, b;
  seg_of(sg, cs, h, b);
  const int c = cs * tiles + j;
  const int64_t row0 = (int64_t)c * kTile;
  float* Pc = P + slot_of(c, h, b) * kD * kD;
  // this CTA's next tile
  const int64_t sgn = j + 1 < tiles ? sg : sg + gridDim.x;
  const int jn = j + 1 < tiles ? j + 1 : 0;
  const bool has_next = sgn < nseg;
  float x[64];
  if (gate_rows(bt, &s->gload, ph, &s->abort, SITE_OUT_TMA, s->r, s->dend, tid, t, half, x) && tid == 0)
    gate_out = -1;
  named_sync(kBarAll, kThreads);  // every row of the gate tile has been read
  if (tid == 0 && j == 0 && !s->abort) {
    // the segment's entering state P (fp32) into the gate tile's space: four
    // boxes of 32 columns with the 128-byte swizzle, so that every thread
    // reads its own row without bank conflicts
    mbar_arrive_expect_tx(&s->ldp, kD * kD * 4);
    const int y = (int)(slot_of(c, h, b) * kD);
#pragma unroll
    for (int bx = 0; bx < 4; ++bx)
      tma_load_2d(reinterpret_cast<uint8_t*>(bt) + bx * (kTile * 128), &map_p, &s->ldp, 32 * bx, y);
    p_ahead = true;
  }
  // the factors of state row t: e^{(b_end - r) of the tile before} carries
  // the state from that tile into this one (after a segment's first tile),
  // then e^{r} makes P'. They are applied one after the other: each lies in
  // [e^{-80}, 1] (the range check bounds both half-tile sums), their product
  // need not be a normal fp32 number.
  const float wcarry = ex2a(dprev * kLog2e);
  const float wrow = ex2a(s->r[t] * kLog2e);
  const float dnext = s->dend[t];
  if (!mbar_wait(&s->load, ph, SITE_OUT_TMA))
    s->abort = 1;
  else if (tid == 0)
    tok_out = -1;
  scale_row_half(sQ, t, half, x, 1.f);   // Q^ = q . E
  scale_row_half(sK, t, half, x, -1.f);  // K^ = k / E
  fence_async_smem();
  tc_fence_before();
  __syncthreads();  // Q^ and K^ are in place
  if (s->abort) goto cleanup;
  {
    const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aX = smem_u32(sX), aA = smem_u32(sA);
    constexpr uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t id_kn = idesc_bf16(128, 128, 0, 1);
    constexpr uint32_t id_nn = idesc_bf16(128, 128, 1, 1);
    if (tid == 0) {
      tc_fence_after();
      for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T0, kmaj(aQ, kk), kmaj(aK, kk), id_kk, kk != 0);
      mma_commit(&s->mma1);
    }
    // under Q^ K^^T: P' = diag(e^{r}) P of row t (this thread's TMEM lane),
    // columns half * 64.., as bf16 into X and (inside a segment) as fp32 into
    // TMEM, where the state update accumulates onto it
    {
      float v[64];
      if (j == 0) {
        const bool pok = mbar_wait(&s->ldp, pph, SITE_OUT_TMA);
        if (pok) {
          pph ^= 1u;
          if (tid == 0) p_ahead = false;
        } else {
          s->abort = 1;  // cleanup waits for this phase once more
        }
        const uint8_t* src = reinterpret_cast<const uint8_t*>(bt) + 2 * half * (kTile * 128);
#pragma unroll
        for (int bb = 0; bb < 2; ++bb)
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const float4 q4 = *reinterpret_cast<const float4*>(src + bb * (kTile * 128) + sw128_offset(t, cc));
            v[bb * 32 + 4 * cc] = q4.x;
            v[bb * 32 + 4 * cc + 1] = q4.y;
            v[bb * 32 + 4 * cc + 2] = q4.z;
            v[bb * 32 + 4 * cc + 3] = q4.w;
          }
      } else {
        uint32_t r0[32], r1[32];
        tmem_ld32(lane_base + TP + half * 64, r0);
        tmem_ld32(lane_base + TP + half * 64 + 32, r1);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          v[u] = __uint_as_float(r0[u]);
          v[32 + u] = __uint_as_float(r1[u]);
        }
      }
      if (j > 0) {
#pragma unroll
        for (int u = 0; u < 64; ++u) v[u] *= wcarry;
      }
#pragma unroll
      for (int u = 0; u < 64; ++u) v[u] *= wrow;
      if (j + 1 < tiles) {
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          uint32_t r[32];
#pragma unroll
          for (int u = 0; u < 32; ++u) r[u] = __float_as_uint(v[c2 * 32 + u]);
          tmem_st32(lane_base + TP + half * 64 + c2 * 32, r);
        }
        tmem_st_wait();
      }
#pragma unroll
      for (int q8 = 0; q8 < 8; ++q8)
        *tile16(sX, t, half * 64 + q8 * 8) =
            make_uint4(pack_bf16(v[q8 * 8], v[q8 * 8 + 1]), pack_bf16(v[q8 * 8 + 2], v[q8 * 8 + 3]),
                       pack_bf16(v[q8 * 8 + 4], v[q8 * 8 + 5]), pack_bf16(v[q8 * 8 + 6], v[q8 * 8 + 7]));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();  // P' is in X; a segment's P has been read
    if (tid == 0 && !s->abort) {
      // P' as the bf16 operand tile goes to this tile's cache slot: the
      // backward loads it back as is
      bulk_store(Pc, sX, kTileBytes);
      tma_store_commit();
      if (has_next) {
        // the next tile's gates into the gate tile (and, at a segment start, its P into L2)
        int csn, hn, bn;
        seg_of(sgn, csn, hn, bn);
        load_gate_tile(bt, &map_g, &s->gload, hn, (csn * tiles + jn) * kTile, bn);
        if (jn == 0) bulk_prefetch_l2(P + slot_of(csn * tiles, hn, bn) * kD * kD, kD * kD * 4);
        gate_out = (int)(ph ^ 1u);
      }
      // the inter term does not wait for the mask
      tc_fence_after();
      for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T1, kmaj(aQ, kk), mnmaj(aX, kk), id_kn, kk != 0);
    }
    // A . causal -> sA (row t, column half)
    if (mbar_wait(&s->mma1, ph, SITE_OUT_MMA)) {
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
      // inside a segment, the state update onto P' in TMEM: + K^^T V (the next
      // tile's factor e^{b_end - r} turns K^ into k e^{b_end - b})
      if (j + 1 < tiles)
        for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + TP, mnmaj(aK, kk), mnmaj(aV, kk), id_nn, 1);
      mma_commit(&s->mma2);
    }
    // O -> sA (free once the MMA has read it) -> TMA store
    if (mbar_wait(&s->mma2, ph, SITE_OUT_MMA)) {
      tc_fence_after();
      if (tid == 0 && has_next) {
        // every MMA has read Q^, K^, V and P': the next tile's tokens go in
        int csn, hn, bn;
        seg_of(sgn, csn, hn, bn);
        load_tokens(hn, (csn * tiles + jn) * kTile, bn);
        tok_out = (int)(ph ^ 1u);
      }
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
    const bool stop = s->abort != 0;
    if (tid == 0 && !stop) {
      tma_store_4d(&map_o, sA, 0, h, (int)row0, b);
      tma_store_4d(&map_o, sA + kBox, 64, h, (int)row0, b);
      tma_store_commit();
      tma_store_wait_read0();  // sA is free for the next tile's mask
    }
    if (stop) goto cleanup;
  }
  dprev = dnext;
  }
  }
cleanup:
  // loads that an abort leaves unused (the current tile's, after a wait that
  // gave up, or the next tile's) land before the CTA exits (bounded waits)
  if (tid == 0 && gate_out >= 0) mbar_wait(&s->gload, (uint32_t)gate_out, SITE_OUT_TMA);
  if (tid == 0 && tok_out >= 0) mbar_wait(&s->load, (uint32_t)tok_out, SITE_OUT_TMA);
  if (tid == 0 && p_ahead) mbar_wait(&s->ldp, pph, SITE_OUT_TMA);
  if (tid == 0) tma_store_wait_read0();  // no store still reads shared memory
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

constexpr int kBwdThreads = 512;  // the gradient kernel: four warps per TMEM lane quadrant

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// D (TMEM) += A (TMEM) B (shared memory descriptor), kind::f16.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Multiplies the 32 bf16 entries of row `row`, columns qt*32.., of a tile by
// exp2(sgn * x[u]) (x in log2 units), in place.
__device__ __forceinline__ void scale_row_quarter(uint8_t* tile, int row, int qt, const float (&x)[32], float sgn) {
#pragma unroll
  for (int c8 = 0; c8 < 4; ++c8) {
    uint4* p = tile16(tile, row, qt * 32 + c8 * 8);
    uint4 w = *p;
    uint32_t* e = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = unpack_bf16(e[u]);
      e[u] = pack_bf16(f.x * ex2a(sgn * x[c8 * 8 + 2 * u]), f.y * ex2a(sgn * x[c8 * 8 + 2 * u + 1]));
    }
    *p = w;
  }
}

// gate_rows for the gradient kernel's 512 threads: threads 0-255 walk the gate
// tile (as walk_tile), then every thread takes row t, columns qt*32.., with
// the same range check, and returns x = (b_t - r) log2 e for them.
__device__ __forceinline__ bool gate_rows_quarter(float* bt, uint64_t* gbar, uint32_t parity, int* abort,
                                                  unsigned int site, float* r, float* dend, int tid, int t, int qt,
                                                  float (&x)[32]) {
  const bool landed = mbar_wait(gbar, parity, site);
  if (!landed) *abort = 1;
  if (tid < 2 * kD) walk_tile(bt, tid, r, dend);
  named_sync(kBarAll, kBwdThreads);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 v = *reinterpret_cast<const float4*>(bt + qt * (kTile * 32) + t * 32 + 4 * (q ^ (t & 7)));
    x[4 * q] = v.x;
    x[4 * q + 1] = v.y;
    x[4 * q + 2] = v.z;
    x[4 * q + 3] = v.w;
  }
  const bool first = t < kTile / 2;  // rows of the second half already hold b_t - r
  bool ok = true;
#pragma unroll
  for (int u = 0; u < 32; ++u) {
    const float y = first ? x[u] - r[qt * 32 + u] : x[u];
    ok = ok && fabsf(y) <= kMaxSpan;
    x[u] = y * kLog2e;
  }
  if (!ok) record_error(LASP_ERR_INVALID_ARG, SITE_GATE_RANGE);
  return landed;
}

// ---------------------------------------------------------------- gradients
struct SmemBwd {
  uint64_t gload, load, ldr, mma1a, mma1b, mma2, mma3, mmar, mmag;
  uint32_t tmem_base;
  int abort;
  alignas(16) float dAd[kTile];  // do_t . v_t, the diagonal of dO V^T (epilogues 1-3)
  alignas(16) float bnd[kD];     // e^{b_end[i]} <R_c[i], P_c[i]>
};

// One persistent CTA per SM, taking segments of S 128-token tiles in launch
// order (segment w, w + grid, ...) and walking each from its last tile to its
// first. The state R_c entering a tile from the right comes, for a segment's
// last tile, from the scan over segments (the workspace slot of that tile's
// last chunk); every other tile's is formed on the way, by the tile after it
// (LASP Appendix A.4: the gated form of the gradient-state recurrence):
//   R_{c-1} = diag(e^{b_end}) R_c + diag(e^{r}) Q^^T dO     (Q^ = q . e^{b - r})
// with Q^^T dO an extra MMA of phase 2 into T0 (idle between epilogue 1 and
// phase 3), combined in fp32 with each thread's share of R_c (kept in
// registers since phase 1 read it) while the T1 products run, and written to
// a scratch slot of the segment (the workspace slot of its first chunk),
// where the next tile's bulk load of R finds it. The scratch is lane-major
// (float4 group g of state row m at float4 g * 128 + m), so that the threads
// of a warp, which own consecutive rows, write one 512-byte run per access;
// phase 1 reads R row-major from the scan's slot (a segment's last tile) or
// lane-major from the scratch.
//
// The log-gate gradient's column sums over the tile's rows,
//   dg_t = sum_{s >= t} dB_s + sum_{s < t} (k . dk^inter)_s + e^{b_end} <R_c, P_c>,
// are two products with triangular 0/1 matrices, U_ts = [s >= t] and L_ts =
// [s < t], held in TMEM as the A operand; dB and k . dk^inter enter as B in
// two bf16 parts each (x = hi + lo, about 16 bits of mantissa), so the sums
// keep nearly fp32 precision.
//
// Most barriers complete once per tile, so their parity flips from tile to
// tile; mmar only on tiles that form a state. Shared memory: Q^, K^, V, dO, X
// (P', loaded as the output kernel cached it, then R'), and the pair sA / sB
// (the gate tile during the walk; then dA . strict and A . causal; then the
// dK and dV outputs); after the last gradient MMA, V, dO, X and K^ hold the
// sums' B operands and Q^ / K^ the fp32 dg tile. TMEM: T0 = dO V^T -> Q^^T dO
// -> (dA . strict)^T Q^ -> dg; T1 = Q^ K^^T -> dV; T2 = dO P'^T + (dA .
// strict) K^ -> q . dq' -> U and L; T3 = log2 E -> V R'^T.
//
// 512 threads: warp w owns tile rows / TMEM lanes 32*(w%4).. and the column
// quarter w/4 (32 columns) of every row-wise step.
__global__ void __launch_bounds__(kBwdThreads, 1) gla_bwd_tc(
    const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_do,
    const __grid_constant__ CUtensorMap map_dk, const __grid_constant__ CUtensorMap map_dv,
    const __grid_constant__ CUtensorMap map_g, const __grid_constant__ CUtensorMap map_dg,
    const float* __restrict__ P, float* __restrict__ R, __nv_bfloat16* __restrict__ dq, int H, int64_t N,
    int64_t t_slots, int stride, int ntx, int S, int64_t nitems, RunIf run_if) {
  if (!runs(run_if)) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = base;
  uint8_t* sK = base + 1 * kTileBytes;
  uint8_t* sV = base + 2 * kTileBytes;
  uint8_t* sD = base + 3 * kTileBytes;
  uint8_t* sX = base + 4 * kTileBytes;
  uint8_t* sA = base + 5 * kTileBytes;
  uint8_t* sB = base + 6 * kTileBytes;
  SmemBwd* s = reinterpret_cast<SmemBwd*>(base + 7 * kTileBytes);
  float* bt = reinterpret_cast<float*>(sA);  // gate tile over sA and sB during the walk
  // r and b_end - r of the gate walk, over arrays first written after phase 0
  float* sr = s->dAd;
  float* sdend = s->bnd;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = (warp & 3) * 32 + lane, qt = warp >> 2, cq = qt * 32;
  // this CTA's k-th tile: tile j = S - 1 - k % S (128 tokens c * 128.., c =
  // seg * S + j) of segment item blockIdx.x + (k / S) * grid (segment seg of
  // head h of sequence b)
  const int nsg = ntx / S;
  const int64_t my_items = nitems > (int64_t)blockIdx.x ? (nitems - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int64_t my_tiles = my_items * S;
  auto tile_of = [&](int64_t k, int& c, int& h, int& b, int& j) {
    const int64_t w = blockIdx.x + (k / S) * (int64_t)gridDim.x;
    j = S - 1 - (int)(k % S);
    c = (int)(w % nsg) * S + j;
    h = (int)((w / nsg) % H);
    b = (int)(w / ((int64_t)nsg * H));
  };
  // P of a tile's first chunk (R of its last is stride - 1 slots on)
  auto pslot_of = [&](int c, int h, int b) { return ((int64_t)b * t_slots + (int64_t)c * stride) * H + h; };
  // the slot R_c of tile c is read from: the scan's (tile's last chunk) for a
  // segment's last tile, the scratch (segment's first chunk) for the others
  auto rslot_of = [&](int c, int h, int b, int j) {
    return j == S - 1 ? pslot_of(c, h, b) + (int64_t)(stride - 1) * H : pslot_of(c - j, h, b);
  };
  auto load_tokens = [&](uint8_t* dst, const CUtensorMap* map, int h, int row, int b) {
    tma_load_4d(dst, map, &s->load, 0, h, row, b);
    tma_load_4d(dst + kBox, map, &s->load, 64, h, row, b);
  };
  // P' = diag(e^{r}) P_c of a tile, as the forward's output kernel left it in
  // the cache slot (the bf16 operand tile, loaded as is)
  auto load_pprime = [&](int64_t ps) { bulk_load(sX, P + ps * kD * kD, kTileBytes, &s->load); };
  if (tid == 0) {
    prefetch_tmap(&map_q);
    prefetch_tmap(&map_k);
    prefetch_tmap(&map_v);
    prefetch_tmap(&map_do);
    prefetch_tmap(&map_g);
    mbar_init(&s->gload, 1);
    mbar_init(&s->load, 1);
    mbar_init(&s->ldr, 1);
    mbar_init(&s->mma1a, 1);
    mbar_init(&s->mma1b, 1);
    mbar_init(&s->mma2, 1);
    mbar_init(&s->mma3, 1);
    mbar_init(&s->mmar, 1);
    mbar_init(&s->mmag, 1);
    s->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s->tmem_base;
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  const uint32_t T0 = 0, T1 = 128, T2 = 256, T3 = 384;
  if (tid == 0 && my_tiles > 0) {
    // the first tile's loads; a later tile's are issued during the tile before
    int c, h, b, j;
    tile_of(0, c, h, b, j);
    const int64_t ps = pslot_of(c, h, b);
    load_gate_tile(bt, &map_g, &s->gload, h, c * kTile, b);
    // R is read by a bulk load later: into L2 now
    bulk_prefetch_l2(R + rslot_of(c, h, b, j) * kD * kD, kD * kD * 4);
    mbar_arrive_expect_tx(&s->load, 5 * kTileBytes);
    load_tokens(sQ, &map_q, h, c * kTile, b);
    load_tokens(sK, &map_k, h, c * kTile, b);
    load_tokens(sV, &map_v, h, c * kTile, b);
    load_tokens(sD, &map_do, h, c * kTile, b);
    load_pprime(ps);
  }
  uint32_t ph = 0;       // parity of every barrier's phase for this CTA's current tile
  uint32_t rph = 0;      // parity of mmar's next phase
  bool r_ahead = false;  // thread 0: R's load into sA/sB is in flight
  // thread 0: the parity of the gate tile's and the token tiles' loads still
  // in flight (issued, not yet waited for), or -1; cleanup waits for them
  int gate_out = my_tiles > 0 ? 0 : -1, tok_out = gate_out;
  for (int64_t k = 0; k < my_tiles; ++k, ph ^= 1u) {
  int c, h, b, j;
  tile_of(k, c, h, b, j);
  const int64_t row0 = (int64_t)c * kTile;
  const int64_t rslot = rslot_of(c, h, b, j);
  const int64_t tok = (((int64_t)b * N + row0 + t) * H + h) * kD;  // row t of every token tensor
  const bool has_next = k + 1 < my_tiles;  // this CTA's next tile
  const bool form = j > 0;  // this tile forms R_{c-1} for the tile before it
  // ---- phase 0: gates, Q^, K^, log2 E -> T3, P' -> X
  float x[32];
  if (gate_rows_quarter(bt, &s->gload, ph, &s->abort, SITE_BWD_TMA, sr, sdend, tid, t, qt, x) && tid == 0)
    gate_out = -1;
  // e^{r}, e^{b_end - r} and e^{b_end} of state row t (feature t)
  const float er = ex2a(sr[t] * kLog2e), wt = ex2a(sdend[t] * kLog2e), eb = er * wt;
  named_sync(kBarAll, kBwdThreads);  // every row of the gate tile has been read
  if (tid == 0) {
    // R_c (fp32) into the gate tile's space while the token tiles arrive
    mbar_arrive_expect_tx(&s->ldr, kD * kD * 4);
    bulk_load(bt, R + rslot * kD * kD, kD * kD * 4, &s->ldr);
    r_ahead = true;
  }
  if (mbar_wait(&s->load, ph, SITE_BWD_TMA)) {
    if (tid == 0) tok_out = -1;
  } else {
    s->abort = 1;
  }
  scale_row_quarter(sQ, t, qt, x, 1.f);   // Q^ = q . E
  scale_row_quarter(sK, t, qt, x, -1.f);  // K^ = k / E
  {
    uint32_t r0[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) r0[u] = __float_as_uint(x[u]);
    tmem_st32(lane_base + T3 + cq, r0);
    tmem_st_wait();
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (s->abort) goto cleanup;
  {
    const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aD = smem_u32(sD);
    const uint32_t aX = smem_u32(sX), aA = smem_u32(sA), aB = smem_u32(sB);
    constexpr uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t id_kn = idesc_bf16(128, 128, 0, 1);
    constexpr uint32_t id_nn = idesc_bf16(128, 128, 1, 1);
    // ---- phase 1: T2 = dO P'^T | T0 = dO V^T, T1 = Q^ K^^T (P' first, so that
    // X takes R' while the other two run)
    if (tid == 0) {
      tc_fence_after();
      for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T2, kmaj(aD, kk), kmaj(aX, kk), id_kk, kk != 0);
      mma_commit(&s->mma1b);
      for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T0, kmaj(aD, kk), kmaj(aV, kk), id_kk, kk != 0);
      for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T1, kmaj(aQ, kk), kmaj(aK, kk), id_kk, kk != 0);
      mma_commit(&s->mma1a);
    }
    // while the MMAs run: row t of R (fp32, from sA/sB; this thread's quarter
    // of the columns) into registers, and that quarter of <R'_t, P'_t> =
    // e^{b_end_t} <R_t, P_t>, with row t of P' read in X (bf16)
    {
      const bool rok = mbar_wait(&s->ldr, ph, SITE_BWD_TMA);
      if (!rok) s->abort = 1;
      if (tid == 0 && rok) r_ahead = false;  // else cleanup waits for it once more
    }
    // R_c, row t, columns cq.. (float4 groups g = qt * 8 + u): row-major from
    // the scan's slot, lane-major from the scratch
    float4 rreg[8];
    {
      const bool rlm = j != S - 1;
      const float4* R4 = reinterpret_cast<const float4*>(bt);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int g = qt * 8 + u;
        rreg[u] = R4[rlm ? g * kD + t : t * (kD / 4) + g];
      }
    }
    named_sync(kBarAll, kBwdThreads);  // every row of R has been read: sA/sB are free
    {
      // e^{b_end - r} <R_t, P'_t> over this thread's quarter of the columns (P'
      // row t in X, bf16); the four quarters' sums meet in sA, one thread per
      // feature adds them into bnd before the masks overwrite sA
      float dot = 0.f;
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        const uint4 pw = *tile16(sX, t, cq + q8 * 8);
        const float2 p0 = unpack_bf16(pw.x), p1 = unpack_bf16(pw.y), p2 = unpack_bf16(pw.z), p3 = unpack_bf16(pw.w);
        const float4 a = rreg[2 * q8], b2 = rreg[2 * q8 + 1];
        dot += p0.x * a.x + p0.y * a.y + p1.x * a.z + p1.y * a.w + p2.x * b2.x + p2.y * b2.y + p3.x * b2.z +
               p3.y * b2.w;
      }
      float* part = reinterpret_cast<float*>(sA);
      part[qt * kD + t] = dot * wt;
      named_sync(kBarAll, kBwdThreads);
      if (tid < kD) s->bnd[tid] = (part[tid] + part[kD + tid]) + (part[2 * kD + tid] + part[3 * kD + tid]);
      named_sync(kBarAll, kBwdThreads);
    }
    // X is free once dO P'^T has read P': R' = diag(e^{b_end - r}) R_c replaces it
    if (mbar_wait(&s->mma1b, ph, SITE_BWD_MMA)) {
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        const float4 a = rreg[2 * q8], b2 = rreg[2 * q8 + 1];
        st_tile16(sX, t, cq + q8 * 8,
                  make_uint4(pack_bf16(a.x * wt, a.y * wt), pack_bf16(a.z * wt, a.w * wt),
                             pack_bf16(b2.x * wt, b2.y * wt), pack_bf16(b2.z * wt, b2.w * wt)));
      }
    } else {
      s->abort = 1;
    }
    // ---- epilogue 1: dA . strict -> sA, A . causal -> sB, the diagonal of dA
    if (mbar_wait(&s->mma1a, ph, SITE_BWD_MMA)) {
      tc_fence_after();
#pragma unroll 1
      for (int c2 = 0; c2 < 4; ++c2) {
        const int col0 = cq + c2 * 8;
        uint32_t ra[8], rs[8];
        tmem_ld8(lane_base + T0 + col0, ra);
        tmem_ld8(lane_base + T1 + col0, rs);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (col0 + u == t) s->dAd[t] = __uint_as_float(ra[u]);
        float fa[8], fs[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int col = col0 + u;
          fa[u] = col < t ? __uint_as_float(ra[u]) : 0.f;
          fs[u] = col <= t ? __uint_as_float(rs[u]) : 0.f;
        }
        *tile16(sA, t, col0) = make_uint4(pack_bf16(fa[0], fa[1]), pack_bf16(fa[2], fa[3]), pack_bf16(fa[4], fa[5]),
                                          pack_bf16(fa[6], fa[7]));
        *tile16(sB, t, col0) = make_uint4(pack_bf16(fs[0], fs[1]), pack_bf16(fs[2], fs[3]), pack_bf16(fs[4], fs[5]),
                                          pack_bf16(fs[6], fs[7]));
      }
    } else {
      s->abort = 1;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (s->abort) goto cleanup;
    // ---- phase 2: T2 += (dA . strict) K^ | T0 = Q^^T dO (when this tile forms
    // R_{c-1}) | T1 = (A . causal)^T dO + K^ R' (phase 1's masks and R' are in
    // place; T1 was read by epilogue 1)
    if (tid == 0) {
      tc_fence_after();
      for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + T2, kmaj(aA, kk), mnmaj(aK, kk), id_kn, 1);
      mma_commit(&s->mma2);
      if (form) {
        for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + T0, mnmaj(aQ, kk), mnmaj(aD, kk), id_nn, kk != 0);
        mma_commit(&s->mmar);
      }
      for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + T1, mnmaj(aB, kk), mnmaj(aD, kk), id_nn, kk != 0);
      for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T1, kmaj(aK, kk), mnmaj(aX, kk), id_kn, 1);
    }
    // ---- R_{c-1} = e^{b_end} R_c + e^{r} T0 (row t, columns cq..; R_c from
    // this thread's registers, read in phase 1), under the T1 products, before
    // epilogue 2 takes its registers; into the segment's scratch slot, lane-major
    // (float4 group g of row t at g * 128 + t), where the next tile's bulk load
    // of R finds it
    if (form) {
      float4* rn = reinterpret_cast<float4*>(R + pslot_of(c - j, h, b) * kD * kD);
      if (mbar_wait(&s->mmar, rph, SITE_BWD_MMA)) {
        tc_fence_after();
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          uint32_t a[16];
          tmem_ld16(lane_base + T0 + cq + c2 * 16, a);
          tmem_ld_wait();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const float4 r4 = rreg[c2 * 4 + q4];
            rn[(qt * 8 + c2 * 4 + q4) * kD + t] =
                make_float4(fmaf(eb, r4.x, er * __uint_as_float(a[4 * q4])),
                            fmaf(eb, r4.y, er * __uint_as_float(a[4 * q4 + 1])),
                            fmaf(eb, r4.z, er * __uint_as_float(a[4 * q4 + 2])),
                            fmaf(eb, r4.w, er * __uint_as_float(a[4 * q4 + 3])));
          }
        }
        fence_async_global();  // the next tile's bulk load of R reads these stores
      } else {
        s->abort = 1;
      }
      rph ^= 1u;
    }
    // ---- epilogue 2: dq' = E . T2; dq = dq' + (do_t . v_t) k_t = E . (T2 + (do_t . v_t) K^_t);
    // q . dq' = Q^ . T2 -> T2
    float xl[32];  // log2 E of row t, columns cq.., kept for epilogue 3
    if (mbar_wait(&s->mma2, ph, SITE_BWD_MMA)) {
      tc_fence_after();
      {
        uint32_t r0[32];
        tmem_ld32(lane_base + T3 + cq, r0);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 32; ++u) xl[u] = __uint_as_float(r0[u]);
      }
      const float dad = s->dAd[t];
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        const int col0 = cq + c2 * 16;
        uint32_t a[16];
        tmem_ld16(lane_base + T2 + col0, a);
        // Q^ and K^ of row t (bf16, shared memory): q . dq' = Q^ . T2 and k_t = K^_t . E_t
        uint32_t qh[8], kh[8];
#pragma unroll
        for (int q4 = 0; q4 < 2; ++q4) {
          const uint4 wq = *tile16(sQ, t, col0 + q4 * 8);
          const uint4 wk = *tile16(sK, t, col0 + q4 * 8);
          qh[4 * q4] = wq.x, qh[4 * q4 + 1] = wq.y, qh[4 * q4 + 2] = wq.z, qh[4 * q4 + 3] = wq.w;
          kh[4 * q4] = wk.x, kh[4 * q4 + 1] = wk.y, kh[4 * q4 + 2] = wk.z, kh[4 * q4 + 3] = wk.w;
        }
        tmem_ld_wait();
        uint32_t out[8];
#pragma unroll
        for (int u2 = 0; u2 < 8; ++u2) {
          const float2 qf = unpack_bf16(qh[u2]), kf = unpack_bf16(kh[u2]);
          const float e0 = ex2a(xl[c2 * 16 + 2 * u2]), e1 = ex2a(xl[c2 * 16 + 2 * u2 + 1]);
          const float t0 = __uint_as_float(a[2 * u2]), t1 = __uint_as_float(a[2 * u2 + 1]);
          out[u2] = pack_bf16(e0 * fmaf(dad, kf.x, t0), e1 * fmaf(dad, kf.y, t1));
          a[2 * u2] = __float_as_uint(qf.x * t0);
          a[2 * u2 + 1] = __float_as_uint(qf.y * t1);
        }
        uint4* dst = reinterpret_cast<uint4*>(dq + tok + col0);
        dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
        dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
        tmem_st16(lane_base + T2 + col0, a);
      }
      tmem_st_wait();
    } else {
      s->abort = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (s->abort) goto cleanup;
    // ---- phase 3: T3 = V R'^T, then T0 = (dA . strict)^T Q^ (every thread has
    // read T0 for R_{c-1} before the barrier above)
    if (tid == 0) {
      tc_fence_after();
      for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + T3, kmaj(aV, kk), kmaj(aX, kk), id_kk, kk != 0);
      for (int kk = 0; kk < kTile / 16; ++kk) mma_bf16(tmem + T0, mnmaj(aA, kk), mnmaj(aQ, kk), id_nn, kk != 0);
      mma_commit(&s->mma3);
    }
    // ---- epilogue 3: dk = E^-1 . (T0 + T3 + (do_s . v_s) Q^_s) -> sA, dv = T1 -> sB;
    // dB = q . dq' - k . dk' = T2 - K^ . T0 and k . dk^inter = K^ . T3, each in
    // two bf16 parts (x = hi + lo, hi = bf16(x), lo = bf16(x - hi)), as the
    // operand tiles of the log-gate gradient's column sums: dB over V and dO,
    // k . dk^inter over X and K^ (each thread overwrites only the K^ entries it
    // has read). The masks of those sums go into TMEM, over this thread's
    // columns of T2 once it has read them: U_ts = [s >= t] and L_ts = [s < t],
    // the rows' K steps 2 qt and 2 qt + 1 at T2 + cq (U) and T2 + cq + 16 (L).
    uint8_t* sBh = sV;
    uint8_t* sBl = sD;
    uint8_t* sKh = sX;
    uint8_t* sKl = sK;
    if (mbar_wait(&s->mma3, ph, SITE_BWD_MMA)) {
      tc_fence_after();
      const float dad = s->dAd[t];
#pragma unroll
      for (int c2 = 0; c2 < 4; ++c2) {
        const int col0 = cq + c2 * 8;
        uint32_t ka[8], kb[8], bq[8];
        tmem_ld8(lane_base + T0 + col0, ka);
        tmem_ld8(lane_base + T3 + col0, kb);
        tmem_ld8(lane_base + T2 + col0, bq);
        const uint4 wq = *tile16(sQ, t, col0), wk = *tile16(sK, t, col0);
        const uint32_t qh[4] = {wq.x, wq.y, wq.z, wq.w}, kh[4] = {wk.x, wk.y, wk.z, wk.w};
        tmem_ld_wait();
        uint32_t out[4], dbh[4], dbl[4], kdh[4], kdl[4];
#pragma unroll
        for (int u2 = 0; u2 < 4; ++u2) {
          const float2 qf = unpack_bf16(qh[u2]), kf = unpack_bf16(kh[u2]);
          const float e0 = ex2a(-xl[c2 * 8 + 2 * u2]), e1 = ex2a(-xl[c2 * 8 + 2 * u2 + 1]);
          const float a0 = __uint_as_float(ka[2 * u2]), a1 = __uint_as_float(ka[2 * u2 + 1]);
          const float b0 = __uint_as_float(kb[2 * u2]), b1 = __uint_as_float(kb[2 * u2 + 1]);
          out[u2] = pack_bf16(e0 * fmaf(dad, qf.x, a0 + b0), e1 * fmaf(dad, qf.y, a1 + b1));
          const float d0 = __uint_as_float(bq[2 * u2]) - kf.x * a0, d1 = __uint_as_float(bq[2 * u2 + 1]) - kf.y * a1;
          const float g0 = kf.x * b0, g1 = kf.y * b1;
          dbh[u2] = pack_bf16(d0, d1);
          kdh[u2] = pack_bf16(g0, g1);
          const float2 dh = unpack_bf16(dbh[u2]), gh = unpack_bf16(kdh[u2]);
          dbl[u2] = pack_bf16(d0 - dh.x, d1 - dh.y);
          kdl[u2] = pack_bf16(g0 - gh.x, g1 - gh.y);
        }
        *tile16(sA, t, col0) = make_uint4(out[0], out[1], out[2], out[3]);
        *tile16(sBh, t, col0) = make_uint4(dbh[0], dbh[1], dbh[2], dbh[3]);
        *tile16(sBl, t, col0) = make_uint4(dbl[0], dbl[1], dbl[2], dbl[3]);
        *tile16(sKh, t, col0) = make_uint4(kdh[0], kdh[1], kdh[2], kdh[3]);
        *tile16(sKl, t, col0) = make_uint4(kdl[0], kdl[1], kdl[2], kdl[3]);
      }
      {
        uint32_t dvv[32];
        tmem_ld32(lane_base + T1 + cq, dvv);
        tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          *tile16(sB, t, cq + q4 * 8) =
              make_uint4(pack_bf16(__uint_as_float(dvv[q4 * 8]), __uint_as_float(dvv[q4 * 8 + 1])),
                         pack_bf16(__uint_as_float(dvv[q4 * 8 + 2]), __uint_as_float(dvv[q4 * 8 + 3])),
                         pack_bf16(__uint_as_float(dvv[q4 * 8 + 4]), __uint_as_float(dvv[q4 * 8 + 5])),
                         pack_bf16(__uint_as_float(dvv[q4 * 8 + 6]), __uint_as_float(dvv[q4 * 8 + 7])));
      }
      {
        // U and L rows t, K elements cq.. (bf16 1 = 0x3f80; element 2w in the low half of word w)
        uint32_t um[16], lm[16];
#pragma unroll
        for (int w = 0; w < 16; ++w) {
          const int s0 = cq + 2 * w;
          um[w] = (s0 >= t ? 0x3f80u : 0u) | (s0 + 1 >= t ? 0x3f800000u : 0u);
          lm[w] = (s0 < t ? 0x3f80u : 0u) | (s0 + 1 < t ? 0x3f800000u : 0u);
        }
        tmem_st16(lane_base + T2 + cq, um);
        tmem_st16(lane_base + T2 + cq + 16, lm);
      }
      tmem_st_wait();
      fence_async_smem();
    } else {
      s->abort = 1;
    }
    tc_fence_before();
    __syncthreads();  // dK, dV and the sums' operands are staged
    tc_fence_after();
    if (s->abort) goto cleanup;
    if (tid == 0) {
      // dK and dV leave now; the sums: T0 = U (dB_hi + dB_lo) + L (kdk_hi + kdk_lo)
      tma_store_4d(&map_dk, sA, 0, h, (int)row0, b);
      tma_store_4d(&map_dk, sA + kBox, 64, h, (int)row0, b);
      tma_store_4d(&map_dv, sB, 0, h, (int)row0, b);
      tma_store_4d(&map_dv, sB + kBox, 64, h, (int)row0, b);
      tma_store_commit();
      const uint32_t aBh = smem_u32(sBh), aBl = smem_u32(sBl), aKh = smem_u32(sKh), aKl = smem_u32(sKl);
      const uint32_t tu = tmem + T2;
      for (int kk = 0; kk < kTile / 16; ++kk)
        mma_bf16_ts(tmem + T0, tu + 32 * (kk >> 1) + 8 * (kk & 1), mnmaj(aBh, kk), id_kn, kk != 0);
      for (int kk = 0; kk < kTile / 16; ++kk)
        mma_bf16_ts(tmem + T0, tu + 32 * (kk >> 1) + 8 * (kk & 1), mnmaj(aBl, kk), id_kn, 1);
      for (int kk = 0; kk < kTile / 16; ++kk)
        mma_bf16_ts(tmem + T0, tu + 32 * (kk >> 1) + 16 + 8 * (kk & 1), mnmaj(aKh, kk), id_kn, 1);
      for (int kk = 0; kk < kTile / 16; ++kk)
        mma_bf16_ts(tmem + T0, tu + 32 * (kk >> 1) + 16 + 8 * (kk & 1), mnmaj(aKl, kk), id_kn, 1);
      mma_commit(&s->mmag);
      if (has_next) {
        // once the dK and dV stores have read sA / sB (the only bulk stores in
        // flight), the next tile's gates go there, under the sums; a segment's
        // entering R into L2 (a formed one is there)
        tma_store_wait_read0();
        int cn, hn, bn, jn;
        tile_of(k + 1, cn, hn, bn, jn);
        load_gate_tile(bt, &map_g, &s->gload, hn, cn * kTile, bn);
        gate_out = (int)(ph ^ 1u);
        if (jn == S - 1) bulk_prefetch_l2(R + rslot_of(cn, hn, bn, jn) * kD * kD, kD * kD * 4);
      }
    }
    // dg_t = sum_{t' >= t} dB_t' + sum_{t' < t} k . dk^inter_t' + e^{b_end} <R_c, P_c>:
    // T0 plus bnd, into an fp32 tile over Q^ and K^ (the gate map's layout),
    // stored by TMA below
    float* fB = reinterpret_cast<float*>(sQ);
    if (mbar_wait(&s->mmag, ph, SITE_BWD_MMA)) {
      tc_fence_after();
      uint32_t dgv[32];
      tmem_ld32(lane_base + T0 + cq, dgv);
      tmem_ld_wait();
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const float4 bn = *reinterpret_cast<const float4*>(s->bnd + cq + 4 * q4);
        *reinterpret_cast<float4*>(fB + gate_slot(t, cq + 4 * q4)) =
            make_float4(__uint_as_float(dgv[4 * q4]) + bn.x, __uint_as_float(dgv[4 * q4 + 1]) + bn.y,
                        __uint_as_float(dgv[4 * q4 + 2]) + bn.z, __uint_as_float(dgv[4 * q4 + 3]) + bn.w);
      }
    } else {
      s->abort = 1;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();  // every thread has read T0 and written its dg; no wait fails after this point
    const bool stop = s->abort != 0;
    if (tid == 0) {
      if (!stop) {
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) tma_store_4d(&map_dg, fB + cb * (kTile * 32), cb * 32, h, (int)row0, b);
        tma_store_commit();
      }
      const bool next = has_next && !stop;
      int cn = 0, hn = 0, bn = 0, jn = 0;
      if (next) tile_of(k + 1, cn, hn, bn, jn);
      if (next) {
        // the sums' operand tiles (V, dO, X) have been read by their MMAs
        mbar_arrive_expect_tx(&s->load, 5 * kTileBytes);
        load_tokens(sV, &map_v, hn, cn * kTile, bn);
        load_tokens(sD, &map_do, hn, cn * kTile, bn);
        load_pprime(pslot_of(cn, hn, bn));
        tok_out = (int)(ph ^ 1u);
      }
      tma_store_wait_read0();  // the dg store has read fB (over Q and K)
      if (next) {
        load_tokens(sQ, &map_q, hn, cn * kTile, bn);
        load_tokens(sK, &map_k, hn, cn * kTile, bn);
      }
    }
    if (stop) goto cleanup;
  }
  }
cleanup:
  // an abort leaves loads unused: they land first
  if (tid == 0 && r_ahead) mbar_wait(&s->ldr, ph, SITE_BWD_TMA);
  if (tid == 0 && gate_out >= 0) mbar_wait(&s->gload, (uint32_t)gate_out, SITE_BWD_TMA);
  if (tid == 0 && tok_out >= 0) mbar_wait(&s->load, (uint32_t)tok_out, SITE_BWD_TMA);
  if (tid == 0) tma_store_wait_read0();  // no store still reads shared memory
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace tc_gla_detail

bool tc_gla_ok(int dtype, int d, int64_t C, int64_t N) {
  // chunks that divide the 128-token tile: a tile's sums regroup the per-chunk
  // intra and inter terms, so states are needed only at tile boundaries
  using tc_gla_detail::kTile;
  return dtype == LASP_BF16 && d == tc_gla_detail::kD && C >= 1 && C <= kTile && kTile % C == 0 && N % kTile == 0;
}

cudaError_t tc_gla_chunk_states(const void* x, const void* y, const float* g, float* M, float* gsum,
                                float* gsum_tile, int B, int H, int64_t N, int kind, int64_t t_slots, int stride,
                                int offset, int tiles, int tstride, cudaStream_t st, int* span_flag, RunIf run) {
  using namespace tc_gla_detail;
  CUtensorMap mx, my;
  if (!make_token_map(&mx, x, B, H, N, kD, kTile) || !make_token_map(&my, y, B, H, N, kD, kTile))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + 2 * (size_t)kTileBytes + sizeof(SmemStates);
  if (tiles < 1 || N % ((int64_t)tiles * kTile) != 0) return cudaErrorInvalidValue;
  auto kern = tiles == 1 ? gla_states_tc<true> : gla_states_tc<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3((unsigned)(N / ((int64_t)tiles * kTile)), H, B), kThreads, smem, st>>>(
      mx, my, g, M, gsum, gsum_tile, H, N, kind, t_slots, stride, offset, tiles, tstride, span_flag, run);
  return cudaGetLastError();
}

cudaError_t tc_gla_chunk_out(const void* q, const void* k, const void* v, const float* g, float* P, void* o,
                             int B, int H, int64_t N, int64_t t_slots, int stride, int tiles, cudaStream_t st,
                             RunIf run) {
  using namespace tc_gla_detail;
  CUtensorMap mq, mk, mv, mo, mg, mp;
  const int ntx = (int)(N / kTile);
  if (tiles < 1 || ntx % tiles != 0) return cudaErrorInvalidValue;
  if (!make_token_map(&mq, q, B, H, N, kD, kTile) || !make_token_map(&mk, k, B, H, N, kD, kTile) ||
      !make_token_map(&mv, v, B, H, N, kD, kTile) || !make_token_map(&mo, o, B, H, N, kD, kTile) ||
      !make_gate_map(&mg, g, B, H, N, kD, kTile) || !make_state_map(&mp, P, (int64_t)B * t_slots * H, kD))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + 7 * (size_t)kTileBytes + sizeof(SmemOut);
  cudaError_t e = cudaFuncSetAttribute(gla_out_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  // one persistent CTA per SM (the kernel holds most of shared memory and all of TMEM)
  const int64_t nseg = (int64_t)B * H * (ntx / tiles);
  const unsigned grid = (unsigned)std::min<int64_t>(nseg, sms);
  gla_out_tc<<<grid, kThreads, smem, st>>>(mq, mk, mv, mo, mg, mp, P, H, N, t_slots, stride, ntx, tiles, nseg, run);
  return cudaGetLastError();
}

cudaError_t tc_gla_chunk_bwd(const void* q, const void* k, const void* v, const void* dout, const float* g,
                             const float* P, float* Rs, void* dq, void* dk, void* dv, float* dg, int B, int H,
                             int64_t N, int64_t t_slots, int stride, int tiles, cudaStream_t st, RunIf run) {
  using namespace tc_gla_detail;
  CUtensorMap mq, mk, mv, mdo, mdk, mdv, mg, mdg;
  if (!make_token_map(&mq, q, B, H, N, kD, kTile) || !make_token_map(&mk, k, B, H, N, kD, kTile) ||
      !make_token_map(&mv, v, B, H, N, kD, kTile) || !make_token_map(&mdo, dout, B, H, N, kD, kTile) ||
      !make_token_map(&mdk, dk, B, H, N, kD, kTile) || !make_token_map(&mdv, dv, B, H, N, kD, kTile) ||
      !make_gate_map(&mg, g, B, H, N, kD, kTile) || !make_gate_map(&mdg, dg, B, H, N, kD, kTile))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + 7 * (size_t)kTileBytes + sizeof(SmemBwd);
  cudaError_t e = cudaFuncSetAttribute(gla_bwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  // one persistent CTA per SM (the kernel holds all of TMEM and most of shared
  // memory), taking segments of `tiles` 128-token tiles
  const int ntx = (int)(N / kTile);
  if (tiles < 1 || ntx % tiles != 0) return cudaErrorInvalidValue;
  const int64_t nitems = (int64_t)B * H * (ntx / tiles);
  const unsigned grid = (unsigned)std::min<int64_t>(nitems, sms);
  gla_bwd_tc<<<grid, kBwdThreads, smem, st>>>(mq, mk, mv, mdo, mdk, mdv, mg, mdg, P, Rs, (__nv_bfloat16*)dq, H, N, t_slots,
                                            stride, ntx, tiles, nitems, run);
  return cudaGetLastError();
}

}  // namespace lasp
