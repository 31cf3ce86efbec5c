// Softmax attention on the 5th-generation tensor cores: the attention layers a
// hybrid model keeps (LASP-2 review page, "Summary": LASP-2H applies the same
// AllGather pattern to standard attention, each rank gathering K_t and V_t).
// Queries of one call sit at global positions p_i = q_offset + i; keys and
// values at positions 0..Nk-1 (the gathered K and V). For bf16, d = 128:
//   s_ij = scale (q_i . k_j) for j <= p_i,  o_i = sum_j softmax_j(s_ij) v_j,
//   lse_i = log sum_{j <= p_i} exp(s_ij)
// and the gradients of sum(o . do).
//
// Forward (one CTA per 128-query tile, heaviest tiles first): the softmax is
// taken online over 128-key tiles. Warp roles, all hand-offs by mbarriers:
//   warp 8 (one thread): TMA loads of the Q tile and of every key tile's K and
//     V into two stages each (K of stage s is refilled once the S MMA that
//     read it has completed, V once the P V MMA has);
//   warp 9 (one thread): S_j = Q K_j^T into one of two TMEM buffers, then
//     O += P_{j-1} V_{j-1}, so the next S is on the tensor pipe while the
//     softmax warps work on the last one;
//   warps 0-7 (two threads per query row: warp w reads TMEM lanes 32 (w % 4)..
//     and the column half w / 4): read S_j from TMEM, mask, keep the running
//     maximum m (log2 units; the two halves of a row exchange their tile
//     maxima through shared memory) and the sum l, write P = exp2(s - m) in
//     bf16 into TMEM as the A operand of the P V MMA. O in TMEM is
//     rescaled only when a row's maximum grows by more than 8 (P stays below
//     2^8 in between): the final O / l uses the same stale m for both, so the
//     result is exact; the rescale waits for the P V MMA before it.
// Epilogue: O / l in bf16 by TMA store, lse = (m + log2 l) ln 2.
//
// Backward (the chain rule through the softmax, with p_ij = exp(s_ij - lse_i)
// recomputed from the forward's lse, delta_i = do_i . o_i):
//   ds_ij = p_ij (do_i . v_j - delta_i),
//   dv_j = sum_i p_ij do_i,  dk_j = scale sum_i ds_ij q_i,  dq_i = scale sum_j ds_ij k_j.
// softmax_delta: delta per query row. softmax_dkdv_tc: one CTA per 128-key
// tile walks the query tiles that see it: S^T = K Q^T and dP^T = V dO^T into
// TMEM, then (sixteen epilogue warps, 32 query columns each) P^T and dS^T in
// bf16 back into TMEM over the columns they came from, then dV += P^T dO and
// dK += dS^T Q; Q and dO stream through a three-slot ring so that the next Q
// tile loads during the current tile.
// softmax_dq_tc: one CTA per 128-query tile walks its key tiles: S = Q K^T,
// dP = dO V^T, dS (sixteen epilogue warps, into TMEM), dQ += dS K. Only the
// tiles on the causal diagonal mask element by element.
// The operands that the epilogues produce (P, P^T, dS^T, dS) stay in TMEM as
// the A operand of the MMA that consumes them: an MMA whose operands both
// come from shared memory takes nearly all of its bandwidth at N = 128. The two gradient kernels
// recompute P separately, so no atomics are needed and the results do not
// depend on scheduling.
#include <algorithm>

#include "kernels.h"
#include "lasp_common.cuh"
#include "sm100.cuh"
#include "tc_kernels.h"
#include "tma_host.h"

namespace lasp {
namespace tc_softmax_detail {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTile = 128;
constexpr uint32_t kTileBytes = kTile * kD * 2;  // 32 KB: two 64-feature boxes
constexpr uint32_t kBox = kTileBytes / 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale = 8.f;  // log2 growth of a row maximum that forces O's rescale

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
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

// ------------------------------------------------------------------ forward
constexpr int kFwdThreads = 320;  // warps 0-7 softmax, 8 TMA, 9 MMA
constexpr int kSoftmaxThreads = 256;
constexpr uint32_t kBarSoftmax = 1;

struct SmemFwd {
  uint64_t q_full, k_full[2], v_full[2], s_full[2], p_full[2], pv_done[2], drain;
  uint32_t tmem_base;
  int abort;
  float red[2][kTile];  // each column half's value of a row (tile maximum, then l)
};

__global__ void __launch_bounds__(kFwdThreads, 1) softmax_fwd_tc(const __grid_constant__ CUtensorMap map_q,
                                                                  const __grid_constant__ CUtensorMap map_k,
                                                                  const __grid_constant__ CUtensorMap map_v,
                                                                  const __grid_constant__ CUtensorMap map_o,
                                                                  float* __restrict__ lse, int H, int64_t Nq,
                                                                  int64_t q_offset, float scale_log2, int qtiles) {
  extern __shared__ uint8_t smem_raw[];
  // the small struct first, then seven 1024-aligned tiles
  SmemFwd* s = reinterpret_cast<SmemFwd*>(smem_raw);
  uint8_t* base = (uint8_t*)(((uintptr_t)(smem_raw + sizeof(SmemFwd)) + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = base;  // Q, then the output tile
  uint8_t* sK = base + kTileBytes;       // two stages
  uint8_t* sV = base + 3 * kTileBytes;   // two stages
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = qtiles - 1 - (int)blockIdx.x;  // heaviest (latest) tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t q0 = (int64_t)qt * kTile;
  // keys up to the last query of the tile that exists
  const int64_t last_pos = q_offset + (q0 + kTile < Nq ? q0 + kTile : Nq) - 1;
  const int nkv = (int)(last_pos / kTile) + 1;
  const volatile int* abort_flag = &s->abort;

  if (tid == 0) {
    prefetch_tmap(&map_q);
    prefetch_tmap(&map_k);
    prefetch_tmap(&map_v);
    prefetch_tmap(&map_o);
    mbar_init(&s->q_full, 1);
    for (int st = 0; st < 2; ++st) {
      mbar_init(&s->k_full[st], 1);
      mbar_init(&s->v_full[st], 1);
      mbar_init(&s->s_full[st], 1);
      mbar_init(&s->p_full[st], kSoftmaxThreads);
      mbar_init(&s->pv_done[st], 1);
    }
    mbar_init(&s->drain, 1);
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
  // S buffers at 0 and 128, O at 256; P in bf16 (the P V MMA's A operand) in
  // two buffers of 64 columns at 384 and 448: K-step kk of buffer st in the 8
  // columns kColP + 64 st + 8 kk, two bf16 per column, the lower K index in
  // the low half
  constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;

  if (warp == 8) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      bool bad = false;
      mbar_arrive_expect_tx(&s->q_full, kTileBytes);
      tma_load_4d(sQ, &map_q, &s->q_full, 0, h, (int)q0, b);
      tma_load_4d(sQ + kBox, &map_q, &s->q_full, 64, h, (int)q0, b);
      int k_out = 0, v_out = 0;  // loads issued (each completes on its stage's barrier)
      for (int j = 0; j < nkv && !bad; ++j) {
        const int st = j & 1;
        const uint32_t use = (uint32_t)(j >> 1);
        if (j >= 2 && !mbar_wait_or_abort(&s->s_full[st], (use - 1) & 1u, SITE_OUT_MMA, abort_flag)) {
          bad = true;  // S_{j-2} has not read K of this stage
          break;
        }
        mbar_arrive_expect_tx(&s->k_full[st], kTileBytes);
        tma_load_4d(sK + st * kTileBytes, &map_k, &s->k_full[st], 0, h, j * kTile, b);
        tma_load_4d(sK + st * kTileBytes + kBox, &map_k, &s->k_full[st], 64, h, j * kTile, b);
        ++k_out;
        if (j >= 2 && !mbar_wait_or_abort(&s->pv_done[st], (use - 1) & 1u, SITE_OUT_MMA, abort_flag)) {
          bad = true;  // P_{j-2} V_{j-2} has not read V of this stage
          break;
        }
        mbar_arrive_expect_tx(&s->v_full[st], kTileBytes);
        tma_load_4d(sV + st * kTileBytes, &map_v, &s->v_full[st], 0, h, j * kTile, b);
        tma_load_4d(sV + st * kTileBytes + kBox, &map_v, &s->v_full[st], 64, h, j * kTile, b);
        ++v_out;
      }
      if (bad) s->abort = 1;
      // every load lands before the CTA can exit: the last one of each stage
      // (bounded waits; earlier ones completed before their stage was refilled)
      for (int j = (k_out > 2 ? k_out - 2 : 0); j < k_out; ++j)
        mbar_wait(&s->k_full[j & 1], (uint32_t)(j >> 1) & 1u, SITE_OUT_TMA);
      for (int j = (v_out > 2 ? v_out - 2 : 0); j < v_out; ++j)
        mbar_wait(&s->v_full[j & 1], (uint32_t)(j >> 1) & 1u, SITE_OUT_TMA);
      mbar_wait(&s->q_full, 0, SITE_OUT_TMA);
    }
  } else if (warp == 9) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t id_kn = idesc_bf16(128, 128, 0, 1);
      const uint32_t aQ = smem_u32(sQ);
      bool bad = !mbar_wait_or_abort(&s->q_full, 0, SITE_OUT_TMA, abort_flag);
      auto pv = [&](int jp) {  // O += P_jp V_jp
        const int sp = jp & 1;
        const uint32_t up = (uint32_t)(jp >> 1) & 1u;
        if (!mbar_wait_or_abort(&s->p_full[sp], up, SITE_OUT_MMA, abort_flag) ||
            !mbar_wait_or_abort(&s->v_full[sp], up, SITE_OUT_TMA, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t aV = smem_u32(sV + sp * kTileBytes);
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_bf16_ts(tmem + kColO, tmem + kColP + 64 * sp + 8 * kk, mnmaj(aV, kk), id_kn,
                      (jp > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&s->pv_done[sp]);
        return true;
      };
      for (int j = 0; j < nkv && !bad; ++j) {
        const int st = j & 1;
        if (!mbar_wait_or_abort(&s->k_full[st], (uint32_t)(j >> 1) & 1u, SITE_OUT_TMA, abort_flag)) {
          bad = true;
          break;
        }
        tc_fence_after();
        const uint32_t aK = smem_u32(sK + st * kTileBytes);
        for (int kk = 0; kk < kD / 16; ++kk)
          mma_bf16(tmem + kColS + st * 128, kmaj(aQ, kk), kmaj(aK, kk), id_kk, kk > 0 ? 1u : 0u);
        mma_commit(&s->s_full[st]);
        if (j >= 1 && !pv(j - 1)) bad = true;
      }
      if (!bad && !pv(nkv - 1)) bad = true;
      if (bad) s->abort = 1;
      // nothing the tensor pipe still runs may outlive the TMEM allocation
      mma_commit(&s->drain);
      mbar_wait(&s->drain, 0, SITE_OUT_MMA);
    }
  } else {
    // ------------------------------------------------------ softmax warps
    const int i = (warp & 3) * 32 + lane;  // query row of the tile = TMEM lane
    const int half = warp >> 2;            // and the column half of it
    const int c0 = half * 64;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int64_t qpos = q_offset + q0 + i;
    float m_used = -INFINITY, l = 0.f;  // l: this half's share of the row sum
    bool bad = false;
    for (int j = 0; j < nkv; ++j) {
      const int st = j & 1;
      const uint32_t use = (uint32_t)(j >> 1) & 1u;
      if (!bad && !mbar_wait_or_abort(&s->s_full[st], use, SITE_OUT_MMA, abort_flag)) bad = true;
      // tcgen05.ld / st are warp-collective: every branch around them is
      // taken by the whole warp
      bad = __any_sync(0xffffffffu, bad);
      float x[64];
      if (!bad) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
          tmem_ld32(lane_base + kColS + st * 128 + c0 + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 32; ++u) x[c * 32 + u] = __uint_as_float(r[u]) * scale_log2;
        }
      } else {
#pragma unroll
        for (int u = 0; u < 64; ++u) x[u] = 0.f;
      }
      const int64_t k0 = (int64_t)j * kTile + c0;
      if (k0 + 63 > qpos) {  // the causal edge crosses this half tile for this row
#pragma unroll
        for (int u = 0; u < 64; ++u)
          if (k0 + u > qpos) x[u] = -INFINITY;
      }
      float mh = x[0];
#pragma unroll
      for (int u = 1; u < 64; ++u) mh = fmaxf(mh, x[u]);
      // the row's tile maximum from both halves: write, barrier, read, barrier
      // (the second keeps the next tile's write from overtaking the read)
      s->red[half][i] = mh;
      named_sync(kBarSoftmax, kSoftmaxThreads);
      const float mt = fmaxf(mh, s->red[half ^ 1][i]);
      named_sync(kBarSoftmax, kSoftmaxThreads);
      // a new maximum far above the one in use: this row's O and l move to it.
      // The warp rescales together when any of its rows needs it (factor 1
      // for the others), after the last P V MMA has written O.
      const bool need = mt > m_used + kRescale;
      const float f = need && j > 0 ? ex2(m_used - mt) : 1.f;
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        if (!bad && !mbar_wait_or_abort(&s->pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, SITE_OUT_MMA,
                                        abort_flag))
          bad = true;
        bad = __any_sync(0xffffffffu, bad);
        if (!bad) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t r[32];
            tmem_ld32(lane_base + kColO + c0 + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 32; ++u) r[u] = __float_as_uint(__uint_as_float(r[u]) * f);
            tmem_st32(lane_base + kColO + c0 + c * 32, r);
          }
          tmem_st_wait();
        }
      }
      if (need) {
        l *= f;
        m_used = mt;
      }
      // P into this stage's TMEM buffer (this thread's 64 columns: K-steps 4
      // half .. 4 half + 3) once the P V MMA of two tiles ago has read it
      if (j >= 2 && !bad &&
          !mbar_wait_or_abort(&s->pv_done[st], (uint32_t)((j - 2) >> 1) & 1u, SITE_OUT_MMA, abort_flag))
        bad = true;
      float rs = 0.f;
      uint32_t pw[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const float p0 = ex2(x[2 * u] - m_used), p1 = ex2(x[2 * u + 1] - m_used);
        rs += p0 + p1;
        pw[u] = pack_bf16(p0, p1);
      }
      tmem_st32(lane_base + kColP + 64 * st + 32 * half, pw);
      tmem_st_wait();
      l += rs;
      tc_fence_before();
      mbar_arrive(&s->p_full[st]);  // arrives even after a failure, so no waiter is left short
    }
    // epilogue: O / l, once the last P V MMA has completed; l of the row is
    // the sum of the two halves'
    const int jl = nkv - 1;
    if (!bad && !mbar_wait_or_abort(&s->pv_done[jl & 1], (uint32_t)(jl >> 1) & 1u, SITE_OUT_MMA, abort_flag))
      bad = true;
    bad = __any_sync(0xffffffffu, bad);
    if (bad) s->abort = 1;
    s->red[half][i] = l;
    named_sync(kBarSoftmax, kSoftmaxThreads);
    const float lr = l + s->red[half ^ 1][i];
    const float inv = 1.f / lr;
    if (!bad) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld32(lane_base + kColO + c0 + c * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8)
          st_tile16(sQ, i, c0 + c * 32 + q8 * 8,
                    make_uint4(pack_bf16(__uint_as_float(r[q8 * 8]) * inv, __uint_as_float(r[q8 * 8 + 1]) * inv),
                               pack_bf16(__uint_as_float(r[q8 * 8 + 2]) * inv, __uint_as_float(r[q8 * 8 + 3]) * inv),
                               pack_bf16(__uint_as_float(r[q8 * 8 + 4]) * inv, __uint_as_float(r[q8 * 8 + 5]) * inv),
                               pack_bf16(__uint_as_float(r[q8 * 8 + 6]) * inv, __uint_as_float(r[q8 * 8 + 7]) * inv)));
      }
      if (half == 0 && q0 + i < Nq) lse[((int64_t)b * H + h) * Nq + q0 + i] = (m_used + __log2f(lr)) * kLn2;
    }
    fence_async_smem();
    named_sync(kBarSoftmax, kSoftmaxThreads);
    if (tid == 0 && !s->abort) {
      tma_store_4d(&map_o, sQ, 0, h, (int)q0, b);
      tma_store_4d(&map_o, sQ + kBox, 64, h, (int)q0, b);
      tma_store_commit();
      tma_store_wait_read0();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ backward
// delta_i = do_i . o_i (fp32) for every query row, [B, H, Nq]: one warp per
// row, four features per lane.
__global__ void __launch_bounds__(256) softmax_delta(const __nv_bfloat16* __restrict__ o,
                                                     const __nv_bfloat16* __restrict__ dout,
                                                     float* __restrict__ delta, int H, int64_t Nq, int64_t rows) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);  // token-major: (b, i, h)
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const uint2 a = *reinterpret_cast<const uint2*>(o + row * kD + lane * 4);
  const uint2 c = *reinterpret_cast<const uint2*>(dout + row * kD + lane * 4);
  const float2 a0 = unpack_bf16(a.x), a1 = unpack_bf16(a.y), c0 = unpack_bf16(c.x), c1 = unpack_bf16(c.y);
  float acc = a0.x * c0.x + a0.y * c0.y + a1.x * c1.x + a1.y * c1.y;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    const int h = (int)(row % H);
    const int64_t i = (row / H) % Nq;
    const int64_t b = row / (H * Nq);
    delta[(b * H + h) * Nq + i] = acc;
  }
}

constexpr uint32_t kBarEpi = 1;  // named barrier of the gradient kernels' epilogue warps
constexpr int kDqThreads = 576;   // softmax_dq_tc: warps 0-15 epilogue, 16 TMA, 17 MMA
constexpr int kDqEpi = 512;  // epilogue threads of both gradient kernels
constexpr int kDkdvThreads = 576;  // softmax_dkdv_tc: warps 0-15 epilogue, 16 TMA, 17 MMA

// 16 consecutive fp32 columns of this thread's TMEM lane (warp-collective).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Reads the S-type and dP-type accumulators of this thread's row (TMEM lane)
// over the 32 columns of chunk cc of column half `half` (half * 64 + cc * 32
// ..), forms p = exp2(s c - lse2) (0 where masked) and ds = p (dp - delta) per
// column, and writes both back into TMEM in bf16, over the accumulator
// columns this thread has just read, as the A operand of the next MMAs: the
// 16 columns of pass ps (K-step kk = 2 sub + ps of those MMAs, sub = 2 half +
// cc) into the 8 columns colS + 32 sub + 8 ps (P) and colP + 32 sub + 8 ps
// (dS), two bf16 per column, the lower K index in the low half. Chunk 0 of
// both halves is the MMAs' K-steps 0, 1, 4, 5, chunk 1 their K-steps 2, 3, 6,
// 7. keep(c) says whether column c is inside the causal mask and the
// sequence; lse2 / dl give the column's values through the callbacks;
// visible = 1 (every column of the chunk inside the mask) or 0 (none) skips
// the per-column test.
template <class Keep, class Lse, class Dl>
__device__ __forceinline__ void p_ds_rows_tmem(uint32_t lane_base, uint32_t colS, uint32_t colP, int half, int cc,
                                               float c2, Keep keep, Lse lse2, Dl dl, int visible) {
  const int col0 = half * 64 + cc * 32;
#pragma unroll 1
  for (int ps = 0; ps < 2; ++ps) {
    const int cb = col0 + ps * 16;
    uint32_t rs[16], rp[16];
    tmem_ld16(lane_base + colS + cb, rs);
    tmem_ld16(lane_base + colP + cb, rp);
    tmem_ld_wait();
    float p[16], ds[16];
    if (visible == 1) {
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int c = cb + u;
        p[u] = ex2(__uint_as_float(rs[u]) * c2 - lse2(c));
        ds[u] = p[u] * (__uint_as_float(rp[u]) - dl(c));
      }
    } else if (visible == 0) {
#pragma unroll
      for (int u = 0; u < 16; ++u) p[u] = ds[u] = 0.f;
    } else {
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int c = cb + u;
        const float e = ex2(__uint_as_float(rs[u]) * c2 - lse2(c));
        p[u] = keep(c) ? e : 0.f;
        ds[u] = p[u] * (__uint_as_float(rp[u]) - dl(c));
      }
    }
    uint32_t wp[8], wd[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      wp[u] = pack_bf16(p[2 * u], p[2 * u + 1]);
      wd[u] = pack_bf16(ds[2 * u], ds[2 * u + 1]);
    }
    tmem_st8(lane_base + colS + col0 + 8 * ps, wp);
    tmem_st8(lane_base + colP + col0 + 8 * ps, wd);
  }
  tmem_st_wait();
}

struct SmemDkdv {
  uint64_t kv_full, full[3], empty[3], ld_full, s_full, p_half, p_full, dv_done, mma2_done, drain;
  uint32_t tmem_base;
  int abort;
  float lse2[kTile], dl[kTile];  // the current query tile's lse (log2 units) and delta
};

__global__ void __launch_bounds__(kDkdvThreads, 1) softmax_dkdv_tc(
    const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_do,
    const __grid_constant__ CUtensorMap map_dk, const __grid_constant__ CUtensorMap map_dv,
    const float* __restrict__ lse, const float* __restrict__ delta, int H, int64_t Nq, int64_t q_offset,
    float scale, int qtiles) {
  extern __shared__ uint8_t smem_raw[];
  // the small struct first, then seven 1024-aligned tiles (all of 227 KB but
  // a little)
  SmemDkdv* s = reinterpret_cast<SmemDkdv*>(smem_raw);
  uint8_t* base = (uint8_t*)(((uintptr_t)(smem_raw + sizeof(SmemDkdv)) + 1023) & ~(uintptr_t)1023);
  uint8_t* sK = base;
  uint8_t* sV = base + kTileBytes;
  uint8_t* ring = base + 2 * kTileBytes;  // three slots: Q_0, dO_0, Q_1, dO_1, ...
  uint8_t* sPt = base + 5 * kTileBytes;   // dK out
  uint8_t* sDSt = base + 6 * kTileBytes;  // dV out
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t k0 = (int64_t)kt * kTile;
  // the query tiles that see a key of this tile: q_offset + i >= k0 for some i
  const int64_t first_q = (k0 > q_offset ? k0 - q_offset : (int64_t)0);
  const int qt0 = first_q < Nq ? (int)(first_q / kTile) : qtiles;
  const int n = qtiles - qt0;  // may be 0: no query reaches these keys
  const volatile int* abort_flag = &s->abort;
  const float c2 = scale * kLog2e;

  if (tid == 0) {
    prefetch_tmap(&map_q);
    prefetch_tmap(&map_k);
    prefetch_tmap(&map_v);
    prefetch_tmap(&map_do);
    prefetch_tmap(&map_dk);
    prefetch_tmap(&map_dv);
    mbar_init(&s->kv_full, 1);
    for (int r = 0; r < 3; ++r) {
      mbar_init(&s->full[r], 1);
      mbar_init(&s->empty[r], 1);
    }
    mbar_init(&s->ld_full, 1);
    mbar_init(&s->s_full, 1);
    mbar_init(&s->p_half, 256);
    mbar_init(&s->p_full, 256);
    mbar_init(&s->dv_done, 1);
    mbar_init(&s->mma2_done, 1);
    mbar_init(&s->drain, 1);
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
  // S^T, then P^T (bf16, the dV MMA's A operand) over its first 64 columns;
  // dP^T, then dS^T (the dK MMA's) likewise; the dV and dK accumulators
  constexpr uint32_t kColS = 0, kColP = 128, kColV = 256, kColK = 384;

  if (warp == 16) {
    // ---------------------------------------------------------- TMA producer
    bool bad = false;
    int issued = 0;  // ring loads issued
    if (lane == 0 && n > 0) {
      mbar_arrive_expect_tx(&s->kv_full, 2 * kTileBytes);
      tma_load_4d(sK, &map_k, &s->kv_full, 0, h, (int)k0, b);
      tma_load_4d(sK + kBox, &map_k, &s->kv_full, 64, h, (int)k0, b);
      tma_load_4d(sV, &map_v, &s->kv_full, 0, h, (int)k0, b);
      tma_load_4d(sV + kBox, &map_v, &s->kv_full, 64, h, (int)k0, b);
    }
    for (int x = 0; x < 2 * n && !bad; ++x) {
      const int i = x >> 1, slot = x % 3;
      const int64_t q0 = (int64_t)(qt0 + i) * kTile;
      if (lane == 0) {
        if (x >= 3 && !mbar_wait_or_abort(&s->empty[slot], (uint32_t)(x / 3 - 1) & 1u, SITE_BWD_MMA, abort_flag))
          bad = true;
        if (!bad) {
          uint8_t* dst = ring + slot * kTileBytes;
          const CUtensorMap* m = (x & 1) ? &map_do : &map_q;
          mbar_arrive_expect_tx(&s->full[slot], kTileBytes);
          tma_load_4d(dst, m, &s->full[slot], 0, h, (int)q0, b);
          tma_load_4d(dst + kBox, m, &s->full[slot], 64, h, (int)q0, b);
          ++issued;
        }
      }
      // the last tile's epilogue has read lse and delta (both chunk groups)
      if (lane == 0 && !bad && (x & 1) == 0 && i > 0 &&
          (!mbar_wait_or_abort(&s->p_half, (uint32_t)(i - 1) & 1u, SITE_BWD_MMA, abort_flag) ||
           !mbar_wait_or_abort(&s->p_full, (uint32_t)(i - 1) & 1u, SITE_BWD_MMA, abort_flag)))
        bad = true;
      bad = __shfl_sync(0xffffffffu, bad, 0);
      if (!bad && (x & 1) == 0) {
        // the tile's lse and delta, by the whole warp; their loads run under
        // the last tile's dV / dK MMAs and this tile's S^T / dP^T
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = lane * 4 + u;
          const int64_t qi = q0 + c;
          const bool in = qi < Nq;
          s->lse2[c] = in ? lse[((int64_t)b * H + h) * Nq + qi] * kLog2e : 0.f;
          s->dl[c] = in ? delta[((int64_t)b * H + h) * Nq + qi] : 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s->ld_full);
      }
    }
    if (lane == 0) {
      if (bad) s->abort = 1;
      for (int x = (issued > 3 ? issued - 3 : 0); x < issued; ++x)
        mbar_wait(&s->full[x % 3], (uint32_t)(x / 3) & 1u, SITE_BWD_TMA);
      if (n > 0) mbar_wait(&s->kv_full, 0, SITE_BWD_TMA);
    }
  } else if (warp == 17) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t id_kn = idesc_bf16(128, 128, 0, 1);
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
      bool bad = !mbar_wait_or_abort(&s->kv_full, 0, SITE_BWD_TMA, abort_flag);
      for (int i = 0; i < n && !bad; ++i) {
        const int xq = 2 * i, xd = 2 * i + 1;
        const int sq = xq % 3, sd = xd % 3;
        const uint32_t aQ = smem_u32(ring + sq * kTileBytes), aO = smem_u32(ring + sd * kTileBytes);
        if (!mbar_wait_or_abort(&s->full[sq], (uint32_t)(xq / 3) & 1u, SITE_BWD_TMA, abort_flag)) {
          bad = true;
          break;
        }
        // S^T overwrites P^T: the last tile's dV MMAs have read it (its dK
        // MMAs are still running, so the wait costs little tensor time)
        if (i > 0 && !mbar_wait_or_abort(&s->dv_done, (uint32_t)(i - 1) & 1u, SITE_BWD_MMA, abort_flag)) {
          bad = true;
          break;
        }
        tc_fence_after();
        for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + kColS, kmaj(aK, kk), kmaj(aQ, kk), id_kk, kk > 0);
        if (!mbar_wait_or_abort(&s->full[sd], (uint32_t)(xd / 3) & 1u, SITE_BWD_TMA, abort_flag)) {
          bad = true;
          break;
        }
        // dP^T overwrites dS^T: the last tile's dK MMAs have read it (under S^T)
        if (i > 0 && !mbar_wait_or_abort(&s->mma2_done, (uint32_t)(i - 1) & 1u, SITE_BWD_MMA, abort_flag)) {
          bad = true;
          break;
        }
        tc_fence_after();
        for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + kColP, kmaj(aV, kk), kmaj(aO, kk), id_kk, kk > 0);
        mma_commit(&s->s_full);
        // dV += P^T dO and dK += dS^T Q over the query columns the epilogue
        // has finished: K-steps 0, 1, 4, 5 (its first chunk), then 2, 3, 6, 7
        bool part_ok = true;
        for (int pc = 0; pc < 2 && part_ok; ++pc) {
          if (!mbar_wait_or_abort(pc == 0 ? &s->p_half : &s->p_full, (uint32_t)i & 1u, SITE_BWD_MMA, abort_flag)) {
            part_ok = false;
            break;
          }
          tc_fence_after();
          // K-step kk's A operand: 8 TMEM columns at 32 (kk / 2) + 8 (kk % 2)
          for (int q = 0; q < 4; ++q) {
            const int kk = (q >> 1) * 4 + pc * 2 + (q & 1);
            mma_bf16_ts(tmem + kColV, tmem + kColS + 32 * (kk >> 1) + 8 * (kk & 1), mnmaj(aO, kk), id_kn,
                        (i > 0 || pc > 0 || q > 0) ? 1u : 0u);
          }
          if (pc == 1) mma_commit(&s->dv_done);
          for (int q = 0; q < 4; ++q) {
            const int kk = (q >> 1) * 4 + pc * 2 + (q & 1);
            mma_bf16_ts(tmem + kColK, tmem + kColP + 32 * (kk >> 1) + 8 * (kk & 1), mnmaj(aQ, kk), id_kn,
                        (i > 0 || pc > 0 || q > 0) ? 1u : 0u);
          }
        }
        if (!part_ok) {
          bad = true;
          break;
        }
        mma_commit(&s->empty[sq]);
        mma_commit(&s->empty[sd]);
        mma_commit(&s->mma2_done);
      }
      if (bad) s->abort = 1;
      mma_commit(&s->drain);
      mbar_wait(&s->drain, 0, SITE_BWD_MMA);
    }
  } else {
    // --------------------------------------------- epilogue warps (0-15)
    // key row of the tile; this thread's 32 query columns sub * 32.., which
    // are chunk cc = sub & 1 of column half sub >> 1 (the p_half / p_full split)
    const int row = (warp & 3) * 32 + lane, sub = warp >> 2;
    const int half = sub >> 1, cc = sub & 1;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int64_t kpos = k0 + row;
    bool bad = false;
    for (int i = 0; i < n; ++i) {
      const int64_t q0 = (int64_t)(qt0 + i) * kTile;
      if (!bad && !mbar_wait_or_abort(&s->s_full, (uint32_t)i & 1u, SITE_BWD_MMA, abort_flag)) bad = true;
      if (!bad && !mbar_wait_or_abort(&s->ld_full, (uint32_t)i & 1u, SITE_BWD_TMA, abort_flag)) bad = true;
      // (the last tile's dV and dK MMAs, which read P^T and dS^T from TMEM,
      // completed before this tile's S^T and dP^T were issued)
      bad = __any_sync(0xffffffffu, bad);  // the TMEM loads below are warp-collective
      const float* L = s->lse2;
      const float* Dl = s->dl;
      auto keep = [&](int c) { return q0 + c < Nq && q_offset + q0 + c >= kpos; };
      // the chunk's columns c = sub * 32 .. + 31: all inside the mask, none, or some
      const int64_t cfirst = q0 + sub * 32, clast = cfirst + 31;
      const int visible = (clast < Nq && q_offset + cfirst >= kpos) ? 1
                          : (cfirst >= Nq || q_offset + clast < kpos) ? 0 : -1;
      if (!bad) {
        tc_fence_after();
        p_ds_rows_tmem(lane_base, kColS, kColP, half, cc, c2, keep, [&](int c) { return L[c]; },
                       [&](int c) { return Dl[c]; }, visible);
      }
      tc_fence_before();
      mbar_arrive(cc == 0 ? &s->p_half : &s->p_full);  // the MMA takes each chunk as it is done
    }
    if (n > 0 && !bad && !mbar_wait_or_abort(&s->mma2_done, (uint32_t)(n - 1) & 1u, SITE_BWD_MMA, abort_flag))
      bad = true;
    bad = __any_sync(0xffffffffu, bad);
    if (bad) s->abort = 1;
    if (!bad) {
      if (n > 0) {
        // dK (times scale) and dV, columns sub * 32.. of row `row`, into the P^T and dS^T tiles
        tc_fence_after();
#pragma unroll 1
        for (int t2 = 0; t2 < 2; ++t2) {
          uint32_t r[32];
          tmem_ld32(lane_base + (t2 == 0 ? kColK : kColV) + sub * 32, r);
          tmem_ld_wait();
          const float f = t2 == 0 ? scale : 1.f;
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __uint_as_float(r[q8 * 8 + u]) * f;
            st_tile16(t2 == 0 ? sPt : sDSt, row, sub * 32 + q8 * 8,
                      make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                                 pack_bf16(v[6], v[7])));
          }
        }
      } else {
        // no query sees these keys: their gradients are zero
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          st_tile16(sPt, row, sub * 32 + c8 * 8, make_uint4(0u, 0u, 0u, 0u));
          st_tile16(sDSt, row, sub * 32 + c8 * 8, make_uint4(0u, 0u, 0u, 0u));
        }
      }
    }
    fence_async_smem();
    named_sync(kBarEpi, kDqEpi);
    if (tid == 0 && !s->abort) {
      tma_store_4d(&map_dk, sPt, 0, h, (int)k0, b);
      tma_store_4d(&map_dk, sPt + kBox, 64, h, (int)k0, b);
      tma_store_4d(&map_dv, sDSt, 0, h, (int)k0, b);
      tma_store_4d(&map_dv, sDSt + kBox, 64, h, (int)k0, b);
      tma_store_commit();
      tma_store_wait_read0();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// softmax_dq_tc: per key tile j, S = Q K_j^T and dP = dO V_j^T (N = 128) into
// TMEM, the epilogue's sixteen warps (four per TMEM lane quarter, 32 key
// columns each: chunk sub & 1 of column half sub >> 1) turn them into dS in
// bf16, and dQ += dS K_j takes the K-steps 0, 1, 4, 5 once the first chunks are
// written and 2, 3, 6, 7 once the second ones are. Only the tile on the causal
// diagonal masks element by element.
struct SmemDq {
  uint64_t qd_full, k_full[2], v_full[2], kv_empty[2], s_full, ds_half, ds_full, dq_done, drain;
  uint32_t tmem_base;
  int abort;
};

__global__ void __launch_bounds__(kDqThreads, 1) softmax_dq_tc(
    const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_do,
    const __grid_constant__ CUtensorMap map_dq, const float* __restrict__ lse, const float* __restrict__ delta,
    int H, int64_t Nq, int64_t q_offset, float scale, int qtiles) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = base;                   // Q, then dQ out
  uint8_t* sO = base + kTileBytes;      // dO
  uint8_t* sK = base + 2 * kTileBytes;  // two stages
  uint8_t* sV = base + 4 * kTileBytes;  // two stages
  SmemDq* s = reinterpret_cast<SmemDq*>(base + 7 * kTileBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = qtiles - 1 - (int)blockIdx.x;  // heaviest tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t q0 = (int64_t)qt * kTile;
  const int64_t last_pos = q_offset + (q0 + kTile < Nq ? q0 + kTile : Nq) - 1;
  const int nkv = (int)(last_pos / kTile) + 1;
  const volatile int* abort_flag = &s->abort;
  const float c2 = scale * kLog2e;

  if (tid == 0) {
    prefetch_tmap(&map_q);
    prefetch_tmap(&map_k);
    prefetch_tmap(&map_v);
    prefetch_tmap(&map_do);
    prefetch_tmap(&map_dq);
    mbar_init(&s->qd_full, 1);
    for (int st = 0; st < 2; ++st) {
      mbar_init(&s->k_full[st], 1);
      mbar_init(&s->v_full[st], 1);
      mbar_init(&s->kv_empty[st], 1);
    }
    mbar_init(&s->s_full, 1);
    mbar_init(&s->ds_half, kDqEpi / 2);
    mbar_init(&s->ds_full, kDqEpi / 2);
    mbar_init(&s->dq_done, 1);
    mbar_init(&s->drain, 1);
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
  // S, dP, the dQ accumulator; dS in bf16 (the dQ MMA's A operand: K-step kk
  // in the 8 columns kColD + 8 kk, two bf16 per column, the lower K index in
  // the low half)
  constexpr uint32_t kColS = 0, kColP = 128, kColQ = 256, kColD = 384;

  if (warp == 16) {
    if (lane == 0) {
      bool bad = false;
      mbar_arrive_expect_tx(&s->qd_full, 2 * kTileBytes);
      tma_load_4d(sQ, &map_q, &s->qd_full, 0, h, (int)q0, b);
      tma_load_4d(sQ + kBox, &map_q, &s->qd_full, 64, h, (int)q0, b);
      tma_load_4d(sO, &map_do, &s->qd_full, 0, h, (int)q0, b);
      tma_load_4d(sO + kBox, &map_do, &s->qd_full, 64, h, (int)q0, b);
      int issued = 0;
      for (int j = 0; j < nkv && !bad; ++j) {
        const int st = j & 1;
        if (j >= 2 &&
            !mbar_wait_or_abort(&s->kv_empty[st], (uint32_t)((j >> 1) - 1) & 1u, SITE_BWD_MMA, abort_flag)) {
          bad = true;
          break;
        }
        mbar_arrive_expect_tx(&s->k_full[st], kTileBytes);
        tma_load_4d(sK + st * kTileBytes, &map_k, &s->k_full[st], 0, h, j * kTile, b);
        tma_load_4d(sK + st * kTileBytes + kBox, &map_k, &s->k_full[st], 64, h, j * kTile, b);
        mbar_arrive_expect_tx(&s->v_full[st], kTileBytes);
        tma_load_4d(sV + st * kTileBytes, &map_v, &s->v_full[st], 0, h, j * kTile, b);
        tma_load_4d(sV + st * kTileBytes + kBox, &map_v, &s->v_full[st], 64, h, j * kTile, b);
        ++issued;
      }
      if (bad) s->abort = 1;
      for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j) {
        mbar_wait(&s->k_full[j & 1], (uint32_t)(j >> 1) & 1u, SITE_BWD_TMA);
        mbar_wait(&s->v_full[j & 1], (uint32_t)(j >> 1) & 1u, SITE_BWD_TMA);
      }
      mbar_wait(&s->qd_full, 0, SITE_BWD_TMA);
    }
  } else if (warp == 17) {
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t id_kn = idesc_bf16(128, 128, 0, 1);
      const uint32_t aQ = smem_u32(sQ), aO = smem_u32(sO);
      bool bad = !mbar_wait_or_abort(&s->qd_full, 0, SITE_BWD_TMA, abort_flag);
      for (int j = 0; j < nkv && !bad; ++j) {
        const int st = j & 1;
        const uint32_t use = (uint32_t)(j >> 1) & 1u;
        const uint32_t aK = smem_u32(sK + st * kTileBytes), aV = smem_u32(sV + st * kTileBytes);
        if (!mbar_wait_or_abort(&s->k_full[st], use, SITE_BWD_TMA, abort_flag)) {
          bad = true;
          break;
        }
        tc_fence_after();
        for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + kColS, kmaj(aQ, kk), kmaj(aK, kk), id_kk, kk > 0);
        if (!mbar_wait_or_abort(&s->v_full[st], use, SITE_BWD_TMA, abort_flag)) {
          bad = true;
          break;
        }
        tc_fence_after();
        for (int kk = 0; kk < kD / 16; ++kk) mma_bf16(tmem + kColP, kmaj(aO, kk), kmaj(aV, kk), id_kk, kk > 0);
        mma_commit(&s->s_full);
        // dQ += dS K over the key columns the epilogue has finished: K-steps
        // 0, 1, 4, 5 (the first chunks), then 2, 3, 6, 7
        bool part_ok = true;
        for (int pc = 0; pc < 2; ++pc) {
          if (!mbar_wait_or_abort(pc == 0 ? &s->ds_half : &s->ds_full, (uint32_t)j & 1u, SITE_BWD_MMA, abort_flag)) {
            part_ok = false;
            break;
          }
          tc_fence_after();
          for (int q = 0; q < 4; ++q) {
            const int kk = (q >> 1) * 4 + pc * 2 + (q & 1);
            mma_bf16_ts(tmem + kColQ, tmem + kColD + 8 * kk, mnmaj(aK, kk), id_kn,
                        (j > 0 || pc > 0 || q > 0) ? 1u : 0u);
          }
        }
        if (!part_ok) {
          bad = true;
          break;
        }
        mma_commit(&s->kv_empty[st]);
        mma_commit(&s->dq_done);
      }
      if (bad) s->abort = 1;
      mma_commit(&s->drain);
      mbar_wait(&s->drain, 0, SITE_BWD_MMA);
    }
  } else {
    // query row `row` of the tile; key columns sub * 32 .. + 31 (two passes of 16)
    const int row = (warp & 3) * 32 + lane, sub = warp >> 2;
    const int cc = sub & 1;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int64_t qi = q0 + row;
    const int64_t qpos = q_offset + qi;
    const bool in = qi < Nq;
    const float lse2 = in ? lse[((int64_t)b * H + h) * Nq + qi] * kLog2e : 0.f;
    const float dl = in ? delta[((int64_t)b * H + h) * Nq + qi] : 0.f;
    bool bad = false;
    for (int j = 0; j < nkv; ++j) {
      const int64_t kc = (int64_t)j * kTile + sub * 32;  // key of this thread's first column
      // columns u <= lim are inside the causal mask (lim >= 31: all, < 0: none)
      const int64_t lim64 = in ? qpos - kc : -1;
      const int lim = lim64 < -1 ? -1 : (lim64 > 31 ? 31 : (int)lim64);
      if (!bad && !mbar_wait_or_abort(&s->s_full, (uint32_t)j & 1u, SITE_BWD_MMA, abort_flag)) bad = true;
      if (j > 0 && !bad && !mbar_wait_or_abort(&s->dq_done, (uint32_t)(j - 1) & 1u, SITE_BWD_MMA, abort_flag))
        bad = true;  // the last dQ MMAs have read dS
      bad = __any_sync(0xffffffffu, bad);  // the TMEM loads below are warp-collective
      if (!bad) {
        tc_fence_after();
#pragma unroll 1
        for (int ps = 0; ps < 2; ++ps) {
          const int cb = sub * 32 + ps * 16;
          uint32_t rs[16], rp[16];
          tmem_ld16(lane_base + kColS + cb, rs);
          tmem_ld16(lane_base + kColP + cb, rp);
          tmem_ld_wait();
          const int lp = lim - ps * 16;  // this pass's columns u <= lp are inside the mask
          float ds[16];
          if (lp >= 15) {
#pragma unroll
            for (int u = 0; u < 16; ++u)
              ds[u] = ex2(__uint_as_float(rs[u]) * c2 - lse2) * (__uint_as_float(rp[u]) - dl);
          } else if (lp < 0) {
#pragma unroll
            for (int u = 0; u < 16; ++u) ds[u] = 0.f;
          } else {
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const float p = u <= lp ? ex2(__uint_as_float(rs[u]) * c2 - lse2) : 0.f;
              ds[u] = p * (__uint_as_float(rp[u]) - dl);
            }
          }
          uint32_t w[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) w[u] = pack_bf16(ds[2 * u], ds[2 * u + 1]);
          tmem_st8(lane_base + kColD + 16 * sub + 8 * ps, w);  // K-step 2 sub + ps
        }
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(cc == 0 ? &s->ds_half : &s->ds_full);  // the MMA takes each chunk group as it is done
    }
    if (!bad && !mbar_wait_or_abort(&s->dq_done, (uint32_t)(nkv - 1) & 1u, SITE_BWD_MMA, abort_flag)) bad = true;
    bad = __any_sync(0xffffffffu, bad);
    if (bad) s->abort = 1;
    if (!bad) {
      // dQ (every MMA that read Q is done): columns sub * 32.. of row `row`, times scale, into the Q tile
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(lane_base + kColQ + sub * 32, r);
      tmem_ld_wait();
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __uint_as_float(r[q8 * 8 + u]) * scale;
        st_tile16(sQ, row, sub * 32 + q8 * 8,
                  make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                             pack_bf16(v[6], v[7])));
      }
    }
    fence_async_smem();
    named_sync(kBarEpi, kDqEpi);
    if (tid == 0 && !s->abort) {
      tma_store_4d(&map_dq, sQ, 0, h, (int)q0, b);
      tma_store_4d(&map_dq, sQ + kBox, 64, h, (int)q0, b);
      tma_store_commit();
      tma_store_wait_read0();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace tc_softmax_detail

bool tc_softmax_ok(int dtype, int d) { return dtype == LASP_BF16 && d == tc_softmax_detail::kD; }

cudaError_t tc_softmax_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int64_t Nq,
                           int64_t Nk, int64_t q_offset, float scale, cudaStream_t st) {
  using namespace tc_softmax_detail;
  CUtensorMap mq, mk, mv, mo;
  if (!make_token_map(&mq, q, B, H, Nq, kD, kTile) || !make_token_map(&mk, k, B, H, Nk, kD, kTile) ||
      !make_token_map(&mv, v, B, H, Nk, kD, kTile) || !make_token_map(&mo, o, B, H, Nq, kD, kTile))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(SmemFwd) + 1023 + 7 * (size_t)kTileBytes;
  cudaError_t e = cudaFuncSetAttribute(softmax_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int qtiles = (int)((Nq + kTile - 1) / kTile);
  softmax_fwd_tc<<<dim3((unsigned)qtiles, H, B), kFwdThreads, smem, st>>>(mq, mk, mv, mo, lse, H, Nq, q_offset,
                                                                          scale * kLog2e, qtiles);
  return cudaGetLastError();
}

}  // namespace lasp

namespace lasp {

cudaError_t tc_softmax_delta(const void* o, const void* dout, float* delta, int B, int H, int64_t Nq,
                             cudaStream_t st) {
  using namespace tc_softmax_detail;
  const int64_t rows = (int64_t)B * Nq * H;
  softmax_delta<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>((const __nv_bfloat16*)o, (const __nv_bfloat16*)dout,
                                                           delta, H, Nq, rows);
  return cudaGetLastError();
}

cudaError_t tc_softmax_dkdv(const void* q, const void* k, const void* v, const float* lse, const void* dout,
                            void* dk, void* dv, const float* delta, int B, int H, int64_t Nq, int64_t Nk,
                            int64_t q_offset, float scale, cudaStream_t st) {
  using namespace tc_softmax_detail;
  CUtensorMap mq, mk, mv, mdo, mdk, mdv;
  if (!make_token_map(&mq, q, B, H, Nq, kD, kTile) || !make_token_map(&mk, k, B, H, Nk, kD, kTile) ||
      !make_token_map(&mv, v, B, H, Nk, kD, kTile) || !make_token_map(&mdo, dout, B, H, Nq, kD, kTile) ||
      !make_token_map(&mdk, dk, B, H, Nk, kD, kTile) || !make_token_map(&mdv, dv, B, H, Nk, kD, kTile))
    return cudaErrorInvalidValue;
  const int qtiles = (int)((Nq + kTile - 1) / kTile);
  const int ktiles = (int)((Nk + kTile - 1) / kTile);
  const size_t smem = sizeof(SmemDkdv) + 1023 + 7 * (size_t)kTileBytes;
  cudaError_t e = cudaFuncSetAttribute(softmax_dkdv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  softmax_dkdv_tc<<<dim3((unsigned)ktiles, H, B), kDkdvThreads, smem, st>>>(mq, mk, mv, mdo, mdk, mdv, lse, delta, H,
                                                                          Nq, q_offset, scale, qtiles);
  return cudaGetLastError();
}

cudaError_t tc_softmax_dq(const void* q, const void* k, const void* v, const float* lse, const void* dout, void* dq,
                          const float* delta, int B, int H, int64_t Nq, int64_t Nk, int64_t q_offset, float scale,
                          cudaStream_t st) {
  using namespace tc_softmax_detail;
  CUtensorMap mq, mk, mv, mdo, mdq;
  if (!make_token_map(&mq, q, B, H, Nq, kD, kTile) || !make_token_map(&mk, k, B, H, Nk, kD, kTile) ||
      !make_token_map(&mv, v, B, H, Nk, kD, kTile) || !make_token_map(&mdo, dout, B, H, Nq, kD, kTile) ||
      !make_token_map(&mdq, dq, B, H, Nq, kD, kTile))
    return cudaErrorInvalidValue;
  const int qtiles = (int)((Nq + kTile - 1) / kTile);
  const size_t smem = 1024 + 7 * (size_t)kTileBytes + sizeof(SmemDq);
  cudaError_t e = cudaFuncSetAttribute(softmax_dq_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  softmax_dq_tc<<<dim3((unsigned)qtiles, H, B), kDqThreads, smem, st>>>(mq, mk, mv, mdo, mdq, lse, delta, H, Nq,
                                                                        q_offset, scale, qtiles);
  return cudaGetLastError();
}

}  // namespace lasp
