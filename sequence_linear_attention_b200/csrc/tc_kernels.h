// Tensor-core (tcgen05 / TMEM / TMA) kernels for bf16 inputs, and the
// predicates that say which sizes they take. The CUDA-core kernels of
// k_simt.cu serve every other size.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace lasp {

// Chunk states on tensor cores: bf16, d = 128, C a multiple of 16. The
// CUDA-core kernels take every size for which a predicate is false.
bool tc_states_ok(int dtype, int d, int64_t C);
cudaError_t tc_chunk_states(const void* a, const void* b, const float* decay, float* M, int B, int H, int64_t N,
                            int d, int C, int kind, cudaStream_t st);

// The same, writing chunk c's state to slot c * slot_stride + slot_offset of
// an array of t_out states per (b, h).
// bh0, nbh: only the (b, h) pairs bh0 .. bh0 + nbh - 1 (b-major; nbh < 0: all).
cudaError_t tc_chunk_states_slots(const void* a, const void* b, const float* decay, float* M, int B, int H,
                                  int64_t N, int d, int C, int kind, int64_t t_out, int slot_stride, int slot_offset,
                                  cudaStream_t st, int64_t bh0 = 0, int64_t nbh = -1);

// Forward walk over segments of G tokens with the state on chip (bf16,
// d = 128, C a multiple of 128 or a divisor of it, N a multiple of max(C, 128),
// G = walk_segment_tokens(N, C)). P must hold, in the slot of each segment's
// first chunk, the state entering that segment; the walk writes o and fills the
// cache: fp32 P_c at the other chunk starts when C > 256, otherwise the bf16
// operand tile of the state entering each 128-token tile in the slot of the
// tile's first chunk (C = 256: both tiles of a chunk in the two halves of its
// slot).
bool tc_fwd_walk_ok(int dtype, int d, int64_t C, int64_t N);
int walk_segment_tokens(int64_t N, int C);
cudaError_t tc_fwd_walk(const void* q, const void* k, const void* v, const float* decay, float* P, void* o, int B,
                        int H, int64_t N, int d, int C, int G, int num_sms, cudaStream_t st, int64_t bh0 = 0,
                        int64_t nbh = -1);

// Backward walk over segments with the gradient state on chip (bf16, d = 128,
// C dividing 128 with N a multiple of 128, or C = 256 with N a multiple of 256). R must hold, in the slot of each
// segment's last chunk, the gradient state entering that chunk from the tokens
// after the segment; the walk writes dq, dk, dv (R of the other chunks stays on
// chip). P is the forward walk's cache of bf16 operand tiles.
bool tc_bwd_walk_ok(int dtype, int d, int64_t C, int64_t N);
cudaError_t tc_bwd_walk(const void* q, const void* k, const void* v, const void* dout, const float* decay,
                        const float* P, float* R, void* dq, void* dk, void* dv, int B, int H, int64_t N, int d, int C,
                        int G, int num_sms, cudaStream_t st, int64_t bh0 = 0, int64_t nbh = -1);

bool tc_out_ok(int dtype, int d, int64_t C);
cudaError_t tc_chunk_out(const void* q, const void* k, const void* v, const float* decay, const float* P, void* o,
                         int B, int H, int64_t N, int d, int C, cudaStream_t st);

bool tc_bwd_ok(int dtype, int d, int64_t C);
cudaError_t tc_chunk_bwd(const void* q, const void* k, const void* v, const void* dout, const float* decay,
                         const float* P, const float* Rs, void* dq, void* dk, void* dv, int B, int H, int64_t N,
                         int d, int C, cudaStream_t st);

// Bidirectional (unmasked) form, bf16, d = 128, N a multiple of 128
// (k_tc_bidir.cu): the fp32 sum of nseg segment states of each (b, h) and its
// bf16 operand tile; and Y = X S (b_kmajor = 0) or X S^T (b_kmajor = 1) per
// 128-token tile of X with S the (b, h)'s tile.
bool tc_bidir_ok(int dtype, int d, int64_t N);
cudaError_t bidir_total(const float* seg, float* total, void* tiles, int B, int H, int nseg, cudaStream_t st);
cudaError_t tc_bidir_apply(const void* x, const void* stiles, void* y, int B, int H, int64_t N, int d, int b_kmajor,
                           int num_sms, cudaStream_t st);

// Gated form on the tensor cores, bf16, d = 128, C dividing 128, N a multiple
// of 128 (k_tc_gla.cu), on 128-token tiles: the states of k_gla_simt.cu per
// tile (kind 0 from (k, v) with the log-gate totals, kind 1 from (q, do)) into
// slot tile * stride + offset of an array of t_slots chunk states; the output
// given P in the slot of each tile's first chunk; the gradients given that P
// and, for segments of `tiles` tiles, the R entering each segment in the slot
// of its last chunk (stride = chunks per tile): the kernel forms every other
// tile's R on its walk through the segment, in the slot of the segment's first
// chunk, which it overwrites.
bool tc_gla_ok(int dtype, int d, int64_t C, int64_t N);
// span_flag (may be NULL): set to 1 when a tile's log-gates span more than the
// factorized form of the output and backward kernels takes; `run` makes a
// launch conditional on such a flag (kernels.h).
cudaError_t tc_gla_chunk_states(const void* x, const void* y, const float* g, float* M, float* gsum,
                                float* gsum_tile, int B, int H, int64_t N, int kind, int64_t t_slots, int stride,
                                int offset, int tiles, int tstride, cudaStream_t st, int* span_flag = nullptr,
                                RunIf run = {});
cudaError_t tc_gla_chunk_out(const void* q, const void* k, const void* v, const float* g, float* P, void* o,
                             int B, int H, int64_t N, int64_t t_slots, int stride, int tiles, cudaStream_t st,
                             RunIf run = {});
cudaError_t tc_gla_chunk_bwd(const void* q, const void* k, const void* v, const void* dout, const float* g,
                             const float* P, float* Rs, void* dq, void* dk, void* dv, float* dg, int B, int H,
                             int64_t N, int64_t t_slots, int stride, int tiles, cudaStream_t st, RunIf run = {});

// Causal softmax attention, bf16, d = 128 (k_tc_softmax.cu): queries at
// positions q_offset + i (i < Nq) against keys / values at 0..Nk-1; lse
// [B, H, Nq] (natural log); delta [B, H, Nq] = rowsum(do . o).
bool tc_softmax_ok(int dtype, int d);
cudaError_t tc_softmax_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int64_t Nq,
                           int64_t Nk, int64_t q_offset, float scale, cudaStream_t st);
cudaError_t tc_softmax_delta(const void* o, const void* dout, float* delta, int B, int H, int64_t Nq,
                             cudaStream_t st);
cudaError_t tc_softmax_dkdv(const void* q, const void* k, const void* v, const float* lse, const void* dout,
                            void* dk, void* dv, const float* delta, int B, int H, int64_t Nq, int64_t Nk,
                            int64_t q_offset, float scale, cudaStream_t st);
cudaError_t tc_softmax_dq(const void* q, const void* k, const void* v, const float* lse, const void* dout, void* dq,
                          const float* delta, int B, int H, int64_t Nq, int64_t Nk, int64_t q_offset, float scale,
                          cudaStream_t st);

}  // namespace lasp
