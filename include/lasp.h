/*
 * lasp.h -- C ABI of the B200 library for chunked causal linear attention
 * with a per-head decay: the single-GPU hot path of LASP / LASP-2.
 *
 * What is computed (page "Linear Attention Sequence Parallelism" (LASP), v3,
 * section 3.2; page "LASP-2" (pith.science review), "The reading"):
 * for every batch b and head h, tokens s = 0..N-1,
 *     kv_s = lambda_h kv_{s-1} + k_s^T v_s        (LASP Eq. 5-6, kv_{-1} = init)
 *     o_s  = q_s kv_s                              (LASP Eq. 4-5)
 * and the gradients of sum(o * dO) (LASP Eq. 12-13). Norm(.) after attention
 * is not applied (LASP section 3.2 omits it in the derivation); there is no
 * feature map and no 1/sqrt(d) scale.
 *
 * The sequence is cut into chunks of C tokens (LASP Algorithm 1, C = N/T);
 * chunk c (0-based) holds tokens c*C .. c*C+C-1.
 *
 * Layouts (all row-major, C order):
 *   token tensors q, k, v, o, dout, dq, dk, dv:  [B, N, H, d]
 *       element type: float (LASP_F32) or bfloat16 (LASP_BF16), the same for all.
 *   state arrays (always float32):  [B, T, H, d, d], T = N / C, or [B, H, d, d]
 *       for a single state per (b, h); element [i][j] pairs key/query feature i
 *       with value/output feature j, e.g. M_c[i][j] = sum_t w_t k_t[i] v_t[j].
 *   decay: float[H], lambda_h in (0, 1], or NULL for lambda = 1 (ordinary
 *       linear attention, LASP section 3.2). NULL and an all-ones array give
 *       bit-identical results.
 *
 * Pointers: every pointer is a DEVICE pointer owned by the caller; the library
 * never allocates, frees or keeps a pointer after the call returns. All
 * tensors must be 16-byte aligned and must not overlap unless stated.
 *
 * Execution: every compute call is asynchronous and stream-ordered on
 * `stream` (a cudaStream_t; NULL = the legacy default stream). Arguments are
 * validated on the host before anything is launched; a non-zero status means
 * nothing was launched. Conditions only the device can see (a decay value
 * outside (0, 1], a wait that exceeded its time limit) are recorded in a
 * per-device status word read by lasp_check_device_status().
 *
 * Supported sizes: B, H >= 1; N >= 0 (N = 0 launches nothing); d in
 * {32, 64, 128}; 1 <= C, C divides N. Larger T * H * d * d products are limited
 * only by device memory.
 *
 * Speed: bf16 runs on the tensor cores for d in {32, 64, 128} and C a multiple
 * of 16; with d = 128 and C in {16, 32, 64, 128, 256} (N a multiple of 128)
 * both passes walk segments of about 1024 tokens with the state on chip, the
 * fastest path. The backward needs the state entering every 128-token tile,
 * which the state cache holds only while a chunk spans at most two tiles: with
 * C > 256 the backward's gradient kernel runs on the CUDA cores, far slower
 * (results are the same for every C). fp32 runs on the CUDA cores.
 */
#ifndef LASP_H
#define LASP_H

#include <stdint.h>

#if defined(__GNUC__)
#define LASP_API __attribute__((visibility("default")))
#else
#define LASP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LASP_OK = 0,
  LASP_ERR_INVALID_ARG = 1, /* bad size, NULL required pointer, bad dtype */
  LASP_ERR_UNSUPPORTED = 2, /* a size the library has no kernel for (e.g. d = 96) */
  LASP_ERR_MISALIGNED = 3,  /* a pointer not 16-byte aligned */
  LASP_ERR_CUDA = 4,        /* a CUDA runtime error (launch failure, no device) */
  LASP_ERR_TIMEOUT = 5      /* a device-side wait exceeded its limit */
} lasp_status;

typedef enum { LASP_F32 = 0, LASP_BF16 = 1 } lasp_dtype;

/*
 * lasp_fwd -- forward pass (LASP Algorithm 2; LASP-2 "The reading": chunk
 * states, prefix over chunk states, intra + inter output).
 *   o[b, s, h, :] = q_s kv_s, with kv_{-1} = init_state[b, h] (or 0).
 * Steps (each a kernel): chunk states M_c = sum_j lambda^{C-1-j} k_j^T v_j
 * (LASP Eq. 10) into state_cache; exclusive decayed prefix over chunks in
 * place, P_c = lambda^C P_{c-1} + M_{c-1}, P_0 = init (LASP-2 prefix sum);
 * output O_c = [(Q_c K_c^T) . Mask] V_c + Lambda Q_c P_c (LASP Eq. 7, 9, 11).
 *   q, k, v:      in,  [B, N, H, d] of `dtype`.
 *   decay:        in,  float[H] or NULL.
 *   o:            out, [B, N, H, d] of `dtype`.
 *   state_cache:  out, B * (N/C) * H * d * d floats (16-byte aligned): the
 *                 cache of chunk-entering states P_c that lasp_bwd reads (LASP
 *                 section 3.4 "KV State Caching"), one d x d slot per (b, c, h).
 *                 Its encoding inside a slot is internal to the library (fp32
 *                 P_c; or, for bf16 with d = 128, C dividing 128 and N a
 *                 multiple of 128, the bf16 operand tile of the state entering
 *                 each 128-token tile, in the slot of the tile's first chunk);
 *                 pass it unchanged to lasp_bwd with the same sizes. The per-chunk states themselves are exposed by
 *                 lasp_chunk_states + lasp_state_prefix. Required.
 *   init_state:   in,  float [B, H, d, d] or NULL: the state entering token 0
 *                 (the prefix of the shards before this one in the LASP-2
 *                 decomposition).
 */
LASP_API int lasp_fwd(const void* q, const void* k, const void* v, const float* decay, void* o,
             int B, int H, int64_t N, int d, int C, int dtype,
             float* state_cache, const float* init_state, void* stream);

/*
 * lasp_bwd -- backward pass (LASP Algorithm 3; LASP-2 suffix sum of dM_t).
 * Gradients of sum(o * dout) with respect to q, k, v.
 * Steps: gradient chunk states dM_c = sum_j lambda^{j+1} q_j^T do_j
 * (LASP Eq. 20 term (Lambda Q_t)^T dO_t) into dstate_ws; exclusive decayed
 * suffix in place, R_c = lambda^C R_{c+1} + dM_{c+1}, R_{T-1} = dstate_in;
 * then dQ, dK, dV per chunk:
 *   dQ_c = [(dO_c V_c^T) . Mask] K_c + Lambda dO_c P_c^T         (Eq. 14, 16)
 *   dK_c = [(dO_c V_c^T) . Mask]^T Q_c + lambda^C Lambda^-1 V_c R_c^T (Eq. 17, 19)
 *   dV_c = [(Q_c K_c^T) . Mask]^T dO_c + lambda^C Lambda^-1 K_c R_c   (Eq. 22, 23)
 *   q, k, v, dout:  in,  [B, N, H, d] of `dtype`.
 *   dq, dk, dv:     out, [B, N, H, d] of `dtype`.
 *   state_cache:    in,  the cache lasp_fwd wrote for the same q, k, v,
 *                   decay, C and init_state. Required.
 *   dstate_ws:      workspace, B * (N/C) * H * d * d floats (16-byte aligned)
 *                   for the gradient states R_c (the gradient state chunk c
 *                   receives from the tokens after it); its contents on return
 *                   are unspecified (lasp_chunk_dstates + lasp_state_prefix
 *                   expose R_c). Required.
 *   init_state:     in,  as given to lasp_fwd (only its effect through
 *                   state_cache matters; may be NULL).
 *   dstate_in:      in,  float [B, H, d, d] or NULL: gradient state entering the
 *                   last token from tokens after the sequence (LASP-2 suffix of
 *                   the later shards).
 *   dinit_state:    out, float [B, H, d, d] or NULL: gradient of the loss with
 *                   respect to init_state, lambda^C R_0 + dM_0 (the dstate_in of
 *                   the previous shard).
 */
LASP_API int lasp_bwd(const void* q, const void* k, const void* v, const float* decay, const void* dout,
             void* dq, void* dk, void* dv, int B, int H, int64_t N, int d, int C, int dtype,
             const float* state_cache, float* dstate_ws, const float* init_state,
             const float* dstate_in, float* dinit_state, void* stream);

/*
 * lasp_chunk_states -- per-chunk memory states (LASP Eq. 10, Algorithm 2 step
 * 16 with KV_{t-1} = 0; LASP-2 "The reading": M_t summarises chunk t):
 *   M[b, c, h][i][j] = sum_{j'=0}^{C-1} lambda_h^{C-1-j'} k_{cC+j'}[i] v_{cC+j'}[j].
 *   q:  unused, may be NULL (kept so the call mirrors lasp_fwd).
 *   k, v:  in, [B, N, H, d] of `dtype`.   M: out, float [B, N/C, H, d, d].
 * C may be as large as N (one state per sequence: the LASP-2 shard state).
 */
LASP_API int lasp_chunk_states(const void* q, const void* k, const void* v, const float* decay, float* M,
                      int B, int H, int64_t N, int d, int C, int dtype, void* stream);

/*
 * lasp_chunk_dstates -- per-chunk gradient states (LASP Eq. 20, Algorithm 3
 * step 18 with dKV_{t+1} = 0):
 *   dM[b, c, h][i][j] = sum_{j'=0}^{C-1} lambda_h^{j'+1} q_{cC+j'}[i] do_{cC+j'}[j].
 *   q, dout: in, [B, N, H, d] of `dtype`.   dM: out, float [B, N/C, H, d, d].
 */
LASP_API int lasp_chunk_dstates(const void* q, const void* dout, const float* decay, float* dM,
                       int B, int H, int64_t N, int d, int C, int dtype, void* stream);

/*
 * lasp_state_prefix -- exclusive decayed scan over chunk states (LASP-2:
 * prefix sum of the gathered M_t in the forward pass, suffix sum of dM_t in
 * the backward pass; LASP Eq. 10 / Eq. 20 give the per-chunk decay lambda^C).
 *   reverse = 0:  P_0 = init; P_c = lambda^C P_{c-1} + M_{c-1};
 *                 total = lambda^C P_{T-1} + M_{T-1}  (state after the last chunk)
 *   reverse = 1:  R_{T-1} = init; R_c = lambda^C R_{c+1} + M_{c+1};
 *                 total = lambda^C R_0 + M_0
 *   M:        in,  float [B, T, H, d, d].
 *   Mprefix:  out, float [B, T, H, d, d]; may be the same pointer as M (in place).
 *   init:     in,  float [B, H, d, d] or NULL (zero).
 *   total:    out, float [B, H, d, d] or NULL.
 *   C:        chunk length in tokens, >= 1 (the decay step is lambda^C).
 */
LASP_API int lasp_state_prefix(const float* M, float* Mprefix, const float* decay, const float* init,
                      float* total, int B, int T, int H, int d, int64_t C, int reverse,
                      void* stream);

/*
 * lasp_chunk_out -- the output step of lasp_fwd on its own (LASP Eq. 7, 9, 11;
 * Algorithm 2 steps 9, 14, 15), given the chunk-entering states P:
 *   O_c[j] = sum_{i<=j} lambda^{j-i} (q_j . k_i) v_i + lambda^{j+1} q_j P_c.
 *   q, k, v: in, [B, N, H, d] of `dtype`.   P: in, float [B, N/C, H, d, d].
 *   o: out, [B, N, H, d] of `dtype`.
 * lasp_fwd = lasp_chunk_states, lasp_state_prefix (in place), lasp_chunk_out.
 */
LASP_API int lasp_chunk_out(const void* q, const void* k, const void* v, const float* decay, const float* P,
                            void* o, int B, int H, int64_t N, int d, int C, int dtype, void* stream);

/*
 * lasp_chunk_grads -- the dQ/dK/dV step of lasp_bwd on its own (LASP Eq. 14,
 * 16, 17, 19, 22, 23; Algorithm 3 steps 7-17), given the chunk-entering
 * states P (from the forward pass) and the gradient states R:
 *   dQ_c[j] = sum_{i<=j} lambda^{j-i} (do_j . v_i) k_i + lambda^{j+1} do_j P_c^T
 *   dK_c[j] = sum_{i>=j} lambda^{i-j} (do_i . v_j) q_i + lambda^{C-1-j} v_j R_c^T
 *   dV_c[j] = sum_{i>=j} lambda^{i-j} (q_i . k_j) do_i + lambda^{C-1-j} k_j R_c
 *   q, k, v, dout: in, [B, N, H, d]; P, R: in, float [B, N/C, H, d, d];
 *   dq, dk, dv: out, [B, N, H, d], all of `dtype`.
 * lasp_bwd = lasp_chunk_dstates, lasp_state_prefix (reverse, in place),
 * lasp_chunk_grads.
 */
LASP_API int lasp_chunk_grads(const void* q, const void* k, const void* v, const void* dout, const float* decay,
                              const float* P, const float* R, void* dq, void* dk, void* dv, int B, int H,
                              int64_t N, int d, int C, int dtype, void* stream);

/*
 * lasp_fwd_states, lasp_fwd_finish -- lasp_fwd in the two parts that the
 * LASP-2 exchange separates (LASP-2 "The reading": every shard computes its
 * memory state M_t, the states are gathered, then each shard takes the prefix
 * of the earlier shards' states and computes its output). Sizes, dtype and
 * state_cache as for lasp_fwd; lasp_fwd is lasp_fwd_states (total NULL)
 * followed by lasp_fwd_finish with the same arguments.
 *   lasp_fwd_states: the first step of lasp_fwd (the chunk states, or on the
 *     tensor-core walk path the segment states, into state_cache) and, if
 *     total (out, float [B, H, d, d]) is non-NULL, the state after the last
 *     token of a sequence that starts from zero:
 *       total = sum_s lambda^{N-1-s} k_s^T v_s   (LASP Eq. 10 with C = N),
 *     the shard state M_t of LASP-2. For N = 0, total is zero.
 *   lasp_fwd_finish: the rest of lasp_fwd on a cache that lasp_fwd_states
 *     filled for the same k, v, decay and sizes: the prefix from init_state
 *     (may be NULL) and the output o.
 */
LASP_API int lasp_fwd_states(const void* k, const void* v, const float* decay, int B, int H, int64_t N, int d, int C,
                             int dtype, float* state_cache, float* total, void* stream);
LASP_API int lasp_fwd_finish(const void* q, const void* k, const void* v, const float* decay, void* o, int B, int H,
                             int64_t N, int d, int C, int dtype, float* state_cache, const float* init_state,
                             void* stream);

/*
 * lasp_bwd_states, lasp_bwd_finish -- lasp_bwd in the same two parts (LASP-2
 * backward: gradient states dM_t, gathered, then the suffix over the later
 * shards and the gradients). Sizes, dtype, state_cache and dstate_ws as for
 * lasp_bwd; lasp_bwd is lasp_bwd_states (total NULL) followed by
 * lasp_bwd_finish.
 *   lasp_bwd_states: the first step of lasp_bwd (the gradient chunk or
 *     segment states into dstate_ws) and, if total (out, float [B, H, d, d])
 *     is non-NULL, the gradient state the sequence passes back to the state
 *     entering its first token when nothing enters from after it:
 *       total = sum_s lambda^{s+1} q_s^T do_s   (LASP Eq. 20 with C = N),
 *     the shard gradient state dM_t of LASP-2. For N = 0, total is zero.
 *   lasp_bwd_finish: the rest of lasp_bwd on a workspace that
 *     lasp_bwd_states filled for the same q, dout, decay and sizes: the suffix
 *     from dstate_in (may be NULL), dinit_state (may be NULL), dq, dk, dv.
 */
LASP_API int lasp_bwd_states(const void* q, const void* dout, const float* decay, int B, int H, int64_t N, int d,
                             int C, int dtype, float* dstate_ws, float* total, void* stream);
LASP_API int lasp_bwd_finish(const void* q, const void* k, const void* v, const float* decay, const void* dout,
                             void* dq, void* dk, void* dv, int B, int H, int64_t N, int d, int C, int dtype,
                             const float* state_cache, float* dstate_ws, const float* dstate_in, float* dinit_state,
                             void* stream);

/*
 * lasp_fwd_states_part, lasp_fwd_finish_part, lasp_bwd_states_part,
 * lasp_bwd_finish_part -- the four split calls above restricted to part `part`
 * of `nparts` (0 <= part < nparts <= B * H) of the (b, h) pairs, taken in
 * b-major order: pairs floor(B H part / nparts) .. floor(B H (part + 1) / nparts) - 1.
 * Calling every part of a step gives exactly the whole call's results; each
 * part reads and writes only its own pairs' slices of every tensor, and the
 * state arrays (total, init_state, dstate_in, dinit_state) stay full
 * [B, H, d, d] arrays of which a part touches its own pairs. This lets LASP-2's
 * exchange of one part's shard states run while the next part's states, and
 * the last part's output, are computed (LASP-2 review page, "Core claim": the
 * AllGather of fixed-size states overlaps computation). nparts = 1 is the
 * whole call; nparts > 1 needs lasp_parts_ok (LASP_ERR_UNSUPPORTED otherwise).
 */
LASP_API int lasp_fwd_states_part(const void* k, const void* v, const float* decay, int B, int H, int64_t N, int d,
                                  int C, int dtype, float* state_cache, float* total, int part, int nparts,
                                  void* stream);
LASP_API int lasp_fwd_finish_part(const void* q, const void* k, const void* v, const float* decay, void* o, int B,
                                  int H, int64_t N, int d, int C, int dtype, float* state_cache,
                                  const float* init_state, int part, int nparts, void* stream);
LASP_API int lasp_bwd_states_part(const void* q, const void* dout, const float* decay, int B, int H, int64_t N, int d,
                                  int C, int dtype, float* dstate_ws, float* total, int part, int nparts,
                                  void* stream);
LASP_API int lasp_bwd_finish_part(const void* q, const void* k, const void* v, const float* decay, const void* dout,
                                  void* dq, void* dk, void* dv, int B, int H, int64_t N, int d, int C, int dtype,
                                  const float* state_cache, float* dstate_ws, const float* dstate_in,
                                  float* dinit_state, int part, int nparts, void* stream);
/* 1 when the part calls accept nparts > 1 for these sizes (both segment walks
 * run: bf16, d = 128, C dividing 128, N a multiple of 128), else 0. */
LASP_API int lasp_parts_ok(int64_t N, int C, int d, int dtype);

/*
 * lasp_bwd_noalloc -- lasp_bwd without the caller-provided workspace.
 * The pages have no counterpart to this call; it exists for callers that
 * cannot allocate device memory: a plain C program or plug-in with no device
 * allocator of its own, or a host application whose memory pool already owns
 * all of the device memory, so that a cudaMalloc would fail (and would
 * synchronize the device if it succeeded).
 * It computes exactly what lasp_bwd computes, with the same arguments except
 * dstate_ws: the gradient-state workspace lives in a fixed 32 MiB array compiled into
 * the library (LASP_NOALLOC_SCRATCH_BYTES), which every GPU that loads the
 * library holds until the process exits. The call allocates nothing.
 *   Limit: B * (N / C) * H * d * d * 4 <= LASP_NOALLOC_SCRATCH_BYTES (for
 *   d = 128: at most 512 chunk-head states); larger problems return
 *   LASP_ERR_UNSUPPORTED before anything is launched.
 *   Set-up: the first call on each device looks up the device address of the
 *   array, with that device current, and caches it; make that first call
 *   before any stream capture.
 *   Sharing: every call uses the same array, which keeps the last call's
 *   contents (nothing in it needs to start at zero). Calls that overlap on the
 *   GPU (on different streams, or from different threads) race on it and must
 *   be serialized by the caller.
 */
#define LASP_NOALLOC_SCRATCH_BYTES (32u << 20)
LASP_API int lasp_bwd_noalloc(const void* q, const void* k, const void* v, const float* decay, const void* dout,
                              void* dq, void* dk, void* dv, int B, int H, int64_t N, int d, int C, int dtype,
                              const float* state_cache, const float* dstate_in, float* dinit_state,
                              void* stream);

/*
 * lasp_check_device_status -- synchronizes `stream`, then returns and clears
 * the first error any kernel of this library recorded on the current device
 * (LASP_OK if none; LASP_ERR_TIMEOUT for a wait that ran out;
 * LASP_ERR_INVALID_ARG for a decay outside (0, 1]; LASP_ERR_CUDA if the
 * synchronization itself failed). `site` (may be NULL) receives the code of
 * the place that recorded it.
 */
LASP_API int lasp_check_device_status(void* stream, int* site);

/* Human-readable name of a status code (static storage). */
LASP_API const char* lasp_status_string(int status);

/*
 * Tracing (a measurement aid; the pages have no counterpart). While enabled,
 * the library brackets each of its kernel launches with two CUDA events on
 * the launch's stream, for up to `capacity` launches.
 *   lasp_trace_enable(capacity): creates the events (no device memory); 0
 *     turns tracing off. Resets the record. Not for concurrent callers.
 *   lasp_trace_read(ids, ms, capacity): waits for the recorded launches,
 *     writes each one's kernel id and duration in milliseconds, clears the
 *     record and returns how many it wrote (a negative status on error).
 *   lasp_kernel_name(id): the kernel's name (static storage).
 */
LASP_API int lasp_trace_enable(int capacity);
LASP_API int lasp_trace_read(int* kernel_ids, float* ms, int capacity);
LASP_API const char* lasp_kernel_name(int kernel_id);

/*
 * lasp_segment_tokens -- the segment length G (tokens) that lasp_fwd uses for
 * a problem of N tokens with chunk size C, head dimension d and `dtype`: the
 * per-segment states and their prefix go to the state_cache slots of each
 * segment's first chunk and a walk carries the state through the segment.
 * Equals C when lasp_fwd computes every chunk state separately; 0 for
 * invalid sizes.
 */
LASP_API int lasp_segment_tokens(int64_t N, int C, int d, int dtype);

/*
 * lasp_set_wait_limit_ns -- sets, for the current device, the time after which
 * a spin-wait inside a kernel gives up, records LASP_ERR_TIMEOUT and lets the
 * kernel return (default 2e9 ns). Synchronous. Used by tests.
 */
LASP_API int lasp_set_wait_limit_ns(uint64_t limit_ns);

/*
 * lasp_wait_probe -- launches one CTA that waits on a barrier nothing arrives
 * on, with the current wait limit, then returns. Lets tests check, without a
 * fault, that a wait that runs out ends with LASP_ERR_TIMEOUT in the status
 * word. Asynchronous on `stream`.
 */
LASP_API int lasp_wait_probe(void* stream);

/* Library version, major * 10000 + minor * 100 + patch. */
LASP_API int lasp_version(void);

/*
 * Bidirectional (unmasked) linear attention: LASP section 3.1, Eq. 3 as the
 * right product O = Q (K^T V) (no Norm, no decay, no mask); the LASP-2 review
 * page ("Summary") gives the unmasked variant as: gather every chunk state
 * M_t, sum them, M_{1:T} = sum_t M_t, and compute Q_t M_{1:T} in every chunk;
 * the backward pass sums dM_t = Q_t^T dO_t the same way. Per (b, h):
 *   M = sum_s k_s^T v_s,  o_s = q_s M;
 *   dM = sum_s q_s^T do_s,  dq_s = do_s M^T,  dk_s = v_s dM^T,  dv_s = k_s dM.
 * Supported: bf16, d = 128, N a multiple of 128 (LASP_ERR_UNSUPPORTED
 * otherwise); N = 0 returns LASP_OK without a launch.
 *
 * lasp_bidir_workspace_floats -- floats of the workspace each pass needs (0
 * for unsupported or invalid sizes). Layout: the segment states (internal),
 * then at lasp_bidir_state_offset the fp32 total state [B, H, d, d] (M after
 * lasp_bidir_fwd, dM after lasp_bidir_bwd; element [i][j] = sum k_i v_j, resp.
 * sum q_i do_j), then its bf16 operand tiles (internal).
 */
LASP_API int64_t lasp_bidir_workspace_floats(int B, int H, int64_t N, int d, int dtype);
LASP_API int64_t lasp_bidir_state_offset(int B, int H, int64_t N, int d, int dtype);

/*
 * lasp_bidir_fwd -- o = q (k^T v) per (b, h).
 *   q, k, v:  in,  [B, N, H, d] bf16.      o: out, [B, N, H, d] bf16.
 *   ws:       out, lasp_bidir_workspace_floats(...) floats (16-byte aligned),
 *             holding M on return; pass it to lasp_bidir_bwd. Required.
 */
LASP_API int lasp_bidir_fwd(const void* q, const void* k, const void* v, void* o, int B, int H, int64_t N, int d,
                            int dtype, float* ws, void* stream);

/*
 * lasp_bidir_bwd -- gradients of sum(o * dout) for lasp_bidir_fwd.
 *   q, k, v, dout:  in,  [B, N, H, d] bf16.   dq, dk, dv: out, [B, N, H, d] bf16.
 *   ws:             in,  the workspace lasp_bidir_fwd filled for the same k, v.
 *   dws:            out, a second workspace of the same size, holding dM on
 *                   return. Required.
 */
LASP_API int lasp_bidir_bwd(const void* q, const void* k, const void* v, const void* dout, void* dq, void* dk,
                            void* dv, int B, int H, int64_t N, int d, int dtype, const float* ws, float* dws,
                            void* stream);

/* ------------------------------------------------------------------------
 * Gated form: a decay that depends on the token and the key feature.
 * Page LASP, Appendix A.4, Eq. 24 (m_t = o_t m_{t-1} + e_t i_t^T), row
 * GLA / GateLoop of Table 5: expand state e_t = k_t, input i_t = v_t, shrink
 * state q_t, memory d x d, oscillation g_t 1^T (the gate of key feature i
 * scales row i of the memory). For every b, h and token s:
 *     kv_s = diag(exp(g_s)) kv_{s-1} + k_s^T v_s,    o_s = q_s kv_s,
 * with g_s[i] the natural log of that gate (g <= 0 for a gate in (0, 1]; any
 * finite value is accepted, but for g > 0 the gate factors can overflow).
 * With g_s[i] = log(lambda_h) this is lasp_fwd's recurrence.
 *
 *   g, dg:  float [B, N, H, d] (always float32, the layout of the token
 *           tensors), the log-gates and the gradient of sum(o * dout) with
 *           respect to them.
 * Chunks: 1 <= C <= 128, C divides N (LASP_ERR_UNSUPPORTED for C > 128).
 * bf16 with d = 128, C dividing 128 and N a multiple of 128 runs on the tensor
 * cores, which factor the decay inside each 128-token tile around the tile's
 * middle token: that holds while the |log-gates| of each 64-token half of a
 * tile sum to at most 79. lasp_gla_fwd checks every tile on the device; when
 * one is beyond that (gates far stronger than any that leave the state
 * anything to carry), the call, and the lasp_gla_bwd given its cache, run the
 * exact CUDA-core kernels instead (slower, same results; no status is
 * recorded and the host is not synchronised). Every other case (fp32 in
 * particular) runs those CUDA-core kernels. In
 * chunk c, b_t = sum_{r<=t} g_{cC+r} (from the chunk start) and the chunk's
 * total log-gate is gsum_c = b_{C-1}. The states of the gated form:
 *   kind 0, (x, y) = (k, v):   M_c  = sum_t diag(exp(gsum_c - b_t)) k_t^T v_t
 *   kind 1, (x, y) = (q, do):  dM_c = sum_t diag(exp(b_t)) q_t^T do_t
 * and the scans step through chunk c with diag(exp(gsum_c)) where lasp_fwd's
 * use lambda^C (LASP-2 prefix / suffix over the chunk states).
 * Pointers, streams and errors as for the calls above.
 */

/* Size, in floats, of the state cache of lasp_gla_fwd / lasp_gla_bwd:
 * B * (N/C) * H * d * (d + 2) + 4 (the last four hold the forward's choice of
 * kernels, read by the backward). -1 for sizes the gated calls reject. */
LASP_API int64_t lasp_gla_cache_floats(int B, int H, int64_t N, int d, int C);

/*
 * lasp_gla_chunk_states -- kind 0: M [B, N/C, H, d, d] from (x, y) = (k, v)
 * and, if gsum (float [B, N/C, H, d]) is non-NULL, the chunk log-gate totals;
 * kind 1: dM from (x, y) = (q, dout) (gsum as for kind 0).
 */
LASP_API int lasp_gla_chunk_states(const void* x, const void* y, const float* g, float* M, float* gsum, int B,
                                   int H, int64_t N, int d, int C, int dtype, int kind, void* stream);

/*
 * lasp_gla_state_prefix -- exclusive scan with a diagonal decay per chunk:
 *   reverse = 0:  P_0 = init; P_c = diag(exp(gsum_{c-1})) P_{c-1} + M_{c-1};
 *                 total = diag(exp(gsum_{T-1})) P_{T-1} + M_{T-1}
 *   reverse = 1:  R_{T-1} = init; R_c = diag(exp(gsum_{c+1})) R_{c+1} + M_{c+1};
 *                 total = diag(exp(gsum_0)) R_0 + M_0
 *   M, Mprefix: float [B, T, H, d, d] (may be the same array); gsum: float
 *   [B, T, H, d]; init, total: float [B, H, d, d] or NULL.
 */
LASP_API int lasp_gla_state_prefix(const float* M, float* Mprefix, const float* gsum, const float* init,
                                   float* total, int B, int T, int H, int d, int reverse, void* stream);

/*
 * lasp_gla_fwd -- o for the gated recurrence. Steps: states (kind 0) and
 * gsum into state_cache, the prefix scan in place (P_c), then per chunk
 *   o_t = (q_t . exp(b_t)) P_c + sum_{s<=t} (sum_i q_t[i] k_s[i] exp(b_t[i] - b_s[i])) v_s.
 *   state_cache: out, lasp_gla_cache_floats(...) floats; pass it unchanged to
 *                lasp_gla_bwd. Required. Its encoding inside a slot is
 *                internal to the library (the tensor-core path keeps states
 *                per segment of about 1024 tokens, and a tile's slot ends up
 *                holding the bf16 operand tile its backward loads).
 *   init_state:  in, float [B, H, d, d] or NULL, the state entering token 0.
 */
LASP_API int lasp_gla_fwd(const void* q, const void* k, const void* v, const float* g, void* o, int B, int H,
                          int64_t N, int d, int C, int dtype, float* state_cache, const float* init_state,
                          void* stream);

/*
 * lasp_gla_bwd -- gradients of sum(o * dout) for lasp_gla_fwd with respect to
 * q, k, v and g. Steps: gradient states (kind 1) into dstate_ws, the suffix
 * scan in place (R_c, the gradient of the state leaving chunk c; dinit), then
 * per chunk, with A_ts = sum_i q_t[i] k_s[i] exp(b_t[i] - b_s[i]) (s <= t):
 *   dq_t = exp(b_t) . (do_t P_c^T) + sum_{s<=t} (do_t . v_s) k_s . exp(b_t - b_s)
 *   dk_s = sum_{t>=s} (do_t . v_s) q_t . exp(b_t - b_s) + exp(gsum_c - b_s) . (v_s R_c^T)
 *   dv_s = sum_{t>=s} A_ts do_t + (k_s . exp(gsum_c - b_s)) R_c
 *   dg_s = sum_{t>=s in the chunk} (q_t . dq_t - k_t . dk_t) + rowsum(R_c . P_{c+1})
 * (P_{c+1} the state leaving the chunk), evaluated without the parts that
 * cancel exactly (each token's s = t pair; the inter part of k . dk for t >= s),
 * so that dg stays accurate to its own size when the gates are strong.
 *   state_cache: in, what lasp_gla_fwd wrote for the same q, k, v, g, C and
 *                init_state. Required.
 *   dstate_ws:   workspace, B * (N/C) * H * d * d floats. Required. Its
 *                contents afterwards are internal (the tensor-core path keeps
 *                one gradient state per segment and a scratch state per
 *                segment; the CUDA-core path R_c per chunk).
 *   dstate_in:   in, float [B, H, d, d] or NULL: gradient with respect to the
 *                state after the last token.
 *   dinit_state: out, float [B, H, d, d] or NULL: gradient with respect to
 *                init_state.
 */
LASP_API int lasp_gla_bwd(const void* q, const void* k, const void* v, const float* g, const void* dout, void* dq,
                          void* dk, void* dv, float* dg, int B, int H, int64_t N, int d, int C, int dtype,
                          const float* state_cache, float* dstate_ws, const float* dstate_in, float* dinit_state,
                          void* stream);

/* ------------------------------------------------------------------------
 * Softmax attention: the standard attention layers a hybrid model keeps.
 * Page LASP-2 review, "Summary" and abstract: LASP-2H applies the same
 * AllGather pattern to standard attention layers, each rank gathering the
 * keys and values (K_t, V_t) of the ranks before it. A call takes a block of
 * queries sitting at global positions p_i = q_offset + i (i = 0..Nq-1) and
 * the keys / values at positions 0..Nk-1 (on one GPU: q_offset = 0 and
 * Nq = Nk = N; in sequence parallelism: the rank's own queries against the
 * gathered keys). For every b, h (causal, scale > 0, usually d^-1/2):
 *     s_ij  = scale (q_i . k_j)                        for j <= p_i
 *     o_i   = sum_{j <= p_i} exp(s_ij - lse_i) v_j
 *     lse_i = log sum_{j <= p_i} exp(s_ij)             (natural log)
 * Supported: bf16, d = 128 (tensor cores); other types and sizes return
 * LASP_ERR_UNSUPPORTED. Requires q_offset + Nq <= Nk (LASP_ERR_INVALID_ARG).
 *   q, o, dout, dq:  [B, Nq, H, d];  k, v, dk, dv: [B, Nk, H, d] (bf16)
 *   lse, delta:      float [B, H, Nq]
 * Pointers, streams and errors as for the calls above; nothing allocates.
 */

/*
 * lasp_softmax_fwd -- o and lse as above (one online-softmax pass over
 * 128-key tiles per 128-query tile).
 */
LASP_API int lasp_softmax_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                              int64_t Nq, int64_t Nk, int64_t q_offset, int d, float scale, int dtype, void* stream);

/*
 * lasp_softmax_bwd -- gradients of sum(o * dout) for lasp_softmax_fwd:
 *     p_ij = exp(s_ij - lse_i),   ds_ij = p_ij (dout_i . v_j - delta_i),
 *     dq_i = scale sum_j ds_ij k_j,  dk_j = scale sum_i ds_ij q_i,  dv_j = sum_i p_ij dout_i,
 * with delta_i = dout_i . o_i (written to `delta`, a workspace the caller
 * owns). o and lse are lasp_softmax_fwd's for the same inputs. Every row of
 * dk and dv is written; keys no query reaches get zeros (in sequence
 * parallelism each rank's dk, dv are summed over the ranks by a
 * reduce-scatter).
 */
LASP_API int lasp_softmax_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                              const void* dout, void* dq, void* dk, void* dv, float* delta, int B, int H, int64_t Nq,
                              int64_t Nk, int64_t q_offset, int d, float scale, int dtype, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LASP_H */
