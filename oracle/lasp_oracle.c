/*
 * lasp_oracle.c -- fp64 CPU oracle for causal linear attention with a per-head
 * decay, as LASP / LASP-2 compute it.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark use this file. It shares no code, header, table or helper
 * with the CUDA library, and the CUDA library never calls it.
 *
 * Sources (page: "Linear Attention Sequence Parallelism" (LASP), v3 full text):
 *   - Eq. 4-6  (section 3.2, forward): kv_s = lambda*kv_{s-1} + k_s v_s^T,
 *              o_s^T = q_s^T kv_s, kv_0 = 0.
 *   - Eq. 12-13 (section 3.2, backward): dq_s^T = do_s^T kv_s^T,
 *              dk_s^T = v_s^T dkv_s^T, dv_s^T = k_s^T dkv_s,
 *              dkv_s = sum_{i>=s} lambda^{i-s} q_i do_i^T.
 *   - Eq. 10 and Algorithm 2 (chunk state update): KV_t = lambda^C KV_{t-1}
 *              + (diag{lambda^{C-1},...,1} K_t)^T V_t.
 *   - Eq. 20 and Algorithm 3 (gradient state): dKV_t = lambda^C dKV_{t+1}
 *              + (Lambda Q_t)^T dO_t with Lambda = diag{lambda,...,lambda^C}.
 * Page "LASP-2" (pith.science review), "The reading" / "Core claim": each chunk
 * is summarised by M_t; a prefix sum over the gathered states gives
 * M_{1:t-1} in the forward pass, a suffix sum over dM_t in the backward pass.
 *
 * Conventions (0-based): per (b, h), tokens s = 0..N-1; chunk c = 0..T-1 with
 * T = N / C; s = c*C + j.  Norm(.) is omitted as on the LASP page (section
 * 3.2, "To streamline derivations ...").  No feature map, no 1/sqrt(d).
 *
 * Tensor arguments are views: a base pointer plus element strides for the
 * batch, token and head indices (sb, sn, sh); the feature index is contiguous.
 * Inputs are float32 (bf16- or fp32-valued data are exact in float32 and in
 * double); all arithmetic and all outputs are double.
 *
 * Every function is plain loops over the definition.  Work is split across
 * OpenMP threads by (b, h) and by blocks of state rows or columns; this only
 * decides which thread evaluates an output element, never the order of the
 * terms summed into it, so results are bit-identical for any thread count.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define BLK 32 /* rows or columns of the d x d state owned by one task */

static double lam_of(const double *lam, int h) { return lam ? lam[h] : 1.0; }

static const float *tok(const float *x, long sb, long sn, long sh, int b, long n, int h) {
  return x + (long)b * sb + n * sn + (long)h * sh;
}
static double *tokd(double *x, long sb, long sn, long sh, int b, long n, int h) {
  return x + (long)b * sb + n * sn + (long)h * sh;
}

/* State arrays [B, H, d, d] (entering or leaving states) and [B, T, H, d, d]. */
static const double *st_bh(const double *x, int H, int d, int b, int h) {
  return x + ((long)b * H + h) * d * d;
}
static double *st_bh_w(double *x, int H, int d, int b, int h) {
  return x + ((long)b * H + h) * d * d;
}
static long st_btc(int T, int H, int d, int b, long c, int h) {
  return (((long)b * T + c) * H + h) * (long)d * d;
}

/*
 * Forward recurrence, Eq. 5:  S <- lambda*S + k_s v_s^T ;  o_s = q_s S.
 * S starts at init[b,h] (the state entering token 0) or 0.
 * Task = (b, h, block of S columns j0..j1): column j of o only needs column j
 * of S.  If final_state is given, it receives S after token N-1.
 */
void oracle_fwd(const float *q, const float *k, const float *v, long sb, long sn, long sh,
                const double *lam, const double *init,
                double *o, long ob, long on, long oh,
                double *final_state, int B, long N, int H, int d) {
  int nblk = (d + BLK - 1) / BLK;
  long ntask = (long)B * H * nblk;
#pragma omp parallel for schedule(dynamic, 1)
  for (long task = 0; task < ntask; ++task) {
    int blk = (int)(task % nblk);
    int h = (int)((task / nblk) % H);
    int b = (int)(task / ((long)nblk * H));
    int j0 = blk * BLK, j1 = j0 + BLK < d ? j0 + BLK : d;
    double l = lam_of(lam, h);
    double *S = (double *)calloc((size_t)d * d, sizeof(double));
    if (init) memcpy(S, st_bh(init, H, d, b, h), sizeof(double) * d * d);
    for (long s = 0; s < N; ++s) {
      const float *qs = tok(q, sb, sn, sh, b, s, h);
      const float *ks = tok(k, sb, sn, sh, b, s, h);
      const float *vs = tok(v, sb, sn, sh, b, s, h);
      double *os = tokd(o, ob, on, oh, b, s, h);
      for (int i = 0; i < d; ++i)
        for (int j = j0; j < j1; ++j) S[i * d + j] = l * S[i * d + j] + (double)ks[i] * vs[j];
      for (int j = j0; j < j1; ++j) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += (double)qs[i] * S[i * d + j];
        os[j] = acc;
      }
    }
    if (final_state) {
      double *F = st_bh_w(final_state, H, d, b, h);
      for (int i = 0; i < d; ++i)
        for (int j = j0; j < j1; ++j) F[i * d + j] = S[i * d + j];
    }
    free(S);
  }
}

/*
 * Backward recurrences, Eq. 12-13.
 *   dq_s[i] = sum_j kv_s[i][j] do_s[j]          (forward sweep, S rows i)
 *   dkv_s   = q_s do_s^T + lambda * dkv_{s+1}     (reverse sweep)
 *   dk_s[i] = sum_j dkv_s[i][j] v_s[j]          (reverse sweep, G rows i)
 *   dv_s[j] = sum_i k_s[i] dkv_s[i][j]          (reverse sweep, G columns j)
 * The reverse sweep starts from dstate_in[b,h] (the gradient state that
 * enters token N-1 from tokens beyond the sequence end, i.e. dkv_{N-1} =
 * q_{N-1} do_{N-1}^T + dstate_in) or 0; init (the forward entering state)
 * enters kv_s as in oracle_fwd.  If dinit is given it receives the gradient
 * of sum(o * do) with respect to init: lambda * dkv_0.
 * Tasks: (b, h, sweep, block); sweep 0 = dq (row blocks of S),
 * 1 = dk (row blocks of G), 2 = dv and dinit (column blocks of G).
 */
void oracle_bwd(const float *q, const float *k, const float *v, const float *dout,
                long sb, long sn, long sh, const double *lam, const double *init,
                const double *dstate_in,
                double *dq, double *dk, double *dv, long gb, long gn, long gh,
                double *dinit, int B, long N, int H, int d) {
  int nblk = (d + BLK - 1) / BLK;
  long ntask = (long)B * H * 3 * nblk;
#pragma omp parallel for schedule(dynamic, 1)
  for (long task = 0; task < ntask; ++task) {
    int blk = (int)(task % nblk);
    int sweep = (int)((task / nblk) % 3);
    int h = (int)((task / (3L * nblk)) % H);
    int b = (int)(task / (3L * nblk * H));
    int r0 = blk * BLK, r1 = r0 + BLK < d ? r0 + BLK : d;
    double l = lam_of(lam, h);
    double *S = (double *)calloc((size_t)d * d, sizeof(double));
    if (sweep == 0) {
      if (init) memcpy(S, st_bh(init, H, d, b, h), sizeof(double) * d * d);
      for (long s = 0; s < N; ++s) {
        const float *ks = tok(k, sb, sn, sh, b, s, h);
        const float *vs = tok(v, sb, sn, sh, b, s, h);
        const float *ds = tok(dout, sb, sn, sh, b, s, h);
        double *dqs = tokd(dq, gb, gn, gh, b, s, h);
        for (int i = r0; i < r1; ++i) {
          double acc = 0.0;
          for (int j = 0; j < d; ++j) {
            S[i * d + j] = l * S[i * d + j] + (double)ks[i] * vs[j];
            acc += S[i * d + j] * ds[j];
          }
          dqs[i] = acc;
        }
      }
    } else {
      double *G = S; /* dkv, exclusive of the current token until it is added */
      if (dstate_in) memcpy(G, st_bh(dstate_in, H, d, b, h), sizeof(double) * d * d);
      for (long s = N - 1; s >= 0; --s) {
        const float *qs = tok(q, sb, sn, sh, b, s, h);
        const float *ks = tok(k, sb, sn, sh, b, s, h);
        const float *vs = tok(v, sb, sn, sh, b, s, h);
        const float *ds = tok(dout, sb, sn, sh, b, s, h);
        if (sweep == 1) {
          double *dks = tokd(dk, gb, gn, gh, b, s, h);
          for (int i = r0; i < r1; ++i) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j) {
              G[i * d + j] += (double)qs[i] * ds[j];
              acc += G[i * d + j] * vs[j];
            }
            dks[i] = acc;
            for (int j = 0; j < d; ++j) G[i * d + j] *= l;
          }
        } else {
          double *dvs = tokd(dv, gb, gn, gh, b, s, h);
          for (int i = 0; i < d; ++i)
            for (int j = r0; j < r1; ++j) G[i * d + j] += (double)qs[i] * ds[j];
          for (int j = r0; j < r1; ++j) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc += (double)ks[i] * G[i * d + j];
            dvs[j] = acc;
          }
          for (int i = 0; i < d; ++i)
            for (int j = r0; j < r1; ++j) G[i * d + j] *= l;
        }
      }
      if (sweep == 2 && dinit) {
        double *D = st_bh_w(dinit, H, d, b, h);
        for (int i = 0; i < d; ++i)
          for (int j = r0; j < r1; ++j) D[i * d + j] = G[i * d + j];
      }
    }
    free(S);
  }
}

/*
 * Per-chunk states, written out from their definition.
 *   kind 0 (forward memory state, Eq. 10 / Algorithm 2):
 *       M_c[i][j] = sum_{t=0}^{C-1} lambda^{C-1-t} a_{cC+t}[i] b_{cC+t}[j]
 *       with (a, b) = (k, v).
 *   kind 1 (gradient state, Eq. 20 / Algorithm 3, term (Lambda Q_t)^T dO_t):
 *       M_c[i][j] = sum_{t=0}^{C-1} lambda^{t+1} a_{cC+t}[i] b_{cC+t}[j]
 *       with (a, b) = (q, do).
 * M is [B, T, H, d, d], T = N / C (the caller guarantees C divides N).
 */
void oracle_chunk_states(const float *a, const float *bm, long sb, long sn, long sh,
                         const double *lam, double *M, int B, long N, int H, int d,
                         long C, int kind) {
  long T = N / C;
  long ntask = (long)B * T * H;
#pragma omp parallel for schedule(dynamic, 1)
  for (long task = 0; task < ntask; ++task) {
    int h = (int)(task % H);
    long c = (task / H) % T;
    int b = (int)(task / ((long)H * T));
    double l = lam_of(lam, h);
    double *Mc = M + st_btc((int)T, H, d, b, c, h);
    for (long e = 0; e < (long)d * d; ++e) Mc[e] = 0.0;
    for (long t = 0; t < C; ++t) {
      double w = kind == 0 ? pow(l, (double)(C - 1 - t)) : pow(l, (double)(t + 1));
      const float *as = tok(a, sb, sn, sh, b, c * C + t, h);
      const float *bs = tok(bm, sb, sn, sh, b, c * C + t, h);
      for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) Mc[i * d + j] += w * (double)as[i] * bs[j];
    }
  }
}

/*
 * Decayed scans over chunk states (LASP-2: prefix sum of the gathered M_t in
 * the forward pass, suffix sum of dM_t in the backward pass; LASP Eq. 10 and
 * Eq. 20 give the decay lambda^C per chunk).
 *   reverse = 0:  P_0 = init (or 0);      P_c = lambda^C P_{c-1} + M_{c-1};
 *                 total = lambda^C P_{T-1} + M_{T-1}.
 *   reverse = 1:  R_{T-1} = init (or 0);  R_c = lambda^C R_{c+1} + M_{c+1};
 *                 total = lambda^C R_0 + M_0.
 * M and P are [B, T, H, d, d]; init and total are [B, H, d, d].
 */
void oracle_state_scan(const double *M, double *P, const double *lam, const double *init,
                       double *total, int B, long T, int H, int d, long C, int reverse) {
  long ntask = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
  for (long task = 0; task < ntask; ++task) {
    int h = (int)(task % H);
    int b = (int)(task / H);
    double g = pow(lam_of(lam, h), (double)C);
    double *acc = (double *)calloc((size_t)d * d, sizeof(double));
    if (init) memcpy(acc, st_bh(init, H, d, b, h), sizeof(double) * d * d);
    for (long n = 0; n < T; ++n) {
      long c = reverse ? T - 1 - n : n;
      const double *Mc = M + st_btc((int)T, H, d, b, c, h);
      double *Pc = P + st_btc((int)T, H, d, b, c, h);
      for (long e = 0; e < (long)d * d; ++e) Pc[e] = acc[e];
      for (long e = 0; e < (long)d * d; ++e) acc[e] = g * acc[e] + Mc[e];
    }
    if (total) memcpy(st_bh_w(total, H, d, b, h), acc, sizeof(double) * d * d);
    free(acc);
  }
}

/*
 * State snapshots from the token recurrences (the state the pages cache for
 * the backward pass, "KV state caching", section 3.4):
 *   kind 0:  P_c = kv_{cC-1}, the forward state after the last token before
 *            chunk c (P_0 = init or 0), run token by token with Eq. 5.
 *   kind 1:  R_c = sum_{s >= (c+1)C} lambda^{s-(c+1)C+1} q_s do_s^T
 *            + lambda^{N-(c+1)C} dstate_in, the gradient state that chunk c
 *            receives from the tokens after it, run token by token with Eq. 13.
 * (a, b) = (k, v) for kind 0 and (q, do) for kind 1; P is [B, T, H, d, d].
 */
void oracle_state_snapshots(const float *a, const float *bm, long sb, long sn, long sh,
                            const double *lam, const double *init, double *P,
                            int B, long N, int H, int d, long C, int kind) {
  long T = N / C;
  long ntask = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
  for (long task = 0; task < ntask; ++task) {
    int h = (int)(task % H);
    int b = (int)(task / H);
    double l = lam_of(lam, h);
    double *S = (double *)calloc((size_t)d * d, sizeof(double));
    if (init) memcpy(S, st_bh(init, H, d, b, h), sizeof(double) * d * d);
    if (kind == 0) {
      for (long s = 0; s < N; ++s) {
        if (s % C == 0) memcpy(P + st_btc((int)T, H, d, b, s / C, h), S, sizeof(double) * d * d);
        const float *as = tok(a, sb, sn, sh, b, s, h);
        const float *bs = tok(bm, sb, sn, sh, b, s, h);
        for (int i = 0; i < d; ++i)
          for (int j = 0; j < d; ++j) S[i * d + j] = l * S[i * d + j] + (double)as[i] * bs[j];
      }
    } else {
      /* S holds the exclusive suffix state at token s (terms from tokens > s). */
      for (long s = N - 1; s >= 0; --s) {
        if (s % C == C - 1) memcpy(P + st_btc((int)T, H, d, b, s / C, h), S, sizeof(double) * d * d);
        const float *as = tok(a, sb, sn, sh, b, s, h);
        const float *bs = tok(bm, sb, sn, sh, b, s, h);
        for (int i = 0; i < d; ++i)
          for (int j = 0; j < d; ++j) S[i * d + j] = l * (S[i * d + j] + (double)as[i] * bs[j]);
      }
    }
    free(S);
  }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * Bidirectional (unmasked) linear attention: LASP Eq. 3 without Norm, the
 * right product O = Q (K^T V); on the LASP-2 page the unmasked variant sums
 * all chunk states, M_{1:T} = sum_t M_t, and every chunk computes Q_t M_{1:T}
 * (no decay).  Per (b, h):
 *   M[i][j] = sum_s k_s[i] v_s[j];           o_s[j] = sum_i q_s[i] M[i][j].
 * M_out (optional, [B, H, d, d]) receives M.
 */
void oracle_bidir_fwd(const float *q, const float *k, const float *v, long sb, long sn, long sh,
                      double *o, long ob, long on, long oh, double *M_out, int B, long N, int H, int d) {
#pragma omp parallel for schedule(dynamic, 1)
  for (long task = 0; task < (long)B * H; ++task) {
    int h = (int)(task % H);
    int b = (int)(task / H);
    double *M = (double *)calloc((size_t)d * d, sizeof(double));
    for (long s = 0; s < N; ++s) {
      const float *ks = tok(k, sb, sn, sh, b, s, h);
      const float *vs = tok(v, sb, sn, sh, b, s, h);
      for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) M[i * d + j] += (double)ks[i] * vs[j];
    }
    for (long s = 0; s < N; ++s) {
      const float *qs = tok(q, sb, sn, sh, b, s, h);
      double *os = tokd(o, ob, on, oh, b, s, h);
      for (int j = 0; j < d; ++j) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += (double)qs[i] * M[i * d + j];
        os[j] = acc;
      }
    }
    if (M_out) memcpy(st_bh_w(M_out, H, d, b, h), M, sizeof(double) * d * d);
    free(M);
  }
}

/*
 * Its gradients for L = sum_s o_s . do_s (the unmasked backward of the
 * LASP-2 page: the gradient state summed over all chunks):
 *   dM[i][j] = sum_s q_s[i] do_s[j];
 *   dq_s[i] = sum_j M[i][j] do_s[j];   dk_s[i] = sum_j dM[i][j] v_s[j];
 *   dv_s[j] = sum_i k_s[i] dM[i][j].
 * dM_out (optional, [B, H, d, d]) receives dM.
 */
void oracle_bidir_bwd(const float *q, const float *k, const float *v, const float *dout, long sb, long sn,
                      long sh, double *dq, double *dk, double *dv, long gb, long gn, long gh, double *dM_out,
                      int B, long N, int H, int d) {
#pragma omp parallel for schedule(dynamic, 1)
  for (long task = 0; task < (long)B * H; ++task) {
    int h = (int)(task % H);
    int b = (int)(task / H);
    double *M = (double *)calloc((size_t)d * d, sizeof(double));
    double *G = (double *)calloc((size_t)d * d, sizeof(double));
    for (long s = 0; s < N; ++s) {
      const float *qs = tok(q, sb, sn, sh, b, s, h);
      const float *ks = tok(k, sb, sn, sh, b, s, h);
      const float *vs = tok(v, sb, sn, sh, b, s, h);
      const float *ds = tok(dout, sb, sn, sh, b, s, h);
      for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) {
          M[i * d + j] += (double)ks[i] * vs[j];
          G[i * d + j] += (double)qs[i] * ds[j];
        }
    }
    for (long s = 0; s < N; ++s) {
      const float *ks = tok(k, sb, sn, sh, b, s, h);
      const float *vs = tok(v, sb, sn, sh, b, s, h);
      const float *ds = tok(dout, sb, sn, sh, b, s, h);
      double *dqs = tokd(dq, gb, gn, gh, b, s, h);
      double *dks = tokd(dk, gb, gn, gh, b, s, h);
      double *dvs = tokd(dv, gb, gn, gh, b, s, h);
      for (int i = 0; i < d; ++i) {
        double aq = 0.0, ak = 0.0, av = 0.0;
        for (int j = 0; j < d; ++j) {
          aq += M[i * d + j] * ds[j];
          ak += G[i * d + j] * vs[j];
          av += (double)ks[j] * G[j * d + i];
        }
        dqs[i] = aq;
        dks[i] = ak;
        dvs[i] = av;
      }
    }
    if (dM_out) memcpy(st_bh_w(dM_out, H, d, b, h), G, sizeof(double) * d * d);
    free(M);
    free(G);
  }
}

/* ------------------------------------------------------------------------
 * Gated form: a decay that depends on the token and the key feature.
 * LASP page, Appendix A.4, Eq. 24, m_t = o_t m_{t-1} + e_t i_t^T, with the
 * GLA / GateLoop row of Table 5: expand state e_t = k_t, input i_t = v_t,
 * shrink state s_t = q_t, memory k x d, and oscillation g_t 1^T, a gate per
 * key feature that scales row i of the memory (elementwise product).  The gate
 * is passed as its natural log a_t[i] (float [B, N, H, d], the same view as
 * q), so that
 *     S_s[i][j] = exp(a_s[i]) S_{s-1}[i][j] + k_s[i] v_s[j],
 *     o_s[j]    = sum_i q_s[i] S_s[i][j].
 * With a_s[i] = log(lambda) everywhere this is oracle_fwd's recurrence.
 * Task = (b, h, block of S columns): column j of o only needs column j of S.
 * init / final_state as in oracle_fwd.
 */
void oracle_gla_fwd(const float *q, const float *k, const float *v, const float *a,
                    long sb, long sn, long sh, const double *init,
                    double *o, long ob, long on, long oh,
                    double *final_state, int B, long N, int H, int d) {
  int nblk = (d + BLK - 1) / BLK;
  long ntask = (long)B * H * nblk;
#pragma omp parallel for schedule(dynamic, 1)
  for (long task = 0; task < ntask; ++task) {
    int blk = (int)(task % nblk);
    int h = (int)((task / nblk) % H);
    int b = (int)(task / ((long)nblk * H));
    int j0 = blk * BLK, j1 = j0 + BLK < d ? j0 + BLK : d;
    double *S = (double *)calloc((size_t)d * d, sizeof(double));
    if (init) memcpy(S, st_bh(init, H, d, b, h), sizeof(double) * d * d);
    for (long s = 0; s < N; ++s) {
      const float *qs = tok(q, sb, sn, sh, b, s, h);
      const float *ks = tok(k, sb, sn, sh, b, s, h);
      const float *vs = tok(v, sb, sn, sh, b, s, h);
      const float *gs = tok(a, sb, sn, sh, b, s, h);
      double *os = tokd(o, ob, on, oh, b, s, h);
      for (int i = 0; i < d; ++i) {
        double g = exp((double)gs[i]);
        for (int j = j0; j < j1; ++j) S[i * d + j] = g * S[i * d + j] + (double)ks[i] * vs[j];
      }
      for (int j = j0; j < j1; ++j) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += (double)qs[i] * S[i * d + j];
        os[j] = acc;
      }
    }
    if (final_state) {
      double *F = st_bh_w(final_state, H, d, b, h);
      for (int i = 0; i < d; ++i)
        for (int j = j0; j < j1; ++j) F[i * d + j] = S[i * d + j];
    }
    free(S);
  }
}

/* Rows r0..r1-1 of the gated state after token s, from the rows after s-1. */
static void gla_rows_step(double *Sr, int r0, int r1, int d, const float *ks, const float *vs,
                          const float *gs) {
  for (int i = r0; i < r1; ++i) {
    double g = exp((double)gs[i]);
    double *row = Sr + (long)(i - r0) * d;
    for (int j = 0; j < d; ++j) row[j] = g * row[j] + (double)ks[i] * vs[j];
  }
}

/*
 * Gradients of L = sum_s o_s . do_s for oracle_gla_fwd, by the chain rule on
 * the recurrence (the gated counterpart of LASP Eq. 12-13).  With G_s the
 * gradient of L with respect to S_s:
 *   G_{N-1} = q_{N-1}^T do_{N-1} + dstate_in,
 *   G_s     = q_s^T do_s + diag(exp(a_{s+1})) G_{s+1};
 *   dq_s[i] = sum_j S_s[i][j] do_s[j]
 *   dk_s[i] = sum_j G_s[i][j] v_s[j]
 *   dv_s[j] = sum_i k_s[i] G_s[i][j]
 *   da_s[i] = exp(a_s[i]) sum_j G_s[i][j] S_{s-1}[i][j]   (S_{-1} = init or 0)
 *   dinit   = diag(exp(a_0)) G_0.
 * Tasks (b, h, sweep, block): sweep 0 = dq (rows of S, forward); sweep 1 = dk
 * and da (rows of G and S, reverse); sweep 2 = dv and dinit (columns of G).
 * Sweep 1 needs S_{s-1} while it walks backward: it keeps the rows of S every
 * K tokens (K about sqrt(N)) on the way forward and, for each block of K
 * tokens, recomputes the rows in between from the kept ones with the same
 * operations in the same order, so they are the very numbers of the forward.
 */
void oracle_gla_bwd(const float *q, const float *k, const float *v, const float *a, const float *dout,
                    long sb, long sn, long sh, const double *init, const double *dstate_in,
                    double *dq, double *dk, double *dv, double *da, long gb, long gn, long gh,
                    double *dinit, int B, long N, int H, int d) {
  int nblk = (d + BLK - 1) / BLK;
  long ntask = (long)B * H * 3 * nblk;
#pragma omp parallel for schedule(dynamic, 1)
  for (long task = 0; task < ntask; ++task) {
    int blk = (int)(task % nblk);
    int sweep = (int)((task / nblk) % 3);
    int h = (int)((task / (3L * nblk)) % H);
    int b = (int)(task / (3L * nblk * H));
    int r0 = blk * BLK, r1 = r0 + BLK < d ? r0 + BLK : d;
    int nr = r1 - r0;
    if (sweep == 0) {
      double *Sr = (double *)calloc((size_t)nr * d, sizeof(double));
      if (init) memcpy(Sr, st_bh(init, H, d, b, h) + (long)r0 * d, sizeof(double) * nr * d);
      for (long s = 0; s < N; ++s) {
        const float *ds = tok(dout, sb, sn, sh, b, s, h);
        double *dqs = tokd(dq, gb, gn, gh, b, s, h);
        gla_rows_step(Sr, r0, r1, d, tok(k, sb, sn, sh, b, s, h), tok(v, sb, sn, sh, b, s, h),
                      tok(a, sb, sn, sh, b, s, h));
        for (int i = r0; i < r1; ++i) {
          double acc = 0.0;
          for (int j = 0; j < d; ++j) acc += Sr[(long)(i - r0) * d + j] * ds[j];
          dqs[i] = acc;
        }
      }
      free(Sr);
    } else if (sweep == 1) {
      long K = (long)ceil(sqrt((double)(N > 0 ? N : 1)));
      long nck = (N + K - 1) / K;
      size_t rows = (size_t)nr * d;
      double *kept = (double *)calloc((size_t)(nck > 0 ? nck : 1) * rows, sizeof(double));
      double *buf = (double *)calloc((size_t)K * rows, sizeof(double));
      double *Sr = (double *)calloc(rows, sizeof(double));
      double *Gr = (double *)calloc(rows, sizeof(double));
      if (init) memcpy(Sr, st_bh(init, H, d, b, h) + (long)r0 * d, sizeof(double) * rows);
      for (long s = 0; s < N; ++s) {
        if (s % K == 0) memcpy(kept + (size_t)(s / K) * rows, Sr, sizeof(double) * rows);
        gla_rows_step(Sr, r0, r1, d, tok(k, sb, sn, sh, b, s, h), tok(v, sb, sn, sh, b, s, h),
                      tok(a, sb, sn, sh, b, s, h));
      }
      if (dstate_in) memcpy(Gr, st_bh(dstate_in, H, d, b, h) + (long)r0 * d, sizeof(double) * rows);
      for (long m = nck - 1; m >= 0; --m) {
        long t0 = m * K, t1 = t0 + K < N ? t0 + K : N;
        memcpy(Sr, kept + (size_t)m * rows, sizeof(double) * rows);
        for (long s = t0; s < t1; ++s) {
          gla_rows_step(Sr, r0, r1, d, tok(k, sb, sn, sh, b, s, h), tok(v, sb, sn, sh, b, s, h),
                        tok(a, sb, sn, sh, b, s, h));
          memcpy(buf + (size_t)(s - t0) * rows, Sr, sizeof(double) * rows);
        }
        for (long s = t1 - 1; s >= t0; --s) {
          const double *prev = s > t0 ? buf + (size_t)(s - 1 - t0) * rows : kept + (size_t)m * rows;
          const float *qs = tok(q, sb, sn, sh, b, s, h);
          const float *vs = tok(v, sb, sn, sh, b, s, h);
          const float *gs = tok(a, sb, sn, sh, b, s, h);
          const float *ds = tok(dout, sb, sn, sh, b, s, h);
          double *dks = tokd(dk, gb, gn, gh, b, s, h);
          double *das = tokd(da, gb, gn, gh, b, s, h);
          for (int i = r0; i < r1; ++i) {
            double g = exp((double)gs[i]);
            double *Gi = Gr + (long)(i - r0) * d;
            const double *Pi = prev + (long)(i - r0) * d;
            double acck = 0.0, acca = 0.0;
            for (int j = 0; j < d; ++j) {
              Gi[j] += (double)qs[i] * ds[j];
              acck += Gi[j] * vs[j];
              acca += Gi[j] * Pi[j];
            }
            dks[i] = acck;
            das[i] = g * acca;
            for (int j = 0; j < d; ++j) Gi[j] *= g;
          }
        }
      }
      free(kept);
      free(buf);
      free(Sr);
      free(Gr);
    } else {
      double *G = (double *)calloc((size_t)d * d, sizeof(double));
      if (dstate_in) memcpy(G, st_bh(dstate_in, H, d, b, h), sizeof(double) * d * d);
      for (long s = N - 1; s >= 0; --s) {
        const float *qs = tok(q, sb, sn, sh, b, s, h);
        const float *ks = tok(k, sb, sn, sh, b, s, h);
        const float *gs = tok(a, sb, sn, sh, b, s, h);
        const float *ds = tok(dout, sb, sn, sh, b, s, h);
        double *dvs = tokd(dv, gb, gn, gh, b, s, h);
        for (int i = 0; i < d; ++i)
          for (int j = r0; j < r1; ++j) G[i * d + j] += (double)qs[i] * ds[j];
        for (int j = r0; j < r1; ++j) {
          double acc = 0.0;
          for (int i = 0; i < d; ++i) acc += (double)ks[i] * G[i * d + j];
          dvs[j] = acc;
        }
        for (int i = 0; i < d; ++i) {
          double g = exp((double)gs[i]);
          for (int j = r0; j < r1; ++j) G[i * d + j] *= g;
        }
      }
      if (dinit) {
        double *D = st_bh_w(dinit, H, d, b, h);
        for (int i = 0; i < d; ++i)
          for (int j = r0; j < r1; ++j) D[i * d + j] = G[i * d + j];
      }
      free(G);
    }
  }
}

/*
 * Per-chunk states of the gated form, written out from their definition (the
 * gated counterparts of LASP Eq. 10 and of Eq. 20's (Lambda Q_t)^T dO_t): with
 * A_c(t0, t1)[i] = sum_{r=t0}^{t1} a_{cC+r}[i] (0 when t0 > t1),
 *   kind 0, (x, y) = (k, v):   M_c[i][j] = sum_t exp(A_c(t+1, C-1)[i]) x_t[i] y_t[j]
 *                              (the gates from token t to the end of the chunk);
 *   kind 1, (x, y) = (q, do):  M_c[i][j] = sum_t exp(A_c(0, t)[i]) x_t[i] y_t[j]
 *                              (the gates from the start of the chunk to token t);
 *   gsum[b, c, h, i] = A_c(0, C-1)[i], the chunk's total log-gate (if gsum is given).
 * M is [B, T, H, d, d] and gsum [B, T, H, d], T = N / C.
 */
void oracle_gla_chunk_states(const float *x, const float *y, const float *a, long sb, long sn, long sh,
                             double *M, double *gsum, int B, long N, int H, int d, long C, int kind) {
  long T = N / C;
  long ntask = (long)B * T * H;
#pragma omp parallel for schedule(dynamic, 1)
  for (long task = 0; task < ntask; ++task) {
    int h = (int)(task % H);
    long c = (task / H) % T;
    int b = (int)(task / ((long)H * T));
    double *Mc = M + st_btc((int)T, H, d, b, c, h);
    double *w = (double *)malloc(sizeof(double) * d);
    for (long e = 0; e < (long)d * d; ++e) Mc[e] = 0.0;
    for (long t = 0; t < C; ++t) {
      long r0 = kind == 0 ? t + 1 : 0, r1 = kind == 0 ? C - 1 : t;
      for (int i = 0; i < d; ++i) {
        double A = 0.0;
        for (long r = r0; r <= r1; ++r) A += (double)tok(a, sb, sn, sh, b, c * C + r, h)[i];
        w[i] = exp(A);
      }
      const float *xs = tok(x, sb, sn, sh, b, c * C + t, h);
      const float *ys = tok(y, sb, sn, sh, b, c * C + t, h);
      for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) Mc[i * d + j] += w[i] * (double)xs[i] * ys[j];
    }
    if (gsum) {
      double *gc = gsum + (((long)b * T + c) * H + h) * d;
      for (int i = 0; i < d; ++i) {
        double A = 0.0;
        for (long r = 0; r < C; ++r) A += (double)tok(a, sb, sn, sh, b, c * C + r, h)[i];
        gc[i] = A;
      }
    }
    free(w);
  }
}

/*
 * Scans over gated chunk states: each step through chunk c scales row i of
 * the carried state by exp(gsum_c[i]) (the product of the chunk's gates).
 *   reverse = 0:  P_0 = init (or 0);     P_c = diag(exp(gsum_{c-1})) P_{c-1} + M_{c-1};
 *                 total = diag(exp(gsum_{T-1})) P_{T-1} + M_{T-1}.
 *   reverse = 1:  R_{T-1} = init (or 0); R_c = diag(exp(gsum_{c+1})) R_{c+1} + M_{c+1};
 *                 total = diag(exp(gsum_0)) R_0 + M_0.
 * M, P: [B, T, H, d, d]; gsum: [B, T, H, d]; init, total: [B, H, d, d].
 */
void oracle_gla_state_scan(const double *M, const double *gsum, double *P, const double *init,
                           double *total, int B, long T, int H, int d, int reverse) {
  long ntask = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
  for (long task = 0; task < ntask; ++task) {
    int h = (int)(task % H);
    int b = (int)(task / H);
    double *acc = (double *)calloc((size_t)d * d, sizeof(double));
    if (init) memcpy(acc, st_bh(init, H, d, b, h), sizeof(double) * d * d);
    for (long n = 0; n < T; ++n) {
      long c = reverse ? T - 1 - n : n;
      const double *Mc = M + st_btc((int)T, H, d, b, c, h);
      const double *gc = gsum + (((long)b * T + c) * H + h) * d;
      double *Pc = P + st_btc((int)T, H, d, b, c, h);
      for (long e = 0; e < (long)d * d; ++e) Pc[e] = acc[e];
      for (int i = 0; i < d; ++i) {
        double g = exp(gc[i]);
        for (int j = 0; j < d; ++j) acc[i * d + j] = g * acc[i * d + j] + Mc[i * d + j];
      }
    }
    if (total) memcpy(st_bh_w(total, H, d, b, h), acc, sizeof(double) * d * d);
    free(acc);
  }
}

/*
 * State snapshots of the gated recurrences (what the backward pass needs at
 * chunk boundaries, LASP section 3.4 "KV State Caching"):
 *   kind 0, (x, y) = (k, v):  P_c = S_{cC-1}, the state entering chunk c
 *            (S_{-1} = init or 0), run token by token;
 *   kind 1, (x, y) = (q, do): R_c = X_{(c+1)C-1}, where X_s is the gradient of
 *            L with respect to S_s carried by the tokens after s:
 *            X_{N-1} = init (the dstate_in) or 0,
 *            X_{s-1} = diag(exp(a_s)) (X_s + q_s^T do_s).
 * P is [B, T, H, d, d].
 */
void oracle_gla_state_snapshots(const float *x, const float *y, const float *a, long sb, long sn, long sh,
                                const double *init, double *P, int B, long N, int H, int d, long C,
                                int kind) {
  long T = N / C;
  long ntask = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
  for (long task = 0; task < ntask; ++task) {
    int h = (int)(task % H);
    int b = (int)(task / H);
    double *S = (double *)calloc((size_t)d * d, sizeof(double));
    if (init) memcpy(S, st_bh(init, H, d, b, h), sizeof(double) * d * d);
    if (kind == 0) {
      for (long s = 0; s < N; ++s) {
        if (s % C == 0) memcpy(P + st_btc((int)T, H, d, b, s / C, h), S, sizeof(double) * d * d);
        const float *xs = tok(x, sb, sn, sh, b, s, h);
        const float *ys = tok(y, sb, sn, sh, b, s, h);
        const float *gs = tok(a, sb, sn, sh, b, s, h);
        for (int i = 0; i < d; ++i) {
          double g = exp((double)gs[i]);
          for (int j = 0; j < d; ++j) S[i * d + j] = g * S[i * d + j] + (double)xs[i] * ys[j];
        }
      }
    } else {
      for (long s = N - 1; s >= 0; --s) {
        if (s % C == C - 1) memcpy(P + st_btc((int)T, H, d, b, s / C, h), S, sizeof(double) * d * d);
        const float *xs = tok(x, sb, sn, sh, b, s, h);
        const float *ys = tok(y, sb, sn, sh, b, s, h);
        const float *gs = tok(a, sb, sn, sh, b, s, h);
        for (int i = 0; i < d; ++i) {
          double g = exp((double)gs[i]);
          for (int j = 0; j < d; ++j) S[i * d + j] = g * (S[i * d + j] + (double)xs[i] * ys[j]);
        }
      }
    }
    free(S);
  }
}

/* ------------------------------------------------------------------------
 * Softmax attention, the layers a hybrid model keeps (LASP-2 review page,
 * "Summary": LASP-2H applies the same AllGather pattern to standard attention
 * layers, each rank gathering K_t and V_t). Standard causal softmax attention,
 * per (b, h), with the queries of this call sitting at global positions
 * p_i = q_offset + i (i = 0..Nq-1) and the keys / values at positions
 * j = 0..Nk-1 (the gathered K and V):
 *   s_ij  = scale * (q_i . k_j)                      for j <= p_i
 *   a_ij  = exp(s_ij) / sum_{j' <= p_i} exp(s_ij')
 *   o_i   = sum_{j <= p_i} a_ij v_j
 *   lse_i = log sum_{j <= p_i} exp(s_ij)             (natural log)
 * The sums over j are taken after subtracting m_i = max_j s_ij (the textbook
 * way to keep exp in range; it cancels in a_ij). Requires q_offset + Nq <= Nk.
 * q, o: [B, Nq, H, d] (views qb/qn/qh, ob/on/oh); k, v: [B, Nk, H, d] (views
 * kb/kn/kh); lse: [B, H, Nq], may be NULL.
 * Task = (b, h, query row): each output row is one thread's sum, in key order.
 */
static double softmax_row_scores(const float *qi, const float *k, long kb, long kn, long kh, int b, int h, long last,
                                 int d, double scale, double *s) {
  double m = -INFINITY;
  for (long j = 0; j <= last; ++j) {
    const float *kj = tok(k, kb, kn, kh, b, j, h);
    double acc = 0.0;
    for (int f = 0; f < d; ++f) acc += (double)qi[f] * kj[f];
    s[j] = scale * acc;
    if (s[j] > m) m = s[j];
  }
  return m;
}

void oracle_softmax_fwd(const float *q, long qb, long qn, long qh, const float *k, const float *v, long kb, long kn,
                        long kh, double *o, long ob, long on, long oh, double *lse, int B, long Nq, long Nk,
                        long q_offset, int H, int d, double scale) {
  (void)Nk;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(q_offset + Nq));
#pragma omp for schedule(dynamic, 16)
    for (long task = 0; task < (long)B * H * Nq; ++task) {
      long i = task % Nq;
      int h = (int)((task / Nq) % H);
      int b = (int)(task / (Nq * H));
      long last = q_offset + i;
      const float *qi = tok(q, qb, qn, qh, b, i, h);
      double m = softmax_row_scores(qi, k, kb, kn, kh, b, h, last, d, scale, s);
      double l = 0.0;
      for (long j = 0; j <= last; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
      }
      double *oi = tokd(o, ob, on, oh, b, i, h);
      for (int f = 0; f < d; ++f) oi[f] = 0.0;
      for (long j = 0; j <= last; ++j) {
        const float *vj = tok(v, kb, kn, kh, b, j, h);
        double a = s[j] / l;
        for (int f = 0; f < d; ++f) oi[f] += a * vj[f];
      }
      if (lse) lse[((long)b * H + h) * Nq + i] = m + log(l);
    }
    free(s);
  }
}

/*
 * Its gradients for L = sum_i o_i . do_i (the chain rule through the softmax):
 *   dv_j  = sum_{i: p_i >= j} a_ij do_i
 *   da_ij = do_i . v_j,   ds_ij = a_ij (da_ij - sum_{j'} a_ij' da_ij')
 *   dq_i  = scale sum_j ds_ij k_j,    dk_j = scale sum_{i: p_i >= j} ds_ij q_i
 * dq: [B, Nq, H, d] (view gb/gn/gh); dk, dv: [B, Nk, H, d] (view eb/en/eh);
 * keys no query reaches get zero gradients. Three passes per (b, h): each
 * query's normaliser and sum_j a_ij da_ij; dq per query; dk and dv per key,
 * each row one thread's sum, in index order.
 */
void oracle_softmax_bwd(const float *q, long qb, long qn, long qh, const float *k, const float *v, long kb, long kn,
                        long kh, const float *dout, double *dq, long gb, long gn, long gh, double *dk, double *dv,
                        long eb, long en, long eh, int B, long Nq, long Nk, long q_offset, int H, int d,
                        double scale) {
  double *lse = (double *)malloc(sizeof(double) * (size_t)B * H * Nq);
  double *rs = (double *)malloc(sizeof(double) * (size_t)B * H * Nq); /* sum_j a_ij da_ij */
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(q_offset + Nq));
#pragma omp for schedule(dynamic, 16)
    for (long task = 0; task < (long)B * H * Nq; ++task) {
      long i = task % Nq;
      int h = (int)((task / Nq) % H);
      int b = (int)(task / (Nq * H));
      long last = q_offset + i;
      const float *qi = tok(q, qb, qn, qh, b, i, h);
      const float *di = tok(dout, qb, qn, qh, b, i, h);
      double m = softmax_row_scores(qi, k, kb, kn, kh, b, h, last, d, scale, s);
      double l = 0.0;
      for (long j = 0; j <= last; ++j) l += exp(s[j] - m);
      double r = 0.0;
      for (long j = 0; j <= last; ++j) {
        const float *vj = tok(v, kb, kn, kh, b, j, h);
        double da = 0.0;
        for (int f = 0; f < d; ++f) da += (double)di[f] * vj[f];
        r += exp(s[j] - m) / l * da;
      }
      lse[task] = m + log(l);
      rs[task] = r;
    }
#pragma omp for schedule(dynamic, 16)
    for (long task = 0; task < (long)B * H * Nq; ++task) {
      long i = task % Nq;
      int h = (int)((task / Nq) % H);
      int b = (int)(task / (Nq * H));
      long last = q_offset + i;
      const float *qi = tok(q, qb, qn, qh, b, i, h);
      const float *di = tok(dout, qb, qn, qh, b, i, h);
      double *dqi = tokd(dq, gb, gn, gh, b, i, h);
      for (int f = 0; f < d; ++f) dqi[f] = 0.0;
      softmax_row_scores(qi, k, kb, kn, kh, b, h, last, d, scale, s);
      for (long j = 0; j <= last; ++j) {
        const float *kj = tok(k, kb, kn, kh, b, j, h);
        const float *vj = tok(v, kb, kn, kh, b, j, h);
        double da = 0.0;
        for (int f = 0; f < d; ++f) da += (double)di[f] * vj[f];
        double a = exp(s[j] - lse[task]);
        double ds = a * (da - rs[task]);
        for (int f = 0; f < d; ++f) dqi[f] += scale * ds * kj[f];
      }
    }
#pragma omp for schedule(dynamic, 16)
    for (long task = 0; task < (long)B * H * Nk; ++task) {
      long j = task % Nk;
      int h = (int)((task / Nk) % H);
      int b = (int)(task / (Nk * H));
      const float *kj = tok(k, kb, kn, kh, b, j, h);
      const float *vj = tok(v, kb, kn, kh, b, j, h);
      double *dkj = tokd(dk, eb, en, eh, b, j, h);
      double *dvj = tokd(dv, eb, en, eh, b, j, h);
      for (int f = 0; f < d; ++f) {
        dkj[f] = 0.0;
        dvj[f] = 0.0;
      }
      long i0 = j > q_offset ? j - q_offset : 0; /* the first query with p_i >= j */
      for (long i = i0; i < Nq; ++i) {
        const float *qi = tok(q, qb, qn, qh, b, i, h);
        const float *di = tok(dout, qb, qn, qh, b, i, h);
        long row = ((long)b * H + h) * Nq + i;
        double sij = 0.0, da = 0.0;
        for (int f = 0; f < d; ++f) {
          sij += (double)qi[f] * kj[f];
          da += (double)di[f] * vj[f];
        }
        double a = exp(scale * sij - lse[row]);
        double ds = a * (da - rs[row]);
        for (int f = 0; f < d; ++f) {
          dvj[f] += a * di[f];
          dkj[f] += scale * ds * qi[f];
        }
      }
    }
    free(s);
  }
  free(lse);
  free(rs);
}
