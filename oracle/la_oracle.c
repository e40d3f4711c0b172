/*
 * la_oracle.c -- float64 CPU oracle for causal linear attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path loads this library:
 * only the test suite, the smoke check in __graft_entry__.py and the
 * cpu_baseline / reference legs of bench.py may load or call it.  It shares no
 * code, header, table or helper with the CUDA library.
 *
 * What it computes (the plain definition, no blocking or reordering):
 *   "1.6 长上下文与高效注意力" (long context and efficient attention), section
 *   线性注意力 (linear attention), the displayed equation
 *       o_t = S_t phi(q_t) / (z_t^T phi(q_t)),
 *       S_t = S_{t-1} + v_t phi(k_t)^T,   z_t = z_{t-1} + phi(k_t),
 *   with S a d_v x d_k matrix started at zero, phi(x) = elu(x) + 1 or the
 *   identity, and a per-head constant decay gamma multiplying the old state:
 *       S_t = gamma S_{t-1} + v_t phi(k_t)^T,  z_t = gamma z_{t-1} + phi(k_t).
 *   gamma = 1 is the page's equation exactly.  The state includes token t
 *   before o_t is read (the sum in the displayed equation runs over j <= t).
 *
 * Functions:
 *   oracle_recurrent  -- the token-by-token recurrence above (prefill).
 *   oracle_chunked    -- the same result regrouped into chunks of C tokens;
 *                        the chunk form is derived in the header comment of
 *                        that function.  It exists to pin the derivation that
 *                        a chunked implementation relies on (results must not
 *                        depend on C beyond rounding).
 *   oracle_step       -- one decode token on a given state, in place.
 *   oracle_final_z    -- the normaliser's key sum z after the last token of
 *                        each sequence (the z a normalised decode continues
 *                        from).
 *   oracle_step_norm  -- one normalised decode token: S and z updated in
 *                        place, o_t = S_t phi(q_t) / (z_t^T phi(q_t)).
 *   oracle_backward   -- dq, dk, dv of sum_t dout_t . o_t for the unnormalised
 *                        recurrence: the adjoint of the definition.
 *   oracle_backward_gated -- the same for the per-token decay, plus the
 *                        gradient of the log decays g.
 *   oracle_backward_gated_norm -- the normalised per-token-decay forward's
 *                        adjoint (dq, dk, dv, dg).
 *   oracle_norm_gate  -- RMSNorm over d_v times a Swish gate, per (token, head).
 *   oracle_gated_delta -- the gated delta rule, token by token.
 *   oracle_gated_delta_chunked -- the same rule regrouped into chunks (the
 *                        WY / UT form of a chunked kernel), to pin that
 *                        algebra against the token-by-token definition.
 *   oracle_recurrent_gated, oracle_step_gated -- the same with a per-token
 *                        (per decode step) decay alpha_t = exp(g_t) in place
 *                        of the per-head constant gamma.
 *
 * Layouts (all row-major, last dimension contiguous):
 *   q, k  [B, T, H, d_k];  v  [B, T, H, d_v];  out  [B, T, H, d_v] (double)
 *   with cu_seqlens != NULL: B must be 1 and sequence n occupies tokens
 *   cu_seqlens[n] .. cu_seqlens[n+1]-1 of the packed T axis.
 *   final_state [n_seqs, H, d_k, d_v] (double) holds S^T (entry [c][r] is
 *   S[r][c]); NULL skips it.
 *   Inputs may be float32, bfloat16 (raw uint16 bits) or float64; they are
 *   upcast to double exactly on every read.
 *
 * Return value: 0 on success, a negative number for a bad argument.
 */
#include <math.h>

/* A task could not allocate its working buffers (inputs too large for this host). */
#define ORC_ERR_NOMEM (-20)
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_F64 2

#define ORC_PHI_IDENTITY 0
#define ORC_PHI_ELU1 1

#define ROWS_PER_TASK 8

static double orc_load(const void *p, int dtype, int64_t i) {
  if (dtype == ORC_F32) return (double)((const float *)p)[i];
  if (dtype == ORC_BF16) {
    uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return ((const double *)p)[i];
}

/* elu with alpha = 1, plus one: x + 1 for x > 0, exp(x) otherwise. */
static double orc_phi(double x, int phi) {
  if (phi == ORC_PHI_ELU1) return x > 0.0 ? x + 1.0 : exp(x);
  return x;
}

static int orc_check(int dtype, int64_t B, int64_t T, int64_t H, int64_t dk,
                     int64_t dv, const int32_t *cu, int64_t n_seqs, int phi) {
  if (dtype < ORC_F32 || dtype > ORC_F64) return -1;
  if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return -2;
  if (phi != ORC_PHI_IDENTITY && phi != ORC_PHI_ELU1) return -3;
  if (cu) {
    if (B != 1 || n_seqs < 0) return -4;
    if (cu[0] != 0) return -5;
    for (int64_t n = 0; n < n_seqs; ++n)
      if (cu[n + 1] < cu[n]) return -6;
    if ((int64_t)cu[n_seqs] > T) return -7;
  } else if (n_seqs != B) {
    return -8;
  }
  return 0;
}

static void orc_seq(const int32_t *cu, int64_t T, int64_t n, int64_t *start,
                    int64_t *len) {
  if (cu) {
    *start = cu[n];
    *len = (int64_t)cu[n + 1] - cu[n];
  } else {
    *start = n * T;
    *len = T;
  }
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * The recurrence, token by token.  Row r of S depends only on column r of v
 * and on phi(k), so the work splits into independent tasks over
 * (sequence, head, block of rows of S); z is recomputed inside each task.
 */
int oracle_recurrent(const void *q, const void *k, const void *v, int dtype,
                     int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                     const double *gamma, const int32_t *cu_seqlens,
                     int64_t n_seqs, int phi, int normalize, double *out,
                     double *final_state, int nthreads) {
  int rc = orc_check(dtype, B, T, H, dk, dv, cu_seqlens, n_seqs, phi);
  if (rc) return rc;
  const int64_t nblk = (dv + ROWS_PER_TASK - 1) / ROWS_PER_TASK;
  const int64_t ntask = n_seqs * H * nblk;
  if (nthreads <= 0) nthreads = oracle_max_threads();

  int oom = 0; /* set when a task could not allocate its buffers */
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
  for (int64_t task = 0; task < ntask; ++task) {
    const int64_t n = task / (H * nblk);
    const int64_t h = (task / nblk) % H;
    const int64_t r0 = (task % nblk) * ROWS_PER_TASK;
    const int64_t nr = dv - r0 < ROWS_PER_TASK ? dv - r0 : ROWS_PER_TASK;
    int64_t start, len;
    orc_seq(cu_seqlens, T, n, &start, &len);
    const double g = gamma[h];

    double *S = (double *)calloc((size_t)(ROWS_PER_TASK * dk), sizeof(double));
    double *z = (double *)calloc((size_t)dk, sizeof(double));
    double *qh = (double *)malloc((size_t)dk * sizeof(double));
    double *kh = (double *)malloc((size_t)dk * sizeof(double));
    if (!S || !z || !qh || !kh) {
      free(S); free(z); free(qh); free(kh);
#pragma omp atomic write
      oom = 1;
      continue;
    }

    for (int64_t t = 0; t < len; ++t) {
      const int64_t tok = start + t;
      const int64_t qk_base = (tok * H + h) * dk;
      const int64_t v_base = (tok * H + h) * dv;
      for (int64_t c = 0; c < dk; ++c) {
        qh[c] = orc_phi(orc_load(q, dtype, qk_base + c), phi);
        kh[c] = orc_phi(orc_load(k, dtype, qk_base + c), phi);
      }
      double den = 1.0;
      if (normalize) {
        den = 0.0;
        for (int64_t c = 0; c < dk; ++c) {
          z[c] = g * z[c] + kh[c];
          den += z[c] * qh[c];
        }
      }
      for (int64_t i = 0; i < nr; ++i) {
        const double vr = orc_load(v, dtype, v_base + r0 + i);
        double *Sr = S + i * dk;
        double num = 0.0;
        for (int64_t c = 0; c < dk; ++c) {
          Sr[c] = g * Sr[c] + vr * kh[c];
          num += Sr[c] * qh[c];
        }
        out[v_base + r0 + i] = num / den;
      }
    }
    if (final_state) {
      double *F = final_state + (n * H + h) * dk * dv;
      for (int64_t i = 0; i < nr; ++i)
        for (int64_t c = 0; c < dk; ++c) F[c * dv + r0 + i] = S[i * dk + c];
    }
    free(S);
    free(z);
    free(qh);
    free(kh);
  }
  return oom ? ORC_ERR_NOMEM : 0;
}

/*
 * The chunked form.  Unrolling the recurrence from a chunk whose first token
 * sees the state S_p (and z_p), for positions i, j = 0 .. C'-1 inside a chunk
 * of C' tokens:
 *   S after token i   = gamma^(i+1) S_p + sum_{j<=i} gamma^(i-j) v_j kh_j^T
 *   o_i (numerator)   = gamma^(i+1) S_p qh_i + sum_{j<=i} gamma^(i-j) (qh_i.kh_j) v_j
 *   den_i             = gamma^(i+1) z_p.qh_i + sum_{j<=i} gamma^(i-j) (qh_i.kh_j)
 *   S_next            = gamma^C' S_p + sum_j gamma^(C'-1-j) v_j kh_j^T
 *   z_next            = gamma^C' z_p + sum_j gamma^(C'-1-j) kh_j
 * Chunks restart at each sequence start; the last chunk of a sequence holds
 * the remaining len mod C tokens when that is not zero.
 */
int oracle_chunked(const void *q, const void *k, const void *v, int dtype,
                   int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                   const double *gamma, const int32_t *cu_seqlens,
                   int64_t n_seqs, int64_t chunk, int phi, int normalize,
                   double *out, double *final_state, int nthreads) {
  int rc = orc_check(dtype, B, T, H, dk, dv, cu_seqlens, n_seqs, phi);
  if (rc) return rc;
  if (chunk <= 0) return -9;
  if (nthreads <= 0) nthreads = oracle_max_threads();

  int oom = 0; /* set when a task could not allocate its buffers */
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
  for (int64_t task = 0; task < n_seqs * H; ++task) {
    const int64_t n = task / H, h = task % H;
    int64_t start, len;
    orc_seq(cu_seqlens, T, n, &start, &len);
    const double g = gamma[h];
    double *S = (double *)calloc((size_t)(dv * dk), sizeof(double)); /* S[r][c] */
    double *Sn = (double *)malloc((size_t)(dv * dk) * sizeof(double));
    double *z = (double *)calloc((size_t)dk, sizeof(double));
    double *zn = (double *)malloc((size_t)dk * sizeof(double));
    double *qh = (double *)malloc((size_t)(chunk * dk) * sizeof(double));
    double *kh = (double *)malloc((size_t)(chunk * dk) * sizeof(double));
    double *vv = (double *)malloc((size_t)(chunk * dv) * sizeof(double));
    if (!S || !Sn || !z || !zn || !qh || !kh || !vv) {
      free(S); free(Sn); free(z); free(zn); free(qh); free(kh); free(vv);
#pragma omp atomic write
      oom = 1;
      continue;
    }

    for (int64_t c0 = 0; c0 < len; c0 += chunk) {
      const int64_t Cp = len - c0 < chunk ? len - c0 : chunk;
      for (int64_t i = 0; i < Cp; ++i) {
        const int64_t tok = start + c0 + i;
        for (int64_t c = 0; c < dk; ++c) {
          qh[i * dk + c] = orc_phi(orc_load(q, dtype, (tok * H + h) * dk + c), phi);
          kh[i * dk + c] = orc_phi(orc_load(k, dtype, (tok * H + h) * dk + c), phi);
        }
        for (int64_t r = 0; r < dv; ++r)
          vv[i * dv + r] = orc_load(v, dtype, (tok * H + h) * dv + r);
      }
      /* outputs of the chunk */
      for (int64_t i = 0; i < Cp; ++i) {
        const double gi1 = pow(g, (double)(i + 1));
        double den = 0.0;
        for (int64_t c = 0; c < dk; ++c) den += z[c] * qh[i * dk + c];
        den *= gi1;
        double *o = out + ((start + c0 + i) * H + h) * dv;
        for (int64_t r = 0; r < dv; ++r) {
          double acc = 0.0;
          for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * qh[i * dk + c];
          o[r] = gi1 * acc;
        }
        for (int64_t j = 0; j <= i; ++j) {
          double a = 0.0;
          for (int64_t c = 0; c < dk; ++c) a += qh[i * dk + c] * kh[j * dk + c];
          const double p = pow(g, (double)(i - j)) * a;
          den += p;
          for (int64_t r = 0; r < dv; ++r) o[r] += p * vv[j * dv + r];
        }
        if (normalize)
          for (int64_t r = 0; r < dv; ++r) o[r] /= den;
      }
      /* state carried to the next chunk */
      const double gC = pow(g, (double)Cp);
      for (int64_t r = 0; r < dv; ++r)
        for (int64_t c = 0; c < dk; ++c) Sn[r * dk + c] = gC * S[r * dk + c];
      for (int64_t c = 0; c < dk; ++c) zn[c] = gC * z[c];
      for (int64_t j = 0; j < Cp; ++j) {
        const double w = pow(g, (double)(Cp - 1 - j));
        for (int64_t c = 0; c < dk; ++c) zn[c] += w * kh[j * dk + c];
        for (int64_t r = 0; r < dv; ++r) {
          const double wv = w * vv[j * dv + r];
          for (int64_t c = 0; c < dk; ++c) Sn[r * dk + c] += wv * kh[j * dk + c];
        }
      }
      memcpy(S, Sn, (size_t)(dv * dk) * sizeof(double));
      memcpy(z, zn, (size_t)dk * sizeof(double));
    }
    if (final_state) {
      double *F = final_state + (n * H + h) * dk * dv;
      for (int64_t r = 0; r < dv; ++r)
        for (int64_t c = 0; c < dk; ++c) F[c * dv + r] = S[r * dk + c];
    }
    free(S);
    free(Sn);
    free(z);
    free(zn);
    free(qh);
    free(kh);
    free(vv);
  }
  return oom ? ORC_ERR_NOMEM : 0;
}

/*
 * One decode token: the recurrence applied once to a given state.
 *   q, k [N, H, d_k];  v [N, H, d_v] (any input dtype above)
 *   state [N, H, d_k, d_v] double, holding S^T, updated in place:
 *       S^T[c][r] <- gamma S^T[c][r] + kh_c v_r
 *   out [N, H, d_v] double:  o_r = sum_c S^T[c][r] qh_c   (after the update)
 */
int oracle_step(const void *q, const void *k, const void *v, int dtype,
                int64_t N, int64_t H, int64_t dk, int64_t dv,
                const double *gamma, double *state, double *out, int phi,
                int nthreads) {
  int rc = orc_check(dtype, 1, 1, H, dk, dv, NULL, 1, phi);
  if (rc) return rc;
  if (N < 0) return -2;
  if (nthreads <= 0) nthreads = oracle_max_threads();

#pragma omp parallel for schedule(static) num_threads(nthreads)
  for (int64_t task = 0; task < N * H; ++task) {
    const int64_t h = task % H;
    const double g = gamma[h];
    double *St = state + task * dk * dv;
    double *o = out + task * dv;
    for (int64_t r = 0; r < dv; ++r) o[r] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
      const double qc = orc_phi(orc_load(q, dtype, task * dk + c), phi);
      const double kc = orc_phi(orc_load(k, dtype, task * dk + c), phi);
      for (int64_t r = 0; r < dv; ++r) {
        const double s = g * St[c * dv + r] + kc * orc_load(v, dtype, task * dv + r);
        St[c * dv + r] = s;
        o[r] += s * qc;
      }
    }
  }
  return 0;
}

/*
 * z after the last token of each sequence, token by token:
 *   z_t = gamma z_{t-1} + phi(k_t),  z_{-1} = 0.
 *   k [B, T, H, d_k] (cu_seqlens as above);  final_z [n_seqs, H, d_k] double.
 */
int oracle_final_z(const void *k, int dtype, int64_t B, int64_t T, int64_t H, int64_t dk,
                   const double *gamma, const int32_t *cu_seqlens, int64_t n_seqs, int phi,
                   double *final_z, int nthreads) {
  int rc = orc_check(dtype, B, T, H, dk, 1, cu_seqlens, n_seqs, phi);
  if (rc) return rc;
  if (nthreads <= 0) nthreads = oracle_max_threads();

#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
  for (int64_t task = 0; task < n_seqs * H; ++task) {
    const int64_t n = task / H, h = task % H;
    int64_t start, len;
    orc_seq(cu_seqlens, T, n, &start, &len);
    double *z = final_z + task * dk;
    for (int64_t c = 0; c < dk; ++c) z[c] = 0.0;
    for (int64_t t = 0; t < len; ++t) {
      const int64_t base = ((start + t) * H + h) * dk;
      for (int64_t c = 0; c < dk; ++c) z[c] = gamma[h] * z[c] + orc_phi(orc_load(k, dtype, base + c), phi);
    }
  }
  return 0;
}

/*
 * One normalised decode token (the displayed equation applied once):
 *   z[c] <- gamma z[c] + kh_c,   S^T[c][r] <- gamma S^T[c][r] + kh_c v_r,
 *   o_r = (sum_c S^T[c][r] qh_c) / (sum_c z[c] qh_c).
 *   q, k [N, H, d_k]; v [N, H, d_v]; state [N, H, d_k, d_v] and z [N, H, d_k]
 *   double, updated in place; out [N, H, d_v] double.
 */
int oracle_step_norm(const void *q, const void *k, const void *v, int dtype,
                     int64_t N, int64_t H, int64_t dk, int64_t dv,
                     const double *gamma, double *state, double *z, double *out, int phi,
                     int nthreads) {
  int rc = orc_check(dtype, 1, 1, H, dk, dv, NULL, 1, phi);
  if (rc) return rc;
  if (N < 0) return -2;
  if (nthreads <= 0) nthreads = oracle_max_threads();

#pragma omp parallel for schedule(static) num_threads(nthreads)
  for (int64_t task = 0; task < N * H; ++task) {
    const int64_t h = task % H;
    const double g = gamma[h];
    double *St = state + task * dk * dv;
    double *zt = z + task * dk;
    double *o = out + task * dv;
    double den = 0.0;
    for (int64_t r = 0; r < dv; ++r) o[r] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
      const double qc = orc_phi(orc_load(q, dtype, task * dk + c), phi);
      const double kc = orc_phi(orc_load(k, dtype, task * dk + c), phi);
      zt[c] = g * zt[c] + kc;
      den += zt[c] * qc;
      for (int64_t r = 0; r < dv; ++r) {
        const double s = g * St[c * dv + r] + kc * orc_load(v, dtype, task * dv + r);
        St[c * dv + r] = s;
        o[r] += s * qc;
      }
    }
    for (int64_t r = 0; r < dv; ++r) o[r] /= den;
  }
  return 0;
}

/*
 * Data-dependent decay ("1.6 长上下文与高效注意力", section 状态空间模型与 Mamba:
 * a state-space recurrence whose decay is a function of the input token, which
 * Mamba-2 restricts to a scalar per step and shows to be linear attention with
 * a decay mask).  The constant gamma of oracle_recurrent becomes a per-token,
 * per-head factor alpha_t = exp(g_t), g_t <= 0 given in log space:
 *     S_t = alpha_t S_{t-1} + v_t phi(k_t)^T,   z_t = alpha_t z_{t-1} + phi(k_t),
 *     o_t = S_t phi(q_t)   [ / (z_t^T phi(q_t)) ].
 *   g  [B, T, H] double (contiguous; packed batches as for q).
 *   Other arguments as for oracle_recurrent; final_z [n_seqs, H, d_k] or NULL.
 */
int oracle_recurrent_gated(const void *q, const void *k, const void *v, int dtype,
                           int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                           const double *g, const int32_t *cu_seqlens, int64_t n_seqs,
                           int phi, int normalize, double *out, double *final_state,
                           double *final_z, int nthreads) {
  int rc = orc_check(dtype, B, T, H, dk, dv, cu_seqlens, n_seqs, phi);
  if (rc) return rc;
  if (!g) return -10;
  if (nthreads <= 0) nthreads = oracle_max_threads();

  int oom = 0; /* set when a task could not allocate its buffers */
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
  for (int64_t task = 0; task < n_seqs * H; ++task) {
    const int64_t n = task / H, h = task % H;
    int64_t start, len;
    orc_seq(cu_seqlens, T, n, &start, &len);
    double *S = (double *)calloc((size_t)(dv * dk), sizeof(double));
    double *z = (double *)calloc((size_t)dk, sizeof(double));
    double *qh = (double *)malloc((size_t)dk * sizeof(double));
    double *kh = (double *)malloc((size_t)dk * sizeof(double));
    if (!S || !z || !qh || !kh) {
      free(S); free(z); free(qh); free(kh);
#pragma omp atomic write
      oom = 1;
      continue;
    }
    for (int64_t t = 0; t < len; ++t) {
      const int64_t row = start + t;  /* token row of the flattened [B * T] grid */
      const double a = exp(g[row * H + h]);
      const int64_t qk_base = (row * H + h) * dk;
      const int64_t v_base = (row * H + h) * dv;
      for (int64_t c = 0; c < dk; ++c) {
        qh[c] = orc_phi(orc_load(q, dtype, qk_base + c), phi);
        kh[c] = orc_phi(orc_load(k, dtype, qk_base + c), phi);
      }
      double den = 0.0;
      for (int64_t c = 0; c < dk; ++c) {
        z[c] = a * z[c] + kh[c];
        den += z[c] * qh[c];
      }
      if (!normalize) den = 1.0;
      for (int64_t r = 0; r < dv; ++r) {
        const double vr = orc_load(v, dtype, v_base + r);
        double *Sr = S + r * dk;
        double num = 0.0;
        for (int64_t c = 0; c < dk; ++c) {
          Sr[c] = a * Sr[c] + vr * kh[c];
          num += Sr[c] * qh[c];
        }
        out[v_base + r] = num / den;
      }
    }
    if (final_state) {
      double *F = final_state + task * dk * dv;
      for (int64_t r = 0; r < dv; ++r)
        for (int64_t c = 0; c < dk; ++c) F[c * dv + r] = S[r * dk + c];
    }
    if (final_z)
      for (int64_t c = 0; c < dk; ++c) final_z[task * dk + c] = z[c];
    free(S);
    free(z);
    free(qh);
    free(kh);
  }
  return oom ? ORC_ERR_NOMEM : 0;
}

/*
 * One decode token with a per-(sequence, head) decay alpha = exp(g[n][h]):
 * oracle_step (z == NULL) or oracle_step_norm (z != NULL) with gamma replaced
 * by alpha.  g [N, H] double.
 */
int oracle_step_gated(const void *q, const void *k, const void *v, int dtype,
                      int64_t N, int64_t H, int64_t dk, int64_t dv,
                      const double *g, double *state, double *z, double *out, int phi,
                      int nthreads) {
  int rc = orc_check(dtype, 1, 1, H, dk, dv, NULL, 1, phi);
  if (rc) return rc;
  if (N < 0) return -2;
  if (nthreads <= 0) nthreads = oracle_max_threads();

#pragma omp parallel for schedule(static) num_threads(nthreads)
  for (int64_t task = 0; task < N * H; ++task) {
    const double a = exp(g[task]);
    double *St = state + task * dk * dv;
    double *o = out + task * dv;
    double den = 0.0;
    for (int64_t r = 0; r < dv; ++r) o[r] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
      const double qc = orc_phi(orc_load(q, dtype, task * dk + c), phi);
      const double kc = orc_phi(orc_load(k, dtype, task * dk + c), phi);
      if (z) {
        z[task * dk + c] = a * z[task * dk + c] + kc;
        den += z[task * dk + c] * qc;
      }
      for (int64_t r = 0; r < dv; ++r) {
        const double s = a * St[c * dv + r] + kc * orc_load(v, dtype, task * dv + r);
        St[c * dv + r] = s;
        o[r] += s * qc;
      }
    }
    if (z)
      for (int64_t r = 0; r < dv; ++r) o[r] /= den;
  }
  return 0;
}

/*
 * Backward of the unnormalised recurrence (per-head gamma), the adjoint of
 * the definition token by token.  With L = sum_t dout_t . o_t:
 *   forward:   S_t = gamma S_{t-1} + v_t kh_t^T,  o_t = S_t qh_t
 *   dqh_t  = S_t^T dout_t
 *   G_t    = dL/dS_t = dout_t qh_t^T + gamma G_{t+1}      (G_{len} = 0)
 *   dkh_t  = G_t^T v_t,   dv_t = G_t kh_t
 *   dq = dqh * phi'(q),   dk = dkh * phi'(k)   (phi' = 1, or for elu + 1:
 *                                                1 if x > 0 else e^x)
 *   dout [B, T, H, d_v]; dq, dk [B, T, H, d_k], dv [B, T, H, d_v] (double).
 * The normalised form is not covered (returns -11 if normalize is set).
 */
static double orc_dphi(double x, int phi) {
  if (phi == ORC_PHI_ELU1) return x > 0.0 ? 1.0 : exp(x);
  return 1.0;
}

int oracle_backward(const void *q, const void *k, const void *v, const void *dout, int dtype,
                    int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                    const double *gamma, const int32_t *cu_seqlens, int64_t n_seqs, int phi,
                    int normalize, double *dq, double *dkk, double *dvv, int nthreads) {
  int rc = orc_check(dtype, B, T, H, dk, dv, cu_seqlens, n_seqs, phi);
  if (rc) return rc;
  if (normalize) return -11;
  if (nthreads <= 0) nthreads = oracle_max_threads();

  int oom = 0; /* set when a task could not allocate its buffers */
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
  for (int64_t task = 0; task < n_seqs * H; ++task) {
    const int64_t n = task / H, h = task % H;
    int64_t start, len;
    orc_seq(cu_seqlens, T, n, &start, &len);
    const double g = gamma[h];
    double *S = (double *)calloc((size_t)(dv * dk), sizeof(double));  /* S[r][c] */
    double *qh = (double *)malloc((size_t)dk * sizeof(double));
    double *kh = (double *)malloc((size_t)dk * sizeof(double));
    if (!S || !qh || !kh) {
      free(S); free(qh); free(kh);
#pragma omp atomic write
      oom = 1;
      continue;
    }
    /* forward in time: dqh_t = S_t^T dout_t */
    for (int64_t t = 0; t < len; ++t) {
      const int64_t row = start + t;
      const int64_t qk = (row * H + h) * dk, vb = (row * H + h) * dv;
      for (int64_t c = 0; c < dk; ++c) kh[c] = orc_phi(orc_load(k, dtype, qk + c), phi);
      for (int64_t r = 0; r < dv; ++r) {
        const double vr = orc_load(v, dtype, vb + r);
        for (int64_t c = 0; c < dk; ++c) S[r * dk + c] = g * S[r * dk + c] + vr * kh[c];
      }
      for (int64_t c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int64_t r = 0; r < dv; ++r) acc += S[r * dk + c] * orc_load(dout, dtype, vb + r);
        const double x = orc_load(q, dtype, qk + c);
        dq[qk + c] = acc * orc_dphi(x, phi);
      }
    }
    /* backward in time: G_t = dout_t qh_t^T + gamma G_{t+1} */
    double *Gm = S;
    memset(Gm, 0, (size_t)(dv * dk) * sizeof(double));
    for (int64_t t = len - 1; t >= 0; --t) {
      const int64_t row = start + t;
      const int64_t qk = (row * H + h) * dk, vb = (row * H + h) * dv;
      for (int64_t c = 0; c < dk; ++c) {
        qh[c] = orc_phi(orc_load(q, dtype, qk + c), phi);
        kh[c] = orc_phi(orc_load(k, dtype, qk + c), phi);
      }
      for (int64_t r = 0; r < dv; ++r) {
        const double d = orc_load(dout, dtype, vb + r);
        for (int64_t c = 0; c < dk; ++c) Gm[r * dk + c] = g * Gm[r * dk + c] + d * qh[c];
      }
      for (int64_t c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int64_t r = 0; r < dv; ++r) acc += Gm[r * dk + c] * orc_load(v, dtype, vb + r);
        dkk[qk + c] = acc * orc_dphi(orc_load(k, dtype, qk + c), phi);
      }
      for (int64_t r = 0; r < dv; ++r) {
        double acc = 0.0;
        for (int64_t c = 0; c < dk; ++c) acc += Gm[r * dk + c] * kh[c];
        dvv[vb + r] = acc;
      }
    }
    free(S);
    free(qh);
    free(kh);
  }
  return oom ? ORC_ERR_NOMEM : 0;
}

/*
 * Backward of the normalised recurrence (per-head gamma), the adjoint of the
 * definition token by token ("1.6 长上下文与高效注意力", section 线性注意力: the
 * output divided by z_t^T phi(q_t)).  With L = sum_t dout_t . o_t:
 *   forward:   S_t = gamma S_{t-1} + v_t kh_t^T,   z_t = gamma z_{t-1} + kh_t,
 *              num_t = S_t qh_t,   den_t = z_t . qh_t,   o_t = num_t / den_t
 *   u_t    = dL/dnum_t = dout_t / den_t
 *   e_t    = dL/dden_t = -(dout_t . o_t) / den_t
 *   dqh_t  = S_t^T u_t + e_t z_t
 *   G_t    = dL/dS_t = u_t qh_t^T + gamma G_{t+1},   g_t = dL/dz_t = e_t qh_t + gamma g_{t+1}
 *   dkh_t  = G_t^T v_t + g_t,   dv_t = G_t kh_t
 *   dq = dqh * phi'(q),   dk = dkh * phi'(k).
 * The forward sweep keeps u_t and e_t of every token of the task (len * (d_v + 1)
 * doubles) for the backward sweep.  Arguments as for oracle_backward.
 */
int oracle_backward_norm(const void *q, const void *k, const void *v, const void *dout, int dtype,
                         int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                         const double *gamma, const int32_t *cu_seqlens, int64_t n_seqs, int phi,
                         double *dq, double *dkk, double *dvv, int nthreads) {
  int rc = orc_check(dtype, B, T, H, dk, dv, cu_seqlens, n_seqs, phi);
  if (rc) return rc;
  if (nthreads <= 0) nthreads = oracle_max_threads();

  int oom = 0; /* set when a task could not allocate its buffers */
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
  for (int64_t task = 0; task < n_seqs * H; ++task) {
    const int64_t n = task / H, h = task % H;
    int64_t start, len;
    orc_seq(cu_seqlens, T, n, &start, &len);
    const double g = gamma[h];
    const size_t nl = (size_t)(len > 0 ? len : 1);
    double *S = (double *)calloc((size_t)(dv * dk), sizeof(double)); /* S[r][c] */
    double *z = (double *)calloc((size_t)dk, sizeof(double));
    double *qh = (double *)malloc((size_t)dk * sizeof(double));
    double *kh = (double *)malloc((size_t)dk * sizeof(double));
    double *U = (double *)malloc(nl * (size_t)dv * sizeof(double)); /* u_t, every t */
    double *E = (double *)malloc(nl * sizeof(double));               /* e_t, every t */
    double *num = (double *)malloc((size_t)dv * sizeof(double));
    if (!S || !z || !qh || !kh || !U || !E || !num) {
      free(S); free(z); free(qh); free(kh); free(U); free(E); free(num);
#pragma omp atomic write
      oom = 1;
      continue;
    }
    /* forward in time: the outputs' adjoints and dqh */
    for (int64_t t = 0; t < len; ++t) {
      const int64_t row = start + t;
      const int64_t qk = (row * H + h) * dk, vb = (row * H + h) * dv;
      for (int64_t c = 0; c < dk; ++c) {
        qh[c] = orc_phi(orc_load(q, dtype, qk + c), phi);
        kh[c] = orc_phi(orc_load(k, dtype, qk + c), phi);
      }
      double den = 0.0;
      for (int64_t c = 0; c < dk; ++c) {
        z[c] = kh[c] + g * z[c];
        den += z[c] * qh[c];
      }
      double dot = 0.0; /* dout_t . o_t */
      for (int64_t r = 0; r < dv; ++r) {
        const double vr = orc_load(v, dtype, vb + r);
        double acc = 0.0;
        for (int64_t c = 0; c < dk; ++c) {
          S[r * dk + c] = g * S[r * dk + c] + vr * kh[c];
          acc += S[r * dk + c] * qh[c];
        }
        num[r] = acc;
        dot += orc_load(dout, dtype, vb + r) * (acc / den);
      }
      double *u = U + (size_t)t * dv;
      for (int64_t r = 0; r < dv; ++r) u[r] = orc_load(dout, dtype, vb + r) / den;
      E[t] = -dot / den;
      for (int64_t c = 0; c < dk; ++c) {
        double acc = E[t] * z[c];
        for (int64_t r = 0; r < dv; ++r) acc += S[r * dk + c] * u[r];
        dq[qk + c] = acc * orc_dphi(orc_load(q, dtype, qk + c), phi);
      }
    }
    /* backward in time: G (in S's buffer) and g (in z's) */
    memset(S, 0, (size_t)(dv * dk) * sizeof(double));
    memset(z, 0, (size_t)dk * sizeof(double));
    for (int64_t t = len - 1; t >= 0; --t) {
      const int64_t row = start + t;
      const int64_t qk = (row * H + h) * dk, vb = (row * H + h) * dv;
      for (int64_t c = 0; c < dk; ++c) {
        qh[c] = orc_phi(orc_load(q, dtype, qk + c), phi);
        kh[c] = orc_phi(orc_load(k, dtype, qk + c), phi);
      }
      const double *u = U + (size_t)t * dv;
      for (int64_t r = 0; r < dv; ++r)
        for (int64_t c = 0; c < dk; ++c) S[r * dk + c] = g * S[r * dk + c] + u[r] * qh[c];
      for (int64_t c = 0; c < dk; ++c) z[c] = g * z[c] + E[t] * qh[c];
      for (int64_t c = 0; c < dk; ++c) {
        double acc = z[c];
        for (int64_t r = 0; r < dv; ++r) acc += S[r * dk + c] * orc_load(v, dtype, vb + r);
        dkk[qk + c] = acc * orc_dphi(orc_load(k, dtype, qk + c), phi);
      }
      for (int64_t r = 0; r < dv; ++r) {
        double acc = 0.0;
        for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * kh[c];
        dvv[vb + r] = acc;
      }
    }
    free(S); free(z); free(qh); free(kh); free(U); free(E); free(num);
  }
  return oom ? ORC_ERR_NOMEM : 0;
}

/*
 * Gradients of L = sum_t dout_t . o_t for the unnormalised recurrence with a
 * per-token decay (oracle_recurrent_gated): the adjoint of that definition,
 * with respect to q, k, v and the log decays g.  With alpha_t = exp(g_t):
 *   forward   S_t = alpha_t S_{t-1} + v_t kh_t^T,  dqh_t = S_t^T dout_t;
 *   backward  D_t = dout_t qh_t^T + alpha_{t+1} D_{t+1}   (D after the last token: 0),
 *             dv_t = D_t kh_t,  dkh_t = D_t^T v_t,
 *             dg_t = alpha_t <D_t, S_{t-1}>   (the Frobenius product; S_{-1} = 0),
 * then dq = dqh phi'(q), dk = dkh phi'(k).  Every state S_{t-1} is kept for
 * the dg step, so this is for test sizes (len * d_v * d_k doubles per task).
 *   g, dg  [B, T, H] double.  Other arguments as for oracle_backward.
 */
int oracle_backward_gated(const void *q, const void *k, const void *v, const void *dout, int dtype,
                          int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                          const double *g, const int32_t *cu_seqlens, int64_t n_seqs, int phi,
                          double *dq, double *dkk, double *dvv, double *dg, int nthreads) {
  int rc = orc_check(dtype, B, T, H, dk, dv, cu_seqlens, n_seqs, phi);
  if (rc) return rc;
  if (!g || !dg) return -10;
  if (nthreads <= 0) nthreads = oracle_max_threads();

  int oom = 0; /* set when a task could not allocate its buffers */
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
  for (int64_t task = 0; task < n_seqs * H; ++task) {
    const int64_t n = task / H, h = task % H;
    int64_t start, len;
    orc_seq(cu_seqlens, T, n, &start, &len);
    const size_t sz = (size_t)(dv * dk);
    double *prev = (double *)calloc((size_t)(len > 0 ? len : 1) * sz, sizeof(double));  /* S_{t-1}, every t */
    double *S = (double *)calloc(sz, sizeof(double));  /* S[r][c] */
    double *D = (double *)calloc(sz, sizeof(double));
    double *qh = (double *)malloc((size_t)dk * sizeof(double));
    double *kh = (double *)malloc((size_t)dk * sizeof(double));
    if (!prev || !S || !D || !qh || !kh) {
      free(prev); free(S); free(D); free(qh); free(kh);
#pragma omp atomic write
      oom = 1;
      continue;
    }
    /* forward in time */
    for (int64_t t = 0; t < len; ++t) {
      const int64_t row = start + t;
      const double a = exp(g[row * H + h]);
      const int64_t qk = (row * H + h) * dk, vb = (row * H + h) * dv;
      memcpy(prev + (size_t)t * sz, S, sz * sizeof(double));
      for (int64_t c = 0; c < dk; ++c) kh[c] = orc_phi(orc_load(k, dtype, qk + c), phi);
      for (int64_t r = 0; r < dv; ++r) {
        const double vr = orc_load(v, dtype, vb + r);
        for (int64_t c = 0; c < dk; ++c) S[r * dk + c] = a * S[r * dk + c] + vr * kh[c];
      }
      for (int64_t c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int64_t r = 0; r < dv; ++r) acc += S[r * dk + c] * orc_load(dout, dtype, vb + r);
        dq[qk + c] = acc * orc_dphi(orc_load(q, dtype, qk + c), phi);
      }
    }
    /* backward in time */
    double a_next = 0.0;  /* alpha_{t+1}; D is zero before the last token anyway */
    for (int64_t t = len - 1; t >= 0; --t) {
      const int64_t row = start + t;
      const double a = exp(g[row * H + h]);
      const int64_t qk = (row * H + h) * dk, vb = (row * H + h) * dv;
      for (int64_t c = 0; c < dk; ++c) {
        qh[c] = orc_phi(orc_load(q, dtype, qk + c), phi);
        kh[c] = orc_phi(orc_load(k, dtype, qk + c), phi);
      }
      for (int64_t r = 0; r < dv; ++r) {
        const double d = orc_load(dout, dtype, vb + r);
        for (int64_t c = 0; c < dk; ++c) D[r * dk + c] = a_next * D[r * dk + c] + d * qh[c];
      }
      for (int64_t c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int64_t r = 0; r < dv; ++r) acc += D[r * dk + c] * orc_load(v, dtype, vb + r);
        dkk[qk + c] = acc * orc_dphi(orc_load(k, dtype, qk + c), phi);
      }
      for (int64_t r = 0; r < dv; ++r) {
        double acc = 0.0;
        for (int64_t c = 0; c < dk; ++c) acc += D[r * dk + c] * kh[c];
        dvv[vb + r] = acc;
      }
      const double *P = prev + (size_t)t * sz;
      double inner = 0.0;
      for (size_t e = 0; e < sz; ++e) inner += D[e] * P[e];
      dg[row * H + h] = a * inner;
      a_next = a;
    }
    free(prev);
    free(S);
    free(D);
    free(qh);
    free(kh);
  }
  return oom ? ORC_ERR_NOMEM : 0;
}

/*
 * Adjoint of the normalised recurrence with the per-token decay alpha_t =
 * exp(g_t) ("1.6 长上下文与高效注意力", section 状态空间模型与 Mamba, with the
 * normaliser of section 线性注意力):
 *   S_t = alpha_t S_{t-1} + v_t kh_t^T,  z_t = alpha_t z_{t-1} + kh_t,
 *   num_t = S_t qh_t,  den_t = z_t . qh_t,  o_t = num_t / den_t.
 * With L = sum_t dout_t . o_t, u_t = dout_t / den_t reaches num_t and
 * e_t = -(dout_t . o_t) / den_t reaches den_t, so
 *   dqh_t = S_t^T u_t + e_t z_t,
 *   G_t = u_t qh_t^T + alpha_{t+1} G_{t+1},   gz_t = e_t qh_t + alpha_{t+1} gz_{t+1},
 *   dkh_t = G_t^T v_t + gz_t,   dv_t = G_t kh_t,
 *   dg_t = alpha_t (<G_t, S_{t-1}> + gz_t . z_{t-1})   (the loss sees g_t only
 *          through alpha_t's two products).
 * The forward sweep keeps every S_{t-1}, z_{t-1}, u_t and e_t of the task.
 */
int oracle_backward_gated_norm(const void *q, const void *k, const void *v, const void *dout, int dtype,
                               int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                               const double *g, const int32_t *cu_seqlens, int64_t n_seqs, int phi,
                               double *dq, double *dkk, double *dvv, double *dg, int nthreads) {
  int rc = orc_check(dtype, B, T, H, dk, dv, cu_seqlens, n_seqs, phi);
  if (rc) return rc;
  if (!g || !dg) return -10;
  if (nthreads <= 0) nthreads = oracle_max_threads();

  int oom = 0; /* set when a task could not allocate its buffers */
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
  for (int64_t task = 0; task < n_seqs * H; ++task) {
    const int64_t n = task / H, h = task % H;
    int64_t start, len;
    orc_seq(cu_seqlens, T, n, &start, &len);
    const size_t sz = (size_t)(dv * dk), L1 = (size_t)(len > 0 ? len : 1);
    double *prevS = (double *)calloc(L1 * sz, sizeof(double));        /* S_{t-1} */
    double *prevz = (double *)calloc(L1 * (size_t)dk, sizeof(double)); /* z_{t-1} */
    double *U = (double *)calloc(L1 * (size_t)dv, sizeof(double));     /* u_t */
    double *E = (double *)calloc(L1, sizeof(double));                  /* e_t */
    double *S = (double *)calloc(sz, sizeof(double));
    double *z = (double *)calloc((size_t)dk, sizeof(double));
    double *G = (double *)calloc(sz, sizeof(double));
    double *gz = (double *)calloc((size_t)dk, sizeof(double));
    double *qh = (double *)malloc((size_t)dk * sizeof(double));
    double *kh = (double *)malloc((size_t)dk * sizeof(double));
    double *num = (double *)malloc((size_t)dv * sizeof(double));
    if (!prevS || !prevz || !U || !E || !S || !z || !G || !gz || !qh || !kh || !num) {
      free(prevS); free(prevz); free(U); free(E); free(S); free(z); free(G); free(gz); free(qh); free(kh);
      free(num);
#pragma omp atomic write
      oom = 1;
      continue;
    }
    /* forward in time: the state, the normaliser, u_t, e_t and dq */
    for (int64_t t = 0; t < len; ++t) {
      const int64_t row = start + t;
      const double a = exp(g[row * H + h]);
      const int64_t qk = (row * H + h) * dk, vb = (row * H + h) * dv;
      memcpy(prevS + (size_t)t * sz, S, sz * sizeof(double));
      memcpy(prevz + (size_t)t * dk, z, (size_t)dk * sizeof(double));
      for (int64_t c = 0; c < dk; ++c) {
        qh[c] = orc_phi(orc_load(q, dtype, qk + c), phi);
        kh[c] = orc_phi(orc_load(k, dtype, qk + c), phi);
        z[c] = a * z[c] + kh[c];
      }
      double den = 0.0;
      for (int64_t c = 0; c < dk; ++c) den += z[c] * qh[c];
      double dot = 0.0;  /* dout . o */
      for (int64_t r = 0; r < dv; ++r) {
        const double vr = orc_load(v, dtype, vb + r);
        double acc = 0.0;
        for (int64_t c = 0; c < dk; ++c) {
          S[r * dk + c] = a * S[r * dk + c] + vr * kh[c];
          acc += S[r * dk + c] * qh[c];
        }
        num[r] = acc;
        dot += orc_load(dout, dtype, vb + r) * (acc / den);
      }
      double *u = U + (size_t)t * dv;
      for (int64_t r = 0; r < dv; ++r) u[r] = orc_load(dout, dtype, vb + r) / den;
      E[t] = -(dot / den);
      for (int64_t c = 0; c < dk; ++c) {
        double acc = z[c] * E[t];
        for (int64_t r = 0; r < dv; ++r) acc += S[r * dk + c] * u[r];
        dq[qk + c] = acc * orc_dphi(orc_load(q, dtype, qk + c), phi);
      }
    }
    /* backward in time: G, gz, dk, dv and dg */
    double a_next = 0.0;  /* alpha_{t+1}; G and gz are zero before the last token anyway */
    for (int64_t t = len - 1; t >= 0; --t) {
      const int64_t row = start + t;
      const double a = exp(g[row * H + h]);
      const int64_t qk = (row * H + h) * dk, vb = (row * H + h) * dv;
      const double *u = U + (size_t)t * dv;
      for (int64_t c = 0; c < dk; ++c) {
        qh[c] = orc_phi(orc_load(q, dtype, qk + c), phi);
        kh[c] = orc_phi(orc_load(k, dtype, qk + c), phi);
        gz[c] = a_next * gz[c] + E[t] * qh[c];
      }
      for (int64_t r = 0; r < dv; ++r)
        for (int64_t c = 0; c < dk; ++c) G[r * dk + c] = a_next * G[r * dk + c] + u[r] * qh[c];
      for (int64_t c = 0; c < dk; ++c) {
        double acc = gz[c];
        for (int64_t r = 0; r < dv; ++r) acc += G[r * dk + c] * orc_load(v, dtype, vb + r);
        dkk[qk + c] = acc * orc_dphi(orc_load(k, dtype, qk + c), phi);
      }
      for (int64_t r = 0; r < dv; ++r) {
        double acc = 0.0;
        for (int64_t c = 0; c < dk; ++c) acc += G[r * dk + c] * kh[c];
        dvv[vb + r] = acc;
      }
      const double *P = prevS + (size_t)t * sz, *Z = prevz + (size_t)t * dk;
      double inner = 0.0;
      for (size_t e = 0; e < sz; ++e) inner += G[e] * P[e];
      for (int64_t c = 0; c < dk; ++c) inner += gz[c] * Z[c];
      dg[row * H + h] = inner * a;
      a_next = a;
    }
    free(prevS); free(prevz); free(U); free(E); free(S); free(z); free(G); free(gz); free(qh); free(kh);
    free(num);
  }
  return oom ? ORC_ERR_NOMEM : 0;
}

/*
 * Output norm and gate ("使用 FlashAttention 内核实现最先进的线性注意力", the
 * paragraph on fused norm-gate operations: RMSNorm fused with a Swish gate;
 * the formula is the plain reading of those two names):
 *   y[r] = o[r] / sqrt(mean_r' o[r']^2 + eps) * w[r] * g[r] * sigmoid(g[r])
 * per (token, head) over the d_v values of o; w [d_v] is shared by all heads.
 *   o, y [rows, d_v] double (y may alias o); g [rows, d_v] (input dtype, see
 *   orc_load); rows = B * T * H.
 */
int oracle_norm_gate(const double *o, const void *g, int dtype, int64_t rows, int64_t dv, const double *w,
                     double eps, double *y, int nthreads) {
  if (rows < 0 || dv <= 0 || !o || !g || !w || !y) return -1;
  if (dtype != ORC_F32 && dtype != ORC_BF16 && dtype != ORC_F64) return -1;
  if (nthreads <= 0) nthreads = oracle_max_threads();

#pragma omp parallel for schedule(static) num_threads(nthreads)
  for (int64_t row = 0; row < rows; ++row) {
    const double *x = o + row * dv;
    double ss = 0.0;
    for (int64_t r = 0; r < dv; ++r) ss += x[r] * x[r];
    const double rstd = 1.0 / sqrt(ss / (double)dv + eps);
    for (int64_t r = 0; r < dv; ++r) {
      const double gv = orc_load(g, dtype, row * dv + r);
      y[row * dv + r] = x[r] * rstd * w[r] * gv / (1.0 + exp(-gv));
    }
  }
  return 0;
}

/*
 * Gated delta rule ("1.6 长上下文与高效注意力", section Gated delta rule, and its
 * listing): with the key normalised to unit length, kt = k_t / max(|k_t|, 1e-12),
 *     S_t = alpha_t S_{t-1} (I - beta_t kt kt^T) + beta_t v_t kt^T,   o_t = S_t q_t
 * per (sequence, head), S (d_v x d_k) starting at init (or zero), alpha_t =
 * exp(g_t).  q is used as given (no feature map), as in the listing.
 *   g, beta [B, T, H] double; init NULL or [n_seqs, H, d_k, d_v] (S^T);
 *   out [B, T, H, d_v]; final_state [n_seqs, H, d_k, d_v] (S^T) or NULL.
 */
int oracle_gated_delta(const void *q, const void *k, const void *v, int dtype, int64_t B, int64_t T,
                       int64_t H, int64_t dk, int64_t dv, const double *g, const double *beta,
                       const int32_t *cu_seqlens, int64_t n_seqs, const double *init, double *out,
                       double *final_state, int nthreads) {
  int rc = orc_check(dtype, B, T, H, dk, dv, cu_seqlens, n_seqs, ORC_PHI_IDENTITY);
  if (rc) return rc;
  if (!g || !beta) return -10;
  if (nthreads <= 0) nthreads = oracle_max_threads();

  int oom = 0; /* set when a task could not allocate its buffers */
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
  for (int64_t task = 0; task < n_seqs * H; ++task) {
    const int64_t n = task / H, h = task % H;
    int64_t start, len;
    orc_seq(cu_seqlens, T, n, &start, &len);
    double *S = (double *)calloc((size_t)(dv * dk), sizeof(double));  /* S[r][c] */
    double *kt = (double *)malloc((size_t)dk * sizeof(double));
    double *u = (double *)malloc((size_t)dv * sizeof(double));
    if (!S || !kt || !u) {
      free(S); free(kt); free(u);
#pragma omp atomic write
      oom = 1;
      continue;
    }
    if (init)
      for (int64_t c = 0; c < dk; ++c)
        for (int64_t r = 0; r < dv; ++r) S[r * dk + c] = init[task * dk * dv + c * dv + r];
    for (int64_t t = 0; t < len; ++t) {
      const int64_t row = start + t;
      const int64_t qk = (row * H + h) * dk, vb = (row * H + h) * dv;
      const double a = exp(g[row * H + h]), b = beta[row * H + h];
      double nrm = 0.0;
      for (int64_t c = 0; c < dk; ++c) {
        kt[c] = orc_load(k, dtype, qk + c);
        nrm += kt[c] * kt[c];
      }
      nrm = sqrt(nrm);
      if (nrm < 1e-12) nrm = 1e-12;
      for (int64_t c = 0; c < dk; ++c) kt[c] /= nrm;
      for (int64_t r = 0; r < dv; ++r) {  /* u = S kt */
        double acc = 0.0;
        for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * kt[c];
        u[r] = acc;
      }
      for (int64_t r = 0; r < dv; ++r) {
        const double vr = orc_load(v, dtype, vb + r);
        double o = 0.0;
        for (int64_t c = 0; c < dk; ++c) {
          S[r * dk + c] = a * (S[r * dk + c] - b * u[r] * kt[c]) + b * vr * kt[c];
          o += S[r * dk + c] * orc_load(q, dtype, qk + c);
        }
        out[vb + r] = o;
      }
    }
    if (final_state)
      for (int64_t c = 0; c < dk; ++c)
        for (int64_t r = 0; r < dv; ++r) final_state[task * dk * dv + c * dv + r] = S[r * dk + c];
    free(S);
    free(kt);
    free(u);
  }
  return oom ? ORC_ERR_NOMEM : 0;
}

/*
 * oracle_gated_delta_chunked -- the gated delta rule restated over chunks of
 * C tokens (float64).  It checks the chunk algebra that a chunked kernel uses
 * against the token-by-token definition; the pages give only the recurrence.
 * Inside a chunk that starts from state S_0, let b_i be the sum of g over the
 * chunk's tokens 0..i and write the update of token i as
 *   S_i = alpha_i S_{i-1} + u_i kt_i^T,   u_i = beta_i (v_i - alpha_i S_{i-1} kt_i),
 * so that S_i = e^{b_i} S_0 + sum_{j<=i} e^{b_i - b_j} u_j kt_j^T.  Putting that
 * S_{i-1} into u_i gives a unit lower-triangular system for the rows u_i:
 *   u_i + sum_{j<i} A_ij u_j = beta_i v_i - beta_i e^{b_i} S_0 kt_i,
 *   A_ij = beta_i e^{b_i - b_j} (kt_i . kt_j)   (j < i),
 * so with T = (I + A)^{-1}:  U = T diag(beta) V - T diag(beta e^b) Kt S_0^T.
 * Then o_i = e^{b_i} S_0 q_i + sum_{j<=i} e^{b_i - b_j} (q_i . kt_j) u_j, and
 * the next chunk starts from e^{b_last} S_0 + sum_j e^{b_last - b_j} u_j kt_j^T.
 * T is formed column by column by forward substitution.  Arguments as for
 * oracle_gated_delta, plus chunk >= 1.
 */
int oracle_gated_delta_chunked(const void *q, const void *k, const void *v, int dtype, int64_t B, int64_t T,
                               int64_t H, int64_t dk, int64_t dv, const double *g, const double *beta,
                               const int32_t *cu_seqlens, int64_t n_seqs, const double *init, int64_t chunk,
                               double *out, double *final_state, int nthreads) {
  int rc = orc_check(dtype, B, T, H, dk, dv, cu_seqlens, n_seqs, ORC_PHI_IDENTITY);
  if (rc) return rc;
  if (!g || !beta) return -10;
  if (chunk < 1) return -11;
  if (nthreads <= 0) nthreads = oracle_max_threads();
  const int64_t C = chunk;

  int oom = 0; /* set when a task could not allocate its buffers */
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
  for (int64_t task = 0; task < n_seqs * H; ++task) {
    const int64_t n = task / H, h = task % H;
    int64_t start, len;
    orc_seq(cu_seqlens, T, n, &start, &len);
    double *S = (double *)calloc((size_t)(dv * dk), sizeof(double)); /* S[r][c] */
    double *Kt = (double *)malloc((size_t)(C * dk) * sizeof(double));
    double *Q = (double *)malloc((size_t)(C * dk) * sizeof(double));
    double *V = (double *)malloc((size_t)(C * dv) * sizeof(double));
    double *A = (double *)malloc((size_t)(C * C) * sizeof(double));
    double *Ti = (double *)malloc((size_t)(C * C) * sizeof(double));
    double *U = (double *)malloc((size_t)(C * dv) * sizeof(double));
    double *X = (double *)malloc((size_t)(C * (dk > dv ? dk : dv)) * sizeof(double));
    double *bcum = (double *)malloc((size_t)C * sizeof(double));
    double *bet = (double *)malloc((size_t)C * sizeof(double));
    if (!S || !Kt || !Q || !V || !A || !Ti || !U || !X || !bcum || !bet) {
      free(S); free(Kt); free(Q); free(V); free(A); free(Ti); free(U); free(X); free(bcum); free(bet);
#pragma omp atomic write
      oom = 1;
      continue;
    }
    if (init)
      for (int64_t c = 0; c < dk; ++c)
        for (int64_t r = 0; r < dv; ++r) S[r * dk + c] = init[task * dk * dv + c * dv + r];
    for (int64_t t0 = 0; t0 < len; t0 += C) {
      const int64_t Cp = len - t0 < C ? len - t0 : C;
      double run = 0.0;
      for (int64_t i = 0; i < Cp; ++i) {
        const int64_t row = start + t0 + i;
        const int64_t qk = (row * H + h) * dk, vb = (row * H + h) * dv;
        run += g[row * H + h];
        bcum[i] = run;
        bet[i] = beta[row * H + h];
        double nrm = 0.0;
        for (int64_t c = 0; c < dk; ++c) {
          Kt[i * dk + c] = orc_load(k, dtype, qk + c);
          Q[i * dk + c] = orc_load(q, dtype, qk + c);
          nrm += Kt[i * dk + c] * Kt[i * dk + c];
        }
        nrm = sqrt(nrm);
        if (nrm < 1e-12) nrm = 1e-12;
        for (int64_t c = 0; c < dk; ++c) Kt[i * dk + c] /= nrm;
        for (int64_t r = 0; r < dv; ++r) V[i * dv + r] = orc_load(v, dtype, vb + r);
      }
      /* A, strictly lower */
      for (int64_t i = 0; i < Cp; ++i)
        for (int64_t j = 0; j < Cp; ++j) {
          double a = 0.0;
          if (j < i) {
            for (int64_t c = 0; c < dk; ++c) a += Kt[i * dk + c] * Kt[j * dk + c];
            a *= bet[i] * exp(bcum[i] - bcum[j]);
          }
          A[i * C + j] = a;
        }
      /* T = (I + A)^{-1}: column j solves (I + A) x = e_j */
      for (int64_t j = 0; j < Cp; ++j)
        for (int64_t i = 0; i < Cp; ++i) {
          double x = i == j ? 1.0 : 0.0;
          for (int64_t m = j; m < i; ++m) x -= A[i * C + m] * Ti[m * C + j];
          Ti[i * C + j] = i < j ? 0.0 : x;
        }
      /* U = T diag(beta) V - T diag(beta e^b) (Kt S_0^T) */
      for (int64_t i = 0; i < Cp; ++i) /* X = Kt S_0^T: X[i][r] = sum_c Kt[i][c] S[r][c] */
        for (int64_t r = 0; r < dv; ++r) {
          double acc = 0.0;
          for (int64_t c = 0; c < dk; ++c) acc += Kt[i * dk + c] * S[r * dk + c];
          X[i * dv + r] = acc;
        }
      for (int64_t i = 0; i < Cp; ++i)
        for (int64_t r = 0; r < dv; ++r) {
          double acc = 0.0;
          for (int64_t j = 0; j <= i; ++j)
            acc += Ti[i * C + j] * bet[j] * (V[j * dv + r] - exp(bcum[j]) * X[j * dv + r]);
          U[i * dv + r] = acc;
        }
      /* outputs */
      for (int64_t i = 0; i < Cp; ++i) {
        const int64_t row = start + t0 + i;
        const int64_t vb = (row * H + h) * dv;
        for (int64_t r = 0; r < dv; ++r) {
          double inter = 0.0;
          for (int64_t c = 0; c < dk; ++c) inter += S[r * dk + c] * Q[i * dk + c];
          double o = exp(bcum[i]) * inter;
          for (int64_t j = 0; j <= i; ++j) {
            double qk = 0.0;
            for (int64_t c = 0; c < dk; ++c) qk += Q[i * dk + c] * Kt[j * dk + c];
            o += exp(bcum[i] - bcum[j]) * qk * U[j * dv + r];
          }
          out[vb + r] = o;
        }
      }
      /* next chunk's start state */
      const double bl = bcum[Cp - 1];
      for (int64_t r = 0; r < dv; ++r)
        for (int64_t c = 0; c < dk; ++c) {
          double acc = exp(bl) * S[r * dk + c];
          for (int64_t j = 0; j < Cp; ++j) acc += exp(bl - bcum[j]) * U[j * dv + r] * Kt[j * dk + c];
          S[r * dk + c] = acc;
        }
    }
    if (final_state)
      for (int64_t c = 0; c < dk; ++c)
        for (int64_t r = 0; r < dv; ++r) final_state[task * dk * dv + c * dv + r] = S[r * dk + c];
    free(S);
    free(Kt);
    free(Q);
    free(V);
    free(A);
    free(Ti);
    free(U);
    free(X);
    free(bcum);
    free(bet);
  }
  return oom ? ORC_ERR_NOMEM : 0;
}
