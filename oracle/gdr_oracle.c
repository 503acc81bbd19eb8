/*
 * gdr_oracle.c -- fp64 CPU oracle of the generalized delta-rule matrix memory.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark load this library.  It shares no code, header or constant with
 * the CUDA library (libgdr) and must never be reached from the product path.
 *
 * What it computes: the plain definition, one token at a time, in double
 * precision, for each (batch, head) independently.  Column form of the state
 * (S is d_v x d_k), as in "Exponential gates and matrix memory: xLSTM and RWKV-7",
 * section 13.1 (state retrieved by S q, transition acting on the right) and
 * section 13.3 (generalized delta rule):
 *
 *     e      = S u_t                                  (read along the erase vector)
 *     S      = S Diag(w_t) - e z_t^T + v_t k_t^T      (= S (Diag(w_t) - u_t z_t^T) + v_t k_t^T)
 *     o_t    = S q_t                                  (readout after the update)
 *
 * with w_t = exp(log_w_t).  The parameter mappings of the forms:
 *   general : u = e1, z = e2, write (v, k)
 *   GDN-2   : "Muir: Linear Attention with Sensitivity-Allocated Gating and
 *             Matched-Filter Readout", section 2.1 eq. (1):
 *             S_t = (I - k^T (b (.) k)) Diag(alpha) S_{t-1} + k^T (w (.) v)  (row form).
 *             Transposed to the column form: decay alpha = w, u = alpha (.) b (.) k,
 *             z = k, written value = wg (.) v (wg = e2, or 1 when e2 is absent).
 *   RWKV-7  : "Exponential gates ...", section 13.3: transition Diag(w) - c a a^T,
 *             write u b^T; here u = c a (c = e2, one scalar per token), z = a (= e1).
 *   GLA     : u = 0 ("Muir ...", section 2.1, channel-wise decay linear attention).
 *
 * Interface: all arrays are float64 and contiguous.  Token-major inputs
 * [B][T][H][d]; the state is passed and returned in the library's storage layout
 * [B][H][d_k][d_v] (key channel j, value channel c), i.e. the transpose of the
 * column-form S used inside.  A decode step is the T = 1 case.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_GENERAL = 0, OR_GDN2 = 1, OR_RWKV7 = 2, OR_GLA = 3 };

/* One (b, h) sequence.  S is d_v x d_k (column form), row-major: S[c * dk + j]. */
static void run_sequence(int form, int b, int h, int B, int T, int H, int dk, int dv,
                         const double *q, const double *k, const double *v,
                         const double *log_w, const double *e1, const double *e2,
                         double *S, double *o, double *u, double *z, double *w,
                         double *vv, double *e) {
  (void)B;
  for (int t = 0; t < T; ++t) {
    const size_t tk = (((size_t)b * T + t) * H + h) * (size_t)dk;  /* [b][t][h][.] over dk */
    const size_t tv = (((size_t)b * T + t) * H + h) * (size_t)dv;  /* [b][t][h][.] over dv */
    const size_t ts = ((size_t)b * T + t) * H + h;                 /* [b][t][h] scalar     */

    for (int j = 0; j < dk; ++j) w[j] = exp(log_w[tk + j]);
    for (int c = 0; c < dv; ++c) vv[c] = v[tv + c];

    switch (form) {
      case OR_GENERAL:
        for (int j = 0; j < dk; ++j) { u[j] = e1[tk + j]; z[j] = e2[tk + j]; }
        break;
      case OR_GDN2:
        /* erase acts on Diag(alpha) S_{t-1}: S_{t-1} Diag(alpha) - (S_{t-1}(alpha.b.k)) k^T */
        for (int j = 0; j < dk; ++j) { u[j] = w[j] * e1[tk + j] * k[tk + j]; z[j] = k[tk + j]; }
        if (e2) for (int c = 0; c < dv; ++c) vv[c] *= e2[tv + c];
        break;
      case OR_RWKV7: {
        const double cc = e2[ts];
        for (int j = 0; j < dk; ++j) { u[j] = cc * e1[tk + j]; z[j] = e1[tk + j]; }
        break;
      }
      default: /* OR_GLA */
        for (int j = 0; j < dk; ++j) { u[j] = 0.0; z[j] = 0.0; }
        break;
    }

    /* e = S u, from the state before this token */
    for (int c = 0; c < dv; ++c) {
      double acc = 0.0;
      for (int j = 0; j < dk; ++j) acc += S[(size_t)c * dk + j] * u[j];
      e[c] = acc;
    }
    /* S = S Diag(w) - e z^T + v k^T */
    for (int c = 0; c < dv; ++c)
      for (int j = 0; j < dk; ++j)
        S[(size_t)c * dk + j] = S[(size_t)c * dk + j] * w[j] - e[c] * z[j] + vv[c] * k[tk + j];
    /* o_t = S q_t */
    for (int c = 0; c < dv; ++c) {
      double acc = 0.0;
      for (int j = 0; j < dk; ++j) acc += S[(size_t)c * dk + j] * q[tk + j];
      o[tv + c] = acc;
    }
  }
}

/*
 * Runs the recurrence for all B*H sequences.  S0 may be NULL (zero state); S_T may
 * be NULL.  n_threads <= 0 lets OpenMP choose.  Returns 0 on success, -1 on bad
 * arguments, -2 when scratch memory could not be allocated.
 */
int oracle_forward(int form, int B, int T, int H, int dk, int dv,
                   const double *q, const double *k, const double *v,
                   const double *log_w, const double *e1, const double *e2,
                   const double *S0, double *o, double *S_T, int n_threads) {
  if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
  if (form < OR_GENERAL || form > OR_GLA) return -1;
  if (T > 0 && (!q || !k || !v || !log_w || !o)) return -1;
  if (T > 0 && form == OR_GENERAL && (!e1 || !e2)) return -1;
  if (T > 0 && form == OR_GDN2 && !e1) return -1;
  if (T > 0 && form == OR_RWKV7 && (!e1 || !e2)) return -1;

  const int n_seq = B * H;
  int failed = 0;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel
#endif
  {
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *scratch = (double *)malloc(sizeof(double) * (size_t)(3 * dk + 2 * dv));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
    for (int s = 0; s < n_seq; ++s) {
      if (!S || !scratch) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
        failed = 1;
        continue;
      }
      const int b = s / H, h = s % H;
      const size_t so = (size_t)s * dk * dv; /* [b][h][dk][dv] */
      for (int c = 0; c < dv; ++c)
        for (int j = 0; j < dk; ++j)
          S[(size_t)c * dk + j] = S0 ? S0[so + (size_t)j * dv + c] : 0.0;
      double *u = scratch, *z = u + dk, *w = z + dk, *vv = w + dk, *e = vv + dv;
      run_sequence(form, b, h, B, T, H, dk, dv, q, k, v, log_w, e1, e2, S, o,
                   u, z, w, vv, e);
      if (S_T)
        for (int c = 0; c < dv; ++c)
          for (int j = 0; j < dk; ++j)
            S_T[so + (size_t)j * dv + c] = S[(size_t)c * dk + j];
    }
    free(S);
    free(scratch);
  }
  return failed ? -2 : 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
