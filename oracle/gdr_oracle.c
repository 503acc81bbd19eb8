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

/* Tokens [t_begin, t_end) of one (b, h) sequence.  S is d_v x d_k (column form),
 * row-major: S[c * dk + j].  o may be NULL (no readout).  On return u, z, w, vv
 * and e hold the last token's erase vector, erase key, decay, written value and
 * e = S_{t-1} u. */
static void run_sequence(int form, int b, int h, int B, int T, int H, int dk, int dv,
                         int t_begin, int t_end,
                         const double *q, const double *k, const double *v,
                         const double *log_w, const double *e1, const double *e2,
                         double *S, double *o, double *u, double *z, double *w,
                         double *vv, double *e) {
  (void)B;
  for (int t = t_begin; t < t_end; ++t) {
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
    for (int c = 0; o && c < dv; ++c) {
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
      run_sequence(form, b, h, B, T, H, dk, dv, 0, T, q, k, v, log_w, e1, e2, S, o,
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

/*
 * Reverse mode of the same loop (the adjoint of each statement of run_sequence,
 * taken in reverse token order).  With the loss L = <dO, o> + <dS_T, S_T>, the
 * adjoint dS of the state after token t collects dO_t q_t^T from the readout and
 * the propagated adjoint of the next token; then, for
 * S_t = S_{t-1} Diag(w) - e z^T + vv k^T with e = S_{t-1} u:
 *
 *     dq = S_t^T dO_t          dvv = dS k          dk  = dS^T vv
 *     de = -dS z               dz  = -dS^T e       dw  = diag(S_{t-1}^T dS)
 *     du = S_{t-1}^T de        dS_{t-1} = dS Diag(w) + de u^T
 *
 * and the form's mapping is differentiated back to its raw arguments:
 *   all forms: d log_w = dw (.) w                        (w = exp(log_w))
 *   general  : d e1 = du, d e2 = dz
 *   GDN-2    : u = w (.) b (.) k, z = k, vv = wg (.) v:
 *              dk += dz + du (.) w (.) b,  d b = du (.) w (.) k,  d log_w += du (.) u,
 *              dv = dvv (.) wg,  d wg = dvv (.) v
 *   RWKV-7   : u = c a, z = a:  d a = c du + dz,  d c = <du, a>
 *   GLA      : u = z = 0 (no erase gradients)
 *
 * States are recomputed from checkpoints taken every kSeg tokens (plain
 * recomputation; the arithmetic is the forward's own loop).
 *
 * Inputs as oracle_forward, plus dO [B][T][H][dv] and dS_T [B][H][dk][dv] (NULL =
 * 0).  Outputs: dq, dk, dlog_w [B][T][H][dk]; dv [B][T][H][dv]; de1 shaped like
 * e1 and de2 like e2 (NULL for a form without them); dS0 [B][H][dk][dv] (may be
 * NULL).  Returns 0, -1 on bad arguments, -2 when scratch memory ran out.
 */
enum { kSeg = 64 };

static void reverse_token(int form, int dk, int dv, size_t tk, size_t tv, size_t ts,
                          const double *q, const double *k, const double *v,
                          const double *e1, const double *e2, const double *dO,
                          const double *S_prev, const double *S_cur, const double *u,
                          const double *z, const double *w, const double *vv,
                          const double *e, double *dS, double *de, double *dvv,
                          double *dq, double *dk_, double *dv_, double *dlog_w,
                          double *de1, double *de2) {
  /* readout o_t = S_t q_t */
  for (int j = 0; j < dk; ++j) {
    double acc = 0.0;
    for (int c = 0; c < dv; ++c) acc += S_cur[(size_t)c * dk + j] * dO[tv + c];
    dq[tk + j] = acc;
  }
  for (int c = 0; c < dv; ++c)
    for (int j = 0; j < dk; ++j) dS[(size_t)c * dk + j] += dO[tv + c] * q[tk + j];
  /* S_t = S_{t-1} Diag(w) - e z^T + vv k^T */
  for (int c = 0; c < dv; ++c) {
    double a = 0.0, b = 0.0;
    for (int j = 0; j < dk; ++j) {
      a += dS[(size_t)c * dk + j] * k[tk + j];
      b += dS[(size_t)c * dk + j] * z[j];
    }
    dvv[c] = a;
    de[c] = -b;
  }
  for (int j = 0; j < dk; ++j) {
    double kw = 0.0, zz = 0.0, ww = 0.0, uu = 0.0;
    for (int c = 0; c < dv; ++c) {
      const double g = dS[(size_t)c * dk + j];
      kw += g * vv[c];
      zz -= g * e[c];
      ww += g * S_prev[(size_t)c * dk + j];
      uu += S_prev[(size_t)c * dk + j] * de[c];   /* e = S_{t-1} u */
    }
    double dkj = kw, dlw = ww * w[j];
    switch (form) {
      case OR_GENERAL:
        de1[tk + j] = uu;
        de2[tk + j] = zz;
        break;
      case OR_GDN2:
        dkj += zz + uu * w[j] * e1[tk + j];
        de1[tk + j] = uu * w[j] * k[tk + j];
        dlw += uu * u[j];
        break;
      case OR_RWKV7:
        de1[tk + j] = uu * e2[ts] + zz;
        break;
      default:
        break;
    }
    dk_[tk + j] = dkj;
    dlog_w[tk + j] = dlw;
  }
  if (form == OR_RWKV7) {
    double acc = 0.0;
    for (int j = 0; j < dk; ++j) {
      double uu = 0.0;
      for (int c = 0; c < dv; ++c) uu += S_prev[(size_t)c * dk + j] * de[c];
      acc += uu * e1[tk + j];
    }
    de2[ts] = acc;
  }
  for (int c = 0; c < dv; ++c) {
    if (form == OR_GDN2 && e2) {
      dv_[tv + c] = dvv[c] * e2[tv + c];
      de2[tv + c] = dvv[c] * v[tv + c];
    } else {
      dv_[tv + c] = dvv[c];
    }
  }
  /* adjoint of S_{t-1} */
  for (int c = 0; c < dv; ++c)
    for (int j = 0; j < dk; ++j)
      dS[(size_t)c * dk + j] = dS[(size_t)c * dk + j] * w[j] + de[c] * u[j];
}

int oracle_backward(int form, int B, int T, int H, int dk, int dv,
                    const double *q, const double *k, const double *v,
                    const double *log_w, const double *e1, const double *e2,
                    const double *S0, const double *dO, const double *dS_T,
                    double *dq, double *dk_, double *dv_, double *dlog_w,
                    double *de1, double *de2, double *dS0, int n_threads) {
  if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
  if (form < OR_GENERAL || form > OR_GLA) return -1;
  if (T > 0 && (!q || !k || !v || !log_w || !dO || !dq || !dk_ || !dv_ || !dlog_w)) return -1;
  if (T > 0 && form == OR_GENERAL && (!e1 || !e2 || !de1 || !de2)) return -1;
  if (T > 0 && form == OR_GDN2 && (!e1 || !de1 || (e2 && !de2))) return -1;
  if (T > 0 && form == OR_RWKV7 && (!e1 || !e2 || !de1 || !de2)) return -1;

  const int n_seq = B * H;
  const int n_ck = (T + kSeg - 1) / kSeg + 1;
  const size_t dd = (size_t)dk * dv;
  int failed = 0;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel
#endif
  {
    double *ck = (double *)malloc(sizeof(double) * dd * (size_t)n_ck);        /* checkpoints */
    double *st = (double *)malloc(sizeof(double) * dd * (size_t)(kSeg + 1));  /* segment states */
    double *par = (double *)malloc(sizeof(double) * (size_t)kSeg * (3 * dk + 2 * dv));
    double *dS = (double *)malloc(sizeof(double) * dd);
    double *scratch = (double *)malloc(sizeof(double) * (size_t)(3 * dk + 4 * dv));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
    for (int sq = 0; sq < n_seq; ++sq) {
      if (!ck || !st || !par || !dS || !scratch) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
        failed = 1;
        continue;
      }
      const int b = sq / H, h = sq % H;
      const size_t so = (size_t)sq * dd;
      double *u = scratch, *z = u + dk, *w = z + dk, *vv = w + dk, *e = vv + dv;
      double *de = e + dv, *dvv = de + dv;
      /* forward pass: checkpoints at t = 0, kSeg, 2 kSeg, ... */
      for (int c = 0; c < dv; ++c)
        for (int j = 0; j < dk; ++j)
          ck[(size_t)c * dk + j] = S0 ? S0[so + j * (size_t)dv + c] : 0.0;
      for (int g = 0; g + 1 < n_ck; ++g) {
        memcpy(ck + (size_t)(g + 1) * dd, ck + (size_t)g * dd, sizeof(double) * dd);
        const int t1 = (g + 1) * kSeg < T ? (g + 1) * kSeg : T;
        run_sequence(form, b, h, B, T, H, dk, dv, g * kSeg, t1, q, k, v, log_w, e1, e2,
                     ck + (size_t)(g + 1) * dd, NULL, u, z, w, vv, e);
      }
      /* reverse pass */
      for (int c = 0; c < dv; ++c)
        for (int j = 0; j < dk; ++j)
          dS[(size_t)c * dk + j] = dS_T ? dS_T[so + (size_t)j * dv + c] : 0.0;
      for (int g = n_ck - 2; g >= 0; --g) {
        const int t0 = g * kSeg, n = (t0 + kSeg < T ? t0 + kSeg : T) - t0;
        memcpy(st, ck + (size_t)g * dd, sizeof(double) * dd);
        for (int i = 0; i < n; ++i) {
          double *S = st + (size_t)(i + 1) * dd;
          double *pp = par + (size_t)i * (3 * dk + 2 * dv);
          memcpy(S, st + (size_t)i * dd, sizeof(double) * dd);
          run_sequence(form, b, h, B, T, H, dk, dv, t0 + i, t0 + i + 1, q, k, v, log_w, e1, e2,
                       S, NULL, pp, pp + dk, pp + 2 * dk, pp + 3 * dk, pp + 3 * dk + dv);
        }
        for (int i = n - 1; i >= 0; --i) {
          const int t = t0 + i;
          const size_t tk = (((size_t)b * T + t) * H + h) * (size_t)dk;
          const size_t tv = (((size_t)b * T + t) * H + h) * (size_t)dv;
          const size_t ts = ((size_t)b * T + t) * H + h;
          const double *pp = par + (size_t)i * (3 * dk + 2 * dv);
          reverse_token(form, dk, dv, tk, tv, ts, q, k, v, e1, e2, dO, st + (size_t)i * dd,
                        st + (size_t)(i + 1) * dd, pp, pp + dk, pp + 2 * dk, pp + 3 * dk,
                        pp + 3 * dk + dv, dS, de, dvv, dq, dk_, dv_, dlog_w, de1, de2);
        }
      }
      if (dS0)
        for (int c = 0; c < dv; ++c)
          for (int j = 0; j < dk; ++j)
            dS0[so + j * (size_t)dv + c] = dS[(size_t)c * dk + j];
    }
    free(ck);
    free(st);
    free(par);
    free(dS);
    free(scratch);
  }
  return failed ? -2 : 0;
}

/*
 * The Muir token mixer around the recurrence ("Muir ...", section 2.1 and section 4,
 * eqs. (8)-(9)): from pre-activations (after the projections and the depthwise causal
 * convolution) and gate logits,
 *
 *     q = l2norm(silu(q_pre)),  k = l2norm(silu(k_pre))  (per head, over d_k),  v = silu(v_pre)
 *     log alpha = -exp(a_log[h]) softplus(z_f),  b = 2 sigmoid(z_b),  w = sigmoid(z_w),
 *     gamma = gamma_stat (.) 2 sigmoid(z_q),     g = z_g
 *     GDN-2 recurrence with q^ = gamma (.) q, erase gate b, write gate w, decay alpha
 *     y_t = rmsnorm(o_t) (.) silu(g_t),  rmsnorm(o)_c = rho_c o_c / sqrt(mean_c o_c^2 + eps)
 *
 * l2norm(x) = x / max(||x||, 1e-12) (a zero vector stays zero).  gamma_stat [H][dk] and
 * rho [dv] may be NULL (all ones).  Inputs [B][T][H][.] as oracle_forward; a_log [H].
 * Outputs y [B][T][H][dv] and, if S_T != NULL, the final state.  Returns as oracle_forward.
 */
static double silu(double x) { return x / (1.0 + exp(-x)); }
static double sigm(double x) { return 1.0 / (1.0 + exp(-x)); }
static double softplus(double x) { return x > 30.0 ? x : log1p(exp(x)); }

int oracle_muir_forward(int B, int T, int H, int dk, int dv,
                        const double *q_pre, const double *k_pre, const double *v_pre,
                        const double *zf, const double *zb, const double *zw,
                        const double *zq, const double *zg, const double *a_log,
                        const double *gamma_stat, const double *rho, double eps,
                        const double *S0, double *y, double *S_T, int n_threads) {
  if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
  if (T > 0 && (!q_pre || !k_pre || !v_pre || !zf || !zb || !zw || !zq || !zg || !a_log || !y))
    return -1;
  const size_t nk = (size_t)B * T * H * dk, nv = (size_t)B * T * H * dv;
  double *q = (double *)calloc(nk ? nk : 1, sizeof(double));
  double *k = (double *)calloc(nk ? nk : 1, sizeof(double));
  double *v = (double *)calloc(nv ? nv : 1, sizeof(double));
  double *lw = (double *)calloc(nk ? nk : 1, sizeof(double));
  double *bg = (double *)calloc(nk ? nk : 1, sizeof(double));
  double *wg = (double *)calloc(nv ? nv : 1, sizeof(double));
  double *o = (double *)calloc(nv ? nv : 1, sizeof(double));
  int rc = -2;
  if (!q || !k || !v || !lw || !bg || !wg || !o) goto done;
  for (size_t tok = 0; tok < (size_t)B * T * H; ++tok) {
    const int h = (int)(tok % H);
    const size_t ok = tok * dk, ov = tok * dv;
    double nq = 0.0, nk2 = 0.0;
    for (int j = 0; j < dk; ++j) {
      q[ok + j] = silu(q_pre[ok + j]);
      k[ok + j] = silu(k_pre[ok + j]);
      nq += q[ok + j] * q[ok + j];
      nk2 += k[ok + j] * k[ok + j];
    }
    nq = sqrt(nq);
    nk2 = sqrt(nk2);
    if (nq < 1e-12) nq = 1e-12;
    if (nk2 < 1e-12) nk2 = 1e-12;
    const double rate = exp(a_log[h]);
    for (int j = 0; j < dk; ++j) {
      const double gam = (gamma_stat ? gamma_stat[(size_t)h * dk + j] : 1.0) * 2.0 * sigm(zq[ok + j]);
      q[ok + j] = gam * q[ok + j] / nq;
      k[ok + j] /= nk2;
      lw[ok + j] = -rate * softplus(zf[ok + j]);
      bg[ok + j] = 2.0 * sigm(zb[ok + j]);
    }
    for (int c = 0; c < dv; ++c) {
      v[ov + c] = silu(v_pre[ov + c]);
      wg[ov + c] = sigm(zw[ov + c]);
    }
  }
  rc = oracle_forward(OR_GDN2, B, T, H, dk, dv, q, k, v, lw, bg, wg, S0, o, S_T, n_threads);
  if (rc != 0) goto done;
  for (size_t tok = 0; tok < (size_t)B * T * H; ++tok) {
    const size_t ov = tok * dv;
    double ms = 0.0;
    for (int c = 0; c < dv; ++c) ms += o[ov + c] * o[ov + c];
    const double inv = 1.0 / sqrt(ms / dv + eps);
    for (int c = 0; c < dv; ++c)
      y[ov + c] = (rho ? rho[c] : 1.0) * o[ov + c] * inv * silu(zg[ov + c]);
  }
done:
  free(q);
  free(k);
  free(v);
  free(lw);
  free(bg);
  free(wg);
  free(o);
  return rc;
}

/*
 * xLSTM's mLSTM cell ("Exponential gates and matrix memory: xLSTM and RWKV-7", section
 * 13.4 and the solution to Exercise 13.6), one head at a time: matrix memory C (d_v x d_k),
 * normalizer n (d_k), scalar gates per (b, t, h): forget f_t = sigmoid(f~_t), input
 * i_t = exp(i~_t).
 *
 *   naive       C_t = f_t C_{t-1} + i_t v_t k_t^T,  n_t = f_t n_{t-1} + i_t k_t,
 *               h_t = C_t q_t / max(|n_t^T q_t|, 1)
 *   stabilized  m_t = max(log f_t + m_{t-1}, i~_t)   (m_0 = -inf for an empty memory)
 *               f'_t = exp(log f_t + m_{t-1} - m_t),  i'_t = exp(i~_t - m_t)
 *               C_t = f'_t C_{t-1} + i'_t v_t k_t^T,  n_t = f'_t n_{t-1} + i'_t k_t
 *               h_t = C_t q_t / max(|n_t^T q_t|, exp(-m_t))
 *
 * (the stabilized memory is the naive one times exp(-m_t); the readout floor scales with
 * it).  Inputs: q, k [B][T][H][dk], v [B][T][H][dv], f_pre, i_pre [B][T][H].  Initial
 * state: C0 [B][H][dk][dv] (storage layout, the transpose of C), n0 [B][H][dk], m0 [B][H];
 * all NULL for an empty memory (stabilized: m0 = -inf).  In the naive mode C0 and n0 are
 * the unscaled memory and m0 is ignored.  Outputs h [B][T][H][dv] and, when non-NULL, the
 * final C_T, n_T, m_T (the naive mode writes m_T = 0).  Returns as oracle_forward.
 */
static double log_sigmoid(double x) { return x >= 0.0 ? -log1p(exp(-x)) : x - log1p(exp(x)); }

int oracle_mlstm_forward(int B, int T, int H, int dk, int dv, int naive,
                         const double *q, const double *k, const double *v,
                         const double *f_pre, const double *i_pre,
                         const double *C0, const double *n0, const double *m0,
                         double *h, double *C_T, double *n_T, double *m_T, int n_threads) {
  if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
  if (T > 0 && (!q || !k || !v || !f_pre || !i_pre || !h)) return -1;
  const int n_seq = B * H;
  int failed = 0;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel
#endif
  {
    double *C = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *nv = (double *)malloc(sizeof(double) * (size_t)dk);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
    for (int sq = 0; sq < n_seq; ++sq) {
      if (!C || !nv) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
        failed = 1;
        continue;
      }
      const int b = sq / H, hh = sq % H;
      const size_t so = (size_t)sq * dk * dv;
      for (int c = 0; c < dv; ++c)
        for (int j = 0; j < dk; ++j) C[(size_t)c * dk + j] = C0 ? C0[so + (size_t)j * dv + c] : 0.0;
      for (int j = 0; j < dk; ++j) nv[j] = n0 ? n0[(size_t)sq * dk + j] : 0.0;
      double m = m0 ? m0[sq] : -INFINITY;
      for (int t = 0; t < T; ++t) {
        const size_t ts = ((size_t)b * T + t) * H + hh;
        const size_t tk = ts * (size_t)dk, tv = ts * (size_t)dv;
        const double lf = log_sigmoid(f_pre[ts]), li = i_pre[ts];
        double fs, is;
        if (naive) {
          fs = exp(lf);
          is = exp(li);
        } else {
          const double mn = fmax(lf + m, li);
          fs = exp(lf + m - mn);   /* 0 when m = -inf: the empty memory is discarded */
          is = exp(li - mn);
          m = mn;
        }
        for (int c = 0; c < dv; ++c)
          for (int j = 0; j < dk; ++j)
            C[(size_t)c * dk + j] = fs * C[(size_t)c * dk + j] + is * v[tv + c] * k[tk + j];
        double den = 0.0;
        for (int j = 0; j < dk; ++j) {
          nv[j] = fs * nv[j] + is * k[tk + j];
          den += nv[j] * q[tk + j];
        }
        const double floor_ = naive ? 1.0 : exp(-m);
        const double dd = fmax(fabs(den), floor_);
        for (int c = 0; c < dv; ++c) {
          double acc = 0.0;
          for (int j = 0; j < dk; ++j) acc += C[(size_t)c * dk + j] * q[tk + j];
          h[tv + c] = acc / dd;
        }
      }
      if (C_T)
        for (int c = 0; c < dv; ++c)
          for (int j = 0; j < dk; ++j) C_T[so + (size_t)j * dv + c] = C[(size_t)c * dk + j];
      if (n_T)
        for (int j = 0; j < dk; ++j) n_T[(size_t)sq * dk + j] = nv[j];
      if (m_T) m_T[sq] = naive ? 0.0 : m;
    }
    free(C);
    free(nv);
  }
  return failed ? -2 : 0;
}
