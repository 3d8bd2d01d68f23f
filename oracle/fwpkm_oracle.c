/*
 * fwpkm_oracle.c -- plain, slow, fp64 CPU oracle of the FwPKM chunked
 * read-then-write step.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the
 * CUDA path is compared against.  It shares no code, header, table or helper
 * with the CUDA path, and only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load it.  The product path never calls it.
 *
 * All arithmetic is double precision; fp32 / bf16 inputs are widened exactly
 * by the caller.  Loops are written in the order the method states them, with
 * no blocking or fusion, so each step can be checked against its source by eye.
 *
 * Sources (pages of the reference, by title and section):
 *   [GS-2]  gist.science "Fast-weight Product Key Memory", section 2
 *           "Methodology", Core Architecture + Key Technical Choices:
 *           two codebooks K1,K2 and top-k over N slots; keys and values updated
 *           by gradient descent on an MSE memorisation loss; negative-entropy
 *           addressing loss on the keys; gate g_t; update after each chunk;
 *           IDW score -log(eps + ||q - K||^2); averaging of the gradient of
 *           slots written several times in a chunk.
 *   [AF]    agifrontier.github.io tutorial: update theta' = theta - eta *
 *           grad L_MSE; query split into two sub-queries, Cartesian-product
 *           addressing; gate g_t.
 *   [SS-TOC] sciencestack.ai table of contents: "Reducing MSE losses to a
 *           scalar by summation", "Weighting gradient by row contribution",
 *           "Weighting MSE loss by token importance", "No gradient clipping",
 *           "Marginal entropy loss".
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *   - slot score s(i,j) = s1(i) + s2(j), slot = i*n + j;
 *   - ties ordered by (score desc, index asc);
 *   - weights = plain softmax over the k selected slot scores;
 *   - L_MSE = sum_t w_t ||yhat_t - v_t||^2 with token weight w_t = g_t
 *     unless a separate per-token weight omega is given (the lookahead
 *     pairing q_t -> v_{t+1} gives the last token of a call weight 0: it has
 *     no target there);
 *   - multi-head: one sub-key pair per head, one shared value table, head
 *     readouts averaged;
 *   - one memory shared by all B sequences; M = B*Tc*H token-heads per chunk;
 *   - marginal p_bar(i) = (1/M) * sum of the softmax weights landing on slot i;
 *     L_addr = -H(p_bar) = sum p_bar log p_bar, reaching the keys only;
 *   - value rows: gradient divided by C_i = sum over its pairs of w/H;
 *     sub-keys: raw summed gradient; no clipping.
 *
 * Parity pins (tests/test_oracle_pins.py): brute-force top-k over all N slots,
 * central finite differences of the loss, closed-form IDW weights and
 * single-access update, eta = 0 invariance, untouched rows unchanged,
 * causality, chaining, sum p_bar = 1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Scoring: IDW score of one query half against one sub-key table.  [GS-2]   */
/* s[i] = -log(eps + sum_d (q_d - K[i][d])^2), direct-difference form.       */
/* dist[i] (optional) receives the squared distance itself.                  */
/* (orc_half_scores_dot, below, is the dot-product score the IDW one is      */
/* chosen over.)                                                            */
/* ------------------------------------------------------------------------ */
void orc_half_scores(const double *q, const double *K, int n, int dh, double eps,
                     double *s, double *dist) {
  for (int i = 0; i < n; ++i) {
    double d = 0.0;
    for (int c = 0; c < dh; ++c) {
      double diff = q[c] - K[(int64_t)i * dh + c];
      d += diff * diff;
    }
    s[i] = -log(eps + d);
    if (dist) dist[i] = d;
  }
}

/* The other scoring the pages set the IDW score against [GS-2 Key Technical */
/* Choices]: the plain dot product s[i] = sum_d q_d K[i][d].                 */
void orc_half_scores_dot(const double *q, const double *K, int n, int dh, double *s) {
  for (int i = 0; i < n; ++i) {
    double d = 0.0;
    for (int c = 0; c < dh; ++c) d += q[c] * K[(int64_t)i * dh + c];
    s[i] = d;
  }
}

/* ------------------------------------------------------------------------ */
/* Top-k under the total order (score desc, index asc).                     */
/* ------------------------------------------------------------------------ */
typedef struct {
  double s;
  int64_t idx;
} scored;

static int cmp_scored(const void *a, const void *b) {
  const scored *x = (const scored *)a, *y = (const scored *)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->idx < y->idx) ? -1 : (x->idx > y->idx ? 1 : 0);
}

/* The k best of n scores; idx_out/s_out receive them best first. */
int orc_topk(const double *s, int n, int k, int64_t *idx_out, double *s_out) {
  if (k < 1 || k > n) return -1;
  scored *all = (scored *)malloc(sizeof(scored) * (size_t)n);
  if (!all) return -3;
  for (int i = 0; i < n; ++i) {
    all[i].s = s[i];
    all[i].idx = i;
  }
  qsort(all, (size_t)n, sizeof(scored), cmp_scored);
  for (int r = 0; r < k; ++r) {
    idx_out[r] = all[r].idx;
    if (s_out) s_out[r] = all[r].s;
  }
  free(all);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Product-key selection [GS-2, AF]: top-k of each half, then the top-k of   */
/* the k*k Cartesian candidates with s = s1(i) + s2(j), slot = i*n + j.      */
/* ia/jb (optional) receive the sub-key index of each half per selection.    */
/* ------------------------------------------------------------------------ */
int orc_pk_select(const double *s1, const double *s2, int n, int k,
                  int64_t *slot, double *score, int64_t *ia, int64_t *jb) {
  if (k < 1 || k > n) return -1;
  int64_t *top1 = (int64_t *)malloc(sizeof(int64_t) * (size_t)k);
  int64_t *top2 = (int64_t *)malloc(sizeof(int64_t) * (size_t)k);
  scored *cand = (scored *)malloc(sizeof(scored) * (size_t)k * (size_t)k);
  if (!top1 || !top2 || !cand) {
    free(top1);
    free(top2);
    free(cand);
    return -3;
  }
  orc_topk(s1, n, k, top1, NULL);
  orc_topk(s2, n, k, top2, NULL);
  for (int a = 0; a < k; ++a)
    for (int b = 0; b < k; ++b) {
      cand[a * k + b].s = s1[top1[a]] + s2[top2[b]];
      cand[a * k + b].idx = top1[a] * (int64_t)n + top2[b];
    }
  qsort(cand, (size_t)k * (size_t)k, sizeof(scored), cmp_scored);
  for (int r = 0; r < k; ++r) {
    slot[r] = cand[r].idx;
    if (score) score[r] = cand[r].s;
    if (ia) ia[r] = cand[r].idx / n;
    if (jb) jb[r] = cand[r].idx % n;
  }
  free(top1);
  free(top2);
  free(cand);
  return 0;
}

/* Brute force over all N = n*n slots (the definition the product-key search
 * must reproduce exactly). */
int orc_brute_select(const double *s1, const double *s2, int n, int k,
                     int64_t *slot, double *score) {
  int64_t N = (int64_t)n * n;
  if (k < 1 || k > N) return -1;
  scored *all = (scored *)malloc(sizeof(scored) * (size_t)N);
  if (!all) return -3;
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j) {
      all[(int64_t)i * n + j].s = s1[i] + s2[j];
      all[(int64_t)i * n + j].idx = (int64_t)i * n + j;
    }
  qsort(all, (size_t)N, sizeof(scored), cmp_scored);
  for (int r = 0; r < k; ++r) {
    slot[r] = all[r].idx;
    if (score) score[r] = all[r].s;
  }
  free(all);
  return 0;
}

/* Softmax over the k selected slot scores (max subtracted). */
void orc_softmax(const double *s, int k, double *w) {
  double mx = s[0];
  for (int r = 1; r < k; ++r)
    if (s[r] > mx) mx = s[r];
  double z = 0.0;
  for (int r = 0; r < k; ++r) {
    w[r] = exp(s[r] - mx);
    z += w[r];
  }
  for (int r = 0; r < k; ++r) w[r] /= z;
}

/* ------------------------------------------------------------------------ */
/* Shapes shared by the chunk routines.                                      */
/* ------------------------------------------------------------------------ */
/* Readings of two points the pages leave open, as options (section 2 of the
 * gist.science page: averaging of repeated-slot gradients; the pypi page's
 * multi-head variant).  Default 0: heads averaged, a value row's gradient
 * divided by its row contribution C_i = sum of w/H.                        */
enum {
  ORC_HEADS_SUM = 1, /* head readouts summed, not averaged                   */
  ORC_AGG_COUNT = 2, /* value-row gradient divided by the row's access count */
  ORC_AGG_SUM = 4,   /* value-row gradient not divided (plain sum)           */
  ORC_SCORE_DOT = 8, /* sub-key score q . K instead of -log(eps + |q - K|^2)  */
};

typedef struct {
  int64_t N;
  int n, dq, dh, dv, k, chunk, H;
  double eps;
  int variant; /* ORC_* bits */
} dims_t;

static int check_dims(int64_t N, int n, int dq, int dv, int topk, int chunk, int heads) {
  if (n < 1 || (int64_t)n * n != N) return -2;
  if (dq < 2 || dq % 2) return -2;
  if (dv < 1 || heads < 1 || chunk < 1) return -2;
  if (topk < 1 || topk > n) return -2;
  return 0;
}

/* Row pointers for token (b, t) of an array laid out [B][T][width]. */
static const double *row_of(const double *base, int T, int b, int t, int width) {
  return base + ((int64_t)b * T + t) * (int64_t)width;
}

/* ------------------------------------------------------------------------ */
/* One chunk: read with the current tables, then (optionally) apply the      */
/* chunk's gradient step.  Tokens t0 .. t0+Tc-1 of every sequence b.         */
/*                                                                          */
/* Token-head m = (b*Tc + tl)*H + h; pair p = m*k + r.                       */
/* omega [B][T] (optional): the MSE weight of each token; NULL = the gate.   */
/*                                                                          */
/* Optional outputs (NULL to skip):                                          */
/*   out      [B][T][dv]   g_t * yhat_t for the chunk's tokens               */
/*   sel_slot [B][T][H][k] selected slots (best first)                       */
/*   sel_w    [B][T][H][k] their softmax weights                              */
/*   gap      [B][T][H]    k-th minus (k+1)-th best slot score over all N     */
/*   dLdV     [N][dv]      raw dL/dV (dense; tiny shapes only)               */
/*   dLdK     [H][2][n][dh] raw dL/dK                                        */
/*   pbar     [N]          marginal slot usage of the chunk                   */
/*   loss     scalar       L_MSE + lambda * (-H(pbar))                       */
/*   n_touched scalar      number of distinct value rows written              */
/* ------------------------------------------------------------------------ */
static int orc_chunk(const dims_t *dm, double *K, double *V, int B, int T, int t0, int Tc,
                     const double *Q, const double *Vt, const double *gate,
                     const double *omega, double eta,
                     double lam, int apply, double *out, int64_t *sel_slot, double *sel_w,
                     double *gap, double *dLdV, double *dLdK, double *pbar_out,
                     double *loss, int64_t *n_touched, int64_t *rowmap) {
  const int n = dm->n, dh = dm->dh, dv = dm->dv, k = dm->k, H = dm->H, dq = dm->dq;
  const int64_t M = (int64_t)B * Tc * H;
  const int64_t P = M * k;
  const int kk = (k + 1 <= n) ? k + 1 : n; /* list length used for the gap */

  int64_t *slot = (int64_t *)malloc(sizeof(int64_t) * P);
  int64_t *ia = (int64_t *)malloc(sizeof(int64_t) * P);
  int64_t *jb = (int64_t *)malloc(sizeof(int64_t) * P);
  double *w = (double *)malloc(sizeof(double) * P);
  double *d1 = (double *)malloc(sizeof(double) * P); /* ||q1 - K1[ia]||^2 */
  double *d2 = (double *)malloc(sizeof(double) * P); /* ||q2 - K2[jb]||^2 */
  double *yhat = (double *)calloc((size_t)B * Tc * dv, sizeof(double));
  double *e = (double *)malloc(sizeof(double) * (size_t)B * Tc * dv);
  int64_t *ulist = (int64_t *)malloc(sizeof(int64_t) * P);
  double *GV = (double *)calloc((size_t)P * dv, sizeof(double));
  double *Csum = (double *)calloc((size_t)P, sizeof(double));
  double *Cnt = (double *)calloc((size_t)P, sizeof(double)); /* accesses per row */
  double *psum = (double *)calloc((size_t)P, sizeof(double));
  double *GK = (double *)calloc((size_t)H * 2 * n * dh, sizeof(double));
  unsigned char *ktouched = (unsigned char *)calloc((size_t)H * 2 * n, 1);
  if (!slot || !ia || !jb || !w || !d1 || !d2 || !yhat || !e || !ulist || !GV || !Csum ||
      !Cnt || !psum || !GK || !ktouched) {
    free(slot); free(ia); free(jb); free(w); free(d1); free(d2); free(yhat); free(e);
    free(ulist); free(GV); free(Csum); free(Cnt); free(psum); free(GK); free(ktouched);
    return -3;
  }
  /* head divisor of the readout and of its gradients: H (heads averaged) or
   * 1 (heads summed) */
  const double Hd = (dm->variant & ORC_HEADS_SUM) ? 1.0 : (double)H;
  int status = 0;
  int64_t U = 0; /* distinct value rows touched by the chunk */

  /* 1. Scores, product-key top-k and softmax per token-head.  [GS-2, AF]   */
#pragma omp parallel
  {
    double *s1 = (double *)malloc(sizeof(double) * n);
    double *s2 = (double *)malloc(sizeof(double) * n);
    double *dd1 = (double *)malloc(sizeof(double) * n);
    double *dd2 = (double *)malloc(sizeof(double) * n);
    double *sc = (double *)malloc(sizeof(double) * (kk > k ? kk : k));
    int64_t *sl = (int64_t *)malloc(sizeof(int64_t) * (kk > k ? kk : k));
    int64_t *a_ = (int64_t *)malloc(sizeof(int64_t) * k);
    int64_t *b_ = (int64_t *)malloc(sizeof(int64_t) * k);
    if (!s1 || !s2 || !dd1 || !dd2 || !sc || !sl || !a_ || !b_) {
#pragma omp atomic write
      status = -3;
    } else {
#pragma omp for schedule(static)
      for (int64_t m = 0; m < M; ++m) {
        int h = (int)(m % H);
        int64_t bt = m / H;
        int b = (int)(bt / Tc), tl = (int)(bt % Tc);
        const double *q = row_of(Q, T, b, t0 + tl, H * dq) + (int64_t)h * dq;
        const double *K1 = K + ((int64_t)h * 2 + 0) * n * dh;
        const double *K2 = K + ((int64_t)h * 2 + 1) * n * dh;
        orc_half_scores(q, K1, n, dh, dm->eps, s1, dd1);      /* first half of q  */
        orc_half_scores(q + dh, K2, n, dh, dm->eps, s2, dd2); /* second half of q */
        if (dm->variant & ORC_SCORE_DOT) { /* the dot-product score instead      */
          orc_half_scores_dot(q, K1, n, dh, s1);
          orc_half_scores_dot(q + dh, K2, n, dh, s2);
        }
        orc_pk_select(s1, s2, n, k, sl, sc, a_, b_);
        orc_softmax(sc, k, w + m * k);
        for (int r = 0; r < k; ++r) {
          slot[m * k + r] = sl[r];
          ia[m * k + r] = a_[r];
          jb[m * k + r] = b_[r];
          d1[m * k + r] = dd1[a_[r]];
          d2[m * k + r] = dd2[b_[r]];
        }
        if (sel_slot || sel_w) {
          int64_t o = (((int64_t)b * T + t0 + tl) * H + h) * k;
          for (int r = 0; r < k; ++r) {
            if (sel_slot) sel_slot[o + r] = sl[r];
            if (sel_w) sel_w[o + r] = w[m * k + r];
          }
        }
        if (gap) {
          double g_ = INFINITY;
          if (kk > k) {
            orc_pk_select(s1, s2, n, kk, sl, sc, NULL, NULL);
            g_ = sc[k - 1] - sc[k];
          }
          gap[((int64_t)b * T + t0 + tl) * H + h] = g_;
        }
      }
    }
    free(s1); free(s2); free(dd1); free(dd2); free(sc); free(sl); free(a_); free(b_);
  }
  if (status) goto done;

  /* 2. Readout [GS-2 "retrieved value"; heads averaged]: yhat_t = (1/H)     */
  /*    sum_h sum_r w V[slot] (Hd = 1: heads summed); out_t = g_t * yhat_t    */
  /*    [GS-2 gate, AF gate]                                                  */
  for (int b = 0; b < B; ++b)
    for (int tl = 0; tl < Tc; ++tl) {
      double *y = yhat + ((int64_t)b * Tc + tl) * dv;
      for (int h = 0; h < H; ++h) {
        int64_t m = ((int64_t)b * Tc + tl) * H + h;
        for (int r = 0; r < k; ++r) {
          const double *vr = V + slot[m * k + r] * dv;
          for (int c = 0; c < dv; ++c) y[c] += w[m * k + r] * vr[c];
        }
      }
      for (int c = 0; c < dv; ++c) y[c] /= Hd;
      double g = row_of(gate, T, b, t0 + tl, 1)[0];
      const double *vt = row_of(Vt, T, b, t0 + tl, dv);
      double *ev = e + ((int64_t)b * Tc + tl) * dv;
      for (int c = 0; c < dv; ++c) ev[c] = y[c] - vt[c];
      if (out) {
        double *o = out + ((int64_t)b * T + t0 + tl) * dv;
        for (int c = 0; c < dv; ++c) o[c] = g * y[c];
      }
    }

  /* 3. Value-row gradient and row contribution per touched slot, and the    */
  /*    marginal usage p_bar.  [GS-2 averaging; SS-TOC row contribution,    */
  /*    token importance, marginal entropy]                                 */
  for (int64_t m = 0; m < M; ++m) {
    int64_t bt = m / H;
    int b = (int)(bt / Tc), tl = (int)(bt % Tc);
    double om = row_of(omega ? omega : gate, T, b, t0 + tl, 1)[0]; /* token weight */
    const double *ev = e + bt * dv;
    for (int r = 0; r < k; ++r) {
      int64_t s_ = slot[m * k + r];
      if (rowmap[s_] < 0) {
        rowmap[s_] = U;
        ulist[U++] = s_;
      }
      int64_t u = rowmap[s_];
      double wr = w[m * k + r];
      for (int c = 0; c < dv; ++c) GV[u * dv + c] += (2.0 * om / Hd) * wr * ev[c];
      Csum[u] += wr / Hd;
      Cnt[u] += 1.0;
      psum[u] += wr;
    }
  }
  /* p_bar(i) = (1/M) sum of weights on slot i. */
  for (int64_t u = 0; u < U; ++u) psum[u] /= (double)M;

  /* 4. Gradient of L w.r.t. the selected slot scores, then the sub-keys.    */
  /*    dL/dw_r = (2 w_t/H) e.V[slot_r] + (lam/M)(log p_bar[slot_r] + 1)      */
  /*    dL/ds_r = w_r (gamma_r - sum_r' w_r' gamma_r')  (softmax Jacobian)    */
  /*    ds/dK_h,i = 2 (q_h - K_h,i) / (eps + d_h(i))   (IDW score)            */
  {
    double *gam = (double *)malloc(sizeof(double) * k);
    if (!gam) {
      status = -3;
      goto done;
    }
    for (int64_t m = 0; m < M; ++m) {
      int h = (int)(m % H);
      int64_t bt = m / H;
      int b = (int)(bt / Tc), tl = (int)(bt % Tc);
      double om = row_of(omega ? omega : gate, T, b, t0 + tl, 1)[0]; /* token weight */
      const double *ev = e + bt * dv;
      const double *q = row_of(Q, T, b, t0 + tl, H * dq) + (int64_t)h * dq;
      double wg = 0.0;
      for (int r = 0; r < k; ++r) {
        const double *vr = V + slot[m * k + r] * dv;
        double dot = 0.0;
        for (int c = 0; c < dv; ++c) dot += ev[c] * vr[c];
        gam[r] = (2.0 * om / Hd) * dot;
        if (lam != 0.0) gam[r] += (lam / (double)M) * (log(psum[rowmap[slot[m * k + r]]]) + 1.0);
        wg += w[m * k + r] * gam[r];
      }
      for (int r = 0; r < k; ++r) {
        double dLds = w[m * k + r] * (gam[r] - wg);
        int64_t i = ia[m * k + r], j = jb[m * k + r];
        double *G1 = GK + (((int64_t)h * 2 + 0) * n + i) * dh;
        double *G2 = GK + (((int64_t)h * 2 + 1) * n + j) * dh;
        const double *K1 = K + (((int64_t)h * 2 + 0) * n + i) * dh;
        const double *K2 = K + (((int64_t)h * 2 + 1) * n + j) * dh;
        if (dm->variant & ORC_SCORE_DOT) {
          /* ds/dK_h,i = q_h for the dot-product score */
          for (int c = 0; c < dh; ++c) {
            G1[c] += dLds * q[c];
            G2[c] += dLds * q[dh + c];
          }
        } else {
          double c1 = dLds * 2.0 / (dm->eps + d1[m * k + r]);
          double c2 = dLds * 2.0 / (dm->eps + d2[m * k + r]);
          for (int c = 0; c < dh; ++c) {
            G1[c] += c1 * (q[c] - K1[c]);
            G2[c] += c2 * (q[dh + c] - K2[c]);
          }
        }
        ktouched[((int64_t)h * 2 + 0) * n + i] = 1;
        ktouched[((int64_t)h * 2 + 1) * n + j] = 1;
      }
    }
    free(gam);
  }

  /* Optional raw-gradient / loss outputs (before any update). */
  if (dLdV)
    for (int64_t u = 0; u < U; ++u)
      for (int c = 0; c < dv; ++c) dLdV[ulist[u] * dv + c] = GV[u * dv + c];
  if (dLdK) memcpy(dLdK, GK, sizeof(double) * (size_t)H * 2 * n * dh);
  if (pbar_out)
    for (int64_t u = 0; u < U; ++u) pbar_out[ulist[u]] = psum[u];
  if (loss) {
    double L = 0.0;
    for (int b = 0; b < B; ++b)
      for (int tl = 0; tl < Tc; ++tl) {
        double om = row_of(omega ? omega : gate, T, b, t0 + tl, 1)[0]; /* token weight */
        const double *ev = e + ((int64_t)b * Tc + tl) * dv;
        double sq = 0.0;
        for (int c = 0; c < dv; ++c) sq += ev[c] * ev[c];
        L += om * sq;
      }
    double negH = 0.0;
    for (int64_t u = 0; u < U; ++u)
      if (psum[u] > 0.0) negH += psum[u] * log(psum[u]);
    *loss = L + lam * negH;
  }
  if (n_touched) *n_touched = U;

  /* 5. Update [AF theta' = theta - eta grad; GS-2 averaging; SS-TOC no     */
  /*    clipping]: V_i -= eta G_i / C_i on touched rows; K -= eta dL/dK.      */
  /*    The divisor of a value row: C_i (row contribution, default), its      */
  /*    access count (ORC_AGG_COUNT), or 1 (ORC_AGG_SUM).                     */
  if (apply) {
    for (int64_t u = 0; u < U; ++u) {
      double *vr = V + ulist[u] * dv;
      if (dm->variant & ORC_AGG_COUNT) Csum[u] = Cnt[u];
      if (dm->variant & ORC_AGG_SUM) Csum[u] = 1.0;
      for (int c = 0; c < dv; ++c) vr[c] -= eta * GV[u * dv + c] / Csum[u];
    }
    for (int64_t row = 0; row < (int64_t)H * 2 * n; ++row)
      if (ktouched[row])
        for (int c = 0; c < dh; ++c) K[row * dh + c] -= eta * GK[row * dh + c];
  }

done:
  for (int64_t u = 0; u < U; ++u) rowmap[ulist[u]] = -1;
  free(slot); free(ia); free(jb); free(w); free(d1); free(d2); free(yhat); free(e);
  free(ulist); free(GV); free(Csum); free(Cnt); free(psum); free(GK); free(ktouched);
  return status;
}

/* ------------------------------------------------------------------------ */
/* Public entry points (ctypes).                                            */
/* ------------------------------------------------------------------------ */

/* Whole call: chunks c = 0 .. ceil(T/chunk)-1 in order, each read with the
 * tables left by the previous chunk [GS-2 causality].  The last chunk may be
 * shorter.  K [H][2][n][dq/2] and V [N][dv] are updated in place; they are the
 * memory carried to the next call.  touched [n_chunks] (optional) receives the
 * number of distinct value rows written per chunk.  omega [B][T] (optional)
 * is the MSE weight of each token; NULL = the gate. */
int orc_step(int64_t N, int n, int dq, int dv, int topk, int chunk, int heads, double eps,
             int variant, double *K, double *V, int B, int T, const double *Q,
             const double *Vt, const double *gate, const double *omega, double eta,
             double lam, double *out, int64_t *sel_slot, double *sel_w, double *gap,
             int64_t *touched, int max_chunks) {
  int rc = check_dims(N, n, dq, dv, topk, chunk, heads);
  if (rc) return rc;
  if (B < 1 || T < 1) return -2;
  if ((variant & ORC_AGG_COUNT) && (variant & ORC_AGG_SUM)) return -1;
  dims_t dm = {N, n, dq, dq / 2, dv, topk, chunk, heads, eps, variant};
  int64_t *rowmap = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
  if (!rowmap) return -3;
  for (int64_t i = 0; i < N; ++i) rowmap[i] = -1;
  int n_chunks = (T + chunk - 1) / chunk;
  if (max_chunks > 0 && max_chunks < n_chunks) n_chunks = max_chunks;
  for (int c = 0; c < n_chunks && !rc; ++c) {
    int t0 = c * chunk;
    int Tc = (T - t0 < chunk) ? T - t0 : chunk;
    int64_t U = 0;
    rc = orc_chunk(&dm, K, V, B, T, t0, Tc, Q, Vt, gate, omega, eta, lam, 1, out, sel_slot,
                   sel_w, gap, NULL, NULL, NULL, NULL, &U, rowmap);
    if (touched) touched[c] = U;
  }
  free(rowmap);
  return rc;
}

/* One chunk (tokens t0 .. t0+Tc-1) without any update: raw gradients, the
 * loss and p_bar for finite-difference and invariant checks. */
int orc_chunk_grads(int64_t N, int n, int dq, int dv, int topk, int chunk, int heads,
                    double eps, int variant, const double *K, const double *V, int B, int T,
                    int t0, int Tc, const double *Q, const double *Vt, const double *gate,
                    const double *omega, double lam, double *dLdV, double *dLdK, double *pbar,
                    double *loss, int64_t *sel_slot, double *sel_w) {
  int rc = check_dims(N, n, dq, dv, topk, chunk, heads);
  if (rc) return rc;
  dims_t dm = {N, n, dq, dq / 2, dv, topk, chunk, heads, eps, variant};
  int64_t *rowmap = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
  if (!rowmap) return -3;
  for (int64_t i = 0; i < N; ++i) rowmap[i] = -1;
  rc = orc_chunk(&dm, (double *)K, (double *)V, B, T, t0, Tc, Q, Vt, gate, omega, 0.0, lam, 0,
                 NULL, sel_slot, sel_w, NULL, dLdV, dLdK, pbar, loss, NULL, rowmap);
  free(rowmap);
  return rc;
}

/* The chunk loss written straight from its definition for a FROZEN selection
 * slots [B][Tc][H][k] (as returned by orc_chunk_grads for the same chunk):
 *   s_r = -log(eps + ||q1 - K1[i_r]||^2) - log(eps + ||q2 - K2[j_r]||^2)
 *   w   = softmax(s);  yhat_t = (1/H) sum_h sum_r w_r V[slot_r]  (summed heads:
 *         no 1/H)
 *   L   = sum_t w_t ||yhat_t - v_t||^2 + lam * sum_i p_bar_i log p_bar_i
 *         (w_t = omega_t if omega is given, else the gate g_t)
 * Used only for finite differences of the analytic gradients. */
double orc_chunk_loss(int64_t N, int n, int dq, int dv, int topk, int heads, double eps,
                      int variant, const double *K, const double *V, int B, int T, int t0,
                      int Tc, const double *Q, const double *Vt, const double *gate,
                      const double *omega, double lam, const int64_t *slots) {
  const int dh = dq / 2, k = topk, H = heads;
  const double Hd = (variant & ORC_HEADS_SUM) ? 1.0 : (double)H;
  const int64_t M = (int64_t)B * Tc * H;
  double *pb = (double *)calloc((size_t)N, sizeof(double));
  double *y = (double *)malloc(sizeof(double) * dv);
  double *s = (double *)malloc(sizeof(double) * k);
  double *w = (double *)malloc(sizeof(double) * k);
  double L = 0.0;
  for (int b = 0; b < B; ++b)
    for (int tl = 0; tl < Tc; ++tl) {
      for (int c = 0; c < dv; ++c) y[c] = 0.0;
      for (int h = 0; h < H; ++h) {
        const double *q = row_of(Q, T, b, t0 + tl, H * dq) + (int64_t)h * dq;
        const int64_t *sl = slots + (((int64_t)b * Tc + tl) * H + h) * k;
        for (int r = 0; r < k; ++r) {
          int64_t i = sl[r] / n, j = sl[r] % n;
          const double *K1 = K + (((int64_t)h * 2 + 0) * n + i) * dh;
          const double *K2 = K + (((int64_t)h * 2 + 1) * n + j) * dh;
          double da = 0.0, db = 0.0;
          for (int c = 0; c < dh; ++c) {
            da += (q[c] - K1[c]) * (q[c] - K1[c]);
            db += (q[dh + c] - K2[c]) * (q[dh + c] - K2[c]);
          }
          s[r] = -log(eps + da) - log(eps + db);
          if (variant & ORC_SCORE_DOT) {
            double pa = 0.0, pb = 0.0;
            for (int c = 0; c < dh; ++c) {
              pa += q[c] * K1[c];
              pb += q[dh + c] * K2[c];
            }
            s[r] = pa + pb;
          }
        }
        orc_softmax(s, k, w);
        for (int r = 0; r < k; ++r) {
          for (int c = 0; c < dv; ++c) y[c] += w[r] * V[sl[r] * dv + c];
          pb[sl[r]] += w[r] / (double)M;
        }
      }
      double wt = row_of(omega ? omega : gate, T, b, t0 + tl, 1)[0];
      const double *vt = row_of(Vt, T, b, t0 + tl, dv);
      double sq = 0.0;
      for (int c = 0; c < dv; ++c) {
        double ec = y[c] / Hd - vt[c];
        sq += ec * ec;
      }
      L += wt * sq;
    }
  double negH = 0.0;
  for (int64_t i = 0; i < N; ++i)
    if (pb[i] > 0.0) negH += pb[i] * log(pb[i]);
  free(pb);
  free(y);
  free(s);
  free(w);
  return L + lam * negH;
}
