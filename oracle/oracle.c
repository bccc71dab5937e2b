/*
 * oracle.c — plain, slow, obviously-correct CPU reference for the
 * pair-biased triangle attention block over a protein pair representation.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The GPU product path
 * never calls it, links it or shares code with it.
 *
 * Everything is computed in IEEE double precision (fp64), with every
 * softmax row materialised in full (no blocking, no online rescaling,
 * except in oracle_attend_blockwise, which exists only so the tests can
 * check the full-softmax evaluation against a different evaluation order).
 *
 * What is computed, and where it comes from:
 *
 *  - The pair representation Z has shape (N, N, c_z), c_z typically 128,
 *    one c_z-vector per residue pair ("token"); it is the dominant cost of
 *    structure models (LightNobel article "蛋白质结构预测模型的量化优化与硬件
 *    加速", §1.1; per-token treatment of the Ns x Ns vectors, §2.2.1).
 *  - LayerNorm is applied per pair before the linear projections (same
 *    article, §2.2.3 group B "after LayerNorm, before the linear layer", and
 *    §3.1 "LayerNorm co-optimised"): mean and biased variance over the c_z
 *    channels, x = (z - mu) / sqrt(var + eps) * gamma + beta.
 *  - Triangular attention is named by the same article (§3.1) without
 *    equations; the block follows the standard starting-node / ending-node
 *    pair-biased triangle attention:
 *      q, k, v = Wq x, Wk x, Wv x   (H heads of width d each)
 *      g       = sigmoid(Wg x + bg) (per channel of H*d)
 *      beta_h  = Wb x               (one logit bias per head)
 *    starting node, for row i, query column j, head h:
 *      s_k  = q_ij . k_ik / sqrt(d) + beta_h(j,k)      over unmasked keys k
 *      o_ij = sum_k softmax_k(s)_k v_ik
 *    ending node, for column j, query row i, head h:
 *      s_k  = q_ij . k_kj / sqrt(d) + beta_h(k,i)      over unmasked keys k
 *      o_ij = sum_k softmax_k(s)_k v_kj
 *    out_ij = z_ij + Wo (g_ij * o_ij) + bo   (residual path: LightNobel
 *    §2.2.3 group A / §3.1).
 *  - The mask is a per-residue key mask: a masked residue k contributes
 *    probability exactly 0 as a key; its own rows and columns are still
 *    computed.  If every key is masked, o = 0 and out = z.
 *  - Training needs the gradients of the attention core with respect to q,
 *    k, v and the logit bias (BioNeMo context-parallelism page, the training
 *    setting its context gaps refer to); oracle_attend_bwd writes them out by
 *    the chain rule through each materialised softmax row.
 *  - Scores are computed on the fly per row; an N x N x H score tensor is
 *    never stored (Design-CP technical summary, §Metodología 1, 2D grid
 *    sharding with ring attention: scores computed without materialising the
 *    full I x I matrix).  The oracle materialises one softmax row at a time.
 *
 * The starting-node and ending-node loops below are written separately, each
 * straight from its own formula; neither is derived from the other through a
 * transpose, so the tests can use the identity ending(Z) = T(start(T(Z)))
 * as an independent check.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Element type of the Z array handed to the oracle.  bf16 and fp32 values
 * are converted to double exactly. */
enum { ORACLE_Z_F64 = 0, ORACLE_Z_F32 = 1, ORACLE_Z_BF16 = 2 };

typedef struct {
  int N, c_z, H, d;
  double eps;
  int z_dtype;                 /* ORACLE_Z_* */
  const void *Z;               /* [N][N][c_z] */
  const unsigned char *mask;   /* [N], 1 = valid key; NULL = all valid */
  const double *gamma, *beta;  /* [c_z] */
  const double *Wq, *Wk, *Wv, *Wg; /* [H*d][c_z] (out x in) */
  const double *bg;            /* [H*d] or NULL */
  const double *Wb;            /* [H][c_z] */
  const double *Wo;            /* [c_z][H*d] */
  const double *bo;            /* [c_z] or NULL */
} oracle_params;

int oracle_version(void) { return 1; }

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Read channel c of pair (a, b) of Z as a double. */
static double z_at(const oracle_params *p, long a, long b, int c) {
  long idx = (a * (long)p->N + b) * (long)p->c_z + c;
  switch (p->z_dtype) {
    case ORACLE_Z_F32:
      return (double)((const float *)p->Z)[idx];
    case ORACLE_Z_BF16: {
      uint32_t bits = (uint32_t)((const uint16_t *)p->Z)[idx] << 16;
      float f;
      memcpy(&f, &bits, sizeof f);
      return (double)f;
    }
    default:
      return ((const double *)p->Z)[idx];
  }
}

/* LayerNorm of one c_z-vector: mean, biased variance, affine. */
static void layer_norm_vec(const double *z, int c_z, double eps,
                           const double *gamma, const double *beta,
                           double *x) {
  double mu = 0.0, var = 0.0;
  for (int c = 0; c < c_z; ++c) mu += z[c];
  mu /= c_z;
  for (int c = 0; c < c_z; ++c) var += (z[c] - mu) * (z[c] - mu);
  var /= c_z;
  double inv = 1.0 / sqrt(var + eps);
  for (int c = 0; c < c_z; ++c) x[c] = (z[c] - mu) * inv * gamma[c] + beta[c];
}

/* y[o] = sum_c W[o][c] x[c] (+ b[o]) for o < n_out. */
static void linear(const double *W, const double *b, const double *x,
                   int n_out, int n_in, double *y) {
  for (int o = 0; o < n_out; ++o) {
    double acc = b ? b[o] : 0.0;
    const double *w = W + (long)o * n_in;
    for (int c = 0; c < n_in; ++c) acc += w[c] * x[c];
    y[o] = acc;
  }
}

static double sigmoid(double t) { return 1.0 / (1.0 + exp(-t)); }

/* Per-pair features of pair (a, b) of Z: q, k, v, g [H*d] and bias [H]. */
typedef struct { double *q, *k, *v, *g, *b; } pair_feat;

static void pair_features(const oracle_params *p, long a, long b,
                          double *zbuf, double *xbuf, pair_feat f) {
  int HD = p->H * p->d;
  for (int c = 0; c < p->c_z; ++c) zbuf[c] = z_at(p, a, b, c);
  layer_norm_vec(zbuf, p->c_z, p->eps, p->gamma, p->beta, xbuf);
  if (f.q) linear(p->Wq, NULL, xbuf, HD, p->c_z, f.q);
  if (f.k) linear(p->Wk, NULL, xbuf, HD, p->c_z, f.k);
  if (f.v) linear(p->Wv, NULL, xbuf, HD, p->c_z, f.v);
  if (f.g) {
    linear(p->Wg, p->bg, xbuf, HD, p->c_z, f.g);
    for (int o = 0; o < HD; ++o) f.g[o] = sigmoid(f.g[o]);
  }
  if (f.b) linear(p->Wb, NULL, xbuf, p->H, p->c_z, f.b);
}

/* ---------------------------------------------------------------------- */
/* Stage functions exported for the tests.                                 */

/* LayerNorm of n independent c_z-vectors. */
int oracle_layer_norm(const double *z, long n, int c_z, double eps,
                      const double *gamma, const double *beta, double *x) {
  if (!z || !x || n < 0 || c_z <= 0) return -1;
#pragma omp parallel for schedule(static)
  for (long t = 0; t < n; ++t)
    layer_norm_vec(z + t * c_z, c_z, eps, gamma, beta, x + t * c_z);
  return 0;
}

/* Features of every pair of Z: q, k, v, g as [N][N][H*d], bias as [H][N][N]
 * (the unmasked logit bias beta_h(a, b) of pair (a, b)).  Any output may be
 * NULL. */
int oracle_pair_features(const oracle_params *p, double *q, double *k,
                         double *v, double *g, double *bias) {
  if (!p || p->N <= 0) return -1;
  long N = p->N;
  int HD = p->H * p->d;
#pragma omp parallel
  {
    double *zb = malloc(sizeof(double) * p->c_z);
    double *xb = malloc(sizeof(double) * p->c_z);
    double *bb = malloc(sizeof(double) * p->H);
#pragma omp for schedule(static)
    for (long ab = 0; ab < N * N; ++ab) {
      long a = ab / N, b = ab % N;
      pair_feat f = {q ? q + ab * HD : NULL, k ? k + ab * HD : NULL,
                     v ? v + ab * HD : NULL, g ? g + ab * HD : NULL,
                     bias ? bb : NULL};
      pair_features(p, a, b, zb, xb, f);
      if (bias)
        for (int h = 0; h < p->H; ++h) bias[((long)h * N + a) * N + b] = bb[h];
    }
    free(zb);
    free(xb);
    free(bb);
  }
  return 0;
}

/* Pair-biased attention with the full softmax row materialised.
 *   q: [Nq][H][d], k, v: [Nk][H][d], bias: [H][Nq][Nk] (added to the scaled
 *   dot product), mask: [Nk] or NULL.
 *   o: [Nq][H][d]; probs (optional): [H][Nq][Nk].
 * Rows with every key masked give o = 0 and an all-zero probability row. */
int oracle_attend(const double *q, const double *k, const double *v,
                  const double *bias, const unsigned char *mask, int Nq,
                  int Nk, int H, int d, double *o, double *probs) {
  if (!q || !k || !v || !bias || !o || Nq < 0 || Nk < 0) return -1;
  double scale = 1.0 / sqrt((double)d);
#pragma omp parallel
  {
    double *s = malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
#pragma omp for collapse(2) schedule(static)
    for (int h = 0; h < H; ++h)
      for (int j = 0; j < Nq; ++j) {
        const double *qj = q + ((long)j * H + h) * d;
        double mx = -INFINITY;
        int any = 0;
        for (int kk = 0; kk < Nk; ++kk) {
          if (mask && !mask[kk]) continue;
          const double *kv = k + ((long)kk * H + h) * d;
          double dot = 0.0;
          for (int c = 0; c < d; ++c) dot += qj[c] * kv[c];
          s[kk] = dot * scale + bias[((long)h * Nq + j) * Nk + kk];
          if (!any || s[kk] > mx) mx = s[kk];
          any = 1;
        }
        double denom = 0.0;
        for (int kk = 0; kk < Nk; ++kk) {
          if (mask && !mask[kk]) { s[kk] = 0.0; continue; }
          s[kk] = exp(s[kk] - mx);
          denom += s[kk];
        }
        double *oj = o + ((long)j * H + h) * d;
        for (int c = 0; c < d; ++c) oj[c] = 0.0;
        for (int kk = 0; kk < Nk; ++kk) {
          double pk = any ? s[kk] / denom : 0.0;
          if (probs) probs[((long)h * Nq + j) * Nk + kk] = pk;
          if (pk == 0.0) continue;
          const double *vv = v + ((long)kk * H + h) * d;
          for (int c = 0; c < d; ++c) oj[c] += pk * vv[c];
        }
      }
    free(s);
  }
  return 0;
}

/* Same attention evaluated block by block over the keys with a running
 * maximum, running denominator and rescaled accumulator (the online-softmax
 * recurrence), block size `block`.  Only used to cross-check oracle_attend. */
int oracle_attend_blockwise(const double *q, const double *k, const double *v,
                            const double *bias, const unsigned char *mask,
                            int Nq, int Nk, int H, int d, int block,
                            double *o) {
  if (!q || !k || !v || !bias || !o || block <= 0) return -1;
  double scale = 1.0 / sqrt((double)d);
  for (int h = 0; h < H; ++h)
    for (int j = 0; j < Nq; ++j) {
      const double *qj = q + ((long)j * H + h) * d;
      double m = -INFINITY, l = 0.0;
      double *acc = calloc(d, sizeof(double));
      double *sb = malloc(sizeof(double) * block);
      for (int k0 = 0; k0 < Nk; k0 += block) {
        int k1 = k0 + block < Nk ? k0 + block : Nk;
        double bm = -INFINITY;
        for (int kk = k0; kk < k1; ++kk) {
          if (mask && !mask[kk]) { sb[kk - k0] = -INFINITY; continue; }
          const double *kv = k + ((long)kk * H + h) * d;
          double dot = 0.0;
          for (int c = 0; c < d; ++c) dot += qj[c] * kv[c];
          sb[kk - k0] = dot * scale + bias[((long)h * Nq + j) * Nk + kk];
          if (sb[kk - k0] > bm) bm = sb[kk - k0];
        }
        if (bm == -INFINITY) continue; /* every key of this block masked */
        double mn = m > bm ? m : bm;
        double corr = (m == -INFINITY) ? 0.0 : exp(m - mn);
        l *= corr;
        for (int c = 0; c < d; ++c) acc[c] *= corr;
        for (int kk = k0; kk < k1; ++kk) {
          if (sb[kk - k0] == -INFINITY) continue;
          double pk = exp(sb[kk - k0] - mn);
          l += pk;
          const double *vv = v + ((long)kk * H + h) * d;
          for (int c = 0; c < d; ++c) acc[c] += pk * vv[c];
        }
        m = mn;
      }
      double *oj = o + ((long)j * H + h) * d;
      for (int c = 0; c < d; ++c) oj[c] = l > 0.0 ? acc[c] / l : 0.0;
      free(acc);
      free(sb);
    }
  return 0;
}

/* ---------------------------------------------------------------------- */
/* Gradients of the attention core (the backward pass).                    */

/* Gradients of oracle_attend with respect to q, k, v and the bias, given the
 * gradient `dout` of a scalar loss with respect to its output o.  Same shapes
 * as oracle_attend: q, dq: [Nq][H][d]; k, v, dk, dv: [Nk][H][d]; bias, dbias:
 * [H][Nq][Nk]; dout: [Nq][H][d].  Every output array is overwritten.
 *
 * Plain chain rule through one softmax row (s_k the scaled dot product plus
 * bias, p = softmax over the unmasked keys, o = sum_k p_k v_k):
 *   dv_k  += p_k dout                       (o is linear in v)
 *   dp_k   = dout . v_k                     (d loss / d p_k)
 *   ds_k   = p_k (dp_k - sum_m p_m dp_m)    (Jacobian of the softmax,
 *                                            diag(p) - p p^T, applied to dp)
 *   dbias_k = ds_k,  dq += ds_k k_k / sqrt(d),  dk_k += ds_k q / sqrt(d)
 * Masked keys have p_k = 0, hence ds_k = 0 and no contribution anywhere; a
 * query whose every key is masked has o = 0 independent of its inputs and
 * gets all-zero gradients. */
int oracle_attend_bwd(const double *q, const double *k, const double *v,
                      const double *bias, const unsigned char *mask,
                      const double *dout, int Nq, int Nk, int H, int d,
                      double *dq, double *dk, double *dv, double *dbias) {
  if (!q || !k || !v || !bias || !dout || !dq || !dk || !dv || !dbias || Nq < 0 || Nk < 0)
    return -1;
  const double scale = 1.0 / sqrt((double)d);
  memset(dq, 0, sizeof(double) * (size_t)Nq * H * d);
  memset(dk, 0, sizeof(double) * (size_t)Nk * H * d);
  memset(dv, 0, sizeof(double) * (size_t)Nk * H * d);
  memset(dbias, 0, sizeof(double) * (size_t)H * Nq * Nk);
  double *p = malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
  double *dp = malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
  /* sequential: dk and dv collect contributions from every query */
  for (int h = 0; h < H; ++h)
    for (int j = 0; j < Nq; ++j) {
      const double *qj = q + ((long)j * H + h) * d;
      const double *gj = dout + ((long)j * H + h) * d;
      double mx = -INFINITY;
      int any = 0;
      for (int kk = 0; kk < Nk; ++kk) {
        if (mask && !mask[kk]) continue;
        const double *kv = k + ((long)kk * H + h) * d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += qj[c] * kv[c];
        p[kk] = dot * scale + bias[((long)h * Nq + j) * Nk + kk];
        if (!any || p[kk] > mx) mx = p[kk];
        any = 1;
      }
      if (!any) continue;
      double denom = 0.0;
      for (int kk = 0; kk < Nk; ++kk) {
        if (mask && !mask[kk]) { p[kk] = 0.0; continue; }
        p[kk] = exp(p[kk] - mx);
        denom += p[kk];
      }
      double pdp = 0.0; /* sum_m p_m dp_m */
      for (int kk = 0; kk < Nk; ++kk) {
        p[kk] /= denom;
        const double *vv = v + ((long)kk * H + h) * d;
        double t = 0.0;
        for (int c = 0; c < d; ++c) t += gj[c] * vv[c];
        dp[kk] = t;
        pdp += p[kk] * t;
      }
      double *dqj = dq + ((long)j * H + h) * d;
      for (int kk = 0; kk < Nk; ++kk) {
        if (p[kk] == 0.0) continue;
        const double ds = p[kk] * (dp[kk] - pdp);
        dbias[((long)h * Nq + j) * Nk + kk] = ds;
        const double *kv = k + ((long)kk * H + h) * d;
        double *dkk = dk + ((long)kk * H + h) * d;
        double *dvk = dv + ((long)kk * H + h) * d;
        for (int c = 0; c < d; ++c) {
          dqj[c] += ds * kv[c] * scale;
          dkk[c] += ds * qj[c] * scale;
          dvk[c] += p[kk] * gj[c];
        }
      }
    }
  free(p);
  free(dp);
  return 0;
}

/* ---------------------------------------------------------------------- */
/* The whole block.                                                        */

/* Softmax over the unmasked entries of s[0..n) (in place, masked entries set
 * to 0), then o[c] = sum_k s[k] * v[k*stride + c] for c < d.  Returns 0 and
 * o = 0 when every entry is masked. */
static int softmax_weighted_sum(double *s, const unsigned char *mask, long n,
                                const double *v, long stride, int d,
                                double *o) {
  double mx = -INFINITY;
  int any = 0;
  for (long kk = 0; kk < n; ++kk) {
    if (mask && !mask[kk]) continue;
    if (!any || s[kk] > mx) mx = s[kk];
    any = 1;
  }
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  if (!any) return 0;
  double denom = 0.0;
  for (long kk = 0; kk < n; ++kk) {
    if (mask && !mask[kk]) { s[kk] = 0.0; continue; }
    s[kk] = exp(s[kk] - mx);
    denom += s[kk];
  }
  for (long kk = 0; kk < n; ++kk) {
    if (s[kk] == 0.0) continue;
    double pk = s[kk] / denom;
    for (int c = 0; c < d; ++c) o[c] += pk * v[kk * stride + c];
  }
  return 1;
}

/* Starting node, row i: out_row[j][c] = out_{i j c} for all j; if o_row is
 * not NULL, also o_row[j][h*d + c] = o_{i j h c}, the attention output before
 * the gate. */
static void start_row(const oracle_params *p, const double *bias_all, long i,
                      double *out_row, double *o_row) {
  long N = p->N;
  int H = p->H, d = p->d, HD = H * d, cz = p->c_z;
  double scale = 1.0 / sqrt((double)d);
  /* features of the pairs (i, x) of this row, indexed by x */
  double *q = malloc(sizeof(double) * N * HD);
  double *k = malloc(sizeof(double) * N * HD);
  double *v = malloc(sizeof(double) * N * HD);
  double *g = malloc(sizeof(double) * N * HD);
  double *zb = malloc(sizeof(double) * cz);
  double *xb = malloc(sizeof(double) * cz);
  double *s = malloc(sizeof(double) * N);
  double *o = malloc(sizeof(double) * HD);
  double *upd = malloc(sizeof(double) * cz);
  for (long x = 0; x < N; ++x) {
    pair_feat f = {q + x * HD, k + x * HD, v + x * HD, g + x * HD, NULL};
    pair_features(p, i, x, zb, xb, f);
  }
  for (long j = 0; j < N; ++j) {
    for (int h = 0; h < H; ++h) {
      /* s_k = q_ij . k_ik / sqrt(d) + beta_h(j, k) */
      for (long kk = 0; kk < N; ++kk) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += q[j * HD + h * d + c] * k[kk * HD + h * d + c];
        s[kk] = dot * scale + bias_all[((long)h * N + j) * N + kk];
      }
      /* o_ij = sum_k p_k v_ik */
      softmax_weighted_sum(s, p->mask, N, v + h * d, HD, d, o + h * d);
    }
    if (o_row)
      for (int t = 0; t < HD; ++t) o_row[j * HD + t] = o[t];
    for (int t = 0; t < HD; ++t) o[t] *= g[j * HD + t];
    linear(p->Wo, p->bo, o, cz, HD, upd);
    for (int c = 0; c < cz; ++c) out_row[j * cz + c] = z_at(p, i, j, c) + upd[c];
  }
  free(q); free(k); free(v); free(g); free(zb); free(xb); free(s); free(o); free(upd);
}

/* Ending node, column j: out_col[i][c] = out_{i j c} for all i; if o_col is
 * not NULL, also o_col[i][h*d + c] = o_{i j h c}, the attention output before
 * the gate. */
static void end_col(const oracle_params *p, const double *bias_all, long j,
                    double *out_col, double *o_col) {
  long N = p->N;
  int H = p->H, d = p->d, HD = H * d, cz = p->c_z;
  double scale = 1.0 / sqrt((double)d);
  /* features of the pairs (x, j) of this column, indexed by x */
  double *q = malloc(sizeof(double) * N * HD);
  double *k = malloc(sizeof(double) * N * HD);
  double *v = malloc(sizeof(double) * N * HD);
  double *g = malloc(sizeof(double) * N * HD);
  double *zb = malloc(sizeof(double) * cz);
  double *xb = malloc(sizeof(double) * cz);
  double *s = malloc(sizeof(double) * N);
  double *o = malloc(sizeof(double) * HD);
  double *upd = malloc(sizeof(double) * cz);
  for (long x = 0; x < N; ++x) {
    pair_feat f = {q + x * HD, k + x * HD, v + x * HD, g + x * HD, NULL};
    pair_features(p, x, j, zb, xb, f);
  }
  for (long i = 0; i < N; ++i) {
    for (int h = 0; h < H; ++h) {
      /* s_k = q_ij . k_kj / sqrt(d) + beta_h(k, i) */
      for (long kk = 0; kk < N; ++kk) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += q[i * HD + h * d + c] * k[kk * HD + h * d + c];
        s[kk] = dot * scale + bias_all[((long)h * N + kk) * N + i];
      }
      /* o_ij = sum_k p_k v_kj */
      softmax_weighted_sum(s, p->mask, N, v + h * d, HD, d, o + h * d);
    }
    if (o_col)
      for (int t = 0; t < HD; ++t) o_col[i * HD + t] = o[t];
    for (int t = 0; t < HD; ++t) o[t] *= g[i * HD + t];
    linear(p->Wo, p->bo, o, cz, HD, upd);
    for (int c = 0; c < cz; ++c) out_col[i * cz + c] = z_at(p, i, j, c) + upd[c];
  }
  free(q); free(k); free(v); free(g); free(zb); free(xb); free(s); free(o); free(upd);
}

/* The whole block for a subset of lines.
 *   orientation 0 (starting node): lines are rows i; out[r][j][c] = out_{lines[r], j, c}
 *   orientation 1 (ending node):   lines are columns j; out[r][i][c] = out_{i, lines[r], c}
 * lines == NULL means every line 0..N-1 (n_lines must then be N).
 * bias_all may be NULL (computed here) or the [H][N][N] array produced by
 * oracle_pair_features, so repeated calls can share it.
 * o_out may be NULL, or [n_lines][N][H*d]: the attention output o (before the
 * gate) of the same pairs, laid out like out. */
int oracle_tri_attn(const oracle_params *p, int orientation, const int *lines,
                    int n_lines, const double *bias_all, double *out, double *o_out) {
  if (!p || !out || p->N <= 0 || p->c_z <= 0 || p->H <= 0 || p->d <= 0)
    return -1;
  if (orientation != 0 && orientation != 1) return -1;
  if (!lines && n_lines != p->N) return -1;
  long N = p->N;
  double *own = NULL;
  if (!bias_all) {
    own = malloc(sizeof(double) * (long)p->H * N * N);
    if (!own) return -2;
    oracle_pair_features(p, NULL, NULL, NULL, NULL, own);
    bias_all = own;
  }
  for (int r = 0; r < n_lines; ++r) {
    int ln = lines ? lines[r] : r;
    if (ln < 0 || ln >= N) { free(own); return -1; }
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n_lines; ++r) {
    long ln = lines ? lines[r] : r;
    double *dst = out + (long)r * N * p->c_z;
    double *odst = o_out ? o_out + (long)r * N * p->H * p->d : NULL;
    if (orientation == 0)
      start_row(p, bias_all, ln, dst, odst);
    else
      end_col(p, bias_all, ln, dst, odst);
  }
  free(own);
  return 0;
}
