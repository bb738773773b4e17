/*
 * MuSe oracle: a plain, slow, fp64 CPU statement of what the MuSe forward
 * operator computes.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * generator with the CUDA library; the two meet only at the seeded input
 * generator, which holds none of the method's arithmetic.
 *
 * Sources (all pages are titled "Multipole Semantic Attention: A Fast
 * Approximation of Softmax Attention for Pretraining"):
 *   [G]  gist.science page, "Technical Summary" -> "Methodology" ->
 *        "Core Mechanisms" (bidirectional clustering, residual decomposition,
 *        two-stage attention, exponential tilting, retrieval) and
 *        "Key Contributions".
 *   [A1] newx.sg page, "Abstract" and "AI Summary" (monopole + dipole
 *        correction, hierarchical block decomposition for causal attention,
 *        O(NCD) / O(NCD log N)).
 * The pages fix the structure but not the details; every reading taken where
 * they are silent is marked READING and listed in the design notes:
 *   - clustering is Lloyd k-means, squared Euclidean distance, ties to the
 *     lowest cluster index, empty clusters keep their previous centroid;
 *   - the seeded initialisation draws C distinct rows with a partial
 *     Fisher-Yates shuffle driven by Vigna's splitmix64;
 *   - the dipole uses the query-cluster centroid nu_i (first-order expansion
 *     of the kept cross term), the tilted mode expands about the tilted
 *     centroid k_hat_ij; the fine-query dipole (an accuracy variant) uses the
 *     query itself: u_qj = (S_j + s M_j q) / n_j;
 *   - the causal scheme is the binary (Fenwick-style) block decomposition.
 *
 * Layouts: Q [B,Hq,N,D], K and V [B,Hkv,N,D], O [B,Hq,N,D], all row-major,
 * all double here (bf16 / f32 inputs convert exactly to double).
 * q-head h reads kv-head h / (Hq/Hkv).
 *
 * Parity status: every function below is pinned by the oracle test-suite
 * (closed forms, invariants, brute force, a library k-means) except the
 * absolute accuracy of the approximation itself, which the pages give no
 * worked example for.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_MONOPOLE 0
#define ORC_DIPOLE 1
#define ORC_TILTED 2
#define ORC_DIPOLE_Q 3
#define ORC_TILTED_DIPOLE 4

/* ------------------------------------------------------------------------ */
/* splitmix64 (Vigna): state advances by the golden-ratio increment, output  */
/* is the increment-mixed state.  READING: seeded initialisation.            */
/* ------------------------------------------------------------------------ */
static const uint64_t SM64_GAMMA = 0x9E3779B97F4A7C15ULL;

uint64_t orc_splitmix64_next(uint64_t *state) {
  uint64_t z = (*state += SM64_GAMMA);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Stream start for (stream id, role); role 0 = keys, 1 = queries. */
uint64_t orc_stream_state(uint64_t seed, uint64_t sid, int role) {
  return seed + SM64_GAMMA * (2ULL * sid + (uint64_t)role + 1ULL);
}

/* The first C entries of a partial Fisher-Yates shuffle of 0..n-1:
 * for c = 0..C-1 swap(perm[c], perm[c + next() % (n - c)]). */
void orc_init_indices(int n, int C, uint64_t seed, uint64_t sid, int role,
                      int *idx_out) {
  int *perm = (int *)malloc(sizeof(int) * (size_t)n);
  for (int i = 0; i < n; ++i) perm[i] = i;
  uint64_t st = orc_stream_state(seed, sid, role);
  for (int c = 0; c < C; ++c) {
    uint64_t r = orc_splitmix64_next(&st);
    int j = c + (int)(r % (uint64_t)(n - c));
    int t = perm[c];
    perm[c] = perm[j];
    perm[j] = t;
  }
  for (int c = 0; c < C; ++c) idx_out[c] = perm[c];
  free(perm);
}

/* ------------------------------------------------------------------------ */
/* k-means: READING of the separate query and key clustering of [G] Core     */
/* Mechanisms, "Bidirectional Semantic Clustering".                          */
/* ------------------------------------------------------------------------ */
static double sqdist(const double *x, const double *c, int D) {
  double s = 0.0;
  for (int d = 0; d < D; ++d) {
    double t = x[d] - c[d];
    s += t * t;
  }
  return s;
}

/* Assignment step: a(x) = argmin_c ||x - c||^2, ties to the lowest c.
 * Returns the inertia sum_x ||x - c_a(x)||^2. */
double orc_kmeans_assign(const double *X, int n, int D, int C,
                         const double *cent, int *assign) {
  double inertia = 0.0;
  for (int t = 0; t < n; ++t) {
    const double *x = X + (size_t)t * D;
    int best = 0;
    double bd = sqdist(x, cent, D);
    for (int c = 1; c < C; ++c) {
      double d = sqdist(x, cent + (size_t)c * D, D);
      if (d < bd) {
        bd = d;
        best = c;
      }
    }
    assign[t] = best;
    inertia += bd;
  }
  return inertia;
}

/* Update step: each centroid becomes the mean of its members (sum in token
 * order); a cluster with no members keeps its previous centroid. */
void orc_kmeans_update(const double *X, int n, int D, int C, const int *assign,
                       double *cent, int *counts) {
  double *sum = (double *)calloc((size_t)C * D, sizeof(double));
  for (int c = 0; c < C; ++c) counts[c] = 0;
  for (int t = 0; t < n; ++t) {
    int a = assign[t];
    counts[a] += 1;
    for (int d = 0; d < D; ++d) sum[(size_t)a * D + d] += X[(size_t)t * D + d];
  }
  for (int c = 0; c < C; ++c)
    if (counts[c] > 0)
      for (int d = 0; d < D; ++d)
        cent[(size_t)c * D + d] = sum[(size_t)c * D + d] / (double)counts[c];
  free(sum);
}

/* Lloyd k-means with `iters` (assign, update) rounds.  Starts from `init`
 * when given, else from the seeded rows.  Outputs the last assignment, the
 * centroids after the last update (the means of that assignment) and the
 * cluster sizes.  `inertia` (optional, [iters]) records each assign step's
 * inertia.  C must satisfy 1 <= C <= n. */
void orc_kmeans(const double *X, int n, int D, int C, int iters, uint64_t seed,
                uint64_t sid, int role, const double *init, int *assign,
                double *cent, int *counts, double *inertia) {
  if (init) {
    memcpy(cent, init, sizeof(double) * (size_t)C * D);
  } else {
    int *idx = (int *)malloc(sizeof(int) * (size_t)C);
    orc_init_indices(n, C, seed, sid, role, idx);
    for (int c = 0; c < C; ++c)
      memcpy(cent + (size_t)c * D, X + (size_t)idx[c] * D, sizeof(double) * D);
    free(idx);
  }
  for (int it = 0; it < iters; ++it) {
    double j = orc_kmeans_assign(X, n, D, C, cent, assign);
    if (inertia) inertia[it] = j;
    orc_kmeans_update(X, n, D, C, assign, cent, counts);
  }
}

/* Centroids and sizes for a given assignment (teacher forcing): the mean of
 * the members; clusters without members get a zero centroid (never used). */
static void centroids_of(const double *X, int n, int D, int C, const int *assign,
                         double *cent, int *counts) {
  memset(cent, 0, sizeof(double) * (size_t)C * D);
  orc_kmeans_update(X, n, D, C, assign, cent, counts);
}

/* ------------------------------------------------------------------------ */
/* Key-cluster summaries: monopole (n_j, mu_j, S_j = sum v) and the dipole    */
/* M_j[e][d] = sum_{t in j} v_t[e] (k_t[d] - mu_j[d]): the correction that   */
/* carries how the keys spread about their centroid ([A1] Abstract).         */
/* ------------------------------------------------------------------------ */
void orc_summaries(const double *K, const double *V, int n, int D, int C,
                   const int *assign, const double *mu, double *S, double *M) {
  memset(S, 0, sizeof(double) * (size_t)C * D);
  if (M) memset(M, 0, sizeof(double) * (size_t)C * D * D);
  for (int t = 0; t < n; ++t) {
    int j = assign[t];
    const double *k = K + (size_t)t * D, *v = V + (size_t)t * D;
    for (int e = 0; e < D; ++e) S[(size_t)j * D + e] += v[e];
    if (M)
      for (int e = 0; e < D; ++e)
        for (int d = 0; d < D; ++d)
          M[((size_t)j * D + e) * D + d] += v[e] * (k[d] - mu[(size_t)j * D + d]);
  }
}

/* ------------------------------------------------------------------------ */
/* One MuSe block problem: a query block (with its clustering) attends a key  */
/* block (with its clustering).  Stage 1 ([G] "Stage 1 (Coarse)",            */
/* "Exponential Tilting", "Cluster Selection") builds, per query cluster i    */
/* and key cluster j, the weight W_ij, the summary value u_ij, the tilted     */
/* centroid k_hat_ij and the selection score s_ij; R_i = top-k1 clusters.     */
/* Stage 2 ([G] "Stage 2 (Refinement)", "Exact Attention") adds, for every    */
/* query, one far-field term per non-retrieved non-empty cluster and one      */
/* exact term per key of the retrieved clusters, into that query's softmax.   */
/* ------------------------------------------------------------------------ */
typedef struct {
  double m, l; /* running max and normaliser */
  double *acc; /* [D] running weighted sum */
} softmax_acc;

/* Plain online softmax: rescale the running sums whenever the max grows. */
static void acc_add(double *m, double *l, double *acc, int D, double logit,
                    const double *val) {
  if (logit > *m) {
    double sc = (*m == -INFINITY) ? 0.0 : exp(*m - logit);
    *l = *l * sc + 1.0;
    for (int d = 0; d < D; ++d) acc[d] = acc[d] * sc + val[d];
    *m = logit;
  } else {
    double w = exp(logit - *m);
    *l += w;
    for (int d = 0; d < D; ++d) acc[d] += w * val[d];
  }
}

static double dot(const double *a, const double *b, int D) {
  double s = 0.0;
  for (int d = 0; d < D; ++d) s += a[d] * b[d];
  return s;
}

typedef struct {
  int n, D, C;
  const double *K, *V; /* [n, D] */
  int *assign, *count;
  double *mu, *S, *M;
} key_block;

typedef struct {
  int n, D, C;
  const double *Q;
  int *assign, *count;
  double *nu;
} query_block;

/* Stage 1.  Outputs (row-major over [Cq][Ck]):
 *   log W, score (score = -inf for empty key clusters), U and Khat
 *   ([Cq][Ck][D]),
 *   R [Cq][k1] (-1 padded), nsel [Cq]. */
static void stage1(const query_block *qb, const key_block *kb, double scale,
                   int mode, int k1, double *logW, double *score, double *U,
                   double *Khat, int *R, int *nsel) {
  const int D = kb->D, Cq = qb->C, Ck = kb->C;
  double *a = (double *)malloc(sizeof(double) * (size_t)(kb->n > 0 ? kb->n : 1));
  for (int i = 0; i < Cq; ++i) {
    const double *nu = qb->nu + (size_t)i * D;
    for (int j = 0; j < Ck; ++j) {
      size_t ij = (size_t)i * Ck + j;
      double *u = U + ij * D, *kh = Khat + ij * D;
      const double *mu = kb->mu + (size_t)j * D, *S = kb->S + (size_t)j * D;
      int nj = kb->count[j];
      if (nj == 0) {
        logW[ij] = -INFINITY;
        score[ij] = -INFINITY;
        for (int d = 0; d < D; ++d) u[d] = kh[d] = 0.0;
        continue;
      }
      if (mode == ORC_MONOPOLE || mode == ORC_DIPOLE || mode == ORC_DIPOLE_Q) {
        logW[ij] = log((double)nj);
        for (int e = 0; e < D; ++e) {
          double x = S[e];
          if (mode == ORC_DIPOLE) {
            /* first-order term of exp(s nu_i . k~): (s/n_j) M_j nu_i
             * (the fine-query dipole adds (s/n_j) M_j q per query in stage 2) */
            const double *Me = kb->M + ((size_t)j * D + e) * D;
            x += scale * dot(Me, nu, D);
          }
          u[e] = x / (double)nj;
        }
        for (int d = 0; d < D; ++d) kh[d] = mu[d];
        score[ij] = scale * dot(nu, mu, D) + log((double)nj);
      } else {
        /* exponential tilting by the query centroid: w_t = exp(s nu.(k_t-mu)) */
        double mx = -INFINITY;
        int cnt = 0;
        for (int t = 0; t < kb->n; ++t) {
          if (kb->assign[t] != j) continue;
          const double *k = kb->K + (size_t)t * D;
          double g = 0.0;
          for (int d = 0; d < D; ++d) g += nu[d] * (k[d] - mu[d]);
          a[t] = scale * g;
          if (a[t] > mx) mx = a[t];
          ++cnt;
        }
        double z = 0.0;
        for (int d = 0; d < D; ++d) u[d] = kh[d] = 0.0;
        for (int t = 0; t < kb->n; ++t) {
          if (kb->assign[t] != j) continue;
          double w = exp(a[t] - mx);
          z += w;
          for (int d = 0; d < D; ++d) {
            u[d] += w * kb->V[(size_t)t * D + d];
            kh[d] += w * kb->K[(size_t)t * D + d];
          }
        }
        for (int d = 0; d < D; ++d) {
          u[d] /= z;
          kh[d] /= z;
        }
        logW[ij] = mx + log(z);
        score[ij] = scale * dot(nu, mu, D) + logW[ij];
        (void)cnt;
      }
    }
    /* top-k1 by score, ties to the lowest cluster index, empty clusters never */
    int taken = 0;
    for (int r = 0; r < k1; ++r) R[(size_t)i * (k1 > 0 ? k1 : 1) + r] = -1;
    for (int r = 0; r < k1; ++r) {
      int best = -1;
      double bs = -INFINITY;
      for (int j = 0; j < Ck; ++j) {
        size_t ij = (size_t)i * Ck + j;
        if (kb->count[j] == 0) continue;
        int dup = 0;
        for (int q = 0; q < taken; ++q)
          if (R[(size_t)i * k1 + q] == j) dup = 1;
        if (dup) continue;
        if (best < 0 || score[ij] > bs) {
          best = j;
          bs = score[ij];
        }
      }
      if (best < 0) break;
      R[(size_t)i * k1 + taken++] = best;
    }
    nsel[i] = taken;
  }
  free(a);
}

/* Stage 2 for every query of the block: far-field terms and exact terms. */
static void stage2(const query_block *qb, const key_block *kb, double scale,
                   int mode, int k1, const double *logW, const double *U,
                   const double *Khat, const int *R, const int *nsel,
                   double *m, double *l, double *acc /* [nq][D] */,
                   long long *n_exact /* nullable, [nq] */) {
  const int D = kb->D, Ck = kb->C;
  char *inR = (char *)malloc((size_t)Ck);
  double *uq = (double *)malloc(sizeof(double) * (size_t)D);
  for (int q = 0; q < qb->n; ++q) {
    const double *x = qb->Q + (size_t)q * D;
    int i = qb->assign[q];
    const double *nu = qb->nu + (size_t)i * D;
    memset(inR, 0, (size_t)Ck);
    for (int r = 0; r < nsel[i]; ++r) inR[R[(size_t)i * k1 + r]] = 1;
    double *aq = acc + (size_t)q * D;
    for (int j = 0; j < Ck; ++j) {
      if (kb->count[j] == 0 || inR[j]) continue;
      size_t ij = (size_t)i * Ck + j;
      double lam;
      if (mode == ORC_TILTED || mode == ORC_TILTED_DIPOLE) {
        const double *kh = Khat + ij * D, *mu = kb->mu + (size_t)j * D;
        double g = 0.0;
        for (int d = 0; d < D; ++d) g += (x[d] - nu[d]) * kh[d];
        lam = scale * g + scale * dot(nu, mu, D) + logW[ij];
      } else {
        lam = scale * dot(x, kb->mu + (size_t)j * D, D) + logW[ij];
      }
      const double *val = U + ij * D;
      if (mode == ORC_DIPOLE_Q) {
        /* the first-order term of exp(s q . k~) with the query itself:
         * u_qj = S_j / n_j + (s / n_j) M_j q */
        for (int e = 0; e < D; ++e)
          uq[e] = val[e] + scale * dot(kb->M + ((size_t)j * D + e) * D, x, D) / (double)kb->count[j];
        val = uq;
      }
      if (mode == ORC_TILTED_DIPOLE) {
        /* the tilted per-pair dipole: the tilt exp(s nu_i . k_t) is kept
         * exactly and exp(s (q - nu_i) . k_t) is expanded to first order
         * about the tilted centroid k^_ij, so the value gains
         * s M^_ij (q - nu_i), M^_ij = sum_t w^_t v_t (k_t - k^_ij)^T with the
         * tilted weights w^_t = exp(s nu_i . (k_t - mu_j) - log W_ij);
         * summed here token by token */
        const double *kh = Khat + ij * D, *mu = kb->mu + (size_t)j * D;
        for (int e = 0; e < D; ++e) uq[e] = val[e];
        for (int t = 0; t < kb->n; ++t) {
          if (kb->assign[t] != j) continue;
          const double *k = kb->K + (size_t)t * D;
          double a = 0.0, g = 0.0;
          for (int d = 0; d < D; ++d) {
            a += nu[d] * (k[d] - mu[d]);
            g += (x[d] - nu[d]) * (k[d] - kh[d]);
          }
          const double w = exp(scale * a - logW[ij]);
          for (int e = 0; e < D; ++e) uq[e] += scale * w * g * kb->V[(size_t)t * D + e];
        }
        val = uq;
      }
      acc_add(&m[q], &l[q], aq, D, lam, val);
    }
    long long ne = 0;
    for (int t = 0; t < kb->n; ++t) {
      if (!inR[kb->assign[t]]) continue;
      acc_add(&m[q], &l[q], aq, D, scale * dot(x, kb->K + (size_t)t * D, D),
              kb->V + (size_t)t * D);
      ++ne;
    }
    if (n_exact) n_exact[q] += ne;
  }
  free(inR);
  free(uq);
}

/* Debug outputs of one block problem (all optional). */
typedef struct {
  int *selected;   /* [Cq][k1] */
  double *U;       /* [Cq][Ck][D] */
  double *logW;    /* [Cq][Ck] */
} block_debug;

static void run_block(const query_block *qb, const key_block *kb, double scale,
                      int mode, int k1, double *m, double *l, double *acc,
                      long long *n_exact, block_debug *dbg) {
  const int D = kb->D, Cq = qb->C, Ck = kb->C;
  size_t cc = (size_t)Cq * Ck;
  double *W = (double *)malloc(sizeof(double) * cc);
  double *score = (double *)malloc(sizeof(double) * cc);
  double *U = (double *)malloc(sizeof(double) * cc * D);
  double *Kh = (double *)malloc(sizeof(double) * cc * D);
  int kk = k1 > 0 ? k1 : 1;
  int *R = (int *)malloc(sizeof(int) * (size_t)Cq * kk);
  int *nsel = (int *)malloc(sizeof(int) * (size_t)Cq);
  stage1(qb, kb, scale, mode, k1, W, score, U, Kh, R, nsel);
  stage2(qb, kb, scale, mode, k1, W, U, Kh, R, nsel, m, l, acc, n_exact);
  if (dbg) {
    if (dbg->selected && k1 > 0) memcpy(dbg->selected, R, sizeof(int) * (size_t)Cq * k1);
    if (dbg->U) memcpy(dbg->U, U, sizeof(double) * cc * D);
    if (dbg->logW) memcpy(dbg->logW, W, sizeof(double) * cc);
  }
  free(W); free(score); free(U); free(Kh); free(R); free(nsel);
}

/* Cluster one block (k-means, or teacher-forced means of a given assignment). */
static void cluster_block(const double *X, int n, int D, int C, int iters,
                          uint64_t seed, uint64_t sid, int role,
                          const int *given, int *assign, double *cent,
                          int *counts) {
  if (given) {
    memcpy(assign, given, sizeof(int) * (size_t)n);
    centroids_of(X, n, D, C, assign, cent, counts);
  } else {
    orc_kmeans(X, n, D, C, iters, seed, sid, role, NULL, assign, cent, counts, NULL);
  }
}

static void make_keys(key_block *kb, const double *K, const double *V, int n,
                      int D, int C, int iters, uint64_t seed, uint64_t sid,
                      const int *given, int need_M) {
  kb->n = n; kb->D = D; kb->C = C; kb->K = K; kb->V = V;
  kb->assign = (int *)malloc(sizeof(int) * (size_t)n);
  kb->count = (int *)malloc(sizeof(int) * (size_t)C);
  kb->mu = (double *)malloc(sizeof(double) * (size_t)C * D);
  kb->S = (double *)malloc(sizeof(double) * (size_t)C * D);
  kb->M = need_M ? (double *)malloc(sizeof(double) * (size_t)C * D * D) : NULL;
  cluster_block(K, n, D, C, iters, seed, sid, 0, given, kb->assign, kb->mu, kb->count);
  orc_summaries(K, V, n, D, C, kb->assign, kb->mu, kb->S, kb->M);
}

static void free_keys(key_block *kb) {
  free(kb->assign); free(kb->count); free(kb->mu); free(kb->S); free(kb->M);
}

static void make_queries(query_block *qb, const double *Q, int n, int D, int C,
                         int iters, uint64_t seed, uint64_t sid,
                         const int *given) {
  qb->n = n; qb->D = D; qb->C = C; qb->Q = Q;
  qb->assign = (int *)malloc(sizeof(int) * (size_t)n);
  qb->count = (int *)malloc(sizeof(int) * (size_t)C);
  qb->nu = (double *)malloc(sizeof(double) * (size_t)C * D);
  cluster_block(Q, n, D, C, iters, seed, sid, 1, given, qb->assign, qb->nu, qb->count);
}

static void free_queries(query_block *qb) {
  free(qb->assign); free(qb->count); free(qb->nu);
}

static void finish(int nq, int D, const double *l, const double *acc, double *O) {
  for (int q = 0; q < nq; ++q)
    for (int d = 0; d < D; ++d) O[(size_t)q * D + d] = acc[(size_t)q * D + d] / l[q];
}

/* ------------------------------------------------------------------------ */
/* Acausal MuSe ([G] Core Mechanisms; [A1] Abstract, O(NCD) acausal form).    */
/* Per (b, kv-head): cluster the keys, summarise; per q-head of the group:    */
/* cluster the queries, stage 1, stage 2.                                     */
/* hq_mask (optional, [B*Hq]): compute only the q-heads whose entry is non-0. */
/* Debug outputs (optional): q_assign [B,Hq,N], k_assign [B,Hkv,N],           */
/* q_cent [B,Hq,Cq,D], k_cent [B,Hkv,Ck,D], k_count [B,Hkv,Ck],               */
/* selected [B,Hq,Cq,k1], n_exact [B,Hq,N] (exact keys per query).            */
/* q_assign_in / k_assign_in (optional) teacher-force the clusterings.        */
/* ks0 / qs0: stream ids of the first key / query row set (0 for a whole     */
/* layer): row set (b, h) draws the seeded start of stream ks0 + b Hkv + h.   */
/* ------------------------------------------------------------------------ */
void orc_muse_acausal(const double *Q, const double *K, const double *V, int B,
                      int Hq, int Hkv, int N, int D, int Cq, int Ck, int iters,
                      uint64_t seed, uint64_t ks0, uint64_t qs0, int k1,
                      double scale, int mode, const unsigned char *hq_mask,
                      const int *q_assign_in, const int *k_assign_in, double *O,
                      int *q_assign, int *k_assign, double *q_cent,
                      double *k_cent, int *k_count, int *selected,
                      long long *n_exact) {
  const int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic)
  for (int bk = 0; bk < B * Hkv; ++bk) {
    int b = bk / Hkv, hk = bk % Hkv;
    int any = 0;
    for (int g = 0; g < G; ++g)
      if (!hq_mask || hq_mask[b * Hq + hk * G + g]) any = 1;
    if (!any) continue;
    size_t koff = (size_t)bk * N;
    key_block kb;
    make_keys(&kb, K + koff * D, V + koff * D, N, D, Ck, iters, seed,
              ks0 + (uint64_t)bk, k_assign_in ? k_assign_in + koff : NULL,
              mode == ORC_DIPOLE || mode == ORC_DIPOLE_Q);
    if (k_assign) memcpy(k_assign + koff, kb.assign, sizeof(int) * (size_t)N);
    if (k_cent) memcpy(k_cent + (size_t)bk * Ck * D, kb.mu, sizeof(double) * (size_t)Ck * D);
    if (k_count) memcpy(k_count + (size_t)bk * Ck, kb.count, sizeof(int) * (size_t)Ck);
    for (int g = 0; g < G; ++g) {
      int hq = hk * G + g, bq = b * Hq + hq;
      if (hq_mask && !hq_mask[bq]) continue;
      size_t qoff = (size_t)bq * N;
      query_block qb;
      make_queries(&qb, Q + qoff * D, N, D, Cq, iters, seed, qs0 + (uint64_t)bq,
                   q_assign_in ? q_assign_in + qoff : NULL);
      double *m = (double *)malloc(sizeof(double) * (size_t)N);
      double *l = (double *)calloc((size_t)N, sizeof(double));
      double *acc = (double *)calloc((size_t)N * D, sizeof(double));
      for (int q = 0; q < N; ++q) m[q] = -INFINITY;
      if (n_exact) memset(n_exact + qoff, 0, sizeof(long long) * (size_t)N);
      block_debug dbg = {selected ? selected + (size_t)bq * Cq * k1 : NULL, NULL, NULL};
      run_block(&qb, &kb, scale, mode, k1, m, l, acc, n_exact ? n_exact + qoff : NULL, &dbg);
      finish(N, D, l, acc, O + qoff * D);
      if (q_assign) memcpy(q_assign + qoff, qb.assign, sizeof(int) * (size_t)N);
      if (q_cent) memcpy(q_cent + (size_t)bq * Cq * D, qb.nu, sizeof(double) * (size_t)Cq * D);
      free(m); free(l); free(acc);
      free_queries(&qb);
    }
    free_keys(&kb);
  }
}

/* ------------------------------------------------------------------------ */
/* Causal MuSe: hierarchical block decomposition ([A1] Abstract: exact       */
/* attention near the diagonal, summaries far from it, O(NCD log N)).        */
/* READING: blocks of L tokens; query block b attends its own block exactly   */
/* (causally) and, for every level l whose bit is set in b, the key block     */
/* [2p s, (2p+1) s) with s = L 2^l and p = b >> (l+1), via one MuSe block     */
/* problem clustered inside those two blocks with C_eff = min(C, s).  The     */
/* levels tile [0, bL) exactly once.  All terms meet in one softmax.          */
/* Debug layouts (optional): q_assign [B,Hq,Lv,N/2], k_assign [B,Hkv,Lv,N/2]  */
/* where entry (l, p s + r) is token r of pair p's block at level l;          */
/* selected [B,Hq,P,C,k1] with P = N/L - 1 block problems numbered level by   */
/* level (rows i >= C_eff left as the caller filled them);                    */
/* n_exact [B,Hq,N] counts exact keys per query including the local block.    */
/* ------------------------------------------------------------------------ */
void orc_muse_causal(const double *Q, const double *K, const double *V, int B,
                     int Hq, int Hkv, int N, int D, int L, int C, int iters,
                     uint64_t seed, uint64_t ks0, uint64_t qs0, int k1,
                     double scale, int mode,
                     const unsigned char *hq_mask, const int *q_assign_in,
                     const int *k_assign_in, double *O, int *q_assign,
                     int *k_assign, int *selected, long long *n_exact) {
  const int G = Hq / Hkv;
  const int nblk = N / L;
  int levels = 0;
  while ((1 << levels) < nblk) ++levels;
  const int pmax = nblk / 2 > 0 ? nblk / 2 : 1;
  const size_t half = (size_t)N / 2;
#pragma omp parallel for schedule(dynamic)
  for (int bk = 0; bk < B * Hkv; ++bk) {
    int b = bk / Hkv, hk = bk % Hkv;
    int any = 0;
    for (int g = 0; g < G; ++g)
      if (!hq_mask || hq_mask[b * Hq + hk * G + g]) any = 1;
    if (!any) continue;
    const double *Kh = K + (size_t)bk * N * D, *Vh = V + (size_t)bk * N * D;
    double *m = (double *)malloc(sizeof(double) * (size_t)G * N);
    double *l = (double *)calloc((size_t)G * N, sizeof(double));
    double *acc = (double *)calloc((size_t)G * N * D, sizeof(double));
    long long *ne = (long long *)calloc((size_t)G * N, sizeof(long long));
    for (size_t i = 0; i < (size_t)G * N; ++i) m[i] = -INFINITY;
    int pbase = 0; /* block problems of the levels below lv */
    for (int lv = 0; lv < levels; ++lv) {
      int s = L << lv;
      int npairs = N / (2 * s);
      int Ce = C < s ? C : s;
      for (int p = 0; p < npairs; ++p) {
        int k0 = 2 * p * s, q0 = (2 * p + 1) * s;
        size_t slot = (size_t)lv * half + (size_t)p * s;
        uint64_t ksid = ((ks0 + (uint64_t)bk) * levels + lv) * pmax + p;
        key_block kb;
        make_keys(&kb, Kh + (size_t)k0 * D, Vh + (size_t)k0 * D, s, D, Ce, iters,
                  seed, ksid,
                  k_assign_in ? k_assign_in + (size_t)bk * levels * half + slot : NULL,
                  mode == ORC_DIPOLE || mode == ORC_DIPOLE_Q);
        if (k_assign)
          memcpy(k_assign + (size_t)bk * levels * half + slot, kb.assign, sizeof(int) * (size_t)s);
        for (int g = 0; g < G; ++g) {
          int hq = hk * G + g, bq = b * Hq + hq;
          if (hq_mask && !hq_mask[bq]) continue;
          const double *Qh = Q + (size_t)bq * N * D;
          uint64_t qsid = ((qs0 + (uint64_t)bq) * levels + lv) * pmax + p;
          query_block qb;
          make_queries(&qb, Qh + (size_t)q0 * D, s, D, Ce, iters, seed, qsid,
                       q_assign_in ? q_assign_in + (size_t)bq * levels * half + slot : NULL);
          if (q_assign)
            memcpy(q_assign + (size_t)bq * levels * half + slot, qb.assign, sizeof(int) * (size_t)s);
          size_t o = (size_t)g * N + q0;
          block_debug dbg = {selected ? selected + ((size_t)bq * (nblk - 1) + pbase + p) *
                                                       (size_t)C * (k1 > 0 ? k1 : 1)
                                      : NULL,
                             NULL, NULL};
          run_block(&qb, &kb, scale, mode, k1, m + o, l + o, acc + o * D, ne + o, &dbg);
          free_queries(&qb);
        }
        free_keys(&kb);
      }
      pbase += npairs;
    }
    /* exact local block: keys t with floor(t/L) == floor(q/L) and t <= q */
    for (int g = 0; g < G; ++g) {
      int hq = hk * G + g, bq = b * Hq + hq;
      if (hq_mask && !hq_mask[bq]) continue;
      const double *Qh = Q + (size_t)bq * N * D;
      for (int q = 0; q < N; ++q) {
        size_t o = (size_t)g * N + q;
        int t0 = (q / L) * L;
        for (int t = t0; t <= q; ++t) {
          acc_add(&m[o], &l[o], acc + o * D, D,
                  scale * dot(Qh + (size_t)q * D, Kh + (size_t)t * D, D),
                  Vh + (size_t)t * D);
          ne[o] += 1;
        }
      }
      finish(N, D, l + (size_t)g * N, acc + (size_t)g * N * D, O + (size_t)bq * N * D);
      if (n_exact) memcpy(n_exact + (size_t)bq * N, ne + (size_t)g * N, sizeof(long long) * (size_t)N);
    }
    free(m); free(l); free(acc); free(ne);
  }
}

/* ------------------------------------------------------------------------ */
/* Exact softmax attention (the quantity MuSe approximates; [G] "Problem      */
/* Statement").  causal != 0 masks keys t > q.                                */
/* ------------------------------------------------------------------------ */
/* One query row: softmax over keys [0, tend) of Kh with values Vh. */
static void exact_row(const double *q, const double *Kh, const double *Vh,
                      int tend, int D, double scale, double *lg, double *e) {
  double mx = -INFINITY;
  for (int t = 0; t < tend; ++t) {
    lg[t] = scale * dot(q, Kh + (size_t)t * D, D);
    if (lg[t] > mx) mx = lg[t];
  }
  double z = 0.0;
  for (int d = 0; d < D; ++d) e[d] = 0.0;
  for (int t = 0; t < tend; ++t) {
    double w = exp(lg[t] - mx);
    z += w;
    for (int d = 0; d < D; ++d) e[d] += w * Vh[(size_t)t * D + d];
  }
  for (int d = 0; d < D; ++d) e[d] /= z;
}

void orc_exact_attn(const double *Q, const double *K, const double *V, int B,
                    int Hq, int Hkv, int N, int D, double scale, int causal,
                    const unsigned char *hq_mask, double *E) {
  const int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic)
  for (int bq = 0; bq < B * Hq; ++bq) {
    if (hq_mask && !hq_mask[bq]) continue;
    int b = bq / Hq, hq = bq % Hq, bk = b * Hkv + hq / G;
    const double *Qh = Q + (size_t)bq * N * D;
    const double *Kh = K + (size_t)bk * N * D, *Vh = V + (size_t)bk * N * D;
    double *lg = (double *)malloc(sizeof(double) * (size_t)N);
    for (int q = 0; q < N; ++q)
      exact_row(Qh + (size_t)q * D, Kh, Vh, causal ? q + 1 : N, D, scale, lg,
                E + ((size_t)bq * N + q) * D);
    free(lg);
  }
}

/* The same for selected query rows of one (b, q-head) bq: E [nrows][D]. */
void orc_exact_attn_rows(const double *Q, const double *K, const double *V,
                         int B, int Hq, int Hkv, int N, int D, double scale,
                         int causal, int bq, int nrows, const int *rows,
                         double *E) {
  const int G = Hq / Hkv;
  int b = bq / Hq, hq = bq % Hq, bk = b * Hkv + hq / G;
  (void)B;
  const double *Qh = Q + (size_t)bq * N * D;
  const double *Kh = K + (size_t)bk * N * D, *Vh = V + (size_t)bk * N * D;
#pragma omp parallel
  {
    double *lg = (double *)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic)
    for (int i = 0; i < nrows; ++i) {
      int q = rows[i];
      exact_row(Qh + (size_t)q * D, Kh, Vh, causal ? q + 1 : N, D, scale, lg,
                E + (size_t)i * D);
    }
    free(lg);
  }
}

/* Stage-1 debug for one acausal (b, q-head) problem under teacher forcing:
 * returns log W [Cq][Ck], U [Cq][Ck][D] and R [Cq][k1] for the given
 * clusterings. */
void orc_stage1_debug(const double *Qh, const double *Kh, const double *Vh,
                      int N, int D, int Cq, int Ck, const int *q_assign,
                      const int *k_assign, int k1, double scale, int mode,
                      double *logW, double *U, int *selected) {
  key_block kb;
  make_keys(&kb, Kh, Vh, N, D, Ck, 1, 0, 0, k_assign, mode == ORC_DIPOLE || mode == ORC_DIPOLE_Q);
  query_block qb;
  make_queries(&qb, Qh, N, D, Cq, 1, 0, 0, q_assign);
  double *m = (double *)malloc(sizeof(double) * (size_t)N);
  double *l = (double *)calloc((size_t)N, sizeof(double));
  double *acc = (double *)calloc((size_t)N * D, sizeof(double));
  for (int q = 0; q < N; ++q) m[q] = -INFINITY;
  block_debug dbg = {selected, U, logW};
  run_block(&qb, &kb, scale, mode, k1, m, l, acc, NULL, &dbg);
  free(m); free(l); free(acc);
  free_queries(&qb);
  free_keys(&kb);
}

/* Threads an OpenMP region of this library would use (1 without OpenMP). */
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
