/*
 * MC-Sparse CPU oracle: plain, slow, fp64.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call this code:
 * only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * Every input is a bf16 tensor (passed as uint16 bit patterns) that is widened
 * exactly to double. One call works on one (batch, head) slice: `x` points at
 * token 0 of that head and consecutive tokens are `stride` elements apart
 * (stride = H * d for the [B, N, H, d] layout).
 *
 * Sources (web pages about the method):
 *  - "MC-Sparse: Deconstructing and Closing the Dense-Sparse Attention Gap in
 *    Diffusion Transformers" (paper listing, thelatestinai.com): Abstract,
 *    Table 4 (token-granular selection), Table 6 (kernel), Table 8 (metadata).
 *  - "MC-Sparse: 高分辨率3D生成怎样减少注意力计算，又保住细结构？"
 *    (aiwillknow.com analysis), "图解主要方法" steps 1-5: Fast PDDP grouping
 *    (step 1), exact-probability top-K (step 2), residual R (step 3), reuse
 *    (step 4), offload and prefetch (step 5).
 *  - aimodeling.com article "Tencent MC-Sparse ... H3 diffusion 1.8x",
 *    section "What MC-Sparse actually does".
 *
 * Readings taken where the pages are silent (each listed in the design notes):
 *  softmax scale 1/sqrt(d), no mask; PDDP uses the exact principal eigenvector
 *  (cyclic Jacobi), and its "fast" variant the top Ritz vector of a k-step
 *  Krylov space from a SplitMix64 start vector, each with the sign fixed so
 *  that its largest-magnitude entry is positive (lowest index on ties); a node of n queries and T = ceil(n/g) tiles
 *  sends the ceil(T/2)*g queries of smallest (projection, token) to the left
 *  child; members of every node are kept in ascending token order; group mass
 *  is a sum; top-K ties go to the lower token index and the K indices are
 *  emitted ascending; sparse attention renormalises over the selected set.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* bf16 widening                                                            */
/* ------------------------------------------------------------------------ */

double orc_bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static void load_row(const uint16_t* x, long stride, int d, int tok, double* out) {
  const uint16_t* r = x + (long)tok * stride;
  for (int e = 0; e < d; ++e) out[e] = orc_bf16_to_f64(r[e]);
}

/* ------------------------------------------------------------------------ */
/* Symmetric eigensolver: cyclic Jacobi (Golub and Van Loan, "Matrix        */
/* Computations", section 8.5, the cyclic-by-row Jacobi method).            */
/* ------------------------------------------------------------------------ */

/*
 * A: n x n symmetric, row-major, overwritten. On return evals[j] and column j
 * of evecs (row-major n x n, evecs[i*n + j]) form the eigenpairs, sorted by
 * eigenvalue descending. Sweeps stop once the off-diagonal Frobenius norm is
 * at most tol * ||A||_F. Returns the number of sweeps, or -1 if max_sweeps
 * ran out.
 */
int orc_jacobi_eigh(int n, double* A, double* evals, double* evecs, double tol, int max_sweeps) {
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j) evecs[i * n + j] = (i == j) ? 1.0 : 0.0;
  double fro = 0.0;
  for (int i = 0; i < n * n; ++i) fro += A[i] * A[i];
  fro = sqrt(fro);
  int sweep = 0;
  for (;;) {
    double off = 0.0;
    for (int p = 0; p < n; ++p)
      for (int q = p + 1; q < n; ++q) off += 2.0 * A[p * n + q] * A[p * n + q];
    if (sqrt(off) <= tol * fro || fro == 0.0) break;
    if (sweep >= max_sweeps) { sweep = -1; break; }
    ++sweep;
    for (int p = 0; p < n - 1; ++p) {
      for (int q = p + 1; q < n; ++q) {
        double apq = A[p * n + q];
        if (apq == 0.0) continue;
        double app = A[p * n + p], aqq = A[q * n + q];
        /* rotation that zeroes A[p][q]: tan(theta) = t, the smaller root */
        double tau = (aqq - app) / (2.0 * apq);
        double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
        double c = 1.0 / sqrt(1.0 + t * t);
        double s = t * c;
        for (int k = 0; k < n; ++k) { /* A <- A J (columns p, q) */
          double akp = A[k * n + p], akq = A[k * n + q];
          A[k * n + p] = c * akp - s * akq;
          A[k * n + q] = s * akp + c * akq;
        }
        for (int k = 0; k < n; ++k) { /* A <- J^T A (rows p, q) */
          double apk = A[p * n + k], aqk = A[q * n + k];
          A[p * n + k] = c * apk - s * aqk;
          A[q * n + k] = s * apk + c * aqk;
        }
        A[p * n + q] = 0.0;
        A[q * n + p] = 0.0;
        for (int k = 0; k < n; ++k) { /* V <- V J */
          double vkp = evecs[k * n + p], vkq = evecs[k * n + q];
          evecs[k * n + p] = c * vkp - s * vkq;
          evecs[k * n + q] = s * vkp + c * vkq;
        }
      }
    }
  }
  /* sort eigenpairs by eigenvalue, descending (selection sort, stable) */
  for (int i = 0; i < n; ++i) evals[i] = A[i * n + i];
  for (int i = 0; i < n; ++i) {
    int best = i;
    for (int j = i + 1; j < n; ++j)
      if (evals[j] > evals[best]) best = j;
    if (best != i) {
      double tv = evals[i]; evals[i] = evals[best]; evals[best] = tv;
      for (int k = 0; k < n; ++k) {
        double tmp = evecs[k * n + i];
        evecs[k * n + i] = evecs[k * n + best];
        evecs[k * n + best] = tmp;
      }
    }
  }
  return sweep;
}

/* ------------------------------------------------------------------------ */
/* Fast PDDP query grouping (aiwillknow analysis, step 1 / Fig. 6 left):    */
/* project on the principal direction, split at the (tile-rounded) median,  */
/* recurse until every leaf is one tile of g queries.                       */
/* ------------------------------------------------------------------------ */

typedef struct { double p; int32_t tok; } proj_t;

static int cmp_proj(const void* a, const void* b) {
  const proj_t* x = (const proj_t*)a;
  const proj_t* y = (const proj_t*)b;
  if (x->p < y->p) return -1;
  if (x->p > y->p) return 1;
  return (x->tok > y->tok) - (x->tok < y->tok);
}

static int cmp_i32(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/* number of queries the left child receives when a node of n queries splits */
int orc_pddp_left_size(int n, int g) {
  int T = (n + g - 1) / g;
  return ((T + 1) / 2) * g;
}

/* The node's rows widened to fp64 (and, for the whitened grouping, each
   channel e multiplied by wscale[e]), their mean mu, and the scatter matrix
   C = sum_i (q_i - mu)(q_i - mu)^T (row-major d x d). */
static void node_moments(const uint16_t* x, long stride, int d, const double* wscale, const int32_t* members,
                         int n, double* rows, double* mu, double* C) {
  for (int i = 0; i < n; ++i) {
    double* r = rows + (size_t)i * d;
    load_row(x, stride, d, members[i], r);
    if (wscale)
      for (int e = 0; e < d; ++e) r[e] *= wscale[e];
  }
  /* centre: mu = mean of the node's queries */
  for (int i = 0; i < n; ++i)
    for (int e = 0; e < d; ++e) mu[e] += rows[(size_t)i * d + e];
  for (int e = 0; e < d; ++e) mu[e] /= (double)n;
  /* scatter matrix C = sum_i (q_i - mu)(q_i - mu)^T */
  for (int i = 0; i < n; ++i) {
    const double* r = rows + (size_t)i * d;
    for (int a = 0; a < d; ++a) {
      double ca = r[a] - mu[a];
      for (int b = 0; b < d; ++b) C[a * d + b] += ca * (r[b] - mu[b]);
    }
  }
}

/* Split along the direction in column 0 of V (row-major d x d): orient it so
   that its largest-magnitude entry (lowest index on ties) is positive, project
   the centred rows, and send the L smallest (projection, token) left. */
static void split_along_column0(const double* V, int d, const double* rows, const double* mu,
                                const int32_t* members, int n, int g, int32_t* left, int32_t* right, double* dir,
                                double* proj, double* split_p) {
  proj_t* pr = (proj_t*)malloc(sizeof(proj_t) * (size_t)n);
  int kmax = 0;
  for (int k = 1; k < d; ++k)
    if (fabs(V[k * d + 0]) > fabs(V[kmax * d + 0])) kmax = k;
  double sgn = V[kmax * d + 0] < 0.0 ? -1.0 : 1.0;
  for (int i = 0; i < n; ++i) {
    const double* r = rows + (size_t)i * d;
    double p = 0.0;
    for (int e = 0; e < d; ++e) p += (r[e] - mu[e]) * (sgn * V[e * d + 0]);
    pr[i].p = p;
    pr[i].tok = members[i];
    if (proj) proj[i] = p;
  }
  if (dir)
    for (int e = 0; e < d; ++e) dir[e] = sgn * V[e * d + 0];
  /* median split: the L smallest (projection, token) go left */
  qsort(pr, (size_t)n, sizeof(proj_t), cmp_proj);
  int L = orc_pddp_left_size(n, g);
  if (split_p) *split_p = pr[L - 1].p;
  for (int i = 0; i < L; ++i) left[i] = pr[i].tok;
  for (int i = L; i < n; ++i) right[i - L] = pr[i].tok;
  qsort(left, (size_t)L, sizeof(int32_t), cmp_i32);
  qsort(right, (size_t)(n - L), sizeof(int32_t), cmp_i32);
  free(pr);
}

/*
 * Split one node. `members` (n tokens) is the node's query set. Writes the
 * left child's L = orc_pddp_left_size(n, g) tokens to `left` and the other
 * n - L to `right`, each in ascending token order. Optional outputs: `dir`
 * (d, the oriented principal direction), `proj` (n, projection of members[i]),
 * `split_p` (the largest left projection), `eig` (2: the two largest
 * eigenvalues of the scatter matrix). Returns 0, or -1 if Jacobi failed.
 */
static int pddp_split_impl(const uint16_t* x, long stride, int d, const double* wscale, const int32_t* members,
                           int n, int g, int32_t* left, int32_t* right, double* dir, double* proj, double* split_p,
                           double* eig) {
  double* rows = (double*)malloc(sizeof(double) * (size_t)n * d);
  double* mu = (double*)calloc((size_t)d, sizeof(double));
  double* C = (double*)calloc((size_t)d * d, sizeof(double));
  double* ev = (double*)malloc(sizeof(double) * (size_t)d);
  double* V = (double*)malloc(sizeof(double) * (size_t)d * d);
  int rc = 0;
  node_moments(x, stride, d, wscale, members, n, rows, mu, C);
  if (orc_jacobi_eigh(d, C, ev, V, 1e-14, 200) < 0) rc = -1;
  /* principal direction = eigenvector of the largest eigenvalue (column 0) */
  if (eig) { eig[0] = ev[0]; eig[1] = d > 1 ? ev[1] : 0.0; }
  split_along_column0(V, d, rows, mu, members, n, g, left, right, dir, proj, split_p);
  free(rows); free(mu); free(C); free(ev); free(V);
  return rc;
}

int orc_pddp_split(const uint16_t* x, long stride, int d, const int32_t* members, int n, int g, int32_t* left,
                   int32_t* right, double* dir, double* proj, double* split_p, double* eig) {
  return pddp_split_impl(x, stride, d, NULL, members, n, g, left, right, dir, proj, split_p, eig);
}

/*
 * Whitened grouping (the project README's TODO "whitening", read as
 * per-channel standardisation): wscale[e] = 1 / sigma_e, sigma_e the
 * population standard deviation of channel e over the head's N queries (mean
 * first, then the mean squared deviation, both in fp64), or 1 for a constant
 * channel. orc_pddp_split_w is orc_pddp_split on the queries with channel e
 * multiplied by wscale[e]; `dir` and `proj` are in the whitened coordinates.
 */
void orc_channel_scale(const uint16_t* x, long stride, int d, int N, double* wscale) {
  for (int e = 0; e < d; ++e) {
    double mu = 0.0, var = 0.0;
    for (int i = 0; i < N; ++i) mu += orc_bf16_to_f64(x[(long)i * stride + e]);
    mu /= (double)N;
    for (int i = 0; i < N; ++i) {
      double t = orc_bf16_to_f64(x[(long)i * stride + e]) - mu;
      var += t * t;
    }
    double sigma = sqrt(var / (double)N);
    wscale[e] = sigma > 0.0 ? 1.0 / sigma : 1.0;
  }
}

int orc_pddp_split_w(const uint16_t* x, long stride, int d, const double* wscale, const int32_t* members, int n,
                     int g, int32_t* left, int32_t* right, double* dir, double* proj, double* split_p, double* eig) {
  return pddp_split_impl(x, stride, d, wscale, members, n, g, left, right, dir, proj, split_p, eig);
}

/* ------------------------------------------------------------------------ */
/* "Fast" PDDP: the split direction from a k-dimensional Krylov space       */
/* ------------------------------------------------------------------------ */

/*
 * Output number `index` (1, 2, ...) of the SplitMix64 generator started from
 * state 0 (S. Vigna's published generator: the state advances by the constant
 * 0x9E3779B97F4A7C15 and each output is the state passed through the
 * xor-shift-multiply finalizer below).
 */
uint64_t orc_splitmix64(uint64_t index) {
  uint64_t z = index * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/*
 * As orc_pddp_split, but the direction is the top Ritz vector of the scatter
 * matrix C on the Krylov space K_k(C, v0) = span(v0, C v0, ..., C^(k-1) v0),
 * v0[e] = 1 + (splitmix64(e + 1) >> 11) * 2^-53 normalised (the method's
 * "fast" variant: a fixed number of Krylov steps; the pages give no count).
 * Rayleigh-Ritz: an orthonormal basis of the space by Gram-Schmidt (two
 * passes per vector; the space ends early once a new vector's norm falls to
 * 1e-13 * trace(C)), H = V^T C V, its top eigenvector y by Jacobi, direction
 * V y. Returns 0, or -1 if Jacobi failed.
 */
int orc_pddp_split_krylov(const uint16_t* x, long stride, int d, const int32_t* members, int n, int g, int k,
                          int32_t* left, int32_t* right, double* dir, double* proj, double* split_p) {
  double* rows = (double*)malloc(sizeof(double) * (size_t)n * d);
  double* mu = (double*)calloc((size_t)d, sizeof(double));
  double* C = (double*)calloc((size_t)d * d, sizeof(double));
  double* B = (double*)calloc((size_t)k * d, sizeof(double));   /* basis vectors as rows */
  double* CB = (double*)calloc((size_t)k * d, sizeof(double));  /* C times each basis vector */
  double* w = (double*)malloc(sizeof(double) * (size_t)d);
  int rc = 0;
  node_moments(x, stride, d, NULL, members, n, rows, mu, C);
  double tr = 0.0;
  for (int e = 0; e < d; ++e) tr += C[e * d + e];
  double nv = 0.0;
  for (int e = 0; e < d; ++e) {
    B[e] = 1.0 + (double)(orc_splitmix64((uint64_t)e + 1) >> 11) * 0x1.0p-53;
    nv += B[e] * B[e];
  }
  for (int e = 0; e < d; ++e) B[e] /= sqrt(nv);
  int m = 1;
  for (int j = 1; j < k && j < d; ++j) {
    /* w = C b_{j-1}, then orthogonalised twice against b_0 .. b_{j-1} */
    for (int a = 0; a < d; ++a) {
      double t = 0.0;
      for (int e = 0; e < d; ++e) t += C[a * d + e] * B[(size_t)(j - 1) * d + e];
      w[a] = t;
    }
    for (int pass = 0; pass < 2; ++pass)
      for (int i = 0; i < j; ++i) {
        double c = 0.0;
        for (int e = 0; e < d; ++e) c += w[e] * B[(size_t)i * d + e];
        for (int e = 0; e < d; ++e) w[e] -= c * B[(size_t)i * d + e];
      }
    double nw = 0.0;
    for (int e = 0; e < d; ++e) nw += w[e] * w[e];
    nw = sqrt(nw);
    if (nw <= 1e-13 * tr) break;
    for (int e = 0; e < d; ++e) B[(size_t)j * d + e] = w[e] / nw;
    m = j + 1;
  }
  /* Rayleigh-Ritz on span(b_0 .. b_{m-1}) */
  for (int i = 0; i < m; ++i)
    for (int a = 0; a < d; ++a) {
      double t = 0.0;
      for (int e = 0; e < d; ++e) t += C[a * d + e] * B[(size_t)i * d + e];
      CB[(size_t)i * d + a] = t;
    }
  double* H = (double*)malloc(sizeof(double) * (size_t)m * m);
  double* hev = (double*)malloc(sizeof(double) * (size_t)m);
  double* Y = (double*)malloc(sizeof(double) * (size_t)m * m);
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < m; ++j) {
      double t = 0.0;
      for (int e = 0; e < d; ++e) t += B[(size_t)i * d + e] * CB[(size_t)j * d + e];
      H[i * m + j] = t;
    }
  for (int i = 0; i < m; ++i)  /* symmetrise the rounding of V^T C V */
    for (int j = i + 1; j < m; ++j) H[i * m + j] = H[j * m + i] = 0.5 * (H[i * m + j] + H[j * m + i]);
  if (orc_jacobi_eigh(m, H, hev, Y, 1e-14, 200) < 0) rc = -1;
  double* V = (double*)calloc((size_t)d * d, sizeof(double));  /* the direction in column 0 */
  double nx = 0.0;
  for (int e = 0; e < d; ++e) {
    double t = 0.0;
    for (int i = 0; i < m; ++i) t += B[(size_t)i * d + e] * Y[i * m + 0];
    V[e * d + 0] = t;
    nx += t * t;
  }
  for (int e = 0; e < d; ++e) V[e * d + 0] /= sqrt(nx);
  split_along_column0(V, d, rows, mu, members, n, g, left, right, dir, proj, split_p);
  free(rows); free(mu); free(C); free(B); free(CB); free(w); free(H); free(hev); free(Y); free(V);
  return rc;
}

static int pddp_krylov_rec(const uint16_t* x, long stride, int d, int32_t* seg, int n, int g, int k) {
  if ((n + g - 1) / g <= 1) return 0;
  int L = orc_pddp_left_size(n, g);
  int32_t* lt = (int32_t*)malloc(sizeof(int32_t) * (size_t)L);
  int32_t* rt = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n - L));
  int rc = orc_pddp_split_krylov(x, stride, d, seg, n, g, k, lt, rt, NULL, NULL, NULL);
  memcpy(seg, lt, sizeof(int32_t) * (size_t)L);
  memcpy(seg + L, rt, sizeof(int32_t) * (size_t)(n - L));
  free(lt);
  free(rt);
  rc |= pddp_krylov_rec(x, stride, d, seg, L, g, k);
  rc |= pddp_krylov_rec(x, stride, d, seg + L, n - L, g, k);
  return rc;
}

/* Full "fast" grouping of one head with k Krylov steps per node (layout as orc_pddp). */
int orc_pddp_krylov(const uint16_t* x, long stride, int d, int N, int g, int k, int32_t* perm) {
  for (int i = 0; i < N; ++i) perm[i] = i;
  return pddp_krylov_rec(x, stride, d, perm, N, g, k);
}

static int pddp_rec(const uint16_t* x, long stride, int d, const double* wscale, int32_t* seg, int n, int g,
                    double* gaps, int* ngaps, int max_gaps) {
  if ((n + g - 1) / g <= 1) return 0; /* a leaf: one tile, ascending tokens */
  int L = orc_pddp_left_size(n, g);
  int32_t* left = (int32_t*)malloc(sizeof(int32_t) * (size_t)L);
  int32_t* right = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n - L));
  double eig[2];
  int rc = pddp_split_impl(x, stride, d, wscale, seg, n, g, left, right, NULL, NULL, NULL, eig);
  if (gaps && *ngaps < max_gaps) gaps[(*ngaps)++] = eig[0] > 0.0 ? (eig[0] - eig[1]) / eig[0] : 0.0;
  memcpy(seg, left, sizeof(int32_t) * (size_t)L);
  memcpy(seg + L, right, sizeof(int32_t) * (size_t)(n - L));
  free(left);
  free(right);
  rc |= pddp_rec(x, stride, d, wscale, seg, L, g, gaps, ngaps, max_gaps);
  rc |= pddp_rec(x, stride, d, wscale, seg + L, n - L, g, gaps, ngaps, max_gaps);
  return rc;
}

/*
 * Full grouping of one head: perm[0..N) lists the leaves depth first (left
 * before right); group j is perm[j*g .. min((j+1)*g, N)). `gaps` (optional,
 * up to max_gaps entries, preorder) receives each internal node's relative
 * eigengap (l1 - l2) / l1. Returns 0 on success.
 */
int orc_pddp(const uint16_t* x, long stride, int d, int N, int g, int32_t* perm, double* gaps, int max_gaps) {
  for (int i = 0; i < N; ++i) perm[i] = i;
  int ng = 0;
  return pddp_rec(x, stride, d, NULL, perm, N, g, gaps, &ng, max_gaps);
}

/* orc_pddp on the whitened queries (wscale from orc_channel_scale). */
int orc_pddp_w(const uint16_t* x, long stride, int d, const double* wscale, int N, int g, int32_t* perm) {
  for (int i = 0; i < N; ++i) perm[i] = i;
  int ng = 0;
  return pddp_rec(x, stride, d, wscale, perm, N, g, NULL, &ng, 0);
}

/* ------------------------------------------------------------------------ */
/* Attention pieces (aiwillknow analysis, steps 2-4; paper Abstract)        */
/* ------------------------------------------------------------------------ */

static double dot_row(const double* qi, const uint16_t* k, long stride, int d, int j) {
  const uint16_t* r = k + (long)j * stride;
  double s = 0.0;
  for (int e = 0; e < d; ++e) s += qi[e] * orc_bf16_to_f64(r[e]);
  return s;
}

/*
 * Attention of query rows `rows` over the key set `keys` (nk tokens; NULL
 * means all N tokens in order): s_ij = scale * q_i . k_j,
 * lse_i = log sum_j exp(s_ij) (max subtracted first),
 * o_i = sum_j exp(s_ij - lse_i) v_j. Outputs o (nrows x d) and lse (nrows,
 * optional).
 */
int orc_attention_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, long stride, int d, int N,
                       double scale, const int32_t* rows, int nrows, const int32_t* keys, int nk, double* o,
                       double* lse) {
  if (!keys) nk = N;
  double* qi = (double*)malloc(sizeof(double) * (size_t)d);
  double* s = (double*)malloc(sizeof(double) * (size_t)nk);
  for (int r = 0; r < nrows; ++r) {
    load_row(q, stride, d, rows[r], qi);
    double m = -INFINITY;
    for (int t = 0; t < nk; ++t) {
      int j = keys ? keys[t] : t;
      s[t] = scale * dot_row(qi, k, stride, d, j);
      if (s[t] > m) m = s[t];
    }
    double l = 0.0;
    for (int t = 0; t < nk; ++t) l += exp(s[t] - m);
    double ls = m + log(l);
    if (lse) lse[r] = ls;
    double* orow = o + (size_t)r * d;
    for (int e = 0; e < d; ++e) orow[e] = 0.0;
    for (int t = 0; t < nk; ++t) {
      int j = keys ? keys[t] : t;
      double p = exp(s[t] - ls);
      const uint16_t* vr = v + (long)j * stride;
      for (int e = 0; e < d; ++e) orow[e] += p * orc_bf16_to_f64(vr[e]);
    }
  }
  free(qi);
  free(s);
  return 0;
}

/*
 * Group attention mass (aiwillknow analysis, step 2): for the group's query
 * rows and every key j, m(j) = sum_i exp(s_ij - lse_i), with lse_i the dense
 * log-sum-exp of row i (recomputed here exactly). mass has N entries.
 */
int orc_group_mass(const uint16_t* q, const uint16_t* k, long stride, int d, int N, double scale,
                   const int32_t* rows, int nrows, double* mass) {
  double* qi = (double*)malloc(sizeof(double) * (size_t)d);
  double* s = (double*)malloc(sizeof(double) * (size_t)N);
  for (int j = 0; j < N; ++j) mass[j] = 0.0;
  for (int r = 0; r < nrows; ++r) {
    load_row(q, stride, d, rows[r], qi);
    double m = -INFINITY;
    for (int j = 0; j < N; ++j) {
      s[j] = scale * dot_row(qi, k, stride, d, j);
      if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int j = 0; j < N; ++j) l += exp(s[j] - m);
    double ls = m + log(l);
    for (int j = 0; j < N; ++j) mass[j] += exp(s[j] - ls);
  }
  free(qi);
  free(s);
  return 0;
}

typedef struct { double m; int32_t j; } mass_t;

static int cmp_mass_desc(const void* a, const void* b) {
  const mass_t* x = (const mass_t*)a;
  const mass_t* y = (const mass_t*)b;
  if (x->m > y->m) return -1;
  if (x->m < y->m) return 1;
  return (x->j > y->j) - (x->j < y->j);
}

/*
 * Token-level top-K (aiwillknow analysis, step 2; paper Table 4 "token"
 * granularity): the K keys of largest mass, ties to the lower index, written
 * to idx in ascending index order.
 */
int orc_topk(const double* mass, int N, int K, int32_t* idx) {
  if (K < 0 || K > N) return -1;
  mass_t* a = (mass_t*)malloc(sizeof(mass_t) * (size_t)N);
  for (int j = 0; j < N; ++j) { a[j].m = mass[j]; a[j].j = j; }
  qsort(a, (size_t)N, sizeof(mass_t), cmp_mass_desc);
  for (int t = 0; t < K; ++t) idx[t] = a[t].j;
  qsort(idx, (size_t)K, sizeof(int32_t), cmp_i32);
  free(a);
  return 0;
}

/*
 * Anchor step for one query group (aiwillknow analysis, steps 2-3; paper
 * Abstract): dense output and lse, group mass, top-K keys, sparse output over
 * the K keys (renormalised), residual R = O_dense - O_sparse.
 * Outputs (all optional except idx): o_dense, o_sparse, resid (nrows x d),
 * lse (nrows), mass (N), idx (K, ascending).
 */
int orc_anchor_group(const uint16_t* q, const uint16_t* k, const uint16_t* v, long stride, int d, int N,
                     double scale, const int32_t* rows, int nrows, int K, double* o_dense, double* o_sparse,
                     double* resid, double* lse, double* mass, int32_t* idx) {
  size_t od = (size_t)nrows * d;
  double* od_ = o_dense ? o_dense : (double*)malloc(sizeof(double) * od);
  double* os_ = o_sparse ? o_sparse : (double*)malloc(sizeof(double) * od);
  double* m_ = mass ? mass : (double*)malloc(sizeof(double) * (size_t)N);
  orc_attention_rows(q, k, v, stride, d, N, scale, rows, nrows, NULL, 0, od_, lse);
  orc_group_mass(q, k, stride, d, N, scale, rows, nrows, m_);
  int rc = orc_topk(m_, N, K, idx);
  orc_attention_rows(q, k, v, stride, d, N, scale, rows, nrows, idx, K, os_, NULL);
  if (resid)
    for (size_t t = 0; t < od; ++t) resid[t] = od_[t] - os_[t];
  if (!o_dense) free(od_);
  if (!o_sparse) free(os_);
  if (!mass) free(m_);
  return rc;
}

/*
 * Reuse step for one group (aiwillknow analysis, step 4): fresh Q/K/V,
 * the anchor's query group and key set, output = sparse attention + R.
 * resid may be NULL (no compensation). o: nrows x d.
 */
int orc_reuse_group(const uint16_t* q, const uint16_t* k, const uint16_t* v, long stride, int d, int N,
                    double scale, const int32_t* rows, int nrows, const int32_t* idx, int K, const double* resid,
                    double* o) {
  orc_attention_rows(q, k, v, stride, d, N, scale, rows, nrows, idx, K, o, NULL);
  if (resid)
    for (size_t t = 0; t < (size_t)nrows * d; ++t) o[t] += resid[t];
  return 0;
}

/*
 * Round doubles to bf16 bit patterns, round to nearest, ties to even, in one
 * step (no intermediate float rounding). Used to store the oracle's residual
 * in the metadata's bf16 format.
 */
void orc_round_bf16(const double* x, long n, uint16_t* out) {
  for (long i = 0; i < n; ++i) {
    double v = x[i];
    if (v == 0.0 || !isfinite(v)) {
      float f = (float)v;
      uint32_t u;
      memcpy(&u, &f, 4);
      out[i] = (uint16_t)(u >> 16);
      continue;
    }
    int e;
    double m = frexp(v, &e);           /* v = m * 2^e, 0.5 <= |m| < 1 */
    double r = nearbyint(m * 256.0);   /* 8 significant bits, ties to even */
    float f = (float)ldexp(r / 256.0, e);
    uint32_t u;
    memcpy(&u, &f, 4);
    out[i] = (uint16_t)(u >> 16);
  }
}
