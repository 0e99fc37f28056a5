// Fast PDDP query grouping (aiwillknow analysis, step 1; paper Fig. 6 left):
// recursive median splits along the principal direction, down to 128-query
// groups. Everything that decides the split runs in fp64.
//
// The tree's shape depends only on N: a node of n queries and T = ceil(n/128)
// tiles sends ceil(T/2)*128 queries left. So the host lists each level's
// internal nodes once, and every level runs for all B*H heads at once:
//   pddp_cov_partial  raw moments sum(x), sum(x x^T) of chunks of at most 2048
//                     rows: the root's rows at level 0, then each parent's
//                     right (smaller) child's rows
//   pddp_node         one CTA per (head, node): raw moments (a right child sums
//                     its chunks; a left child takes its parent's moments minus
//                     its sibling's chunks, so only half the rows of a level are
//                     read for moments), scatter matrix C, top eigenvector
//                     by Lanczos with full reorthogonalisation (restarted), the
//                     sign rule (largest |v_k| positive, lowest k on ties),
//                     projections p_i = (x_i - mu).v, an exact radix select of
//                     the L-th smallest (p, position), and a stable partition of
//                     the node's members into the next level's permutation.
// Members of a node stay in ascending token order (every partition is stable
// and the root starts as the identity), so position order is token order.
//
// Whitened grouping (the README TODO's "whitening", read as per-channel
// standardisation of each head's queries): pddp_channel_scale computes, per
// (batch, head), w_c = 1/sigma_c with sigma_c the standard deviation of channel
// c over the head's N queries (w_c = 1 for a constant channel). PDDP on the
// whitened queries x' = W x (W = diag(w)) has the scatter matrix W C W, whose
// top eigenvector v' is oriented by the same sign rule, and the projections
// (x' - mu').v' = (x - mu).(W v'): each node scales its scatter matrix and its
// projection direction and is otherwise unchanged.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <vector>

#include "mcs_ptx.cuh"

namespace mcs {

namespace {

constexpr int kPddpThreads = 256;
constexpr int kPddpWarps = kPddpThreads / 32;
constexpr int kChunkRows = 2048;
// Lanczos cycles of at most kKrylovMax steps, each restarted from the previous
// cycle's Ritz vector. One cycle suffices for almost every node; a top
// eigenvalue inside a tight cluster (relative gap ~1e-3 with dozens of
// eigenvalues just below) can take three or four.
constexpr int kLanczosCycles = 8;
// Convergence checks at steps 47, 63, ... Measured on the Wan-14B and 3-D asset
// workloads: nodes converge after 42-43 steps on average (checking every 4
// steps from step 23), but each check (multisection of the tridiagonal's top
// eigenvalue, inverse iteration) costs several steps, and that schedule took
// 108 ms per grouping against 82 ms for this one (49 steps on average).
constexpr int kKrylovMax = kPddpKrylovMax;  // basis vectors per Lanczos cycle (shared memory); a cycle
                                            // that ends unconverged restarts from its Ritz vector
constexpr int kFirstCheck = 47;  // first Lanczos step with a convergence check
constexpr int kCheckEvery = 16;  // steps between later checks
constexpr int kStageRows = 32;
constexpr int kRankSelectMax = 768;  // nodes up to this size select the split key by direct ranks
constexpr int kSelUnroll = 4;        // key loads in flight per thread in the select and partition sweeps

// An internal node of the tree: members cur[off .. off + n), of which the
// first L go left. Its raw moments (sum x, sum x x^T) come from the chunks
// [chunk0, chunk0 + nchunk) of its level: the node's own rows (derive == 0),
// or its right sibling's rows, subtracted from the moments of its parent,
// node `parent` of the previous level (derive == 1).
struct Node {
  int off, n, L;
  int chunk0, nchunk;
  int derive, parent;
};

// Rows cur[off + r0 .. off + r1) of one head, whose raw moments one CTA sums.
struct Chunk {
  int off, r0, r1;
};

__host__ __device__ inline int tiles_of(int n) { return (n + MCS_GROUP_SIZE - 1) / MCS_GROUP_SIZE; }
__host__ __device__ inline int left_size(int n) { return ((tiles_of(n) + 1) / 2) * MCS_GROUP_SIZE; }

// The whole plan of a grouping of N queries (it depends only on N), written
// identically by the host (for launch sizes) and by the device (the tables the
// kernels read). Level 0 holds the root, whose moments are summed from chunks
// of all N rows. Each deeper level holds the internal children of the
// previous level's nodes, left before right; for every parent with an
// internal child, the chunks cover the RIGHT child's rows (the smaller half,
// a leaf or not): the right child sums them, the left child subtracts them
// from its parent's moments. lvl_node[l] / lvl_chunk[l] index the first node
// / chunk of level l; entries [nlevels] close the last level. Returns nlevels.
__host__ __device__ inline int build_plan(int N, Node* nodes, Chunk* chunks, int* lvl_node, int* lvl_chunk) {
  int nn = 0, nc = 0;
  lvl_node[0] = 0;
  lvl_chunk[0] = 0;
  if (tiles_of(N) <= 1) return 0;
  Node root{0, N, left_size(N), 0, 0, 0, -1};
  for (int r = 0; r < N; r += kChunkRows) chunks[nc++] = Chunk{0, r, r + kChunkRows < N ? r + kChunkRows : N};
  root.nchunk = nc;
  nodes[nn++] = root;
  int nl = 1, lo = 0, hi = nn;
  for (;;) {
    lvl_node[nl] = nn;
    lvl_chunk[nl] = nc;
    for (int i = lo; i < hi; ++i) {
      const Node p = nodes[i];
      const int nL = p.L, nR = p.n - p.L;
      const bool left_int = tiles_of(nL) >= 2, right_int = tiles_of(nR) >= 2;
      if (!left_int && !right_int) continue;
      const int c0 = nc - lvl_chunk[nl];
      for (int r = 0; r < nR; r += kChunkRows) chunks[nc++] = Chunk{p.off + nL, r, r + kChunkRows < nR ? r + kChunkRows : nR};
      const int cn = nc - lvl_chunk[nl] - c0;
      if (left_int) nodes[nn++] = Node{p.off, nL, left_size(nL), c0, cn, 1, i - lo};
      if (right_int) nodes[nn++] = Node{p.off + nL, nR, left_size(nR), c0, cn, 0, -1};
    }
    if (nn == lvl_node[nl]) return nl;
    lo = hi;
    hi = nn;
    ++nl;
  }
}

// bounds for the plan's tables: internal nodes < leaves; per level at most one
// chunk per parent plus one per kChunkRows rows
__host__ __device__ inline int plan_max_nodes(int N) { return tiles_of(N) + 1; }
__host__ __device__ inline int plan_max_chunks(int N) { return tiles_of(N) + 40 * (N / kChunkRows + 2); }
constexpr int kMaxLevels = 40;

struct LevelArgs {
  int B, H, N, nnodes, nchunks;
  const Node* nodes;
  const Chunk* chunks;
  const uint16_t* q;
  const int32_t* cur;  // [P, N]
  int32_t* nxt;        // [P, N]
  double* keys;        // [P, N]
  double* partial;     // [P, nchunks, pstride]
  const double* mom_in;  // [P, max_nodes, pstride]: raw moments of the previous level's nodes
  double* mom_out;       // [P, max_nodes, pstride]: raw moments of this level's nodes
  int max_nodes;
  int* status;
  int krylov_steps;    // 0: Lanczos to convergence; k > 0: the top Ritz vector after k steps
  const double* wscale;  // [P, D] channel scales of the whitened grouping, or null
};

template <int D>
struct PCfg {
  static constexpr int BLK = D / 16;                   // chunk partials: per-thread block of the d x d matrix
  static constexpr int PSTRIDE = D + D * (D + 1) / 2;  // sum(x) then packed upper sum(x x^T)
  static constexpr int VEC = kStageRows * D / (8 * kPddpThreads);  // 16-byte loads per thread per stage
  // Node kernel: thread t holds row t / TPR of the scatter matrix, columns
  // [CPT * (t % TPR), + CPT), so a matvec needs one shuffle per TPR step.
  static constexpr int TPR = kPddpThreads / D;
  static constexpr int CPT = D / TPR;
  // Krylov vectors in shared memory: TPV segments of EPT elements, each followed
  // by two doubles of padding (row stride VS). The Gram-Schmidt dot products
  // (TPV threads per basis vector, one segment each) and the matvec (TPR
  // segments per row) then read 16-byte pairs without bank conflicts.
  static constexpr int TPV = 4;
  static constexpr int EPT = D / TPV;
  static constexpr int VS = D + 2 * TPV;
  static_assert(kPddpThreads % D == 0 && EPT % 4 == 0 && CPT % EPT == 0, "node kernel layout");
};

// position of element c of a Krylov vector in the padded layout
template <int D>
__device__ __forceinline__ int vpos(int c) {
  return c + 2 * (c / PCfg<D>::EPT);
}

__device__ __forceinline__ int packed_index(int a, int b, int d) {  // a <= b
  return a * d - a * (a - 1) / 2 + (b - a);
}

__device__ __forceinline__ double bf16d(uint16_t x) {
  return static_cast<double>(__uint_as_float(static_cast<uint32_t>(x) << 16));
}

// Register prefetch of one stage (kStageRows rows of the node, tokens from cur).
template <int D>
__device__ __forceinline__ void load_stage(uint4 (&reg)[PCfg<D>::VEC], const uint16_t* q, const int32_t* cur,
                                           int r0, int cnt, int b, int h, int N, int H) {
#pragma unroll
  for (int v = 0; v < PCfg<D>::VEC; ++v) {
    const int e = (v * kPddpThreads + threadIdx.x) * 8;
    const int r = e / D, c = e % D;
    uint4 x = make_uint4(0, 0, 0, 0);
    if (r < cnt) {
      const int tok = cur[r0 + r];
      x = __ldg(reinterpret_cast<const uint4*>(q + ((static_cast<size_t>(b) * N + tok) * H + h) * D + c));
    }
    reg[v] = x;
  }
}

template <int D>
__device__ __forceinline__ void store_stage(double* X, const uint4 (&reg)[PCfg<D>::VEC]) {
#pragma unroll
  for (int v = 0; v < PCfg<D>::VEC; ++v) {
    const int e = (v * kPddpThreads + threadIdx.x) * 8;
    const uint16_t* hv = reinterpret_cast<const uint16_t*>(&reg[v]);
#pragma unroll
    for (int i = 0; i < 8; ++i) X[e + i] = bf16d(hv[i]);
  }
}

// Raw moments of rows [r0, r1): acc[i][j] += x_a x_b with a = ti + 16 i and
// b = tj + 16 j (ti = tid / 16, tj = tid % 16), s1 += x_t for threads t < D.
// Only blocks i <= j are accumulated: every entry a < b of the symmetric
// matrix lies in one of them (blocks i > j hold only entries a > b), and the
// diagonal blocks are computed whole. Stages are prefetched one ahead.
template <int D>
__device__ void accumulate_moments(double* X, const uint16_t* q, const int32_t* cur, int r0, int r1, int b, int h,
                                   int N, int H, double (&acc)[PCfg<D>::BLK][PCfg<D>::BLK], double& s1) {
  constexpr int BLK = PCfg<D>::BLK;
  const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
  uint4 reg[PCfg<D>::VEC];
  load_stage<D>(reg, q, cur, r0, min(kStageRows, r1 - r0), b, h, N, H);
  for (int base = r0; base < r1; base += kStageRows) {
    const int cnt = min(kStageRows, r1 - base);
    __syncthreads();
    store_stage<D>(X, reg);
    __syncthreads();
    if (base + kStageRows < r1) load_stage<D>(reg, q, cur, base + kStageRows, min(kStageRows, r1 - base - kStageRows), b, h, N, H);
#pragma unroll 2
    for (int r = 0; r < cnt; ++r) {
      double av[BLK], bv[BLK];
#pragma unroll
      for (int i = 0; i < BLK; ++i) {  // rows ti + 16 i, columns tj + 16 j: conflict-free reads
        av[i] = X[r * D + ti + 16 * i];
        bv[i] = X[r * D + tj + 16 * i];
      }
#pragma unroll
      for (int i = 0; i < BLK; ++i)
#pragma unroll
        for (int j = i; j < BLK; ++j) acc[i][j] = fma(av[i], bv[j], acc[i][j]);
      if (threadIdx.x < D) s1 += X[r * D + threadIdx.x];
    }
  }
  __syncthreads();
}

__device__ __forceinline__ uint64_t key_bits(double x) {
  x = x + 0.0;  // -0 -> +0
  uint64_t u = static_cast<uint64_t>(__double_as_longlong(x));
  return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Number of eigenvalues of the symmetric tridiagonal (al, be) below sigma: the
// sign changes along the leading principal minors p_i = det(T_i - sigma I),
// p_i = (al_i - sigma) p_{i-1} - be_{i-1}^2 p_{i-2} (p_{-1} = 1). A minor that
// is exactly zero counts as a change of sign. The pair (p_{i-1}, p_i) is
// rescaled when it leaves [1e-150, 1e150], which keeps every sign. This is the
// classic Sturm count without the division of its ratio form: the serial
// chain is one FMA per step instead of one fp64 division.
__device__ int sturm_count(const double* al, const double* be, int m, double sigma) {
  double pm1 = 1.0, p = al[0] - sigma;
  bool prev = p == 0.0 ? true : p < 0.0;
  int cnt = prev;
  for (int i = 1; i < m; ++i) {
    const double t = be[i - 1] * be[i - 1] * pm1;
    const double pn = fma(al[i] - sigma, p, -t);
    pm1 = p;
    p = pn;
    const double a = fabs(p);
    if (a > 1e150 || (a < 1e-150 && fabs(pm1) < 1e-150 && a != 0.0)) {
      const double sc = a > 1e150 ? 1e-150 : 1e150;
      p *= sc;
      pm1 *= sc;
    }
    const bool neg = p == 0.0 ? !prev : p < 0.0;
    cnt += neg != prev;
    prev = neg;
  }
  return cnt;
}

// Whole block: largest eigenvalue of the m x m tridiagonal by multisection.
// Each round splits the bracket [lo, hi] at 256 points, one Sturm count per
// thread; the lowest point with every eigenvalue below it bounds the top one
// from above. About seven rounds reach full double precision. Every thread
// must call it (it synchronises the block); all return the same value.
__device__ double tridiag_top_eigenvalue(const double* al, const double* be, int m, int* scratch,
                                         double* bracket) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    double lo = 1e308, hi = -1e308;
    for (int i = 0; i < m; ++i) {
      const double r = (i > 0 ? fabs(be[i - 1]) : 0.0) + (i < m - 1 ? fabs(be[i]) : 0.0);
      lo = fmin(lo, al[i] - r);
      hi = fmax(hi, al[i] + r);
    }
    const double pad = 1e-12 * fmax(fabs(lo), fabs(hi)) + 1e-300;
    bracket[0] = lo - pad;
    bracket[1] = hi + pad;
  }
  __syncthreads();
  double lo = bracket[0], hi = bracket[1];
  constexpr int kPts = kPddpThreads;
  for (int round = 0; round < 16; ++round) {
    const double w = (hi - lo) / (kPts + 1);
    const double x = lo + w * (tid + 1);
    const bool above = sturm_count(al, be, m, x) == m;  // x above the top eigenvalue
    const unsigned mask = __ballot_sync(0xffffffffu, above);
    if (lane == 0) scratch[warp] = mask ? warp * 32 + __ffs(mask) - 1 : kPts;
    __syncthreads();
    int first = kPts;
#pragma unroll
    for (int i = 0; i < kPddpWarps; ++i) first = min(first, scratch[i]);
    __syncthreads();  // scratch is rewritten next round
    const double nlo = first == 0 ? lo : lo + w * first;
    const double nhi = first == kPts ? hi : lo + w * (first + 1);
    if (nhi - nlo >= hi - lo) break;
    lo = nlo;
    hi = nhi;
    if (hi - lo <= 4e-16 * fmax(fabs(lo), fabs(hi))) break;
  }
  return 0.5 * (lo + hi);
}

// One whole warp: eigenvector of the m x m tridiagonal for eigenvalue theta,
// by inverse iteration. T - theta I is factored once (partial pivoting; row i
// swaps with i+1 when |sub-diagonal| > |pivot|) and the multipliers, swap
// flags and reciprocal pivots are kept, so the solves need no division. The
// serial steps (the factorisation, forward elimination, back substitution)
// run on lane 0; norms, scalings and the reciprocals on all lanes. theta comes
// from multisection to full precision, so two solves reach the eigenvector.
__device__ void tridiag_eigenvector(const double* al, const double* be, int m, double theta, double* y,
                                    double* dd, double* du, double* du2, double* rr, double* fm, int* piv) {
  const int lane = threadIdx.x & 31;
  double tnorm = 0.0;
  for (int i = lane; i < m; i += 32)
    tnorm = fmax(tnorm, fabs(al[i]) + (i ? fabs(be[i - 1]) : 0.0) + (i < m - 1 ? fabs(be[i]) : 0.0));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tnorm = fmax(tnorm, __shfl_xor_sync(0xffffffffu, tnorm, o));
  const double tiny = 1e-15 * tnorm + 1e-300;
  // factor: dd = pivots (then their reciprocals), du / du2 = first / second super-diagonals of U
  for (int i = lane; i < m; i += 32) {
    dd[i] = al[i] - theta;
    du[i] = i < m - 1 ? be[i] : 0.0;
    du2[i] = 0.0;
    y[i] = 1.0;
  }
  __syncwarp();
  if (lane == 0) {
    for (int i = 0; i < m - 1; ++i) {
      const double dl = be[i];
      if (fabs(dd[i]) >= fabs(dl)) {
        if (dd[i] == 0.0) dd[i] = tiny;
        const double f = dl / dd[i];
        dd[i + 1] -= f * du[i];
        fm[i] = f;
        piv[i] = 0;
      } else {
        const double f = dd[i] / dl;
        const double d1 = dd[i + 1], u1 = (i + 1 < m - 1) ? du[i + 1] : 0.0;
        dd[i] = dl;
        const double u0 = du[i];
        du[i] = d1;
        du2[i] = u1;
        dd[i + 1] = u0 - f * d1;
        if (i + 1 < m - 1) du[i + 1] = -f * u1;
        fm[i] = f;
        piv[i] = 1;
      }
    }
    if (dd[m - 1] == 0.0) dd[m - 1] = tiny;
  }
  __syncwarp();
  for (int i = lane; i < m; i += 32) dd[i] = 1.0 / dd[i];
  __syncwarp();
  for (int iter = 0; iter < 2; ++iter) {
    double nrm = 0.0;
    for (int i = lane; i < m; i += 32) nrm += y[i] * y[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nrm += __shfl_xor_sync(0xffffffffu, nrm, o);
    const double inv = 1.0 / sqrt(nrm);
    for (int i = lane; i < m; i += 32) rr[i] = y[i] * inv;
    __syncwarp();
    if (lane == 0) {
      for (int i = 0; i < m - 1; ++i) {  // the same row operations on the right-hand side
        if (piv[i]) {
          const double r0 = rr[i], r1 = rr[i + 1];
          rr[i] = r1;
          rr[i + 1] = r0 - fm[i] * r1;
        } else {
          rr[i + 1] -= fm[i] * rr[i];
        }
      }
      y[m - 1] = rr[m - 1] * dd[m - 1];
      if (m > 1) y[m - 2] = (rr[m - 2] - du[m - 2] * y[m - 1]) * dd[m - 2];
      for (int i = m - 3; i >= 0; --i) y[i] = (rr[i] - du[i] * y[i + 1] - du2[i] * y[i + 2]) * dd[i];
    }
    __syncwarp();
  }
  double nrm = 0.0;
  for (int i = lane; i < m; i += 32) nrm += y[i] * y[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nrm += __shfl_xor_sync(0xffffffffu, nrm, o);
  nrm = sqrt(nrm);
  for (int i = lane; i < m; i += 32) y[i] /= nrm;
  __syncwarp();
}

template <int D>
struct NodeSmem {
  // Krylov basis (KMAX rows); before it the node's raw moments, after it the
  // per-warp digit histograms (kPddpWarps x 2048 ints), whichever is largest
  static constexpr int KMAX = kKrylovMax < D ? kKrylovMax : D;
  static constexpr int VB = KMAX * PCfg<D>::VS;
  static constexpr int VSZ0 = VB > kPddpWarps * 2048 / 2 ? VB : kPddpWarps * 2048 / 2;
  static constexpr int VSZ = VSZ0 > PCfg<D>::PSTRIDE ? VSZ0 : PCfg<D>::PSTRIDE;
  double V[VSZ];
  double wv[2][PCfg<D>::VS];  // C v_j, then its Gram-Schmidt remainder (padded layout), double-buffered
  double mu[D], v0[D];
  double al[D], be[D], y[D];
  double tdd[D], tdu[D], tdu2[D], trr[D], tfm[D], coef[D];
  int tpiv[D];
  double red[kPddpWarps];
  int hist[2048];
  int wcnt[kPddpWarps][2];  // per warp segment: keys below T, keys equal to T
  int wleft[kPddpWarps], wright[kPddpWarps], weq[kPddpWarps];
  int iscal[8];
  double dscal[8];
  unsigned long long kscal;
  uint32_t tmem_slot;
};
// two node CTAs per SM: shared memory (and TMEM: 2 D columns each) for both
static_assert(sizeof(NodeSmem<128>) <= 110 * 1024 && sizeof(NodeSmem<64>) <= 110 * 1024, "node smem");

__device__ double block_sum(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int i = 0; i < kPddpWarps; ++i) t += red[i];
  return t;
}

// w = (C v) / div, row r of C in TMEM lane r (D doubles as 2D 32-bit columns,
// low word first), computed by threads r < D (whole warps); v and w in the
// padded layout.
template <int D>
__device__ __forceinline__ void tmem_matvec(uint32_t trow, const double* v, double* w, double div) {
  double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int cb = 0; cb < D / 32; ++cb) {  // 32 doubles (64 columns) per TMEM wait
    float u[64];
    tmem_ld32(trow + cb * 64, u);
    tmem_ld32(trow + cb * 64 + 32, u + 32);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 32; k += 2) {
      const double2 x = *reinterpret_cast<const double2*>(v + vpos<D>(cb * 32 + k));
      const double c0 = __hiloint2double(__float_as_int(u[2 * k + 1]), __float_as_int(u[2 * k]));
      const double c1 = __hiloint2double(__float_as_int(u[2 * k + 3]), __float_as_int(u[2 * k + 2]));
      acc[k & 7] = fma(c0, x.x, acc[k & 7]);
      acc[(k + 1) & 7] = fma(c1, x.y, acc[(k + 1) & 7]);
    }
  }
  const double t = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
  w[vpos<D>(threadIdx.x)] = div == 1.0 ? t : t / div;
}

}  // namespace

// Whitened grouping: w[(b,h), c] = 1 / sigma_c over the head's N queries
// (population standard deviation, two fp64 passes), 1 for a constant channel.
// One CTA per (b, h); kPddpThreads / D threads share a channel.
template <int D>
__global__ void __launch_bounds__(kPddpThreads) pddp_channel_scale(const uint16_t* q, int H, int N, double* w) {
  constexpr int R = kPddpThreads / D;  // threads per channel
  __shared__ double red[kPddpThreads];
  const int prob = blockIdx.x, b = prob / H, h = prob % H;
  const int c = threadIdx.x % D, r = threadIdx.x / D;
  const uint16_t* base = q + (static_cast<size_t>(b) * N * H + h) * D + c;
  const size_t stride = static_cast<size_t>(H) * D;
  double s = 0.0;
  for (int i = r; i < N; i += R) s += bf16d(base[i * stride]);
  red[threadIdx.x] = s;
  __syncthreads();
  double mu = 0.0;
  for (int k = 0; k < R; ++k) mu += red[k * D + c];
  mu /= N;
  __syncthreads();
  double v = 0.0;
  for (int i = r; i < N; i += R) {
    const double t = bf16d(base[i * stride]) - mu;
    v = fma(t, t, v);
  }
  red[threadIdx.x] = v;
  __syncthreads();
  if (r == 0) {
    double var = 0.0;
    for (int k = 0; k < R; ++k) var += red[k * D + c];
    const double sigma = sqrt(var / N);
    w[static_cast<size_t>(prob) * D + c] = sigma > 0.0 ? 1.0 / sigma : 1.0;
  }
}

template <int D>
__global__ void __launch_bounds__(kPddpThreads) pddp_cov_partial(const LevelArgs a) {
  constexpr int BLK = PCfg<D>::BLK;
  constexpr int PS = PCfg<D>::PSTRIDE;
  __shared__ double X[kStageRows * D];
  const int ci = blockIdx.x % a.nchunks;
  const int prob = blockIdx.x / a.nchunks;
  const int b = prob / a.H, h = prob % a.H;
  const Chunk ch = a.chunks[ci];
  const int32_t* cur = a.cur + static_cast<size_t>(prob) * a.N + ch.off;
  double acc[BLK][BLK];
#pragma unroll
  for (int i = 0; i < BLK; ++i)
#pragma unroll
    for (int j = 0; j < BLK; ++j) acc[i][j] = 0.0;
  double s1 = 0.0;
  accumulate_moments<D>(X, a.q, cur, ch.r0, ch.r1, b, h, a.N, a.H, acc, s1);
  double* out = a.partial + (static_cast<size_t>(prob) * a.nchunks + ci) * PS;
  if (threadIdx.x < D) out[threadIdx.x] = s1;
  const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
#pragma unroll
  for (int i = 0; i < BLK; ++i)
#pragma unroll
    for (int j = 0; j < BLK; ++j) {
      const int r = ti + 16 * i, c = tj + 16 * j;
      if (r <= c) out[D + packed_index(r, c, D)] = acc[i][j];
    }
}

template <int D>
__global__ void __launch_bounds__(kPddpThreads, 2) pddp_node(const LevelArgs a) {
  constexpr int PS = PCfg<D>::PSTRIDE;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  NodeSmem<D>& S = *reinterpret_cast<NodeSmem<D>*>(smem_raw);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ni = blockIdx.x % a.nnodes;
  const int prob = blockIdx.x / a.nnodes;
  const int b = prob / a.H, h = prob % a.H;
  const Node nd = a.nodes[ni];
  const int n = nd.n;
  const int32_t* cur = a.cur + static_cast<size_t>(prob) * a.N + nd.off;
  int32_t* nxt = a.nxt + static_cast<size_t>(prob) * a.N + nd.off;
  double* keys = a.keys + static_cast<size_t>(prob) * a.N + nd.off;

  // ---------------- 1. scatter matrix C = sum(x x^T) - n mu mu^T, kept in TMEM
  // Raw moments of the node, assembled in shared memory (coalesced reads): its
  // own chunks summed in a fixed order, or, for a left child, its parent's
  // moments minus its right sibling's chunks. Thread r < D then writes row r
  // of the symmetric matrix (fp64) to TMEM lane r, where the matvecs read it:
  // with C out of the register file, two nodes share an SM.
  using P = PCfg<D>;
  using SM = NodeSmem<D>;
  constexpr uint32_t kTmemCols = 2 * D;
  if (warp == 0) {
    tmem_alloc(&S.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  double* M = S.V;  // packed like a chunk partial: sum x, then the upper triangle of sum x x^T
  {
    const double* pm =
        nd.derive ? a.mom_in + (static_cast<size_t>(prob) * a.max_nodes + nd.parent) * PS : nullptr;
    const double sign = nd.derive ? -1.0 : 1.0;  // subtracted from the parent's, or summed
    const double* part = a.partial + (static_cast<size_t>(prob) * a.nchunks + nd.chunk0) * PS;
    for (int e = tid; e < PS; e += kPddpThreads) {
      double m = pm ? pm[e] : 0.0;
      for (int c = 0; c < nd.nchunk; ++c) m = fma(sign, part[static_cast<size_t>(c) * PS + e], m);
      M[e] = m;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t trow = S.tmem_slot + (static_cast<uint32_t>(32 * (warp & 3)) << 16);  // lane = row tid
  if (nd.L >= 2 * MCS_GROUP_SIZE) {  // the node's raw moments, for its left child at the next level
    double* om = a.mom_out + (static_cast<size_t>(prob) * a.max_nodes + ni) * PS;
    for (int e = tid; e < PS; e += kPddpThreads) om[e] = M[e];
  }
  if (tid < D) S.mu[tid] = M[tid] / n;
  __syncthreads();
  const double* wsc = a.wscale ? a.wscale + static_cast<size_t>(prob) * D : nullptr;
  double diag = 0.0;  // C[tid][tid]
  if (tid < D) {
    const int r = tid;
    const double mur = S.mu[r], wr = wsc ? wsc[r] : 1.0;
    for (int cb = 0; cb < D / 16; ++cb) {  // 16 doubles = 32 TMEM columns per store
      float u[32];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int c = cb * 16 + k;
        // n mu_r mu_c and w_r w_c as commutative products: C stays exactly symmetric
        double x = M[D + (r <= c ? packed_index(r, c, D) : packed_index(c, r, D))] -
                   static_cast<double>(n) * (mur * S.mu[c]);
        if (wsc) x *= wr * wsc[c];  // whitened grouping: W C W
        if (c == r) diag = x;
        u[2 * k] = __int_as_float(__double2loint(x));
        u[2 * k + 1] = __int_as_float(__double2hiint(x));
      }
      tmem_st32(trow + cb * 32, u);
    }
    tmem_wait_st();
  }
  __syncthreads();  // M is overwritten by the Krylov basis below

  // ---------------- 2. principal direction: Lanczos with full reorthogonalisation
  {  // trace(C) = sum of eigenvalues >= the top one: a scale for "beta is negligible"
    const double tr = block_sum(diag, S.red);
    if (tid == 0) S.dscal[3] = tr + 1e-300;
    __syncthreads();
  }
  if (tid < D) {  // deterministic start vector (splitmix-style hash of the index)
    uint64_t z = 0x9E3779B97F4A7C15ull * (tid + 1);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    S.v0[tid] = 1.0 + static_cast<double>(z >> 11) * 0x1.0p-53;
  }
  __syncthreads();
  {
    const double nv = block_sum(tid < D ? S.v0[tid] * S.v0[tid] : 0.0, S.red);
    if (tid < D) S.v0[tid] /= sqrt(nv);
    __syncthreads();
  }
  int steps_total = 0;  // Lanczos steps over all cycles (diagnostic counter)
  double* V = S.V;      // Krylov basis, row j = v_j in the padded layout (row stride VS)
  for (int cycle = 0; cycle < kLanczosCycles; ++cycle) {
    if (tid < D) V[vpos<D>(tid)] = S.v0[tid];
    __syncthreads();
    int m_used = SM::KMAX;
    bool converged = false;
    int wb = 0;  // S.wv[wb] holds C v_j
    if (tid < D) tmem_matvec<D>(trow, V, S.wv[0], 1.0);
    __syncthreads();
    for (int j = 0; j < SM::KMAX; ++j) {
      double* w = S.wv[wb];
      // two classical Gram-Schmidt passes against v_0 .. v_j; alpha_j is the v_j
      // coefficient; the second pass also yields |w|^2 for beta_j
      double alpha = 0.0;
      for (int pass = 0; pass < 2; ++pass) {
        {  // c_i = v_i . w: TPV threads per basis vector (one segment each), 64 vectors at a time
          const int q = tid % P::TPV;
          const double* ws = w + q * (P::EPT + 2);
          for (int i0 = 0; i0 <= j; i0 += kPddpThreads / P::TPV) {
            const int i = i0 + tid / P::TPV;
            double t = 0.0;
            if (i <= j) {
              const double* vi = V + i * P::VS + q * (P::EPT + 2);
              double a4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
              for (int k = 0; k < P::EPT; k += 2) {
                const double2 x = *reinterpret_cast<const double2*>(vi + k);
                const double2 y = *reinterpret_cast<const double2*>(ws + k);
                a4[k & 3] = fma(x.x, y.x, a4[k & 3]);
                a4[(k + 1) & 3] = fma(x.y, y.y, a4[(k + 1) & 3]);
              }
              t = (a4[0] + a4[1]) + (a4[2] + a4[3]);
            }
#pragma unroll
            for (int o = 1; o < P::TPV; o <<= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
            if (q == 0 && i <= j) S.coef[i] = t;
          }
        }
        __syncthreads();
        alpha += S.coef[j];
        double t = 0.0;
        if (tid < D) {  // w -= sum_i c_i v_i with four independent partial sums
          const int pc = vpos<D>(tid);
          double q4[4] = {0.0, 0.0, 0.0, 0.0};
          int i = 0;
          for (; i + 3 <= j; i += 4) {
            const double2 c01 = *reinterpret_cast<const double2*>(S.coef + i);
            const double2 c23 = *reinterpret_cast<const double2*>(S.coef + i + 2);
            q4[0] = fma(c01.x, V[i * P::VS + pc], q4[0]);
            q4[1] = fma(c01.y, V[(i + 1) * P::VS + pc], q4[1]);
            q4[2] = fma(c23.x, V[(i + 2) * P::VS + pc], q4[2]);
            q4[3] = fma(c23.y, V[(i + 3) * P::VS + pc], q4[3]);
          }
          for (; i <= j; ++i) q4[0] = fma(S.coef[i], V[i * P::VS + pc], q4[0]);
          t = w[pc] - ((q4[0] + q4[1]) + (q4[2] + q4[3]));
          w[pc] = t;
        }
        if (pass == 1) {
          double q2 = t * t;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) q2 += __shfl_xor_sync(0xffffffffu, q2, o);
          if (lane == 0) S.red[warp] = q2;
        }
        __syncthreads();
      }
      double wsq = 0.0;
#pragma unroll
      for (int i = 0; i < kPddpWarps; ++i) wsq += S.red[i];
      const double beta = sqrt(wsq);
      if (tid == 0) {
        S.al[j] = alpha;
        S.be[j] = beta;
      }
      const bool fixed_end = a.krylov_steps > 0 && j + 1 >= a.krylov_steps;
      const bool last = (j == SM::KMAX - 1) || beta <= 1e-13 * fabs(S.dscal[3]) || fixed_end;
      // convergence checks from step kFirstCheck on, every kCheckEvery steps
      if (last || (a.krylov_steps == 0 && j >= kFirstCheck && ((j - kFirstCheck) % kCheckEvery) == 0)) {
        __syncthreads();
        const double th = tridiag_top_eigenvalue(S.al, S.be, j + 1, S.iscal, S.dscal + 4);
        if (warp == 0) {
          tridiag_eigenvector(S.al, S.be, j + 1, th, S.y, S.tdd, S.tdu, S.tdu2, S.trr, S.tfm, S.tpiv);
          if (lane == 0) {
            S.dscal[0] = th;
            S.dscal[1] = beta * fabs(S.y[j]);
          }
        }
        __syncthreads();
        const double theta = S.dscal[0], resid = S.dscal[1];
        if (resid <= 1e-14 * fabs(theta) || last) {
          converged = resid <= 1e-12 * fabs(theta) || beta <= 1e-13 * fabs(S.dscal[3]) || fixed_end;
          m_used = j + 1;
          break;
        }
      }
      // v_{j+1} = w / beta, and C v_{j+1} (from w, divided by beta) into the other buffer
      if (tid < D) V[(j + 1) * P::VS + vpos<D>(tid)] = w[vpos<D>(tid)] / beta;
      if (tid < D) tmem_matvec<D>(trow, w, S.wv[wb ^ 1], beta);
      wb ^= 1;
      __syncthreads();
    }
    // Ritz vector x = V y
    double* x = S.wv[wb ^ 1];  // free: the last matvec wrote S.wv[wb]
    if (tid < D) {
      double t = 0.0;
      for (int i = 0; i < m_used; ++i) t = fma(V[i * P::VS + vpos<D>(tid)], S.y[i], t);
      x[tid] = t;
    }
    __syncthreads();
    const double nx = sqrt(block_sum(tid < D ? x[tid] * x[tid] : 0.0, S.red));
    if (tid < D) S.v0[tid] = x[tid] / nx;
    __syncthreads();
    steps_total += m_used;
    if (converged) break;
  }
  if (tid == 0 && a.status) {
    atomicAdd(a.status + MCS_SW_LANCZOS_STEPS, steps_total);
    atomicAdd(a.status + MCS_SW_LANCZOS_NODES, 1);
  }
  // orientation: the entry of largest magnitude (lowest index on ties) is positive
  if (tid == 0) {
    int kmax = 0;
    for (int k = 1; k < D; ++k)
      if (fabs(S.v0[k]) > fabs(S.v0[kmax])) kmax = k;
    S.dscal[2] = S.v0[kmax] < 0.0 ? -1.0 : 1.0;
  }
  __syncthreads();
  if (tid < D) S.v0[tid] *= S.dscal[2];
  __syncthreads();

  // ---------------- 3. projections p_i = (x_i - mu) . v
  // A warp takes 16 members at a time: lane u fetches the token of member
  // i0 + u one batch ahead, every lane loads its D/32 elements of the 16 rows,
  // and the 16 partial dot products are summed across the warp by recursive
  // halving (each step hands half of the open sums to the partner lane), two
  // shuffles per member instead of ten.
  {
    constexpr int PER = D / 32;  // elements per lane
    constexpr int kB = 16;       // members per warp per batch
    double vv[PER], mm[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      vv[e] = S.v0[lane * PER + e];
      if (wsc) vv[e] *= wsc[lane * PER + e];  // whitened: project along W v'
      mm[e] = S.mu[lane * PER + e];
    }
    const size_t row_stride = static_cast<size_t>(a.H) * D;
    const uint16_t* qh = a.q + (static_cast<size_t>(b) * a.N * a.H + h) * D + lane * PER;
    constexpr int kStep = kPddpWarps * kB;
    int tok_next = (lane < kB && warp * kB + lane < n) ? cur[warp * kB + lane] : 0;
    for (int i0 = warp * kB; i0 < n; i0 += kStep) {
      const int tok_l = tok_next;  // token of member i0 + lane (lanes < kB; 0 past the node)
      tok_next = (lane < kB && i0 + kStep + lane < n) ? cur[i0 + kStep + lane] : 0;
      uint16_t xs[kB][PER];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int tok = __shfl_sync(0xffffffffu, tok_l, u);
        const uint16_t* xr = qh + static_cast<size_t>(tok) * row_stride;
        if (PER == 4) {
          const uint2 w2 = __ldg(reinterpret_cast<const uint2*>(xr));
          const uint16_t* hv = reinterpret_cast<const uint16_t*>(&w2);
#pragma unroll
          for (int e = 0; e < PER; ++e) xs[u][e] = hv[e];
        } else {
          const uint32_t w1 = __ldg(reinterpret_cast<const uint32_t*>(xr));
          const uint16_t* hv = reinterpret_cast<const uint16_t*>(&w1);
#pragma unroll
          for (int e = 0; e < PER; ++e) xs[u][e] = hv[e];
        }
      }
      double t[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        double acc = 0.0;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc = fma(bf16d(xs[u][e]) - mm[e], vv[e], acc);
        t[u] = acc;
      }
      // recursive halving over lane bits 4..1: after the step with offset o a
      // lane holds half as many sums, each over twice as many lanes
#pragma unroll
      for (int m = kB / 2, o = 16; m >= 1; m >>= 1, o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int r = 0; r < m; ++r) {
          const double send = up ? t[r] : t[r + m];
          const double keep = up ? t[r + m] : t[r];
          t[r] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      t[0] += __shfl_xor_sync(0xffffffffu, t[0], 1);
      const int row = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
      if ((lane & 1) == 0 && i0 + row < n) keys[i0 + row] = t[0];
    }
  }
  __syncthreads();

  // ---------------- 4. select: the L-th smallest key T, and how many keys equal
  // to T go left (`need`, the first ones in position order)
  uint64_t prefix = 0, pmask = 0;
  int need = nd.L;  // rank (1-based) of the wanted key among those matching the prefix
  if (n <= kRankSelectMax) {
    // small node: direct ranks, every thread scanning all keys (in shared
    // memory, read in step: broadcasts) for the ranks of its own keys
    uint64_t* sk = reinterpret_cast<uint64_t*>(S.V);  // the basis is no longer needed
    for (int i = tid; i < n; i += kPddpThreads) sk[i] = key_bits(keys[i]);
    __syncthreads();
    for (int i = tid; i < n; i += kPddpThreads) {
      const uint64_t k = sk[i];
      int lt = 0, eq = 0;
#pragma unroll 4
      for (int o = 0; o < n; ++o) {
        const uint64_t x = sk[o];
        lt += x < k;
        eq += x == k;
      }
      if (lt < nd.L && nd.L <= lt + eq) {  // k is T; threads holding equal keys write the same
        S.kscal = k;
        S.iscal[1] = nd.L - lt;
      }
    }
    __syncthreads();
    prefix = S.kscal;
    need = S.iscal[1];
  }
  // larger nodes: radix select on the 64-bit keys (11-bit digits)
  int* whist = reinterpret_cast<int*>(S.V);  // [kPddpWarps][2048], the basis is no longer needed
  const int shifts[6] = {53, 42, 31, 20, 9, 0};
  const int widths[6] = {11, 11, 11, 11, 11, 9};
  for (int pass = 0; n > kRankSelectMax && pass < 6; ++pass) {
    const int nb = 1 << widths[pass];
    for (int i = lane; i < nb; i += 32) whist[warp * 2048 + i] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kPddpThreads * kSelUnroll) {
      uint64_t kr[kSelUnroll];  // the keys' loads all in flight before any is used
#pragma unroll
      for (int u = 0; u < kSelUnroll; ++u) {
        const int i = base + u * kPddpThreads + tid;
        kr[u] = i < n ? key_bits(keys[i]) : 0ull;
      }
#pragma unroll
      for (int u = 0; u < kSelUnroll; ++u) {
        const int i = base + u * kPddpThreads + tid;
        const uint64_t k = kr[u];
        const bool in = i < n && (k & pmask) == prefix;
        const unsigned act = __ballot_sync(0xffffffffu, in);
        if (in) {
          const int digit = static_cast<int>((k >> shifts[pass]) & static_cast<uint64_t>(nb - 1));
          const unsigned peers = __match_any_sync(act, digit);
          if (lane == __ffs(peers) - 1) atomicAdd(&whist[warp * 2048 + digit], __popc(peers));
        }
      }
    }
    __syncthreads();
    for (int i = tid; i < nb; i += kPddpThreads) {
      int t = 0;
#pragma unroll
      for (int w = 0; w < kPddpWarps; ++w) t += whist[w * 2048 + i];
      S.hist[i] = t;
    }
    __syncthreads();
    if (warp == 0) {  // lane l owns bins [l*per, (l+1)*per); ascending
      const int per = nb / 32;
      int sum = 0;
      for (int i = 0; i < per; ++i) sum += S.hist[lane * per + i];
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int excl = incl - sum;
      if (excl < need && incl >= need) {
        int acc = excl;
        for (int i = 0; i < per; ++i) {
          const int bin = lane * per + i;
          if (acc + S.hist[bin] >= need) {
            S.iscal[0] = bin;
            S.iscal[1] = acc;
            break;
          }
          acc += S.hist[bin];
        }
      }
    }
    __syncthreads();
    need -= S.iscal[1];
    prefix |= static_cast<uint64_t>(S.iscal[0]) << shifts[pass];
    pmask |= static_cast<uint64_t>(nb - 1) << shifts[pass];
    __syncthreads();
  }
  // keys below the threshold go left, then the first `need` equal keys in position order

  // ---------------- 5. stable partition over warp segments
  const int seg = ((n + kPddpWarps - 1) / kPddpWarps + 31) / 32 * 32;
  const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);
  {
    int lt = 0, eq = 0;
    for (int base = s0; base < s1; base += 32 * kSelUnroll) {
      uint64_t kr[kSelUnroll];
#pragma unroll
      for (int u = 0; u < kSelUnroll; ++u) {
        const int i = base + 32 * u + lane;
        kr[u] = i < s1 ? key_bits(keys[i]) : 0ull;
      }
#pragma unroll
      for (int u = 0; u < kSelUnroll; ++u) {
        const int i = base + 32 * u + lane;
        lt += __popc(__ballot_sync(0xffffffffu, i < s1 && kr[u] < prefix));
        eq += __popc(__ballot_sync(0xffffffffu, i < s1 && kr[u] == prefix));
      }
    }
    if (lane == 0) {
      S.wcnt[warp][0] = lt;
      S.wcnt[warp][1] = eq;
    }
  }
  __syncthreads();
  if (tid == 0) {
    int left = 0, right = 0, eqs = 0;
    for (int w = 0; w < kPddpWarps; ++w) {
      const int len = max(0, min(n, w * seg + seg) - min(n, w * seg));
      const int eq_take = max(0, min(S.wcnt[w][1], need - eqs));
      S.wleft[w] = left;
      S.wright[w] = right;
      S.weq[w] = eqs;
      left += S.wcnt[w][0] + eq_take;
      right += len - S.wcnt[w][0] - eq_take;
      eqs += S.wcnt[w][1];
    }
    S.iscal[2] = left;
  }
  __syncthreads();
  {
    int lo = S.wleft[warp], ro = S.wright[warp], es = S.weq[warp];
    for (int base = s0; base < s1; base += 32 * kSelUnroll) {
      uint64_t kr[kSelUnroll];
      int tr[kSelUnroll];
#pragma unroll
      for (int u = 0; u < kSelUnroll; ++u) {
        const int i = base + 32 * u + lane;
        kr[u] = i < s1 ? key_bits(keys[i]) : 0ull;
        tr[u] = i < s1 ? cur[i] : 0;
      }
#pragma unroll
      for (int u = 0; u < kSelUnroll; ++u) {
      const int i = base + 32 * u + lane;
      const bool valid = i < s1;
      const uint64_t k = kr[u];
      const bool eq = valid && k == prefix;
      const unsigned eqb = __ballot_sync(0xffffffffu, eq);
      const bool go_left = valid && (k < prefix || (eq && es + __popc(eqb & lanemask_lt()) < need));
      const unsigned lb = __ballot_sync(0xffffffffu, go_left);
      const unsigned vb = __ballot_sync(0xffffffffu, valid);
      if (valid) {
        const int tok = tr[u];
        if (go_left) nxt[lo + __popc(lb & lanemask_lt())] = tok;
        else nxt[nd.L + ro + __popc((vb & ~lb) & lanemask_lt())] = tok;
      }
      lo += __popc(lb);
      ro += __popc(vb & ~lb);
      es += __popc(eqb);
      }
    }
  }
  if (tid == 0 && S.iscal[2] != nd.L) record_status(a.status, MCS_ERR_BAD_INDEX, -2000000 - S.iscal[2]);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(S.tmem_slot, kTmemCols);
  }
}

__global__ void pddp_identity(int32_t* perm, int P, int N) {
  const size_t total = static_cast<size_t>(P) * N;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    perm[i] = static_cast<int32_t>(i % N);
}

// Level-by-level list of the internal nodes (and the 2048-row chunks of big
// nodes), numbered per level; one thread, same order as the host plan.
__global__ void pddp_plan_kernel(int N, Node* nodes, Chunk* chunks) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int lvl_node[kMaxLevels + 1], lvl_chunk[kMaxLevels + 1];
  build_plan(N, nodes, chunks, lvl_node, lvl_chunk);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

namespace {

struct Plan {
  std::vector<std::vector<Node>> levels;
  std::vector<std::vector<Chunk>> chunks;
  size_t max_nodes = 0, max_chunks = 0;
};

Plan make_plan(int N) {
  Plan pl;
  std::vector<Node> nodes(plan_max_nodes(N));
  std::vector<Chunk> chunks(plan_max_chunks(N));
  int lvl_node[kMaxLevels + 1], lvl_chunk[kMaxLevels + 1];
  const int nl = build_plan(N, nodes.data(), chunks.data(), lvl_node, lvl_chunk);
  for (int l = 0; l < nl; ++l) {
    pl.levels.emplace_back(nodes.begin() + lvl_node[l], nodes.begin() + lvl_node[l + 1]);
    pl.chunks.emplace_back(chunks.begin() + lvl_chunk[l], chunks.begin() + lvl_chunk[l + 1]);
    pl.max_nodes = std::max(pl.max_nodes, pl.levels.back().size());
    pl.max_chunks = std::max(pl.max_chunks, pl.chunks.back().size());
  }
  return pl;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

struct PddpWs {
  size_t tmp, keys, nodes, chunks, partial, mom, wscale, total;
};

PddpWs pddp_layout(int B, int H, int N, int d, const Plan& pl) {
  PddpWs w{};
  const size_t P = static_cast<size_t>(B) * H;
  size_t off = 0;
  w.tmp = off; off = align256(off + P * N * sizeof(int32_t));
  w.keys = off; off = align256(off + P * N * sizeof(double));
  size_t nn = 0, nc = 0;
  for (size_t l = 0; l < pl.levels.size(); ++l) { nn += pl.levels[l].size(); nc += pl.chunks[l].size(); }
  w.nodes = off; off = align256(off + (nn + 1) * sizeof(Node));
  w.chunks = off; off = align256(off + (nc + 1) * sizeof(Chunk));
  const size_t ps = static_cast<size_t>(d) + static_cast<size_t>(d) * (d + 1) / 2;
  w.partial = off; off = align256(off + P * pl.max_chunks * ps * sizeof(double));
  w.mom = off; off = align256(off + 2 * P * pl.max_nodes * ps * sizeof(double));  // two levels' moments
  w.wscale = off; off = align256(off + P * d * sizeof(double));
  w.total = off;
  return w;
}

template <int D>
cudaError_t run_levels(int B, int H, int N, const uint16_t* q, int32_t* perm, uint8_t* ws, const Plan& pl,
                       const PddpWs& L, int* status, int krylov_steps, bool whiten, cudaStream_t s) {
  const int P = B * H;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(pddp_node<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sizeof(NodeSmem<D>)));
    if (e != cudaSuccess) return e;
    attr = true;
  }
  // node and chunk tables of all levels, generated on the device in the
  // host plan's order (the tree depends only on N)
  std::vector<size_t> node_off, chunk_off;
  size_t nn = 0, nc = 0;
  for (size_t l = 0; l < pl.levels.size(); ++l) {
    node_off.push_back(nn);
    chunk_off.push_back(nc);
    nn += pl.levels[l].size();
    nc += pl.chunks[l].size();
  }
  Node* dnodes = reinterpret_cast<Node*>(ws + L.nodes);
  Chunk* dchunks = reinterpret_cast<Chunk*>(ws + L.chunks);
  cudaError_t e;
  pddp_plan_kernel<<<1, 1, 0, s>>>(N, dnodes, dchunks);
  note_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  int32_t* tmp = reinterpret_cast<int32_t*>(ws + L.tmp);
  int32_t* cur = perm;
  int32_t* nxt = tmp;
  pddp_identity<<<592, 256, 0, s>>>(cur, P, N);
  note_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  double* wscale = whiten ? reinterpret_cast<double*>(ws + L.wscale) : nullptr;
  if (whiten) {
    pddp_channel_scale<D><<<P, kPddpThreads, 0, s>>>(q, H, N, wscale);
    note_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  for (size_t l = 0; l < pl.levels.size(); ++l) {
    if ((e = cudaMemcpyAsync(nxt, cur, static_cast<size_t>(P) * N * sizeof(int32_t), cudaMemcpyDeviceToDevice, s)) !=
        cudaSuccess)
      return e;
    LevelArgs a{};
    a.B = B; a.H = H; a.N = N;
    a.nnodes = static_cast<int>(pl.levels[l].size());
    a.nchunks = static_cast<int>(pl.chunks[l].size());
    a.nodes = dnodes + node_off[l];
    a.chunks = dchunks + chunk_off[l];
    a.q = q;
    a.cur = cur;
    a.nxt = nxt;
    a.keys = reinterpret_cast<double*>(ws + L.keys);
    a.partial = reinterpret_cast<double*>(ws + L.partial);
    {
      double* mom = reinterpret_cast<double*>(ws + L.mom);
      const size_t lvl = static_cast<size_t>(P) * pl.max_nodes * PCfg<D>::PSTRIDE;
      a.mom_in = mom + ((l + 1) & 1) * lvl;   // written by the previous level
      a.mom_out = mom + (l & 1) * lvl;
      a.max_nodes = static_cast<int>(pl.max_nodes);
    }
    a.status = status;
    a.krylov_steps = krylov_steps;
    a.wscale = wscale;
    if (a.nchunks > 0) {
      pddp_cov_partial<D><<<P * a.nchunks, kPddpThreads, 0, s>>>(a);
      note_launches(1);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    pddp_node<D><<<P * a.nnodes, kPddpThreads, sizeof(NodeSmem<D>), s>>>(a);
    note_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    std::swap(cur, nxt);
  }
  if (cur != perm)
    return cudaMemcpyAsync(perm, cur, static_cast<size_t>(P) * N * sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
  return cudaSuccess;
}

}  // namespace

size_t pddp_workspace_bytes(int B, int H, int N, int d) {
  const Plan pl = make_plan(N);
  return pddp_layout(B, H, N, d, pl).total;
}

cudaError_t pddp_run(int B, int H, int N, int d, const uint16_t* q, int32_t* perm, void* ws, size_t ws_bytes,
                     int* status, int krylov_steps, bool whiten, cudaStream_t s) {
  const Plan pl = make_plan(N);
  const PddpWs L = pddp_layout(B, H, N, d, pl);
  if (ws_bytes < L.total) return cudaErrorInvalidValue;
  uint8_t* w = static_cast<uint8_t*>(ws);
  if (d == 128) return run_levels<128>(B, H, N, q, perm, w, pl, L, status, krylov_steps, whiten, s);
  if (d == 64) return run_levels<64>(B, H, N, q, perm, w, pl, L, status, krylov_steps, whiten, s);
  return cudaErrorInvalidValue;
}

}  // namespace mcs
