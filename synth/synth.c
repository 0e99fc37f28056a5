/*
 * Seeded synthetic Q/K/V for the MC-Sparse workloads.
 *
 * This file produces INPUTS only. It holds none of the attention, grouping or
 * selection arithmetic; both the CUDA path and the CPU oracle read the tensors
 * it writes.
 *
 * Random numbers are counter based: splitmix64 (Steele, Lea and Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014) hashes a stream key
 * and an element counter into 64 bits, and the Box-Muller transform (Box and
 * Muller, 1958) turns two uniforms into one standard normal. A stream key mixes
 * (seed, tensor, step, layer, head, component), so any single head of any step
 * can be regenerated alone.
 *
 * Value models (per head, d channels, N tokens):
 *   model 0, "low-rank":  X = Z + alpha * sum_{r<8} a_{i,r} c_r, with c_r ~ N(0, I_d)
 *                         shared by Q and K, a_{i,r} ~ N(0,1) drawn per tensor,
 *                         alpha = sqrt(3 / sqrt(8 d)); V = Z.
 *   model 1, "field":     X = gamma * F + Z. F is an iid N(0,1) field over the
 *                         (T, Y, X) token grid, blurred per channel by a separable
 *                         periodic Gaussian (sigma = 2 tokens per axis, truncated
 *                         at 3 sigma) and divided by the blur's exact std gain.
 *                         Q and K share one field per head; V has its own.
 *   heavy_k:              K's Z is Student-t (nu = 4) scaled to unit variance.
 *   drift:                X_t = X_0 + drift * sum_{s=1..t} W_s, W_s ~ N(0,1).
 * Token index n = (t * Y + y) * X + x. Output is bf16 (round to nearest even).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { T_Q = 0, T_K = 1, T_V = 2 };
enum { C_Z = 1, C_A = 2, C_C = 3, C_F = 4, C_W = 5, C_CHI = 6 };

static inline uint64_t sm64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

static uint64_t stream_key(uint64_t seed, int tensor, int step, int layer, int head, int comp) {
  uint64_t k = sm64(seed);
  k = sm64(k ^ (uint64_t)(tensor + 1));
  k = sm64(k ^ (uint64_t)(step + 1) * 0x100000001B3ull);
  k = sm64(k ^ (uint64_t)(layer + 1) * 0xC2B2AE3D27D4EB4Full);
  k = sm64(k ^ (uint64_t)(head + 1) * 0x165667B19E3779F9ull);
  k = sm64(k ^ (uint64_t)(comp + 1) * 0x27D4EB2F165667C5ull);
  return k;
}

/* Standard normal number `i` of stream `key`. */
static inline double normal_at(uint64_t key, uint64_t i) {
  uint64_t a = sm64(key ^ sm64(2 * i));
  uint64_t b = sm64(key ^ sm64(2 * i + 1));
  double u1 = ((double)(a >> 11) + 1.0) * 0x1.0p-53; /* (0, 1] */
  double u2 = (double)(b >> 11) * 0x1.0p-53;         /* [0, 1) */
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925 * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* Periodic separable Gaussian blur of one channel field along one axis. */
static void blur_axis(float* f, float* tmp, int T, int Y, int X, int axis, const double* w, int R) {
  int n = T * Y * X;
  int len = axis == 0 ? T : (axis == 1 ? Y : X);
  int stride = axis == 0 ? Y * X : (axis == 1 ? X : 1);
  int* wrap = (int*)malloc(sizeof(int) * (size_t)len * (2 * R + 1));
  for (int p = 0; p < len; ++p)
    for (int k = -R; k <= R; ++k) wrap[p * (2 * R + 1) + k + R] = ((p + k) % len + len) % len;
  for (int i = 0; i < n; ++i) {
    int p = (i / stride) % len;
    int base = i - p * stride;
    const int* wp = wrap + p * (2 * R + 1);
    double acc = 0.0;
    for (int k = 0; k < 2 * R + 1; ++k) acc += w[k] * (double)f[base + wp[k] * stride];
    tmp[i] = (float)acc;
  }
  memcpy(f, tmp, sizeof(float) * (size_t)n);
  free(wrap);
}

typedef struct {
  int model, tensor, step, layer, head, N, d, T, Y, X, heavy_k;
  uint64_t seed;
  double gamma, drift;
  float* out; /* N*d, row = token */
} head_job;

static void gen_head(const head_job* j) {
  const int N = j->N, d = j->d;
  float* out = j->out;
  /* noise Z (or Student-t for K when heavy_k) */
  uint64_t kz = stream_key(j->seed, j->tensor, 0, j->layer, j->head, C_Z);
  if (j->heavy_k && j->tensor == T_K) {
    uint64_t kc = stream_key(j->seed, j->tensor, 0, j->layer, j->head, C_CHI);
    for (long i = 0; i < (long)N * d; ++i) {
      double chi = 0.0;
      for (int r = 0; r < 4; ++r) { double g = normal_at(kc, (uint64_t)i * 4 + r); chi += g * g; }
      double t = normal_at(kz, (uint64_t)i) / sqrt(chi / 4.0);
      out[i] = (float)(t / sqrt(2.0)); /* Var(t_4) = 2 */
    }
  } else {
    for (long i = 0; i < (long)N * d; ++i) out[i] = (float)normal_at(kz, (uint64_t)i);
  }
  if (j->model == 0) {
    if (j->tensor != T_V) {
      const int Rk = 8;
      double alpha = sqrt(3.0 / sqrt(8.0 * d));
      uint64_t kc = stream_key(j->seed, 99, 0, j->layer, j->head, C_C); /* shared by Q and K */
      uint64_t ka = stream_key(j->seed, j->tensor, 0, j->layer, j->head, C_A);
      double* c = (double*)malloc(sizeof(double) * Rk * d);
      for (int i = 0; i < Rk * d; ++i) c[i] = normal_at(kc, (uint64_t)i);
      for (int i = 0; i < N; ++i) {
        double a[8];
        for (int r = 0; r < Rk; ++r) a[r] = normal_at(ka, (uint64_t)i * Rk + r);
        for (int e = 0; e < d; ++e) {
          double s = 0.0;
          for (int r = 0; r < Rk; ++r) s += a[r] * c[r * d + e];
          out[(long)i * d + e] = (float)((double)out[(long)i * d + e] + alpha * s);
        }
      }
      free(c);
    }
  } else {
    /* smooth field shared by Q and K (component tag 98), own field for V (97) */
    int ftag = (j->tensor == T_V) ? 97 : 98;
    uint64_t kf = stream_key(j->seed, ftag, 0, j->layer, j->head, C_F);
    const int R = 6;
    double w[13], ws = 0.0, w2 = 0.0;
    for (int k = -R; k <= R; ++k) { w[k + R] = exp(-(double)(k * k) / (2.0 * 2.0 * 2.0)); ws += w[k + R]; }
    for (int k = 0; k < 2 * R + 1; ++k) { w[k] /= ws; w2 += w[k] * w[k]; }
    double gain = sqrt(w2 * w2 * w2); /* std of the 3-axis blur of unit white noise */
    float* f = (float*)malloc(sizeof(float) * (size_t)N);
    float* tmp = (float*)malloc(sizeof(float) * (size_t)N);
    for (int e = 0; e < d; ++e) {
      for (int i = 0; i < N; ++i) f[i] = (float)normal_at(kf, (uint64_t)e * (uint64_t)N + (uint64_t)i);
      for (int ax = 0; ax < 3; ++ax) blur_axis(f, tmp, j->T, j->Y, j->X, ax, w, R);
      for (int i = 0; i < N; ++i)
        out[(long)i * d + e] = (float)((double)out[(long)i * d + e] + j->gamma * (double)f[i] / gain);
    }
    free(f);
    free(tmp);
  }
  for (int s = 1; s <= j->step; ++s) {
    uint64_t kw = stream_key(j->seed, j->tensor, s, j->layer, j->head, C_W);
    for (long i = 0; i < (long)N * d; ++i) out[i] = (float)((double)out[i] + j->drift * normal_at(kw, (uint64_t)i));
  }
}

typedef struct {
  head_job base;
  int Hd, hb, h0, h1;
  uint16_t* dst; /* [N, Hd, d]: heads hb .. hb+Hd-1 of batch entry 0 */
  int rc;
} fill_job;

static void* fill_worker(void* p) {
  fill_job* fj = (fill_job*)p;
  size_t nd = (size_t)fj->base.N * fj->base.d;
  float* buf = (float*)malloc(sizeof(float) * nd);
  if (!buf) { fj->rc = 1; return NULL; }
  for (int h = fj->h0; h < fj->h1; ++h) {
    head_job j = fj->base;
    j.head = h;
    j.out = buf;
    gen_head(&j);
    for (int i = 0; i < j.N; ++i)
      for (int e = 0; e < j.d; ++e)
        fj->dst[((size_t)i * fj->Hd + (h - fj->hb)) * j.d + e] = f32_to_bf16_rne(buf[(size_t)i * j.d + e]);
  }
  free(buf);
  fj->rc = 0;
  return NULL;
}

/*
 * Fill dst = bf16 [N, h_end - h_begin, d] (one batch entry) with heads
 * [h_begin, h_end) of the given tensor/step/layer; H is the workload's head
 * count. Returns 0 on success.
 */
int synth_fill(int model, uint64_t seed, int tensor, int step, int layer, int H, int h_begin, int h_end, int N,
               int d, int T, int Y, int X, double gamma, double drift, int heavy_k, int nthreads, uint16_t* dst) {
  if (N <= 0 || d <= 0 || H <= 0 || h_begin < 0 || h_end > H || h_begin >= h_end) return 2;
  if (model == 1 && (long)T * Y * X != N) return 3;
  if (nthreads < 1) nthreads = 1;
  int nh = h_end - h_begin;
  if (nthreads > nh) nthreads = nh;
  pthread_t th[256];
  fill_job jobs[256];
  if (nthreads > 256) nthreads = 256;
  for (int t = 0; t < nthreads; ++t) {
    head_job b = {model, tensor, step, layer, 0, N, d, T, Y, X, heavy_k, seed, gamma, drift, NULL};
    jobs[t].base = b;
    jobs[t].Hd = nh;
    jobs[t].hb = h_begin;
    jobs[t].h0 = h_begin + (int)((long)nh * t / nthreads);
    jobs[t].h1 = h_begin + (int)((long)nh * (t + 1) / nthreads);
    jobs[t].dst = dst;
    jobs[t].rc = 0;
    pthread_create(&th[t], NULL, fill_worker, &jobs[t]);
  }
  int rc = 0;
  for (int t = 0; t < nthreads; ++t) {
    pthread_join(th[t], NULL);
    rc |= jobs[t].rc;
  }
  return rc;
}
