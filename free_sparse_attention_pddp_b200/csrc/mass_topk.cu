// Anchor passes 2 and 3 of MC-Sparse (aiwillknow analysis, step 2; paper
// Table 4 "token" granularity): exact attention probabilities from a second
// QK^T pass, per-group probability mass, and token-level top-K selection.
//
// Mass pass: one CTA per (b, h, 128-key tile). It keeps its K tile in shared
// memory and streams every query group of the head through S^T = K_tile Q_g^T
// (UMMA, M = 128 keys, N = 128 queries). Each TMEM lane is one key, so a
// consumer thread turns its 128 columns into probabilities
// p_ij = 2^(s_ij*scale*log2e - lse_i*log2e) and sums them: m_g(j) with no
// cross-thread reduction. Output: fp32 mass [B, hn, G, N].
//
// Top-K: one CTA per (b, h, g). A 3-pass radix select (11/11/10 bits of the
// fp32 key) finds the K-th largest mass T. Keys above T(1+eps) are taken, keys
// below T(1-eps) dropped; keys in the band are re-scored in fp64 (exact bf16
// products, double exp, the dense pass's lse) and ranked by (mass desc, index
// asc). The selection is written in ascending index order.
#include <cuda_bf16.h>
#include <math_constants.h>

#include <cub/block/block_scan.cuh>

#include "mcs_ptx.cuh"

namespace mcs {

namespace {

constexpr int kMassThreads = 192;

template <int D>
struct MassCfg {
  static constexpr int KB = D / 64;
  static constexpr uint32_t TILE = 128u * D * 2u;
  static constexpr int NQ = 3;  // query-tile stages
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_Q = TILE;
  static constexpr uint32_t OFF_LSE = OFF_Q + NQ * TILE;  // NQ x 128 floats
  static constexpr uint32_t OFF_BAR = OFF_LSE + NQ * 512;
  static constexpr uint32_t NBAR = 1 + 2 * NQ + 4 + 1;
  static constexpr uint32_t SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 256;
};

__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kMassThreads, 1)
    mass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const MassParams p) {
  using C = MassCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sQ = smem + C::OFF_Q;
  float* sL = reinterpret_cast<float*>(smem + C::OFF_LSE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* k_full = bars;
  uint64_t* q_full = bars + 1;        // [NQ]
  uint64_t* q_empty = q_full + C::NQ; // [NQ]
  uint64_t* s_full = q_empty + C::NQ; // [2]
  uint64_t* s_empty = s_full + 2;     // [2]
  uint64_t* drain_bar = s_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kt = blockIdx.x % p.G;  // key tile
  const int bh = blockIdx.x / p.G;  // over B * hn
  const int b = bh / p.hn;
  const int hl = bh % p.hn;
  const int h = p.h0 + hl;
  const size_t head_base = static_cast<size_t>(b) * p.H + h;

  if (threadIdx.x == 0) {
    mbar_init(k_full, 1);
    for (int i = 0; i < C::NQ; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1 + 128);  // UMMA done (commit) + every consumer read the lse slice
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 128);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wctx{abort_flag, p.status, p.wait_limit_ns};
  int issued = 0;

  if (warp == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    int kr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int j = kt * 128 + lane * 4 + i;
      if (j >= p.N) j = p.N - 1;
      kr[i] = (b * p.N + j) * p.H + h;
    }
    if (lane == 0) mbar_arrive_expect_tx(k_full, C::TILE);
    __syncwarp();
#pragma unroll
    for (int kb = 0; kb < C::KB; ++kb)
      tma_gather4(&tm_k, k_full, sK + kb * 16384 + lane * 512, kb * 64, kr[0], kr[1], kr[2], kr[3]);
    for (int g = 0; g < p.G; ++g) {
      const int st = g % C::NQ;
      if (g >= C::NQ && !mbar_wait(&q_empty[st], ((g / C::NQ) & 1) ^ 1, wctx, MCS_WHERE_MASS_PRODUCER)) break;
      int qr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        int pos = g * 128 + lane * 4 + i;
        if (pos >= p.N) pos = p.N - 1;
        int tok = p.perm[head_base * p.N + pos];
        if (tok < 0 || tok >= p.N) {
          record_status(p.status, MCS_ERR_BAD_INDEX, tok);
          tok = 0;
        }
        qr[i] = (b * p.N + tok) * p.H + h;
      }
      if (lane == 0) mbar_arrive_expect_tx(&q_full[st], C::TILE + 512);
      __syncwarp();
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb)
        tma_gather4(&tm_q, &q_full[st], sQ + st * C::TILE + kb * 16384 + lane * 512, kb * 64, qr[0], qr[1], qr[2],
                    qr[3]);
      if (lane == 0)
        bulk_copy_g2s(sL + st * 128, p.lse_perm + head_base * (static_cast<size_t>(p.G) * 128) + g * 128, 512,
                      &q_full[st]);
      issued = g + 1;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, false, false);
      const uint32_t aK = smem_u32(sK), aQ = smem_u32(sQ);
      bool ok = mbar_wait(k_full, 0, wctx, MCS_WHERE_MASS_MMA);
      for (int g = 0; ok && g < p.G; ++g) {
        const int st = g % C::NQ;
        const int sb = g & 1;
        if (!mbar_wait(&q_full[st], (g / C::NQ) & 1, wctx, MCS_WHERE_MASS_MMA)) break;
        if (g >= 2 && !mbar_wait(&s_empty[sb], ((g - 2) >> 1) & 1, wctx, MCS_WHERE_MASS_MMA)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_bf16_ss(tmem + sb * 128, sdesc_sw128(aK + off, 16, 1024),
                       sdesc_sw128(aQ + st * C::TILE + off, 16, 1024), IDESC, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[sb]);
        umma_commit(&q_empty[st]);
      }
    }
    __syncwarp();
  } else {
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // key within the tile
    const int key = kt * 128 + row;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const float c = p.scale_log2;
    float* out = p.mass + (static_cast<size_t>(b) * p.hn + hl) * static_cast<size_t>(p.G) * p.N;
    for (int g = 0; g < p.G; ++g) {
      const int sb = g & 1;
      const int st = g % C::NQ;
      if (!mbar_wait_warp(&s_full[sb], (g >> 1) & 1, wctx, MCS_WHERE_MASS_CONSUMER)) break;
      tc_fence_after();
      float sv[128];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld32(tmem + lane_addr + sb * 128 + q * 32, sv + q * 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_empty[sb]);
      // the group's lse slice arrived with its query tile; the stage is not
      // refilled before these threads arrive on q_empty below
      if (!mbar_wait_warp(&q_full[st], (g / C::NQ) & 1, wctx, MCS_WHERE_MASS_CONSUMER)) break;
      const float* lse = sL + st * 128;
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
      for (int i = 0; i < 128; i += 2) {
        acc0 += fast_exp2(fmaf(sv[i], c, -lse[i] * 1.4426950408889634f));
        acc1 += fast_exp2(fmaf(sv[i + 1], c, -lse[i + 1] * 1.4426950408889634f));
      }
      mbar_arrive(&q_empty[st]);
      if (key < p.N) out[static_cast<size_t>(g) * p.N + key] = acc0 + acc1;
    }
  }

  __syncthreads();
  if (*abort_flag) {
    volatile int never = 0;
    const WaitCtx drain_ctx{&never, nullptr, 50000000ull};
    if (warp == 0 && lane == 0)
      for (int g = max(0, issued - C::NQ); g < issued; ++g)
        mbar_wait(&q_full[g % C::NQ], (g / C::NQ) & 1, drain_ctx, MCS_WHERE_DRAIN);
    if (warp == 1 && lane == 0) {
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0, drain_ctx, MCS_WHERE_DRAIN);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// top-K
// ---------------------------------------------------------------------------

namespace {
constexpr int kTopkThreads = 1024;
constexpr int kBandMax = 2048;
using BlockScan = cub::BlockScan<int, kTopkThreads>;

struct TopkSmem {
  int hist[2048];
  int band_idx[kBandMax];
  double band_m[kBandMax];
  float lse[128];
  int scalars[8];
  typename BlockScan::TempStorage scan;
};

// inclusive suffix search over hist[0..nbins): the bin holding the need-th
// largest key; returns the bin and the count of keys in higher bins
__device__ void find_bin(const int* hist, int nbins, int need, int* out_bin, int* out_above, int* scratch) {
  // one warp: each lane owns a contiguous chunk of bins, highest chunk first
  const int lane = threadIdx.x & 31;
  const int per = nbins / 32;
  const int hi = nbins - lane * per;  // chunk [hi - per, hi)
  int sum = 0;
  for (int bidx = hi - 1; bidx >= hi - per; --bidx) sum += hist[bidx];
  // exclusive prefix over lanes (lane 0 = highest bins)
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const int excl = incl - sum;
  if (excl < need && incl >= need) {
    int acc = excl;
    for (int bidx = hi - 1; bidx >= hi - per; --bidx) {
      if (acc + hist[bidx] >= need) {
        *out_bin = bidx;
        *out_above = acc;
        break;
      }
      acc += hist[bidx];
    }
  }
  (void)scratch;
}
}  // namespace

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(const TopkParams p) {
  extern __shared__ uint8_t smem_raw[];
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(smem_raw);
  uint32_t* selbits = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkSmem));  // N bits
  float* qrows = reinterpret_cast<float*>(selbits + ((p.N + 31) / 32 + 3) / 4 * 4);  // 128 x d fp32

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.x % p.G;
  const int bh = blockIdx.x / p.G;
  const int b = bh / p.hn;
  const int hl = bh % p.hn;
  const int h = p.h0 + hl;
  const size_t head_base = static_cast<size_t>(b) * p.H + h;
  const float* mrow = p.mass + ((static_cast<size_t>(b) * p.hn + hl) * p.G + g) * static_cast<size_t>(p.N);
  const int N = p.N;

  // ---------------- radix select of the K-th largest fp32 key
  uint32_t prefix = 0, pmask = 0;
  int need = p.K;
  const int shifts[3] = {21, 10, 0};
  const int nbits[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int nb = 1 << nbits[pass];
    for (int i = tid; i < nb; i += kTopkThreads) S.hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < N; j += kTopkThreads) {
      const uint32_t key = __float_as_uint(mrow[j]);
      if ((key & pmask) == prefix) atomicAdd(&S.hist[(key >> shifts[pass]) & (nb - 1)], 1);
    }
    __syncthreads();
    if (warp == 0) find_bin(S.hist, nb, need, &S.scalars[0], &S.scalars[1], nullptr);
    __syncthreads();
    const int bin = S.scalars[0];
    need -= S.scalars[1];
    prefix |= static_cast<uint32_t>(bin) << shifts[pass];
    pmask |= static_cast<uint32_t>(nb - 1) << shifts[pass];
    __syncthreads();
  }
  const uint32_t Tkey = prefix;  // K-th largest key; `need` keys equal to it are taken in the fp32 ranking
  const float Tval = __uint_as_float(Tkey);
  const float hi = Tval * (1.f + p.band_rel);
  const float lo = Tval * (1.f - p.band_rel);

  // ---------------- band: keys with lo <= m <= hi, collected in index order
  int c_in = 0, nband = 0;
  for (int base = 0; base < N; base += kTopkThreads) {
    const int j = base + tid;
    const float m = j < N ? mrow[j] : 0.f;
    const int inb = (j < N && m >= lo && m <= hi) ? 1 : 0;
    const int above = (j < N && m > hi) ? 1 : 0;
    int pos, tot;
    BlockScan(S.scan).ExclusiveSum(inb, pos, tot);
    __syncthreads();
    if (inb && nband + pos < kBandMax) S.band_idx[nband + pos] = j;
    nband += tot;
    int a_tot;
    int dummy;
    BlockScan(S.scan).ExclusiveSum(above, dummy, a_tot);
    __syncthreads();
    c_in += a_tot;
  }
  for (int i = tid; i < (N + 31) / 32; i += kTopkThreads) selbits[i] = 0;
  const bool overflow = nband > kBandMax;
  const int take = p.K - c_in;  // 1 <= take <= nband when no overflow
  __syncthreads();

  if (!overflow) {
    // load this group's query rows (fp32) and lse
    const int nrows = min(128, N - g * 128);
    for (int e = tid; e < 128 * p.d; e += kTopkThreads) {
      const int r = e / p.d, c = e % p.d;
      float x = 0.f;
      if (r < nrows) {
        const int tok = p.perm[head_base * N + g * 128 + r];
        x = __uint_as_float(static_cast<uint32_t>(p.q[((static_cast<size_t>(b) * N + tok) * p.H + h) * p.d + c]) << 16);
      }
      qrows[e] = x;
    }
    if (tid < 128) S.lse[tid] = p.lse_perm[head_base * (static_cast<size_t>(p.G) * 128) + g * 128 + tid];
    __syncthreads();
    // fp64 rescoring: one warp per band key, lanes over queries
    const double scale = p.scale;
    for (int t = warp; t < nband; t += kTopkThreads / 32) {
      const int j = S.band_idx[t];
      const uint16_t* krow = p.k + ((static_cast<size_t>(b) * N + j) * p.H + h) * p.d;
      double acc = 0.0;
      for (int r = lane; r < nrows; r += 32) {
        const float* qr = qrows + r * p.d;
        double dot = 0.0;
        for (int c = 0; c < p.d; ++c)
          dot = fma(static_cast<double>(qr[c]),
                    static_cast<double>(__uint_as_float(static_cast<uint32_t>(krow[c]) << 16)), dot);
        acc += exp(dot * scale - static_cast<double>(S.lse[r]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) S.band_m[t] = acc;
    }
    __syncthreads();
    // rank inside the band by (mass desc, index asc); take the first `take`
    for (int t = tid; t < nband; t += kTopkThreads) {
      const double mt = S.band_m[t];
      const int jt = S.band_idx[t];
      int rank = 0;
      for (int u = 0; u < nband; ++u) {
        const double mu = S.band_m[u];
        rank += (mu > mt || (mu == mt && S.band_idx[u] < jt)) ? 1 : 0;
      }
      if (rank < take) atomicOr(&selbits[jt >> 5], 1u << (jt & 31));
    }
    if (tid == 0) atomicAdd(p.status + MCS_SW_REFINED, nband);
  } else {
    if (tid == 0) atomicAdd(p.status + MCS_SW_BAND_OVERFLOW, 1);
  }
  __syncthreads();

  // ---------------- write the selection in ascending index order
  int32_t* outp = p.kv_idx + (head_base * p.G + g) * static_cast<size_t>(p.K);
  int written = 0, eq_seen = 0;
  for (int base = 0; base < N; base += kTopkThreads) {
    const int j = base + tid;
    int flag = 0, eq = 0;
    if (j < N) {
      const float m = mrow[j];
      if (!overflow) {
        flag = (m > hi) || ((selbits[j >> 5] >> (j & 31)) & 1u);
      } else {
        const uint32_t key = __float_as_uint(m);
        eq = key == Tkey;
        flag = key > Tkey;
      }
    }
    if (overflow) {  // fp32 fallback: equal keys taken in index order
      int eq_pos, eq_tot;
      BlockScan(S.scan).ExclusiveSum(eq, eq_pos, eq_tot);
      __syncthreads();
      if (eq && eq_seen + eq_pos < need) flag = 1;
      eq_seen += eq_tot;
    }
    int pos, tot;
    BlockScan(S.scan).ExclusiveSum(flag, pos, tot);
    __syncthreads();
    if (flag && written + pos < p.K) outp[written + pos] = j;
    written += tot;
  }
  if (tid == 0 && written != p.K) record_status(p.status, MCS_ERR_BAD_INDEX, -1000000 - written);
}

template <int D>
static cudaError_t launch_mass_t(const CUtensorMap* tq, const CUtensorMap* tk, const MassParams& p,
                                 cudaStream_t s) {
  using C = MassCfg<D>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(mass_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  mass_kernel<D><<<p.B * p.hn * p.G, kMassThreads, C::SMEM, s>>>(*tq, *tk, p);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_mass(int d, const CUtensorMap* tq, const CUtensorMap* tk, const MassParams& p, cudaStream_t s) {
  if (d == 128) return launch_mass_t<128>(tq, tk, p, s);
  if (d == 64) return launch_mass_t<64>(tq, tk, p, s);
  return cudaErrorInvalidValue;
}

size_t topk_smem_bytes(int N, int d) {
  return sizeof(TopkSmem) + static_cast<size_t>(((N + 31) / 32 + 3) / 4 * 4) * 4 + 128ull * d * 4;
}

cudaError_t launch_topk(const TopkParams& p, cudaStream_t s) {
  const size_t smem = topk_smem_bytes(p.N, p.d);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  topk_kernel<<<p.B * p.hn * p.G, kTopkThreads, smem, s>>>(p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace mcs
