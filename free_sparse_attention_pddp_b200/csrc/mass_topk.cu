// Anchor passes 2 and 3 of MC-Sparse (aiwillknow analysis, step 2; paper
// Table 4 "token" granularity): exact attention probabilities from a second
// QK^T pass, per-group probability mass, and token-level top-K selection.
//
// Mass pass: one CTA per (b, h, 128-key tile). It keeps its K tile in shared
// memory and streams every query group of the head (from a copy of Q laid out
// in group order, one tiled TMA box per group) through S^T = K_tile Q_g^T
// (UMMA, M = 128 keys, N = 128 queries). Three consumer warpgroups take the
// groups in turn, each with its own TMEM S buffer, so one warpgroup's loads and
// reductions overlap the others' exponentials. A query tile's stage is free
// again as soon as its UMMAs complete; the group's lse slice, which its
// consumer reads throughout, travels in a separate, deeper ring, so the tile
// loads run ahead of the consumers by the whole ring. Each TMEM lane is one key, so a
// consumer thread turns its 128 columns
// into probabilities
// p_ij = 2^(s_ij*scale*log2e - lse2_i) (lse2 = lse*log2e; the dense pass stores -lse2, so
// each exponent is one fused multiply-add) and sums them: m_g(j) with no
// cross-thread reduction. Output: fp32 mass [B, hn, G, N].
//
// Top-K: one CTA per (b, h, g). Two sweeps over the group's fp32 mass row find
// the K-th largest mass T (a 4096-bin histogram of the key's top 12 bits, then
// the keys of T's bin gathered into shared memory for an exact radix select).
// Keys above T(1+eps) are taken, keys below T(1-eps) dropped; keys in the band
// are re-scored in fp64 (exact bf16 products, double exp, the dense pass's lse
// read as its fp32 hi + lo pair)
// and ranked by (mass desc, index asc). The selection is written in ascending
// index order. Rare rows (see topk_kernel) take a general seven-sweep path with
// the same result.
#include <cuda_bf16.h>
#include <math_constants.h>


#include "mcs_ptx.cuh"

namespace mcs {

namespace {

constexpr int kMassConsumers = 3;  // consumer warpgroups, one TMEM S buffer each (four would spill at 96 registers)
constexpr int kMassThreads = 64 + 128 * kMassConsumers;  // producer warp, UMMA warp, consumers

template <int D>
struct MassCfg {
  static constexpr int KB = D / 64;
  static constexpr uint32_t TILE = 128u * D * 2u;
  static constexpr int NQ = 5;  // query-tile stages, each free again once its UMMAs completed
  static constexpr int NL = 8;  // lse slices (512 B), held until the group's consumer finished
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_Q = TILE;
  static constexpr uint32_t OFF_LSE = OFF_Q + NQ * TILE;  // NL x 128 floats
  static constexpr uint32_t OFF_BAR = OFF_LSE + NL * 512;
  static constexpr uint32_t NBAR = 1 + 2 * NQ + 2 * NL + 2 * kMassConsumers + 1;
  static constexpr uint32_t SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  // one 128-column S buffer per consumer warpgroup; allocations are powers of two
  static constexpr uint32_t TMEM_COLS = 128 * kMassConsumers <= 256 ? 256 : 512;
  static_assert(128 * kMassConsumers <= 512, "TMEM holds at most four S buffers");
};

__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* dst, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

}  // namespace

// Queries in group order, one 128-row tile per group: qp[b,h,pos] = q[b, perm[pos], h]
// (rows past N repeat the last query; the mass pass gives them probability 0).
__global__ void permute_queries(const uint16_t* q, const int32_t* perm, uint16_t* qp, int B, int H, int N, int G,
                                int d, int* status) {
  const int per_row = d / 8;  // 16-byte pieces per row
  const size_t rows = static_cast<size_t>(B) * H * G * 128;
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < rows * per_row;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t r = e / per_row;
    const int c = static_cast<int>(e % per_row);
    const int pos0 = static_cast<int>(r % (static_cast<size_t>(G) * 128));
    const size_t bh = r / (static_cast<size_t>(G) * 128);
    const int b = static_cast<int>(bh / H), h = static_cast<int>(bh % H);
    const int pos = pos0 < N ? pos0 : N - 1;
    int tok = perm[bh * N + pos];
    if (tok < 0 || tok >= N) {
      record_status(status, MCS_ERR_BAD_INDEX, tok);
      tok = 0;
    }
    const uint4* src = reinterpret_cast<const uint4*>(q + ((static_cast<size_t>(b) * N + tok) * H + h) * d) + c;
    reinterpret_cast<uint4*>(qp + r * d)[c] = __ldg(src);
  }
}

template <int D>
__global__ void __launch_bounds__(kMassThreads, 1)
    mass_kernel(const __grid_constant__ CUtensorMap tm_qp, const __grid_constant__ CUtensorMap tm_k,
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
  uint64_t* l_full = q_empty + C::NQ; // [NL]
  uint64_t* l_empty = l_full + C::NL; // [NL]
  uint64_t* s_full = l_empty + C::NL; // [kMassConsumers]: buffer c holds the groups of consumer warpgroup c
  uint64_t* s_empty = s_full + kMassConsumers;
  uint64_t* drain_bar = s_empty + kMassConsumers;
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
      mbar_init(&q_empty[i], 1);  // the group's UMMAs completed (commit)
    }
    for (int i = 0; i < C::NL; ++i) {
      mbar_init(&l_full[i], 1);
      mbar_init(&l_empty[i], 128);  // the consumer warpgroup is done with the slice
    }
    for (int i = 0; i < kMassConsumers; ++i) {
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
  // The CTAs of one wave hold consecutive key tiles of one head; each starts
  // its sweep over the query groups at its own key tile's index, so at any
  // moment they read different query tiles (spread over the L2) instead of
  // all requesting the same one.
  auto rot = [&](int g) { const int r = g + kt; return r < p.G ? r : r - p.G; };

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tm_qp);
      prefetch_tensormap(&tm_k);
      // the key tile: 128 consecutive tokens of head h (box {64, 1, 128})
      mbar_arrive_expect_tx(k_full, C::TILE);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb) tma_load_3d(&tm_k, k_full, sK + kb * 16384, kb * 64, h, b * p.N + kt * 128);
      const int qrow0 = static_cast<int>(head_base * p.G * 128);
      for (int g = 0; g < p.G; ++g) {
        const int st = g % C::NQ, sl = g % C::NL;
        if (g >= C::NQ && !mbar_wait(&q_empty[st], ((g / C::NQ) & 1) ^ 1, wctx, MCS_WHERE_MASS_PRODUCER)) break;
        if (g >= C::NL && !mbar_wait(&l_empty[sl], ((g / C::NL) & 1) ^ 1, wctx, MCS_WHERE_MASS_PRODUCER)) break;
        mbar_arrive_expect_tx(&q_full[st], C::TILE);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_2d(&tm_qp, &q_full[st], sQ + st * C::TILE + kb * 16384, kb * 64, qrow0 + rot(g) * 128);
        mbar_arrive_expect_tx(&l_full[sl], 512);
        bulk_copy_g2s(sL + sl * 128, p.lse_perm + head_base * (static_cast<size_t>(p.G) * 128) + rot(g) * 128, 512,
                      &l_full[sl]);
        issued = g + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // one lane runs the schedule and issues the UMMAs
      constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, false, false);
      // descriptors built once; each UMMA steps them with one add
      const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
      bool ok = mbar_wait(k_full, 0, wctx, MCS_WHERE_MASS_MMA);
      for (int g = 0; ok && g < p.G; ++g) {
        const int st = g % C::NQ;
        const int sb = g % kMassConsumers;
        if (!mbar_wait(&q_full[st], (g / C::NQ) & 1, wctx, MCS_WHERE_MASS_MMA)) break;
        if (g >= kMassConsumers &&
            !mbar_wait(&s_empty[sb], ((g - kMassConsumers) / kMassConsumers) & 1, wctx, MCS_WHERE_MASS_MMA))
          break;
        tc_fence_after();
        const uint64_t dQs = sdesc_advance(dQ, st * C::TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_bf16_ss(tmem + sb * 128, sdesc_advance(dK, off), sdesc_advance(dQs, off), IDESC, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[sb]);
        umma_commit(&q_empty[st]);
      }
    }
    __syncwarp();
  } else {
    const int wg = (warp - 2) >> 2;  // consumer warpgroup: groups g with g % kMassConsumers == wg
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // key within the tile
    const int key = kt * 128 + row;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const float c = p.scale_log2;
    const uint64_t c2 = f2_pack(c, c);
    float* out = p.mass + (static_cast<size_t>(b) * p.hn + hl) * static_cast<size_t>(p.G) * p.N;
    for (int g = wg; g < p.G; g += kMassConsumers) {
      const int sb = wg;
      const int sl = g % C::NL;
      if (!mbar_wait_warp(&s_full[sb], (g / kMassConsumers) & 1, wctx, MCS_WHERE_MASS_CONSUMER)) break;
      tc_fence_after();
      // the group's lse slice; not refilled before this warpgroup arrives on l_empty below
      if (!mbar_wait_warp(&l_full[sl], (g / C::NL) & 1, wctx, MCS_WHERE_MASS_CONSUMER)) break;
      // p = 2^(s * scale * log2e - lse2) over the group's 128 query rows, in
      // two halves of 64 columns and in pairs: one packed fused multiply-add with -lse2,
      // MUFU ex2 for three pairs in four and the FMA-pipe polynomial for the
      // fourth (rows past N have -lse2 = -inf and give 0 either way), packed
      // accumulation; the S buffer is released once both halves are loaded
      const float2* lse2 = reinterpret_cast<const float2*>(sL + sl * 128);  // -lse, log2 units
      uint64_t acc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = f2_pack(0.f, 0.f);
#pragma unroll 1
      for (int hv = 0; hv < 2; ++hv) {  // rolled: one half's 64 scores live at a time
        float sv[64];
        tmem_ld32(tmem + lane_addr + sb * 128 + hv * 64, sv);
        tmem_ld32(tmem + lane_addr + sb * 128 + hv * 64 + 32, sv + 32);
        tmem_wait_ld();
        if (hv == 1) {
          tc_fence_before();
          mbar_arrive(&s_empty[sb]);
        }
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const float2 l = lse2[hv * 32 + q];
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(sv[2 * q], sv[2 * q + 1]), c2, f2_pack(l.x, l.y)), x0, x1);
          if ((q & 3) == 3) {
            exp2_poly2(x0, x1);
          } else {
            x0 = fast_exp2(x0);
            x1 = fast_exp2(x1);
          }
          acc[q & 3] = f2_add(acc[q & 3], f2_pack(x0, x1));
        }
      }
      mbar_arrive(&l_empty[sl]);
      float r[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) f2_unpack(acc[i], r[2 * i], r[2 * i + 1]);
      if (key < p.N)
        out[static_cast<size_t>(rot(g)) * p.N + key] = ((r[0] + r[1]) + (r[2] + r[3])) + ((r[4] + r[5]) + (r[6] + r[7]));
    }
  }

  __syncthreads();
  if (*abort_flag) {
    volatile int never = 0;
    const WaitCtx drain_ctx{&never, nullptr, 50000000ull};
    if (warp == 0 && lane == 0)
      for (int g = max(0, issued - C::NL); g < issued; ++g) {
        if (g >= issued - C::NQ) mbar_wait(&q_full[g % C::NQ], (g / C::NQ) & 1, drain_ctx, MCS_WHERE_DRAIN);
        mbar_wait(&l_full[g % C::NL], (g / C::NL) & 1, drain_ctx, MCS_WHERE_DRAIN);
      }
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
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kBandMax = 2048;
constexpr int kUnroll = 8;          // sweep steps whose loads are issued together (the mass row streams from L2)
constexpr int kBinShift = 20;       // two-sweep path: bins of key >> 20 (sign, exponent, top 3 mantissa bits)
constexpr int kBins = 1 << (32 - kBinShift);
constexpr uint32_t kBinNonFinite = 0x7F800000u >> kBinShift;  // first bin of +inf / NaN keys
constexpr int kCandMax = 8192;      // keys of the K-th largest key's bin held in shared memory
static_assert(kBins == 4 * kTopkThreads, "each thread owns four bins in the bin scan");

enum {  // TopkSmem::scalars
  SC_BIN = 0, SC_ABOVE, SC_HIGH, SC_NCAND, SC_DIG, SC_ACC, SC_NBAND, SC_ABOVE_HI, SC_TOTAL,
  SC_BAND, SC_CIN, SC_EQ, SC_COUNT = 16
};

struct TopkSmem {
  union {
    int whist[kTopkWarps][256];  // seven-sweep path: warp-private digit histograms
    int bins[kBins];             // two-sweep path: key-bin histogram, then candidate digit histograms
  };
  int hist[256];
  int band_idx[kBandMax];
  double band_m[kBandMax];
  double nlse2[128];            // the group's negated lse, log2 units (hi + lo, in fp64)
  int wcnt[kTopkWarps][4];     // per warp segment: band, above hi, above T, equal T
  int woff[kTopkWarps][4];     // exclusive offsets of the same
  int wsel[kTopkWarps];        // selected band keys per warp segment
  int wout[kTopkWarps];        // output offset per warp segment
  int wscan[kTopkWarps];       // block scans: per-warp totals
  int scalars[SC_COUNT];
};

// Dynamic shared memory: TopkSmem | selection bitmap (N bits) | group queries fp32 128 x (d+1) |
// candidate keys | candidate indices.
struct TopkLayout {
  size_t sel, qrows, cand_key, cand_idx, base_bytes;
};

__host__ __device__ inline TopkLayout topk_layout(int N, int d, int cap) {
  TopkLayout L;
  L.sel = sizeof(TopkSmem);
  L.qrows = L.sel + static_cast<size_t>(((N + 31) / 32 + 3) / 4 * 4) * 4;
  L.cand_key = L.qrows + 128ull * (d + 1) * 4;
  L.base_bytes = L.cand_key;
  L.cand_idx = L.cand_key + static_cast<size_t>(cap) * 4;
  return L;
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Inclusive prefix sum of v over the block's threads in thread order. Ends with a barrier.
__device__ __forceinline__ int block_incl_scan(int v, int* wscan) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wscan[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int w = wscan[lane];
    int z = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, z, o);
      if (lane >= o) z += y;
    }
    wscan[lane] = z - w;
  }
  __syncthreads();
  return x + wscan[warp];
}

// The group's queries as fp32 rows (padded to d+1) and their lse: the operands of the fp64 re-scoring.
__device__ void stage_group_queries(const TopkParams& p, TopkSmem& S, float* qrows, int b, int h, int g,
                                    size_t head_base) {
  const int N = p.N, d = p.d, ld = d + 1, c8n = d / 8;
  const int nrows = min(128, N - g * 128);
  for (int e = threadIdx.x; e < 128 * c8n; e += kTopkThreads) {
    const int r = e / c8n, c8 = e % c8n;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (r < nrows) {
      const int tok = p.perm[head_base * N + g * 128 + r];
      w = __ldg(reinterpret_cast<const uint4*>(p.q + ((static_cast<size_t>(b) * N + tok) * p.H + h) * d) + c8);
    }
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
    float* dst = qrows + r * ld + c8 * 8;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      dst[2 * t] = __uint_as_float(u[t] << 16);
      dst[2 * t + 1] = __uint_as_float(u[t] & 0xffff0000u);
    }
  }
  if (threadIdx.x < 128) {
    const size_t r = head_base * (static_cast<size_t>(p.G) * 128) + g * 128 + threadIdx.x;
    S.nlse2[threadIdx.x] = static_cast<double>(p.lse_perm[r]) + static_cast<double>(p.lse_perm_lo[r]);
  }
}

// fp64 re-scoring of the nband keys in S.band_idx (exact bf16 products, double exp, the dense pass's lse),
// then ranking by (mass desc, index asc): the first `take` get their bit set in `selbits` (and, when
// seg > 0, are counted per warp segment of `seg` keys in S.wsel). Starts and ends with a barrier.
__device__ void rescore_and_select(const TopkParams& p, TopkSmem& S, float* qrows, uint32_t* selbits, int nband,
                                   int take, int b, int h, int g, size_t head_base, int seg) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  stage_group_queries(p, S, qrows, b, h, g, head_base);
  __syncthreads();
  const int N = p.N, ld = p.d + 1;
  const int nrows = min(128, N - g * 128);
  const double scale = p.scale;
  const double ln2 = 0.693147180559945309417232121458;
  // one warp per band key, lanes over the group's queries (rows lane + 32i, four independent sums);
  // the key row is staged as fp32 in the warp's slice of the (now unused) histogram space
  float* kf = reinterpret_cast<float*>(S.bins) + warp * (kBins / kTopkWarps);
  static_assert(kBins / kTopkWarps >= 128, "a warp's slice holds one key row");
  for (int t = warp; t < nband; t += kTopkWarps) {
    const int j = S.band_idx[t];
    const uint16_t* krow = p.k + ((static_cast<size_t>(b) * N + j) * p.H + h) * p.d;
    for (int c = lane; c < p.d; c += 32) kf[c] = __uint_as_float(static_cast<uint32_t>(__ldg(krow + c)) << 16);
    __syncwarp();
    double dot[4] = {0.0, 0.0, 0.0, 0.0};
    for (int c = 0; c < p.d; ++c) {
      const double kc = static_cast<double>(kf[c]);
#pragma unroll
      for (int i = 0; i < 4; ++i) dot[i] = fma(static_cast<double>(qrows[(lane + 32 * i) * ld + c]), kc, dot[i]);
    }
    double acc = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = lane + 32 * i;
      if (r < nrows) acc += exp(dot[i] * scale + S.nlse2[r] * ln2);
    }
    __syncwarp();
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) S.band_m[t] = acc;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < nband; t += kTopkThreads) {
    const double mt = S.band_m[t];
    const int jt = S.band_idx[t];
    int rank = 0;
    for (int u = 0; u < nband; ++u) {
      const double mu = S.band_m[u];
      rank += (mu > mt || (mu == mt && S.band_idx[u] < jt)) ? 1 : 0;
    }
    if (rank < take) {
      atomicOr(&selbits[jt >> 5], 1u << (jt & 31));
      if (seg > 0) atomicAdd(&S.wsel[jt / seg], 1);
    }
  }
  if (threadIdx.x == 0) atomicAdd(p.status + MCS_SW_REFINED, nband);
  __syncthreads();
}

// The general selection: a 4 x 8-bit radix select of the K-th largest key, then sweeps for the per-segment
// counts, the band, and the ordered write. Handles every input, including bands wider than kBandMax
// (fp32 ranking, ties to the lower index) and keys that are not finite and non-negative.
__device__ __noinline__ void topk_full_sweeps(const TopkParams& p, TopkSmem& S, uint32_t* selbits, float* qrows,
                                              int b, int h, int g, size_t head_base, const float* mrow,
                                              int32_t* outp) {
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int N = p.N;
  uint32_t prefix = 0, pmask = 0;
  int need = p.K;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = lane; i < 256; i += 32) S.whist[warp][i] = 0;
    __syncthreads();
    for (int base = 0; base < N; base += kTopkThreads * kUnroll) {
      uint32_t kb[kUnroll];  // loads of kUnroll sweep steps in flight at once
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = base + u * kTopkThreads + tid;
        kb[u] = j < N ? __float_as_uint(mrow[j]) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = base + u * kTopkThreads + tid;
        const uint32_t key = kb[u];
        const bool in = (j < N) && ((key & pmask) == prefix);
        const unsigned act = __ballot_sync(0xffffffffu, in);
        if (in) {
          const uint32_t digit = (key >> shift) & 255u;
          const unsigned peers = __match_any_sync(act, digit);
          if (lane == __ffs(peers) - 1) atomicAdd(&S.whist[warp][digit], __popc(peers));
        }
      }
    }
    __syncthreads();
    if (tid < 256) {
      int t = 0;
      for (int w = 0; w < kTopkWarps; ++w) t += S.whist[w][tid];
      S.hist[tid] = t;
    }
    __syncthreads();
    if (warp == 0) {  // lane l owns bins [248 - 8l, 256 - 8l); walk from the top
      int sum = 0;
      for (int i = 0; i < 8; ++i) sum += S.hist[255 - 8 * lane - i];
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int excl = incl - sum;
      if (excl < need && incl >= need) {
        int acc = excl;
        for (int i = 0; i < 8; ++i) {
          const int bin = 255 - 8 * lane - i;
          if (acc + S.hist[bin] >= need) {
            S.scalars[SC_DIG] = bin;
            S.scalars[SC_ACC] = acc;
            break;
          }
          acc += S.hist[bin];
        }
      }
    }
    __syncthreads();
    need -= S.scalars[SC_ACC];
    prefix |= static_cast<uint32_t>(S.scalars[SC_DIG]) << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t Tkey = prefix;  // the K-th largest key; `need` keys equal to it complete the fp32 ranking
  const float Tval = __uint_as_float(Tkey);
  const float hi = Tval * (1.f + p.band_rel);
  const float lo = Tval * (1.f - p.band_rel);

  // warp segments: counts of band / above-hi / above-T / equal-T keys
  const int seg = ((N + kTopkWarps - 1) / kTopkWarps + 31) / 32 * 32;
  const int s0 = min(N, warp * seg), s1 = min(N, s0 + seg);
  {
    int c[4] = {0, 0, 0, 0};
    for (int base0 = s0; base0 < s1; base0 += 32 * kUnroll) {
      float mb[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = base0 + 32 * u + lane;
        mb[u] = j < s1 ? mrow[j] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = base0 + 32 * u + lane;
        const float m = mb[u];
        const uint32_t key = __float_as_uint(m);
        const bool valid = j < s1;
        c[0] += __popc(__ballot_sync(0xffffffffu, valid && m >= lo && m <= hi));
        c[1] += __popc(__ballot_sync(0xffffffffu, valid && m > hi));
        c[2] += __popc(__ballot_sync(0xffffffffu, valid && key > Tkey));
        c[3] += __popc(__ballot_sync(0xffffffffu, valid && key == Tkey));
      }
    }
    if (lane < 4) S.wcnt[warp][lane] = c[lane];
    if (lane == 0) S.wsel[warp] = 0;
  }
  for (int i = tid; i < (N + 31) / 32; i += kTopkThreads) selbits[i] = 0;
  __syncthreads();
  if (tid < 4) {
    int acc = 0;
    for (int w = 0; w < kTopkWarps; ++w) {
      S.woff[w][tid] = acc;
      acc += S.wcnt[w][tid];
    }
    S.scalars[SC_BAND + tid] = acc;  // totals: band, above hi, above T, equal T
  }
  __syncthreads();
  const int nband = S.scalars[SC_BAND];
  const int c_in = S.scalars[SC_CIN];
  const bool overflow = nband > kBandMax;
  const int take = p.K - c_in;  // 1 <= take <= nband

  if (!overflow) {
    // collect the band in index order
    int off = S.woff[warp][0];
    for (int base0 = s0; base0 < s1; base0 += 32 * kUnroll) {
      float mb[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = base0 + 32 * u + lane;
        mb[u] = j < s1 ? mrow[j] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = base0 + 32 * u + lane;
        const bool inb = j < s1 && mb[u] >= lo && mb[u] <= hi;
        const unsigned bal = __ballot_sync(0xffffffffu, inb);
        if (inb) S.band_idx[off + __popc(bal & lanemask_lt())] = j;
        off += __popc(bal);
      }
    }
    rescore_and_select(p, S, qrows, selbits, nband, take, b, h, g, head_base, seg);
  } else {
    if (tid == 0) atomicAdd(p.status + MCS_SW_BAND_OVERFLOW, 1);
    __syncthreads();
  }
  // output offsets per warp segment, then the ordered write
  if (tid == 0) {
    int acc = 0;
    for (int w = 0; w < kTopkWarps; ++w) {
      S.wout[w] = acc;
      if (!overflow) {
        acc += S.wcnt[w][1] + S.wsel[w];
      } else {
        const int eq_take = max(0, min(S.wcnt[w][3], need - S.woff[w][3]));
        acc += S.wcnt[w][2] + eq_take;
      }
    }
    S.scalars[SC_TOTAL] = acc;
  }
  __syncthreads();
  {
    int off = S.wout[warp];
    int eq_seen = S.woff[warp][3];
    for (int base0 = s0; base0 < s1; base0 += 32 * kUnroll) {
      float mb[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = base0 + 32 * u + lane;
        mb[u] = j < s1 ? mrow[j] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = base0 + 32 * u + lane;
        const bool valid = j < s1;
        const float m = mb[u];
        bool flag;
        if (!overflow) {
          flag = valid && (m > hi || ((selbits[j >> 5] >> (j & 31)) & 1u));
        } else {
          const uint32_t key = __float_as_uint(m);
          const bool eq = valid && key == Tkey;
          const unsigned eqb = __ballot_sync(0xffffffffu, eq);
          flag = valid && (key > Tkey || (eq && eq_seen + __popc(eqb & lanemask_lt()) < need));
          eq_seen += __popc(eqb);
        }
        const unsigned fb = __ballot_sync(0xffffffffu, flag);
        if (flag) {
          const int pos = off + __popc(fb & lanemask_lt());
          if (pos < p.K) outp[pos] = j;
        }
        off += __popc(fb);
      }
    }
  }
  if (tid == 0 && S.scalars[SC_TOTAL] != p.K) record_status(p.status, MCS_ERR_BAD_INDEX, -1000000 - S.scalars[SC_TOTAL]);
}
}  // namespace

// One CTA per (b, h, g). The usual case takes two sweeps over the group's mass row:
//  1. a histogram of key >> 20 (4096 bins of 1/8 binade) locates the bin d1 holding the K-th largest key;
//  2. keys above d1 go into a shared-memory bitmap (they are above the band: see below) and the keys of
//     bin d1 into a shared-memory list.
// The exact K-th largest key T comes from a radix select over that list; when the band [T(1-eps), T(1+eps)]
// lies inside bin d1, every band key is in the list, the band is re-scored and ranked as in the general
// path, and the selection is written from the bitmap in ascending index order. Otherwise (bin d1 larger
// than the list, a band crossing a bin edge, more than kBandMax band keys, keys that are not finite and
// non-negative) the CTA runs the general seven-sweep selection, which gives the same result.
__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(const TopkParams p) {
  extern __shared__ uint8_t smem_raw[];
  const TopkLayout L = topk_layout(p.N, p.d, p.cand_cap);
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(smem_raw);
  uint32_t* selbits = reinterpret_cast<uint32_t*>(smem_raw + L.sel);
  float* qrows = reinterpret_cast<float*>(smem_raw + L.qrows);
  uint32_t* cand_key = reinterpret_cast<uint32_t*>(smem_raw + L.cand_key);
  int* cand_idx = reinterpret_cast<int*>(smem_raw + L.cand_idx);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.x % p.G;
  const int bh = blockIdx.x / p.G;
  const int b = bh / p.hn;
  const int hl = bh % p.hn;
  const int h = p.h0 + hl;
  const size_t head_base = static_cast<size_t>(b) * p.H + h;
  const float* mrow = p.mass + ((static_cast<size_t>(b) * p.hn + hl) * p.G + g) * static_cast<size_t>(p.N);
  int32_t* outp = p.kv_idx + (head_base * p.G + g) * static_cast<size_t>(p.K);
  const int N = p.N;

  // ---- sweep 1: histogram of key >> 20
  for (int i = tid; i < kBins; i += kTopkThreads) S.bins[i] = 0;
  if (tid == 0) {
    S.scalars[SC_NCAND] = 0;
    S.scalars[SC_NBAND] = 0;
    S.scalars[SC_ABOVE_HI] = 0;
    S.scalars[SC_HIGH] = 0;
  }
  __syncthreads();
  for (int base = 0; base < N; base += kTopkThreads * kUnroll) {
    uint32_t kb[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int j = base + u * kTopkThreads + tid;
      kb[u] = j < N ? __float_as_uint(mrow[j]) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int j = base + u * kTopkThreads + tid;
      if (j < N) atomicAdd(&S.bins[kb[u] >> kBinShift], 1);
    }
  }
  __syncthreads();
  // ---- the bin d1 of the K-th largest key: thread t owns bins 4095-4t down to 4092-4t
  {
    int c4[4], sum = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      c4[i] = S.bins[kBins - 1 - 4 * tid - i];
      sum += c4[i];
    }
    const int incl = block_incl_scan(sum, S.wscan);
    const int excl = incl - sum;
    if (excl < p.K && incl >= p.K) {
      int acc = excl;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (acc + c4[i] >= p.K) {
          S.scalars[SC_BIN] = kBins - 1 - 4 * tid - i;
          S.scalars[SC_ABOVE] = acc;
          break;
        }
        acc += c4[i];
      }
    }
    // keys in bins >= kBinNonFinite (+inf, NaN, negative): thread (kBins - kBinNonFinite) / 4 - 1 ends there
    if (tid == (kBins - static_cast<int>(kBinNonFinite)) / 4 - 1) S.scalars[SC_HIGH] = incl;
  }
  __syncthreads();
  const int d1 = S.scalars[SC_BIN];
  const int above = S.scalars[SC_ABOVE];  // keys in bins above d1
  const int ncand = S.bins[d1];
  bool fast = !p.force_full && ncand <= p.cand_cap && S.scalars[SC_HIGH] == 0;  // block-uniform
  __syncthreads();

  if (fast) {
    // ---- sweep 2: bins above d1 into the bitmap (one ballot word per warp step), bin d1 into the list
    for (int base = 0; base < N; base += kTopkThreads * kUnroll) {
      uint32_t kb[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = base + u * kTopkThreads + tid;
        kb[u] = j < N ? __float_as_uint(mrow[j]) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = base + u * kTopkThreads + tid;
        const int j0 = j - lane;  // first key of this warp's 32-key word
        const bool valid = j < N;
        const uint32_t bin = kb[u] >> kBinShift;
        const unsigned word = __ballot_sync(0xffffffffu, valid && bin > static_cast<uint32_t>(d1));
        if (lane == 0 && j0 < N) selbits[j0 >> 5] = word;
        const bool isc = valid && bin == static_cast<uint32_t>(d1);
        const unsigned cb = __ballot_sync(0xffffffffu, isc);
        if (cb) {
          int off = 0;
          if (lane == 0) off = atomicAdd(&S.scalars[SC_NCAND], __popc(cb));
          off = __shfl_sync(0xffffffffu, off, 0);
          const int c = off + __popc(cb & lanemask_lt());
          if (isc && c < p.cand_cap) {
            cand_key[c] = kb[u];
            cand_idx[c] = j;
          }
        }
      }
    }
    __syncthreads();
    // ---- exact K-th largest key: radix select over the list (bits 19..10, then 9..0)
    uint32_t prefix = static_cast<uint32_t>(d1) << kBinShift, pmask = ~0u << kBinShift;
    int need = p.K - above;  // 1 <= need <= ncand
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = 10 - 10 * pass;
      S.bins[tid] = 0;
      __syncthreads();
      for (int c = tid; c < ncand; c += kTopkThreads) {
        const uint32_t key = cand_key[c];
        if ((key & pmask) == prefix) atomicAdd(&S.bins[(key >> shift) & 1023u], 1);
      }
      __syncthreads();
      const int v = S.bins[1023 - tid];  // thread t owns digit 1023 - t
      const int incl = block_incl_scan(v, S.wscan);
      if (incl - v < need && incl >= need) {
        S.scalars[SC_DIG] = 1023 - tid;
        S.scalars[SC_ACC] = incl - v;
      }
      __syncthreads();
      need -= S.scalars[SC_ACC];
      prefix |= static_cast<uint32_t>(S.scalars[SC_DIG]) << shift;
      pmask |= 1023u << shift;
      __syncthreads();
    }
    const float Tval = __uint_as_float(prefix);
    const float hi = Tval * (1.f + p.band_rel);
    const float lo = Tval * (1.f - p.band_rel);
    fast = (__float_as_uint(hi) >> kBinShift) == static_cast<uint32_t>(d1) &&
           (__float_as_uint(lo) >> kBinShift) == static_cast<uint32_t>(d1);
    if (fast) {
      // ---- classify the list: above the band (bitmap), in the band (band list)
      for (int c0 = 0; c0 < ncand; c0 += kTopkThreads) {
        const int c = c0 + tid;
        const bool valid = c < ncand;
        const float m = valid ? __uint_as_float(cand_key[c]) : 0.f;
        const int j = valid ? cand_idx[c] : 0;
        const bool up = valid && m > hi;
        const bool inb = valid && m >= lo && m <= hi;
        if (up) atomicOr(&selbits[j >> 5], 1u << (j & 31));
        const unsigned ub = __ballot_sync(0xffffffffu, up);
        if (lane == 0 && ub) atomicAdd(&S.scalars[SC_ABOVE_HI], __popc(ub));
        const unsigned bb = __ballot_sync(0xffffffffu, inb);
        if (bb) {
          int off = 0;
          if (lane == 0) off = atomicAdd(&S.scalars[SC_NBAND], __popc(bb));
          off = __shfl_sync(0xffffffffu, off, 0);
          const int t = off + __popc(bb & lanemask_lt());
          if (inb && t < kBandMax) S.band_idx[t] = j;
        }
      }
      __syncthreads();
      const int nband = S.scalars[SC_NBAND];
      const int take = p.K - above - S.scalars[SC_ABOVE_HI];  // 1 <= take <= nband
      fast = nband <= kBandMax;
      if (fast) rescore_and_select(p, S, qrows, selbits, nband, take, b, h, g, head_base, 0);
    }
  }
  if (!fast) {
    if (tid == 0) atomicAdd(p.status + MCS_SW_TOPK_FULL, 1);
    __syncthreads();
    topk_full_sweeps(p, S, selbits, qrows, b, h, g, head_base, mrow, outp);
    return;
  }
  // ---- ordered write from the bitmap: warp w owns a contiguous range of words
  const int nwords = (N + 31) / 32;
  const int wpw = (nwords + kTopkWarps - 1) / kTopkWarps;
  const int w0 = min(nwords, warp * wpw), w1 = min(nwords, w0 + wpw);
  {
    int cnt = 0;
    for (int i = w0 + lane; i < w1; i += 32) cnt += __popc(selbits[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) S.wout[warp] = cnt;
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int w = 0; w < kTopkWarps; ++w) {
      const int c = S.wout[w];
      S.wout[w] = acc;
      acc += c;
    }
    S.scalars[SC_TOTAL] = acc;
  }
  __syncthreads();
  int off = S.wout[warp];
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int i = i0 + lane;
    uint32_t bits = i < w1 ? selbits[i] : 0u;
    const int c = __popc(bits);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = off + incl - c;
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      if (pos < p.K) outp[pos] = i * 32 + bit;
      ++pos;
    }
    off += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (tid == 0 && S.scalars[SC_TOTAL] != p.K) record_status(p.status, MCS_ERR_BAD_INDEX, -1000000 - S.scalars[SC_TOTAL]);
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

cudaError_t launch_permute_queries(const uint16_t* q, const int32_t* perm, uint16_t* qp, int B, int H, int N, int G,
                                   int d, int* status, cudaStream_t s) {
  permute_queries<<<148 * 8, 256, 0, s>>>(q, perm, qp, B, H, N, G, d, status);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_mass(int d, const CUtensorMap* tq, const CUtensorMap* tk, const MassParams& p, cudaStream_t s) {
  if (d == 128) return launch_mass_t<128>(tq, tk, p, s);
  if (d == 64) return launch_mass_t<64>(tq, tk, p, s);
  return cudaErrorInvalidValue;
}

size_t topk_smem_bytes(int N, int d) { return topk_layout(N, d, 0).base_bytes; }

cudaError_t launch_topk(const TopkParams& p0, cudaStream_t s) {
  constexpr size_t kSmemMax = 227 * 1024;
  const size_t base = topk_smem_bytes(p0.N, p0.d);
  if (base > kSmemMax) return cudaErrorInvalidValue;
  TopkParams p = p0;
  // the candidate list takes what shared memory is left, up to kCandMax keys (8 bytes each)
  const size_t room = (kSmemMax - base) / 8;
  p.cand_cap = static_cast<int>(room < static_cast<size_t>(kCandMax) ? room : kCandMax) & ~31;
  const size_t smem = topk_layout(p.N, p.d, p.cand_cap).cand_idx + static_cast<size_t>(p.cand_cap) * 4;
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  topk_kernel<<<p.B * p.hn * p.G, kTopkThreads, smem, s>>>(p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace mcs
