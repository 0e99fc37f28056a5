// Anchor passes 2 and 3 of MC-Sparse (aiwillknow analysis, step 2; paper
// Table 4 "token" granularity): exact attention probabilities from a second
// QK^T pass, per-group probability mass, and token-level top-K selection.
//
// Mass pass: one CTA per (b, h, 128-key tile). It keeps its K tile in shared
// memory and streams every query group of the head (from a copy of Q laid out
// in group order, one tiled TMA box per group) through S^T = K_tile Q_g^T
// (UMMA, M = 128 keys, N = 128 queries). Three consumer warpgroups take the
// groups in turn, each with its own TMEM S buffer, so one warpgroup's loads and
// reductions overlap the others' exponentials. Each TMEM lane is one key, so a
// consumer thread turns its 128 columns
// into probabilities
// p_ij = 2^(s_ij*scale*log2e - lse2_i) (lse2 = lse*log2e) and sums them: m_g(j) with no
// cross-thread reduction. Output: fp32 mass [B, hn, G, N].
//
// Top-K: one CTA per (b, h, g). A 3-pass radix select (11/11/10 bits of the
// fp32 key) finds the K-th largest mass T. Keys above T(1+eps) are taken, keys
// below T(1-eps) dropped; keys in the band are re-scored in fp64 (exact bf16
// products, double exp, the dense pass's lse) and ranked by (mass desc, index
// asc). The selection is written in ascending index order.
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
  static constexpr int NQ = 5;  // query-tile stages
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_Q = TILE;
  static constexpr uint32_t OFF_LSE = OFF_Q + NQ * TILE;  // NQ x 128 floats
  static constexpr uint32_t OFF_BAR = OFF_LSE + NQ * 512;
  static constexpr uint32_t NBAR = 1 + 2 * NQ + 2 * kMassConsumers + 1;
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
  uint64_t* s_full = q_empty + C::NQ; // [kMassConsumers]: buffer c holds the groups of consumer warpgroup c
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
      mbar_init(&q_empty[i], 1 + 128);  // UMMA done (commit) + the consumer warpgroup read the lse slice
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
        const int st = g % C::NQ;
        if (g >= C::NQ && !mbar_wait(&q_empty[st], ((g / C::NQ) & 1) ^ 1, wctx, MCS_WHERE_MASS_PRODUCER)) break;
        mbar_arrive_expect_tx(&q_full[st], C::TILE + 512);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_2d(&tm_qp, &q_full[st], sQ + st * C::TILE + kb * 16384, kb * 64, qrow0 + g * 128);
        bulk_copy_g2s(sL + st * 128, p.lse_perm + head_base * (static_cast<size_t>(p.G) * 128) + g * 128, 512,
                      &q_full[st]);
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
      const int st = g % C::NQ;
      if (!mbar_wait_warp(&s_full[sb], (g / kMassConsumers) & 1, wctx, MCS_WHERE_MASS_CONSUMER)) break;
      tc_fence_after();
      // the group's lse slice arrived with its query tile; the stage is not
      // refilled before this warpgroup arrives on q_empty below
      if (!mbar_wait_warp(&q_full[st], (g / C::NQ) & 1, wctx, MCS_WHERE_MASS_CONSUMER)) break;
      // p = 2^(s * scale * log2e - lse2) over the group's 128 query rows, in
      // two halves of 64 columns and in pairs: packed multiply and subtract,
      // MUFU ex2 for three pairs in four and the FMA-pipe polynomial for the
      // fourth (rows past N have lse2 = +inf and give 0 either way), packed
      // accumulation; the S buffer is released once both halves are loaded
      const float2* lse2 = reinterpret_cast<const float2*>(sL + st * 128);  // log2 units
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
          f2_unpack(f2_sub(f2_mul(f2_pack(sv[2 * q], sv[2 * q + 1]), c2), f2_pack(l.x, l.y)), x0, x1);
          if ((q & 3) == 3) {
            exp2_poly2(x0, x1);
          } else {
            x0 = fast_exp2(x0);
            x1 = fast_exp2(x1);
          }
          acc[q & 3] = f2_add(acc[q & 3], f2_pack(x0, x1));
        }
      }
      mbar_arrive(&q_empty[st]);
      float r[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) f2_unpack(acc[i], r[2 * i], r[2 * i + 1]);
      if (key < p.N)
        out[static_cast<size_t>(g) * p.N + key] = ((r[0] + r[1]) + (r[2] + r[3])) + ((r[4] + r[5]) + (r[6] + r[7]));
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
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kBandMax = 2048;
constexpr int kUnroll = 8;  // sweep steps whose loads are issued together (the mass row streams from L2)

struct TopkSmem {
  int whist[kTopkWarps][256];  // warp-private digit histograms
  int hist[256];
  int band_idx[kBandMax];
  double band_m[kBandMax];
  float lse2[128];
  int wcnt[kTopkWarps][4];     // per warp segment: band, above hi, above T, equal T
  int woff[kTopkWarps][4];     // exclusive offsets of the same
  int wsel[kTopkWarps];        // selected band keys per warp segment
  int wout[kTopkWarps];        // output offset per warp segment
  int scalars[8];
};

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}
}  // namespace

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(const TopkParams p) {
  extern __shared__ uint8_t smem_raw[];
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(smem_raw);
  uint32_t* selbits = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkSmem));  // N bits
  const int nsel_words = ((p.N + 31) / 32 + 3) / 4 * 4;
  float* qrows = reinterpret_cast<float*>(selbits + nsel_words);                   // 128 x (d+1) fp32

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

  // ---------------- radix select of the K-th largest fp32 key (4 x 8 bits, MSB first)
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
            S.scalars[0] = bin;
            S.scalars[1] = acc;
            break;
          }
          acc += S.hist[bin];
        }
      }
    }
    __syncthreads();
    need -= S.scalars[1];
    prefix |= static_cast<uint32_t>(S.scalars[0]) << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t Tkey = prefix;  // the K-th largest key; `need` keys equal to it complete the fp32 ranking
  const float Tval = __uint_as_float(Tkey);
  const float hi = Tval * (1.f + p.band_rel);
  const float lo = Tval * (1.f - p.band_rel);

  // ---------------- warp segments: counts of band / above-hi / above-T / equal-T keys
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
    S.scalars[2 + tid] = acc;  // totals: band, above hi, above T, equal T
  }
  __syncthreads();
  const int nband = S.scalars[2];
  const int c_in = S.scalars[3];
  const bool overflow = nband > kBandMax;
  const int take = p.K - c_in;  // 1 <= take <= nband

  if (!overflow) {
    // collect the band in index order
    {
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
    }
    // this group's queries (fp32, rows padded to d+1) and their lse
    const int nrows = min(128, N - g * 128);
    const int ld = p.d + 1;
    for (int e = tid; e < 128 * p.d; e += kTopkThreads) {
      const int r = e / p.d, c = e % p.d;
      float x = 0.f;
      if (r < nrows) {
        const int tok = p.perm[head_base * N + g * 128 + r];
        x = __uint_as_float(static_cast<uint32_t>(p.q[((static_cast<size_t>(b) * N + tok) * p.H + h) * p.d + c])
                            << 16);
      }
      qrows[r * ld + c] = x;
    }
    if (tid < 128) S.lse2[tid] = p.lse_perm[head_base * (static_cast<size_t>(p.G) * 128) + g * 128 + tid];
    __syncthreads();
    // fp64 re-scoring: one warp per band key, lanes over the group's queries
    const double scale = p.scale;
    const double ln2 = 0.693147180559945309417232121458;
    for (int t = warp; t < nband; t += kTopkWarps) {
      const int j = S.band_idx[t];
      const uint16_t* krow = p.k + ((static_cast<size_t>(b) * N + j) * p.H + h) * p.d;
      double acc = 0.0;
      for (int r = lane; r < nrows; r += 32) {
        const float* qr = qrows + r * ld;
        double dot = 0.0;
        for (int c = 0; c < p.d; ++c)
          dot = fma(static_cast<double>(qr[c]),
                    static_cast<double>(__uint_as_float(static_cast<uint32_t>(__ldg(krow + c)) << 16)), dot);
        acc += exp(dot * scale - static_cast<double>(S.lse2[r]) * ln2);
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
      if (rank < take) {
        atomicOr(&selbits[jt >> 5], 1u << (jt & 31));
        atomicAdd(&S.wsel[jt / seg], 1);
      }
    }
    if (tid == 0) atomicAdd(p.status + MCS_SW_REFINED, nband);
  } else {
    if (tid == 0) atomicAdd(p.status + MCS_SW_BAND_OVERFLOW, 1);
  }
  __syncthreads();
  // ---------------- output offsets per warp segment, then the ordered write
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
    S.scalars[6] = acc;
  }
  __syncthreads();
  int32_t* outp = p.kv_idx + (head_base * p.G + g) * static_cast<size_t>(p.K);
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
  if (tid == 0 && S.scalars[6] != p.K) record_status(p.status, MCS_ERR_BAD_INDEX, -1000000 - S.scalars[6]);
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

size_t topk_smem_bytes(int N, int d) {
  return sizeof(TopkSmem) + static_cast<size_t>(((N + 31) / 32 + 3) / 4 * 4) * 4 + 128ull * (d + 1) * 4;
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
