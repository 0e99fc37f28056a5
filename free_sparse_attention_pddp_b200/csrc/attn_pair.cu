// Dense attention over PAIRS of 128-query tiles per CTA (d = 128): the dense
// baseline (ATTN_DENSE), same arithmetic and outputs as the one-tile kernel in
// attn.cu, which keeps the anchor's dense pass (measured: this layout is
// about 5 % faster for plain attention and about 1.5 % slower with the anchor's
// fp64 row sums and lse export).
//
// Why pairs: with one query tile per CTA, the softmax of a key tile has to
// finish before its PV product, and its two key-half warps on each SM
// sub-partition run the same phases at the same time, so the tile period is
// the softmax's own latency chain. Here the two query tiles A and B of a CTA
// share every K/V tile and the tensor pipe alternates between them:
//   S_A(j) = Q_A K_j^T | O_B += P_B(j-1) V_j-1 | S_B(j) = Q_B K_j^T | O_A += P_A(j) V_j
// so the softmax of A's key tile j runs while the pipe computes B's products
// and the other way round: the two softmax warpgroups (one per tile, one
// thread per query row, all 128 keys of the tile) work out of phase.
//
// TMEM (512 columns): S_A | S_B | O_A | O_B, 128 each; P_t (bf16 pairs, key k
// in column k/2) overwrites the first 64 columns of S_t and is the TS-form A
// operand of O_t += P_t V. Online softmax with a lazy rescale of O_t, as in
// attn.cu.
//
// Threads (384): warp 0 issues the UMMAs (lane 0), warps 1-3 gather the two
// query tiles (tile::gather4) and stream K/V tiles with tiled TMA (two
// stages), warps 4-7 run tile A's softmax, warps 8-11 tile B's. setmaxnreg
// moves registers from warpgroup 0 (64) to the softmax warpgroups (216).
#include <cuda_bf16.h>
#include <math_constants.h>

#include "mcs_ptx.cuh"

namespace mcs {

namespace {

constexpr int kPairThreads = 384;
constexpr int kPairLaunchRegs = 168;  // 65536 / 384 rounded down to a multiple of 8
constexpr int kPairLowRegs = 64;      // warpgroup 0: UMMA issuer and producers
constexpr int kPairSoftRegs = 216;    // the two softmax warpgroups (no spills in either role)
static_assert(128 * kPairLowRegs + 256 * kPairSoftRegs <= kPairThreads * kPairLaunchRegs, "register split");
constexpr float kPairRescaleThreshold = 4.0f;  // log2 units, as in attn.cu

struct PairCfg {
  static constexpr int D = 128;
  static constexpr int KB = D / 64;
  static constexpr uint32_t TILE = 128u * D * 2u;  // 32 KB: one 128-row bf16 tile
  static constexpr int NS = 2;                      // K/V stages
  static constexpr uint32_t OFF_Q = 0;              // Q_A, Q_B
  static constexpr uint32_t OFF_K = 2 * TILE;
  static constexpr uint32_t OFF_V = OFF_K + NS * TILE;
  static constexpr uint32_t OFF_BAR = OFF_V + NS * TILE;
  // q_full[2], k_full[NS], v_full[NS], kv_empty[NS], s_full[2], p_full[2], p_empty[2], drain
  static constexpr uint32_t NBAR = 2 + 3 * NS + 2 + 2 + 2 + 1;
  static constexpr uint32_t SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
};

__device__ __forceinline__ uint32_t pack_bf16x2_p(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int ID, int NTHREADS>
__device__ __forceinline__ void named_barrier_p() {
  asm volatile("barrier.sync %0, %1;" ::"n"(ID), "n"(NTHREADS) : "memory");
}

}  // namespace

__global__ void __launch_bounds__(kPairThreads, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = PairCfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;                 // [tile]
  uint64_t* k_full = q_full + 2;           // [stage]
  uint64_t* v_full = k_full + C::NS;       // [stage]
  uint64_t* kv_empty = v_full + C::NS;     // [stage]
  uint64_t* s_full = kv_empty + C::NS;     // [tile]: S_t(j) computed
  uint64_t* p_full = s_full + 2;           // [tile]: P_t(j) written (and O_t rescaled)
  uint64_t* p_empty = p_full + 2;          // [tile]: O_t += P_t(j) V_j done
  uint64_t* drain_bar = p_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int npair = (p.G + 1) >> 1;
  const int pair = blockIdx.x % npair;
  const int bh = blockIdx.x / npair;
  const int hc = p.hc > 0 ? p.hc : p.H;
  const int b = bh / hc;
  const int h = p.h0 + bh % hc;
  const int T = (p.kv_count + 127) >> 7;
  // each CTA starts its key sweep at its own pair's index (spreads L2 reads)
  const int kt0 = pair % T;
  auto key_tile = [&](int i) { const int r = i + kt0; return r < T ? r : r - T; };
  constexpr int kGather = C::KB * 32;  // gathering threads: 4 query rows of one column block each, both tiles

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) mbar_init(&q_full[t], kGather);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&p_empty[t], 1);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wctx{abort_flag, p.status, p.wait_limit_ns};
  int issued = 0;  // producer: K/V tiles whose loads were issued

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPairLowRegs));
    if (warp == 0) {
      // ---------------------------------------------------------------- UMMA issuer
      if (lane == 0) {
        constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, false, true);
        const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
        const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
        const uint64_t dV = sdesc_sw128(smem_u32(sV), 16384, 1024);
        // S_t(j) = Q_t K_j^T into the 128 columns of tile t
        auto issue_s = [&](int t, int j) {
          const uint64_t dQt = sdesc_advance(dQ, t * C::TILE);
          const uint64_t dKs = sdesc_advance(dK, (j % C::NS) * C::TILE);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_bf16_ss(tmem + t * 128, sdesc_advance(dQt, off), sdesc_advance(dKs, off), IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[t]);
        };
        // O_t += P_t(j) V_j: P_t as bf16 pairs in the first 64 columns of tile
        // t's S (8 columns per 16 keys), V rows 16 kk .. 16 kk + 15
        auto issue_o = [&](int t, int j) {
          const uint64_t dVs = sdesc_advance(dV, (j % C::NS) * C::TILE);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, sdesc_advance(dVs, kk * 2048), IDESC_O,
                         (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&p_empty[t]);
        };
        bool ok = mbar_wait(&q_full[0], 0, wctx, MCS_WHERE_ATTN_MMA) && mbar_wait(&q_full[1], 0, wctx, MCS_WHERE_ATTN_MMA);
        // order per key tile: S_A(j), O_B += P_B(j-1) V_j-1, S_B(j), O_A += P_A(j) V_j. UMMAs run in
        // order, so S_t(j+1) overwrites P_t(j) only after the product that reads it.
        for (int it = 0; ok && it <= T; ++it) {
          const int s = it % C::NS;
          if (it < T) {
            if (!mbar_wait(&k_full[s], (it / C::NS) & 1, wctx, MCS_WHERE_ATTN_MMA)) break;
            tc_fence_after();
            issue_s(0, it);
          }
          if (it >= 1) {
            const int j = it - 1;
            if (!mbar_wait(&p_full[1], j & 1, wctx, MCS_WHERE_ATTN_MMA)) break;
            tc_fence_after();
            issue_o(1, j);                       // V_j arrived before O_A's product of step j
            umma_commit(&kv_empty[j % C::NS]);  // every UMMA reading K_j and V_j has been issued
          }
          if (it < T) {
            issue_s(1, it);
            if (!mbar_wait(&v_full[s], (it / C::NS) & 1, wctx, MCS_WHERE_ATTN_MMA)) break;
            if (!mbar_wait(&p_full[0], it & 1, wctx, MCS_WHERE_ATTN_MMA)) break;
            tc_fence_after();
            issue_o(0, it);
          }
        }
      }
      __syncwarp();
    } else {
      // ---------------------------------------------------------------- TMA producers
      const int pt = threadIdx.x - 32;
      if (pt == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
      }
      const size_t head_base = static_cast<size_t>(b) * p.H + h;
      // thread pt < KB*32 gathers query rows 4g..4g+3 of column block kb (g = pt % 32) of both tiles
      if (pt < kGather) {
        const int kb = pt >> 5, grp = pt & 31;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          int qr[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            int pos = (2 * pair + t) * 128 + grp * 4 + i;
            if (pos >= p.N) pos = p.N - 1;  // tail rows (and a missing last tile) repeat the last query
            int tok = p.perm ? p.perm[head_base * p.N + pos] : pos;
            if (tok < 0 || tok >= p.N) {
              record_status(p.status, MCS_ERR_BAD_INDEX, tok);
              tok = 0;
            }
            qr[i] = (b * p.N + tok) * p.H + h;
          }
          mbar_arrive_expect_tx(&q_full[t], 512);
          tma_gather4(&tm_q, &q_full[t], sQ + t * C::TILE + kb * 16384 + grp * 512, kb * 64, qr[0], qr[1], qr[2],
                      qr[3]);
        }
      }
      for (int it = 0; pt == 0 && it < T; ++it) {
        const int s = it % C::NS;
        if (it >= C::NS) {
          if (!mbar_wait(&kv_empty[s], ((it / C::NS) & 1) ^ 1, wctx, MCS_WHERE_ATTN_PRODUCER)) break;
        }
        if ((p.debug_flags & 1) && it == 0) continue;  // test knob: never deliver tile 0
        mbar_arrive_expect_tx(&k_full[s], C::TILE);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d(&tm_k, &k_full[s], sK + s * C::TILE + kb * 16384, kb * 64, h, b * p.N + key_tile(it) * 128);
        mbar_arrive_expect_tx(&v_full[s], C::TILE);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d(&tm_v, &v_full[s], sV + s * C::TILE + kb * 16384, kb * 64, h, b * p.N + key_tile(it) * 128);
        issued = it + 1;
      }
      __syncwarp();
    }
    // back to the launch allocation once the softmax warpgroups returned theirs
    named_barrier_p<1, kPairThreads>();
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPairLaunchRegs));
  } else {
    // ---------------------------------------------------------------- softmax + epilogue of tile t
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPairSoftRegs));
    const int t = (warp - 4) >> 2;  // query tile of this warpgroup
    const int wq = warp & 3;        // TMEM lane quarter this warp may access
    const int row = wq * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_addr + t * 128;
    const uint32_t tO = tmem + lane_addr + 256 + t * 128;
    const int tile = 2 * pair + t;  // == G for the missing second tile of an odd G
    const int pos = tile * 128 + row;
    const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
    float m = -CUDART_INF_F;  // running max of scaled scores, log2 units
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      if (!mbar_wait_warp(&s_full[t], j & 1, wctx, MCS_WHERE_ATTN_SOFTMAX)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[128];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tS + c4 * 32, sv + c4 * 32);
      tmem_wait_ld();
      const int valid = p.kv_count - key_tile(j) * 128;  // keys of this tile (>= 1)
      if (valid < 128) {
#pragma unroll
        for (int c = 0; c < 128; ++c) sv[c] = (c < valid) ? sv[c] : -CUDART_INF_F;
      }
      // row max: eight chains of three-input max
      float mc[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float a = sv[k * 16];
#pragma unroll
        for (int e = 1; e < 15; e += 2) a = fmax3(a, sv[k * 16 + e], sv[k * 16 + e + 1]);
        mc[k] = fmaxf(a, sv[k * 16 + 15]);
      }
      const float mx =
          fmaxf(fmax3(fmaxf(mc[0], mc[1]), mc[2], mc[3]), fmax3(fmaxf(mc[4], mc[5]), mc[6], mc[7])) * p.scale_log2;
      const bool need = mx > m + kPairRescaleThreshold;
      float alpha = 1.f;
      bool rescale = false;  // warp-uniform: some row of this warp moves its max
      if (j == 0) {
        m = mx;
      } else {
        rescale = __any_sync(0xffffffffu, need);
        if (need) {
          alpha = fast_exp2(m - mx);
          m = mx;
        }
      }
      const uint64_t negm = f2_pack(-m, -m);  // m is finite: every key tile holds a key
#pragma unroll
      for (int q = 0; q < 64; ++q) {
        const uint64_t s2 = f2_pack(sv[2 * q], sv[2 * q + 1]);
        const uint64_t x = f2_fma(s2, scale2, negm);  // s*c - m, rounded once
        float x0, x1;
        f2_unpack(x, x0, x1);
        sv[2 * q] = fast_exp2(x0);
        sv[2 * q + 1] = fast_exp2(x1);
      }
      if (valid < 128) {  // masked keys (their exponent is -inf): exactly 0
#pragma unroll
        for (int c = 0; c < 128; ++c) sv[c] = (c < valid) ? sv[c] : 0.f;
      }
      // P (bf16 pairs) over the first 64 columns of this tile's S: S_t(j+1) is
      // issued into them only after O_t += P_t(j) V_j, and UMMAs run in order
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2_p(sv[64 * h2 + 2 * c], sv[64 * h2 + 2 * c + 1]);
        tmem_st32u(tS + h2 * 32, pk);
      }
      // the tile's row sum as a balanced tree of packed adds (depth 7)
      uint64_t acc[32];
#pragma unroll
      for (int q = 0; q < 32; ++q)
        acc[q] = f2_add(f2_pack(sv[2 * q], sv[2 * q + 1]), f2_pack(sv[2 * q + 64], sv[2 * q + 65]));
#pragma unroll
      for (int w = 16; w >= 1; w >>= 1) {
#pragma unroll
        for (int q = 0; q < w; ++q) acc[q] = f2_add(acc[q], acc[q + w]);
      }
      float r0, r1;
      f2_unpack(acc[0], r0, r1);
      l = l * alpha + (r0 + r1);
      tmem_wait_st();
      if (rescale) {
        // O_t holds tiles < j scaled by the old max: once O_t += P_t(j-1) V_j-1
        // is done, scale it by alpha before O_t += P_t(j) V_j (which waits for p_full)
        if (!mbar_wait_warp(&p_empty[t], (j - 1) & 1, wctx, MCS_WHERE_ATTN_SOFTMAX)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float ov[32];
          tmem_ld32(tO + c * 32, ov);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tmem_st32(tO + c * 32, ov);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    // ---------------------------------------------------------------- epilogue of tile t
    const bool fin = ok && mbar_wait_warp(&p_empty[t], (T - 1) & 1, wctx, MCS_WHERE_ATTN_EPILOGUE);
    if (fin && tile < p.G) {
      tc_fence_after();
      const float inv_L = 1.f / l;
      const bool row_valid = pos < p.N;
      const size_t head_base = static_cast<size_t>(b) * p.H + h;
      int tok = pos;
      if (row_valid && p.perm) tok = p.perm[head_base * p.N + pos];
      if (tok < 0 || tok >= p.N) tok = 0;
      if (row_valid && p.lse_out) {
        const float lse2 = m + log2f(l);
        p.lse_out[head_base * p.N + tok] = lse2 * 0.69314718055994530942f;
      }
      uint16_t* orow = p.o + (static_cast<size_t>(b) * p.N + tok) * p.H * D + static_cast<size_t>(h) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        float ov[32];
        tmem_ld32(tO + cc * 32, ov);
        tmem_wait_ld();
        if (!row_valid) continue;
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] *= inv_L;
        uint4* odst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 w;
          w.x = pack_bf16x2_p(ov[8 * i + 0], ov[8 * i + 1]);
          w.y = pack_bf16x2_p(ov[8 * i + 2], ov[8 * i + 3]);
          w.z = pack_bf16x2_p(ov[8 * i + 4], ov[8 * i + 5]);
          w.w = pack_bf16x2_p(ov[8 * i + 6], ov[8 * i + 7]);
          odst[i] = w;
        }
      }
    }
    __syncwarp();
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPairLaunchRegs));
    named_barrier_p<1, kPairThreads>();
  }

  // ------------------------------------------------------------------ teardown
  // All roles have left their loops. After an abort, wait (bounded, ignoring
  // the abort flag) for copies and UMMAs this CTA issued, then free TMEM.
  __syncthreads();
  if (*abort_flag) {
    volatile int never = 0;
    const WaitCtx drain_ctx{&never, nullptr, 50000000ull};
    if (threadIdx.x == 32) {
      for (int it = max(0, issued - C::NS); it < issued; ++it) {
        const int s = it % C::NS;
        mbar_wait(&k_full[s], (it / C::NS) & 1, drain_ctx, MCS_WHERE_DRAIN);
        mbar_wait(&v_full[s], (it / C::NS) & 1, drain_ctx, MCS_WHERE_DRAIN);
      }
    }
    if (warp == 0 && lane == 0) {
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0, drain_ctx, MCS_WHERE_DRAIN);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

cudaError_t launch_attention_pair(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                                  const AttnParams& p, cudaStream_t s) {
  static bool attr_set = false;
  auto kern = attn_pair_kernel;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg::SMEM);
    if (e != cudaSuccess) return e;
    // the setmaxnreg split assumes exactly kPairLaunchRegs registers per thread
    // at launch; with fewer, a register increase could never be satisfied
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kPairLaunchRegs) return cudaErrorInvalidKernelImage;
    attr_set = true;
  }
  const int hc = p.hc > 0 ? p.hc : p.H;
  const unsigned grid = static_cast<unsigned>(p.B) * hc * ((p.G + 1) / 2);
  if (grid == 0) return cudaSuccess;
  kern<<<grid, kPairThreads, PairCfg::SMEM, s>>>(*tq, *tk, *tv, p);
  return cudaGetLastError();
}

}  // namespace mcs
