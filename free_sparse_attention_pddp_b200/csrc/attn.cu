// Attention over one 128-query tile per CTA, tcgen05/TMEM on sm_100a.
//
// One kernel body serves three passes of the MC-Sparse path:
//   ATTN_DENSE          all N keys in order (dense baseline; anchor pass 1,
//                       which also exports fp32 O_dense and lse in group order)
//   ATTN_REUSE          the group's K cached keys, o = sparse + R (reuse step,
//                       aiwillknow analysis step 4; paper Table 6 kernel)
//   ATTN_ANCHOR_SPARSE  the group's K keys at the anchor, R = O_dense - sparse
//                       (aiwillknow analysis step 3)
// Queries of a tile are gathered by the grouping permutation and keys/values by
// index with TMA tile::gather4 (4 rows of 128 B per instruction, 128-byte
// swizzle) straight into the UMMA operand layout; selection crosses KV block
// boundaries with no padding (paper Table 4, token granularity).
//
// Warp roles (288 threads):
//   warps 0-3  TMA producers: gathered tiles take 2*32*(d/64) gather4 per K/V
//              tile, one per producer thread (a single issuing warp cannot
//              keep up with random 128-byte rows); dense K/V tiles are one
//              tiled 3-D TMA box (64 x 1 x 128) per 128-byte column block
//   warp 4     TMEM owner and UMMA issuer: S = Q K^T into one of two TMEM
//              S buffers, then O += P V with P read from TMEM (TS form) and V
//              an MN-major shared-memory operand
//   warps 5-8  softmax: one thread per query row; online softmax with a lazy
//              rescale (the running max only moves when it grows by more than
//              a factor of 2, which keeps the dominant probability close to 1
//              where bf16 P is accurate, and rescales of O in TMEM rare), P
//              written as bf16 pairs over its S columns; then the epilogue.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "mcs_ptx.cuh"

namespace mcs {

namespace {

// Thread layout per mode. Dense: 4 TMA producer warps (thread 0 issues the
// tiled loads, threads < 64 the query gather), UMMA warp 4, softmax warps 5-8.
// Gathered modes: 16 cp.async loader warps (random 256-byte rows: 16-byte
// pieces from 512 threads sustain the highest gather rate), softmax warps
// 16-19, UMMA warp 20, warps 21-23 idle; registers move from the loader and
// UMMA warpgroups to the softmax warpgroup with setmaxnreg.
template <int MODE>
struct Roles {
  static constexpr bool kCpAsync = MODE != ATTN_DENSE;
  static constexpr int kThreads = kCpAsync ? 768 : 288;
  static constexpr int kLoaders = kCpAsync ? 512 : 128;
  static constexpr int kMmaWarp = kCpAsync ? 20 : 4;
  static constexpr int kLoaderRegs = 40, kSoftRegs = 256, kMmaRegs = 40;
  static constexpr int kLaunchRegs = 80;  // 65536 / 768 rounded down to a multiple of 8  // within the 768 x 80 launch pool
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// arrive on `bar` once every cp.async this thread issued so far has landed
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Named barrier 1 over the whole CTA, reached from different role branches
// (hence the non-aligned form). In the gathered modes it orders the register
// hand-back: the softmax warpgroup returns its extra registers before arriving,
// and the other warpgroups take theirs back only after it, so no increase can
// claim registers that the softmax warpgroup's initial increase still needs.
template <int NTHREADS>
__device__ __forceinline__ void role_barrier() {
  asm volatile("barrier.sync 1, %0;" ::"n"(NTHREADS) : "memory");
}
constexpr float kRescaleThreshold = 1.0f;  // log2 units: rescale O when the row max grows by more than 2x

template <int D>
struct AttnCfg {
  static constexpr int KB = D / 64;                 // 128-byte column blocks per row
  static constexpr uint32_t TILE = 128u * D * 2u;   // one 128-row bf16 tile
  static constexpr int NS = (D == 128) ? 3 : 5;     // K/V pipeline stages
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = TILE;
  static constexpr uint32_t OFF_V = OFF_K + NS * TILE;
  static constexpr uint32_t OFF_BAR = OFF_V + NS * TILE;
  static constexpr uint32_t NBAR = 1 + 3 * NS + 6 + 1;
  static constexpr uint32_t SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + alignment slack
  static constexpr uint32_t TMEM_COLS = 512;  // S0 | S1 | O; P (bf16) overwrites the first half of its S
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

}  // namespace

template <int D, int MODE>
__global__ void __launch_bounds__(Roles<MODE>::kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = AttnCfg<D>;
  using R = Roles<MODE>;
  constexpr int kMmaWarp = R::kMmaWarp;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + C::NS;
  uint64_t* kv_empty = v_full + C::NS;
  uint64_t* s_full = kv_empty + C::NS;  // [2]
  uint64_t* p_full = s_full + 2;        // [2]
  uint64_t* p_empty = p_full + 2;       // [2]  PV done on that P buffer
  uint64_t* drain_bar = p_empty + 2;    // abort path: all issued UMMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile = blockIdx.x % p.G;
  const int bh = blockIdx.x / p.G;
  const int b = bh / p.H;
  const int h = bh % p.H;
  const int T = (p.kv_count + 127) >> 7;

  constexpr int kGatherPerTile = C::KB * 32;  // dense: query gather4 per 128-row tile, one per thread
  if (threadIdx.x == 0) {
    mbar_init(q_full, R::kCpAsync ? R::kLoaders : kGatherPerTile);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&k_full[s], R::kCpAsync ? R::kLoaders : 1);
      mbar_init(&v_full[s], R::kCpAsync ? R::kLoaders : 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&p_empty[i], 1);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wctx{abort_flag, p.status, p.wait_limit_ns};
  int issued = 0;  // producer: K/V tiles whose loads were issued

  if (threadIdx.x < R::kLoaders && R::kCpAsync) {
    // ---------------------------------------------------------------- cp.async loaders
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R::kLoaderRegs));
    const int lt = threadIdx.x;
    constexpr int CH = D / 8;                // 16-byte pieces per row
    constexpr int PER = 128 * CH / R::kLoaders;  // rows per thread per tile: lt/CH + (512/CH) i
    constexpr int RSTEP = R::kLoaders / CH;
    const int ch = lt % CH;
    const int row0 = lt / CH;
    const size_t head_base = static_cast<size_t>(b) * p.H + h;
    const uint32_t soff = (ch >> 3) * 16384;
    // the query tile, gathered by the grouping permutation
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int row = row0 + RSTEP * i;
      int pos = tile * 128 + row;
      if (pos >= p.N) pos = p.N - 1;  // tail rows repeat the last valid query
      int tok = p.perm[head_base * p.N + pos];
      if (tok < 0 || tok >= p.N) {
        record_status(p.status, MCS_ERR_BAD_INDEX, tok);
        tok = 0;
      }
      cp_async16(sQ + soff + sw128_offset(row, ch & 7),
                 p.q + ((static_cast<size_t>(b) * p.N + tok) * p.H + h) * D + ch * 8);
    }
    cp_async_arrive_noinc(q_full);
    const int32_t* idx_list = p.kv_idx + (head_base * p.G + tile) * static_cast<size_t>(p.kv_count);
    auto load_tokens = [&](int it, int (&tok)[PER]) {
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        int c = it * 128 + row0 + RSTEP * i;
        if (c >= p.kv_count) c = p.kv_count - 1;  // masked in softmax
        int t = __ldg(idx_list + c);
        if (t < 0 || t >= p.N) {
          record_status(p.status, MCS_ERR_BAD_INDEX, t);
          t = 0;
        }
        tok[i] = t;
      }
    };
    int tok[PER], tok_next[PER];
    load_tokens(0, tok_next);
    for (int it = 0; it < T; ++it) {
      const int s = it % C::NS;
#pragma unroll
      for (int i = 0; i < PER; ++i) tok[i] = tok_next[i];
      if (it + 1 < T) load_tokens(it + 1, tok_next);  // in flight while this tile is issued
      if (it >= C::NS) {
        if (!mbar_wait(&kv_empty[s], ((it / C::NS) & 1) ^ 1, wctx, MCS_WHERE_ATTN_PRODUCER)) break;
      }
      if ((p.debug_flags & 1) && it == 0) continue;  // test knob: never deliver tile 0
#pragma unroll
      for (int i = 0; i < PER; ++i)
        cp_async16(sK + s * C::TILE + soff + sw128_offset(row0 + RSTEP * i, ch & 7),
                   p.k + ((static_cast<size_t>(b) * p.N + tok[i]) * p.H + h) * D + ch * 8);
      cp_async_arrive_noinc(&k_full[s]);
#pragma unroll
      for (int i = 0; i < PER; ++i)
        cp_async16(sV + s * C::TILE + soff + sw128_offset(row0 + RSTEP * i, ch & 7),
                   p.v + ((static_cast<size_t>(b) * p.N + tok[i]) * p.H + h) * D + ch * 8);
      cp_async_arrive_noinc(&v_full[s]);
      issued = it + 1;
    }
    cp_async_wait_all();
    // back to the launch allocation so the shared teardown below sees one
    // limit, once the softmax warpgroup has returned its registers
    role_barrier<R::kThreads>();
    __syncwarp();  // setmaxnreg wants the whole warp converged
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R::kLaunchRegs));
  } else if (threadIdx.x < R::kLoaders) {
    // ---------------------------------------------------------------- TMA producers (dense)
    const int pt = threadIdx.x;
    if (pt == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
    }
    const size_t head_base = static_cast<size_t>(b) * p.H + h;
    // thread pt < KB*32 gathers query rows 4g..4g+3 of column block kb (g = pt % 32)
    if (pt < kGatherPerTile) {
      const int kb = pt >> 5, grp = pt & 31;
      int qr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        int pos = tile * 128 + grp * 4 + i;
        if (pos >= p.N) pos = p.N - 1;  // tail rows repeat the last valid query
        int tok = p.perm ? p.perm[head_base * p.N + pos] : pos;
        if (tok < 0 || tok >= p.N) {
          record_status(p.status, MCS_ERR_BAD_INDEX, tok);
          tok = 0;
        }
        qr[i] = (b * p.N + tok) * p.H + h;
      }
      mbar_arrive_expect_tx(q_full, 512);
      tma_gather4(&tm_q, q_full, sQ + kb * 16384 + grp * 512, kb * 64, qr[0], qr[1], qr[2], qr[3]);
    }
    for (int it = 0; pt == 0 && it < T; ++it) {
      const int s = it % C::NS;
      if (it >= C::NS) {
        if (!mbar_wait(&kv_empty[s], ((it / C::NS) & 1) ^ 1, wctx, MCS_WHERE_ATTN_PRODUCER)) break;
      }
      if ((p.debug_flags & 1) && it == 0) continue;  // test knob: never deliver tile 0
      // 128 consecutive tokens of head h: box {64, 1, 128} of the [B*N, H, d] view
      mbar_arrive_expect_tx(&k_full[s], C::TILE);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb)
        tma_load_3d(&tm_k, &k_full[s], sK + s * C::TILE + kb * 16384, kb * 64, h, b * p.N + it * 128);
      mbar_arrive_expect_tx(&v_full[s], C::TILE);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb)
        tma_load_3d(&tm_v, &v_full[s], sV + s * C::TILE + kb * 16384, kb * 64, h, b * p.N + it * 128);
      issued = it + 1;
    }
  } else if (R::kCpAsync ? (warp >= kMmaWarp) : (warp == kMmaWarp)) {
    // ---------------------------------------------------------------- UMMA issuer (and idle warps)
    if (R::kCpAsync) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R::kMmaRegs));
    if (warp == kMmaWarp && lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, false, true);
      const uint32_t tO = tmem + 256;
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
      bool ok = mbar_wait(q_full, 0, wctx, MCS_WHERE_ATTN_MMA);
      for (int it = 0; ok && it <= T; ++it) {
        if (it < T) {
          const int s = it % C::NS;
          if (!mbar_wait(&k_full[s], (it / C::NS) & 1, wctx, MCS_WHERE_ATTN_MMA)) break;
          tc_fence_after();
          const uint32_t tS = tmem + (it & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_bf16_ss(tS, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(aK + s * C::TILE + off, 16, 1024),
                         IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[it & 1]);
        }
        if (it >= 1) {
          const int j = it - 1;
          const int s = j % C::NS;
          const int pb = j & 1;
          if (!mbar_wait(&p_full[pb], (j >> 1) & 1, wctx, MCS_WHERE_ATTN_MMA)) break;
          if (!mbar_wait(&v_full[s], (j / C::NS) & 1, wctx, MCS_WHERE_ATTN_MMA)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // P_j (bf16 in TMEM, 8 columns per 16 keys) times V_j
            umma_bf16_ts(tO, tmem + pb * 128 + kk * 8, sdesc_sw128(aV + s * C::TILE + kk * 2048, 16384, 1024),
                         IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&kv_empty[s]);
          umma_commit(&p_empty[pb]);
        }
      }
    }
    __syncwarp();
    if (R::kCpAsync) {
      role_barrier<R::kThreads>();
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R::kLaunchRegs));
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    if (R::kCpAsync) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R::kSoftRegs));
    const int wq = warp & 3;  // TMEM lane quarter this warp may access
    const int row = wq * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const int pos = tile * 128 + row;
    float m = -CUDART_INF_F;  // running max of scaled scores, log2 units
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int pb = j & 1;
      if (!mbar_wait_warp(&s_full[pb], (j >> 1) & 1, wctx, MCS_WHERE_ATTN_SOFTMAX)) { ok = false; break; }
      tc_fence_after();
      float sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_addr + pb * 128 + c * 32, sv + c * 32);
      tmem_wait_ld();
      const int valid = min(128, p.kv_count - j * 128);
      if (valid < 128) {  // last, partial tile: masked keys get probability 0
#pragma unroll
        for (int c = 0; c < 128; ++c) sv[c] = (c < valid) ? sv[c] : -CUDART_INF_F;
      }
      // row max of the raw scores with 8 independent chains
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = sv[i];
#pragma unroll
      for (int c = 8; c < 128; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], sv[c]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * p.scale_log2;
      bool need = (mx > m + kRescaleThreshold);
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
      // p = 2^(s*scale*log2e - m): one FFMA and one MUFU ex2 per score
      const float neg_m = -m;
      float rs8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) rs8[i] = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        sv[c] = fast_exp2(fmaf(sv[c], p.scale_log2, neg_m));
        rs8[c & 7] += sv[c];
      }
      l = l * alpha + (((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7])));
      // P_j (bf16 pairs) over the first 64 columns of this S buffer; S_{j+2} is
      // issued into the same buffer only after PV_j, and UMMAs run in order
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(sv[half * 64 + 2 * c], sv[half * 64 + 2 * c + 1]);
        tmem_st32u(tmem + lane_addr + pb * 128 + half * 32, pk);
      }
      tmem_wait_st();
      if (rescale) {
        // O holds tiles < j scaled by the old max: once PV_{j-1} is done, scale
        // it by alpha before PV_j (which waits for this warp's p_full arrival)
        if (!mbar_wait_warp(&p_empty[(j - 1) & 1], ((j - 1) >> 1) & 1, wctx, MCS_WHERE_ATTN_SOFTMAX)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float ov[32];
          tmem_ld32(tmem + lane_addr + 256 + c * 32, ov);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tmem_st32(tmem + lane_addr + 256 + c * 32, ov);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&p_full[pb]);
    }
    // ---------------------------------------------------------------- epilogue
    if (ok && mbar_wait_warp(&p_empty[(T - 1) & 1], ((T - 1) >> 1) & 1, wctx, MCS_WHERE_ATTN_EPILOGUE)) {
      tc_fence_after();
      const bool row_valid = pos < p.N;
      const size_t head_base = static_cast<size_t>(b) * p.H + h;
      const size_t prow_idx = head_base * (static_cast<size_t>(p.G) * 128) + pos;  // padded perm-order row
      int tok = pos;
      if (row_valid && p.perm) tok = p.perm[head_base * p.N + pos];
      if (tok < 0 || tok >= p.N) tok = 0;
      const float inv_l = 1.f / l;
      const float lse2 = m + log2f(l);  // log2 of sum_j 2^(s_ij*scale*log2e)
      const float lse = lse2 * 0.69314718055994530942f;
      if (MODE == ATTN_DENSE) {
        if (p.lse_perm_out) p.lse_perm_out[prow_idx] = row_valid ? lse2 : CUDART_INF_F;
        if (row_valid && p.lse_out) p.lse_out[head_base * p.N + tok] = lse;
      }
      uint16_t* orow = p.o + (static_cast<size_t>(b) * p.N + tok) * p.H * D + static_cast<size_t>(h) * D;
      const size_t rrow = (head_base * p.N + (row_valid ? pos : 0)) * D;  // resid rows: [B,H,N,d] perm order
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float ov[32];
        tmem_ld32(tmem + lane_addr + 256 + c * 32, ov);
        tmem_wait_ld();
        if (!row_valid) continue;
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] *= inv_l;
        if (MODE == ATTN_DENSE && p.o_dense_out) {
          float4* dst = reinterpret_cast<float4*>(p.o_dense_out + prow_idx * D + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_float4(ov[4 * i], ov[4 * i + 1], ov[4 * i + 2], ov[4 * i + 3]);
        }
        if (MODE == ATTN_REUSE && p.resid_in) {
          const uint4* rsrc = reinterpret_cast<const uint4*>(p.resid_in + rrow + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 rv = rsrc[i];
            const uint16_t* rh = reinterpret_cast<const uint16_t*>(&rv);
#pragma unroll
            for (int e = 0; e < 8; ++e) ov[i * 8 + e] += bf16_to_f32(rh[e]);
          }
        }
        if (MODE == ATTN_ANCHOR_SPARSE) {
          const float4* dsrc = reinterpret_cast<const float4*>(p.o_dense_in + prow_idx * D + c * 32);
          uint4* rdst = reinterpret_cast<uint4*>(p.resid_out + rrow + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float4 d0 = dsrc[2 * i], d1 = dsrc[2 * i + 1];
            uint4 w;
            w.x = pack_bf16x2(d0.x - ov[8 * i + 0], d0.y - ov[8 * i + 1]);
            w.y = pack_bf16x2(d0.z - ov[8 * i + 2], d0.w - ov[8 * i + 3]);
            w.z = pack_bf16x2(d1.x - ov[8 * i + 4], d1.y - ov[8 * i + 5]);
            w.w = pack_bf16x2(d1.z - ov[8 * i + 6], d1.w - ov[8 * i + 7]);
            rdst[i] = w;
          }
        } else {
          uint4* odst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16x2(ov[8 * i + 0], ov[8 * i + 1]);
            w.y = pack_bf16x2(ov[8 * i + 2], ov[8 * i + 3]);
            w.z = pack_bf16x2(ov[8 * i + 4], ov[8 * i + 5]);
            w.w = pack_bf16x2(ov[8 * i + 6], ov[8 * i + 7]);
            odst[i] = w;
          }
        }
      }
    }
    if (R::kCpAsync) {
      __syncwarp();
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R::kLaunchRegs));
      role_barrier<R::kThreads>();
    }
  }

  // ------------------------------------------------------------------ teardown
  // All roles have left their loops. After an abort, wait (bounded, ignoring
  // the abort flag) for copies and UMMAs this CTA issued, then free TMEM.
  __syncthreads();
  if (*abort_flag) {
    volatile int never = 0;
    const WaitCtx drain_ctx{&never, nullptr, 50000000ull};
    if (warp == 0 && lane == 0) {
      for (int it = max(0, issued - C::NS); it < issued; ++it) {
        const int s = it % C::NS;
        mbar_wait(&k_full[s], (it / C::NS) & 1, drain_ctx, MCS_WHERE_DRAIN);
        mbar_wait(&v_full[s], (it / C::NS) & 1, drain_ctx, MCS_WHERE_DRAIN);
      }
    }
    if (warp == kMmaWarp && lane == 0) {
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0, drain_ctx, MCS_WHERE_DRAIN);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D, int MODE>
static cudaError_t launch_attn_t(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                                 const AttnParams& p, cudaStream_t s) {
  using C = AttnCfg<D>;
  static bool attr_set = false;
  auto kern = attn_kernel<D, MODE>;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid(static_cast<unsigned>(p.B * p.H * p.G));
  kern<<<grid, Roles<MODE>::kThreads, C::SMEM, s>>>(*tq, *tk, *tv, p);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_attention(int d, AttnMode mode, const CUtensorMap* tq, const CUtensorMap* tk,
                             const CUtensorMap* tv, const AttnParams& p, cudaStream_t s) {
  if (d == 128) {
    switch (mode) {
      case ATTN_DENSE: return launch_attn_t<128, ATTN_DENSE>(tq, tk, tv, p, s);
      case ATTN_REUSE: return launch_attn_t<128, ATTN_REUSE>(tq, tk, tv, p, s);
      case ATTN_ANCHOR_SPARSE: return launch_attn_t<128, ATTN_ANCHOR_SPARSE>(tq, tk, tv, p, s);
    }
  } else if (d == 64) {
    switch (mode) {
      case ATTN_DENSE: return launch_attn_t<64, ATTN_DENSE>(tq, tk, tv, p, s);
      case ATTN_REUSE: return launch_attn_t<64, ATTN_REUSE>(tq, tk, tv, p, s);
      case ATTN_ANCHOR_SPARSE: return launch_attn_t<64, ATTN_ANCHOR_SPARSE>(tq, tk, tv, p, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace mcs
