// Attention over one 128-query tile per CTA, tcgen05/TMEM on sm_100a.
//
// One kernel body serves four passes of the MC-Sparse path:
//   ATTN_DENSE          all N keys in order (dense baseline)
//   ATTN_ANCHOR_DENSE   the same over queries in group order (anchor pass 1),
//                       exporting fp32 O_dense and the lse as an fp32 hi/lo pair
//   ATTN_REUSE          the group's K cached keys, o = sparse + R (reuse step,
//                       aiwillknow analysis step 4; paper Table 6 kernel)
//   ATTN_ANCHOR_SPARSE  the group's K keys at the anchor, R = O_dense - sparse
//                       (aiwillknow analysis step 3)
// Queries of a tile come in grouping-permutation order and keys/values by index
// (paper Table 4, token granularity: selection crosses KV block boundaries
// with no padding), straight into the 128-byte-swizzled UMMA operand layout.
//
// Work split of a 128-key tile j. The UMMA warp computes S_j = Q K_j^T into one
// of two TMEM S buffers. Two softmax warpgroups then take the two column halves
// of S_j (keys 0-63 and 64-127 of the tile), one thread per query row each.
// Each half keeps its own running max m_h and sum l_h and its own fp32 output
// accumulator O_h in TMEM, so the halves never synchronise inside the key loop:
// the UMMA warp accumulates O_h += P_h V_h as soon as half h has written P_h
// (bf16 pairs in TMEM, read by the TS form of the MMA). The epilogue merges the
// halves exactly: with m = max(m_0, m_1) and c_h = 2^(m_h - m),
//   O = (c_0 O_0 + c_1 O_1) / (c_0 l_0 + c_1 l_1),   lse = m + log2(c_0 l_0 + c_1 l_1)
// (the split-key form of online softmax). Two warps per SM sub-partition run
// softmax, so one warp's TMEM loads and reductions overlap the other's exps.
//
// Online softmax uses a lazy rescale: a half's running max only moves when its
// tile max exceeds it by more than kRescaleThreshold (log2 units), which keeps
// every probability below 16 (bf16 rounds it relatively, as any other) and makes rescales of O_h in
// TMEM rare. Scores are exponentiated in base 2 on the MUFU ex2 unit.
//
// Accuracy of the anchor's lse (ATTN_ANCHOR_DENSE), which the fp64 selection
// re-score divides by: the exponent s*c - m is formed with c split into fp32
// hi + lo parts (two FMAs, so the scale's fp32 rounding does not enter), each
// tile's 64 probabilities of a row are summed as a balanced tree (depth 6), the
// tile sums accumulate in fp64, every rescale of that sum (and the epilogue's
// merge of the halves) uses an fp64 2^(m_old - m_new), and lse2 = m + log2(l)
// is formed in fp64 and stored as an fp32 hi/lo pair.
//
// Thread layouts:
//   dense (384 threads): warp 0 UMMA, warps 1-3 TMA producers (thread 32
//     issues one tiled 3-D box per 128-byte column block of K and V; threads
//     32 .. 32 + 32*d/64 gather the query rows with tile::gather4), warps 4-11
//     softmax.
//   gathered (640 threads): warp 0 UMMA (warps 1-3 idle), warps 4-11 cp.async
//     loaders (16-byte pieces of the random 2*d-byte K/V rows from 256 threads
//     sustain a higher gather rate than TMA gather4), warps 12-19 softmax.
//     Registers move from the loader and UMMA warpgroups to the softmax
//     warpgroups with setmaxnreg (96 at launch; d = 128: 48 / 40 / 168,
//     d = 64: 40 / 40 / 176).
#include <cuda_bf16.h>
#include <math_constants.h>

#include <type_traits>

#include "mcs_ptx.cuh"

namespace mcs {

namespace {

// The UMMA issuer is lane 0 of warp 0.
template <int D, int MODE>
struct Roles {
  static constexpr bool kCpAsync = MODE == ATTN_REUSE || MODE == ATTN_ANCHOR_SPARSE;
  static constexpr int kMmaWarp = 0;
  static constexpr int kMmaWarps = kCpAsync ? 4 : 1;      // a whole warpgroup where setmaxnreg is used
  static constexpr int kLoader0 = kMmaWarps * 32;         // first loader / producer thread
  // loader / producer threads: 256 cp.async loaders keep the gather ahead of the
  // tensor pipe while leaving issue slots to the softmax warps (measured: 512
  // loaders were 1.5-7 % slower per pass)
  static constexpr int kLoaders = kCpAsync ? 256 : 96;
  static constexpr int kSoftWarp0 = (kLoader0 + kLoaders) / 32;  // first of 8 softmax warps
  static constexpr int kThreads = (kSoftWarp0 + 8) * 32;
  // registers per thread at launch: 65536 / kThreads rounded down to a multiple of 8
  static constexpr int kLaunchRegs = (65536 / kThreads) & ~7;
  // register shares chosen so that ptxas spills in no role (d = 128: loaders
  // 48, softmax 168; d = 64: loaders 40, softmax 176)
  static constexpr int kLoaderRegs = D == 128 ? 48 : 40, kMmaRegs = 40;
  // everything the loader and UMMA warpgroups give up goes to the 256 softmax
  // threads (rounded down to a multiple of 8)
  static constexpr int kSoftRegs =
      (kLaunchRegs + (kLoaders * (kLaunchRegs - kLoaderRegs) + 128 * (kLaunchRegs - kMmaRegs)) / 256) & ~7;
  static_assert(!kCpAsync || (kSoftRegs % 8 == 0 && kSoftRegs <= 256), "setmaxnreg counts");
  static_assert(!kCpAsync || (kLoaders * kLoaderRegs + 128 * kMmaRegs + 256 * kSoftRegs <= kThreads * kLaunchRegs),
                "register split exceeds the launch allocation");
};

// log2 units: rescale O_h when m_h would grow by more than 16x. Measured on the
// Wan-14B shape against 1.0: anchor dense pass 2.5 % and reuse step 3 % faster,
// every parity test green; 8.0 was faster still but its bf16 outputs left the
// parity tolerance in three tests.
constexpr float kRescaleThreshold = 4.0f;

template <int D>
struct AttnCfg {
  static constexpr int KB = D / 64;                 // 128-byte column blocks per row
  static constexpr uint32_t TILE = 128u * D * 2u;   // one 128-row bf16 tile
  static constexpr int NS = (D == 128) ? 3 : 5;     // K/V pipeline stages
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = TILE;
  static constexpr uint32_t OFF_V = OFF_K + NS * TILE;
  static constexpr uint32_t OFF_BAR = OFF_V + NS * TILE;
  static constexpr uint32_t NBAR = 1 + 3 * NS + 2 + 4 + 4 + 1;
  static constexpr uint32_t SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + alignment slack
  // TMEM columns: S0 | S1 | O_0 (D) | O_1 (D); P_h (bf16 pairs) overwrites the
  // first 32 columns of its own half of S
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(256 + 2 * D <= TMEM_COLS, "TMEM layout");
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// arrive on `bar` once every cp.async this thread issued so far has landed
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Named barrier over NTHREADS threads, reached from different role branches
// (hence the non-aligned form). Barrier 1 (whole CTA, gathered modes) orders
// the register hand-back: the softmax warpgroups return their extra registers
// before arriving and the other warpgroups take theirs back only after it, so
// no increase can claim registers that a softmax increase still needs.
// Barrier 2 joins the two softmax warpgroups before the epilogue merge.
template <int ID, int NTHREADS>
__device__ __forceinline__ void named_barrier() {
  asm volatile("barrier.sync %0, %1;" ::"n"(ID), "n"(NTHREADS) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

}  // namespace

template <int D, int MODE>
__global__ void __launch_bounds__(Roles<D, MODE>::kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = AttnCfg<D>;
  using R = Roles<D, MODE>;
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
  uint64_t* s_full = kv_empty + C::NS;  // [buffer]
  uint64_t* p_full = s_full + 2;        // [half * 2 + buffer]: P_h written
  uint64_t* p_empty = p_full + 4;       // [half * 2 + buffer]: PV of half h done on that buffer
  uint64_t* drain_bar = p_empty + 4;    // abort path: all issued UMMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile = blockIdx.x % p.G;
  const int bh = blockIdx.x / p.G;
  const int hc = p.hc > 0 ? p.hc : p.H;  // heads of this launch
  const int b = bh / hc;
  const int h = p.h0 + bh % hc;
  const int T = (p.kv_count + 127) >> 7;
  // Dense modes: the CTAs of one wave hold consecutive query tiles of one
  // head, and each starts its sweep over the key tiles at its own tile's
  // index (wrapping around), so at any moment they read different K/V tiles
  // instead of all requesting the same one from the L2.
  constexpr bool kDenseKeys = MODE == ATTN_DENSE || MODE == ATTN_ANCHOR_DENSE;
  const int kt0 = kDenseKeys ? tile % T : 0;
  auto key_tile = [&](int i) { const int r = i + kt0; return r < T ? r : r - T; };

  constexpr int kGatherPerTile = C::KB * 32;  // dense: query gather4 per 128-row tile, one per thread
  if (threadIdx.x == 0) {
    mbar_init(q_full, R::kCpAsync ? R::kLoaders : kGatherPerTile);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&k_full[s], R::kCpAsync ? R::kLoaders : 1);
      mbar_init(&v_full[s], R::kCpAsync ? R::kLoaders : 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&s_full[i], 1);
    for (int i = 0; i < 4; ++i) {
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

  if (warp < R::kMmaWarps) {
    // ---------------------------------------------------------------- UMMA issuer (and idle warps)
    if (R::kCpAsync) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R::kMmaRegs));
    if (warp == kMmaWarp && lane == 0) {
      // one lane runs the schedule and issues the UMMAs; the rest of its warp
      // waits below (measured: a lone issuing lane feeds the tensor pipe about
      // 20 % faster than a converged warp issuing through a lane predicate)
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, false, true);
      // descriptors built once; each UMMA steps them with one add
      const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(sV), 16384, 1024);
      bool ok = mbar_wait(q_full, 0, wctx, MCS_WHERE_ATTN_MMA);
      for (int it = 0; ok && it <= T; ++it) {
        if (it < T) {
          const int s = it % C::NS;
          if (!mbar_wait(&k_full[s], (it / C::NS) & 1, wctx, MCS_WHERE_ATTN_MMA)) break;
          tc_fence_after();
          const uint32_t tS = tmem + (it & 1) * 128;
          const uint64_t dKs = sdesc_advance(dK, s * C::TILE);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_bf16_ss(tS, sdesc_advance(dQ, off), sdesc_advance(dKs, off), IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[it & 1]);
        }
        if (it >= 1) {
          const int j = it - 1;
          const int s = j % C::NS;
          const int pb = j & 1;
          if (!mbar_wait(&v_full[s], (j / C::NS) & 1, wctx, MCS_WHERE_ATTN_MMA)) break;
          // O_h += P_h V_h: P_h (64 keys as bf16 pairs, 8 TMEM columns per 16
          // keys) at the start of half h of S buffer pb; V rows 64h .. 64h+63
          const uint64_t dVs = sdesc_advance(dV, s * C::TILE);
          bool got = true;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            if (!mbar_wait(&p_full[hf * 2 + pb], (j >> 1) & 1, wctx, MCS_WHERE_ATTN_MMA)) {
              got = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ts(tmem + 256 + hf * D, tmem + pb * 128 + hf * 64 + kk * 8,
                              sdesc_advance(dVs, (hf * 4 + kk) * 2048), IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
            if (hf == 1) umma_commit(&kv_empty[s]);
            umma_commit(&p_empty[hf * 2 + pb]);
          }
          if (!got) break;
        }
      }
    }
    __syncwarp();
    if (R::kCpAsync) {
      named_barrier<1, R::kThreads>();
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R::kLaunchRegs));
    }
  } else if (R::kCpAsync && threadIdx.x < R::kLoader0 + R::kLoaders) {
    // ---------------------------------------------------------------- cp.async loaders
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R::kLoaderRegs));
    constexpr int CH = D / 8;                  // 16-byte pieces per row
    constexpr int RSTEP = R::kLoaders / CH;    // rows between one thread's pieces
    constexpr int PER = 128 / RSTEP;           // rows per thread per tile
    constexpr uint32_t ISTEP = RSTEP * 128u;   // bytes between them in a column block
    static_assert(!R::kCpAsync || (RSTEP % 8 == 0 && 128 % RSTEP == 0), "one swizzle phase per thread");
    const int lt = threadIdx.x - R::kLoader0;
    const int ch = lt % CH;
    const int row0 = lt / CH;
    const size_t head_base = static_cast<size_t>(b) * p.H + h;
    // piece (row0 + RSTEP*i, ch) of a tile: rows row0 + RSTEP*i share row0's
    // swizzle phase, so every piece is dst0 + ISTEP*i
    const uint32_t dst0 = (ch >> 3) * 16384u + sw128_offset(row0, ch & 7);
    const uint32_t rstride = static_cast<uint32_t>(p.H) * D * 2u;  // bytes between tokens of a head
    const size_t col0 = (static_cast<size_t>(b) * p.N * p.H + h) * D * 2u + ch * 16u;
    const char* qbase = reinterpret_cast<const char*>(p.q) + col0;
    const char* kbase = reinterpret_cast<const char*>(p.k) + col0;
    const char* vbase = reinterpret_cast<const char*>(p.v) + col0;
    uint32_t bad = 0;
    int bad_value = 0;
    // the query tile, gathered by the grouping permutation
    {
      const uint32_t sq = smem_u32(sQ) + dst0;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        int pos = tile * 128 + row0 + RSTEP * i;
        if (pos >= p.N) pos = p.N - 1;  // tail rows repeat the last valid query
        int tok = p.perm[head_base * p.N + pos];
        if (static_cast<uint32_t>(tok) >= static_cast<uint32_t>(p.N)) {
          if (!bad) bad_value = tok;
          bad = 1;
          tok = 0;
        }
        cp_async16(sq + ISTEP * i, qbase + static_cast<uint64_t>(static_cast<uint32_t>(tok)) * rstride);
      }
      cp_async_arrive_noinc(q_full);
    }
    const int32_t* idx_list = p.kv_idx + (head_base * p.G + tile) * static_cast<size_t>(p.kv_count);
    const int full_tiles = p.kv_count >> 7;
    auto load_tokens = [&](int it, uint32_t (&tok)[PER]) {
      if (it < full_tiles) {
        const int32_t* src = idx_list + it * 128 + row0;
#pragma unroll
        for (int i = 0; i < PER; ++i) tok[i] = static_cast<uint32_t>(__ldg(src + RSTEP * i));
      } else {
#pragma unroll
        for (int i = 0; i < PER; ++i)  // keys past K repeat the last one; softmax masks them
          tok[i] = static_cast<uint32_t>(__ldg(idx_list + min(it * 128 + row0 + RSTEP * i, p.kv_count - 1)));
      }
      uint32_t hi = tok[0];
#pragma unroll
      for (int i = 1; i < PER; ++i) hi = max(hi, tok[i]);  // unsigned: a negative index is huge
      if (hi >= static_cast<uint32_t>(p.N)) {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          if (tok[i] >= static_cast<uint32_t>(p.N)) {
            if (!bad) bad_value = static_cast<int>(tok[i]);
            bad = 1;
            tok[i] = 0;
          }
        }
      }
    };
    uint32_t tok[PER], tok_next[PER];
    load_tokens(0, tok_next);
    const uint32_t sk0 = smem_u32(sK) + dst0, sv0 = smem_u32(sV) + dst0;
    int s = 0;
    uint32_t ph = 0;  // (it / NS) & 1
    for (int it = 0; it < T; ++it) {
#pragma unroll
      for (int i = 0; i < PER; ++i) tok[i] = tok_next[i];
      if (it + 1 < T) load_tokens(it + 1, tok_next);  // in flight while this tile is issued
      if (it >= C::NS) {
        if (!mbar_wait(&kv_empty[s], ph ^ 1u, wctx, MCS_WHERE_ATTN_PRODUCER)) break;
      }
      if (!((p.debug_flags & 1) && it == 0)) {  // test knob: never deliver tile 0
        const uint32_t sk = sk0 + s * C::TILE, sv = sv0 + s * C::TILE;
#pragma unroll
        for (int i = 0; i < PER; ++i)
          cp_async16(sk + ISTEP * i, kbase + static_cast<uint64_t>(tok[i]) * rstride);
        cp_async_arrive_noinc(&k_full[s]);
#pragma unroll
        for (int i = 0; i < PER; ++i)
          cp_async16(sv + ISTEP * i, vbase + static_cast<uint64_t>(tok[i]) * rstride);
        cp_async_arrive_noinc(&v_full[s]);
        issued = it + 1;
      }
      if (++s == C::NS) {
        s = 0;
        ph ^= 1u;
      }
    }
    cp_async_wait_all();
    if (bad) record_status(p.status, MCS_ERR_BAD_INDEX, bad_value);
    // back to the launch allocation so the shared teardown below sees one
    // limit, once the softmax warpgroups have returned their registers
    named_barrier<1, R::kThreads>();
    __syncwarp();  // setmaxnreg wants the whole warp converged
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R::kLaunchRegs));
  } else if (threadIdx.x < R::kLoader0 + R::kLoaders) {
    // ---------------------------------------------------------------- TMA producers (dense)
    const int pt = threadIdx.x - R::kLoader0;
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
        tma_load_3d(&tm_k, &k_full[s], sK + s * C::TILE + kb * 16384, kb * 64, h, b * p.N + key_tile(it) * 128);
      mbar_arrive_expect_tx(&v_full[s], C::TILE);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb)
        tma_load_3d(&tm_v, &v_full[s], sV + s * C::TILE + kb * 16384, kb * 64, h, b * p.N + key_tile(it) * 128);
      issued = it + 1;
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    if (R::kCpAsync) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R::kSoftRegs));
    const int half = (warp - R::kSoftWarp0) >> 2;  // column half of S; O_half accumulator
    const int wq = warp & 3;                       // TMEM lane quarter this warp may access
    const int row = wq * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_addr + half * 64;  // + 128 * buffer
    const uint32_t tO = tmem + lane_addr + 256;        // O_0 at +0, O_1 at +D
    const int pos = tile * 128 + row;
    constexpr bool kExport = MODE == ATTN_ANCHOR_DENSE;
    using LAcc = typename std::conditional<kExport, double, float>::type;  // row-sum accumulator
    const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
    const uint64_t scale2_lo = f2_pack(p.scale_log2_lo, p.scale_log2_lo);
    float m = -CUDART_INF_F;  // running max of scaled scores of this half, log2 units
    LAcc l = 0;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int pb = j & 1;
      if (!mbar_wait_warp(&s_full[pb], (j >> 1) & 1, wctx, MCS_WHERE_ATTN_SOFTMAX)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[64];
      tmem_ld32(tS + pb * 128, sv);
      tmem_ld32(tS + pb * 128 + 32, sv + 32);
      tmem_wait_ld();
      const int valid = p.kv_count - key_tile(j) * 128 - half * 64;  // existing keys of this half (may be <= 0)
      if (valid < 64) {
#pragma unroll
        for (int c = 0; c < 64; ++c) sv[c] = (c < valid) ? sv[c] : -CUDART_INF_F;
      }
      // row max: four chains of three-input max
      float mc[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float a = sv[k * 16];
#pragma unroll
        for (int e = 1; e < 15; e += 2) a = fmax3(a, sv[k * 16 + e], sv[k * 16 + e + 1]);
        mc[k] = fmaxf(a, sv[k * 16 + 15]);
      }
      const float mx = fmax3(fmaxf(mc[0], mc[1]), mc[2], mc[3]) * p.scale_log2;
      const bool need = mx > m + kRescaleThreshold;
      float alpha = 1.f;
      LAcc alpha_l = 1;      // the row sum's rescale factor (fp64 2^(m_old - m_new) in the export mode)
      bool rescale = false;  // warp-uniform: some row of this warp moves its max
      if (j == 0) {
        m = mx;
      } else {
        rescale = __any_sync(0xffffffffu, need);
        if (need) {
          alpha = fast_exp2(m - mx);  // 0 when nothing of this half was seen yet
          if (kExport)
            alpha_l = static_cast<LAcc>(exp2(static_cast<double>(m) - static_cast<double>(mx)));
          else
            alpha_l = static_cast<LAcc>(alpha);
          m = mx;
        }
      }
      // p = 2^(s * scale * log2 e - m); m is -inf only while every key of this
      // half so far was masked, and then every p is 0
      const float mu = (m == -CUDART_INF_F) ? 0.f : m;
      const uint64_t negm = f2_pack(-mu, -mu);
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const uint64_t s2 = f2_pack(sv[2 * q], sv[2 * q + 1]);
        uint64_t x = f2_fma(s2, scale2, negm);      // s*c_hi - m, rounded once
        if (kExport) x = f2_fma(s2, scale2_lo, x);  // + s*c_lo: the exponent to ~1 ulp of itself
        float x0, x1;
        f2_unpack(x, x0, x1);
        sv[2 * q] = fast_exp2(x0);
        sv[2 * q + 1] = fast_exp2(x1);
      }
      if (valid < 64) {  // masked keys: -inf * c_lo can be NaN, so zero them after the exponentials
#pragma unroll
        for (int c = 0; c < 64; ++c) sv[c] = (c < valid) ? sv[c] : 0.f;
      }
      // the tile's row sum as a balanced tree of packed adds (depth 6)
      uint64_t acc[16];
#pragma unroll
      for (int q = 0; q < 16; ++q)
        acc[q] = f2_add(f2_pack(sv[2 * q], sv[2 * q + 1]), f2_pack(sv[2 * q + 32], sv[2 * q + 33]));
#pragma unroll
      for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
        for (int q = 0; q < w; ++q) acc[q] = f2_add(acc[q], acc[q + w]);
      }
      float r0, r1;
      f2_unpack(acc[0], r0, r1);
      l = l * alpha_l + static_cast<LAcc>(r0 + r1);
      // P_h (bf16 pairs) over the first 32 columns of this half of the S
      // buffer; S_{j+2} is issued into the same buffer only after PV_j, and
      // UMMAs run in order
      {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(sv[2 * c], sv[2 * c + 1]);
        tmem_st32u(tS + pb * 128, pk);
      }
      tmem_wait_st();
      if (rescale) {
        // O_h holds tiles < j scaled by the old max: once PV_{j-1} of this half
        // is done, scale it by alpha before PV_j (which waits for p_full)
        if (!mbar_wait_warp(&p_empty[half * 2 + ((j - 1) & 1)], ((j - 1) >> 1) & 1, wctx,
                            MCS_WHERE_ATTN_SOFTMAX)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float ov[32];
          tmem_ld32(tO + half * D + c * 32, ov);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tmem_st32(tO + half * D + c * 32, ov);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&p_full[half * 2 + pb]);
    }
    // ---------------------------------------------------------------- epilogue
    // Both halves' last PV done -> exchange (m_h, l_h) through the dead Q tile
    // (every UMMA that reads it has completed) and merge; half h writes output
    // columns [h*D/2, (h+1)*D/2) of its row.
    const int lastb = (T - 1) & 1, lastp = ((T - 1) >> 1) & 1;
    const bool fin = ok && mbar_wait_warp(&p_empty[lastb], lastp, wctx, MCS_WHERE_ATTN_EPILOGUE) &&
                     mbar_wait_warp(&p_empty[2 + lastb], lastp, wctx, MCS_WHERE_ATTN_EPILOGUE);
    float* mx_x = reinterpret_cast<float*>(sQ);                 // [2][128] running max
    LAcc* l_x = reinterpret_cast<LAcc*>(sQ + 2 * 128 * sizeof(LAcc));  // [2][128] row sums
    if (fin) {
      mx_x[half * 128 + row] = m;
      l_x[half * 128 + row] = l;
    }
    named_barrier<2, 256>();
    if (fin) {
      tc_fence_after();
      const float m0 = mx_x[row], m1 = mx_x[128 + row];
      const float mm = fmaxf(m0, m1);  // finite: half 0 of tile 0 always holds a key
      const float c0 = fast_exp2(m0 - mm), c1 = fast_exp2(m1 - mm);  // 2^-inf = 0
      LAcc L;
      if (kExport)
        L = l_x[row] * exp2(static_cast<double>(m0) - static_cast<double>(mm)) +
            l_x[128 + row] * exp2(static_cast<double>(m1) - static_cast<double>(mm));
      else
        L = l_x[row] * c0 + l_x[128 + row] * c1;
      const float inv_L = 1.f / static_cast<float>(L);
      const float f0 = c0 * inv_L, f1 = c1 * inv_L;
      const bool row_valid = pos < p.N;
      const size_t head_base = static_cast<size_t>(b) * p.H + h;
      const size_t prow_idx = head_base * (static_cast<size_t>(p.G) * 128) + pos;  // padded perm-order row
      int tok = pos;
      if (row_valid && p.perm) tok = p.perm[head_base * p.N + pos];
      if (tok < 0 || tok >= p.N) tok = 0;
      if (half == 0 && (MODE == ATTN_DENSE || kExport)) {
        if (kExport) {
          // log2 of sum_j 2^(s_ij*scale*log2e), in fp64; exported negated as hi + lo
          const double lse2 = static_cast<double>(mm) + log2(static_cast<double>(L));
          const float nhi = static_cast<float>(-lse2);
          if (p.lse_perm_out) p.lse_perm_out[prow_idx] = row_valid ? nhi : -CUDART_INF_F;
          if (p.lse_perm_lo_out)
            p.lse_perm_lo_out[prow_idx] = row_valid ? static_cast<float>(-lse2 - static_cast<double>(nhi)) : 0.f;
          if (row_valid && p.lse_out)
            p.lse_out[head_base * p.N + tok] = static_cast<float>(lse2 * 0.69314718055994530942);
        } else if (row_valid && p.lse_out) {
          const float lse2 = mm + log2f(static_cast<float>(L));
          p.lse_out[head_base * p.N + tok] = lse2 * 0.69314718055994530942f;
        }
      }
      uint16_t* orow = p.o + (static_cast<size_t>(b) * p.N + tok) * p.H * D + static_cast<size_t>(h) * D;
      const size_t rrow = (head_base * p.N + (row_valid ? pos : 0)) * D;  // resid rows: [B,H,N,d] perm order
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        const int col = half * (D / 2) + cc * 32;
        float ov[32], o1[32];
        tmem_ld32(tO + col, ov);
        tmem_ld32(tO + D + col, o1);
        tmem_wait_ld();
        if (!row_valid) continue;
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] = ov[i] * f0 + o1[i] * f1;
        if (kExport && p.o_dense_out) {
          float4* dst = reinterpret_cast<float4*>(p.o_dense_out + prow_idx * D + col);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_float4(ov[4 * i], ov[4 * i + 1], ov[4 * i + 2], ov[4 * i + 3]);
        }
        if (MODE == ATTN_REUSE && p.resid_in) {
          const uint4* rsrc = reinterpret_cast<const uint4*>(p.resid_in + rrow + col);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 rv = rsrc[i];
            const uint16_t* rh = reinterpret_cast<const uint16_t*>(&rv);
#pragma unroll
            for (int e = 0; e < 8; ++e) ov[i * 8 + e] += bf16_to_f32(rh[e]);
          }
        }
        if (MODE == ATTN_ANCHOR_SPARSE) {
          const float4* dsrc = reinterpret_cast<const float4*>(p.o_dense_in + prow_idx * D + col);
          uint4* rdst = reinterpret_cast<uint4*>(p.resid_out + rrow + col);
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
          uint4* odst = reinterpret_cast<uint4*>(orow + col);
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
      named_barrier<1, R::kThreads>();
    }
  }

  // ------------------------------------------------------------------ teardown
  // All roles have left their loops. After an abort, wait (bounded, ignoring
  // the abort flag) for copies and UMMAs this CTA issued, then free TMEM.
  __syncthreads();
  if (*abort_flag) {
    volatile int never = 0;
    const WaitCtx drain_ctx{&never, nullptr, 50000000ull};
    if (threadIdx.x == R::kLoader0 && !R::kCpAsync) {  // cp.async loaders waited for their own copies
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
  using R = Roles<D, MODE>;
  static bool attr_set = false;
  auto kern = attn_kernel<D, MODE>;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    if (R::kCpAsync) {
      // the setmaxnreg split assumes exactly kLaunchRegs registers per thread at
      // launch; with fewer, a register increase could never be satisfied
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, kern);
      if (e != cudaSuccess) return e;
      if (fa.numRegs != R::kLaunchRegs) return cudaErrorInvalidKernelImage;
    }
    attr_set = true;
  }
  dim3 grid(static_cast<unsigned>(p.B * (p.hc > 0 ? p.hc : p.H) * p.G));
  kern<<<grid, R::kThreads, C::SMEM, s>>>(*tq, *tk, *tv, p);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_attention(int d, AttnMode mode, const CUtensorMap* tq, const CUtensorMap* tk,
                             const CUtensorMap* tv, const AttnParams& p, cudaStream_t s) {
  if (d == 128 && mode == ATTN_DENSE && !(p.debug_flags & 4)) return launch_attention_pair(tq, tk, tv, p, s);
  if (d == 128) {
    switch (mode) {
      case ATTN_DENSE: return launch_attn_t<128, ATTN_DENSE>(tq, tk, tv, p, s);
      case ATTN_ANCHOR_DENSE: return launch_attn_t<128, ATTN_ANCHOR_DENSE>(tq, tk, tv, p, s);
      case ATTN_REUSE: return launch_attn_t<128, ATTN_REUSE>(tq, tk, tv, p, s);
      case ATTN_ANCHOR_SPARSE: return launch_attn_t<128, ATTN_ANCHOR_SPARSE>(tq, tk, tv, p, s);
    }
  } else if (d == 64) {
    switch (mode) {
      case ATTN_DENSE: return launch_attn_t<64, ATTN_DENSE>(tq, tk, tv, p, s);
      case ATTN_ANCHOR_DENSE: return launch_attn_t<64, ATTN_ANCHOR_DENSE>(tq, tk, tv, p, s);
      case ATTN_REUSE: return launch_attn_t<64, ATTN_REUSE>(tq, tk, tv, p, s);
      case ATTN_ANCHOR_SPARSE: return launch_attn_t<64, ATTN_ANCHOR_SPARSE>(tq, tk, tv, p, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace mcs
