// Internal declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/mcs.h"

// status block word indices (int32 words at the start of the workspace)
#define MCS_SW_STATUS 0
#define MCS_SW_DETAIL 1
#define MCS_SW_BAND_OVERFLOW 2
#define MCS_SW_REFINED 3
#define MCS_SW_TOPK_FULL 4
#define MCS_SW_LANCZOS_STEPS 5  // grouping: Lanczos steps summed over all nodes (a diagnostic)
#define MCS_SW_LANCZOS_NODES 6  // grouping: nodes that ran Lanczos

// where-codes recorded as the status detail when a bounded wait expires
enum {
  MCS_WHERE_ATTN_PRODUCER = 1,
  MCS_WHERE_ATTN_MMA = 2,
  MCS_WHERE_ATTN_SOFTMAX = 3,
  MCS_WHERE_ATTN_EPILOGUE = 4,
  MCS_WHERE_MASS_PRODUCER = 11,
  MCS_WHERE_MASS_MMA = 12,
  MCS_WHERE_MASS_CONSUMER = 13,
  MCS_WHERE_DRAIN = 20,
};

namespace mcs {

// Basis vectors of one Lanczos cycle in the grouping's node kernel (its shared
// memory holds that many): the most Krylov steps a fixed-step grouping takes.
constexpr int kPddpKrylovMax = 64;

// ATTN_ANCHOR_DENSE is ATTN_DENSE plus the anchor's exports (fp32 O_dense, the
// lse as an fp32 hi/lo pair) computed with the exact-exponent arithmetic the
// fp64 selection re-score relies on.
enum AttnMode { ATTN_DENSE = 0, ATTN_REUSE = 1, ATTN_ANCHOR_SPARSE = 2, ATTN_ANCHOR_DENSE = 3 };

struct AttnParams {
  int B, H, N;
  int h0, hc;       // heads [h0, h0 + hc) of this launch (hc == 0: all H); strides use H
  int G;            // query tiles per (b,h)
  int kv_count;     // keys per tile list: N (dense) or K (sparse)
  float scale_log2;    // softmax scale * log2(e), rounded to fp32
  float scale_log2_lo; // the rounding residual: scale * log2(e) - scale_log2 (used by ATTN_ANCHOR_DENSE)
  const uint16_t *q, *k, *v;     // bf16 [B,N,H,d] (read directly by the gathered modes)
  const int32_t* perm;           // [B,H,N] or null (identity query order)
  const int32_t* kv_idx;         // [B,H,G,K] (sparse modes)
  const uint16_t* resid_in;      // reuse: bf16 [B,H,N,d] perm order (nullable)
  const float* o_dense_in;       // anchor sparse: fp32 [B,H,G*128,d] perm order
  uint16_t* o;                   // bf16 [B,N,H,d] token order (dense, reuse)
  float* o_dense_out;            // anchor dense: fp32 [B,H,G*128,d] perm order (nullable)
  float* lse_out;                // token order [B,H,N] (nullable)
  float* lse_perm_out;           // perm order [B,H,G*128], NEGATED lse in log2 units, -inf past N (nullable)
  float* lse_perm_lo_out;        // same rows: -lse2 - lse_perm_out in fp32 (the low part; 0 past N; nullable)
  uint16_t* resid_out;           // anchor sparse: bf16 [B,H,N,d] perm order
  int* status;                   // status block
  uint64_t wait_limit_ns;
  int debug_flags;
};

struct MassParams {
  int B, H, N, G, h0, hn;  // heads [h0, h0+hn) of this chunk
  float scale_log2;
  const int32_t* perm;     // [B,H,N] (unused by the kernel; queries come in group order)
  const float* lse_perm;   // [B,H,G*128] negated lse in log2 units (-lse * log2 e), -inf past N
  float* mass;             // [B,hn,G,N] for the chunk
  int* status;
  uint64_t wait_limit_ns;
};

struct TopkParams {
  int B, H, N, G, K, d, h0, hn;
  double scale;            // softmax scale (natural), in fp64 as the caller's shape defines it
  const float* mass;       // [B,hn,G,N]
  const uint16_t* q;       // bf16 [B,N,H,d]
  const uint16_t* k;
  const int32_t* perm;
  const float* lse_perm;   // [B,H,G*128] negated lse in log2 units (high part)
  const float* lse_perm_lo;  // [B,H,G*128] its low part: -lse2 = lse_perm + lse_perm_lo (fp64 sum)
  int32_t* kv_idx;         // [B,H,G,K]
  int* status;
  float band_rel;          // relative half-width of the uncertain band
  int cand_cap;            // set by launch_topk: keys of one bin the two-sweep path holds in shared memory
  int force_full;          // test hook: every group takes the general seven-sweep path
};

// launchers (return cudaSuccess or the launch error)
// plain dense attention (ATTN_DENSE) at d = 128 over pairs of query tiles (attn_pair.cu)
cudaError_t launch_attention_pair(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                                  const AttnParams& p, cudaStream_t s);
cudaError_t launch_attention(int d, AttnMode mode, const CUtensorMap* tq, const CUtensorMap* tk,
                             const CUtensorMap* tv, const AttnParams& p, cudaStream_t s);
cudaError_t launch_mass(int d, const CUtensorMap* tqp, const CUtensorMap* tk, const MassParams& p,
                        cudaStream_t s);
cudaError_t launch_permute_queries(const uint16_t* q, const int32_t* perm, uint16_t* qp, int B, int H, int N, int G,
                                   int d, int* status, cudaStream_t s);
cudaError_t launch_topk(const TopkParams& p, cudaStream_t s);
// packed selection (uint32 [rows, ceil(N/32)]) <-> ascending index lists (int32 [rows, K])
size_t meta_pack_smem_bytes(int N);
cudaError_t launch_meta_pack(const int32_t* idx, uint32_t* mask, long long rows, int N, int K, int* status,
                             cudaStream_t s);
cudaError_t launch_meta_unpack(const uint32_t* mask, int32_t* idx, long long rows, int N, int K, int* status,
                               cudaStream_t s);

// PDDP grouping: enqueue the whole recursion (fp64) for all heads
struct PddpPlan;
// krylov_steps: 0 = principal direction to convergence; k > 0 = top Ritz vector after k Lanczos steps;
// whiten: group the per-channel standardised queries
cudaError_t pddp_run(int B, int H, int N, int d, const uint16_t* q, int32_t* perm, void* ws, size_t ws_bytes,
                     int* status, int krylov_steps, bool whiten, cudaStream_t s);
size_t pddp_workspace_bytes(int B, int H, int N, int d);

// process-wide test knobs (see mcs_debug_set in api.cu)
int debug_flags();

// count of kernel launches this library made in the process (diagnostics)
void note_launches(int n);

}  // namespace mcs
