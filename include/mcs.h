/*
 * mcs.h — C ABI of the B200 (sm_100a) MC-Sparse hot path.
 *
 * MC-Sparse (Meta-Cached Sparse Attention) groups similar queries into
 * tile-sized groups, selects individual KV tokens per group from exact attention
 * probabilities at an "anchor" denoising step, caches the residual between dense
 * and sparse attention, and reuses query groups, KV indices and residual on the
 * following steps with fresh Q/K/V. Sources: the paper listing "MC-Sparse:
 * Deconstructing and Closing the Dense-Sparse Attention Gap in Diffusion
 * Transformers" (thelatestinai.com, Abstract; Tables 4, 6, 8) and the
 * aiwillknow.com analysis "MC-Sparse：高分辨率3D生成怎样减少注意力计算，又保住细结构？"
 * (section 图解主要方法, steps 1-5).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Device pointers are caller-owned (allocated by the caller, e.g. PyTorch);
 *    the library never allocates or frees device memory. Every compute call is
 *    asynchronous on the caller's stream and returns after enqueueing.
 *    Host memory appears only where a call says so: mcs_sparse_host (q, k, v
 *    and o on the host), mcs_meta_copy (one side of the copy), and the info
 *    words of mcs_poll_status and mcs_sparse_noalloc.
 *  - Tensors (row-major, contiguous, 16-byte aligned):
 *      q, k, v, o : bf16 [B, N, H, d]    (token-major, heads interleaved)
 *      perm       : int32 [B, H, N]      query permutation; group t of head
 *                                        (b,h) is perm[b,h, t*128 .. t*128+127]
 *                                        (the last group may be shorter)
 *      kv_idx     : int32 [B, H, G, K]   G = ceil(N/128); each row strictly
 *                                        ascending token indices in [0, N)
 *      resid      : bf16 [B, H, N, d]    residual R in permutation order: row t
 *                                        of head (b,h) belongs to query perm[b,h,t]
 *      lse        : fp32 [B, H, N]       log-sum-exp of scaled scores, token order
 *  - Supported shapes: d in {64, 128}; group == 128; 1 <= K <= N; N >= 1;
 *    B*N*H < 2^31. scale <= 0 selects 1/sqrt(d).
 *  - Workspace: `ws` of at least mcs_workspace_bytes(shape, op) bytes,
 *    256-byte aligned, caller-owned. Its first 256 bytes are the status block;
 *    they must be zero before the first call (allocate zeroed, or call
 *    mcs_poll_status once). Calls never clear it; device-side errors (a bound
 *    wait that expired, an index out of range) set it and the affected blocks
 *    stop; mcs_poll_status reports and clears it. Calls that share one
 *    workspace must be ordered on one stream.
 *  - Host-side validation happens before anything is enqueued: a bad argument
 *    returns an error and enqueues nothing. There is no fallback path.
 */
#ifndef MCS_H_
#define MCS_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MCS_GROUP_SIZE 128
#define MCS_STATUS_BYTES 256
#define MCS_INFO_WORDS 8

typedef enum mcs_status {
  MCS_OK = 0,
  MCS_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misalignment, small workspace */
  MCS_ERR_UNSUPPORTED = 2,  /* d not in {64,128}, group != 128, no sm_100 device   */
  MCS_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed                   */
  MCS_ERR_TIMEOUT = 4,      /* a bounded device wait expired (reported on poll)    */
  MCS_ERR_BAD_INDEX = 5     /* an index input was out of range (reported on poll)  */
} mcs_status;

typedef struct mcs_shape {
  int B, H, N, d;
  int group; /* query group size; must be 128 (one UMMA M tile) */
  int topk;  /* K: selected KV tokens per group (mcs_anchor, mcs_sparse) */
  float scale;
} mcs_shape;

typedef enum mcs_op { MCS_OP_GROUP = 0, MCS_OP_ANCHOR = 1, MCS_OP_SPARSE = 2, MCS_OP_DENSE = 3 } mcs_op;

/* Bytes of workspace `op` needs for `shape` (>= MCS_STATUS_BYTES); 0 if the
 * shape is invalid or unsupported. */
size_t mcs_workspace_bytes(const mcs_shape* shape, mcs_op op);

/*
 * Fast PDDP query grouping (aiwillknow analysis, step 1; paper Fig. 6 left).
 * Per (b,h): starting from all N queries, a node of n queries and
 * T = ceil(n/128) tiles is centred, its principal direction (top eigenvector of
 * the scatter matrix, oriented so its largest-magnitude entry is positive) is
 * found, and the ceil(T/2)*128 queries of smallest (projection, token index) go
 * to the left child, the rest to the right; children recurse until T == 1.
 * perm lists the leaves depth first, left before right, each leaf in ascending
 * token order. Arithmetic is fp64 (scatter, eigenvector, projections).
 * In: q. Out: perm [B,H,N]. Workspace: mcs_workspace_bytes(.., MCS_OP_GROUP).
 */
mcs_status mcs_group(const mcs_shape* shape, const void* q, int32_t* perm, void* ws, size_t ws_bytes,
                     cudaStream_t stream);

/*
 * "Fast" PDDP grouping (aiwillknow analysis, step 1 names the method Fast
 * PDDP; paper Table 7 times it; the pages give no iteration count): the same
 * tree, centring, projections, tile-rounded median split and output as
 * mcs_group, but each node's split direction is the top Ritz vector after
 * exactly krylov_steps Lanczos steps (full reorthogonalisation, one cycle)
 * instead of the converged principal eigenvector. The grouping is then an
 * approximation of mcs_group's: every output is still a valid grouping (a
 * permutation of each head's tokens, split at every node by the computed
 * projection), and where a node's leading eigenvalue is well separated a few
 * steps already give mcs_group's split. 2 <= krylov_steps <= min(d, 64) (one
 * Lanczos cycle holds at most 64 basis vectors), else MCS_ERR_INVALID_ARG; everything else as mcs_group (same workspace).
 */
mcs_status mcs_group_fast(const mcs_shape* shape, const void* q, int32_t* perm, int krylov_steps, void* ws,
                          size_t ws_bytes, cudaStream_t stream);

/*
 * Grouping with options (aiwillknow analysis, step 1; the project README's
 * TODO quoted on the aimodeling.com pages asks to "expose and validate
 * whitening support" without defining it). krylov_steps: 0 = mcs_group's
 * converged direction, 2..min(d, 64) = mcs_group_fast's. flags: MCS_GROUP_WHITEN groups
 * the per-channel standardised queries: per (b,h), channel c of every query is
 * divided by the standard deviation sigma_c of that channel over the head's N
 * queries (a constant channel is left as is), then the same tree, sign rule,
 * median split and output as mcs_group follow, all in fp64. The queries
 * themselves are not modified. Other flag bits, or krylov_steps outside
 * {0} U [2, min(d, 64)], return MCS_ERR_INVALID_ARG; same workspace as mcs_group.
 */
#define MCS_GROUP_WHITEN 1
mcs_status mcs_group_ex(const mcs_shape* shape, const void* q, int32_t* perm, int krylov_steps, int flags,
                        void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Anchor step (aiwillknow analysis, steps 2-3; paper Abstract, Table 4).
 * For every group g of perm: dense attention O_dense and lse over all N keys;
 * exact probabilities p_ij = exp(s_ij - lse_i) from a second QK^T pass; group
 * mass m_g(j) = sum_{i in g} p_ij; the K keys of largest mass (ties to the
 * lower index, emitted ascending) -> kv_idx; sparse attention over those keys,
 * renormalised over them -> O_sparse; resid = O_dense - O_sparse (bf16, perm
 * order). o receives O_dense (bf16, token order). lse (nullable) receives the
 * dense lse (token order).
 * Keys whose fp32 mass lies within a small band of the K-th largest are
 * re-ranked with fp64 scores, so selection matches exact-probability ranking.
 * stage_events (nullable) = 5 created events recorded before the dense pass, the
 * mass pass, the selection, the sparse pass, and after it (for timing
 * breakdowns; with several head chunks the mass/selection boundary is the first
 * chunk's). A null entry is an invalid argument.
 */
mcs_status mcs_anchor(const mcs_shape* shape, const void* q, const void* k, const void* v, const int32_t* perm,
                      void* o, int32_t* kv_idx, void* resid, float* lse, void* ws, size_t ws_bytes,
                      cudaStream_t stream, cudaEvent_t* stage_events);

/*
 * Reuse step (aiwillknow analysis, step 4; paper Abstract, Table 6 kernel):
 * fresh q/k/v, cached perm, kv_idx and resid. For query i of group g:
 * o_i = sum_{j in kv_idx[g]} softmax_j(scale * q_i.k_j) v_j + resid_i, written
 * bf16 to token order. resid may be NULL (plain token-sparse attention).
 */
mcs_status mcs_sparse(const mcs_shape* shape, const void* q, const void* k, const void* v, const int32_t* perm,
                      const int32_t* kv_idx, const void* resid, void* o, void* ws, size_t ws_bytes,
                      cudaStream_t stream);

/*
 * The reuse step (as mcs_sparse) for callers that cannot allocate device
 * memory where they run it -- for example a runtime that reserves all device
 * memory up front and hands out only tensor buffers, or a plug-in that must
 * not touch the allocator. The pages have no counterpart to this call; it
 * exists for such callers.
 * No workspace argument: the kernel's only scratch, its 256-byte status block,
 * is a static device array that each GPU loading this library holds until
 * the process exits. Limit: the shape's MCS_OP_SPARSE workspace must fit in
 * 256 bytes (true for every supported shape today); a larger need returns
 * MCS_ERR_INVALID_ARG. The call allocates nothing (no cudaMalloc, no
 * allocating library routine). The first call on a device resolves the
 * array's device address for that device and caches it for the life of the
 * process, so make that first call before any stream capture, and do not use
 * this entry point again on a device after cudaDeviceReset (the cached
 * address would be stale). Every call clears the array (an asynchronous
 * memset on `stream`) and reuses it, so calls whose kernels overlap on the GPU
 * race on it and may report each other's status.
 * info (nullable, host memory, MCS_INFO_WORDS int32 words): when given, the
 * call waits for `stream`, fills info as mcs_poll_status does and returns the
 * device status; info is written only when the call gets that far (its return
 * value is then MCS_OK or a device-side code). On a host-side error (invalid
 * arguments, a CUDA error while enqueueing) info is left unwritten. When info
 * is NULL the call returns after enqueueing and device-side errors are not
 * reported.
 */
mcs_status mcs_sparse_noalloc(const mcs_shape* shape, const void* q, const void* k, const void* v,
                              const int32_t* perm, const int32_t* kv_idx, const void* resid, void* o,
                              int32_t* info, cudaStream_t stream);

/*
 * The reuse step (as mcs_sparse) with q, k, v and o in HOST memory: the call a
 * user makes when the step's inputs arrive from, and its output returns to, the
 * host. Attention is independent per head, so the heads are split into
 * head_chunks contiguous ranges (chunk c = heads [c*H/n, (c+1)*H/n)), and for
 * each range the copy of its q/k/v columns into the device buffers (on
 * copy_in), the reuse kernel over those heads (on stream) and the copy of its o
 * columns back (on copy_out) are chained by events, so the copies of one chunk
 * overlap the kernel of another. The pages have no counterpart to this call;
 * its arithmetic is exactly mcs_sparse's (bit-identical output for any
 * head_chunks).
 * Layouts: q_host, k_host, v_host, o_host and q_dev, k_dev, v_dev, o_dev are
 * bf16 [B, N, H, d] (token order). Host buffers should be pinned
 * (cudaHostAlloc) for the copies to run asynchronously; pageable memory works
 * but serialises. perm, kv_idx and resid are device buffers as in mcs_sparse;
 * the caller owns every buffer and keeps them alive until `stream` has passed
 * the call. Ordering: the copies start after work enqueued on `stream` before
 * the call, and `stream` is ordered after the last output copy, so
 * synchronising `stream` makes o_host valid. copy_in and copy_out should be
 * non-blocking streams other than `stream`; any streams give the same result,
 * but shared or blocking ones serialise the copies with the kernels.
 * 1 <= head_chunks <= min(H, 64), else
 * MCS_ERR_INVALID_ARG; device-side errors land in ws as for mcs_sparse.
 */
mcs_status mcs_sparse_host(const mcs_shape* shape, const void* q_host, const void* k_host, const void* v_host,
                           const int32_t* perm, const int32_t* kv_idx, const void* resid, void* o_host,
                           void* q_dev, void* k_dev, void* v_dev, void* o_dev, int head_chunks, void* ws,
                           size_t ws_bytes, cudaStream_t stream, cudaStream_t copy_in, cudaStream_t copy_out);

/*
 * Dense attention baseline (the denominator of the paper's Table 6 speedups):
 * o = softmax(scale * q k^T) v over all N keys, bf16 token order; lse
 * (nullable) fp32 [B,H,N].
 */
mcs_status mcs_dense(const mcs_shape* shape, const void* q, const void* k, const void* v, void* o, float* lse,
                     void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Metadata offload / prefetch (aiwillknow analysis, step 5; paper Table 8):
 * the per-layer metadata (kv_idx and resid) leaves the GPU after the anchor
 * and the next layer's copy comes back while the current layer computes.
 * Enqueues on the `side` stream: a wait for `wait` (nullable; e.g. an event
 * recorded after the anchor that wrote the metadata, or after the last kernel
 * that read the device buffer about to be overwritten), then an asynchronous
 * copy of `bytes` bytes, device->host when to_host != 0, else host->device,
 * then a record of `done` (nullable; the compute stream waits on it before it
 * uses prefetched metadata). The host buffer must be pinned for the copy to
 * overlap compute; pageable memory works but serialises. bytes == 0 enqueues
 * nothing. Null dst/src with bytes > 0 is an invalid argument.
 */
mcs_status mcs_meta_copy(void* dst, const void* src, size_t bytes, int to_host, cudaStream_t side, cudaEvent_t wait,
                         cudaEvent_t done);

/*
 * Packed selection for metadata offload (aiwillknow analysis, step 5; paper
 * Table 8 counts the selection as int32 lists). The pages have no packed
 * form; this one is exact and smaller than the lists whenever K > N/32.
 * Layout: uint32 words [B, H, G, W], W = ceil(N/32), G = ceil(N/group); in
 * row (b, h, g), bit (j mod 32) of word floor(j/32) is set exactly when key j
 * is in the group's selection, and bits at positions >= N are zero.
 * mcs_meta_mask_bytes: bytes of that array (0 for an invalid shape; topk is
 * required).
 * mcs_meta_pack: kv_idx [B,H,G,K] (strictly ascending lists, as mcs_anchor
 * writes them) -> mask. mcs_meta_unpack: mask -> kv_idx, ascending.
 * Both are device-to-device, enqueued on `stream`, and allocate nothing; ws is
 * any workspace of at least MCS_STATUS_BYTES (e.g. the MCS_OP_SPARSE one),
 * whose status block receives MCS_ERR_BAD_INDEX for an index out of range or
 * out of order (pack), or for a row whose popcount is not K or with bits at
 * positions >= N (unpack); the caller reads it with mcs_poll_status. Writes
 * never leave the destination rows. Invalid shapes or null pointers return
 * MCS_ERR_INVALID_ARG; N above 1,859,584 (a row's words beyond 227 KB of
 * shared memory) returns MCS_ERR_UNSUPPORTED from mcs_meta_pack.
 */
size_t mcs_meta_mask_bytes(const mcs_shape* shape);
mcs_status mcs_meta_pack(const mcs_shape* shape, const int32_t* kv_idx, uint32_t* mask, void* ws, size_t ws_bytes,
                         cudaStream_t stream);
mcs_status mcs_meta_unpack(const mcs_shape* shape, const uint32_t* mask, int32_t* kv_idx, void* ws,
                           size_t ws_bytes, cudaStream_t stream);

/*
 * Synchronises `stream`, reads the status block of `ws`, clears it, and returns
 * the recorded status (MCS_OK if none). info (nullable) receives
 * MCS_INFO_WORDS int32 words: [0] status, [1] detail (where/which index),
 * [2] anchor selections whose uncertain band overflowed and fell back to fp32
 * ranking, [3] keys re-ranked in fp64, [4] anchor selections that took the
 * general seven-sweep top-K path instead of the two-sweep one (same result;
 * a performance counter), [5] grouping: Lanczos steps summed over all nodes,
 * [6] grouping: nodes (performance counters; [5] / [6] is the mean number of
 * steps to convergence), [7] reserved.
 */
mcs_status mcs_poll_status(void* ws, int32_t* info, cudaStream_t stream);

/* Static, human-readable name of a status code. */
const char* mcs_status_string(mcs_status status);

#ifdef __cplusplus
}
#endif

#endif /* MCS_H_ */
