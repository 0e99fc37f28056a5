// C ABI entry points of the MC-Sparse library (declared in include/mcs.h):
// host-side validation, TMA tensor-map encoding, workspace layout, and the
// launch sequence of each call. No device memory is allocated here.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "mcs_internal.h"
#include "../../include/mcs_test.h"

namespace mcs {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
int g_debug_flags = 0;
std::atomic<long long> g_launches{0};
cudaEvent_t const* g_chunk_events = nullptr;  // measurement hook: events around the anchor's chunk launches
int g_chunk_event_count = 0;

constexpr uint64_t kWaitLimitNs = 2000000000ull;    // 2 s per bounded device wait
constexpr size_t kMassBudget = size_t(2) << 30;      // bytes of mass matrix per head chunk
// Half-width of the fp32-mass uncertainty band around the K-th largest mass,
// 2^-11 relative. A group's fp32 mass carries at most ~1e-4 relative error
// (one exponential pair in four on the FMA-pipe polynomial, 7.5e-5; fp32 sums
// over 128 rows; fp32 tensor-core scores; the lse), so two keys can only swap
// order in fp32 when their exact masses are within ~2e-4: every such key lies
// inside the band, with a margin of about 2.5, and is re-ranked in fp64.
constexpr float kBandRel = 4.8828125e-4f;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

mcs_status encode_init() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode ? MCS_OK : MCS_ERR_CUDA;
}

// 2-D map over the rows of a [B, N, H, d] bf16 tensor (row = one head of one
// token), box {64 elements, 1 row}, 128-byte swizzle: the gather4 source.
mcs_status rows_map(CUtensorMap* m, const void* base, uint64_t rows, int d) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), rows};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MCS_OK : MCS_ERR_CUDA;
}

// 3-D map over the same tensor viewed as [B*N, H, d], box {64, 1, 128}: 128
// consecutive tokens of one head per load (dense key/value tiles).
mcs_status tokens_map(CUtensorMap* m, const void* base, uint64_t tokens, int H, int d) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), tokens};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MCS_OK : MCS_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mcs_status check_device() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MCS_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return MCS_ERR_CUDA;
  return major == 10 ? MCS_OK : MCS_ERR_UNSUPPORTED;
}

mcs_status check_shape(const mcs_shape* s, bool need_topk) {
  if (!s) return MCS_ERR_INVALID_ARG;
  if (s->B < 1 || s->H < 1 || s->N < 1 || s->d < 1) return MCS_ERR_INVALID_ARG;
  if (static_cast<long long>(s->B) * s->N * s->H >= (1ll << 31)) return MCS_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return MCS_ERR_UNSUPPORTED;
  if (s->group != MCS_GROUP_SIZE) return MCS_ERR_UNSUPPORTED;
  if (need_topk && (s->topk < 1 || s->topk > s->N)) return MCS_ERR_INVALID_ARG;
  if (!(s->scale == s->scale) || isinf(s->scale)) return MCS_ERR_INVALID_ARG;
  return MCS_OK;
}

// softmax scale in fp64: the caller's value, or 1/sqrt(d)
double scale_of(const mcs_shape* s) { return s->scale > 0.f ? static_cast<double>(s->scale) : 1.0 / sqrt(static_cast<double>(s->d)); }

// scale * log2(e) as an fp32 value and its fp32 rounding residual
void scale_log2_parts(const mcs_shape* s, float* hi, float* lo) {
  const double c = scale_of(s) * 1.4426950408889634074;
  *hi = static_cast<float>(c);
  *lo = static_cast<float>(c - static_cast<double>(*hi));
}
int groups_of(const mcs_shape* s) { return (s->N + MCS_GROUP_SIZE - 1) / MCS_GROUP_SIZE; }

// anchor workspace layout
struct AnchorWs {
  size_t o_dense, lse_perm, lse_perm_lo, qp, mass, total;
  int heads_per_chunk;
};

AnchorWs anchor_layout(const mcs_shape* s) {
  AnchorWs w{};
  const size_t G = groups_of(s);
  const size_t rows = static_cast<size_t>(s->B) * s->H * G * MCS_GROUP_SIZE;
  size_t off = MCS_STATUS_BYTES;
  w.o_dense = off;
  off = align_up(off + rows * s->d * sizeof(float), 256);
  w.lse_perm = off;
  off = align_up(off + rows * sizeof(float), 256);
  w.lse_perm_lo = off;
  off = align_up(off + rows * sizeof(float), 256);
  w.qp = off;  // queries in group order, bf16 [B, H, G*128, d]
  off = align_up(off + rows * s->d * 2, 256);
  const size_t per_head = static_cast<size_t>(s->B) * G * s->N * sizeof(float);
  size_t hc = kMassBudget / per_head;
  if (hc < 1) hc = 1;
  if (hc > static_cast<size_t>(s->H)) hc = s->H;
  w.heads_per_chunk = static_cast<int>(hc);
  w.mass = off;
  off = align_up(off + hc * per_head, 256);
  w.total = off;
  return w;
}

mcs_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MCS_OK : MCS_ERR_CUDA; }

}  // namespace

int debug_flags() { return g_debug_flags; }
void note_launches(int n) { g_launches += n; }

}  // namespace mcs

using namespace mcs;

extern "C" {

size_t mcs_workspace_bytes(const mcs_shape* s, mcs_op op) {
  if (check_shape(s, op == MCS_OP_ANCHOR || op == MCS_OP_SPARSE) != MCS_OK) return 0;
  switch (op) {
    case MCS_OP_DENSE:
    case MCS_OP_SPARSE:
      return MCS_STATUS_BYTES;
    case MCS_OP_ANCHOR:
      return anchor_layout(s).total;
    case MCS_OP_GROUP:
      return MCS_STATUS_BYTES + pddp_workspace_bytes(s->B, s->H, s->N, s->d);
  }
  return 0;
}

const char* mcs_status_string(mcs_status st) {
  switch (st) {
    case MCS_OK: return "MCS_OK";
    case MCS_ERR_INVALID_ARG: return "MCS_ERR_INVALID_ARG";
    case MCS_ERR_UNSUPPORTED: return "MCS_ERR_UNSUPPORTED";
    case MCS_ERR_CUDA: return "MCS_ERR_CUDA";
    case MCS_ERR_TIMEOUT: return "MCS_ERR_TIMEOUT";
    case MCS_ERR_BAD_INDEX: return "MCS_ERR_BAD_INDEX";
  }
  return "MCS_ERR_UNKNOWN";
}

mcs_status mcs_dense(const mcs_shape* s, const void* q, const void* k, const void* v, void* o, float* lse, void* ws,
                     size_t ws_bytes, cudaStream_t stream) {
  mcs_status st = check_shape(s, false);
  if (st != MCS_OK) return st;
  if (!q || !k || !v || !o || !ws) return MCS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)))
    return MCS_ERR_INVALID_ARG;
  if (ws_bytes < mcs_workspace_bytes(s, MCS_OP_DENSE)) return MCS_ERR_INVALID_ARG;
  if ((st = check_device()) != MCS_OK) return st;
  if ((st = encode_init()) != MCS_OK) return st;
  const uint64_t rows = static_cast<uint64_t>(s->B) * s->N * s->H;
  CUtensorMap tq, tk, tv;
  if (rows_map(&tq, q, rows, s->d) || tokens_map(&tk, k, static_cast<uint64_t>(s->B) * s->N, s->H, s->d) ||
      tokens_map(&tv, v, static_cast<uint64_t>(s->B) * s->N, s->H, s->d))
    return MCS_ERR_CUDA;
  AttnParams p{};
  p.B = s->B; p.H = s->H; p.N = s->N; p.G = groups_of(s);
  p.kv_count = s->N;
  scale_log2_parts(s, &p.scale_log2, &p.scale_log2_lo);
  p.o = static_cast<uint16_t*>(o);
  p.lse_out = lse;
  p.status = static_cast<int*>(ws);
  p.wait_limit_ns = kWaitLimitNs;
  p.debug_flags = g_debug_flags;
  return cuda_status(launch_attention(s->d, ATTN_DENSE, &tq, &tk, &tv, p, stream));
}

}  // extern "C"

namespace {

// The reuse step over heads [h0, h0 + hc) of full-size tensors (hc == 0: all).
mcs_status launch_reuse(const mcs_shape* s, const void* q, const void* k, const void* v, const int32_t* perm,
                        const int32_t* kv_idx, const void* resid, void* o, void* ws, int h0, int hc,
                        cudaStream_t stream) {
  mcs_status st;
  if ((st = encode_init()) != MCS_OK) return st;
  const uint64_t rows = static_cast<uint64_t>(s->B) * s->N * s->H;
  CUtensorMap tq, tk, tv;
  if (rows_map(&tq, q, rows, s->d) || rows_map(&tk, k, rows, s->d) || rows_map(&tv, v, rows, s->d))
    return MCS_ERR_CUDA;
  AttnParams p{};
  p.B = s->B; p.H = s->H; p.N = s->N; p.G = groups_of(s);
  p.h0 = h0;
  p.hc = hc;
  p.kv_count = s->topk;
  scale_log2_parts(s, &p.scale_log2, &p.scale_log2_lo);
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.perm = perm;
  p.kv_idx = kv_idx;
  p.resid_in = static_cast<const uint16_t*>(resid);
  p.o = static_cast<uint16_t*>(o);
  p.status = static_cast<int*>(ws);
  p.wait_limit_ns = kWaitLimitNs;
  p.debug_flags = g_debug_flags;
  return cuda_status(launch_attention(s->d, ATTN_REUSE, &tq, &tk, &tv, p, stream));
}

}  // namespace

extern "C" {

mcs_status mcs_sparse(const mcs_shape* s, const void* q, const void* k, const void* v, const int32_t* perm,
                      const int32_t* kv_idx, const void* resid, void* o, void* ws, size_t ws_bytes,
                      cudaStream_t stream) {
  mcs_status st = check_shape(s, true);
  if (st != MCS_OK) return st;
  if (!q || !k || !v || !perm || !kv_idx || !o || !ws) return MCS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (resid && !aligned16(resid)))
    return MCS_ERR_INVALID_ARG;
  if (ws_bytes < mcs_workspace_bytes(s, MCS_OP_SPARSE)) return MCS_ERR_INVALID_ARG;
  if ((st = check_device()) != MCS_OK) return st;
  return launch_reuse(s, q, k, v, perm, kv_idx, resid, o, ws, 0, 0, stream);
}

mcs_status mcs_sparse_host(const mcs_shape* s, const void* q_host, const void* k_host, const void* v_host,
                           const int32_t* perm, const int32_t* kv_idx, const void* resid, void* o_host,
                           void* q_dev, void* k_dev, void* v_dev, void* o_dev, int head_chunks, void* ws,
                           size_t ws_bytes, cudaStream_t stream, cudaStream_t copy_in, cudaStream_t copy_out) {
  mcs_status st = check_shape(s, true);
  if (st != MCS_OK) return st;
  if (!q_host || !k_host || !v_host || !o_host || !q_dev || !k_dev || !v_dev || !o_dev || !perm || !kv_idx || !ws)
    return MCS_ERR_INVALID_ARG;
  if (!aligned16(q_dev) || !aligned16(k_dev) || !aligned16(v_dev) || !aligned16(o_dev) ||
      (resid && !aligned16(resid)))
    return MCS_ERR_INVALID_ARG;
  if (head_chunks < 1 || head_chunks > s->H || head_chunks > 64) return MCS_ERR_INVALID_ARG;
  if (ws_bytes < mcs_workspace_bytes(s, MCS_OP_SPARSE)) return MCS_ERR_INVALID_ARG;
  if ((st = check_device()) != MCS_OK) return st;
  // events of this call (host-side objects; released once their work is done)
  const int nev = 2 * head_chunks + 2;
  cudaEvent_t ev[2 * 64 + 2];
  int made = 0;
  for (; made < nev; ++made)
    if (cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming) != cudaSuccess) break;
  auto finish = [&](mcs_status r) {
    for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
    return r;
  };
  if (made < nev) return finish(MCS_ERR_CUDA);
  cudaEvent_t start = ev[0], out_done = ev[1];
  // the copies into the device buffers start after earlier work on `stream`
  if (cudaEventRecord(start, stream) != cudaSuccess || cudaStreamWaitEvent(copy_in, start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(copy_out, start, 0) != cudaSuccess)
    return finish(MCS_ERR_CUDA);
  const size_t pitch = static_cast<size_t>(s->H) * s->d * 2;  // bytes per token row
  const size_t height = static_cast<size_t>(s->B) * s->N;
  const void* hin[3] = {q_host, k_host, v_host};
  void* din[3] = {q_dev, k_dev, v_dev};
  for (int c = 0; c < head_chunks; ++c) {
    const int h0 = static_cast<int>(static_cast<long long>(c) * s->H / head_chunks);
    const int h1 = static_cast<int>(static_cast<long long>(c + 1) * s->H / head_chunks);
    const size_t off = static_cast<size_t>(h0) * s->d * 2, width = static_cast<size_t>(h1 - h0) * s->d * 2;
    cudaEvent_t landed = ev[2 + 2 * c], computed = ev[3 + 2 * c];
    for (int t = 0; t < 3; ++t)
      if (cudaMemcpy2DAsync(static_cast<char*>(din[t]) + off, pitch, static_cast<const char*>(hin[t]) + off, pitch,
                            width, height, cudaMemcpyHostToDevice, copy_in) != cudaSuccess)
        return finish(MCS_ERR_CUDA);
    if (cudaEventRecord(landed, copy_in) != cudaSuccess || cudaStreamWaitEvent(stream, landed, 0) != cudaSuccess)
      return finish(MCS_ERR_CUDA);
    if ((st = launch_reuse(s, q_dev, k_dev, v_dev, perm, kv_idx, resid, o_dev, ws, h0, h1 - h0, stream)) != MCS_OK)
      return finish(st);
    if (cudaEventRecord(computed, stream) != cudaSuccess || cudaStreamWaitEvent(copy_out, computed, 0) != cudaSuccess)
      return finish(MCS_ERR_CUDA);
    if (cudaMemcpy2DAsync(static_cast<char*>(o_host) + off, pitch, static_cast<const char*>(o_dev) + off, pitch,
                          width, height, cudaMemcpyDeviceToHost, copy_out) != cudaSuccess)
      return finish(MCS_ERR_CUDA);
  }
  // completion of the whole call, output copies included, is ordered on `stream`
  if (cudaEventRecord(out_done, copy_out) != cudaSuccess || cudaStreamWaitEvent(stream, out_done, 0) != cudaSuccess)
    return finish(MCS_ERR_CUDA);
  return finish(MCS_OK);
}

mcs_status mcs_anchor(const mcs_shape* s, const void* q, const void* k, const void* v, const int32_t* perm, void* o,
                      int32_t* kv_idx, void* resid, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream,
                      cudaEvent_t* ev) {
  mcs_status st = check_shape(s, true);
  if (st != MCS_OK) return st;
  if (!q || !k || !v || !perm || !o || !kv_idx || !resid || !ws) return MCS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(resid) ||
      (lse && !aligned16(lse)))
    return MCS_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MCS_ERR_INVALID_ARG;
  if (ws_bytes < mcs_workspace_bytes(s, MCS_OP_ANCHOR)) return MCS_ERR_INVALID_ARG;
  if (ev)
    for (int i = 0; i < 5; ++i)
      if (!ev[i]) return MCS_ERR_INVALID_ARG;
  if ((st = check_device()) != MCS_OK) return st;
  if ((st = encode_init()) != MCS_OK) return st;
  const AnchorWs L = anchor_layout(s);
  uint8_t* w = static_cast<uint8_t*>(ws);
  const uint64_t rows = static_cast<uint64_t>(s->B) * s->N * s->H;
  CUtensorMap tq, tk, tv;
  if (rows_map(&tq, q, rows, s->d) || rows_map(&tk, k, rows, s->d) || rows_map(&tv, v, rows, s->d))
    return MCS_ERR_CUDA;
  const int G = groups_of(s);
  float scale_log2 = 0.f, scale_log2_lo = 0.f;
  scale_log2_parts(s, &scale_log2, &scale_log2_lo);
  float* o_dense = reinterpret_cast<float*>(w + L.o_dense);
  float* lse_perm = reinterpret_cast<float*>(w + L.lse_perm);
  float* lse_perm_lo = reinterpret_cast<float*>(w + L.lse_perm_lo);
  float* mass = reinterpret_cast<float*>(w + L.mass);
  int* status = static_cast<int*>(ws);
  if (ev && cudaEventRecord(ev[0], stream) != cudaSuccess) return MCS_ERR_CUDA;
  // pass 1: dense attention + lse, queries in group order
  AttnParams pd{};
  pd.B = s->B; pd.H = s->H; pd.N = s->N; pd.G = G;
  pd.kv_count = s->N;
  pd.scale_log2 = scale_log2;
  pd.scale_log2_lo = scale_log2_lo;
  pd.perm = perm;
  pd.o = static_cast<uint16_t*>(o);
  pd.o_dense_out = o_dense;
  pd.lse_out = lse;
  pd.lse_perm_out = lse_perm;
  pd.lse_perm_lo_out = lse_perm_lo;
  pd.status = status;
  pd.wait_limit_ns = kWaitLimitNs;
  pd.debug_flags = g_debug_flags;
  CUtensorMap tk3, tv3;
  if (tokens_map(&tk3, k, static_cast<uint64_t>(s->B) * s->N, s->H, s->d) ||
      tokens_map(&tv3, v, static_cast<uint64_t>(s->B) * s->N, s->H, s->d))
    return MCS_ERR_CUDA;
  if (launch_attention(s->d, ATTN_ANCHOR_DENSE, &tq, &tk3, &tv3, pd, stream) != cudaSuccess)
    return MCS_ERR_CUDA;
  if (ev && cudaEventRecord(ev[1], stream) != cudaSuccess) return MCS_ERR_CUDA;
  // passes 2-3: exact probabilities -> group mass -> top-K, one head chunk at a time.
  // The mass pass streams queries in group order from one permuted copy.
  uint16_t* qp = reinterpret_cast<uint16_t*>(w + L.qp);
  if (launch_permute_queries(static_cast<const uint16_t*>(q), perm, qp, s->B, s->H, s->N, G, s->d, status, stream) !=
      cudaSuccess)
    return MCS_ERR_CUDA;
  CUtensorMap tqp;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(s->d), static_cast<cuuint64_t>(s->B) * s->H * G * 128};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(s->d) * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    if (g_encode(&tqp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qp, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MCS_ERR_CUDA;
  }
  for (int h0 = 0, c = 0; h0 < s->H; h0 += L.heads_per_chunk, ++c) {
    const int hn = (s->H - h0 < L.heads_per_chunk) ? (s->H - h0) : L.heads_per_chunk;
    cudaEvent_t const* cev = (g_chunk_events && 3 * c + 2 < g_chunk_event_count) ? g_chunk_events + 3 * c : nullptr;
    if (cev && cudaEventRecord(cev[0], stream) != cudaSuccess) return MCS_ERR_CUDA;
    MassParams pm{};
    pm.B = s->B; pm.H = s->H; pm.N = s->N; pm.G = G; pm.h0 = h0; pm.hn = hn;
    pm.scale_log2 = scale_log2;
    pm.perm = perm;
    pm.lse_perm = lse_perm;
    pm.mass = mass;
    pm.status = status;
    pm.wait_limit_ns = kWaitLimitNs;
    if (launch_mass(s->d, &tqp, &tk3, pm, stream) != cudaSuccess) return MCS_ERR_CUDA;
    if (ev && h0 == 0 && cudaEventRecord(ev[2], stream) != cudaSuccess) return MCS_ERR_CUDA;
    if (cev && cudaEventRecord(cev[1], stream) != cudaSuccess) return MCS_ERR_CUDA;
    TopkParams pt{};
    pt.B = s->B; pt.H = s->H; pt.N = s->N; pt.G = G; pt.K = s->topk; pt.d = s->d; pt.h0 = h0; pt.hn = hn;
    pt.scale = scale_of(s);
    pt.mass = mass;
    pt.q = static_cast<const uint16_t*>(q);
    pt.k = static_cast<const uint16_t*>(k);
    pt.perm = perm;
    pt.lse_perm = lse_perm;
    pt.lse_perm_lo = lse_perm_lo;
    pt.kv_idx = kv_idx;
    pt.status = status;
    pt.band_rel = kBandRel;
    pt.force_full = (g_debug_flags & 2) != 0;
    if (launch_topk(pt, stream) != cudaSuccess) return MCS_ERR_CUDA;
    if (cev && cudaEventRecord(cev[2], stream) != cudaSuccess) return MCS_ERR_CUDA;
  }
  if (ev && cudaEventRecord(ev[3], stream) != cudaSuccess) return MCS_ERR_CUDA;
  // pass 4: sparse attention over the selection at the anchor, R = O_dense - O_sparse
  AttnParams ps{};
  ps.B = s->B; ps.H = s->H; ps.N = s->N; ps.G = G;
  ps.kv_count = s->topk;
  ps.scale_log2 = scale_log2;
  ps.scale_log2_lo = scale_log2_lo;
  ps.q = static_cast<const uint16_t*>(q);
  ps.k = static_cast<const uint16_t*>(k);
  ps.v = static_cast<const uint16_t*>(v);
  ps.perm = perm;
  ps.kv_idx = kv_idx;
  ps.o_dense_in = o_dense;
  ps.resid_out = static_cast<uint16_t*>(resid);
  ps.status = status;
  ps.wait_limit_ns = kWaitLimitNs;
  ps.debug_flags = g_debug_flags;
  if (launch_attention(s->d, ATTN_ANCHOR_SPARSE, &tq, &tk, &tv, ps, stream) != cudaSuccess)
    return MCS_ERR_CUDA;
  if (ev && cudaEventRecord(ev[4], stream) != cudaSuccess) return MCS_ERR_CUDA;
  return MCS_OK;
}

}  // extern "C"

namespace {

mcs_status group_call(const mcs_shape* s, const void* q, int32_t* perm, void* ws, size_t ws_bytes,
                      int krylov_steps, bool whiten, cudaStream_t stream) {
  mcs_status st = check_shape(s, false);
  if (st != MCS_OK) return st;
  if (!q || !perm || !ws) return MCS_ERR_INVALID_ARG;
  if (!aligned16(q) || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MCS_ERR_INVALID_ARG;
  if (ws_bytes < mcs_workspace_bytes(s, MCS_OP_GROUP)) return MCS_ERR_INVALID_ARG;
  if ((st = check_device()) != MCS_OK) return st;
  uint8_t* w = static_cast<uint8_t*>(ws);
  return cuda_status(pddp_run(s->B, s->H, s->N, s->d, static_cast<const uint16_t*>(q), perm, w + MCS_STATUS_BYTES,
                              ws_bytes - MCS_STATUS_BYTES, static_cast<int*>(ws), krylov_steps, whiten, stream));
}

}  // namespace

extern "C" {

mcs_status mcs_group(const mcs_shape* s, const void* q, int32_t* perm, void* ws, size_t ws_bytes,
                     cudaStream_t stream) {
  return group_call(s, q, perm, ws, ws_bytes, 0, false, stream);
}

mcs_status mcs_group_fast(const mcs_shape* s, const void* q, int32_t* perm, int krylov_steps, void* ws,
                          size_t ws_bytes, cudaStream_t stream) {
  if (!s || krylov_steps < 2 || krylov_steps > std::min(s->d, kPddpKrylovMax)) return MCS_ERR_INVALID_ARG;
  return group_call(s, q, perm, ws, ws_bytes, krylov_steps, false, stream);
}

mcs_status mcs_group_ex(const mcs_shape* s, const void* q, int32_t* perm, int krylov_steps, int flags, void* ws,
                        size_t ws_bytes, cudaStream_t stream) {
  if (!s || (krylov_steps != 0 && (krylov_steps < 2 || krylov_steps > std::min(s->d, kPddpKrylovMax))))
    return MCS_ERR_INVALID_ARG;
  if ((flags & ~MCS_GROUP_WHITEN) != 0) return MCS_ERR_INVALID_ARG;
  return group_call(s, q, perm, ws, ws_bytes, krylov_steps, (flags & MCS_GROUP_WHITEN) != 0, stream);
}

size_t mcs_meta_mask_bytes(const mcs_shape* s) {
  if (check_shape(s, true) != MCS_OK) return 0;
  return static_cast<size_t>(s->B) * s->H * groups_of(s) * ((static_cast<size_t>(s->N) + 31) / 32) * 4;
}

mcs_status mcs_meta_pack(const mcs_shape* s, const int32_t* kv_idx, uint32_t* mask, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  mcs_status st = check_shape(s, true);
  if (st != MCS_OK) return st;
  if (!kv_idx || !mask || !ws) return MCS_ERR_INVALID_ARG;
  if (ws_bytes < MCS_STATUS_BYTES) return MCS_ERR_INVALID_ARG;
  if (meta_pack_smem_bytes(s->N) > 227 * 1024) return MCS_ERR_UNSUPPORTED;
  if ((st = check_device()) != MCS_OK) return st;
  const long long rows = static_cast<long long>(s->B) * s->H * groups_of(s);
  return cuda_status(launch_meta_pack(kv_idx, mask, rows, s->N, s->topk, static_cast<int*>(ws), stream));
}

mcs_status mcs_meta_unpack(const mcs_shape* s, const uint32_t* mask, int32_t* kv_idx, void* ws, size_t ws_bytes,
                           cudaStream_t stream) {
  mcs_status st = check_shape(s, true);
  if (st != MCS_OK) return st;
  if (!kv_idx || !mask || !ws) return MCS_ERR_INVALID_ARG;
  if (ws_bytes < MCS_STATUS_BYTES) return MCS_ERR_INVALID_ARG;
  if ((st = check_device()) != MCS_OK) return st;
  const long long rows = static_cast<long long>(s->B) * s->H * groups_of(s);
  return cuda_status(launch_meta_unpack(mask, kv_idx, rows, s->N, s->topk, static_cast<int*>(ws), stream));
}

mcs_status mcs_meta_copy(void* dst, const void* src, size_t bytes, int to_host, cudaStream_t side, cudaEvent_t wait,
                         cudaEvent_t done) {
  if (bytes == 0) return MCS_OK;
  if (!dst || !src) return MCS_ERR_INVALID_ARG;
  if (wait && cudaStreamWaitEvent(side, wait, 0) != cudaSuccess) return MCS_ERR_CUDA;
  cudaError_t e = cudaMemcpyAsync(dst, src, bytes, to_host ? cudaMemcpyDeviceToHost : cudaMemcpyHostToDevice, side);
  if (e != cudaSuccess) return MCS_ERR_CUDA;
  if (done && cudaEventRecord(done, side) != cudaSuccess) return MCS_ERR_CUDA;
  return MCS_OK;
}

mcs_status mcs_poll_status(void* ws, int32_t* info, cudaStream_t stream) {
  if (!ws) return MCS_ERR_INVALID_ARG;
  int32_t words[MCS_INFO_WORDS];
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MCS_ERR_CUDA;
  if (cudaMemcpy(words, ws, sizeof(words), cudaMemcpyDeviceToHost) != cudaSuccess) return MCS_ERR_CUDA;
  if (cudaMemset(ws, 0, MCS_STATUS_BYTES) != cudaSuccess) return MCS_ERR_CUDA;
  if (info) memcpy(info, words, sizeof(words));
  return static_cast<mcs_status>(words[MCS_SW_STATUS]);
}

// Test hooks declared in include/mcs_test.h.
void mcs_debug_set_flags(int flags) { g_debug_flags = flags; }
void mcs_debug_set_anchor_chunk_events(void* const* ev, int n) {
  g_chunk_events = reinterpret_cast<cudaEvent_t const*>(ev);
  g_chunk_event_count = ev ? n : 0;
}
long long mcs_debug_launch_count(void) { return g_launches.load(); }

}  // extern "C"
