// Packed selection metadata for offload.
//
// The cached metadata of a layer is the residual R and, per (batch, head,
// query group), the K selected key indices (paper Table 8 counts them as int32
// lists; aiwillknow analysis, step 5, moves them to host memory between
// anchors). At the densities the method runs at, a group's selection is
// smaller as an N-bit mask than as K int32 indices whenever K > N/32. The
// packed form, uint32 words [B, H, G, ceil(N/32)]:
//   bit (j mod 32) of word floor(j / 32) of row (b, h, g) is set exactly when
//   key j is in the group's selection; bits at positions >= N are zero.
// Packing and unpacking are exact inverses for strictly ascending lists, so the
// reuse step reads the same indices whichever form crossed the PCIe link.
//
// meta_pack_kernel: one CTA per row; the row's words are built in shared
// memory with atomic ORs (indices checked for range and strict ascent) and
// written out coalesced.
// meta_unpack_kernel: one CTA per row; eight warps own contiguous word ranges;
// per-warp popcounts and an exclusive scan give each warp's output offset, then
// each lane expands one word at a time into ascending indices. A row whose
// popcount is not K, or with bits at positions >= N, is reported as a bad
// index; no write lands outside the row's K slots.
#include "mcs_ptx.cuh"

namespace mcs {

namespace {
constexpr int kMetaThreads = 256;
constexpr int kMetaWarps = kMetaThreads / 32;
}  // namespace

__global__ void __launch_bounds__(kMetaThreads) meta_pack_kernel(const int32_t* idx, uint32_t* mask, int N, int K,
                                                                 int W, int* status) {
  extern __shared__ uint32_t words[];
  const size_t row = blockIdx.x;
  const int32_t* in = idx + row * static_cast<size_t>(K);
  uint32_t* out = mask + row * static_cast<size_t>(W);
  for (int w = threadIdx.x; w < W; w += kMetaThreads) words[w] = 0u;
  __syncthreads();
  int bad = 0, bad_value = 0;
  for (int t = threadIdx.x; t < K; t += kMetaThreads) {
    const int j = __ldg(in + t);
    const bool ok = j >= 0 && j < N && (t == 0 || __ldg(in + t - 1) < j);
    if (ok) {
      atomicOr(&words[j >> 5], 1u << (j & 31));
    } else if (!bad) {
      bad = 1;
      bad_value = j;
    }
  }
  if (bad) record_status(status, MCS_ERR_BAD_INDEX, bad_value);
  __syncthreads();
  for (int w = threadIdx.x; w < W; w += kMetaThreads) out[w] = words[w];
}

__global__ void __launch_bounds__(kMetaThreads) meta_unpack_kernel(const uint32_t* mask, int32_t* idx, int N, int K,
                                                                   int W, int* status) {
  __shared__ int wout[kMetaWarps];
  const size_t row = blockIdx.x;
  const uint32_t* in = mask + row * static_cast<size_t>(W);
  int32_t* out = idx + row * static_cast<size_t>(K);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpw = (W + kMetaWarps - 1) / kMetaWarps;
  const int w0 = min(W, warp * wpw), w1 = min(W, w0 + wpw);
  // bits at or above N in the last word must be clear
  const uint32_t tail_mask = (N & 31) ? ~((1u << (N & 31)) - 1u) : 0u;
  int cnt = 0;
  for (int w = w0 + lane; w < w1; w += 32) cnt += __popc(__ldg(in + w));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) wout[warp] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int w = 0; w < kMetaWarps; ++w) {
      const int c = wout[w];
      wout[w] = acc;
      acc += c;
    }
    const bool tail_bad = (__ldg(in + W - 1) & tail_mask) != 0u;
    if (acc != K || tail_bad) record_status(status, MCS_ERR_BAD_INDEX, tail_bad ? -2 : -1000000 - acc);
  }
  __syncthreads();
  int off = wout[warp];
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int w = i0 + lane;
    uint32_t bits = w < w1 ? __ldg(in + w) : 0u;
    if (w == W - 1) bits &= ~tail_mask;
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
      bits &= bits - 1u;
      if (pos < K) out[pos] = w * 32 + bit;
      ++pos;
    }
    off += __shfl_sync(0xffffffffu, incl, 31);
  }
}

size_t meta_pack_smem_bytes(int N) { return static_cast<size_t>((N + 31) / 32) * 4; }

cudaError_t launch_meta_pack(const int32_t* idx, uint32_t* mask, long long rows, int N, int K, int* status,
                             cudaStream_t s) {
  const int W = (N + 31) / 32;
  const size_t smem = meta_pack_smem_bytes(N);
  if (rows <= 0 || rows > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(meta_pack_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  meta_pack_kernel<<<static_cast<unsigned>(rows), kMetaThreads, smem, s>>>(idx, mask, N, K, W, status);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_meta_unpack(const uint32_t* mask, int32_t* idx, long long rows, int N, int K, int* status,
                               cudaStream_t s) {
  const int W = (N + 31) / 32;
  if (rows <= 0 || rows > 0x7fffffffLL) return cudaErrorInvalidValue;
  meta_unpack_kernel<<<static_cast<unsigned>(rows), kMetaThreads, 0, s>>>(mask, idx, N, K, W, status);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace mcs
