// Token-to-expert permutation: an exact, deterministic counting sort of the T*k
// (token, slot) pairs by expert, stable by the flat pair index p = t*k + j.
//
// This is the gathered dispatch that the Tenstorrent card calls "per-token gathered
// expert prefill" (tokens grouped per expert instead of running every expert on every
// token), computed exactly:
//   histogram -> exclusive scan (expert_offsets) -> stable scatter (sorted_src, inv_pos).
// Up to kPermSmallMax pairs one block does everything; beyond that, per-block
// histograms, one scan block, and a per-block stable scatter over at most
// kPermMaxBlocks blocks of a multiple of kPermThreads pairs each.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "permute_impl.cuh"

namespace moe {

constexpr int kPermThreads = 1024;
constexpr int kPermSmallMax = 2048;  // pairs handled by the single-block path
constexpr int kPermMaxBlocks = 256;  // blocks of the multi-block path at most

// Pairs per block of the multi-block path: one pass of the block's threads when that
// keeps the grid within kPermMaxBlocks, else the smallest multiple that does.
int pairs_per_block(int n) {
  const int64_t per = (static_cast<int64_t>(n) + kPermMaxBlocks - 1) / kPermMaxBlocks;
  return static_cast<int>(std::max<int64_t>(1, (per + kPermThreads - 1) / kPermThreads) *
                          kPermThreads);
}

__global__ void __launch_bounds__(kPermThreads) permute_small_kernel(
    int n, int E, const int* __restrict__ idx, int* __restrict__ offsets,
    int* __restrict__ sorted_src, int* __restrict__ inv_pos) {
  __shared__ PermuteSmem<kPermThreads> s;
  pdl_wait();
  pdl_trigger();
  permute_block<kPermThreads>(n, E, idx, offsets, sorted_src, inv_pos, s);
}

// Multi-block pass 1: per-block histograms block_hist[b][e].
__global__ void __launch_bounds__(kPermThreads) permute_hist_kernel(int n, int E, int ppb,
                                                                    const int* __restrict__ idx,
                                                                    int* __restrict__ block_hist) {
  __shared__ int cnt[kPermMaxE];
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  for (int e = tid; e < E; e += kPermThreads) cnt[e] = 0;
  __syncthreads();
  const int p0 = blockIdx.x * ppb;
  const int p1 = min(n, p0 + ppb);
  for (int p = p0 + tid; p < p1; p += kPermThreads) {
    const int e = idx[p];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int e = tid; e < E; e += kPermThreads) block_hist[blockIdx.x * E + e] = cnt[e];
}

// Multi-block pass 2 (one block): offsets and each block's first position per expert.
__global__ void __launch_bounds__(kPermMaxE) permute_scan_kernel(int nb, int E,
                                                                 const int* __restrict__ block_hist,
                                                                 int* __restrict__ block_base,
                                                                 int* __restrict__ offsets) {
  __shared__ int tot[kPermMaxE];
  __shared__ int off[kPermMaxE + 1];
  const int e = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (e < E) {
    int s = 0;
    for (int b = 0; b < nb; ++b) s += block_hist[b * E + e];
    tot[e] = s;
  }
  __syncthreads();
  if (threadIdx.x < 32) warp_exclusive_scan(tot, off, E);
  __syncthreads();
  if (e < E) {
    int run = off[e];
    offsets[e] = run;
    for (int b = 0; b < nb; ++b) {
      block_base[b * E + e] = run;
      run += block_hist[b * E + e];
    }
  }
  if (e == 0) offsets[E] = off[E];
}

// Multi-block pass 3: stable scatter of each block's pairs.
__global__ void __launch_bounds__(kPermThreads) permute_scatter_kernel(
    int n, int E, int ppb, const int* __restrict__ idx, const int* __restrict__ block_base,
    int* __restrict__ sorted_src, int* __restrict__ inv_pos) {
  __shared__ int base[kPermMaxE];
  __shared__ int wcnt[kPermThreads / 32][kPermMaxE];
  pdl_wait();
  pdl_trigger();
  for (int e = threadIdx.x; e < E; e += kPermThreads) base[e] = block_base[blockIdx.x * E + e];
  __syncthreads();
  const int p0 = blockIdx.x * ppb;
  scatter_range<kPermThreads>(p0, min(n, p0 + ppb), E, idx, base, wcnt, sorted_src, inv_pos);
}

int permute_blocks(int n) {
  if (n <= kPermSmallMax) return 0;
  const int ppb = pairs_per_block(n);
  return (n + ppb - 1) / ppb;
}

cudaError_t launch_permute(int n, int E, const int* topk_idx, int* offsets, int* sorted_src,
                           int* inv_pos, int* block_hist, int* block_base, cudaStream_t s,
                           bool pdl) {
  const int nb = permute_blocks(n);
  if (nb == 0)
    return launch_k(permute_small_kernel, dim3(1), dim3(kPermThreads), 0, s, pdl, n, E, topk_idx,
                    offsets, sorted_src, inv_pos);
  const int ppb = pairs_per_block(n);
  cudaError_t e = launch_k(permute_hist_kernel, dim3(nb), dim3(kPermThreads), 0, s, pdl, n, E,
                           ppb, topk_idx, block_hist);
  if (e != cudaSuccess) return e;
  e = launch_k(permute_scan_kernel, dim3(1), dim3(kPermMaxE), 0, s, true, nb, E,
               (const int*)block_hist, block_base, offsets);
  if (e != cudaSuccess) return e;
  return launch_k(permute_scatter_kernel, dim3(nb), dim3(kPermThreads), 0, s, true, n, E, ppb,
                  topk_idx, (const int*)block_base, sorted_src, inv_pos);
}

// dst[q] = src[sorted_src[q] / k] for the n sorted pairs; one thread per 16 bytes.
// A pair index outside [0, T*k) yields a zero row (never an out-of-bounds read).
__global__ void __launch_bounds__(256) gather_rows_kernel(int n, int k, int H, int T,
                                                          const int* __restrict__ sorted_src,
                                                          const uint16_t* __restrict__ src,
                                                          uint16_t* __restrict__ dst) {
  const int nch = H >> 3;
  pdl_wait();
  pdl_trigger();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (i >= static_cast<int64_t>(n) * nch) return;
  const int q = static_cast<int>(i / nch), c = static_cast<int>(i % nch);
  const int p = sorted_src[q];
  const int t = (p >= 0 && p < n) ? p / k : -1;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (t >= 0 && t < T) v = __ldg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(t) * H) + c);
  reinterpret_cast<uint4*>(dst + static_cast<size_t>(q) * H)[c] = v;
}

cudaError_t launch_gather_rows(int n, int k, int H, int T, const int* sorted_src,
                               const uint16_t* src, uint16_t* dst, cudaStream_t s, bool pdl) {
  const int64_t total = static_cast<int64_t>(n) * (H >> 3);
  return launch_k(gather_rows_kernel, dim3(static_cast<unsigned>((total + 255) / 256)), dim3(256),
                  0, s, pdl, n, k, H, T, sorted_src, src, dst);
}

}  // namespace moe
