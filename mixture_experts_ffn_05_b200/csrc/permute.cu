// Token-to-expert permutation: an exact, deterministic counting sort of the T*k
// (token, slot) pairs by expert, stable by the flat pair index p = t*k + j.
//
// This is the gathered dispatch that the Tenstorrent card calls "per-token gathered
// expert prefill" (tokens grouped per expert instead of running every expert on every
// token), computed exactly:
//   histogram -> exclusive scan (expert_offsets) -> stable scatter (sorted_src, inv_pos).
// Ranks inside a warp come from __match_any_sync + popc, ranks across warps and blocks
// from per-warp and per-block counts summed in index order, so no result depends on
// the order in which atomics land.
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kPermThreads = 1024;
constexpr int kPermMaxE = 256;
constexpr int kPermPerBlock = 4096;   // pairs per block of the multi-block path
constexpr int kPermSmallMax = 8192;   // pairs handled by the single-block path

// Stable scatter of the pairs [p0, p1) given base[e] = first output position of this
// range's pairs of expert e (advanced as it goes).  Runs on all 1024 threads.
__device__ void scatter_range(int p0, int p1, int E, const int* __restrict__ idx,
                              int* __restrict__ base, int (*wcnt)[kPermMaxE],
                              int* __restrict__ sorted_src, int* __restrict__ inv_pos) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int c0 = p0; c0 < p1; c0 += kPermThreads) {
    const int p = c0 + tid;
    int e = -1;
    if (p < p1) {
      e = idx[p];
      if (e < 0 || e >= E) e = -1;  // invalid ids are dropped
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    for (int i = tid; i < 32 * kPermMaxE; i += kPermThreads) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    if (e >= 0 && rank == 0) wcnt[warp][e] = __popc(peers);
    __syncthreads();
    if (tid < E) {
      int run = base[tid];
      for (int w = 0; w < 32; ++w) {
        const int c = wcnt[w][tid];
        wcnt[w][tid] = run;
        run += c;
      }
      base[tid] = run;
    }
    __syncthreads();
    if (e >= 0) {
      const int pos = wcnt[warp][e] + rank;
      sorted_src[pos] = p;
      inv_pos[p] = pos;
    }
    __syncthreads();
  }
}

// Exclusive scan of cnt[0..E) into out[0..E], by one warp.  out[E] = total.
__device__ void warp_exclusive_scan(const int* cnt, int* out, int E) {
  const int lane = threadIdx.x & 31;
  int carry = 0;
  for (int b = 0; b < E; b += 32) {
    const int e = b + lane;
    int v = (e < E) ? cnt[e] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (e < E) out[e] = carry + incl - v;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) out[E] = carry;
}

// Single block: n <= kPermSmallMax pairs.
__global__ void __launch_bounds__(kPermThreads) permute_small_kernel(
    int n, int E, const int* __restrict__ idx, int* __restrict__ offsets,
    int* __restrict__ sorted_src, int* __restrict__ inv_pos) {
  __shared__ int cnt[kPermMaxE];
  __shared__ int off[kPermMaxE + 1];
  __shared__ int wcnt[32][kPermMaxE];
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += kPermThreads) cnt[e] = 0;
  __syncthreads();
  for (int p = tid; p < n; p += kPermThreads) {
    const int e = idx[p];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  if (tid < 32) warp_exclusive_scan(cnt, off, E);
  __syncthreads();
  for (int e = tid; e <= E; e += kPermThreads) offsets[e] = off[e];
  if (tid < E) cnt[tid] = off[tid];  // cnt becomes the running base
  __syncthreads();
  scatter_range(0, n, E, idx, cnt, wcnt, sorted_src, inv_pos);
}

// Multi-block pass 1: per-block histograms block_hist[b][e].
__global__ void __launch_bounds__(kPermThreads) permute_hist_kernel(int n, int E,
                                                                    const int* __restrict__ idx,
                                                                    int* __restrict__ block_hist) {
  __shared__ int cnt[kPermMaxE];
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += kPermThreads) cnt[e] = 0;
  __syncthreads();
  const int p0 = blockIdx.x * kPermPerBlock;
  const int p1 = min(n, p0 + kPermPerBlock);
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
    int n, int E, const int* __restrict__ idx, const int* __restrict__ block_base,
    int* __restrict__ sorted_src, int* __restrict__ inv_pos) {
  __shared__ int base[kPermMaxE];
  __shared__ int wcnt[32][kPermMaxE];
  for (int e = threadIdx.x; e < E; e += kPermThreads) base[e] = block_base[blockIdx.x * E + e];
  __syncthreads();
  const int p0 = blockIdx.x * kPermPerBlock;
  scatter_range(p0, min(n, p0 + kPermPerBlock), E, idx, base, wcnt, sorted_src, inv_pos);
}

int permute_blocks(int n) {
  return n <= kPermSmallMax ? 0 : (n + kPermPerBlock - 1) / kPermPerBlock;
}

cudaError_t launch_permute(int n, int E, const int* topk_idx, int* offsets, int* sorted_src,
                           int* inv_pos, int* block_hist, int* block_base, cudaStream_t s) {
  const int nb = permute_blocks(n);
  if (nb == 0) {
    permute_small_kernel<<<1, kPermThreads, 0, s>>>(n, E, topk_idx, offsets, sorted_src, inv_pos);
    return cudaGetLastError();
  }
  permute_hist_kernel<<<nb, kPermThreads, 0, s>>>(n, E, topk_idx, block_hist);
  permute_scan_kernel<<<1, kPermMaxE, 0, s>>>(nb, E, block_hist, block_base, offsets);
  permute_scatter_kernel<<<nb, kPermThreads, 0, s>>>(n, E, topk_idx, block_base, sorted_src,
                                                     inv_pos);
  return cudaGetLastError();
}

// dst[q] = src[sorted_src[q] / k] for the n sorted pairs: one warp per row of H bf16.
// A pair index outside [0, T*k) yields a zero row (never an out-of-bounds read).
__global__ void __launch_bounds__(256) gather_rows_kernel(int n, int k, int H, int T,
                                                          const int* __restrict__ sorted_src,
                                                          const uint16_t* __restrict__ src,
                                                          uint16_t* __restrict__ dst) {
  const int q = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (q >= n) return;
  const int lane = threadIdx.x & 31;
  const int p = sorted_src[q];
  const int t = (p >= 0 && p < n) ? p / k : -1;
  uint4* d = reinterpret_cast<uint4*>(dst + static_cast<size_t>(q) * H);
  if (t < 0 || t >= T) {
    for (int c = lane; c < (H >> 3); c += 32) d[c] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const uint4* s = reinterpret_cast<const uint4*>(src + static_cast<size_t>(t) * H);
  for (int c = lane; c < (H >> 3); c += 32) d[c] = __ldg(s + c);
}

cudaError_t launch_gather_rows(int n, int k, int H, int T, const int* sorted_src,
                               const uint16_t* src, uint16_t* dst, cudaStream_t s) {
  gather_rows_kernel<<<(n + 7) / 8, 256, 0, s>>>(n, k, H, T, sorted_src, src, dst);
  return cudaGetLastError();
}

}  // namespace moe
