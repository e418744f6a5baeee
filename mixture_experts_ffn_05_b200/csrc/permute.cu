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

// dst[q] = src[sorted_src[q] / k] for the n sorted pairs.  One warp per row: each lane
// requests up to 8 of the row's 16-byte chunks before storing any, so a warp keeps
// 4 KB of loads in flight.  A pair index outside [0, T*k) yields a zero row (never an
// out-of-bounds read).
constexpr int kGatherWarps = 8;
// From this many pairs on, the rows are written token by token (each source row read
// once); below, pair by pair (more warps for a small batch).
constexpr int kScatterMinPairs = 4096;

template <bool F16>
__global__ void __launch_bounds__(32 * kGatherWarps) gather_rows_kernel(
    int n, int k, int H, int T, const int* __restrict__ sorted_src,
    const uint16_t* __restrict__ src, uint16_t* __restrict__ dst) {
  const int nch = H >> 3;
  pdl_wait();
  pdl_trigger();
  const int q = static_cast<int>(blockIdx.x) * kGatherWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (q >= n) return;
  const int p = sorted_src[q];
  const int t = (p >= 0 && p < n) ? p / k : -1;
  const uint4* s = (t >= 0 && t < T) ? reinterpret_cast<const uint4*>(src + static_cast<size_t>(t) * H)
                                     : nullptr;
  uint4* d = reinterpret_cast<uint4*>(dst + static_cast<size_t>(q) * H);
  for (int c0 = lane; c0 < nch; c0 += 32 * 8) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = c0 + 32 * u;
      v[u] = (s != nullptr && c < nch) ? __ldg(s + c) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = c0 + 32 * u;
      if (c < nch) d[c] = F16 ? bf16x8_to_f16x8(v[u]) : v[u];
    }
  }
}

// The same rows written token by token: warp t reads row t of src once and writes it to the
// sorted position of each of its k pairs (pos = inv_pos[t k + j], taken only where
// sorted_src[pos] names the pair back, so that dropped pairs write nothing).  For large
// batches: each source row is read once instead of k times, from HBM once it no longer
// sits in L2.  Every row the matmuls read (the positions below the pair count) is written.
template <bool F16>
__global__ void __launch_bounds__(32 * kGatherWarps) scatter_rows_kernel(
    int T, int k, int H, int n, const int* __restrict__ inv_pos,
    const int* __restrict__ sorted_src, const uint16_t* __restrict__ src,
    uint16_t* __restrict__ dst) {
  const int nch = H >> 3;
  pdl_wait();
  pdl_trigger();
  const int t = static_cast<int>(blockIdx.x) * kGatherWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  // lane j < k: the destination of pair (t, j), or -1
  int pos = -1;
  if (lane < k) {
    const int p = t * k + lane;
    const int q = __ldg(inv_pos + p);
    if (q >= 0 && q < n && __ldg(sorted_src + q) == p) pos = q;
  }
  const uint4* srow = reinterpret_cast<const uint4*>(src + static_cast<size_t>(t) * H);
  for (int c0 = lane; c0 < nch; c0 += 32 * 8) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = c0 + 32 * u;
      v[u] = c < nch ? __ldg(srow + c) : make_uint4(0u, 0u, 0u, 0u);
      if (F16) v[u] = bf16x8_to_f16x8(v[u]);
    }
    for (int j = 0; j < k; ++j) {
      const int q = __shfl_sync(0xffffffffu, pos, j);
      if (q < 0) continue;
      uint4* d = reinterpret_cast<uint4*>(dst + static_cast<size_t>(q) * H);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + 32 * u;
        if (c < nch) d[c] = v[u];
      }
    }
  }
}

// The fp8 variant's activations (dynamic per-token E4M3 quantisation, the "Gemma 4 26B-A4B
// IT" recipe page, "Quantized Variants"): row q of the matmul operand is source row r(q)
// quantised with its own scale s = max|row| / 448 (fp32; 1 for an all-zero row), codes
// E4M3(v / s) rounded to nearest even, saturating.  One warp per row, two passes over the
// row (the second from cache).  r(q) = sorted_src[q] / k (the gather of the routed rows),
// or q with sorted_src NULL (h, already in sorted order).
__global__ void __launch_bounds__(32 * kGatherWarps) gather_quant_fp8_kernel(
    int n, int k, int cols, int T, const int* __restrict__ sorted_src,
    const uint16_t* __restrict__ src, uint8_t* __restrict__ dst, float* __restrict__ scales) {
  const int nch = cols >> 3;
  pdl_wait();
  pdl_trigger();
  const int q = static_cast<int>(blockIdx.x) * kGatherWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (q >= n) return;
  int t = q;
  if (sorted_src != nullptr) {
    const int p = sorted_src[q];
    t = (p >= 0 && p < n) ? p / k : -1;
  }
  const bool ok = t >= 0 && t < T;
  const uint4* s = reinterpret_cast<const uint4*>(src + static_cast<size_t>(ok ? t : 0) * cols);
  float amax = 0.f;
  if (ok) {
    for (int c0 = lane; c0 < nch; c0 += 32 * 4) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u;
        v[u] = c < nch ? __ldg(s + c) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float f[8];
        unpack8(v[u], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
      }
    }
  }
  amax = warp_max(amax);
  const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  if (lane == 0) scales[q] = sc;
  uint2* d = reinterpret_cast<uint2*>(dst + static_cast<size_t>(q) * cols);
  for (int c = lane; c < nch; c += 32) {
    uint32_t packed[2] = {0u, 0u};
    if (ok) {
      float f[8];
      unpack8(__ldg(s + c), f);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        packed[i >> 2] |= static_cast<uint32_t>(e4m3_bits_sat(__fdiv_rn(f[i], sc))) << (8 * (i & 3));
    }
    d[c] = make_uint2(packed[0], packed[1]);
  }
}

cudaError_t launch_gather_quant_fp8(int n, int k, int cols, int T, const int* sorted_src,
                                    const uint16_t* src, uint8_t* dst, float* scales,
                                    cudaStream_t s, bool pdl) {
  const int blocks = (n + kGatherWarps - 1) / kGatherWarps;
  return launch_k(gather_quant_fp8_kernel, dim3(static_cast<unsigned>(blocks)),
                  dim3(32 * kGatherWarps), 0, s, pdl, n, k, cols, T, sorted_src, src, dst, scales);
}

cudaError_t launch_gather_rows(int n, int k, int H, int T, const int* sorted_src,
                               const int* inv_pos, const uint16_t* src, uint16_t* dst,
                               bool to_f16, cudaStream_t s, bool pdl) {
  if (inv_pos != nullptr && n >= kScatterMinPairs && k <= 32) {
    const int tb = (T + kGatherWarps - 1) / kGatherWarps;
    return to_f16 ? launch_k(scatter_rows_kernel<true>, dim3(static_cast<unsigned>(tb)),
                             dim3(32 * kGatherWarps), 0, s, pdl, T, k, H, n, inv_pos, sorted_src,
                             src, dst)
                  : launch_k(scatter_rows_kernel<false>, dim3(static_cast<unsigned>(tb)),
                             dim3(32 * kGatherWarps), 0, s, pdl, T, k, H, n, inv_pos, sorted_src,
                             src, dst);
  }
  const int blocks = (n + kGatherWarps - 1) / kGatherWarps;
  return to_f16 ? launch_k(gather_rows_kernel<true>, dim3(static_cast<unsigned>(blocks)),
                           dim3(32 * kGatherWarps), 0, s, pdl, n, k, H, T, sorted_src, src, dst)
                : launch_k(gather_rows_kernel<false>, dim3(static_cast<unsigned>(blocks)),
                           dim3(32 * kGatherWarps), 0, s, pdl, n, k, H, T, sorted_src, src, dst);
}

}  // namespace moe
