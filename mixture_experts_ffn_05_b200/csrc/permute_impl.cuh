// Block-level stable counting sort of (token, slot) pairs by expert, shared by the
// permutation kernels and the fused router.  NT threads (a multiple of 32, <= 1024).
//
// Ranks inside a warp come from __match_any_sync + popc, ranks across warps from
// per-warp counts summed in warp order, so no result depends on the order in which
// atomics land.  Ids outside [0, E) are dropped.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kPermMaxE = 256;

// bf16 -> fp16 of 8 values (exact for |v| in the fp16 normal range; smaller values keep
// fp16 subnormal precision, 2^-24 absolute).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4& u) {
  float f[8];
  unpack8(u, f);
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 h = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
    o[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int NT>
struct PermuteSmem {
  int cnt[kPermMaxE];
  int off[kPermMaxE + 1];
  int wcnt[NT / 32][kPermMaxE];
};

// Exclusive scan of cnt[0..E) into out[0..E] by one warp; out[E] = total.
__device__ __forceinline__ void warp_exclusive_scan(const int* cnt, int* out, int E) {
  const int lane = threadIdx.x & 31;
  int carry = 0;
  for (int b = 0; b < E; b += 32) {
    const int e = b + lane;
    const int v = (e < E) ? cnt[e] : 0;
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

// Stable scatter of the pairs [p0, p1): base[e] holds the first output position of
// this range's pairs of expert e and is advanced as the range is consumed.
template <int NT>
__device__ void scatter_range(int p0, int p1, int E, const int* idx, int* base,
                              int (*wcnt)[kPermMaxE], int* __restrict__ sorted_src,
                              int* __restrict__ inv_pos) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int c0 = p0; c0 < p1; c0 += NT) {
    const int p = c0 + tid;
    int e = -1;
    if (p < p1) {
      e = __ldcg(idx + p);
      if (e < 0 || e >= E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    for (int i = tid; i < NW * kPermMaxE; i += NT) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    if (e >= 0 && rank == 0) wcnt[warp][e] = __popc(peers);
    __syncthreads();
    for (int ee = tid; ee < E; ee += NT) {
      int run = base[ee];
      for (int w = 0; w < NW; ++w) {
        const int c = wcnt[w][ee];
        wcnt[w][ee] = run;
        run += c;
      }
      base[ee] = run;
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

// The whole sort of n pairs by one block: histogram, scan, stable scatter.
template <int NT>
__device__ void permute_block(int n, int E, const int* idx, int* __restrict__ offsets,
                              int* __restrict__ sorted_src, int* __restrict__ inv_pos,
                              PermuteSmem<NT>& s) {
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += NT) s.cnt[e] = 0;
  __syncthreads();
  for (int p = tid; p < n; p += NT) {
    const int e = __ldcg(idx + p);
    if (e >= 0 && e < E) atomicAdd(&s.cnt[e], 1);
  }
  __syncthreads();
  if (tid < 32) warp_exclusive_scan(s.cnt, s.off, E);
  __syncthreads();
  for (int e = tid; e <= E; e += NT) offsets[e] = s.off[e];
  for (int e = tid; e < E; e += NT) s.cnt[e] = s.off[e];  // cnt becomes the running base
  __syncthreads();
  scatter_range<NT>(0, n, E, idx, s.cnt, s.wcnt, sorted_src, inv_pos);
}

}  // namespace moe
