// Combine of the expert outputs, the post norms and the residual.
//
// ONNX export card, "Truthful graph contracts", "MoE topology" row: the block returns
// post_ff_norm(dense + moe) + residual; the Inferentia2 card's "four feed-forward
// layernorms" add a post norm on each branch:
//   m   = sum_{j=0..k-1} w[t,j] * Y[inv_pos[t*k + j]]        (fixed slot order)
//   out = x + N_post_ff( N_post_dense(d) + N_post_moe(m) ),  N_g(v) = v / rms(v) * g
// Y (the expert outputs in sorted order, unweighted) arrives in fp16 and d in fp32; all
// sums are fp32 and the output is rounded to bf16 once.  A slot whose inv_pos does not point back
// at it through sorted_src (a pair the permutation dropped) contributes nothing.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kCombMaxThreads = 768;  // H <= 6144: one 8-column chunk per thread
constexpr int kCombManyTokens = 256;  // from here on, occupancy over slots in flight

// Sums of two values over the block in a fixed order (deterministic).
__device__ __forceinline__ float2 block_sum2(float a, float b, float2* red) {
  a = warp_sum(a);
  b = warp_sum(b);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red may still be read by a previous call
  if (lane == 0) red[warp] = make_float2(a, b);
  __syncthreads();
  float2 s = make_float2(0.f, 0.f);
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
    s.x += red[w].x;
    s.y += red[w].y;
  }
  return s;
}

// 8 fp32 values from two 16-byte loads.
__device__ __forceinline__ void load8f(const float* p, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// Row of Y and routing weight of each slot of token t, in shared memory (row -1: none).
__device__ __forceinline__ void load_slots(int t, int k, int n, const int* __restrict__ inv_pos,
                                           const int* __restrict__ sorted_src,
                                           const float* __restrict__ topk_w, int* s_q,
                                           float* s_w) {
  if (threadIdx.x < k) {
    const int p = t * k + threadIdx.x;
    const int q = inv_pos[p];
    // sorted_src == NULL: the permutation comes from this library's own sort (no check)
    const bool ok = q >= 0 && q < n && (sorted_src == nullptr || sorted_src[q] == p);
    s_q[threadIdx.x] = ok ? q : -1;
    s_w[threadIdx.x] = topk_w[p];
  }
  __syncthreads();
}

// One CTA per token, one 8-column chunk per thread; every input is requested before
// the first reduction.  NSLOT slots of Y (16 bytes of fp16 each per thread) are in
// flight at a time.  The kernel is latency-bound (two dependent round trips, inv_pos
// then Y, and two block reductions per token), so MINB resident CTAs per SM matter more
// than slots in flight: up to H = 3072, 4 slots and 4 CTAs of 352-384 threads (at most
// 40 registers) measured 22% faster than 8 slots and 2 CTAs at T = 16384.
template <int MAXT, int NSLOT, int MINB>
__global__ void __launch_bounds__(MAXT, MINB) combine_block_kernel(
    int H, int k, float eps, const uint16_t* __restrict__ x, const uint16_t* __restrict__ y,
    const int* __restrict__ inv_pos, const int* __restrict__ sorted_src,
    const float* __restrict__ topk_w, const float* __restrict__ dense,
    const uint16_t* __restrict__ g_pm,
    const uint16_t* __restrict__ g_pd, const uint16_t* __restrict__ g_ff,
    uint16_t* __restrict__ out, uint16_t* __restrict__ moe_out) {
  __shared__ float2 red[MAXT / 32];
  __shared__ int s_q[16];
  __shared__ float s_w[16];
  const int t = blockIdx.x;
  const int c = threadIdx.x;
  const bool on = c < (H >> 3);
  const int cc = on ? c : 0;
  // Read before the dependency wait: the residual, and the slot table.  inv_pos and
  // topk_w come from the routing kernels, which completed before the kernel this one
  // follows could start (the gather and GEMM launches wait for them); only Y and the dense
  // output are the previous kernel's results.  (The gains, read late, are cache-resident.)
  const uint4 vx = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H) + cc);
  load_slots(t, k, gridDim.x * k, inv_pos, sorted_src, topk_w, s_q, s_w);
  pdl_wait();
  pdl_trigger();
  float m[8], d[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = d[i] = 0.f;
  {
    load8f(dense + static_cast<size_t>(t) * H + cc * 8, d);
    for (int j0 = 0; j0 < k; j0 += NSLOT) {  // NSLOT slots in flight, summed in slot order
      uint4 raw[NSLOT];
#pragma unroll
      for (int j = 0; j < NSLOT; ++j)
        raw[j] = (j0 + j < k && s_q[j0 + j] >= 0)
                     ? __ldg(reinterpret_cast<const uint4*>(y + static_cast<size_t>(s_q[j0 + j]) * H) + cc)
                     : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int j = 0; j < NSLOT; ++j)
        if (j0 + j < k && s_q[j0 + j] >= 0) {
          const float w = s_w[j0 + j];
          float f[8];
          unpack8_f16(raw[j], f);
#pragma unroll
          for (int i = 0; i < 8; ++i) m[i] = fmaf(w, f[i], m[i]);
        }
    }
    if (!on) {
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] = d[i] = 0.f;
    }
    if (on && moe_out) reinterpret_cast<uint4*>(moe_out + static_cast<size_t>(t) * H)[c] = pack8(m);
  }
  float ssm = 0.f, ssd = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    ssm = fmaf(m[i], m[i], ssm);
    ssd = fmaf(d[i], d[i], ssd);
  }
  const float2 ss = block_sum2(ssm, ssd, red);
  const float rm = g_pm ? 1.0f / sqrtf(ss.x / H + eps) : 1.f;
  const float rd = g_pd ? 1.0f / sqrtf(ss.y / H + eps) : 1.f;
  float sum[8], ga[8], gb[8];
  unpack8(g_pd ? __ldg(reinterpret_cast<const uint4*>(g_pd) + cc) : make_uint4(0u, 0u, 0u, 0u), ga);
  unpack8(g_pm ? __ldg(reinterpret_cast<const uint4*>(g_pm) + cc) : make_uint4(0u, 0u, 0u, 0u), gb);
  float ssc = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float av = g_pd ? d[i] * rd * ga[i] : d[i];
    const float bv = g_pm ? m[i] * rm * gb[i] : m[i];
    sum[i] = av + bv;
    ssc = fmaf(sum[i], sum[i], ssc);
  }
  const float rc = 1.0f / sqrtf(block_sum2(ssc, 0.f, red).x / H + eps);
  if (on) {
    float xf[8], g[8], o[8];
    unpack8(vx, xf);
    unpack8(__ldg(reinterpret_cast<const uint4*>(g_ff) + cc), g);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = xf[i] + sum[i] * rc * g[i];
    reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H)[c] = pack8(o);
  }
}

// moe_out[t] = sum_j w[t,j] * Y[inv_pos[t*k + j]] in fp32, slot order, rounded to bf16.
__global__ void __launch_bounds__(256) combine_moe_kernel(int H, int k,
                                                          const uint16_t* __restrict__ y,
                                                          const int* __restrict__ inv_pos,
                                                          const int* __restrict__ sorted_src,
                                                          const float* __restrict__ topk_w,
                                                          uint16_t* __restrict__ moe_out) {
  __shared__ int s_q[16];
  __shared__ float s_w[16];
  const int t = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  load_slots(t, k, gridDim.x * k, inv_pos, sorted_src, topk_w, s_q, s_w);
  for (int c = threadIdx.x; c < (H >> 3); c += 256) {
    float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      if (s_q[j] < 0) continue;
      float f[8];
      unpack8_f16(__ldg(reinterpret_cast<const uint4*>(y + static_cast<size_t>(s_q[j]) * H) + c), f);
      const float w = s_w[j];
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] = fmaf(w, f[i], m[i]);
    }
    reinterpret_cast<uint4*>(moe_out + static_cast<size_t>(t) * H)[c] = pack8(m);
  }
}

cudaError_t launch_combine_block(int T, int H, int k, float eps, const uint16_t* x,
                                 const uint16_t* y, const int* inv_pos, const int* sorted_src,
                                 const float* topk_w, const float* dense,
                                 const uint16_t* g_post_moe, const uint16_t* g_post_dense,
                                 const uint16_t* g_post_ff, uint16_t* out, uint16_t* moe_out,
                                 cudaStream_t s, bool pdl) {
  const int threads = std::max(32, ((H >> 3) + 31) / 32 * 32);
  // Many tokens: resident CTAs hide the latency (4 slots in flight, 4 CTAs per SM).  Few
  // tokens (up to about two CTAs per SM): every slot in flight at once (k <= 16), so that
  // a token's Y rows cost one round trip.
  if (threads <= 384 && T >= kCombManyTokens)
    return launch_k(combine_block_kernel<384, 4, 4>, dim3(T), dim3(threads), 0, s, pdl, H, k, eps,
                    x, y, inv_pos, sorted_src, topk_w, dense, g_post_moe, g_post_dense,
                    g_post_ff, out, moe_out);
  if (threads <= 384)
    return launch_k(combine_block_kernel<384, 16, 1>, dim3(T), dim3(threads), 0, s, pdl, H, k,
                    eps, x, y, inv_pos, sorted_src, topk_w, dense, g_post_moe, g_post_dense,
                    g_post_ff, out, moe_out);
  return launch_k(combine_block_kernel<kCombMaxThreads, 8, 1>, dim3(T), dim3(threads), 0, s, pdl,
                  H, k, eps, x, y, inv_pos, sorted_src, topk_w, dense, g_post_moe,
                  g_post_dense, g_post_ff, out, moe_out);
}

cudaError_t launch_combine_moe(int T, int H, int k, const uint16_t* y, const int* inv_pos,
                               const int* sorted_src, const float* topk_w, uint16_t* moe_out,
                               cudaStream_t s, bool pdl) {
  return launch_k(combine_moe_kernel, dim3(T), dim3(256), 0, s, pdl, H, k, y, inv_pos,
                  sorted_src, topk_w, moe_out);
}

}  // namespace moe
