// Combine of the expert outputs, the post norms and the residual.
//
// ONNX export card, "Truthful graph contracts", "MoE topology" row: the block returns
// post_ff_norm(dense + moe) + residual; the Inferentia2 card's "four feed-forward
// layernorms" add a post norm on each branch:
//   m   = sum_{j=0..k-1} Y[t*k + j]          (weights already applied, fixed slot order)
//   out = x + N_post_ff( N_post_dense(d) + N_post_moe(m) ),  N_g(v) = v / rms(v) * g
// All sums in fp32; the output is rounded to bf16 once.  One CTA of 128 threads per
// token; each thread owns chunks of 8 columns.
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kCombThreads = 128;
constexpr int kCombMaxChunks = 6;  // H <= 6144: 768 chunks of 8 over 128 threads

__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red may still be read by a previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < kCombThreads / 32; ++w) s += red[w];  // fixed order
  return s;
}

__global__ void __launch_bounds__(kCombThreads) combine_block_kernel(
    int H, int k, float eps, const uint16_t* __restrict__ x, const uint16_t* __restrict__ y,
    const uint16_t* __restrict__ dense, const uint16_t* __restrict__ g_pm,
    const uint16_t* __restrict__ g_pd, const uint16_t* __restrict__ g_ff,
    uint16_t* __restrict__ out, uint16_t* __restrict__ moe_out) {
  __shared__ float red[kCombThreads / 32];
  const int t = blockIdx.x;
  const int nch = H >> 3;
  float m[kCombMaxChunks][8], d[kCombMaxChunks][8];
  float ssm = 0.f, ssd = 0.f;
#pragma unroll
  for (int u = 0; u < kCombMaxChunks; ++u) {
    const int c = threadIdx.x + u * kCombThreads;
    if (c < nch) {
#pragma unroll
      for (int i = 0; i < 8; ++i) m[u][i] = 0.f;
      for (int j = 0; j < k; ++j) {
        float f[8];
        unpack8(__ldg(reinterpret_cast<const uint4*>(y + (static_cast<size_t>(t) * k + j) * H) + c), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) m[u][i] += f[i];
      }
      unpack8(__ldg(reinterpret_cast<const uint4*>(dense + static_cast<size_t>(t) * H) + c), d[u]);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        ssm = fmaf(m[u][i], m[u][i], ssm);
        ssd = fmaf(d[u][i], d[u][i], ssd);
      }
      if (moe_out) reinterpret_cast<uint4*>(moe_out + static_cast<size_t>(t) * H)[c] = pack8(m[u]);
    }
  }
  const float rm = g_pm ? 1.0f / sqrtf(block_sum(ssm, red) / H + eps) : 1.f;
  const float rd = g_pd ? 1.0f / sqrtf(block_sum(ssd, red) / H + eps) : 1.f;
  float ssc = 0.f;
#pragma unroll
  for (int u = 0; u < kCombMaxChunks; ++u) {
    const int c = threadIdx.x + u * kCombThreads;
    if (c < nch) {
      float ga[8], gb[8];
      if (g_pd) unpack8(__ldg(reinterpret_cast<const uint4*>(g_pd) + c), ga);
      if (g_pm) unpack8(__ldg(reinterpret_cast<const uint4*>(g_pm) + c), gb);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float a = g_pd ? d[u][i] * rd * ga[i] : d[u][i];
        const float b = g_pm ? m[u][i] * rm * gb[i] : m[u][i];
        m[u][i] = a + b;  // reuse m for the sum
        ssc = fmaf(m[u][i], m[u][i], ssc);
      }
    }
  }
  const float rc = 1.0f / sqrtf(block_sum(ssc, red) / H + eps);
#pragma unroll
  for (int u = 0; u < kCombMaxChunks; ++u) {
    const int c = threadIdx.x + u * kCombThreads;
    if (c < nch) {
      float xf[8], g[8], o[8];
      unpack8(__ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H) + c), xf);
      unpack8(__ldg(reinterpret_cast<const uint4*>(g_ff) + c), g);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = xf[i] + m[u][i] * rc * g[i];
      reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H)[c] = pack8(o);
    }
  }
}

// moe_out[t] = sum_j Y[t*k + j] in fp32, slot order, rounded to bf16.
__global__ void __launch_bounds__(kCombThreads) combine_moe_kernel(int H, int k,
                                                                   const uint16_t* __restrict__ y,
                                                                   uint16_t* __restrict__ moe_out) {
  const int t = blockIdx.x;
  for (int c = threadIdx.x; c < (H >> 3); c += kCombThreads) {
    float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      float f[8];
      unpack8(__ldg(reinterpret_cast<const uint4*>(y + (static_cast<size_t>(t) * k + j) * H) + c), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] += f[i];
    }
    reinterpret_cast<uint4*>(moe_out + static_cast<size_t>(t) * H)[c] = pack8(m);
  }
}

cudaError_t launch_combine_block(int T, int H, int k, float eps, const uint16_t* x,
                                 const uint16_t* y, const uint16_t* dense,
                                 const uint16_t* g_post_moe, const uint16_t* g_post_dense,
                                 const uint16_t* g_post_ff, uint16_t* out, uint16_t* moe_out,
                                 cudaStream_t s) {
  combine_block_kernel<<<T, kCombThreads, 0, s>>>(H, k, eps, x, y, dense, g_post_moe,
                                                  g_post_dense, g_post_ff, out, moe_out);
  return cudaGetLastError();
}

cudaError_t launch_combine_moe(int T, int H, int k, const uint16_t* y, uint16_t* moe_out,
                               cudaStream_t s) {
  combine_moe_kernel<<<T, kCombThreads, 0, s>>>(H, k, y, moe_out);
  return cudaGetLastError();
}

}  // namespace moe
