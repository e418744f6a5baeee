// Router of the MoE block and the pre norms of both branches.
//
// Follows the router of the ONNX export card ("Truthful graph contracts", Router row):
// scale-free RMSNorm -> learned scale x hidden_size^-0.5 -> linear to E logits ->
// softmax (fp32) -> top-k -> renormalise -> per_expert_scale.  The same rms(x) serves
// the pre norms of the MoE and dense branches, so this kernel also writes
// xn_moe = xhat * g_pre_moe and xn_dense = xhat * g_pre_dense.
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kRouterTokens = 8;    // tokens per CTA (one warp each in the norm phase)
constexpr int kRouterExperts = 16;  // experts per CTA (two per warp)

// Grid (ceil(T / 8), ceil(E / 16)), 256 threads.  Dynamic smem: 8 * H floats (z).
__global__ void __launch_bounds__(256) router_logits_kernel(
    int T, int H, int E, float eps, float inv_sqrt_h, const uint16_t* __restrict__ x,
    const uint16_t* __restrict__ rscale, const uint16_t* __restrict__ wr,
    const float* __restrict__ bias, const uint16_t* __restrict__ gm,
    const uint16_t* __restrict__ gd, uint16_t* __restrict__ xn_moe,
    uint16_t* __restrict__ xn_dense, float* __restrict__ logits) {
  extern __shared__ float z[];  // [kRouterTokens][H]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kRouterTokens;
  const int nchunk = H >> 3;  // 8 values per 16-byte chunk

  // ---- phase 1: rms(x) per token, z = xhat * scale * H^-0.5, and the pre norms
  {
    const int t = t0 + warp;
    float* zt = z + warp * H;
    if (t < T) {
      const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H);
      float ss = 0.f;
      for (int c = lane; c < nchunk; c += 32) {
        float f[8];
        unpack8(__ldg(xr + c), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
      }
      ss = warp_sum(ss);
      const float r = 1.0f / sqrtf(ss / static_cast<float>(H) + eps);
      const bool write_norms = (blockIdx.y == 0);
      for (int c = lane; c < nchunk; c += 32) {
        float f[8], s[8];
        unpack8(__ldg(xr + c), f);
        unpack8(__ldg(reinterpret_cast<const uint4*>(rscale) + c), s);
        float xh[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) xh[i] = f[i] * r;
        float4* zz = reinterpret_cast<float4*>(zt + c * 8);
        zz[0] = make_float4(xh[0] * s[0] * inv_sqrt_h, xh[1] * s[1] * inv_sqrt_h,
                            xh[2] * s[2] * inv_sqrt_h, xh[3] * s[3] * inv_sqrt_h);
        zz[1] = make_float4(xh[4] * s[4] * inv_sqrt_h, xh[5] * s[5] * inv_sqrt_h,
                            xh[6] * s[6] * inv_sqrt_h, xh[7] * s[7] * inv_sqrt_h);
        if (write_norms) {
          float a[8], b[8], g[8];
          unpack8(__ldg(reinterpret_cast<const uint4*>(gm) + c), g);
#pragma unroll
          for (int i = 0; i < 8; ++i) a[i] = xh[i] * g[i];
          unpack8(__ldg(reinterpret_cast<const uint4*>(gd) + c), g);
#pragma unroll
          for (int i = 0; i < 8; ++i) b[i] = xh[i] * g[i];
          reinterpret_cast<uint4*>(xn_moe + static_cast<size_t>(t) * H)[c] = pack8(a);
          reinterpret_cast<uint4*>(xn_dense + static_cast<size_t>(t) * H)[c] = pack8(b);
        }
      }
    } else {
      for (int i = lane; i < H; i += 32) zt[i] = 0.f;
    }
  }
  __syncthreads();

  // ---- phase 2: two experts per warp against all tokens of the CTA
  const int ea = blockIdx.y * kRouterExperts + 2 * warp;
  const int eb = ea + 1;
  const bool va = ea < E, vb = eb < E;
  float acc[2][kRouterTokens];
#pragma unroll
  for (int t = 0; t < kRouterTokens; ++t) acc[0][t] = acc[1][t] = 0.f;
  const uint4* wa = reinterpret_cast<const uint4*>(wr + static_cast<size_t>(va ? ea : 0) * H);
  const uint4* wb = reinterpret_cast<const uint4*>(wr + static_cast<size_t>(vb ? eb : 0) * H);
  for (int c = lane; c < nchunk; c += 32) {
    float fa[8], fb[8];
    unpack8(__ldg(wa + c), fa);
    unpack8(__ldg(wb + c), fb);
#pragma unroll
    for (int t = 0; t < kRouterTokens; ++t) {
      const float4* zz = reinterpret_cast<const float4*>(z + t * H + c * 8);
      const float4 z0 = zz[0], z1 = zz[1];
      const float zv[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        acc[0][t] = fmaf(fa[i], zv[i], acc[0][t]);
        acc[1][t] = fmaf(fb[i], zv[i], acc[1][t]);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kRouterTokens; ++t) {
    acc[0][t] = warp_sum(acc[0][t]);
    acc[1][t] = warp_sum(acc[1][t]);
  }
  if (lane < kRouterTokens) {
    const int t = t0 + lane;
    float la = 0.f, lb = 0.f;
#pragma unroll
    for (int i = 0; i < kRouterTokens; ++i)
      if (i == lane) { la = acc[0][i]; lb = acc[1][i]; }
    if (t < T) {
      if (va) logits[static_cast<size_t>(t) * E + ea] = la + (bias ? bias[ea] : 0.f);
      if (vb) logits[static_cast<size_t>(t) * E + eb] = lb + (bias ? bias[eb] : 0.f);
    }
  }
}

// One warp per token: top-k of the logits (ties to the lower expert id), then the
// softmax restricted to the selected experts (the full-softmax denominator cancels
// in the renormalisation), then per_expert_scale.
__global__ void __launch_bounds__(256) router_topk_kernel(int T, int E, int k,
                                                          const float* __restrict__ logits,
                                                          const uint16_t* __restrict__ pes,
                                                          int* __restrict__ topk_idx,
                                                          float* __restrict__ topk_w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  float v[8];
  unsigned taken = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    float l = (e < E) ? logits[static_cast<size_t>(t) * E + e] : -INFINITY;
    v[i] = (l != l) ? -INFINITY : l;  // NaN sorts last
    if (e >= E) taken |= 1u << i;
  }
  float sel_v[16];
  int sel_i[16];
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (!(taken & (1u << i)) && (v[i] > bv || (v[i] == bv && e < bi))) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    sel_v[j] = bv;
    sel_i[j] = bi;
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
  }
  const float m = sel_v[0];
  float e_sum = 0.f;
  float ex[16];
  for (int j = 0; j < k; ++j) {
    ex[j] = expf(sel_v[j] - m);
    e_sum += ex[j];
  }
  for (int j = 0; j < k; ++j) {
    if (lane == j) {
      const float p = __uint_as_float(static_cast<uint32_t>(pes[sel_i[j]]) << 16);
      topk_idx[static_cast<size_t>(t) * k + j] = sel_i[j];
      topk_w[static_cast<size_t>(t) * k + j] = ex[j] / e_sum * p;
    }
  }
}

cudaError_t launch_router_logits(int T, int H, int E, float eps, float inv_sqrt_h,
                                 const uint16_t* x, const uint16_t* router_scale,
                                 const uint16_t* w_router, const float* bias,
                                 const uint16_t* g_pre_moe, const uint16_t* g_pre_dense,
                                 uint16_t* xn_moe, uint16_t* xn_dense, float* logits,
                                 cudaStream_t s) {
  const size_t smem = static_cast<size_t>(kRouterTokens) * H * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(router_logits_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid((T + kRouterTokens - 1) / kRouterTokens, (E + kRouterExperts - 1) / kRouterExperts);
  router_logits_kernel<<<grid, 256, smem, s>>>(T, H, E, eps, inv_sqrt_h, x, router_scale,
                                               w_router, bias, g_pre_moe, g_pre_dense, xn_moe,
                                               xn_dense, logits);
  return cudaGetLastError();
}

cudaError_t launch_router_topk(int T, int E, int k, const float* logits,
                               const uint16_t* per_expert_scale, int* topk_idx, float* topk_w,
                               cudaStream_t s) {
  router_topk_kernel<<<(T + 7) / 8, 256, 0, s>>>(T, E, k, logits, per_expert_scale, topk_idx,
                                                 topk_w);
  return cudaGetLastError();
}

}  // namespace moe
