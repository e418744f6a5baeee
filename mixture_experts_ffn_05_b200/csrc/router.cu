// Router of the MoE block and the pre norms of both branches, in one launch.
//
// Follows the router of the ONNX export card ("Truthful graph contracts", Router row):
// scale-free RMSNorm -> learned scale x hidden_size^-0.5 -> linear to E logits ->
// softmax (fp32) -> top-k -> renormalise -> per_expert_scale.  The same rms(x) serves
// the pre norms of the MoE and dense branches, so the kernel also writes
// xn_moe = xhat * g_pre_moe and xn_dense = xhat * g_pre_dense.
//
// Grid (token blocks of 8, expert slices).  Every CTA normalises its 8 tokens into
// shared memory (z = xhat * scale * H^-0.5, fp32) and computes the logits of its expert
// slice; each warp owns one eighth of H for all experts of the slice, and the eight
// partial sums are added in warp order.  The last CTA of a token block to finish (an
// atomic counter) takes the top-k of its 8 tokens.  When asked, the last token block to
// finish then runs the token-to-expert counting sort for the whole batch, so a decode
// step routes and sorts in a single launch.  Counters reset themselves after use.
#include "common.cuh"
#include "internal.h"
#include "permute_impl.cuh"

namespace moe {

constexpr int kRT = 8;        // tokens per CTA
constexpr int kRThreads = 256;

// Top-k of one token's logits (ties to the lower expert id), then the softmax restricted
// to the selected experts (the full-softmax denominator cancels in the renormalisation),
// then per_expert_scale.  One warp; logits read from global memory (L2).
__device__ void topk_one_token(int t, int E, int k, const float* logits,
                               const uint16_t* __restrict__ pes, int* __restrict__ topk_idx,
                               float* __restrict__ topk_w) {
  const int lane = threadIdx.x & 31;
  float v[8];
  unsigned taken = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    const float l = (e < E) ? __ldcg(logits + static_cast<size_t>(t) * E + e) : -INFINITY;
    v[i] = (l != l) ? -INFINITY : l;  // NaN sorts last
    if (e >= E) taken |= 1u << i;
  }
  float m = 0.f, e_sum = 0.f, my_ex = 0.f;
  int my_i = 0;
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
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (j == 0) m = bv;
    const float ex = expf(bv - m);
    e_sum += ex;
    if (lane == j) {
      my_ex = ex;
      my_i = bi;
    }
  }
  if (lane < k) {
    const float p = __uint_as_float(static_cast<uint32_t>(pes[my_i]) << 16);
    topk_idx[static_cast<size_t>(t) * k + lane] = my_i;
    topk_w[static_cast<size_t>(t) * k + lane] = my_ex / e_sum * p;
  }
}

struct RouterArgs {
  int T, H, E, k;
  float eps, inv_sqrt_h;
  const uint16_t* x;
  const uint16_t* rscale;
  const uint16_t* wr;
  const float* bias;
  const uint16_t* pes;
  const uint16_t* gm;
  const uint16_t* gd;
  uint16_t* xn_moe;
  uint16_t* xn_dense;
  float* logits;
  int* topk_idx;
  float* topk_w;
  unsigned* counters;  // [token blocks + 1], zero on entry, zero again on exit
  // counting sort of all T*k pairs by the last token block (NULL = not here)
  int* offsets;
  int* sorted_src;
  int* inv_pos;
};

template <int EB>
__global__ void __launch_bounds__(kRThreads) router_kernel(const RouterArgs a) {
  extern __shared__ float z[];  // [kRT][H]
  __shared__ float part[8][EB * kRT];
  __shared__ int flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = a.H, E = a.E;
  const int t0 = blockIdx.x * kRT;
  const int nch = H >> 3;  // chunks of 8 values
  pdl_wait();
  pdl_trigger();

  // ---- normalise the CTA's tokens into z; the first expert slice writes the pre norms
  {
    const int t = t0 + warp;
    float* zt = z + warp * H;
    if (t < a.T) {
      const uint4* xr = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * H);
      // loads are issued in batches so that a warp has several in flight at once
      float ss = 0.f;
      for (int c0 = lane; c0 < nch; c0 += 32 * 4) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + 32 * u;
          v[u] = c < nch ? __ldg(xr + c) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float f[8];
          unpack8(v[u], f);
#pragma unroll
          for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
        }
      }
      ss = warp_sum(ss);
      const float r = 1.0f / sqrtf(ss / static_cast<float>(H) + a.eps);
      const bool norms = blockIdx.y == 0;
      for (int c0 = lane; c0 < nch; c0 += 32 * 2) {
        uint4 vx[2], vs[2], vm[2], vd[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c = min(c0 + 32 * u, nch - 1);
          vx[u] = __ldg(xr + c);
          vs[u] = __ldg(reinterpret_cast<const uint4*>(a.rscale) + c);
          if (norms) {
            vm[u] = __ldg(reinterpret_cast<const uint4*>(a.gm) + c);
            vd[u] = __ldg(reinterpret_cast<const uint4*>(a.gd) + c);
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c = c0 + 32 * u;
          if (c >= nch) break;
          float f[8], s[8], xh[8];
          unpack8(vx[u], f);
          unpack8(vs[u], s);
#pragma unroll
          for (int i = 0; i < 8; ++i) xh[i] = f[i] * r;
          float4* zz = reinterpret_cast<float4*>(zt + c * 8);
          zz[0] = make_float4(xh[0] * s[0] * a.inv_sqrt_h, xh[1] * s[1] * a.inv_sqrt_h,
                              xh[2] * s[2] * a.inv_sqrt_h, xh[3] * s[3] * a.inv_sqrt_h);
          zz[1] = make_float4(xh[4] * s[4] * a.inv_sqrt_h, xh[5] * s[5] * a.inv_sqrt_h,
                              xh[6] * s[6] * a.inv_sqrt_h, xh[7] * s[7] * a.inv_sqrt_h);
          if (norms) {
            float o1[8], o2[8], g[8];
            unpack8(vm[u], g);
#pragma unroll
            for (int i = 0; i < 8; ++i) o1[i] = xh[i] * g[i];
            unpack8(vd[u], g);
#pragma unroll
            for (int i = 0; i < 8; ++i) o2[i] = xh[i] * g[i];
            reinterpret_cast<uint4*>(a.xn_moe + static_cast<size_t>(t) * H)[c] = pack8(o1);
            reinterpret_cast<uint4*>(a.xn_dense + static_cast<size_t>(t) * H)[c] = pack8(o2);
          }
        }
      }
    } else {
      for (int i = lane; i < H; i += 32) zt[i] = 0.f;
    }
  }
  __syncthreads();

  // ---- logits of the slice: warp w sums its eighth of H, 4 experts x 8 tokens at a time
  const int e0 = blockIdx.y * EB;
  const int cb = warp * nch / 8, ce = (warp + 1) * nch / 8;
#pragma unroll 1
  for (int g = 0; g < EB / 4; ++g) {
    float acc[4][kRT];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int t = 0; t < kRT; ++t) acc[i][t] = 0.f;
    const uint4* wrow[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = min(e0 + 4 * g + i, E - 1);
      wrow[i] = reinterpret_cast<const uint4*>(a.wr + static_cast<size_t>(e) * H);
    }
    for (int c = cb + lane; c < ce; c += 32) {
      float w[4][8];
#pragma unroll
      for (int i = 0; i < 4; ++i) unpack8(__ldg(wrow[i] + c), w[i]);
#pragma unroll
      for (int t = 0; t < kRT; ++t) {
        const float4* zz = reinterpret_cast<const float4*>(z + t * H + c * 8);
        const float4 z0 = zz[0], z1 = zz[1];
        const float zv[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[i][t] = fmaf(w[i][q], zv[q], acc[i][t]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int t = 0; t < kRT; ++t) {
        const float s = warp_sum(acc[i][t]);
        if (lane == 0) part[warp][(4 * g + i) * kRT + t] = s;
      }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < EB * kRT; j += kRThreads) {
    const int e = e0 + j / kRT, t = t0 + j % kRT;
    if (e < E && t < a.T) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) s += part[w][j];
      a.logits[static_cast<size_t>(t) * E + e] = s + (a.bias ? a.bias[e] : 0.f);
    }
  }

  // ---- the last slice of this token block takes the top-k
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned old = atomicAdd(a.counters + blockIdx.x, 1u);
    flag = old == gridDim.y - 1;
    if (flag) {
      a.counters[blockIdx.x] = 0u;
      __threadfence();
    }
  }
  __syncthreads();
  if (!flag) return;
  if (t0 + warp < a.T) topk_one_token(t0 + warp, E, a.k, a.logits, a.pes, a.topk_idx, a.topk_w);
  if (a.offsets == nullptr) return;

  // ---- the last token block sorts every (token, slot) pair by expert
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned old = atomicAdd(a.counters + gridDim.x, 1u);
    flag = old == gridDim.x - 1;
    if (flag) {
      a.counters[gridDim.x] = 0u;
      __threadfence();
    }
  }
  __syncthreads();
  if (!flag) return;
  __shared__ PermuteSmem<kRThreads> ps;
  permute_block<kRThreads>(a.T * a.k, E, a.topk_idx, a.offsets, a.sorted_src, a.inv_pos, ps);
}

template <int EB>
static cudaError_t launch_eb(const RouterArgs& a, cudaStream_t s, bool pdl) {
  const size_t smem = static_cast<size_t>(kRT) * a.H * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(router_kernel<EB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid((a.T + kRT - 1) / kRT, (a.E + EB - 1) / EB);
  return launch_k(router_kernel<EB>, grid, dim3(kRThreads), smem, s, pdl, a);
}

int router_counters(int T) { return (T + kRT - 1) / kRT + 1; }

cudaError_t launch_router(int T, int H, int E, int k, float eps, const uint16_t* x,
                          const uint16_t* router_scale, const uint16_t* w_router,
                          const float* bias, const uint16_t* per_expert_scale,
                          const uint16_t* g_pre_moe, const uint16_t* g_pre_dense,
                          uint16_t* xn_moe, uint16_t* xn_dense, float* logits, int* topk_idx,
                          float* topk_w, unsigned* counters, int* offsets, int* sorted_src,
                          int* inv_pos, cudaStream_t s, bool pdl) {
  RouterArgs a{T, H, E, k, eps, 1.0f / sqrtf(static_cast<float>(H)), x, router_scale, w_router,
               bias, per_expert_scale, g_pre_moe, g_pre_dense, xn_moe, xn_dense, logits,
               topk_idx, topk_w, counters, offsets, sorted_src, inv_pos};
  // Narrow expert slices for small batches (more CTAs streaming W_r), wide ones for
  // large batches (fewer redundant normalisations).
  if (T <= 64) return launch_eb<4>(a, s, pdl);
  return launch_eb<32>(a, s, pdl);
}

}  // namespace moe
