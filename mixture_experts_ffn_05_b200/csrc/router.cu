// Router of the MoE block and the pre norms of both branches, in one launch.
//
// Follows the router of the ONNX export card ("Truthful graph contracts", Router row):
// scale-free RMSNorm -> learned scale x hidden_size^-0.5 -> linear to E logits ->
// softmax (fp32) -> top-k -> renormalise -> per_expert_scale.  The same rms(x) serves
// the pre norms of the MoE and dense branches, so the kernel also writes
// xn_moe = xhat * g_pre_moe and xn_dense = xhat * g_pre_dense.
//
// Grid (token blocks of 8, expert slices).  Every CTA stages its 8 tokens in shared
// memory as z' = x * scale * H^-0.5 (fp32) in the same pass that sums x^2, and computes
// the logits of its expert slice as (z' . W_r[e]) / rms(x): the norm factor is a
// per-token scalar, so it can be applied after the dot product.  Each warp owns one
// eighth of H for all experts of the slice, and the eight partial sums are added in
// warp order.  The last CTA of a token block to finish (an
// atomic counter) takes the top-k of its 8 tokens.  When asked, the last token block to
// finish then runs the token-to-expert counting sort for the whole batch, so a decode
// step routes and sorts in a single launch.  Counters reset themselves after use.
#include "common.cuh"
#include "internal.h"
#include "permute_impl.cuh"

namespace moe {

constexpr int kRT = 8;        // tokens per CTA
constexpr int kRThreads = 256;

// Orderable 64-bit key of (logit, expert): a larger key is a larger logit, and for equal
// logits a smaller expert id.  NaN sorts below every number.
__device__ __forceinline__ unsigned long long topk_key(float l, int e) {
  if (l != l) l = -INFINITY;
  uint32_t u = __float_as_uint(l);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // monotone in the float value
  return (static_cast<unsigned long long>(u) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(e));
}

__device__ __forceinline__ float key_logit(unsigned long long key) {
  uint32_t u = static_cast<uint32_t>(key >> 32);
  u = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
  return __uint_as_float(u);
}

// Top-k of one token's logits (ties to the lower expert id), then the softmax restricted
// to the selected experts (the full-softmax denominator cancels in the renormalisation),
// then per_expert_scale.  One warp: each lane sorts its (up to 8) candidates, then each
// of the k rounds takes the warp maximum of the lanes' best remaining keys.
__device__ void topk_one_token(int t, int E, int k, const float* logits, const uint16_t* pes,
                               int* __restrict__ topk_idx, float* __restrict__ topk_w,
                               int* s_ids = nullptr) {
  const int lane = threadIdx.x & 31;
  unsigned long long key[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    key[i] = (e < E) ? topk_key(__ldcg(logits + static_cast<size_t>(t) * E + e), e) : 0ull;
  }
  // sort the lane's 8 keys in descending order (odd-even transposition, registers only)
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int i = r & 1; i + 1 < 8; i += 2)
      if (key[i] < key[i + 1]) {
        const unsigned long long tmp = key[i];
        key[i] = key[i + 1];
        key[i + 1] = tmp;
      }
  unsigned long long mine = 0ull;  // lane j keeps the j-th selected key
  for (int j = 0; j < k; ++j) {
    unsigned long long best = key[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other > best ? other : best;
    }
    if (key[0] == best) {  // keys are unique: exactly one lane pops its head
#pragma unroll
      for (int i = 0; i < 7; ++i) key[i] = key[i + 1];
      key[7] = 0ull;
    }
    if (lane == j) mine = best;
  }
  const float top = key_logit(__shfl_sync(0xffffffffu, mine, 0));
  const int my_i = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(mine));
  const float ex = lane < k ? expf(key_logit(mine) - top) : 0.f;
  float e_sum = 0.f;  // sum in slot order, the same order on every run
  for (int j = 0; j < k; ++j) e_sum += __shfl_sync(0xffffffffu, ex, j);
  if (lane < k) {
    const float p = __uint_as_float(static_cast<uint32_t>(pes[my_i]) << 16);
    topk_idx[static_cast<size_t>(t) * k + lane] = my_i;
    topk_w[static_cast<size_t>(t) * k + lane] = ex / e_sum * p;
    if (s_ids) s_ids[t * k + lane] = my_i;
  }
}

// Stable counting sort of n <= 128 (token, slot) pairs held in shared memory, by the
// first four warps of the CTA: ranks inside a warp from __match_any_sync + popc, across
// warps from per-warp counts in warp order, so the order is by (expert, p) exactly as in
// the general sort.  All threads of the CTA call it.
__device__ void sort_small(int n, int E, const int* s_ids, int (*s_wcnt)[kPermMaxE],
                           int* s_tot, int* s_off, int* __restrict__ offsets,
                           int* __restrict__ sorted_src, int* __restrict__ inv_pos) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < 4 * kPermMaxE; i += blockDim.x) (&s_wcnt[0][0])[i] = 0;
  __syncthreads();
  int e = -1, rank = 0;
  if (warp < 4) {
    e = tid < n ? s_ids[tid] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    rank = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && rank == 0) s_wcnt[warp][e] = __popc(peers);
  }
  __syncthreads();
  for (int x = tid; x < E; x += blockDim.x)
    s_tot[x] = s_wcnt[0][x] + s_wcnt[1][x] + s_wcnt[2][x] + s_wcnt[3][x];
  __syncthreads();
  if (tid < 32) warp_exclusive_scan(s_tot, s_off, E);
  __syncthreads();
  for (int i = tid; i <= E; i += blockDim.x) offsets[i] = s_off[i];
  if (e >= 0) {
    int pos = s_off[e] + rank;
    for (int w = 0; w < warp; ++w) pos += s_wcnt[w][e];
    sorted_src[pos] = tid;
    inv_pos[tid] = pos;
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
  unsigned* status;    // device status word (a bounded wait that ran out)
  int stage_w;         // copy the slice's W_r rows to shared memory first
  // counting sort of all T*k pairs by the last token block (NULL = not here)
  int* offsets;
  int* sorted_src;
  int* inv_pos;
};

// Narrow expert slices (EB <= kStageEB) copy their W_r rows into shared memory with 1-D
// bulk copies at the start, overlapping the pass over x.
constexpr int kStageEB = 4;

template <int EB>
__global__ void __launch_bounds__(kRThreads) router_kernel(const RouterArgs a) {
  extern __shared__ __align__(16) float z[];  // [kRT][H], then (narrow slices) W_r rows
  __shared__ float part[8][EB * kRT];
  __shared__ int flag;
  __shared__ __align__(8) uint64_t wbar;
  __shared__ uint16_t s_pes[kPermMaxE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < a.E; e += kRThreads) s_pes[e] = a.pes[e];
  const int H = a.H, E = a.E;
  const int t0 = blockIdx.x * kRT;
  const int nch = H >> 3;  // chunks of 8 values
  const bool stage_w = a.stage_w != 0;
  uint16_t* wsm = reinterpret_cast<uint16_t*>(z + kRT * H);  // [EB][H] bf16
  if (stage_w && threadIdx.x == 0) {
    // W_r is a weight (not produced by an earlier kernel), so it is fetched before the
    // dependency wait
    mbar_init(&wbar, 1);
    mbar_fence_init();
    mbar_arrive_expect_tx(&wbar, EB * H * 2);
    for (int i = 0; i < EB; ++i) {
      const int e = min(blockIdx.y * EB + i, E - 1);
      bulk_load_1d(wsm + i * H, a.wr + static_cast<size_t>(e) * H, H * 2, &wbar);
    }
  }
  pdl_wait();
  pdl_trigger();

  // ---- one pass over the CTA's tokens: z' = x * scale * H^-0.5 (the norm factor
  // 1/rms(x) is a per-token scalar, applied to the logits at the end) and sum(x^2)
  __shared__ float rinv[kRT];
  {
    const int t = t0 + warp;
    float* zt = z + warp * H;
    if (t < a.T) {
      const uint4* xr = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * H);
      const uint4* sr = reinterpret_cast<const uint4*>(a.rscale);
      float ss = 0.f;
      for (int c0 = lane; c0 < nch; c0 += 32 * 4) {
        uint4 vx[4], vs[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // 8 loads in flight per lane
          const int c = min(c0 + 32 * u, nch - 1);
          vx[u] = __ldg(xr + c);
          vs[u] = __ldg(sr + c);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + 32 * u;
          if (c < nch) {
            float f[8], sc[8];
            unpack8(vx[u], f);
            unpack8(vs[u], sc);
#pragma unroll
            for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
            float4* zz = reinterpret_cast<float4*>(zt + c * 8);
            zz[0] = make_float4(f[0] * sc[0] * a.inv_sqrt_h, f[1] * sc[1] * a.inv_sqrt_h,
                                f[2] * sc[2] * a.inv_sqrt_h, f[3] * sc[3] * a.inv_sqrt_h);
            zz[1] = make_float4(f[4] * sc[4] * a.inv_sqrt_h, f[5] * sc[5] * a.inv_sqrt_h,
                                f[6] * sc[6] * a.inv_sqrt_h, f[7] * sc[7] * a.inv_sqrt_h);
          }
        }
      }
      ss = warp_sum(ss);
      if (lane == 0) rinv[warp] = 1.0f / sqrtf(ss / static_cast<float>(H) + a.eps);
    } else {
      for (int i = lane; i < H; i += 32) zt[i] = 0.f;
      if (lane == 0) rinv[warp] = 0.f;
    }
  }
  __syncthreads();

  // ---- logits of the slice: warp w sums its eighth of H, 4 experts x 8 tokens at a time
  const int e0 = blockIdx.y * EB;
  const int cb = warp * nch / 8, ce = (warp + 1) * nch / 8;
  if (stage_w) {
    if (threadIdx.x == 0) flag = mbar_wait(&wbar, 0, 2000000000ull, nullptr) ? 1 : 0;
    __syncthreads();
    if (!flag) {  // the copy did not land in time: report it, leave the outputs alone
      if (threadIdx.x == 0) record_status(a.status, kStatusTimeout);
      return;
    }
  }
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
      wrow[i] = stage_w ? reinterpret_cast<const uint4*>(wsm + (4 * g + i) * H)
                        : reinterpret_cast<const uint4*>(a.wr + static_cast<size_t>(e) * H);
    }
    for (int c0 = cb + lane; c0 < ce; c0 += 64) {
      uint4 wv[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u)  // both chunks' weights in flight before any math
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = min(c0 + 32 * u, ce - 1);
          wv[u][i] = stage_w ? wrow[i][c] : __ldg(wrow[i] + c);
        }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c = c0 + 32 * u;
        if (c < ce) {
          float w[4][8];
#pragma unroll
          for (int i = 0; i < 4; ++i) unpack8(wv[u][i], w[i]);
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
      }
    }
    // transpose-reduce the 32 sums over the warp: after 5 halving steps (31 shuffles)
    // lane l holds the full sum of value index l = i * 8 + t
    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int t = 0; t < kRT; ++t) v[i * kRT + t] = acc[i][t];
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
      const bool upper = (lane & w) != 0;
#pragma unroll
      for (int j = 0; j < w; ++j) {
        const float send = upper ? v[j] : v[j + w];
        const float keep = upper ? v[j + w] : v[j];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, w);
      }
    }
    // lane l now holds value index l (the halving kept bit b of the index where bit b of
    // the lane is set)
    part[warp][4 * g * kRT + lane] = v[0];
  }
  __syncthreads();
  for (int j = threadIdx.x; j < EB * kRT; j += kRThreads) {
    const int e = e0 + j / kRT, tl = j % kRT, t = t0 + tl;
    if (e < E && t < a.T) {
      float sm = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) sm += part[w][j];
      a.logits[static_cast<size_t>(t) * E + e] = sm * rinv[tl] + (a.bias ? a.bias[e] : 0.f);
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
  // ---- every expert slice writes its share of the pre norms of both branches:
  // columns [y, y + gridDim.y, ...) in chunks of 8, for the CTA's tokens
  {
    const int t = t0 + warp;
    if (t < a.T) {
      const float r = rinv[warp];
      const uint4* xr = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * H);
      for (int c = blockIdx.y + gridDim.y * lane; c < nch; c += gridDim.y * 32) {
        float f[8], gm[8], gd[8], o1[8], o2[8];
        unpack8(__ldg(xr + c), f);
        unpack8(__ldg(reinterpret_cast<const uint4*>(a.gm) + c), gm);
        unpack8(__ldg(reinterpret_cast<const uint4*>(a.gd) + c), gd);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float xh = f[i] * r;
          o1[i] = xh * gm[i];
          o2[i] = xh * gd[i];
        }
        reinterpret_cast<uint4*>(a.xn_moe + static_cast<size_t>(t) * H)[c] = pack8(o1);
        reinterpret_cast<uint4*>(a.xn_dense + static_cast<size_t>(t) * H)[c] = pack8(o2);
      }
    }
  }
  __syncthreads();
  if (!flag) return;
  __shared__ int s_ids[kRT * 16];
  const bool small_sort = a.offsets != nullptr && gridDim.x == 1;  // every pair is here
  if (t0 + warp < a.T)
    topk_one_token(t0 + warp, E, a.k, a.logits, s_pes, a.topk_idx, a.topk_w,
                   small_sort ? s_ids : nullptr);
  if (a.offsets == nullptr) return;
  if (small_sort) {
    __shared__ int s_wcnt[4][kPermMaxE];
    __shared__ int s_tot[kPermMaxE];
    __shared__ int s_off[kPermMaxE + 1];
    __syncthreads();
    sort_small(a.T * a.k, E, s_ids, s_wcnt, s_tot, s_off, a.offsets, a.sorted_src, a.inv_pos);
    return;
  }

  // ---- the last token block sorts every (token, slot) pair by expert
  __syncthreads();
  if (gridDim.x > 1) {
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
  }
  __shared__ PermuteSmem<kRThreads> ps;
  permute_block<kRThreads>(a.T * a.k, E, a.topk_idx, a.offsets, a.sorted_src, a.inv_pos, ps);
}

template <int EB>
static cudaError_t launch_eb(const RouterArgs& a, cudaStream_t s, bool pdl) {
  const size_t zbytes = static_cast<size_t>(kRT) * a.H * sizeof(float);
  const size_t wbytes = static_cast<size_t>(EB) * a.H * 2;
  RouterArgs b = a;
  b.stage_w = (EB <= kStageEB && zbytes + wbytes <= 160 * 1024) ? 1 : 0;
  const size_t smem = zbytes + (b.stage_w ? wbytes : 0);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(router_kernel<EB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid((a.T + kRT - 1) / kRT, (a.E + EB - 1) / EB);
  return launch_k(router_kernel<EB>, grid, dim3(kRThreads), smem, s, pdl, b);
}

int router_counters(int T) { return (T + kRT - 1) / kRT + 1; }

cudaError_t launch_router(int T, int H, int E, int k, float eps, const uint16_t* x,
                          const uint16_t* router_scale, const uint16_t* w_router,
                          const float* bias, const uint16_t* per_expert_scale,
                          const uint16_t* g_pre_moe, const uint16_t* g_pre_dense,
                          uint16_t* xn_moe, uint16_t* xn_dense, float* logits, int* topk_idx,
                          float* topk_w, unsigned* counters, unsigned* status, int* offsets,
                          int* sorted_src, int* inv_pos, cudaStream_t s, bool pdl) {
  RouterArgs a{T, H, E, k, eps, 1.0f / sqrtf(static_cast<float>(H)), x, router_scale, w_router,
               bias, per_expert_scale, g_pre_moe, g_pre_dense, xn_moe, xn_dense, logits,
               topk_idx, topk_w, counters, status, 0, offsets, sorted_src, inv_pos};
  // Narrow expert slices for small batches (more CTAs streaming W_r), wide ones for
  // large batches (fewer redundant normalisations).
  if (T <= 64) return launch_eb<4>(a, s, pdl);
  return launch_eb<32>(a, s, pdl);
}

}  // namespace moe
