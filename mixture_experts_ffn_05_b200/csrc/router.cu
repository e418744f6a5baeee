// Router of the MoE block and the pre norms of both branches, in one launch (batches of
// up to 128 tokens; larger ones take the tensor-memory router, router_tc.cu).
//
// Follows the router of the ONNX export card ("Truthful graph contracts", Router row):
// scale-free RMSNorm -> learned scale x hidden_size^-0.5 -> linear to E logits ->
// softmax (fp32) -> top-k -> renormalise -> per_expert_scale.  The same rms(x) serves
// the pre norms of the MoE and dense branches, so the kernel also writes
// xn_moe = xhat * g_pre_moe and xn_dense = xhat * g_pre_dense.
//
// Grid (token blocks of 8, expert slices of EB <= 8), sized to about one CTA per SM.  A
// CTA copies its W_r rows and the router scale into shared memory with bulk copies
// before the dependency wait (weights do not come from an earlier kernel), then its
// token rows.  The norm factor 1/rms(x) is a per-token scalar, so the logits are
// rinv * (x . W'[e]) + b[e] with W' = scale * W_r * H^-0.5 formed in fp32.  The dot
// products run on mma.sync (m16n8k16, bf16 operands, fp32 accumulation) with W' split
// into two bf16 terms, W' = hi + lo + d, |d| <= 2^-16 |W'| (the split of the
// tensor-memory router): A rows 0..7 hold hi of the slice's experts, rows 8..15 lo, B
// the 8 tokens as they are, so every product is exact and the two halves of the
// accumulator add up to the logit.  Warp w takes every 16th K step, and the 16 partial
// sums are added in warp order; the same pass sums x^2 per token.  Every expert slice
// writes its share of the columns of xn_moe and xn_dense.  The last slice of a token
// block to finish (an acq_rel counter) takes the top-k of its 8 tokens; when asked, the
// last token block then runs the token-to-expert counting sort for the whole batch, so
// a decode step routes and sorts in one launch.  Counters reset themselves after use.
#include "common.cuh"
#include "internal.h"
#include "warp_mma.cuh"
#include "permute_impl.cuh"

namespace moe {

constexpr int kRT = 8;          // tokens per CTA (the MMA's N)
constexpr int kRThreads = 512;  // 16 warps
constexpr int kRWarps = kRThreads / 32;
constexpr int kRMaxEB = 8;      // experts per CTA (the MMA's M holds hi and lo of each)

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
// then per_expert_scale.  One warp: each lane sorts its KPL candidates (experts lane +
// 32 i), then each of the k rounds takes the warp maximum of the lanes' best remaining
// keys, high word first, then the low word among the lanes that share it.
template <int KPL>
__device__ void topk_one_token(int t, int E, int k, const float* logits, const uint16_t* pes,
                               int* __restrict__ topk_idx, float* __restrict__ topk_w,
                               int* s_ids = nullptr) {
  const int lane = threadIdx.x & 31;
  unsigned long long key[KPL];
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    const int e = lane + 32 * i;
    key[i] = (e < E) ? topk_key(__ldcg(logits + static_cast<size_t>(t) * E + e), e) : 0ull;
  }
  // sort the lane's keys in descending order (odd-even transposition, registers only)
#pragma unroll
  for (int r = 0; r < KPL; ++r)
#pragma unroll
    for (int i = r & 1; i + 1 < KPL; i += 2)
      if (key[i] < key[i + 1]) {
        const unsigned long long tmp = key[i];
        key[i] = key[i + 1];
        key[i + 1] = tmp;
      }
  unsigned long long mine = 0ull;  // lane j keeps the j-th selected key
  for (int j = 0; j < k; ++j) {
    const uint32_t hi = static_cast<uint32_t>(key[0] >> 32);
    const uint32_t bh = __reduce_max_sync(0xffffffffu, hi);
    const uint32_t bl = __reduce_max_sync(0xffffffffu, hi == bh ? static_cast<uint32_t>(key[0]) : 0u);
    const unsigned long long best = (static_cast<unsigned long long>(bh) << 32) | bl;
    if (key[0] == best) {  // keys are unique: exactly one lane pops its head
#pragma unroll
      for (int i = 0; i + 1 < KPL; ++i) key[i] = key[i + 1];
      key[KPL - 1] = 0ull;
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
  // counting sort of all T*k pairs by the last token block (NULL = not here)
  int* offsets;
  int* sorted_src;
  int* inv_pos;
  // with the sort of a single token block: the routed rows of xn_moe in sorted order
  // (fp16 when aperm_f16), or NULL
  uint16_t* aperm;
  int aperm_f16;
};

// Two floats rounded to bf16 (nearest even), the first in the low half.
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int EB>
__global__ void __launch_bounds__(kRThreads, 1) router_kernel(const RouterArgs a) {
  // x rows [8], W_r rows [EB] and the scale row, each padded by 32 bytes so that the eight
  // rows read by the lanes of one phase start in distinct banks
  extern __shared__ __align__(128) uint8_t r_smem[];
  __shared__ float part[kRWarps][kRMaxEB][kRT];
  __shared__ float ssp[kRWarps][kRT];
  __shared__ float rinv[kRT];
  __shared__ int flag;
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint16_t s_pes[kPermMaxE];
  __shared__ int s_ids[kRT * 16];
  __shared__ int s_tok[kRT * 16];  // router gather: the token of each sorted position
  __shared__ PermuteSmem<kRThreads> ps;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int H = a.H, E = a.E;
  const int t0 = blockIdx.x * kRT, e0 = blockIdx.y * EB;
  const int nt = min(kRT, a.T - t0);  // tokens of the block
  const int ne = min(EB, E - e0);     // experts of the slice
  const uint32_t row_bytes = static_cast<uint32_t>(H) * 2u;
  const int RS = H + 16;  // padded row stride in elements
  uint16_t* xs = reinterpret_cast<uint16_t*>(r_smem);
  uint16_t* wsm = xs + kRT * RS;
  uint16_t* ssc = wsm + EB * RS;
  if (tid == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
    mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(ne + 1 + nt) * row_bytes);
    for (int i = 0; i < ne; ++i)
      bulk_load_1d(wsm + i * RS, a.wr + static_cast<size_t>(e0 + i) * H, row_bytes, &bar);
    bulk_load_1d(ssc, a.rscale, row_bytes, &bar);
  }
  for (int e = tid; e < E; e += kRThreads) s_pes[e] = a.pes[e];
  // this slice's share of the pre-norm columns: chunks [cb, ce) of 8 values, for each token
  const int nch = H >> 3;
  const int cb = static_cast<int>(static_cast<int64_t>(blockIdx.y) * nch / gridDim.y);
  const int ce = static_cast<int>(static_cast<int64_t>(blockIdx.y + 1) * nch / gridDim.y);
  const int nc = ce - cb, npairs = nc * nt;
  uint4 gm0 = make_uint4(0u, 0u, 0u, 0u), gd0 = gm0;  // the gains of the first pair, early
  if (tid < npairs) {
    gm0 = __ldg(reinterpret_cast<const uint4*>(a.gm) + cb + tid % nc);
    gd0 = __ldg(reinterpret_cast<const uint4*>(a.gd) + cb + tid % nc);
  }
  pdl_wait();
  pdl_trigger();
  if (tid == 0) {
    for (int i = 0; i < nt; ++i)
      bulk_load_1d(xs + i * RS, a.x + static_cast<size_t>(t0 + i) * H, row_bytes, &bar);
    flag = mbar_wait(&bar, 0, 2000000000ull, nullptr) ? 1 : 0;
  }
  __syncthreads();
  if (!flag) {  // the copies did not land in time: report it, leave the outputs alone
    if (tid == 0) record_status(a.status, kStatusTimeout);
    return;
  }

  // ---- logits of the slice and sum(x^2): warp w takes K steps w, w + 16, ...; lane (g, t)
  // takes elements [16 s + 4t, +4) of step s (a permutation of K applied to both operands)
  {
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    float ss = 0.f;
    const bool xok = g < nt, wok = g < ne;
    const uint16_t* xr = xs + g * RS + 4 * t;
    const uint16_t* wr = wsm + g * RS + 4 * t;
    const uint16_t* sr = ssc + 4 * t;
    const float ish = a.inv_sqrt_h;
#pragma unroll 2
    for (int st = warp; st < (H >> 4); st += kRWarps) {
      const int k0 = st * 16;
      uint2 xv = make_uint2(0u, 0u);
      if (xok) xv = *reinterpret_cast<const uint2*>(xr + k0);
      const float x0 = bf16lo(xv.x), x1 = bf16hi(xv.x), x2 = bf16lo(xv.y), x3 = bf16hi(xv.y);
      ss = fmaf(x0, x0, ss);
      ss = fmaf(x1, x1, ss);
      ss = fmaf(x2, x2, ss);
      ss = fmaf(x3, x3, ss);
      uint32_t h01 = 0u, h23 = 0u, l01 = 0u, l23 = 0u;
      if (wok) {
        const uint2 wv = *reinterpret_cast<const uint2*>(wr + k0);
        const uint2 sv = *reinterpret_cast<const uint2*>(sr + k0);
        const float v0 = bf16lo(wv.x) * bf16lo(sv.x) * ish, v1 = bf16hi(wv.x) * bf16hi(sv.x) * ish;
        const float v2 = bf16lo(wv.y) * bf16lo(sv.y) * ish, v3 = bf16hi(wv.y) * bf16hi(sv.y) * ish;
        h01 = cvt_bf16x2(v0, v1);
        h23 = cvt_bf16x2(v2, v3);
        l01 = cvt_bf16x2(v0 - bf16lo(h01), v1 - bf16hi(h01));
        l23 = cvt_bf16x2(v2 - bf16lo(h23), v3 - bf16hi(h23));
      }
      mma16816<true>(c, h01, l01, h23, l23, xv.x, xv.y);
    }
    // C rows g (hi) and g + 8 (lo) of expert g, columns (tokens) 2t and 2t + 1
    if (g < EB) {
      part[warp][g][2 * t] = c[0] + c[2];
      part[warp][g][2 * t + 1] = c[1] + c[3];
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    if (t == 0) ssp[warp][g] = ss;
  }
  __syncthreads();
  if (tid < EB * kRT) {
    const int e = tid / kRT, tl = tid % kRT;
    float sq = 0.f, dot = 0.f;
#pragma unroll
    for (int w = 0; w < kRWarps; ++w) {
      sq += ssp[w][tl];
      dot += part[w][e][tl];
    }
    const float r = 1.0f / sqrtf(sq / static_cast<float>(H) + a.eps);
    if (e == 0) rinv[tl] = r;
    if (e < ne && tl < nt)
      a.logits[static_cast<size_t>(t0 + tl) * E + e0 + e] = dot * r + (a.bias ? a.bias[e0 + e] : 0.f);
  }
  // ---- the last slice of this token block takes the top-k.  The barrier orders every
  // thread's logits before the elected thread's atomic, whose acq_rel also acquires the
  // other slices' logits for the last one; the pre norms are written while it is in flight.
  __syncthreads();
  unsigned old = 0;
  if (tid == 0) old = atom_add_acq_rel_gpu(a.counters + blockIdx.x, 1u);
  // ---- the slice's share of the pre norms of both branches
  for (int j = tid; j < npairs; j += kRThreads) {
    const int c = cb + j % nc, tl = j / nc;
    float f[8], gm[8], gd[8], o1[8], o2[8];
    unpack8(*reinterpret_cast<const uint4*>(xs + tl * RS + c * 8), f);
    unpack8(j == tid ? gm0 : __ldg(reinterpret_cast<const uint4*>(a.gm) + c), gm);
    unpack8(j == tid ? gd0 : __ldg(reinterpret_cast<const uint4*>(a.gd) + c), gd);
    const float r = rinv[tl];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float xh = f[i] * r;
      o1[i] = xh * gm[i];
      o2[i] = xh * gd[i];
    }
    reinterpret_cast<uint4*>(a.xn_moe + static_cast<size_t>(t0 + tl) * H)[c] = pack8(o1);
    reinterpret_cast<uint4*>(a.xn_dense + static_cast<size_t>(t0 + tl) * H)[c] = pack8(o2);
  }
  if (tid == 0) {
    flag = old == gridDim.y - 1;
    if (flag) a.counters[blockIdx.x] = 0u;
  }
  __syncthreads();
  if (!flag) return;
  const bool small_sort = a.offsets != nullptr && gridDim.x == 1;  // every pair is here
  if (warp < nt) {
    if (E <= 128)
      topk_one_token<4>(t0 + warp, E, a.k, a.logits, s_pes, a.topk_idx, a.topk_w,
                        small_sort ? s_ids : nullptr);
    else
      topk_one_token<8>(t0 + warp, E, a.k, a.logits, s_pes, a.topk_idx, a.topk_w,
                        small_sort ? s_ids : nullptr);
  }
  if (a.offsets == nullptr) return;
  if (small_sort) {
    __syncthreads();
    sort_small(a.T * a.k, E, s_ids, ps.wcnt, ps.cnt, ps.off, a.offsets, a.sorted_src, a.inv_pos);
    if (a.aperm != nullptr) {
      // the gather of the routed rows, for a batch this small cheaper here than as a launch
      // of its own: the other slices' xn_moe columns were acquired with the counter.  The
      // token of each sorted position goes to shared memory first, then every thread
      // requests all of its chunks before storing any (one round trip).
      const int n = a.T * a.k, nch = H >> 3;
      __syncthreads();  // sorted_src is written
      if (tid < n) s_tok[tid] = __ldcg(a.sorted_src + tid) / a.k;
      __syncthreads();
      constexpr int U = 6;
      for (int i0 = tid; i0 < n * nch; i0 += kRThreads * U) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = i0 + u * kRThreads;
          if (i < n * nch) {
            const int q = i / nch, c = i - q * nch;
            v[u] = __ldcg(reinterpret_cast<const uint4*>(a.xn_moe + static_cast<size_t>(s_tok[q]) * H) + c);
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = i0 + u * kRThreads;
          if (i < n * nch) {
            const int q = i / nch, c = i - q * nch;
            reinterpret_cast<uint4*>(a.aperm + static_cast<size_t>(q) * H)[c] =
                a.aperm_f16 ? bf16x8_to_f16x8(v[u]) : v[u];
          }
        }
      }
    }
    return;
  }

  // ---- the last token block sorts every (token, slot) pair by expert
  __syncthreads();
  if (tid == 0) {
    const unsigned old = atom_add_acq_rel_gpu(a.counters + gridDim.x, 1u);
    flag = old == gridDim.x - 1;
    if (flag) a.counters[gridDim.x] = 0u;
  }
  __syncthreads();
  if (!flag) return;
  permute_block<kRThreads>(a.T * a.k, E, a.topk_idx, a.offsets, a.sorted_src, a.inv_pos, ps);
}

// Dynamic shared memory of a CTA with EB experts.
static size_t router_smem(int H, int EB) { return static_cast<size_t>(kRT + EB + 1) * (H + 16) * 2; }

// Experts per CTA: about one CTA per SM (token blocks x expert slices), within the
// shared-memory budget.
static int router_eb(int T, int H, int E) {
  const int tb = (T + kRT - 1) / kRT;
  int eb = 1;
  while (eb < kRMaxEB && tb * ((E + eb - 1) / eb) > 160) eb *= 2;
  while (eb > 1 && router_smem(H, eb) > 176 * 1024) eb /= 2;
  return eb;
}

template <int EB>
static cudaError_t launch_eb(const RouterArgs& a, cudaStream_t s, bool pdl) {
  const size_t smem = router_smem(a.H, EB);
  cudaError_t e = cudaFuncSetAttribute(router_kernel<EB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((a.T + kRT - 1) / kRT, (a.E + EB - 1) / EB);
  return launch_k(router_kernel<EB>, grid, dim3(kRThreads), smem, s, pdl, a);
}

int router_counters(int T) { return (T + kRT - 1) / kRT + 1; }

cudaError_t launch_router(int T, int H, int E, int k, float eps, const uint16_t* x,
                          const uint16_t* router_scale, const uint16_t* w_router,
                          const float* bias, const uint16_t* per_expert_scale,
                          const uint16_t* g_pre_moe, const uint16_t* g_pre_dense,
                          uint16_t* xn_moe, uint16_t* xn_dense, float* logits, int* topk_idx,
                          float* topk_w, unsigned* counters, unsigned* status, int* offsets,
                          int* sorted_src, int* inv_pos, uint16_t* aperm, bool aperm_f16,
                          cudaStream_t s, bool pdl) {
  if (aperm != nullptr && (offsets == nullptr || T > kRT)) return cudaErrorInvalidValue;
  RouterArgs a{T, H, E, k, eps, 1.0f / sqrtf(static_cast<float>(H)), x, router_scale, w_router,
               bias, per_expert_scale, g_pre_moe, g_pre_dense, xn_moe, xn_dense, logits,
               topk_idx, topk_w, counters, status, offsets, sorted_src, inv_pos, aperm,
               aperm_f16 ? 1 : 0};
  switch (router_eb(T, H, E)) {
    case 1: return launch_eb<1>(a, s, pdl);
    case 2: return launch_eb<2>(a, s, pdl);
    case 4: return launch_eb<4>(a, s, pdl);
    default: return launch_eb<8>(a, s, pdl);
  }
}

}  // namespace moe
