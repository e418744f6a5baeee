// Router of the MoE block for large batches, on the tensor cores.
//
// Computes what router.cu computes (the ONNX export card, "Truthful graph contracts",
// Router row: scale-free RMSNorm -> learned scale x hidden_size^-0.5 -> linear to E
// logits -> softmax (fp32) -> top-k -> renormalise -> per_expert_scale, plus the pre
// norms of both branches), with the logits as a bf16 GEMM on tcgen05.
//
// The logit of token t and expert e is
//     l[t,e] = rinv[t] * sum_h x[t,h] * W'[e,h] + bias[e],   W'[e,h] = s[h] W_r[e,h] / sqrt(H)
// with rinv[t] = 1 / sqrt(mean_h x[t,h]^2 + eps).  x is bf16 and goes to the tensor cores
// as it is.  W' is fp32; a preparation kernel splits it into two bf16 matrices,
// W' = W'hi + W'lo + d with |d| <= 2^-16 |W'|, and the kernel accumulates x.W'hi and
// x.W'lo in fp32 (one MMA of N = 2 ne over both, each into its own accumulator columns,
// added when read), so the logits carry the accuracy of an fp32 dot product (every bf16 x
// bf16 product is exact in fp32).
//
// One CTA per 128 tokens (the 128 TMEM lanes) and slice of the experts (the N dimension:
// all E experts when the batch has enough token tiles to fill the GPU, else E/2, E/4 or
// E/8 of them, so that small batches still spread over most SMs).
// Warp roles:
//   0      TMA producer: per 64-wide K step the x tile and the W'hi, W'lo tiles
//          (phase 1), then the x tiles again, several per ring stage (phase 2);
//   1      MMA issuer (one MMA per 16 K over W'hi and W'lo, two for slices wider than
//          128 experts) and TMEM owner;
//   2..5   sums of x^2 of one token row per thread, read from the x tiles of phase 1;
//          afterwards the top-k of the same row from its TMEM lane (one expert slice),
//          or the row's logits of the slice to global memory (several slices: the last
//          CTA of a token tile to finish then takes the top-k of its 128 tokens, one
//          warp per token);
//   6..13  phase 2: xn_moe = x * rinv * g_pre_moe and xn_dense = x * rinv * g_pre_dense,
//          for the CTA's share of the columns (its slice of the 64-wide K steps).
// Every wait is bounded.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kTcTokens = 128;
constexpr int kTcThreads = 448;
constexpr int kTcMaxStages = 8;
constexpr int kTcSmemBudget = 192 * 1024;
constexpr uint32_t kTcTile = 128 * 128;  // one x tile: 128 rows of 64 bf16
constexpr int kTcWriterThreads = 256;    // warps 6..13
constexpr int kTcMaxE = 256;
// the selection of a several-slice tile stages 128 x (E + 1) logits in the ring, whose
// size is at least the budget less one stage of the widest slice (128 experts)
static_assert(kTcSmemBudget - (static_cast<int>(kTcTile) + 2 * 128 * 128) >=
                  kTcTokens * (kTcMaxE + 1) * 4,
              "ring too small for the logits of a tile");

struct RouterTcArgs {
  int T, H, E, k;
  int ne;               // experts per CTA (a multiple of 16: the MMA N)
  int slices;           // expert slices (gridDim.y); ne * slices >= E
  int stages;           // ring stages
  int stage_bytes;      // x tile + W'hi tile + W'lo tile
  int tiles_per_stage;  // x tiles per stage in phase 2
  float eps;
  const float* bias;
  const uint16_t* pes;
  const uint16_t* gm;
  const uint16_t* gd;
  uint16_t* xn_moe;
  uint16_t* xn_dense;
  int* topk_idx;
  float* topk_w;
  float* logits;       // [T][E], several slices only
  unsigned* counters;  // one per token tile, zero on entry and on exit (several slices)
  unsigned* status;
  uint64_t timeout_ns;
};

// Order-preserving map of a float to an unsigned key; NaN maps to the key of -inf.
// Key 0 is below every float.
__device__ __forceinline__ uint32_t order_key(float l) {
  if (l != l) l = -INFINITY;
  const uint32_t u = __float_as_uint(l);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Top-k of one token's logits, fed in ascending expert order: a strictly larger key
// enters the sorted list, so among equal logits the lower expert id comes first.
template <int KMAX>
struct TopK {
  uint32_t key[KMAX];
  int id[KMAX];

  __device__ __forceinline__ void init() {
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      key[j] = 0u;
      id[j] = 0;
    }
  }

  // The new key's place is the number of kept keys >= it (they are sorted, so those are
  // a prefix); every slot then updates independently of the others, so a push is a few
  // dependent steps and no branch (a shifting insertion is a chain of KMAX steps, and in
  // a warp of 32 rows nearly every push inserts somewhere).
  __device__ __forceinline__ void push(float l, int e) {
    const uint32_t ck = order_key(l);
    int pos = 0;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) pos += key[j] >= ck ? 1 : 0;
#pragma unroll
    for (int j = KMAX - 1; j > 0; --j) {
      key[j] = j < pos ? key[j] : (j == pos ? ck : key[j - 1]);
      id[j] = j < pos ? id[j] : (j == pos ? e : id[j - 1]);
    }
    key[0] = pos > 0 ? key[0] : ck;
    id[0] = pos > 0 ? id[0] : e;
  }

  // softmax restricted to the selected experts (the full denominator cancels in the
  // renormalisation), summed in slot order; then per_expert_scale
  __device__ __forceinline__ void write(int t, int k, const uint16_t* pes, int* topk_idx,
                                        float* topk_w) const {
    const float top = key_value(key[0]);
    float ex[KMAX];
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      ex[j] = 0.f;
      if (j < k) {
        ex[j] = expf(key_value(key[j]) - top);
        sum += ex[j];
      }
    }
    int* oi = topk_idx + static_cast<size_t>(t) * k;
    float* ow = topk_w + static_cast<size_t>(t) * k;
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k) {
        oi[j] = id[j];
        ow[j] = ex[j] / sum * __uint_as_float(static_cast<uint32_t>(pes[id[j]]) << 16);
      }
  }
};

// All lanes wait; the warp continues only if every lane saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns,
                                          const volatile int* abort) {
  const bool ok = mbar_wait(bar, parity, timeout_ns, abort);
  return __all_sync(0xffffffffu, ok);
}

// Top-k of one row of E <= 32 KPL logits in shared memory by one warp (ties to the lower
// expert id): lane i holds experts i, i + 32, ...; each of the k rounds takes the warp
// maximum of the lanes' best remaining 64-bit keys (ordered logit, then the inverted
// expert id), high word first, then the low word among the lanes that share it.  Then
// the weights as TopK::write computes them.
template <int KPL>
__device__ __forceinline__ void topk_row_warp(const float* row, int E, int k, int t,
                                              const uint16_t* pes, int* topk_idx,
                                              float* topk_w) {
  const int lane = threadIdx.x & 31;
  unsigned long long key[KPL];
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < E ? (static_cast<unsigned long long>(order_key(row[e])) << 32) |
                         (0xFFFFFFFFu - static_cast<uint32_t>(e))
                   : 0ull;
  }
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
    if (key[0] == best) {
#pragma unroll
      for (int i = 0; i + 1 < KPL; ++i) key[i] = key[i + 1];
      key[KPL - 1] = 0ull;
    }
    if (lane == j) mine = best;
  }
  const float top = key_value(static_cast<uint32_t>(__shfl_sync(0xffffffffu, mine, 0) >> 32));
  const int my_e = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(mine));
  const float ex = lane < k ? expf(key_value(static_cast<uint32_t>(mine >> 32)) - top) : 0.f;
  float sum = 0.f;  // in slot order
  for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, ex, j);
  if (lane < k) {
    topk_idx[static_cast<size_t>(t) * k + lane] = my_e;
    topk_w[static_cast<size_t>(t) * k + lane] =
        ex / sum * __uint_as_float(static_cast<uint32_t>(pes[my_e]) << 16);
  }
}

template <int KMAX>
__global__ void __launch_bounds__(kTcThreads, 1)
    router_tc_kernel(const __grid_constant__ RouterTcMaps maps, const RouterTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t full[kTcMaxStages];
  __shared__ __align__(8) uint64_t empty1[kTcMaxStages];  // phase-1 releases: MMA + 4 row warps
  __shared__ __align__(8) uint64_t empty2[kTcMaxStages];  // phase-2 releases: 8 writer warps
  __shared__ __align__(8) uint64_t acc_full;
  __shared__ __align__(8) uint64_t drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int s_abort;
  __shared__ float s_rinv[kTcTokens];
  __shared__ int s_last;
  __shared__ float s_bias[kTcMaxE];
  __shared__ uint16_t s_pes[kTcMaxE];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kTcTokens;
  const int e0 = blockIdx.y * a.ne;  // first expert of this CTA's slice
  const int KS = a.H / 64;
  const int S = a.stages;
  // phase 2 covers this slice's share of the K steps
  const int ks0 = static_cast<int>(blockIdx.y) * KS / a.slices;
  const int ks1 = static_cast<int>(blockIdx.y + 1) * KS / a.slices;
  const int J2 = (ks1 - ks0 + a.tiles_per_stage - 1) / a.tiles_per_stage;
  const uint32_t b_bytes = static_cast<uint32_t>(a.ne) * 128u;
  // W'hi and W'lo rows sit back to back in a stage, so with 2 ne <= 256 one MMA of N = 2 ne
  // multiplies both: accumulator columns [0, ne) hold x.W'hi, [ne, 2 ne) x.W'lo (two
  // independent sums, added when read).  Wider slices take two MMAs into one accumulator.
  const bool merged = 2 * a.ne <= 256;
  const int acc_cols = merged ? 2 * a.ne : a.ne;
  const uint32_t tmem_cols = acc_cols <= 32 ? 32u : acc_cols <= 64 ? 64u : acc_cols <= 128 ? 128u : 256u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty1[s], 5);
      mbar_init(&empty2[s], kTcWriterThreads / 32);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&drain, 1);
    s_abort = 0;
    mbar_fence_init();
  }
  // caller inputs (not written by the preparation kernel): read before the dependency wait
  for (int e = threadIdx.x; e < a.E; e += kTcThreads) {
    s_pes[e] = a.pes[e];
    s_bias[e] = a.bias ? a.bias[e] : 0.f;
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&maps.x);
    tma_prefetch_map(&maps.whi);
    tma_prefetch_map(&maps.wlo);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t keep = policy_evict_last();  // x is read twice, W' by every CTA
      bool ok = true;
      int issued = 0;
      pdl_wait();  // W'hi and W'lo come from the preparation kernel
      for (int j = 0; j < KS + J2; ++j) {
        const int s = j % S;
        if (j >= S) {
          const int jp = j - S;  // the previous job on this stage
          if (jp < KS) {
            ok = mbar_wait(&empty1[s], (jp / S) & 1, a.timeout_ns, &s_abort);
          } else {
            const int first2 = KS + ((s - KS % S) + S) % S;  // first phase-2 job on stage s
            ok = mbar_wait(&empty2[s], ((jp - first2) / S) & 1, a.timeout_ns, &s_abort);
          }
          if (!ok) break;
        }
        uint8_t* st = ring + static_cast<size_t>(s) * a.stage_bytes;
        if (j < KS) {
          mbar_arrive_expect_tx(&full[s], kTcTile + 2 * b_bytes);
          tma_load_2d(st, &maps.x, &full[s], j * 64, t0, keep);
          tma_load_2d(st + kTcTile, &maps.whi, &full[s], j * 64, e0, keep);
          tma_load_2d(st + kTcTile + b_bytes, &maps.wlo, &full[s], j * 64, e0, keep);
        } else {
          const int q0 = ks0 + (j - KS) * a.tiles_per_stage;
          const int nt = min(a.tiles_per_stage, ks1 - q0);
          mbar_arrive_expect_tx(&full[s], nt * kTcTile);
          for (int i = 0; i < nt; ++i)
            tma_load_2d(st + i * kTcTile, &maps.x, &full[s], (q0 + i) * 64, t0, keep);
        }
        issued = j + 1;
      }
      if (!ok) {
        record_status(a.status, kStatusTimeout);
        s_abort = 1;
        // let the copies already issued land before the CTA can exit
        for (int j = max(0, issued - S); j < issued; ++j)
          mbar_wait(&full[j % S], (j / S) & 1, a.timeout_ns, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, acc_cols);
      bool ok = true;
      int done = 0;
      for (int j = 0; j < KS; ++j) {
        const int s = j % S;
        if (!mbar_wait(&full[s], (j / S) & 1, a.timeout_ns, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(ring + static_cast<size_t>(s) * a.stage_bytes);
        // one 32-byte K slice per MMA: descriptors advance by 2 (16-byte units)
        const uint64_t ad = sdesc_k_sw128(sa);
        const uint64_t bh = sdesc_k_sw128(sa + kTcTile);
        if (merged) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) umma_bf16(tmem, ad + 2 * kk, bh + 2 * kk, idesc, (j | kk) != 0);
        } else {
          const uint64_t bl = sdesc_k_sw128(sa + kTcTile + b_bytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            umma_bf16(tmem, ad + 2 * kk, bh + 2 * kk, idesc, (j | kk) != 0);
            umma_bf16(tmem, ad + 2 * kk, bl + 2 * kk, idesc, 1u);
          }
        }
        umma_commit(&empty1[s]);
        done = j + 1;
      }
      if (ok) {
        umma_commit(&acc_full);
      } else {
        record_status(a.status, kStatusTimeout);
        s_abort = 1;
        if (done > 0) {  // the MMAs already issued finish before TMEM is released
          umma_commit(&drain);
          mbar_wait(&drain, 0, a.timeout_ns, nullptr);
        }
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ token rows
    const int q = warp & 3;  // TMEM lane quarter of this warp
    const int r = q * 32 + lane;
    // a thread sums a whole row: 8-term partial sums in fp32, accumulated in fp64, so
    // the norm factor is as accurate as the warp-parallel sum of the small-batch router
    double ss = 0.0;
    bool ok = true;
    for (int j = 0; j < KS; ++j) {
      const int s = j % S;
      if (!warp_wait(&full[s], (j / S) & 1, a.timeout_ns, &s_abort)) {
        ok = false;
        break;
      }
      const uint8_t* row = ring + static_cast<size_t>(s) * a.stage_bytes + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float f[8];
        unpack8(*reinterpret_cast<const uint4*>(row + ((c ^ (r & 7)) << 4)), f);
        float p = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) p = fmaf(f[i], f[i], p);
        ss += static_cast<double>(p);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty1[s]);
    }
    const float rinv = static_cast<float>(1.0 / sqrt(ss / a.H + static_cast<double>(a.eps)));
    s_rinv[r] = rinv;
    named_sync(1, 32 * 12);  // warps 2..13: the norm factors are in shared memory
    if (ok) ok = warp_wait(&acc_full, 0, a.timeout_ns, &s_abort);
    if (!ok) {
      if (lane == 0) {
        record_status(a.status, kStatusTimeout);
        s_abort = 1;
      }
    } else {
      tc_fence_after();
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
      const int t = t0 + r;
      if (a.slices == 1) {
        TopK<KMAX> tk;
        tk.init();
        for (int c = 0; c < a.ne; c += 16) {
          float v[16];
          tmem_ld16(lane_base + c, v);
          if (merged) {
            float w[16];
            tmem_ld16(lane_base + a.ne + c, w);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] += w[i];
          }
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c + i < a.E) tk.push(v[i] * rinv + s_bias[c + i], c + i);
        }
        if (t < a.T) tk.write(t, a.k, s_pes, a.topk_idx, a.topk_w);
      } else {
        // the slice's logits to global memory; the last CTA of the tile selects
        for (int c = 0; c < a.ne; c += 16) {
          float v[16];
          tmem_ld16(lane_base + c, v);
          if (merged) {
            float w[16];
            tmem_ld16(lane_base + a.ne + c, w);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] += w[i];
          }
          if (t < a.T) {
            float* lr = a.logits + static_cast<size_t>(t) * a.E + e0 + c;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (e0 + c + i < a.E) lr[i] = v[i] * rinv + s_bias[e0 + c + i];
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ pre-norm writers
    named_sync(1, 32 * 12);
    const int wt = threadIdx.x - 6 * 32;
    const uint4* gm = reinterpret_cast<const uint4*>(a.gm);
    const uint4* gd = reinterpret_cast<const uint4*>(a.gd);
    for (int j = KS; j < KS + J2; ++j) {
      const int s = j % S;
      if (!warp_wait(&full[s], (j / S) & 1, a.timeout_ns, &s_abort)) {
        if (lane == 0) {
          record_status(a.status, kStatusTimeout);
          s_abort = 1;
        }
        break;
      }
      const uint8_t* st = ring + static_cast<size_t>(s) * a.stage_bytes;
      const int q0 = ks0 + (j - KS) * a.tiles_per_stage;
      const int nt = min(a.tiles_per_stage, ks1 - q0);
      for (int i = 0; i < nt; ++i) {
        const uint8_t* tile = st + i * kTcTile;
        const int cb = (q0 + i) * 8;  // first 8-wide chunk of this tile's columns
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int idx = wt + kTcWriterThreads * u;
          const int r = idx >> 3, c = idx & 7;
          const int t = t0 + r;
          const uint4 v = *reinterpret_cast<const uint4*>(tile + r * 128 + ((c ^ (r & 7)) << 4));
          if (t < a.T) {
            const float rv = s_rinv[r];
            float f[8], g1[8], g2[8], o1[8], o2[8];
            unpack8(v, f);
            unpack8(__ldg(gm + cb + c), g1);
            unpack8(__ldg(gd + cb + c), g2);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float xh = f[e] * rv;
              o1[e] = xh * g1[e];
              o2[e] = xh * g2[e];
            }
            reinterpret_cast<uint4*>(a.xn_moe + static_cast<size_t>(t) * a.H)[cb + c] = pack8(o1);
            reinterpret_cast<uint4*>(a.xn_dense + static_cast<size_t>(t) * a.H)[cb + c] = pack8(o2);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty2[s]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
  if (a.slices == 1) return;

  // ---- several slices: the last CTA of this token tile to finish takes the top-k
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned old = atomicAdd(a.counters + blockIdx.x, 1u);
    s_last = old == gridDim.y - 1;
    if (s_last) {
      a.counters[blockIdx.x] = 0u;
      __threadfence();
    }
  }
  __syncthreads();
  if (!s_last) return;
  // The tile's logits go through shared memory (the ring is free now): coalesced loads by
  // the whole CTA, rows padded to E + 1 floats so that the row-per-thread reads of the
  // selection hit distinct banks.  (Read straight from global memory, each thread's
  // row-wise loads made every warp request touch 32 rows; the selection took ~30 us.)
  // With several slices a stage holds at least 144 KB of the 192 KB ring, more than
  // the 128 x 257 floats of E = 256.
  const int rows = min(kTcTokens, a.T - t0);
  const int ld = a.E + 1;
  float* sl = reinterpret_cast<float*>(ring);
  const float* src = a.logits + static_cast<size_t>(t0) * a.E;
  const int n = rows * a.E;
  if ((a.E & 3) == 0) {  // 16-byte loads (a row starts on a 16-byte boundary)
    const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll 8
    for (int i = threadIdx.x; i < n / 4; i += kTcThreads) {
      const float4 v = __ldcg(s4 + i);
      float* d = sl + (4 * i / a.E) * ld + (4 * i) % a.E;
      d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
    }
  } else {
#pragma unroll 8
    for (int i = threadIdx.x; i < n; i += kTcThreads) sl[(i / a.E) * ld + i % a.E] = __ldcg(src + i);
  }
  __syncthreads();
  // one warp per row (a thread per row took ~15 us for the 128 rows of a tile)
  for (int r = warp; r < rows; r += kTcThreads / 32) {
    if (a.E <= 128)
      topk_row_warp<4>(sl + r * ld, a.E, a.k, t0 + r, s_pes, a.topk_idx, a.topk_w);
    else
      topk_row_warp<8>(sl + r * ld, a.E, a.k, t0 + r, s_pes, a.topk_idx, a.topk_w);
  }
}

// W'hi, W'lo = the two-term bf16 split of s[h] * W_r[e,h] / sqrt(H); one thread per 8.
__global__ void __launch_bounds__(256) router_prep_kernel(int E, int H, float inv_sqrt_h,
                                                          const uint16_t* __restrict__ w,
                                                          const uint16_t* __restrict__ scale,
                                                          uint16_t* __restrict__ whi,
                                                          uint16_t* __restrict__ wlo) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const int nch = H >> 3;
  if (i >= static_cast<int64_t>(E) * nch) return;
  const int c = static_cast<int>(i % nch);
  float f[8], sc[8], hi[8], lo[8];
  unpack8(__ldg(reinterpret_cast<const uint4*>(w) + i), f);
  unpack8(__ldg(reinterpret_cast<const uint4*>(scale) + c), sc);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float v = f[q] * sc[q] * inv_sqrt_h;
    hi[q] = __uint_as_float(static_cast<uint32_t>(bf16_bits(v)) << 16);
    lo[q] = v - hi[q];
  }
  reinterpret_cast<uint4*>(whi)[i] = pack8(hi);
  reinterpret_cast<uint4*>(wlo)[i] = pack8(lo);
}

bool router_uses_tc(int T) { return T > kRouterTcMinT; }

int router_tc_slices(int T, int E) {
  const int tiles = (T + kTcTokens - 1) / kTcTokens;
  const int groups16 = (E + 15) / 16;  // every slice is a multiple of 16 experts
  int sl = 1;
  while (sl < 8 && tiles * sl * 2 <= 148 && groups16 % (sl * 2) == 0) sl *= 2;
  return sl;
}

template <int KMAX>
static cudaError_t launch_tc(const RouterTcMaps& maps, const RouterTcArgs& a, size_t smem,
                             cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(router_tc_kernel<KMAX>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_k(router_tc_kernel<KMAX>,
                  dim3((a.T + kTcTokens - 1) / kTcTokens, a.slices), dim3(kTcThreads), smem, s,
                  true, maps, a);
}

cudaError_t launch_router_tc(const RouterTcMaps& maps, int T, int H, int E, int k, float eps,
                             const uint16_t* w_router, const uint16_t* router_scale,
                             uint16_t* whi, uint16_t* wlo, const float* bias,
                             const uint16_t* per_expert_scale, const uint16_t* g_pre_moe,
                             const uint16_t* g_pre_dense, uint16_t* xn_moe, uint16_t* xn_dense,
                             int* topk_idx, float* topk_w, float* logits, unsigned* counters,
                             unsigned* status, uint64_t timeout_ns, cudaStream_t s, bool pdl) {
  const int64_t nch = static_cast<int64_t>(E) * (H / 8);
  cudaError_t e = launch_k(router_prep_kernel, dim3(static_cast<unsigned>((nch + 255) / 256)),
                           dim3(256), 0, s, pdl, E, H, 1.0f / sqrtf(static_cast<float>(H)),
                           w_router, router_scale, whi, wlo);
  if (e != cudaSuccess) return e;
  RouterTcArgs a{};
  a.T = T; a.H = H; a.E = E; a.k = k;
  a.slices = router_tc_slices(T, E);
  a.ne = (E + 15) / 16 * 16 / a.slices;
  a.stage_bytes = static_cast<int>(kTcTile) + 2 * a.ne * 128;
  a.stages = std::min(kTcMaxStages, kTcSmemBudget / a.stage_bytes);
  a.tiles_per_stage = a.stage_bytes / static_cast<int>(kTcTile);
  a.eps = eps;
  a.bias = bias; a.pes = per_expert_scale; a.gm = g_pre_moe; a.gd = g_pre_dense;
  a.xn_moe = xn_moe; a.xn_dense = xn_dense; a.topk_idx = topk_idx; a.topk_w = topk_w;
  a.logits = logits; a.counters = counters; a.status = status; a.timeout_ns = timeout_ns;
  const size_t smem = static_cast<size_t>(a.stages) * a.stage_bytes + 1024;
  return k <= 8 ? launch_tc<8>(maps, a, smem, s) : launch_tc<16>(maps, a, smem, s);
}

}  // namespace moe
