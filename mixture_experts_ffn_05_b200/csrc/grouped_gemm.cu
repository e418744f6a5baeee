// Persistent grouped GEMM on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// Used for both halves of every expert MLP and of the shared dense MLP:
//   gate_up (kind 0): h[pos][i] = gelu_tanh(g) * u, g/u = xn[pos] . W_gate_up[e][i or I+i]
//   down    (kind 1): Y[pos][o] = h[pos] . W_down[e][o]   (fp16, bf16 or fp32)
// pos is the token row in sorted (expert-major) order; the routing weights are applied
// where the slots of a token are summed (combine.cu).  (ONNX export card, "Truthful graph
// contracts", "Mixture of Experts" and "MoE topology" rows; Inferentia2 card, "How it
// works": expert outputs weighted by the routing weight.)
//
// Orientation: the weights are the M operand (128 rows per tile, streamed once from
// HBM by TMA), the tokens of one expert are the N operand (BN columns).  A decode
// batch puts a handful of tokens on each expert, so N is small and the kernel is a
// weight stream; a prefill batch fills N up to 256.  A gate_up tile holds 64 features as
// 8 gate rows, the 8 matching up rows, the next 8 gate rows, ... (one 5-D TMA box), so
// the gate and up rows of a feature are 8 TMEM lanes apart.
//
// Work list: for each problem (experts, then the optional dense MLP), for each group,
// for each M tile (PAIR: pair of M tiles), for each N tile of BN tokens, `split` pieces
// along K.  Narrow tiles deal pieces round-robin to the persistent grid (one CTA per
// SM); wide single-CTA tiles take them from a global counter.  When split > 1 each piece
// stores its fp32 partial tile; the last piece to arrive (an atomic counter) sums all
// partials in piece order, so the result does not depend on arrival order or schedule.
//
// Warp roles (320 threads; 448 with the int8 converters): warp 0 issues TMA loads into a
// ring of shared-memory stages, warp 1 issues every tcgen05.mma of the CTA into one of
// 1-4 TMEM accumulators, and two groups of four warps (2-5 and 6-9) read the
// accumulator back (tcgen05.ld) and run the epilogue while later
// pieces are being multiplied (wide tiles: both groups, alternate column chunks; BN = 16:
// alternate pieces).  Operand kinds per problem: bf16 (kind::f16); E4M3 codes with a
// scale per weight row and per token row (kind::f8f6f4, the FP8-dynamic variant of the
// "Gemma 4 26B-A4B IT" recipe page); int8 weights with per-channel scales (the int8 build
// of the Inferentia2 card), which warps 10-13 convert to fp16 in tensor memory, exactly,
// for MMAs that take A from TMEM.  Row scales multiply the fp32 accumulator in the
// epilogue (they factor out of the K sum).  Every wait is bounded; a wait that runs out
// records a timeout in the status word and the CTA winds down.
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kMaxSplit = 4;       // K pieces per tile at most
constexpr int kMaxEntries = 258;   // groups of problem 0 (<= 256) + problem 1 (1) + 1
constexpr int kConvWarp0 = 10;     // first converter warp of the int8 variant
constexpr int kConvWarps = 4;      // converter warps, 32 rows of the 128-row tile each

// W8 = false: the A tile (weights, bf16) goes from HBM to shared memory by TMA, already
//   in the 128-byte-swizzled K-major layout the MMA reads.
// PAIR = true (bf16 only, wide token tiles): clusters of two CTAs run M = 256 MMAs
//   (cta_group::2).  A work item covers two neighbouring M tiles, one per CTA, and
//   both CTAs load half of the item's token rows, so each CTA streams 16 KB of
//   weights and 16 KB of tokens per 64-wide K step for a 128 x 256 share of the
//   product (instead of 16 + 32 KB alone): a third less shared-memory fill traffic per
//   FLOP, which is what bounds the wide tiles.
// W8 = true: TMA lands the A tile of an int8 problem as 128 rows of 128 codes (128-byte
//   swizzled); four converter warps turn each row into fp16 in registers and store it in
//   tensor memory, from which the MMA reads its A operand (tcgen05.mma with A in TMEM),
//   so the converted tile never passes through shared memory.  A bf16 problem in the same
//   launch (the dense MLP) is read by the MMA from shared memory as usual.  The int8 row
//   scales are applied in the epilogue.
template <int BN, bool W8, bool PAIR>
struct Cfg {
  static_assert(!(W8 && PAIR), "CTA pairs take bf16 weights only");
  static constexpr int kThreads = W8 ? 448 : 320;  // producer, MMA, 2x4 epilogue (+4 converters)
  static constexpr int kABytes = 128 * 64 * 2;     // bf16 A tile: 128 weight rows x 64 K
  static constexpr int kBRows = PAIR ? BN / 2 : BN;  // token rows in this CTA's B tile
  static constexpr int kBBytes = kBRows * 64 * 2;
  // W8 stages hold a raw A tile of 16 KB (int8 codes for 128 K, or bf16 for 64 K) and
  // up to two B tiles (an int8 step covers two 64-wide MMA sub-steps).
  static constexpr int kBSlots = W8 ? 2 : 1;
  static constexpr int kStage = kABytes + kBSlots * kBBytes;
  static constexpr int kStages = PAIR ? (BN <= 128 ? 8 : 6)
                                : W8 ? (BN <= 32 ? 8 : (BN <= 64 ? 6 : (BN <= 128 ? 4 : 2)))
                                     : (BN <= 32 ? 8 : (BN <= 64 ? 7 : (BN <= 128 ? 6 : 4)));
  // W8: TMEM buffers for converted A tiles, 64 columns (128 K of fp16 pairs) each
  static constexpr int kConv = W8 ? 4 : 0;
  // W8 with at least kConv ring stages: TMEM buffer j % kConv serves k-step j, and it is
  // free once stage (j - kConv) % kStages has been released (its MMAs done), so the
  // converters wait on that stage's empty barrier and the MMA warp commits once per
  // k-step.  With fewer stages than buffers (BN = 256) a phase of that barrier could be
  // passed twice before the wait, so that variant keeps a barrier of its own per buffer.
  static constexpr bool kMergedRelease = W8 && kStages >= kConv;
  // TMEM accumulators: 4 for narrow tiles (the epilogue of a weight-streaming piece is
  // latency-bound and must not hold up the MMAs), 2 for wide ones (512 columns max, less
  // the converted A buffers of the W8 variant).
  static constexpr int kAcc = BN <= 64 ? 4 : (W8 && BN >= 256 ? 1 : 2);
  // BN >= 32: both epilogue groups drain every tile, each taking alternate 16-column
  // chunks, so an accumulator is released in half the time (such launches never split
  // K); BN = 16: the groups take alternate pieces
  static constexpr bool kColSplit = BN >= 32;
  static constexpr int kTaCol = kAcc * BN;  // first TMEM column of the A buffers
  static constexpr int kTmemCols =
      W8 ? 512 : (kAcc * BN < 32 ? 32 : kAcc * BN);
  static_assert(kTaCol + kConv * 64 <= kTmemCols, "tensor memory");
  // after the stages: barriers, bookkeeping, the output staging buffers
  static constexpr int kBarOff = kStages * kStage;
  // Single CTAs with wide tiles take their pieces from a global counter (the fastest SMs
  // take more, which shortens the tail of long pieces); the producer passes them to the
  // other roles through a queue of kQ slots.  Narrow (weight-streaming) tiles keep the
  // round-robin deal, which measured faster for their short pieces.
  static constexpr bool kDyn = !PAIR && BN >= 64;
  static constexpr int kQ = 8;
  static constexpr int kQConsumers = 1 + 2 + (W8 ? kConvWarps : 0);  // MMA, 2 groups, converters
  static constexpr int kNumBars = 2 * kStages + 2 * kConv + 2 * kAcc + 1 + 2 * kQ;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  // tmem slot, abort, bcast x2, group piece broadcast 2 x 2, queue slots
  static constexpr int kMiscInts = 8 + kQ;
  static constexpr int kPreOff = kMiscOff + kMiscInts * 4;
  static constexpr int kTabInts = 4 * kMaxEntries;  // pre, cnt, b0, ng
  // output staging (transposes a warp's slice of the tile so that each lane stores 16 or
  // 32 contiguous bytes): two 1 KB buffers per epilogue warp (one where two do not fit
  // next to the pipeline)
  static constexpr int kStgBytes = 1024;
  static constexpr int kStgOff = ((kPreOff + kTabInts * 4) + 127) & ~127;
  static constexpr int kStgBufs = (kStgOff + 8 * 2 * kStgBytes + 1024 <= 232448) ? 2 : 1;
  static constexpr int kSmem = kStgOff + 8 * kStgBufs * kStgBytes + 1024;  // + alignment slack
  static_assert(kStage % 1024 == 0, "stages must keep 1024-byte alignment");
  static_assert(kSmem <= 232448, "shared memory");
};

// ---- int8 -> fp16 in the converter warps (int8 expert problems take fp16 operands).
// For a code q in [-127, 127], the fp16 number whose exponent is that of 1024 and whose
// low mantissa bits hold the byte q + 128 is 1024 + q + 128 (fp16 has 10 mantissa bits),
// and subtracting 1152 in fp16 leaves q exactly (exponent-bias construction).  One byte
// permute builds two such halves from a word of biased codes; one fp16x2 subtraction
// finishes both.  sel 0x5140 takes codes 0 and 1 of the word, 0x5342 codes 2 and 3.
__device__ __forceinline__ uint32_t i8x2_to_f16x2(uint32_t biased_word, uint32_t sel) {
  const uint32_t h = __byte_perm(biased_word, 0x64646464u, sel);
  uint32_t r;
  asm("sub.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(0x64806480u));
  return r;
}

// A converter warp owns 32 rows of the tile.  Its lanes read the warp's slice of the raw
// tile contiguously (16 bytes per lane per step, conflict-free), so a lane converts a
// piece of a row; the converted rows keep the 128-byte swizzle of the MMA operand:
// 16-byte chunk c of row r at chunk position c ^ (r % 8) (1024-byte-aligned sub-tile).
//   int8 raw rows are 128 codes (two 64-wide sub-tiles): step j, lane l -> row
//     4j + l/8, codes 16*(l%8)..+15 -> sub-tile (l%8)/4, chunks 2*(l%4) and 2*(l%4)+1.
//   bf16 raw rows are 64 values (one sub-tile): step j, lane l -> row 4j + l/8, chunk l%8.
// A converter warp owns 32 rows of the tile, one per lane (its TMEM lane quarter).  A
// lane reads its row's 128 codes from the swizzled tile (chunk c of row r at chunk
// position c ^ (r % 8): the 32 lanes of a load hit 8 distinct positions), converts them
// to 64 fp16 pairs and stores them in 64 consecutive TMEM columns of its lane: column j
// holds codes 2j (low half) and 2j+1, the layout of an M x K fp16 A operand in TMEM.
__device__ __forceinline__ void convert_row_i8_to_tmem(const uint8_t* raw, int r,
                                                       uint32_t taddr) {
#pragma unroll
  for (int h = 0; h < 4; ++h) {  // 32 codes -> 16 columns at a time
    uint32_t o[16];
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int c = 2 * h + cc;
      const uint4 q = *reinterpret_cast<const uint4*>(raw + r * 128 + ((c ^ (r & 7)) << 4));
      const uint32_t w[4] = {q.x ^ 0x80808080u, q.y ^ 0x80808080u, q.z ^ 0x80808080u,
                             q.w ^ 0x80808080u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        o[8 * cc + 2 * i] = i8x2_to_f16x2(w[i], 0x5140u);
        o[8 * cc + 2 * i + 1] = i8x2_to_f16x2(w[i], 0x5342u);
      }
    }
    tmem_st16(taddr + 16 * h, o);
  }
}

struct Piece {
  int p, g, m, n, s;
  int k0, k1;
  int b_row0, n_valid;
  int first_piece;
};

__device__ __forceinline__ int find_entry(const int* pre, int nent, int piece) {
  int lo = 0, hi = nent - 1;  // largest i with pre[i] <= piece
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= piece) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// With PAIR, pc.m numbers pairs of M tiles.
template <int BN>
__device__ __forceinline__ Piece decode_piece(int piece, const GemmParams& P, const int* pre,
                                              const int* b0, const int* ng, int nent) {
  Piece pc;
  const int i = find_entry(pre, nent, piece);
  const int G0 = P.prob[0].groups;
  pc.p = i < G0 ? 0 : 1;
  pc.g = i < G0 ? i : i - G0;
  const GemmProblem& pr = P.prob[pc.p];
  const int ntl = (ng[i] + BN - 1) / BN;
  const int local = piece - pre[i];
  pc.s = local % pr.split;
  const int tl = local / pr.split;
  pc.n = tl % ntl;
  pc.m = tl / ntl;
  pc.k0 = pc.s * pr.k_steps / pr.split;
  pc.k1 = (pc.s + 1) * pr.k_steps / pr.split;
  pc.b_row0 = b0[i];
  pc.n_valid = min(BN, ng[i] - pc.n * BN);
  pc.first_piece = piece - pc.s;
  return pc;
}

// Transposed staging tiles of one epilogue warp (16-bit values, 16 token columns).
// gate_up: [16 tokens][16 features], 32 bytes a token; down: [16 tokens][32 features],
// 64 bytes a token.  The 16-byte chunks of a token are rotated by its index so that the
// eight rows that one stmatrix matrix writes, and eight lanes' 16-byte reads, fall on
// distinct banks.
__device__ __forceinline__ uint32_t stg_glu_off(int tok, int chunk) {
  return static_cast<uint32_t>(tok * 32 + ((chunk ^ ((tok >> 2) & 1)) << 4));
}
__device__ __forceinline__ uint32_t stg_dn_off(int tok, int chunk) {
  return static_cast<uint32_t>(tok * 64 + ((chunk ^ ((tok >> 1) & 3)) << 4));
}
__device__ __forceinline__ uint32_t pack16(float lo, float hi, int mode) {
  // mode 0: bf16, 1: fp16, 2: fp16 saturating at +-65504
  const uint16_t a = mode == 0 ? bf16_bits(lo) : (mode == 1 ? f16_bits(lo) : f16_bits_sat(lo));
  const uint16_t b = mode == 0 ? bf16_bits(hi) : (mode == 1 ? f16_bits(hi) : f16_bits_sat(hi));
  return static_cast<uint32_t>(a) | (static_cast<uint32_t>(b) << 16);
}

template <int BN, bool W8, bool PAIR>
__global__ void __launch_bounds__((Cfg<BN, W8, PAIR>::kThreads), 1)
    grouped_gemm_kernel(const __grid_constant__ GemmMaps maps, const GemmParams P) {
  using C = Cfg<BN, W8, PAIR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + C::kStages;
  uint64_t* conv_full = empty + C::kStages;  // converted A tile in TMEM buffer i is ready
  uint64_t* conv_empty = conv_full + C::kConv;
  uint64_t* acc_full = conv_empty + C::kConv;
  uint64_t* acc_empty = acc_full + C::kAcc;
  uint64_t* drain = acc_empty + C::kAcc;
  uint64_t* q_full = drain + 1;
  uint64_t* q_empty = q_full + C::kQ;
  int* misc = reinterpret_cast<int*>(smem + C::kMiscOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 0);
  volatile int* abort_flag = misc + 1;
  volatile int* bcast = misc + 2;        // [2], one per epilogue group
  volatile int* gpiece = misc + 4;       // [2][2]: each group's piece ids, by parity
  volatile int* q_piece = misc + 8;      // [kQ]
  int* pre = reinterpret_cast<int*>(smem + C::kPreOff);
  int* cnt = pre + kMaxEntries;
  int* b0 = cnt + kMaxEntries;
  int* ng = b0 + kMaxEntries;
  uint8_t* stg_all = smem + C::kStgOff;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nent = P.prob[0].groups + (P.nprob > 1 ? P.prob[1].groups : 0);
  // work items: one per CTA, or (PAIR) one per cluster of two, dealt round-robin
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int first_item = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int item_stride = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  // ---- setup: barriers, TMEM, the piece table
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full[i], 1);
      // W8: the stage is free once the MMA (B) and every converter warp (raw A) are done
      mbar_init(&empty[i], W8 ? 1 + kConvWarps : 1);
    }
    for (int i = 0; i < C::kConv; ++i) {
      mbar_init(&conv_full[i], kConvWarps);
      mbar_init(&conv_empty[i], 1);
    }
    for (int i = 0; i < C::kAcc; ++i) {
      mbar_init(&acc_full[i], 1);
      // every epilogue thread that drains the buffer arrives; PAIR: both CTAs' (leader's)
      mbar_init(&acc_empty[i], (PAIR ? 2 : 1) * (C::kColSplit ? 256 : 128));
    }
    mbar_init(drain, 1);
    for (int i = 0; i < C::kQ; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], C::kQConsumers);
    }
    mbar_fence_init();
    *abort_flag = 0;
    tma_prefetch_map(&maps.a[0]);
    tma_prefetch_map(&maps.b[0]);
    if (P.nprob > 1) {
      tma_prefetch_map(&maps.a[1]);
      tma_prefetch_map(&maps.b[1]);
    }
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(tmem_slot, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::kTmemCols);
      tmem_relinquish();
    }
  }
  // the peer's barriers are initialised before either CTA signals the other
  if (PAIR) cluster_sync();
  // Everything up to the producer's first token-tile load overlaps the previous kernel
  // on the stream.  The routing tables read here (offsets) come from kernels that
  // completed before that kernel started; only the token tiles (gathered rows, h) are
  // its own results, and the producer loads them after the dependency wait.
  pdl_trigger();
  for (int i = threadIdx.x; i < nent; i += C::kThreads) {
    const int p = i < P.prob[0].groups ? 0 : 1;
    const int g = p == 0 ? i : i - P.prob[0].groups;
    const GemmProblem& pr = P.prob[p];
    int s0, n;
    if (pr.offsets) {
      // Segments are clamped to [0, b_rows) so a bad offsets table cannot move any
      // access out of the B operand or the outputs.
      const int brows = pr.n_tokens;
      int a = pr.offsets[g], b = pr.offsets[g + 1];
      a = max(0, min(a, brows));
      b = max(a, min(b, brows));
      s0 = a;
      n = b - a;
    } else {
      s0 = 0;
      n = pr.n_tokens;
    }
    b0[i] = s0;
    ng[i] = n;
    const int m_items = PAIR ? (pr.m_tiles + 1) / 2 : pr.m_tiles;
    cnt[i] = m_items * ((n + BN - 1) / BN) * pr.split;
  }
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < nent; base += 32) {
      const int i = base + lane;
      const int v = i < nent ? cnt[i] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (i < nent) pre[i] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) pre[nent] = carry;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = pre[nent];
  const uint64_t tmo = P.timeout_ns;

  // The piece queue (kDyn): the producer pushes each piece it takes, then -1; every
  // consumer role pops the same sequence (one elected thread per role).
  auto q_push = [&](int n_pushed, int v) -> bool {
    const int slot = n_pushed % C::kQ;
    if (n_pushed >= C::kQ &&
        !mbar_wait(&q_empty[slot], static_cast<uint32_t>((n_pushed / C::kQ) - 1) & 1u, tmo,
                   abort_flag))
      return false;
    q_piece[slot] = v;
    mbar_arrive(&q_full[slot]);
    return true;
  };
  auto q_pop = [&](int n_popped, int* v) -> bool {
    const int slot = n_popped % C::kQ;
    if (!mbar_wait(&q_full[slot], static_cast<uint32_t>(n_popped / C::kQ) & 1u, tmo, abort_flag))
      return false;
    *v = q_piece[slot];
    mbar_arrive(&q_empty[slot]);
    return true;
  };

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();  // weights: read once
      const uint64_t pol_b = policy_evict_last();   // tokens: reused by every M tile
      int stage = 0;
      uint32_t phase = 0;
      int armed[C::kStages];
      for (int i = 0; i < C::kStages; ++i) armed[i] = -1;
      bool ok = true;
      // Weight tiles are never written by an earlier kernel, so the first ring fill of
      // them is issued before the dependency wait; the token-tile loads of those stages
      // are held here and issued after it.
      bool waited = false;
      int nd = 0, steps = 0;
      uint8_t* d_dst[2 * C::kStages];
      const CUtensorMap* d_map[2 * C::kStages];
      int d_c0[2 * C::kStages], d_c1[2 * C::kStages];
      uint64_t* d_bar[2 * C::kStages];
      auto load_b = [&](uint8_t* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
        if (waited) {
          if (PAIR)
            tma_load_2d_pair(dst, map, cluster_addr(bar, 0), c0, c1, pol_b);
          else
            tma_load_2d(dst, map, bar, c0, c1, pol_b);
        } else {
          d_dst[nd] = dst; d_map[nd] = map; d_c0[nd] = c0; d_c1[nd] = c1; d_bar[nd] = bar;
          ++nd;
        }
      };
      auto release_b = [&]() {
        pdl_wait();
        waited = true;
        for (int i = 0; i < nd; ++i) load_b(d_dst[i], d_map[i], d_c0[i], d_c1[i], d_bar[i]);
        nd = 0;
      };
      int n_pushed = 0;
      int piece = C::kDyn ? static_cast<int>(atomicAdd(P.sched, 1u)) : first_item;
      for (; piece < total && ok;) {
        // the next piece is taken one ahead, so the atomic's latency hides behind loads
        const int next = C::kDyn ? static_cast<int>(atomicAdd(P.sched, 1u)) : piece + item_stride;
        if (C::kDyn && !q_push(n_pushed++, piece)) {
          ok = false;
          break;
        }
        const Piece pc = decode_piece<BN>(piece, P, pre, b0, ng, nent);
        const GemmProblem& pr = P.prob[pc.p];
        const CUtensorMap* ma = &maps.a[pr.map];
        const CUtensorMap* mb = &maps.b[pr.map];
        // this CTA's M tile; PAIR: the second tile of an odd count lies past the group's
        // rows (zero-filled for gate_up, another group's rows for down: never stored)
        const int mt = PAIR ? 2 * pc.m + static_cast<int>(rank) : pc.m;
        const int arow = pc.g * pr.w_rows_per_group + mt * 128;  // down only
        // PAIR: the leader loads the first half of the item's (16-rounded) token columns,
        // the other CTA the second half
        const int half = ((pc.n_valid + 15) & ~15) >> 1;
        const int brow = pc.b_row0 + pc.n * BN + (PAIR ? static_cast<int>(rank) * half : 0);
        // a step covers 64 K (bf16), 128 K of int8 codes (two fp16 B sub-tiles) or 128 K of
        // E4M3 codes (one B tile of 128-byte rows); the A tile is 16 KB in every case
        const bool i8p = W8 && pr.w8;
        const int kw = (i8p || pr.fp8) ? 128 : 64;
        const int nb = i8p ? 2 : 1;
        for (int ks = pc.k0; ks < pc.k1; ++ks) {
          if (!waited && steps == C::kStages) release_b();  // the ring is full
          if (!mbar_wait(&empty[stage], phase ^ 1u, tmo, abort_flag)) {
            ok = false;
            break;
          }
          ++steps;
          uint8_t* sa = smem + stage * C::kStage;
          if (PAIR) {
            // both CTAs' bytes land on the leader's barrier; the leader expects them all
            const uint32_t fb = cluster_addr(&full[stage], 0);
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * (C::kABytes + C::kBBytes));
            if (pr.kind == 0)
              tma_load_5d_pair(sa, ma, fb, ks * kw, 0, 0, mt * 8, pc.g, pol_w);
            else
              tma_load_2d_pair(sa, ma, fb, ks * kw, arow, pol_w);
            load_b(sa + C::kABytes, mb, ks * kw, brow, &full[stage]);
          } else {
            mbar_arrive_expect_tx(&full[stage], C::kABytes + nb * C::kBBytes);
            if (pr.kind == 0)  // 8 gate rows, the 8 matching up rows, ... (one 5-D box)
              tma_load_5d(sa, ma, &full[stage], ks * kw, 0, 0, pc.m * 8, pc.g, pol_w);
            else
              tma_load_2d(sa, ma, &full[stage], ks * kw, arow, pol_w);
            for (int b = 0; b < nb; ++b)
              load_b(sa + C::kABytes + b * C::kBBytes, mb, ks * kw + 64 * b, brow, &full[stage]);
          }
          armed[stage] = static_cast<int>(phase);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        piece = next;
      }
      if (C::kDyn && ok && !q_push(n_pushed++, -1)) ok = false;  // end of the sequence
      if (!waited) release_b();  // fewer steps than stages, or a wait that gave up
      if (!ok) {
        record_status(P.status, kStatusTimeout);
        *abort_flag = 1;
        // Let every copy already issued land before the CTA winds down (PAIR: the
        // leader's barriers count both CTAs' copies).
        if (!PAIR || leader)
          for (int i = 0; i < C::kStages; ++i)
            if (armed[i] >= 0) mbar_wait(&full[i], static_cast<uint32_t>(armed[i]), tmo, nullptr);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer (PAIR: the leader's, for both CTAs) =================
    if (lane == 0 && (!PAIR || leader)) {
      int stage = 0;
      uint32_t phase = 0;
      int cs = 0;
      uint32_t cph = 0;
      uint32_t kj = 0;      // k-steps issued so far (kMergedRelease: buffer kj % kConv)
      uint32_t cphm = 0;    // kMergedRelease: bit b = uses of buffer b so far, mod 2
      int ab = 0;
      uint32_t aph = 0;
      bool ok = true, issued = false;
      // PAIR: stage and accumulator releases go to the barriers of both CTAs
      const uint32_t peer_empty0 = PAIR ? cluster_addr(&empty[0], 1) : 0u;
      const uint32_t peer_acc0 = PAIR ? cluster_addr(&acc_full[0], 1) : 0u;
      int n_popped = 0;
      for (int piece = first_item; ok; piece += item_stride) {
        if (C::kDyn && !q_pop(n_popped++, &piece)) {
          ok = false;
          break;
        }
        if (piece < 0 || piece >= total) break;
        const Piece pc = decode_piece<BN>(piece, P, pre, b0, ng, nent);
        const int ncol = (pc.n_valid + 15) & ~15;
        // E4M3 operands take the A/B format code 0, as fp16 does under kind::f16
        const bool f8 = P.prob[pc.p].fp8 != 0;
        const uint32_t idesc = (P.prob[pc.p].f16 || f8) ? idesc_f16_f32(PAIR ? 256 : 128, ncol)
                                                        : idesc_bf16_f32(PAIR ? 256 : 128, ncol);
        if (!mbar_wait(&acc_empty[ab], aph ^ 1u, tmo, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(ab * BN);
        // int8 problems (W8): A comes from the TMEM buffer the converters filled
        const bool a_tmem = W8 && P.prob[pc.p].w8;
        // The k-step loop exists once per operand kind (bf16/fp16 from shared memory, E4M3
        // from shared memory, int8-as-fp16 from TMEM), chosen per piece: this thread issues
        // every MMA of the CTA, and a branch per MMA measured 25% at decode.
        auto k_loop = [&](auto kind_tag) {
          constexpr int kKind = decltype(kind_tag)::value;  // 0 f16 kinds, 1 E4M3, 2 TMEM A
          for (int ks = pc.k0; ks < pc.k1; ++ks, ++kj) {
            if (C::kMergedRelease) cs = static_cast<int>(kj % C::kConv);
            const uint32_t cpar = C::kMergedRelease ? (cphm >> cs) & 1u : cph;
            if (!mbar_wait(&full[stage], phase, tmo, abort_flag) ||
                (kKind == 2 && !mbar_wait(&conv_full[cs], cpar, tmo, abort_flag))) {
              ok = false;
              return;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + stage * C::kStage);
            if constexpr (kKind == 2) {
              // a 128-K step: two 64-wide sub-steps; A sub-step `sub`, K slice kk sits in
              // TMEM columns [32 sub + 8 kk, +8) of the buffer
              const uint32_t ta = tmem_base + static_cast<uint32_t>(C::kTaCol + cs * 64);
              for (int sub = 0; sub < 2; ++sub) {
                const uint64_t bd = sdesc_k_sw128(sa + C::kABytes + sub * C::kBBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  umma_ta(d, ta + 32 * sub + 8 * kk, bd + 2 * kk, idesc,
                          (ks > pc.k0 || sub > 0 || kk > 0) ? 1u : 0u);
              }
              if (C::kMergedRelease) {
                cphm ^= 1u << cs;  // the stage's release below also frees the buffer
              } else {
                umma_commit(&conv_empty[cs]);
                if (++cs == C::kConv) {
                  cs = 0;
                  cph ^= 1u;
                }
              }
            } else {
              const uint64_t ad = sdesc_k_sw128(sa);
              const uint64_t bd = sdesc_k_sw128(sa + C::kABytes);
              // four MMAs per 128-byte row: K = 16 bf16 or K = 32 E4M3 each
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t acc = (ks > pc.k0 || kk > 0) ? 1u : 0u;
                if constexpr (kKind == 1) {
                  if (PAIR)
                    umma_f8_pair(d, ad + 2 * kk, bd + 2 * kk, idesc, acc);
                  else
                    umma_f8(d, ad + 2 * kk, bd + 2 * kk, idesc, acc);
                } else {
                  if (PAIR)
                    umma_bf16_pair(d, ad + 2 * kk, bd + 2 * kk, idesc, acc);
                  else
                    umma_bf16(d, ad + 2 * kk, bd + 2 * kk, idesc, acc);
                }
              }
            }
            if (PAIR) {
              umma_commit_pair(smem_u32(&empty[stage]));
              umma_commit_pair(peer_empty0 + stage * 8);
            } else {
              umma_commit(&empty[stage]);
            }
            issued = true;
            if (++stage == C::kStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
        };
        if (W8 && a_tmem)
          k_loop(std::integral_constant<int, 2>{});
        else if (f8)
          k_loop(std::integral_constant<int, 1>{});
        else
          k_loop(std::integral_constant<int, 0>{});
        if (!ok) break;
        if (PAIR) {
          umma_commit_pair(smem_u32(&acc_full[ab]));
          umma_commit_pair(peer_acc0 + ab * 8);
        } else {
          umma_commit(&acc_full[ab]);
        }
        if (++ab == C::kAcc) {
          ab = 0;
          aph ^= 1u;
        }
      }
      if (!ok) {
        record_status(P.status, kStatusTimeout);
        *abort_flag = 1;
        if (issued) {  // wait for the MMAs in flight before TMEM is released
          if (PAIR)
            umma_commit_pair(smem_u32(drain));
          else
            umma_commit(drain);
          mbar_wait(drain, 0, tmo, nullptr);
        }
      }
    }
  } else if (W8 && warp >= kConvWarp0) {
    // ================= converters (W8): int8 A tile -> fp16 in TMEM ==================
    // Each warp owns 32 rows of the tile (one per lane, its TMEM lane quarter) and runs on
    // its own: an elected lane waits for the stage (and, for an int8 problem, a free TMEM
    // buffer), the warp converts and stores, and lane 0 arrives for the warp.  Stages of
    // a bf16 problem need no conversion: the warp only takes part in releasing them.
    int stage = 0;
    uint32_t phase = 0;
    int cs = 0;
    uint32_t cph = 0;
    uint32_t kj = 0;  // k-steps seen so far, in the MMA warp's order
    bool ok = true;
    int n_popped = 0;
    for (int piece = first_item; ok; piece += item_stride) {
      if (C::kDyn) {
        int v = -2;
        if (lane == 0 && !q_pop(n_popped, &v)) v = -2;
        ++n_popped;
        piece = __shfl_sync(0xffffffffu, v, 0);
        if (piece == -2) {
          ok = false;
          break;
        }
      }
      if (piece < 0 || piece >= total) break;
      const Piece pc = decode_piece<BN>(piece, P, pre, b0, ng, nent);
      const bool i8 = P.prob[pc.p].w8 != 0;
      const int q = warp & 3;  // TMEM lane quarter
      for (int ks = pc.k0; ks < pc.k1; ++ks, ++kj) {
        if (C::kMergedRelease) cs = static_cast<int>(kj % C::kConv);
        int good = 1;
        if (lane == 0) {
          bool free_buf = true;
          if (i8) {
            if (C::kMergedRelease) {
              // the MMAs of k-step kj - kConv, the buffer's last user, are done once that
              // step's stage has been released
              if (kj >= static_cast<uint32_t>(C::kConv)) {
                const uint32_t jp = kj - C::kConv;
                free_buf = mbar_wait(&empty[jp % C::kStages], (jp / C::kStages) & 1u, tmo,
                                     abort_flag);
              }
            } else {
              free_buf = mbar_wait(&conv_empty[cs], cph ^ 1u, tmo, abort_flag);
            }
          }
          good = (mbar_wait(&full[stage], phase, tmo, abort_flag) && free_buf) ? 1 : 0;
        }
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) {
          ok = false;
          break;
        }
        if (i8) {
          tc_fence_after();
          const uint8_t* raw = smem + stage * C::kStage;
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                 static_cast<uint32_t>(C::kTaCol + cs * 64);
          convert_row_i8_to_tmem(raw, q * 32 + lane, taddr);
          tmem_st_wait();
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) {
          if (i8) mbar_arrive(&conv_full[cs]);
          mbar_arrive(&empty[stage]);
        }
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
        if (!C::kMergedRelease && i8 && ++cs == C::kConv) {
          cs = 0;
          cph ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      record_status(P.status, kStatusTimeout);
      *abort_flag = 1;
    }
  } else {
    // ================= epilogue: two groups of 4 warps ==================================
    // Warp w reads TMEM lanes 32*(w%4)..+31; each group covers all 128 lanes.  The groups
    // take alternate 16-column chunks of every tile (kColSplit) or, at BN = 16, alternate
    // pieces, which keeps the latency-bound part of a split-K epilogue (partials,
    // counters) off the MMA's path.
    // Each warp then writes its own slice of the output tile: it stages the values in its
    // shared-memory buffers, transposed, so that every lane stores 16 or 32 contiguous
    // bytes of an output row (a warp store covers 512 bytes).
    //   gate_up: lanes l and l^8 hold the gate and up row of one feature (the A tile is
    //     8 gate rows, the matching 8 up rows, ...); a shuffle pairs them, the gate lane
    //     finishes columns 0-7 of each 16 and the up lane columns 8-15.  Warp q covers
    //     features 16q..16q+15 of the tile's 64.
    //   down: lane l holds output row 32q + l of the tile's 128.
    // Output rows are the tile's B rows (sorted order); columns past the tile's valid
    // count are not stored.
    const int grp = (warp - 2) >> 2;
    const int q = warp & 3;
    const int et = threadIdx.x - 64 - 128 * grp;
    const uint32_t bar = 1 + grp;
    volatile int* gb = bcast + grp;
    uint8_t* stg = stg_all + (warp - 2) * C::kStgBufs * C::kStgBytes;
    int nstg = 0;  // staging buffers used by this warp so far
    int local = 0;
    for (int piece = first_item;; piece += item_stride, ++local) {
      if (C::kDyn) {
        // the group's elected thread pops; the slot alternates by parity, so it is not
        // rewritten before every thread of the group has read it
        volatile int* slot = gpiece + 2 * grp + (local & 1);
        if (et == 0) {
          int v = -2;
          *slot = q_pop(local, &v) ? v : -2;
        }
        named_sync(bar, 128);
        piece = *slot;
        if (piece == -2) {
          if (et == 0) {
            record_status(P.status, kStatusTimeout);
            *abort_flag = 1;
          }
          break;
        }
      }
      if (piece < 0 || piece >= total) break;
      if (!C::kColSplit && (local & 1) != grp) continue;
      const int ab = local % C::kAcc;
      const uint32_t aph = static_cast<uint32_t>(local / C::kAcc) & 1u;
      const Piece pc = decode_piece<BN>(piece, P, pre, b0, ng, nent);
      const GemmProblem& pr = P.prob[pc.p];
      if (et == 0) *gb = mbar_wait(&acc_full[ab], aph, tmo, abort_flag) ? 1 : 0;
      named_sync(bar, 128);
      if (!*gb) {
        if (et == 0) {
          record_status(P.status, kStatusTimeout);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(ab * BN);
      const int row = q * 32 + lane;  // accumulator row = TMEM lane
      const int ncols = (pc.n_valid + 15) & ~15;
      const int mt = PAIR ? 2 * pc.m + static_cast<int>(rank) : pc.m;  // this CTA's M tile
      bool last = mt < pr.m_tiles;  // PAIR: the second tile of an odd count is not stored
      if (pr.split > 1) {  // (never with PAIR)
        float* part = P.partials + static_cast<size_t>(piece) * BN * 128;
        for (int c0 = 0; c0 < ncols; c0 += 16) {
          float v[16];
          tmem_ld16(tbase + c0, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) __stcg(part + (c0 + i) * 128 + row, v[i]);
        }
        // Publish with one release: the barrier orders every thread's partial before the
        // elected thread's atomic, whose acq_rel also acquires the other pieces' partials.
        named_sync(bar, 128);
        if (et == 0) {
          const unsigned old = atom_add_acq_rel_gpu(P.counters + pc.first_piece, 1u);
          const int l = (old == static_cast<unsigned>(pr.split - 1)) ? 1 : 0;
          if (l) P.counters[pc.first_piece] = 0u;  // ready for the next launch
          *gb = l;
        }
        named_sync(bar, 128);
        last = *gb != 0;
      }
      if (last && pr.split == 1 && (pr.kind == 0 || pr.out_type != kOutF32)) {
        // 16-bit outputs of a whole-K tile: the accumulator is read 16 rows x 16 columns at
        // a time (tcgen05.ld 16x256b: thread t holds rows t/4 and t/4+8 of each 16, columns
        // 2(t%4)..+1 of each 8), which is stmatrix's fragment layout; stmatrix.trans writes
        // it to shared memory as [token][features] and each lane stores 16 contiguous bytes
        const int pos0 = pc.b_row0 + pc.n * BN;  // output row of column 0
        const int fq = lane >> 2;
        float sc[4] = {1.f, 1.f, 1.f, 1.f};  // [16-row half][row t/4, row t/4 + 8]
        if (pr.wscale) {
          const float* wsr = pr.wscale + static_cast<size_t>(pc.g) * pr.w_rows_per_group;
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              // gate_up: rows 16h+fq (gate) and 16h+fq+8 (up) of warp q are feature
              // 8(2q+h)+fq of the tile's 64; down: rows are output features
              const int wr = pr.kind == 0 ? mt * 64 + 8 * (2 * q + h) + fq + (u ? pr.nw : 0)
                                          : mt * 128 + 32 * q + 16 * h + 8 * u + fq;
              sc[2 * h + u] = wsr[wr];
            }
        }
        const int mode = pr.kind == 0 ? (pr.f16 ? 1 : 0) : (pr.out_type == kOutF16 ? 2 : 0);
        const int mi = lane >> 3;  // the stmatrix matrix this lane addresses, row lane % 8
        const float* xsc = pr.xscale ? pr.xscale + pos0 : nullptr;  // fp8: per column
        for (int c0 = C::kColSplit ? 16 * grp : 0; c0 < ncols; c0 += C::kColSplit ? 32 : 16) {
          uint32_t r[8], s[8];
          tmem_ld_16x256b_x2(tbase + c0, r);
          tmem_ld_16x256b_x2(tbase + (16u << 16) + c0, s);
          tmem_ld_wait_16(r, s);
          float a[2][8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            a[0][i] = __uint_as_float(r[i]) * sc[(i >> 1) & 1];
            a[1][i] = __uint_as_float(s[i]) * sc[2 + ((i >> 1) & 1)];
          }
          if (xsc != nullptr) {
            // this thread's columns: 2m, 2m+1, 8+2m, 9+2m of the chunk (m = lane % 4)
            float xs[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int col = c0 + 8 * (j >> 1) + 2 * (lane & 3) + (j & 1);
              xs[j] = col < pc.n_valid ? __ldg(xsc + col) : 0.f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              a[0][i] *= xs[((i >> 2) << 1) | (i & 1)];
              a[1][i] *= xs[((i >> 2) << 1) | (i & 1)];
            }
          }
          uint8_t* buf = stg + (nstg % C::kStgBufs) * C::kStgBytes;
          ++nstg;
          __syncwarp();  // this buffer's reads of an earlier chunk are done
          const uint32_t sb = smem_u32(buf);
          if (pr.kind == 0) {
            // a[h][4j], a[h][4j+1]: gate of feature 8h+fq at columns 8j+2(t%4), +1;
            // a[h][4j+2], a[h][4j+3]: up of the same feature and columns.  Matrix 2h+j:
            // features 8h.. x columns 8j..
            uint32_t m4[4];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int j = 0; j < 2; ++j)
                m4[2 * h + j] = pack16(gelu_tanh(a[h][4 * j]) * a[h][4 * j + 2],
                                       gelu_tanh(a[h][4 * j + 1]) * a[h][4 * j + 3], mode);
            stmatrix_x4_trans(sb + stg_glu_off((lane & 7) + 8 * (mi & 1), mi >> 1), m4[0], m4[1],
                              m4[2], m4[3]);
            __syncwarp();
            const int tok = lane >> 1, ch = lane & 1;
            if (c0 + tok < pc.n_valid) {
              const uint4 val = *reinterpret_cast<const uint4*>(buf + stg_glu_off(tok, ch));
              *reinterpret_cast<uint4*>(static_cast<uint16_t*>(pr.out) +
                                        static_cast<size_t>(pos0 + c0 + tok) * pr.out_ld +
                                        mt * 64 + 16 * q + 8 * ch) = val;
            }
          } else {
            // half h, matrix i: rows 16h + 8(i&1).. x columns 8(i>>1)..
            const int tok_w = (lane & 7) + 8 * (mi >> 1);
#pragma unroll
            for (int h = 0; h < 2; ++h)
              stmatrix_x4_trans(sb + stg_dn_off(tok_w, 2 * h + (mi & 1)),
                                pack16(a[h][0], a[h][1], mode), pack16(a[h][2], a[h][3], mode),
                                pack16(a[h][4], a[h][5], mode), pack16(a[h][6], a[h][7], mode));
            __syncwarp();
#pragma unroll
            for (int rnd = 0; rnd < 2; ++rnd) {
              const int tok = 8 * rnd + (lane >> 2), g = lane & 3;
              if (c0 + tok < pc.n_valid) {
                const uint4 val = *reinterpret_cast<const uint4*>(buf + stg_dn_off(tok, g));
                *reinterpret_cast<uint4*>(static_cast<uint16_t*>(pr.out) +
                                          static_cast<size_t>(pos0 + c0 + tok) * pr.out_ld +
                                          mt * 128 + 32 * q + 8 * g) = val;
              }
            }
          }
        }
      } else if (last) {
        const int pos0 = pc.b_row0 + pc.n * BN;  // output row of column 0
        float sc = 1.f;
        if (pr.wscale) {
          // gate_up row r of the tile: feature 8*(r/16) + r%8 of its 64, gate or up by bit 3
          const int wr = pr.kind == 0
                             ? mt * 64 + 8 * (row >> 4) + (row & 7) + ((row & 8) ? pr.nw : 0)
                             : mt * 128 + row;
          sc = pr.wscale[static_cast<size_t>(pc.g) * pr.w_rows_per_group + wr];
        }
        for (int c0 = C::kColSplit ? 16 * grp : 0; c0 < ncols; c0 += C::kColSplit ? 32 : 16) {
          float v[16];
          tmem_ld16(tbase + c0, v);
          if (pr.split > 1) {
            // every other piece's partial is loaded first, then all are summed in piece
            // order (the same order whichever piece arrives last)
            float pv[kMaxSplit][16];
#pragma unroll
            for (int s2 = 0; s2 < kMaxSplit; ++s2) {
              if (s2 < pr.split && s2 != pc.s) {
                const float* qp = P.partials + static_cast<size_t>(pc.first_piece + s2) * BN * 128;
#pragma unroll
                for (int i = 0; i < 16; ++i) pv[s2][i] = __ldcg(qp + (c0 + i) * 128 + row);
              }
            }
            float acc[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < kMaxSplit; ++s2) {
              if (s2 < pr.split) {
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i] += (s2 == pc.s) ? v[i] : pv[s2][i];
              }
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = acc[i];
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] *= sc;
          if (pr.xscale != nullptr) {  // fp8: the B rows' (tokens') scales, per column
#pragma unroll
            for (int i = 0; i < 16; ++i)
              v[i] *= c0 + i < pc.n_valid ? __ldg(pr.xscale + pos0 + c0 + i) : 0.f;
          }
          if (pr.kind == 0) {
            // pair gate and up, 8 columns per lane
            const bool up = (lane & 8) != 0;
            float h[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float mine = up ? v[8 + i] : v[i];          // gate: cols 0-7, up: 8-15
              const float give = up ? v[i] : v[8 + i];          // what the partner needs
              const float other = __shfl_xor_sync(0xffffffffu, give, 8);
              h[i] = up ? gelu_tanh(other) * mine : gelu_tanh(mine) * other;
            }
            uint8_t* buf = stg + (nstg % C::kStgBufs) * C::kStgBytes;
            ++nstg;
            __syncwarp();  // the buffer's last reads (two chunks ago) are done
            // [16 columns][16 features] bf16, then one 16-byte store per lane: lane l
            // writes features 8*(l&1)..+7 of column l/2
            uint16_t* b16 = reinterpret_cast<uint16_t*>(buf);
            const int f = 8 * (lane >> 4) + (lane & 7);
            const int cb = up ? 8 : 0;
#pragma unroll
            for (int i = 0; i < 8; ++i)
              b16[(cb + i) * 16 + f] = pr.f16 ? f16_bits(h[i]) : bf16_bits(h[i]);
            __syncwarp();
            const int fx = mt * 64 + 16 * q;  // first output feature of this warp
            const int c = lane >> 1;
            if (c0 + c < pc.n_valid) {
              const uint4 val = *reinterpret_cast<const uint4*>(b16 + c * 16 + 8 * (lane & 1));
              *reinterpret_cast<uint4*>(static_cast<uint16_t*>(pr.out) +
                                        static_cast<size_t>(pos0 + c0 + c) * pr.out_ld + fx +
                                        8 * (lane & 1)) = val;
            }
          } else {
            // two halves of 8 columns: [8 columns][32 rows] fp32 or bf16, then lane l
            // writes rows 8*(l&3)..+7 of column l/4
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              uint8_t* buf = stg + (nstg % C::kStgBufs) * C::kStgBytes;
              ++nstg;
              __syncwarp();
              if (pr.out_type == kOutF32) {
                float* bf = reinterpret_cast<float*>(buf);
#pragma unroll
                for (int i = 0; i < 8; ++i) bf[i * 32 + lane] = v[8 * hh + i];
              } else {
                uint16_t* bh = reinterpret_cast<uint16_t*>(buf);
                if (pr.out_type == kOutF16) {
#pragma unroll
                  for (int i = 0; i < 8; ++i) bh[i * 32 + lane] = f16_bits_sat(v[8 * hh + i]);
                } else {
#pragma unroll
                  for (int i = 0; i < 8; ++i) bh[i * 32 + lane] = bf16_bits(v[8 * hh + i]);
                }
              }
              __syncwarp();
              const int cc = c0 + 8 * hh;
              const int fx = mt * 128 + 32 * q;
              const int c = lane >> 2, g = lane & 3;
              if (cc + c < pc.n_valid) {
                const size_t o = static_cast<size_t>(pos0 + cc + c) * pr.out_ld + fx + 8 * g;
                if (pr.out_type == kOutF32) {
                  const float4* src = reinterpret_cast<const float4*>(buf) + c * 8 + 2 * g;
                  float4* dst = reinterpret_cast<float4*>(static_cast<float*>(pr.out) + o);
                  dst[0] = src[0];
                  dst[1] = src[1];
                } else {
                  *reinterpret_cast<uint4*>(static_cast<uint16_t*>(pr.out) + o) =
                      *(reinterpret_cast<const uint4*>(buf) + c * 4 + g);
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      named_sync(bar, 128);  // every flag of this piece is read before the next is written
      if (PAIR)
        mbar_arrive_cluster(cluster_addr(&acc_empty[ab], 0));  // the leader's MMA waits
      else
        mbar_arrive(&acc_empty[ab]);
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (C::kDyn && threadIdx.x == 0) {
    // the last CTA to finish returns the piece counter to zero for the next launch
    __threadfence();
    if (atomicAdd(P.sched + 1, 1u) == gridDim.x - 1) {
      P.sched[0] = 0u;
      P.sched[1] = 0u;
      __threadfence();
    }
  }
  // PAIR: neither CTA releases TMEM or exits while its peer may still signal it or read
  // its shared memory
  if (PAIR) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if (PAIR)
      tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else
      tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <int BN, bool W8, bool PAIR>
static cudaError_t launch_bn(const GemmMaps& maps, const GemmParams& p, int grid, cudaStream_t s,
                             bool pdl) {
  using C = Cfg<BN, W8, PAIR>;
  auto kernel = grouped_gemm_kernel<BN, W8, PAIR>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  if (!PAIR) return launch_k(kernel, dim3(grid), dim3(C::kThreads), C::kSmem, s, pdl, maps, p);
  // clusters of two CTAs (an even grid), optionally a programmatic dependent launch
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid & ~1);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, maps, p);
}

template <bool W8>
static cudaError_t launch_w(int bn, const GemmMaps& maps, const GemmParams& p, int grid,
                            cudaStream_t s, bool pdl) {
  switch (bn) {
    case 16: return launch_bn<16, W8, false>(maps, p, grid, s, pdl);
    case 32: return launch_bn<32, W8, false>(maps, p, grid, s, pdl);
    case 64: return launch_bn<64, W8, false>(maps, p, grid, s, pdl);
    case 128: return launch_bn<128, W8, false>(maps, p, grid, s, pdl);
    case 256: return launch_bn<256, W8, false>(maps, p, grid, s, pdl);
  }
  return cudaErrorInvalidValue;
}

bool gemm_pairs_allowed(int bn, bool int8_weights) { return !int8_weights && bn >= 128; }

cudaError_t launch_grouped_gemm(int bn, const GemmMaps& maps, const GemmParams& p, int grid,
                                cudaStream_t s, bool pdl) {
  // split K only with BN = 16 (wider tiles split their epilogue by columns instead)
  for (int i = 0; i < p.nprob; ++i)
    if (bn != 16 && p.prob[i].split > 1) return cudaErrorInvalidValue;
  if (p.pairs) {
    if (!gemm_pairs_allowed(bn, p.int8_weights != 0)) return cudaErrorInvalidValue;

    if (bn == 128) return launch_bn<128, false, true>(maps, p, grid, s, pdl);
    if (bn == 256) return launch_bn<256, false, true>(maps, p, grid, s, pdl);
    return cudaErrorInvalidValue;
  }
  return p.int8_weights ? launch_w<true>(bn, maps, p, grid, s, pdl)
                        : launch_w<false>(bn, maps, p, grid, s, pdl);
}

}  // namespace moe
