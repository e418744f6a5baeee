// Weight-streaming grouped GEMM for small batches (decode), with the weights dequantised
// in registers.
//
// Computes the same two launches as the tensor-memory grouped GEMM (grouped_gemm.cu):
//   gate_up (kind 0): h[pos][f] = gelu_tanh(g) * u,  g/u = b[pos] . W[e][f or F+f]
//   down    (kind 1): Y[pos][o] = b[pos] . W[e][o]
// for the routed experts and the shared dense MLP (ONNX export card, "Truthful graph
// contracts", "Mixture of Experts" and "MoE topology" rows).  A decode batch puts one to a
// few tokens on each expert, so the work is a stream of weight bytes with a handful of
// multiply-adds per byte.  With 8-bit or 4-bit weights ("Gemma-4 26B-A4B (MoE, int8
// experts) on AWS Inferentia2", "How it works": per-channel int8; "Gemma 4 26B-A4B IT",
// variant list: NVFP4) the codes must be widened before a tensor-core instruction can use
// them; the tensor-memory kernel does that through shared or tensor memory, a chain of
// waits per k-step.  Here the codes are widened to fp16 in registers and fed to mma.sync
// (m16n8k16, fp32 accumulation), which at decode sizes has tensor throughput to spare.
//
// Work: a tile of 64 weight rows of one group against a chunk of up to 8 nt of its tokens
// (nt n-tiles of 8: groups of many tokens read each weight tile once per wide unit),
// over a range of K (the tile's K is split into pieces when a launch has too few tiles to
// keep every SM streaming; the last piece to finish adds the others' fp32 partial sums in
// piece order, so results do not depend on timing).  Pieces are dealt round-robin.
// Inside a CTA, warp w multiplies tile rows 16w .. 16w + 15 (gate_up: 8 gate rows and the
// 8 matching up rows; down: 16 output rows).
//
// Data movement: every K item (128 bytes of each weight row) is copied by all 128 threads
// with cp.async into a ring of shared-memory stages, eight threads per 128-byte row, so
// each L2 request carries a whole line; the item's token rows (and NVFP4 block scales) come
// with it.  One barrier per item releases the stage.
//
// Operand layout inside a 64-wide K step: lane (g, t) (g = lane / 4, t = lane % 4) takes
// elements [16t, 16t + 16) of its strip's rows g and g + 8 and of token g.  MMA j of the
// step takes elements 16t + 4j + {0, 1} as its K columns (2t, 2t + 1) and 16t + 4j +
// {2, 3} as (2t + 8, 2t + 9): a permutation of K applied to both operands, which leaves
// every dot product unchanged and lets each lane use 16 contiguous elements.
//
// Weight formats (A operand):
//   bf16: as stored; the tokens are bf16 (kind bf16 MMA).
//   int8: codes q with an fp32 scale per row; q becomes fp16 exactly (the exponent-bias
//     construction of the converter warps in grouped_gemm.cu); tokens are fp16 (the
//     gather writes them so); the row scale multiplies the fp32 sum.
//   nvfp4: E2M1 codes, 8 to a 32-bit word (nibbles 0-3: elements 0, 2, 4, 6 of the word's
//     8; nibbles 4-7: elements 1, 3, 5, 7), one E4M3 scale per 16 elements of a row and one
//     fp32 scale per matrix.  A code's three magnitude bits placed as the low exponent bits
//     and the top mantissa bit of an fp16 number give exactly its value times 2^-14 (fp16
//     subnormals and normals line up with E2M1's); times the block scale the product is
//     still exact in fp16 (at most 6 significant bits, a multiple of 2^-24, at most 0.17);
//     2^14 and the matrix scale multiply the fp32 sum.  Tokens are fp16.
#include "common.cuh"
#include "internal.h"
#include "warp_mma.cuh"

namespace moe {

constexpr int kStreamWarps = 4;
constexpr int kStreamThreads = 32 * kStreamWarps;
constexpr int kStreamRows = kStreamTileRows;  // weight rows per tile
constexpr int kStreamMaxEntries = 258;
constexpr int kStreamRingBytes = 40 * 1024;

// ---- operand widening helpers

// Two int8 codes of a word of biased codes (q + 128) -> fp16x2 (see grouped_gemm.cu).
__device__ __forceinline__ uint32_t s_i8x2_f16x2(uint32_t biased, uint32_t sel) {
  const uint32_t h = __byte_perm(biased, 0x64646464u, sel);
  uint32_t r;
  asm("sub.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(0x64806480u));
  return r;
}

// Two E2M1 codes already shifted into bits 12..9 and 28..25 -> fp16x2 of their values
// times 2^-14: the magnitude bits become the exponent's low bits and the mantissa's top
// bit; the sign, left at exponent bit 12, is moved to bit 15 (adding 7 x 2^12 to the
// isolated bit carries it there).
__device__ __forceinline__ uint32_t e2m1x2_f16x2(uint32_t x) {
  x &= 0x1E001E00u;
  return x + 7u * (x & 0x10001000u);
}

// fp16x2 of the E4M3 code in the low byte of v, in both halves (exact).
__device__ __forceinline__ uint32_t e4m3_to_f16x2_both(uint32_t v) {
  uint32_t r;
  const uint16_t two = static_cast<uint16_t>((v & 0xFFu) | ((v & 0xFFu) << 8));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(two));
  return r;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- stage geometry per weight format
// An item is 128 bytes of each of the tile's 64 weight rows: 64 K of bf16, 128 K of int8,
// 256 K of NVFP4.  Stage layout: [64 rows][128 B] weights, [8 tokens][item K x 2 B] token
// rows, NVFP4: [64 rows][16 B] block scales.  16-byte chunks are placed with an XOR of the
// row (token) parity, so that the 16-byte reads of the eight lanes of a phase (rows g and
// g + 1) fall on distinct banks.
template <int WT>
struct Geo;
template <>
struct Geo<kStreamBf16> {
  static constexpr int kSteps = 1;       // 64-wide K steps per item
  static constexpr int kBRow = 128;      // token bytes per item
  static constexpr int kBs = 0;          // block-scale bytes per stage
  static constexpr int kASwz = 1;        // XOR of odd rows' chunk index
};
template <>
struct Geo<kStreamInt8> {
  static constexpr int kSteps = 2;
  static constexpr int kBRow = 256;
  static constexpr int kBs = 0;
  static constexpr int kASwz = 4;
};
template <>
struct Geo<kStreamNvfp4> {
  static constexpr int kSteps = 4;
  static constexpr int kBRow = 512;
  static constexpr int kBs = kStreamRows * 16;
  static constexpr int kASwz = 2;
};
template <int WT, int NT>
struct Stage {
  static constexpr int kA = kStreamRows * 128;
  static constexpr int kB = 8 * NT * Geo<WT>::kBRow;
  static constexpr int kBytes = kA + kB + Geo<WT>::kBs;
  static constexpr int kCount = kStreamRingBytes / kBytes;
  static_assert(kCount >= 3, "ring too small");
};

__device__ __forceinline__ uint32_t a_off(int row, int chunk, int swz) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ ((row & 1) * swz)) << 4));
}
__device__ __forceinline__ uint32_t b_off(int tok, int chunk, int row_bytes) {
  return static_cast<uint32_t>(tok * row_bytes + ((chunk ^ (tok & 1)) << 4));
}

// ---- pieces
struct Piece {
  int p, gg, m, c, s;     // problem, group, tile, token chunk, K piece
  int tok0, n_valid;      // token rows of the chunk
  int it0, it1;           // K items of the piece
  int unit;               // (tile, chunk) index for the split-K counters
  int64_t part0;          // float offset of split 0's partial tile of this unit
};

struct Tables {
  int* pre;   // [nent + 1] first piece of each (problem, group) entry
  int* b0s;   // token segment of each entry
  int* ngs;
  int* upre;  // [nent + 1] first unit of each entry
  int nent, G0;
};

__device__ __forceinline__ int s_find_entry(const int* pre, int nent, int u) {
  int lo = 0, hi = nent - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__host__ __device__ __forceinline__ int stream_items_of(int K, int wtype) {
  const int bytes = wtype == kStreamBf16 ? K * 2 : wtype == kStreamInt8 ? K : K / 2;
  return (bytes + 127) / 128;
}

__device__ __forceinline__ Piece piece_of(int piece, const StreamParams& P, const Tables& tb) {
  Piece pc;
  const int i = s_find_entry(tb.pre, tb.nent, piece);
  pc.p = i < tb.G0 ? 0 : 1;
  pc.gg = pc.p == 0 ? i : i - tb.G0;
  const StreamProblem& pr = P.prob[pc.p];
  const int local = piece - tb.pre[i];
  const int tiles = pr.rows / kStreamRows;
  const int split = pr.split, nc = kStreamChunk * pr.nt;
  pc.s = local % split;
  const int ul = local / split;          // unit within the entry: chunk-major
  pc.m = ul % tiles;
  pc.c = ul / tiles;
  pc.tok0 = tb.b0s[i] + pc.c * nc;
  pc.n_valid = min(nc, tb.ngs[i] - pc.c * nc);
  const int items = stream_items_of(pr.K, pr.wtype);
  pc.it0 = pc.s * items / split;
  pc.it1 = (pc.s + 1) * items / split;
  pc.unit = tb.upre[i] + ul;
  // partial tiles [piece][64][nc] fp32, problem 0's pieces first
  const int first = piece - pc.s;
  const int p0end = tb.pre[tb.G0];
  pc.part0 = pc.p == 0 ? static_cast<int64_t>(first) * kStreamRows * nc
                       : static_cast<int64_t>(p0end) * kStreamRows * kStreamChunk * P.prob[0].nt +
                             static_cast<int64_t>(first - p0end) * kStreamRows * nc;
  return pc;
}

// Weight row of tile row r (0..63): gate_up strips are 8 gate rows and the 8 matching up
// rows of 8 features; down rows are consecutive.
__device__ __forceinline__ int weight_row(const StreamProblem& pr, int m, int r) {
  if (pr.kind != 0) return m * kStreamRows + r;
  const int w = r >> 4, rr = r & 15;
  const int f = m * 32 + 8 * w + (rr & 7);
  return rr < 8 ? f : pr.F + f;
}

// This thread's share of every item copy of one piece, with the addresses worked out once
// per piece: weight chunk c = tid % 8 of tile rows tid / 8 + 16 j (j < 4); NVFP4 block-scale
// word tid % 4 of rows tid / 4 + 32 j (j < 2); token-row chunks q = tid + 128 j.
struct CopyPlan {
  const uint8_t* a[4];   // weight row + chunk offset
  const uint8_t* bs[2];  // nvfp4: block-scale row + word offset
  const uint16_t* b[4];  // token row + chunk offset (NULL past the valid tokens)
  int a_lim;             // bytes of a row: chunk copies stop at it
  int bs_lim;            // nvfp4: block scales per row
  int b_lim;             // elements of a token row
};

template <int WT, int NT>
__device__ __forceinline__ void plan_piece(CopyPlan& cp, const StreamProblem& pr, const Piece& pc) {
  using Gm = Geo<WT>;
  const int tid = threadIdx.x;
  const size_t row_bytes = WT == kStreamBf16 ? static_cast<size_t>(pr.K) * 2
                           : WT == kStreamInt8 ? static_cast<size_t>(pr.K)
                                               : static_cast<size_t>(pr.K) / 2;
  const size_t grow = static_cast<size_t>(pc.gg) * pr.rows;
  const uint8_t* wb = static_cast<const uint8_t*>(pr.w);
  const int c = tid & 7;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    cp.a[j] = wb + (grow + weight_row(pr, pc.m, (tid >> 3) + 16 * j)) * row_bytes + c * 16;
  cp.a_lim = static_cast<int>(row_bytes) - c * 16;  // this thread's chunk exists while it * 128 < a_lim
  if constexpr (WT == kStreamNvfp4) {
    const int nblk = pr.K / 16;
#pragma unroll
    for (int j = 0; j < 2; ++j)
      cp.bs[j] = pr.bscale + (grow + weight_row(pr, pc.m, (tid >> 2) + 32 * j)) * static_cast<size_t>(nblk) +
                 (tid & 3) * 4;
    cp.bs_lim = nblk - (tid & 3) * 4;
  }
  constexpr int kChunks = Gm::kBRow / 16;  // chunks of 8 elements per token row and item
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int q = tid + j * kStreamThreads;
    const int tk = q / kChunks, ch = q % kChunks;
    cp.b[j] = (q < 8 * NT * kChunks && tk < pc.n_valid)
                  ? pr.b + static_cast<size_t>(pc.tok0 + tk) * pr.K + ch * 8
                  : nullptr;
  }
  cp.b_lim = pr.K;
}

// This thread's byte offsets inside a stage, fixed for the whole kernel (worked out once
// so that no swizzle arithmetic runs per item): the chunks it reads for each K step of an
// item (weight rows g and g + 8 of its warp's strip, token g) and the chunks it copies.
template <int WT>
struct Offs {
  uint32_t a[Geo<WT>::kSteps][2][2];  // [step][row g, g + 8][first, second 16-byte chunk]
  uint32_t b[Geo<WT>::kSteps][2];     // token g: the two chunks of a step
  uint32_t bs[2];                     // nvfp4: block-scale bytes of rows g and g + 8 (+ 4h + t)
  uint32_t cpa[4];                    // the 16-byte weight chunks it copies
  uint32_t cpb[4];                    // the 16-byte token chunks it copies
  uint32_t cpbs[2];                   // nvfp4: the block-scale words it copies
};

template <int WT, int NT>
__device__ __forceinline__ Offs<WT> make_offs(int warp, int lane) {
  using Gm = Geo<WT>;
  Offs<WT> o;
  const int g = lane >> 2, t = lane & 3, tid = threadIdx.x;
  const int r0 = 16 * warp + g, r1 = r0 + 8;
#pragma unroll
  for (int h = 0; h < Gm::kSteps; ++h) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = rr ? r1 : r0;
      if constexpr (WT == kStreamBf16) {
        o.a[h][rr][0] = a_off(r, 2 * t, Gm::kASwz);
        o.a[h][rr][1] = a_off(r, 2 * t + 1, Gm::kASwz);
      } else if constexpr (WT == kStreamInt8) {
        o.a[h][rr][0] = o.a[h][rr][1] = a_off(r, 4 * h + t, Gm::kASwz);
      } else {  // 8 bytes: bytes [32h + 8t, +8) of the row
        o.a[h][rr][0] = o.a[h][rr][1] = a_off(r, 2 * h + (t >> 1), Gm::kASwz) + 8 * (t & 1);
      }
    }
    o.b[h][0] = Stage<WT, NT>::kA + b_off(g, 8 * h + 2 * t, Gm::kBRow);
    o.b[h][1] = Stage<WT, NT>::kA + b_off(g, 8 * h + 2 * t + 1, Gm::kBRow);
  }
  o.bs[0] = Stage<WT, NT>::kA + Stage<WT, NT>::kB + r0 * 16 + t;
  o.bs[1] = Stage<WT, NT>::kA + Stage<WT, NT>::kB + r1 * 16 + t;
#pragma unroll
  for (int j = 0; j < 4; ++j) o.cpa[j] = a_off((tid >> 3) + 16 * j, tid & 7, Gm::kASwz);
  constexpr int kChunks = Gm::kBRow / 16;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int q = tid + j * kStreamThreads;
    o.cpb[j] = Stage<WT, NT>::kA + b_off(q / kChunks, q % kChunks, Gm::kBRow);
  }
#pragma unroll
  for (int j = 0; j < 2; ++j)
    o.cpbs[j] = Stage<WT, NT>::kA + Stage<WT, NT>::kB + ((tid >> 2) + 32 * j) * 16 + (tid & 3) * 4;
  return o;
}

// Copies of item `it` of the planned piece into the stage at shared address `st`.
template <int WT, int NT>
__device__ __forceinline__ void issue_item(uint32_t st, const CopyPlan& cp, const Offs<WT>& of,
                                           int it, bool weights, bool tokens) {
  using Gm = Geo<WT>;
  const int tid = threadIdx.x;
  if (weights) {
    const bool ok = it * 128 < cp.a_lim;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      cp_async16(st + of.cpa[j], ok ? cp.a[j] + it * 128 : cp.a[j], ok ? 16u : 0u);
    if constexpr (WT == kStreamNvfp4) {
      const bool okb = it * 16 < cp.bs_lim;
#pragma unroll
      for (int j = 0; j < 2; ++j)
        cp_async4(st + of.cpbs[j], okb ? cp.bs[j] + it * 16 : cp.bs[j], okb ? 4u : 0u);
    }
  }
  if (tokens) {
    constexpr int kChunks = Gm::kBRow / 16;
    const int k0 = it * 64 * Gm::kSteps;
#pragma unroll
    for (int j = 0; j < (8 * NT * kChunks + kStreamThreads - 1) / kStreamThreads; ++j) {
      const int q = tid + j * kStreamThreads;
      if (q < 8 * NT * kChunks) {
        const bool ok = cp.b[j] != nullptr && k0 + (q % kChunks) * 8 < cp.b_lim;
        const void* src = ok ? static_cast<const void*>(cp.b[j] + k0) : static_cast<const void*>(cp.a[0]);
        cp_async16(st + of.cpb[j], src, ok ? 16u : 0u);
      }
    }
  }
}

// The fp16/bf16 pairs of step h of the item: rows g (w[0..7]) and g + 8 (w[8..15]) of the
// warp's strip.
template <int WT>
__device__ __forceinline__ void widen(const uint8_t* st, const Offs<WT>& of, int h,
                                      uint32_t (&w)[16]) {
  if constexpr (WT == kStreamBf16) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const uint4 a = *reinterpret_cast<const uint4*>(st + of.a[h][rr][0]);
      const uint4 b = *reinterpret_cast<const uint4*>(st + of.a[h][rr][1]);
      w[8 * rr + 0] = a.x; w[8 * rr + 1] = a.y; w[8 * rr + 2] = a.z; w[8 * rr + 3] = a.w;
      w[8 * rr + 4] = b.x; w[8 * rr + 5] = b.y; w[8 * rr + 6] = b.z; w[8 * rr + 7] = b.w;
    }
  } else if constexpr (WT == kStreamInt8) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const uint4 v = *reinterpret_cast<const uint4*>(st + of.a[h][rr][0]);
      const uint32_t q[4] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u, v.z ^ 0x80808080u,
                             v.w ^ 0x80808080u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        w[8 * rr + 2 * i] = s_i8x2_f16x2(q[i], 0x5140u);
        w[8 * rr + 2 * i + 1] = s_i8x2_f16x2(q[i], 0x5342u);
      }
    }
  } else {
    // step h: 16 codes of each row, block 4h + t of the item
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const uint2 v = *reinterpret_cast<const uint2*>(st + of.a[h][rr][0]);
      const uint32_t b = e4m3_to_f16x2_both(st[of.bs[rr] + 4 * h]);
      const uint32_t words[2] = {v.x, v.y};
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t x = words[i];
        uint32_t* o = w + 8 * rr + 4 * i;
        o[0] = hmul2_u32(e2m1x2_f16x2(x << 9), b);
        o[1] = hmul2_u32(e2m1x2_f16x2(x << 5), b);
        o[2] = hmul2_u32(e2m1x2_f16x2(x << 1), b);
        o[3] = hmul2_u32(e2m1x2_f16x2(x >> 3), b);
      }
    }
  }
}

// One item against the unit's NT n-tiles: the weights are widened once per step and feed
// every n-tile (token g + 8n of the chunk).  With one n-tile, consecutive steps alternate
// between two accumulator sets, so that an MMA does not wait for the previous one.
template <int WT, int NT>
__device__ __forceinline__ void consume_item(const uint8_t* st, const Offs<WT>& of, int nsteps,
                                             float (&acc)[NT + (NT == 1)][4]) {
  using Gm = Geo<WT>;
#pragma unroll
  for (int h = 0; h < Gm::kSteps; ++h) {
    if (h < nsteps) {
      uint32_t w[16];
      widen<WT>(st, of, h, w);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        // token g + 8n, elements [64h + 16t, +16)
        const uint4 b0 = *reinterpret_cast<const uint4*>(st + of.b[h][0] + n * 8 * Gm::kBRow);
        const uint4 b1 = *reinterpret_cast<const uint4*>(st + of.b[h][1] + n * 8 * Gm::kBRow);
        const uint32_t b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
        float(&c)[4] = acc[NT == 1 ? (h & 1) : n];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma16816<WT == kStreamBf16>(c, w[2 * j], w[8 + 2 * j], w[2 * j + 1], w[8 + 2 * j + 1],
                                      b[2 * j], b[2 * j + 1]);
      }
    }
  }
}

// The scales of this lane's two output rows (g and g + 8 of its warp's strip): int8 one
// per row, nvfp4 the matrix scale times 2^14, bf16 none.  Loaded when a piece starts, so
// that the epilogue does not wait for them.
__device__ __forceinline__ float2 row_scales(const StreamProblem& pr, const Piece& pc) {
  const int warp = threadIdx.x >> 5, g = (threadIdx.x & 31) >> 2;
  const int r0 = 16 * warp + g;
  const size_t grow = static_cast<size_t>(pc.gg) * pr.rows;
  if (pr.wtype == kStreamInt8)
    return make_float2(__ldg(pr.wscale + grow + weight_row(pr, pc.m, r0)),
                       __ldg(pr.wscale + grow + weight_row(pr, pc.m, r0 + 8)));
  if (pr.wtype == kStreamNvfp4) {
    const float s = __ldg(pr.wscale + pc.gg) * 16384.0f;
    return make_float2(s, s);
  }
  return make_float2(1.f, 1.f);
}

// The epilogue of n-tile n of one unit from its (full-K) sums v: lane (g, t) of warp w
// holds rows g and g + 8 of strip w for tokens 8n + 2t and 8n + 2t + 1 of the chunk.
__device__ __forceinline__ void store_unit(const StreamProblem& pr, const Piece& pc, int warp,
                                           int g, int t, int n, const float (&v)[4], float2 sc) {
  const int r0 = 16 * warp + g;
  const int wr0 = weight_row(pr, pc.m, r0), wr1 = weight_row(pr, pc.m, r0 + 8);
  const float s0 = sc.x, s1 = sc.y;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int col = 8 * n + 2 * t + q;
    if (col >= pc.n_valid) continue;
    const size_t pos = static_cast<size_t>(pc.tok0 + col);
    if (pr.kind == 0) {  // row r0: gate of feature wr0, row r0 + 8: its up row
      const float hv = gelu_tanh(v[q] * s0) * (v[2 + q] * s1);
      uint16_t* o = static_cast<uint16_t*>(pr.out) + pos * pr.out_ld + wr0;
      *o = pr.out_type == kOutF16 ? f16_bits(hv) : bf16_bits(hv);
    } else {
      const float y0 = v[q] * s0, y1 = v[2 + q] * s1;
      const size_t o0 = pos * pr.out_ld + wr0, o1 = pos * pr.out_ld + wr1;
      if (pr.out_type == kOutF32) {
        static_cast<float*>(pr.out)[o0] = y0;
        static_cast<float*>(pr.out)[o1] = y1;
      } else if (pr.out_type == kOutF16) {
        static_cast<uint16_t*>(pr.out)[o0] = f16_bits_sat(y0);
        static_cast<uint16_t*>(pr.out)[o1] = f16_bits_sat(y1);
      } else {
        static_cast<uint16_t*>(pr.out)[o0] = bf16_bits(y0);
        static_cast<uint16_t*>(pr.out)[o1] = bf16_bits(y1);
      }
    }
  }
}

// The end of one piece: its partial sums, or (unsplit tiles, and the last piece of a split
// tile) the full sums and the epilogue.  All threads of the CTA.
template <int NT>
__device__ __forceinline__ void finish_piece(const StreamParams& P, const StreamProblem& pr,
                                             const Piece& pc, float (&v)[NT][4], float2 sc,
                                             volatile int* flag) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  constexpr int NC = kStreamChunk * NT;
  if (pr.split > 1) {
    // partial tile [64 rows][NC tokens] fp32: lane (g, t) of warp w writes rows 16w + g and
    // 16w + g + 8, tokens 8n + 2t and 8n + 2t + 1
    float* part = P.partials + pc.part0 + static_cast<int64_t>(pc.s) * (kStreamRows * NC);
    const int r = 16 * warp + g;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      __stcg(reinterpret_cast<float2*>(part + r * NC + 8 * n + 2 * t), make_float2(v[n][0], v[n][1]));
      __stcg(reinterpret_cast<float2*>(part + (r + 8) * NC + 8 * n + 2 * t),
             make_float2(v[n][2], v[n][3]));
    }
    // one release for the CTA: the barrier orders every thread's partial before the
    // elected thread's atomic, whose acq_rel also acquires the other pieces' partials
    __syncthreads();
    if (threadIdx.x == 0) {
      const unsigned old = atom_add_acq_rel_gpu(P.counters + pc.unit, 1u);
      const int last = old == static_cast<unsigned>(pr.split - 1) ? 1 : 0;
      if (last) P.counters[pc.unit] = 0u;  // ready for the next launch
      *flag = last;
    }
    __syncthreads();
    const bool last = *flag != 0;
    __syncthreads();  // every thread has read the flag before it is written again
    if (!last) return;
    // the last piece: every piece's partial, added in piece order
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int q = 0; q < 4; ++q) v[n][q] = 0.f;
    for (int s2 = 0; s2 < pr.split; ++s2) {
      const float* pp = P.partials + pc.part0 + static_cast<int64_t>(s2) * (kStreamRows * NC);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const float2 x = __ldcg(reinterpret_cast<const float2*>(pp + r * NC + 8 * n + 2 * t));
        const float2 y = __ldcg(reinterpret_cast<const float2*>(pp + (r + 8) * NC + 8 * n + 2 * t));
        v[n][0] += x.x; v[n][1] += x.y; v[n][2] += y.x; v[n][3] += y.y;
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NT; ++n) store_unit(pr, pc, warp, g, t, n, v[n], sc);
}

// Pieces are dealt round-robin over the launch: the CTA's k-th piece is blockIdx.x +
// k * gridDim.x (the host sizes the pieces of both problems to about the same bytes).
__device__ __forceinline__ int cta_piece(int k) {
  return static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
}

// The copy side of the ring: walks this CTA's pieces of one problem item by item.
struct IssueCursor {
  int k, item;  // the CTA's piece index and item within the piece
  int piece;
  bool next;    // the piece is exhausted: move to piece k + 1 at the next issue
  Piece pc;
  CopyPlan cp;
};

template <int WT, int NT>
__device__ __forceinline__ void cursor_set(IssueCursor& c, int piece, const StreamParams& P,
                                           const StreamProblem& pr, const Tables& tb, int end) {
  c.piece = piece;
  c.item = 0;
  c.next = false;
  if (piece < end) {
    c.pc = piece_of(piece, P, tb);
    plan_piece<WT, NT>(c.cp, pr, c.pc);
  }
}

// Issues the cursor's item and steps past it (moving to the CTA's next piece at the next
// issue once the piece is exhausted).
template <int WT, int NT>
__device__ __forceinline__ void cursor_issue(IssueCursor& c, uint32_t st, const Offs<WT>& of,
                                             const StreamParams& P, const StreamProblem& pr,
                                             const Tables& tb, int end, bool weights,
                                             bool tokens) {
  if (c.next) {
    ++c.k;
    cursor_set<WT, NT>(c, cta_piece(c.k), P, pr, tb, end);
  }
  if (c.piece >= end) return;
  issue_item<WT, NT>(st, c.cp, of, c.pc.it0 + c.item, weights, tokens);
  if (++c.item == c.pc.it1 - c.pc.it0) c.next = true;
}

// This CTA's pieces of one problem (ids below `end`), starting at its k-th piece, through
// one ring that runs S - 1 items ahead continuously, across piece boundaries: the next
// piece's first copies are in flight while a piece's partial sums are exchanged and stored.
// Returns the index of the CTA's first piece not handled (of the next problem, or done).
template <int WT, int NT>
__device__ int run_problem(const StreamParams& P, const StreamProblem& pr, int k, int end,
                           const Tables& tb, uint8_t* ring, bool& waited, volatile int* flag) {
  constexpr int S = Stage<WT, NT>::kCount;
  constexpr int SB = Stage<WT, NT>::kBytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t r0 = smem_u32(ring);
  const int steps_total = pr.K >> 6;
  const Offs<WT> of = make_offs<WT, NT>(warp, lane);
  IssueCursor ic;
  ic.k = k;
  cursor_set<WT, NT>(ic, cta_piece(k), P, pr, tb, end);
  // prologue: S - 1 items in flight.  Weight copies do not depend on the previous kernel;
  // before the first dependency wait they are issued ahead of the token copies.
  if (!waited) {
    IssueCursor wc = ic;
#pragma unroll 1
    for (int q = 0; q < S - 1; ++q)
      cursor_issue<WT, NT>(wc, r0 + q * SB, of, P, pr, tb, end, true, false);
    pdl_wait();
    waited = true;
#pragma unroll 1
    for (int q = 0; q < S - 1; ++q) {
      cursor_issue<WT, NT>(ic, r0 + q * SB, of, P, pr, tb, end, false, true);
      cp_async_commit();
    }
  } else {
#pragma unroll 1
    for (int q = 0; q < S - 1; ++q) {
      cursor_issue<WT, NT>(ic, r0 + q * SB, of, P, pr, tb, end, true, true);
      cp_async_commit();
    }
  }
  int consumed = 0;
#pragma unroll 1
  for (;;) {
    const int piece = cta_piece(k);
    if (piece >= end) break;
    const Piece pc = piece_of(piece, P, tb);
    const float2 sc = row_scales(pr, pc);
    const int n = pc.it1 - pc.it0;
    float acc[NT + (NT == 1)][4];
#pragma unroll
    for (int n = 0; n < NT + (NT == 1); ++n)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[n][q] = 0.f;
#pragma unroll 1
    for (int i = 0; i < n; ++i) {
      cp_async_wait<S - 2>();  // this thread's copies of the item being consumed have landed
      __syncthreads();         // everyone's have, and everyone is done with the item before
      cursor_issue<WT, NT>(ic, r0 + ((consumed + S - 1) % S) * SB, of, P, pr, tb, end, true, true);
      cp_async_commit();
      const int it = pc.it0 + i;
      const int nsteps = min(Geo<WT>::kSteps, steps_total - it * Geo<WT>::kSteps);
      consume_item<WT, NT>(ring + (consumed % S) * SB, of, nsteps, acc);
      ++consumed;
    }
    float v[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int q = 0; q < 4; ++q) v[n][q] = NT == 1 ? acc[0][q] + acc[NT == 1 ? 1 : 0][q] : acc[n][q];
    finish_piece<NT>(P, pr, pc, v, sc, flag);
    ++k;
  }
  cp_async_wait<0>();
  __syncthreads();  // the ring is free for the next problem
  return k;
}

__global__ void __launch_bounds__(kStreamThreads, 5) stream_gemm_kernel(const StreamParams P) {
  extern __shared__ __align__(128) uint8_t s_ring[];
  __shared__ int pre[kStreamMaxEntries + 1];
  __shared__ int upre[kStreamMaxEntries + 1];
  __shared__ int b0s[kStreamMaxEntries];
  __shared__ int ngs[kStreamMaxEntries];
  __shared__ int s_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G0 = P.prob[0].groups;
  const int nent = G0 + (P.nprob > 1 ? P.prob[1].groups : 0);

  // ---- the piece table (routing offsets come from kernels that completed before the
  // previous kernel on the stream started); pre/upre first hold the counts
  for (int i = threadIdx.x; i < nent; i += kStreamThreads) {
    const int p = i < G0 ? 0 : 1;
    const int gg = p == 0 ? i : i - G0;
    const StreamProblem& pr = P.prob[p];
    int s0 = 0, n = pr.n_tokens;
    if (pr.offsets) {
      int a = pr.offsets[gg], b = pr.offsets[gg + 1];
      a = max(0, min(a, pr.n_tokens));
      b = max(a, min(b, pr.n_tokens));
      s0 = a;
      n = b - a;
    }
    b0s[i] = s0;
    ngs[i] = n;
    const int nc = kStreamChunk * pr.nt;
    const int units = (pr.rows / kStreamRows) * ((n + nc - 1) / nc);
    upre[i] = units;
    pre[i] = units * pr.split;
  }
  __syncthreads();
  if (warp == 0) {
    for (int which = 0; which < 2; ++which) {
      int* arr = which ? upre : pre;
      int carry = 0;
      for (int base = 0; base < nent; base += 32) {
        const int i = base + lane;
        const int v = i < nent ? arr[i] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        __syncwarp();
        if (i < nent) arr[i] = carry + incl - v;
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) arr[nent] = carry;
    }
  }
  __syncthreads();
  pdl_trigger();
  const Tables tb{pre, b0s, ngs, upre, nent, G0};
  const int total = pre[nent];
  const int u1 = pre[G0];  // problem 0's pieces are [0, u1), problem 1's [u1, total)
  bool waited = false;
  int k = 0;
  // (the problem index is unrolled, so that each problem is read from parameter space at
  // a fixed offset rather than copied to local memory)
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    if (p >= P.nprob) break;
    const StreamProblem& pr = P.prob[p];
    const int ue = p == 0 ? u1 : total;
    if (pr.wtype == kStreamInt8) {
      if (pr.nt == 2)
        k = run_problem<kStreamInt8, 2>(P, pr, k, ue, tb, s_ring, waited, &s_flag);
      else
        k = run_problem<kStreamInt8, 1>(P, pr, k, ue, tb, s_ring, waited, &s_flag);
    } else if (pr.wtype == kStreamNvfp4) {
      k = run_problem<kStreamNvfp4, 1>(P, pr, k, ue, tb, s_ring, waited, &s_flag);
    } else {
      if (pr.nt == 4)
        k = run_problem<kStreamBf16, 4>(P, pr, k, ue, tb, s_ring, waited, &s_flag);
      else if (pr.nt == 2)
        k = run_problem<kStreamBf16, 2>(P, pr, k, ue, tb, s_ring, waited, &s_flag);
      else
        k = run_problem<kStreamBf16, 1>(P, pr, k, ue, tb, s_ring, waited, &s_flag);
    }
  }
  if (!waited) pdl_wait();
}

int stream_items(int K, int wtype) { return stream_items_of(K, wtype); }

cudaError_t launch_stream_gemm(const StreamParams& p, int sms, cudaStream_t s, bool pdl) {
  for (int i = 0; i < p.nprob; ++i) {
    const StreamProblem& pr = p.prob[i];
    if (pr.K % 64 || pr.rows % kStreamRows || (pr.kind == 0 && pr.rows != 2 * pr.F)) return cudaErrorInvalidValue;
    if (pr.wtype == kStreamNvfp4 && pr.bscale == nullptr) return cudaErrorInvalidValue;
    if (pr.wtype != kStreamBf16 && pr.wscale == nullptr) return cudaErrorInvalidValue;
    if (pr.split < 1 || pr.split > stream_items_of(pr.K, pr.wtype)) return cudaErrorInvalidValue;
    if (pr.nt != 1 && pr.nt != 2 && pr.nt != 4) return cudaErrorInvalidValue;
    if (pr.nt > stream_max_nt(pr.wtype)) return cudaErrorInvalidValue;
    if (pr.split > 1 && (p.partials == nullptr || p.counters == nullptr)) return cudaErrorInvalidValue;
  }
  const int ctas = stream_gemm_ctas(sms);
  if (ctas <= 0) return cudaErrorInvalidValue;
  return launch_k(stream_gemm_kernel, dim3(ctas), dim3(kStreamThreads), kStreamRingBytes, s, pdl, p);
}

int stream_gemm_ctas(int sms) {
  static int per_sm = 0;  // CTAs resident per SM (the kernel's resources decide it)
  if (per_sm == 0) {
    if (cudaFuncSetAttribute(stream_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kStreamRingBytes) != cudaSuccess)
      return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, stream_gemm_kernel, kStreamThreads,
                                                      kStreamRingBytes) != cudaSuccess)
      return 0;
    per_sm = n > 0 ? n : 1;
  }
  return sms * per_sm;
}

}  // namespace moe
