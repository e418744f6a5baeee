// Host-side declarations shared by the kernel files and the C interface (moe_ffn.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// One GEMM problem of a grouped launch.  The weights are the M operand (rows of a
// K-major matrix streamed by TMA), the tokens the N operand.  Output row = B row.
//   kind 0 (gate_up): each M tile holds 64 features of one group as 8 gate rows, the
//     8 matching up rows, the next 8 gate rows, ... (a 5-D tensor map over
//     [group][gate|up][feature/8][8][K]); the epilogue writes h = gelu_tanh(gate) * up
//     as bf16.
//   kind 1 (down): each M tile is 128 rows of the output; the epilogue scales by the
//     int8 row scale (if any) and writes bf16 or fp32.
struct GemmProblem {
  int kind;              // 0 gate_up, 1 down
  int groups;            // experts, or 1 for the dense MLP
  const int* offsets;    // [groups+1] token segments in the B operand; NULL = one group
  int n_tokens;          // rows of the B operand and of the output (segments are
                         // clamped to it); the single group's tokens if offsets == NULL
  int k_steps;           // K / 64
  int m_tiles;           // gate_up: Nw / 64;  down: rows / 128
  int w_rows_per_group;  // gate_up: 2 * Nw;   down: rows
  int nw;                // gate_up: Nw (first up row); down: unused
  int split;             // pieces per tile along K (>= 1)
  int map;               // tensor-map pair: 0 or 1
  void* out;             // output: bf16 or fp16 (gate_up, see f16), or out_type (down)
  int out_type;          // down: kOutBf16, kOutF32 or kOutF16 (the block's branch outputs
                         // before the combine keep more precision than bf16: the dense
                         // output fp32, the expert outputs fp16)
  int out_ld;            // elements per output row
  const float* wscale;   // int8 row scales [groups][w_rows_per_group]; NULL for bf16
  int w8;                // A operand is int8 codes (needs a launch with int8_weights)
  int f16;               // A and B are fp16 (int8 codes are converted to fp16, exact);
                         // gate_up writes h in fp16
  int fp8;               // A and B are E4M3 codes (kind::f8f6f4 MMAs, 128 K per step)
  const float* xscale;   // fp8: scale of each B row (sorted order), applied per column
                         // in the epilogue with wscale; NULL otherwise
};

constexpr int kOutBf16 = 0, kOutF32 = 1, kOutF16 = 2;

struct GemmParams {
  GemmProblem prob[2];
  int nprob;
  int int8_weights;     // a problem has int8 A: use the variant with converter warps
  int pairs;            // run on CTA pairs (see gemm_pairs_allowed)
  float* partials;      // split-K partial tiles, [piece][BN][128] fp32
  unsigned* counters;   // split-K arrival counters, zero between launches
  unsigned* sched;      // [2] piece counter and finished CTAs (single-CTA launches), zero
                        // between launches; launches that may overlap need their own
  unsigned* status;     // device status word
  uint64_t timeout_ns;  // bound of every wait
};

struct GemmMaps {
  CUtensorMap a[2];  // weights of problem map 0 / 1
  CUtensorMap b[2];  // tokens of problem map 0 / 1
};

// Launches kernel<<<grid, block, smem, s>>>(args...).  With pdl the launch is a
// programmatic dependent of the previous kernel on s: it may start (and run its setup)
// before that kernel ends, and waits in pdl_wait() before reading its results.  The
// first kernel of every entry point is launched without it, so that nothing overlaps
// work that an earlier call left on the stream.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Launchers.  All return cudaSuccess or the launch error.
// Router + pre norms + top-k in one launch; when offsets != NULL (and T*k fits the
// single-block sort, see permute_blocks) also the token-to-expert counting sort, and with
// aperm != NULL (a single token block, T <= 8) the gather of the routed rows of xn_moe in
// sorted order into aperm (fp16 when aperm_f16).
// counters: router_counters(T) words, zero on entry (left zero on exit).
cudaError_t launch_router(int T, int H, int E, int k, float eps, const uint16_t* x,
                          const uint16_t* router_scale, const uint16_t* w_router,
                          const float* bias, const uint16_t* per_expert_scale,
                          const uint16_t* g_pre_moe, const uint16_t* g_pre_dense,
                          uint16_t* xn_moe, uint16_t* xn_dense, float* logits, int* topk_idx,
                          float* topk_w, unsigned* counters, unsigned* status, int* offsets,
                          int* sorted_src, int* inv_pos, uint16_t* aperm, bool aperm_f16,
                          cudaStream_t s, bool pdl = false);
int router_counters(int T);

// The tensor-core router (router_tc.cu) serves batches of more than kRouterTcMinT
// tokens.  It needs two E x H bf16 buffers for the split W' = s * W_r / sqrt(H), the
// logits buffer [T][E] fp32 and one counter per 128 tokens when it splits the experts
// into router_tc_slices(T, E) > 1 slices, and the tensor maps below: x [T][H] with
// 64 x 128 boxes, W'hi and W'lo [E][H] with 64 x (E rounded up to 16) / slices boxes,
// all with 128-byte swizzling.
constexpr int kRouterTcMinT = 128;
bool router_uses_tc(int T);
int router_tc_slices(int T, int E);
struct RouterTcMaps {
  CUtensorMap x, whi, wlo;
};
cudaError_t launch_router_tc(const RouterTcMaps& maps, int T, int H, int E, int k, float eps,
                             const uint16_t* w_router, const uint16_t* router_scale,
                             uint16_t* whi, uint16_t* wlo, const float* bias,
                             const uint16_t* per_expert_scale, const uint16_t* g_pre_moe,
                             const uint16_t* g_pre_dense, uint16_t* xn_moe, uint16_t* xn_dense,
                             int* topk_idx, float* topk_w, float* logits, unsigned* counters,
                             unsigned* status, uint64_t timeout_ns, cudaStream_t s,
                             bool pdl = false);
cudaError_t launch_permute(int n, int E, const int* topk_idx, int* offsets, int* sorted_src,
                           int* inv_pos, int* block_hist, int* block_base, cudaStream_t s,
                           bool pdl = false);
int permute_blocks(int n);  // blocks of the multi-block path, <= 256 (0 = single-block path)
// dst[q] = src row sorted_src[q] / k for the n sorted positions; to_f16: write the rows
// as fp16 (the operand type of int8 experts) instead of bf16.  With inv_pos (the inverse
// permutation) large batches are written token by token.
cudaError_t launch_gather_rows(int n, int k, int H, int T, const int* sorted_src,
                               const int* inv_pos, const uint16_t* src, uint16_t* dst,
                               bool to_f16, cudaStream_t s, bool pdl = false);
// A launch may run on CTA pairs (GemmParams::pairs) when its weights are bf16 and its
// token tiles are 128 or 256 wide; its B maps then take boxes of bn / 2 rows (each CTA
// loads half of a tile's token rows), and the grid is even.  A pair takes two M tiles:
// with an odd count the second CTA of the last pair computes on zero or foreign weight
// rows and stores nothing.
bool gemm_pairs_allowed(int bn, bool int8_weights);
cudaError_t launch_grouped_gemm(int bn, const GemmMaps& maps, const GemmParams& p, int grid,
                                cudaStream_t s, bool pdl = false);
// y holds the expert outputs in sorted order (row inv_pos[t*k+j] for slot j of token
// t), unweighted; the combine applies topk_w.  With sorted_src != NULL a slot counts
// only if sorted_src[inv_pos[p]] == p (a caller-supplied permutation may have dropped
// pairs); NULL skips that check (the permutation is this library's own).
cudaError_t launch_combine_block(int T, int H, int k, float eps, const uint16_t* x,
                                 const uint16_t* y, const int* inv_pos, const int* sorted_src,
                                 const float* topk_w, const float* dense,
                                 const uint16_t* g_post_moe, const uint16_t* g_post_dense,
                                 const uint16_t* g_post_ff, uint16_t* out, uint16_t* moe_out,
                                 cudaStream_t s, bool pdl = false);
cudaError_t launch_combine_moe(int T, int H, int k, const uint16_t* y, const int* inv_pos,
                               const int* sorted_src, const float* topk_w, uint16_t* moe_out,
                               cudaStream_t s, bool pdl = false);
cudaError_t launch_wait_selftest(unsigned* status, uint64_t timeout_ns, cudaStream_t s);

// The weight-streaming grouped GEMM of small batches (stream_gemm.cu): the same gate_up and
// down problems as GemmProblem, with the weights dequantised in registers.
constexpr int kStreamBf16 = 0, kStreamInt8 = 1, kStreamNvfp4 = 2;
struct StreamProblem {
  int kind;              // 0 gate_up (writes h = gelu_tanh(gate) * up), 1 down
  int wtype;             // kStreamBf16 (bf16 B), kStreamInt8 or kStreamNvfp4 (fp16 B)
  int groups;            // experts, or 1 for the dense MLP
  const int* offsets;    // [groups+1] token segments of b; NULL = one group of n_tokens
  int n_tokens;          // rows of b and of the output
  int K;                 // reduction length, a multiple of 64
  int rows;              // weight rows per group (gate_up: 2F), a multiple of 16
  int F;                 // gate_up: features (first up row)
  const void* w;         // [groups][rows][K] bf16 / int8, or [groups][rows][K/2] packed E2M1
  const float* wscale;   // int8: [groups][rows] row scales; nvfp4: [groups] matrix scales
  const uint8_t* bscale; // nvfp4: [groups][rows][K/16] E4M3 block scales
  const uint16_t* b;     // [n_tokens][K] token rows (bf16, or fp16 for int8 / nvfp4)
  void* out;             // gate_up: h [n_tokens][out_ld]; down: [n_tokens][out_ld]
  int out_type;          // kOutBf16, kOutF16 (gate_up: h's format) or kOutF32 (down)
  int out_ld;
  int split;             // pieces per tile along K (1 .. stream_items(K, wtype))
  int nt;                // tokens per unit in n-tiles of 8 (1 .. stream_max_nt(wtype))
};
struct StreamParams {
  StreamProblem prob[2];
  int nprob;
  float* partials;       // split-K partial tiles, [piece][64][8 * nt] fp32, problem 0's first
  unsigned* counters;    // split-K arrival counters, one per (tile, chunk); zero between launches
};
// Tiles of 64 weight rows against chunks of 8 * nt tokens; K in items of 128 bytes of a row.
constexpr int kStreamTileRows = 64, kStreamChunk = 8;
int stream_items(int K, int wtype);
// The widest unit (n-tiles of 8 tokens) a weight format allows: 4 for bf16, 2 for int8,
// 1 for NVFP4.
constexpr int stream_max_nt(int wtype) {
  return wtype == kStreamBf16 ? 4 : wtype == kStreamInt8 ? 2 : 1;
}
// CTAs of one launch (a persistent grid of every CTA that fits at once).
int stream_gemm_ctas(int sms);
cudaError_t launch_stream_gemm(const StreamParams& p, int sms, cudaStream_t s, bool pdl);
// dst[q] = E4M3 codes of row r(q) of src divided by scales[q] = max|row| / 448 (1 for an
// all-zero row), r(q) = sorted_src[q] / k, or q when sorted_src is NULL; a source row
// outside [0, T) gives a zero row.  cols a multiple of 8.
cudaError_t launch_gather_quant_fp8(int n, int k, int cols, int T, const int* sorted_src,
                                    const uint16_t* src, uint8_t* dst, float* scales,
                                    cudaStream_t s, bool pdl);
cudaError_t launch_quantize_fp8(const uint16_t* w, int64_t rows, int cols, uint8_t* q,
                                float* scales, cudaStream_t s);
cudaError_t launch_quantize_int8(const uint16_t* w, int64_t rows, int cols, int8_t* q,
                                 float* scales, cudaStream_t s);
// matrices x [rows][cols] bf16 -> packed E2M1 codes [.][rows][cols/2], E4M3 block scales
// [.][rows][cols/16], fp32 matrix scales [matrices]; cols a multiple of 16.
cudaError_t launch_quantize_nvfp4(const uint16_t* w, int64_t matrices, int64_t rows, int cols,
                                  uint8_t* q, uint8_t* bscale, float* tensor_scale,
                                  cudaStream_t s);

}  // namespace moe
