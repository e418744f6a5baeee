/*
 * moe_ffn.h - C interface of the hybrid mixture-of-experts feed-forward block
 * (Gemma-4-26B-A4B shape) on NVIDIA B200 (sm_100a).
 *
 * The block, per token x (one row of H values):
 *
 *   xhat       = x / sqrt(mean(x^2) + eps)                      scale-free RMSNorm
 *   router     : z = xhat * router_scale * H^-0.5, logits = z W_r^T (+ bias),
 *                softmax (fp32) -> top-k -> renormalise -> * per_expert_scale
 *   experts    : for each selected expert e with weight w:
 *                g, u = xn_moe W_gate_up[e]^T (gate rows, then up rows),
 *                h = gelu_tanh(g) * u,  y = h W_down[e]^T,  moe += w * y
 *   dense MLP  : the same gated-GELU MLP with intermediate D on xn_dense
 *   out        = x + N_post_ff( N_post_dense(dense) + N_post_moe(moe) )
 *
 * where xn_moe = xhat * g_pre_moe, xn_dense = xhat * g_pre_dense and
 * N_g(v) = v / sqrt(mean(v^2) + eps) * g.
 *
 * Sources: "Gemma-4 26B-A4B-it - ONNX MoE text decoder", table "Truthful graph
 * contracts" (rows "Mixture of Experts", "MoE topology", "Router");
 * "Gemma-4 26B-A4B (MoE) on AWS Inferentia2", sections "The architecture (a
 * dual-path FFN)" and "How it works (the recipe)"; "Gemma-4 26B-A4B (MoE, int8
 * experts) on AWS Inferentia2" for the per-channel int8 expert weights.
 *
 * Conventions for every entry point
 *   - bf16 values are passed as their 16-bit patterns (moe_bf16_t).
 *   - All tensors are row-major with the reduction (K) dimension contiguous.
 *   - Every pointer is device memory owned by the caller, 16-byte aligned, unless
 *     marked "host".  The library never allocates or frees memory in these calls;
 *     scratch comes from the caller's workspace `ws` of `ws_bytes` bytes, which must
 *     be at least moe_workspace_size(cfg, T) and 256-byte aligned.  A new workspace
 *     must be zeroed once before its first use (e.g. cudaMemsetAsync); every call that
 *     completes leaves its counters at zero again, so later calls need no clearing.
 *     After MOE_ERR_DEVICE_TIMEOUT, zero the workspace again.  A workspace that was
 *     not zeroed gives wrong results, never an out-of-bounds access or a hang.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every call
 *     only enqueues work on that stream and returns; results are ready when the
 *     stream reaches that point.  Calls on different streams must not share `ws`.
 *   - Size limits: H a multiple of 128 (128..6144), I and D multiples of 64
 *     (128..16384), 1 <= E <= 256, 1 <= k <= min(E, 16), 0 <= T, T*k < 2^31.
 *     T = 0 returns MOE_OK at once (before any pointer is checked) and launches
 *     nothing.
 *   - Argument errors are found on the host before anything is launched and
 *     return MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED or MOE_ERR_WORKSPACE.  A failed
 *     launch returns MOE_ERR_CUDA.  Nothing throws across this interface.
 *   - The GPU kernels bound every wait they make.  A wait that runs out records
 *     MOE_ERR_DEVICE_TIMEOUT in a status word inside `ws`, and the kernel returns;
 *     moe_check_device_status() reads and clears it.
 *   - Results are deterministic: the same inputs give the same bits on every run.
 */
#ifndef MOE_FFN_H
#define MOE_FFN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16_t; /* bf16 bit pattern */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,    /* a pointer, size or layout argument is invalid */
  MOE_ERR_UNSUPPORTED = 2,    /* sizes outside the limits above */
  MOE_ERR_WORKSPACE = 3,      /* ws NULL, misaligned or smaller than required */
  MOE_ERR_CUDA = 4,           /* a CUDA runtime or driver call failed */
  MOE_ERR_DEVICE_TIMEOUT = 5  /* a bounded device wait ran out (see above) */
} moe_status_t;

typedef enum {
  MOE_W_BF16 = 0,    /* expert weights in bf16 */
  MOE_W_INT8 = 1,    /* expert weights int8, one fp32 scale per output row */
  MOE_W_FP8_E4M3 = 2, /* expert weights E4M3, one fp32 scale per output row; the expert
                         matmuls' activations are quantised to E4M3 per token row */
  MOE_W_NVFP4 = 3     /* expert weights NVFP4: E2M1 codes, an E4M3 scale per 16 weights of a
                         row and an fp32 scale per matrix; weight-only */
} moe_wdtype_t;

/* Sizes of one layer. */
typedef struct {
  int32_t hidden;        /* H */
  int32_t num_experts;   /* E */
  int32_t top_k;         /* k */
  int32_t expert_inter;  /* I: intermediate size of each expert */
  int32_t dense_inter;   /* D: intermediate size of the shared dense MLP */
  float eps;             /* RMSNorm epsilon, > 0 */
  int32_t expert_wdtype; /* moe_wdtype_t */
} moe_config_t;

/* Expert weights, read-only; may be shared by concurrent calls.
 *   w_gate_up [E][2I][H]  rows 0..I-1 are the gate projection, rows I..2I-1 the up
 *                         projection (the pages' fused gate_up weight);
 *   w_down    [E][H][I];
 *   bf16 (MOE_W_BF16): s_gate_up and s_down must be NULL.
 *   int8 (MOE_W_INT8): the weight is q * s, with s_gate_up [E][2I] and s_down [E][H]
 *                      fp32 per-output-row scales (see moe_quantize_int8).
 *   fp8 (MOE_W_FP8_E4M3): the same layout of E4M3 codes (uint8) with the same scales
 *                      (see moe_quantize_fp8).  This is the "FP8-dynamic" variant ("Gemma 4
 *                      26B-A4B IT" recipe page, "Quantized Variants": E4M3 weights with
 *                      dynamic per-token activation quantisation): each expert matmul's
 *                      input rows (a routed token's xn_moe, its h) are quantised with
 *                      their own scale max|row| / 448, codes rounded to nearest even and
 *                      saturating; the products accumulate in fp32.
 *   nvfp4 (MOE_W_NVFP4): "NVFP4 (4-bit) quantized weights" ("Gemma 4 26B-A4B IT" recipe
 *                      page, variant list), weight-only: the weight is q * b * t with q an
 *                      E2M1 value (0, 0.5, 1, 1.5, 2, 3, 4, 6 and negatives; code = sign << 3
 *                      | index), b an E4M3 scale per 16 consecutive weights of a row and t an
 *                      fp32 scale per matrix (see moe_quantize_nvfp4):
 *                        w_gate_up [E][2I][H/2] bytes, w_down [E][H][I/2]: codes packed 8 to a
 *                          little-endian 32-bit word, nibbles 0-3 = elements 0, 2, 4, 6 of the
 *                          word's 8 consecutive weights, nibbles 4-7 = elements 1, 3, 5, 7;
 *                        b_gate_up [E][2I][H/16], b_down [E][H][I/16]: E4M3 codes;
 *                        s_gate_up [E], s_down [E]: t of each expert's two matrices.
 *                      Activations stay 16-bit (fp16 inside the expert matmuls, as for int8).
 *   b_gate_up and b_down must be NULL for the other formats. */
typedef struct {
  const void* w_gate_up;
  const void* w_down;
  const float* s_gate_up;
  const float* s_down;
  const uint8_t* b_gate_up;  /* nvfp4 block scales, else NULL */
  const uint8_t* b_down;
} moe_expert_weights_t;

/* All weights of one block. */
typedef struct {
  const moe_bf16_t* router_scale;     /* [H] learned router scale */
  const moe_bf16_t* w_router;         /* [E][H] */
  const float* logit_bias;            /* [E] fp32 added to the logits, or NULL */
  const moe_bf16_t* per_expert_scale; /* [E] */
  const moe_bf16_t* g_pre_moe;        /* [H] gain of the MoE branch's pre norm */
  const moe_bf16_t* g_pre_dense;      /* [H] gain of the dense branch's pre norm */
  const moe_bf16_t* g_post_moe;       /* [H] or NULL: post norm of the MoE branch skipped */
  const moe_bf16_t* g_post_dense;     /* [H] or NULL: post norm of the dense branch skipped */
  const moe_bf16_t* g_post_ff;        /* [H] gain of the final post_ff norm */
  moe_expert_weights_t experts;
  const moe_bf16_t* w_dense_gate_up;  /* [2D][H] gate rows then up rows */
  const moe_bf16_t* w_dense_down;     /* [H][D] */
} moe_block_weights_t;

/* Bytes of workspace every call below needs for T tokens (0 if cfg is invalid).
 * Host function; launches nothing. */
size_t moe_workspace_size(const moe_config_t* cfg, int32_t T);

/* Router and pre norms (ONNX export card, "Truthful graph contracts", Router row;
 * Inferentia2 card, "The architecture").
 *   x [T][H] bf16 (the un-normed block input).
 *   Outputs: topk_idx [T][k] int32 expert ids, ordered by logit descending and, for
 *   equal logits, by expert id ascending; topk_w [T][k] fp32 routing weights
 *   (renormalised over the k selected, then times per_expert_scale);
 *   xn_moe, xn_dense [T][H] bf16 = xhat * g_pre_moe, xhat * g_pre_dense.
 *   logit_bias may be NULL. */
moe_status_t moe_router(const moe_config_t* cfg, int32_t T, const moe_bf16_t* x,
                        const moe_bf16_t* router_scale, const moe_bf16_t* w_router,
                        const float* logit_bias, const moe_bf16_t* per_expert_scale,
                        const moe_bf16_t* g_pre_moe, const moe_bf16_t* g_pre_dense,
                        int32_t* topk_idx, float* topk_w, moe_bf16_t* xn_moe,
                        moe_bf16_t* xn_dense, void* ws, size_t ws_bytes, void* stream);

/* Token-to-expert permutation (a counting sort; the gathered-per-expert dispatch of
 * the Tenstorrent card's "gathered expert prefill", computed exactly).
 *   topk_idx [T][k] int32 in [0, E).  The flat pair index is p = t*k + j.
 *   expert_offsets [E+1]: expert e's pairs occupy [offsets[e], offsets[e+1]).
 *   sorted_src [T*k]: the pairs grouped by expert, in increasing p within a group.
 *   inv_pos [T*k]: inv_pos[p] is the position of pair p in sorted_src.
 *   An id outside [0, E) returns nothing useful; the kernel does not read or write
 *   out of bounds for it (such pairs are dropped and the offsets count the rest). */
moe_status_t moe_permute(const moe_config_t* cfg, int32_t T, const int32_t* topk_idx,
                         int32_t* expert_offsets, int32_t* sorted_src, int32_t* inv_pos,
                         void* ws, size_t ws_bytes, void* stream);

/* The token-to-expert permutation of moe_permute for callers that cannot hand the
 * library any scratch memory: plugin hosts that pass only input and output buffers and
 * offer no allocator, processes whose device memory is already reserved by another
 * framework's caching allocator, and latency-critical loops that must not call
 * cudaMalloc (which can synchronise the device).  The model pages have no counterpart;
 * this is an interface convenience, computing exactly what moe_permute computes.
 *   Arguments and results as in moe_permute, without `ws`.
 *   Scratch: a fixed array of MOE_PERMUTE_NOALLOC_SCRATCH_BYTES (512 KiB) in the
 *   library's device memory, present on every GPU that loads the library until the
 *   process exits.  Nothing is allocated or freed by this call.
 *   Limits: T*k <= MOE_PERMUTE_NOALLOC_MAX_PAIRS (2^20); larger batches return
 *   MOE_ERR_UNSUPPORTED before anything is launched (use moe_permute with a workspace).
 *   Every call looks up the scratch array's address in the calling thread's current
 *   context (an allocation-free lookup), so a device reset or another context on the
 *   same device never leaves a stale address behind.  The first call in a context may
 *   load the library's device code there: make it before any stream capture.
 *   Every call shares the one scratch array: calls whose kernels overlap on the GPU (on
 *   different streams, or from several threads) race and must be serialised by the
 *   caller.  Each call fully writes the scratch it reads, so nothing carries over. */
#define MOE_PERMUTE_NOALLOC_MAX_PAIRS (1 << 20)
#define MOE_PERMUTE_NOALLOC_SCRATCH_BYTES (512 * 1024)
moe_status_t moe_permute_noalloc(const moe_config_t* cfg, int32_t T, const int32_t* topk_idx,
                                 int32_t* expert_offsets, int32_t* sorted_src,
                                 int32_t* inv_pos, void* stream);

/* Routed experts (ONNX export card, "Mixture of Experts" row; Inferentia2 card,
 * "How it works": outputs weighted by the routing weights and summed).
 *   xn_moe [T][H] bf16; topk_w [T][k] fp32; expert_offsets, sorted_src, inv_pos as
 *   produced by moe_permute.
 *   moe_out [T][H] bf16 = sum_j topk_w[t][j] * MLP_{e(t,j)}(xn_moe[t]), the branch
 *   output before its post norm.  Accumulation is fp32; between the steps h is stored
 *   as bf16 (fp16 with int8 or NVFP4 experts, E4M3 codes with a row scale with fp8
 *   experts) and each pair's unweighted expert output as fp16; the weighted sum over the
 *   slots is taken in fp32, in slot order. */
moe_status_t moe_ffn_forward(const moe_config_t* cfg, int32_t T, const moe_bf16_t* xn_moe,
                             const float* topk_w, const int32_t* expert_offsets,
                             const int32_t* sorted_src, const int32_t* inv_pos,
                             const moe_expert_weights_t* experts, moe_bf16_t* moe_out,
                             void* ws, size_t ws_bytes, void* stream);

/* Shared dense MLP (ONNX export card, "MoE topology" row).
 *   xn_dense [T][H]; w_gate_up [2D][H] (gate rows, then up rows); w_down [H][D].
 *   dense_out [T][H] bf16 = gelu_tanh(xn g^T) * (xn u^T) W_down^T, fp32 accumulation. */
moe_status_t dense_mlp_forward(const moe_config_t* cfg, int32_t T, const moe_bf16_t* xn_dense,
                               const moe_bf16_t* w_gate_up, const moe_bf16_t* w_down,
                               moe_bf16_t* dense_out, void* ws, size_t ws_bytes, void* stream);

/* The whole block: router -> permute -> experts and dense MLP -> combine, post norms
 * and residual (ONNX export card, "MoE topology" row).
 *   x [T][H] bf16 input; out [T][H] bf16.  moe_out [T][H] bf16 may be NULL; when given
 *   it receives the MoE branch output before its post norm.
 *   stage_events: NULL, or a host array of MOE_BLOCK_EVENTS cudaEvent_t that the call
 *   records on `stream` at its stage boundaries, for timing each stage:
 *     [0] start  [1] router done (with the permutation for small batches)
 *     [2] permutation done  [3] row gather done  [4] gate_up GEMMs done
 *     [5] down GEMMs done  [6] combine done */
#define MOE_BLOCK_EVENTS 7
moe_status_t moe_block_forward(const moe_config_t* cfg, int32_t T, const moe_bf16_t* x,
                               const moe_block_weights_t* w, moe_bf16_t* out,
                               moe_bf16_t* moe_out, void* ws, size_t ws_bytes, void* stream,
                               void* const* stage_events);

/* Chunked prefill over a stack of blocks (the Tenstorrent card's "Configurable knobs":
 * GEMMA4_CHUNKED_PREFILL, GEMMA4_PREFILL_CHUNK_SIZE 16384 "snapped to 1024, capped at
 * 32768").  The blocks of one layer stack are chained through the residual (block l's `out`
 * is block l+1's `x`); the block is row-independent, so a long prompt runs as consecutive
 * chunks of at most moe_stack_chunk_tokens(chunk_tokens) tokens, every chunk through every
 * layer, with a workspace sized for one chunk instead of the whole prompt.
 *   moe_stack_chunk_tokens: the chunk length used for a requested one: rounded down to a
 *     multiple of 1024, at least 1024, at most 32768.  Host function.
 *   moe_stack_workspace_size: bytes of workspace for chunks of that length (0 if cfg is
 *     invalid); 256-byte aligned, zeroed once before first use like the block workspace.
 *   moe_stack_forward: x [T][H] -> out [T][H] through layers[0..n_layers-1] (host array of
 *     weight structs; the device pointers inside as for moe_block_forward), chunk after
 *     chunk on `stream`; x and out must not overlap.  n_layers >= 1.  Errors as for
 *     moe_block_forward; the first failing call's status is returned. */
int32_t moe_stack_chunk_tokens(int32_t chunk_tokens);
size_t moe_stack_workspace_size(const moe_config_t* cfg, int32_t chunk_tokens);
moe_status_t moe_stack_forward(const moe_config_t* cfg, int32_t T, const moe_bf16_t* x,
                               const moe_block_weights_t* layers, int32_t n_layers,
                               moe_bf16_t* out, int32_t chunk_tokens, void* ws,
                               size_t ws_bytes, void* stream);

/* Per-output-row symmetric int8 quantisation ("Gemma-4 26B-A4B (MoE, int8 experts)",
 * "How it works": per-channel symmetric INT8 expert weights).
 *   w [rows][cols] bf16 -> q [rows][cols] int8, scales [rows] fp32, computed in fp32:
 *   s = max|w| / 127 (s = 1 for an all-zero row), q = round-half-even(w / s) clamped to
 *   [-127, 127].  cols a multiple of 8 (1..65536), rows >= 0. */
moe_status_t moe_quantize_int8(const moe_bf16_t* w, int64_t rows, int32_t cols, int8_t* q,
                               float* scales, void* stream);

/* Per-output-row E4M3 quantisation for MOE_W_FP8_E4M3, in fp32: s = max|w| / 448 (s = 1
 * for an all-zero row), q = E4M3 code of w / s, rounded to nearest even, saturating at
 * +-448 ("Gemma 4 26B-A4B IT", "Quantized Variants").  w [rows][cols] bf16 -> q
 * [rows][cols] uint8 codes, scales [rows] fp32; cols a multiple of 8 (8..65536),
 * rows >= 0; w and q 16-byte aligned. */
moe_status_t moe_quantize_fp8(const moe_bf16_t* w, int64_t rows, int32_t cols, uint8_t* q,
                              float* scales, void* stream);

/* NVFP4 quantisation of `matrices` bf16 weight matrices of [rows][cols] each, weight-only
 * ("Gemma 4 26B-A4B IT" recipe page, variant list: "NVFP4 (4-bit) quantized weights"; the
 * format is named there, not defined: this is the public NVFP4 format, quantised as
 * follows), computed in fp32:
 *   t = max|W| / (448 * 6) over the matrix (t = 1 for an all-zero matrix);
 *   per block of 16 consecutive weights of a row: b = E4M3(max|block| / 6 / t), rounded to
 *   nearest even, saturating at 448;
 *   codes: E2M1(w / (b * t)) rounded to nearest, ties to the even code, saturating at +-6;
 *   a block whose scale is 0 gets code 0 throughout.
 * Outputs (layouts as in moe_expert_weights_t): q [matrices][rows][cols/2] packed codes,
 * block_scales [matrices][rows][cols/16] E4M3 codes, tensor_scales [matrices] fp32 t.
 * cols a multiple of 16 (16..65536), rows >= 1, matrices >= 0; w 16-byte aligned, q
 * 8-byte aligned, tensor_scales 4-byte aligned.  tensor_scales is also used as scratch
 * (it is cleared and filled by the call). */
moe_status_t moe_quantize_nvfp4(const moe_bf16_t* w, int64_t matrices, int64_t rows,
                                int32_t cols, uint8_t* q, uint8_t* block_scales,
                                float* tensor_scales, void* stream);

/* Waits for `stream`, then reads and clears the device status word in `ws`.
 * Returns MOE_OK, MOE_ERR_DEVICE_TIMEOUT, or MOE_ERR_CUDA if the stream failed. */
moe_status_t moe_check_device_status(void* ws, size_t ws_bytes, void* stream);

/* Self-test of the failure path of the bounded device waits (this library's own health
 * check; the pages define no such call).  Enqueues one kernel that waits on a barrier
 * that nothing completes, for `timeout_ns` nanoseconds (1e3 .. 1e10), then records
 * MOE_ERR_DEVICE_TIMEOUT in the status word of `ws` exactly as a kernel of the block
 * does when one of its waits runs out, and returns.  The GPU context stays usable; a
 * following moe_check_device_status() returns MOE_ERR_DEVICE_TIMEOUT and clears the
 * word.  Only the status word is written.  ws: 256-byte aligned, ws_bytes >= 256;
 * otherwise MOE_ERR_WORKSPACE; a timeout out of range gives MOE_ERR_INVALID_ARG. */
moe_status_t moe_wait_selftest(void* ws, size_t ws_bytes, uint64_t timeout_ns, void* stream);

/* Number of kernels that one moe_block_forward(cfg, T, ...) launches (host-only, no
 * GPU needed): the router (1, or 2 for the tensor-core router of T > 128: weight prep and
 * router), the permutation (0 when the router sorts in the same launch, else 1 or 3),
 * the row gather (0 when the router also gathers: bf16 experts, T <= 8 and T*k <= 32),
 * the gate_up and down GEMMs and the combine (1 each), and for MOE_W_FP8_E4M3 the
 * quantisation of h between the GEMMs.  0 for T = 0;
 * -1 when cfg or T is invalid (the arguments moe_block_forward would reject). */
int32_t moe_block_launch_count(const moe_config_t* cfg, int32_t T);

/* A short constant English description of a status code. */
const char* moe_status_string(moe_status_t status);

/* Version of this interface (increases when a signature or a calling contract changes;
 * 2: the workspace is zeroed once by the caller, MOE_BLOCK_EVENTS is 7;
 * 3: moe_wait_selftest; 4: moe_block_launch_count; 5: MOE_W_FP8_E4M3, moe_quantize_fp8;
 * 6: MOE_W_NVFP4, moe_quantize_nvfp4, block-scale fields in moe_expert_weights_t;
 * 7: moe_stack_chunk_tokens, moe_stack_workspace_size, moe_stack_forward). */
int32_t moe_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_FFN_H */
