// C interface of the hybrid MoE feed-forward block: argument checks, workspace layout,
// TMA tensor maps and the launch sequence.  See include/moe_ffn.h for the contract.
#include <cudaTypedefs.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "internal.h"
#include "moe_ffn.h"

using namespace moe;

namespace {

constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // bound of every device wait: 2 s
constexpr size_t kAlign = 1024;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- sizes and checks

struct Dims {
  int T, H, E, k, I, D;
  float eps;
  int int8;  // int8 expert weights (converted to fp16 on the way to the tensor cores)
  int fp8;   // E4M3 expert weights and per-token E4M3 activations of the expert matmuls
  int nvfp4; // NVFP4 expert weights (weight-only; fp16 activations like int8)
};

moe_status_t check_cfg(const moe_config_t* c, int32_t T, Dims* d) {
  if (c == nullptr) return MOE_ERR_INVALID_ARG;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (!(c->eps > 0.f) || !(c->eps < 1e30f)) return MOE_ERR_INVALID_ARG;
  if (c->expert_wdtype != MOE_W_BF16 && c->expert_wdtype != MOE_W_INT8 &&
      c->expert_wdtype != MOE_W_FP8_E4M3 && c->expert_wdtype != MOE_W_NVFP4)
    return MOE_ERR_INVALID_ARG;
  if (c->hidden < 128 || c->hidden > 6144 || c->hidden % 128) return MOE_ERR_UNSUPPORTED;
  // I, D >= 128: with a 64-wide dense intermediate the bf16 rounding of the GEMM operands
  // alone can reach the accuracy bar at the largest H, E and k (an emulation over seeds)
  if (c->expert_inter < 128 || c->expert_inter > 16384 || c->expert_inter % 64) return MOE_ERR_UNSUPPORTED;
  if (c->dense_inter < 128 || c->dense_inter > 16384 || c->dense_inter % 64) return MOE_ERR_UNSUPPORTED;
  if (c->num_experts < 1 || c->num_experts > 256) return MOE_ERR_UNSUPPORTED;
  if (c->top_k < 1 || c->top_k > 16 || c->top_k > c->num_experts) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(T) * c->top_k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  // every weight tensor must be addressable by a 32-bit TMA row coordinate
  if (static_cast<int64_t>(c->num_experts) * 2 * c->expert_inter >= (int64_t(1) << 31) ||
      static_cast<int64_t>(c->num_experts) * c->hidden >= (int64_t(1) << 31))
    return MOE_ERR_UNSUPPORTED;
  d->T = T;
  d->H = c->hidden;
  d->E = c->num_experts;
  d->k = c->top_k;
  d->I = c->expert_inter;
  d->D = c->dense_inter;
  d->eps = c->eps;
  d->int8 = c->expert_wdtype == MOE_W_INT8;
  d->fp8 = c->expert_wdtype == MOE_W_FP8_E4M3;
  d->nvfp4 = c->expert_wdtype == MOE_W_NVFP4;
  return MOE_OK;
}

// Token-tile width of the GEMMs: about twice the mean number of tokens per expert.
int choose_bn(const Dims& d) {
  const double avg = static_cast<double>(d.T) * d.k / d.E;
  int bn = 16;
  while (bn < 256 && bn < 2.0 * avg) bn *= 2;
  return bn;
}

// K pieces per tile: only for the narrowest token tiles (weight-streaming batches), and
// only when a launch has too few tiles to keep every SM streaming to the end (fewer than
// kSplitTilesPerSm per SM); the partial sums cost more than the balance gains beyond.
// Pieces keep about 22 k-steps (each piece costs a partial store and an arrival: at
// decode T = 8 the gate_up launch measured 6% faster with pieces of 22 k-steps than of
// 11), or about 11 when a launch has fewer than two tiles per SM (T = 1).
constexpr int kSplitTilesPerSm = 8;
constexpr int kAssumedSms = 148;  // a B200; only shifts the threshold if the GPU differs

int choose_split(int k_steps, int bn, double tiles) {
  if (bn != 16 || tiles >= kSplitTilesPerSm * kAssumedSms) return 1;
  const int per = tiles < 2 * kAssumedSms ? 11 : 22;
  return std::max(1, std::min(std::min(k_steps, 4), (k_steps + per - 1) / per));
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Expected number of experts that receive at least one of T*k uniformly routed pairs
// (fewer when the routing is skewed, which only makes splitting more useful).
double expected_used_experts(const Dims& d) {
  const double pairs = static_cast<double>(d.T) * d.k;
  return d.E * (1.0 - std::pow(1.0 - 1.0 / d.E, pairs));
}

// Batches up to this many tokens with 8-bit integer expert weights run the expert and
// dense GEMMs on the weight-streaming kernel (stream_gemm.cu), which widens the codes in
// registers; larger ones on the tensor-memory kernel with converter warps.  NVFP4 expert
// weights always take the weight-streaming kernel.
constexpr int kStreamMaxT = 256;

bool stream_path(const Dims& d) { return d.nvfp4 || (d.int8 && d.T <= kStreamMaxT); }

// Batches of at most this many (token, slot) pairs in one token block of the small-batch
// router have their routed rows gathered by the router's last CTA, after its sort, instead
// of by a launch of its own (a few rows: less than the launch and its kernel boundary;
// bf16 T = 1 step 52.7 -> 50.8 us).  With int8 or NVFP4 experts it measured slower (T = 1
// +4% and +7%: the weight-streaming GEMM's weight requests, issued before its dependency
// wait, then overlap only the router's tail), and fp8 rows are quantised on the way, so
// those keep the separate gather.
constexpr int kRouterGatherMaxPairs = 32;

bool router_gathers(const Dims& d) {
  return d.T <= 8 && d.T * d.k <= kRouterGatherMaxPairs && !d.fp8 && !d.int8 && !d.nvfp4;
}

// K pieces of the weight-streaming kernel's tiles.  Pieces are dealt round-robin, so the
// pieces of both problems of a launch are sized to about the same bytes: about four per CTA
// of the launch (five CTAs per SM assumed), at least 32 KB and four K items each.
constexpr int kStreamAssumedCtas = 5 * kAssumedSms;

struct StreamSplits {
  int gu_e, gu_d, dn_e, dn_d;  // K pieces: gate_up experts / dense, down experts / dense
  int nt_e, nt_d;              // token n-tiles of 8 per unit: experts / dense (both launches)
  int64_t units, pieces;       // upper bounds over the two launches
  int64_t partial_floats;      // upper bound of the split-K partials of one launch
};

int stream_split(double tile_bytes, double target, int items) {
  const int want = static_cast<int>(std::lround(tile_bytes / target));
  return std::max(1, std::min(want, items / 4));
}

// Token n-tiles per unit for a group of about `mean` tokens: a weight tile is read once
// per unit, so groups of many tokens take wide units (up to the ring's limit for the
// weight format: three stages must fit).
int stream_nt(double mean, int wtype) {
  const int cap = stream_max_nt(wtype);
  int nt = 1;
  while (nt < cap && mean > kStreamChunk * nt) nt *= 2;
  return nt;
}

StreamSplits stream_splits(const Dims& d) {
  StreamSplits ss{};
  const int64_t T = d.T, Tk = static_cast<int64_t>(d.T) * d.k;
  const double u = expected_used_experts(d);
  const int wt = d.nvfp4 ? kStreamNvfp4 : d.int8 ? kStreamInt8 : kStreamBf16;
  ss.nt_e = stream_nt(static_cast<double>(Tk) / std::max(u, 1.0), wt);
  ss.nt_d = stream_nt(static_cast<double>(T), kStreamBf16);
  const int nc_e = kStreamChunk * ss.nt_e, nc_d = kStreamChunk * ss.nt_d;
  const double dense_chunks = static_cast<double>(ceil_div(T, nc_d));
  const double exp_chunks = u * std::max(1.0, static_cast<double>(Tk) / std::max(u, 1.0) / nc_e);
  const int tiles_gu_e = 2 * d.I / kStreamTileRows, tiles_gu_d = 2 * d.D / kStreamTileRows;
  const int tiles_dn = d.H / kStreamTileRows;
  // bytes of one tile (64 rows of the full K)
  const double t_gu_e = 128.0 * kStreamTileRows * stream_items(d.H, wt);
  const double t_gu_d = 128.0 * kStreamTileRows * stream_items(d.H, kStreamBf16);
  const double t_dn_e = 128.0 * kStreamTileRows * stream_items(d.I, wt);
  const double t_dn_d = 128.0 * kStreamTileRows * stream_items(d.D, kStreamBf16);
  const double gu_bytes = exp_chunks * tiles_gu_e * t_gu_e + dense_chunks * tiles_gu_d * t_gu_d;
  const double dn_bytes = (exp_chunks * t_dn_e + dense_chunks * t_dn_d) * tiles_dn;
  const double tgt_gu = std::max(32.0 * 1024, gu_bytes / (4.0 * kStreamAssumedCtas));
  const double tgt_dn = std::max(32.0 * 1024, dn_bytes / (4.0 * kStreamAssumedCtas));
  ss.gu_e = stream_split(t_gu_e, tgt_gu, stream_items(d.H, wt));
  ss.gu_d = stream_split(t_gu_d, tgt_gu, stream_items(d.H, kStreamBf16));
  ss.dn_e = stream_split(t_dn_e, tgt_dn, stream_items(d.I, wt));
  ss.dn_d = stream_split(t_dn_d, tgt_dn, stream_items(d.D, kStreamBf16));
  // upper bounds: every non-empty expert has a partial chunk
  const int64_t ch_e = std::min<int64_t>(d.E, Tk) + ceil_div(Tk, nc_e);
  const int64_t ch_d = ceil_div(T, nc_d);
  const int64_t u_gu = ch_e * tiles_gu_e + ch_d * tiles_gu_d, u_dn = (ch_e + ch_d) * tiles_dn;
  ss.units = std::max(u_gu, u_dn);
  const int64_t p_gu_e = ch_e * tiles_gu_e * ss.gu_e, p_gu_d = ch_d * tiles_gu_d * ss.gu_d;
  const int64_t p_dn_e = ch_e * tiles_dn * ss.dn_e, p_dn_d = ch_d * tiles_dn * ss.dn_d;
  ss.pieces = std::max(p_gu_e + p_gu_d, p_dn_e + p_dn_d);
  // partials: [piece][64 rows][8 * nt tokens] fp32, problem by problem
  ss.partial_floats = kStreamTileRows * std::max(p_gu_e * nc_e + p_gu_d * nc_d,
                                                 p_dn_e * nc_e + p_dn_d * nc_d);
  return ss;
}

struct Layout {
  size_t status, rcounters, counters, logits, bhist, bbase, topk_idx, topk_w, offsets, sorted, inv;
  size_t xn_moe, xn_dense, aperm, h, y, hd, dense, partials, wr_hi, wr_lo, sched, total;
  size_t sx, h8, sh;  // fp8: token-row scales of the gathered rows, h in E4M3, h's scales
  size_t counters_bytes;
  int bn, split_gu, split_dgu, split_d, split_dd;
  StreamSplits ss;    // the weight-streaming kernel's splits (stream_path only)
};

Layout layout_of(const Dims& d) {
  Layout L{};
  const int64_t T = d.T, Tk = static_cast<int64_t>(d.T) * d.k;
  L.bn = choose_bn(d);
  const int kw = (d.int8 || d.fp8) ? 128 : 64;  // K per pipeline step of the expert GEMMs
  // expected tiles of the two launches (experts and the dense MLP share each launch)
  const double u = expected_used_experts(d);
  const double dense_nt = static_cast<double>(ceil_div(T, L.bn));
  const double tiles_gu = u * (d.I / 64) + dense_nt * (d.D / 64);
  const double tiles_dn = u * (d.H / 128) + dense_nt * (d.H / 128);
  L.split_gu = choose_split((d.H + kw - 1) / kw, L.bn, tiles_gu);
  L.split_dgu = choose_split(d.H / 64, L.bn, tiles_gu);
  L.split_d = choose_split((d.I + kw - 1) / kw, L.bn, tiles_dn);
  L.split_dd = choose_split(d.D / 64, L.bn, tiles_dn);
  // Upper bound of the N tiles: every non-empty expert has a partial tile.
  const int64_t ntl_e = std::min<int64_t>(d.E, Tk) + ceil_div(Tk, L.bn);
  const int64_t ntl_d = ceil_div(T, L.bn);
  const int64_t pieces_gu = (d.I / 64) * ntl_e * L.split_gu + (d.D / 64) * ntl_d * L.split_dgu;
  const int64_t pieces_dn = (d.H / 128) * ntl_e * L.split_d + (d.H / 128) * ntl_d * L.split_dd;
  int64_t pieces = std::max(pieces_gu, pieces_dn);
  bool any_split = L.split_gu > 1 || L.split_dgu > 1 || L.split_d > 1 || L.split_dd > 1;
  int64_t partial_bytes = any_split ? pieces * L.bn * 128 * 4 : 0;
  if (stream_path(d)) {
    // the weight-streaming kernel: one counter per (tile, chunk), [64][8] fp32 per piece
    L.ss = stream_splits(d);
    pieces = std::max(pieces, L.ss.units);
    const bool ssplit = L.ss.gu_e > 1 || L.ss.gu_d > 1 || L.ss.dn_e > 1 || L.ss.dn_d > 1;
    if (ssplit) partial_bytes = std::max<int64_t>(partial_bytes, L.ss.partial_floats * 4);
    any_split = any_split || ssplit;
  }
  const int nb = permute_blocks(static_cast<int>(Tk));

  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + std::max<size_t>(bytes, 1), kAlign);
    return at;
  };
  // status word, router counters and GEMM counters are contiguous: one memset clears them
  L.status = 0;
  L.rcounters = 256;
  L.counters = align_up(L.rcounters + static_cast<size_t>(router_counters(d.T)) * 4, 256);
  L.counters_bytes = static_cast<size_t>(pieces) * 4;
  off = align_up(L.counters + L.counters_bytes, kAlign);
  L.logits = take(static_cast<size_t>(T) * d.E * 4);
  L.bhist = take(static_cast<size_t>(nb) * d.E * 4);
  L.bbase = take(static_cast<size_t>(nb) * d.E * 4);
  L.topk_idx = take(Tk * 4);
  L.topk_w = take(Tk * 4);
  L.offsets = take((d.E + 1) * 4);
  L.sorted = take(Tk * 4);
  L.inv = take(Tk * 4);
  L.xn_moe = take(T * d.H * 2);
  L.xn_dense = take(T * d.H * 2);
  L.aperm = take(Tk * d.H * 2);
  L.h = take(Tk * d.I * 2);
  L.y = take(Tk * d.H * 2);
  L.hd = take(T * d.D * 2);
  L.dense = take(T * d.H * 4);
  L.partials = take(static_cast<size_t>(partial_bytes));
  // the tensor-core router's two-term split of the scaled router weights
  const size_t wr_bytes = router_uses_tc(d.T) ? static_cast<size_t>(d.E) * d.H * 2 : 0;
  L.wr_hi = take(wr_bytes);
  L.wr_lo = take(wr_bytes);
  L.sched = take(16);  // the GEMM launches' piece counters: [0..1] gate_up, [2..3] down
  // fp8: the gathered rows' E4M3 codes share the aperm buffer; their scales, h in E4M3
  // and h's row scales
  L.sx = take(d.fp8 ? Tk * 4 : 0);
  L.h8 = take(d.fp8 ? Tk * d.I : 0);
  L.sh = take(d.fp8 ? Tk * 4 : 0);
  L.total = off;
  return L;
}

moe_status_t check_ws(const Dims& d, void* ws, size_t ws_bytes, Layout* L) {
  *L = layout_of(d);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_WORKSPACE;
  if (ws_bytes < L->total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// ---------------------------------------------------------------- devices and TMA

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
int g_sm_count[64] = {0};

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

// K-major 2-D map: rows x cols elements, box of 128 bytes of K x box_rows rows.
bool encode_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows,
               CUtensorMapDataType dt, int elem_bytes, CUtensorMapSwizzle swz) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encoder();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * elem_bytes};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem_bytes), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  const CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 tile as the MMA reads it (128-byte swizzle).
bool encode_bf16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  return encode_2d(m, base, rows, cols, box_rows, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

// int8 weight tile for the converter warps: 128-byte rows of 128 codes, 128-byte swizzle.
bool encode_i8(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  return encode_2d(m, base, rows, cols, box_rows, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

// gate_up weights [groups][2F][K] (gate rows 0..F-1, up rows F..2F-1) as a 5-D map over
// (K, row in 8, gate|up, feature group of 8, group): one box of 128 bytes of K x 8 rows x
// gate|up x 8 groups lands as 8 gate rows, the matching 8 up rows, the next 8 gate
// rows, ...  The strides are not increasing (gate|up is outside the feature groups in
// memory but inside them in the box).
bool encode_gate_up(CUtensorMap* m, const void* base, int64_t groups, int64_t F, int64_t K,
                    bool int8) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encoder();
  if (fn == nullptr) return false;
  const int es = int8 ? 1 : 2;
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(K), 8, 2, static_cast<cuuint64_t>(F / 8),
                        static_cast<cuuint64_t>(groups)};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(K * es), static_cast<cuuint64_t>(F * K * es),
                           static_cast<cuuint64_t>(8 * K * es),
                           static_cast<cuuint64_t>(2 * F * K * es)};
  cuuint32_t box[5] = {static_cast<cuuint32_t>(128 / es), 8, 2, 8, 1};
  cuuint32_t el[5] = {1, 1, 1, 1, 1};
  const CUresult r =
      fn(m, int8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
         const_cast<void*>(base), dims, strides, box, el, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// ---------------------------------------------------------------- the expert / dense GEMMs

struct GemmJob {
  // experts (problem 0), may be absent
  bool experts;
  const void* a_rows;        // gathered xn_moe rows, [Tk][H]: bf16, fp16 (int8 experts)
                             // or E4M3 codes (fp8 experts)
  const float* a_scales;     // fp8: the gathered rows' scales [Tk]
  const void* w_gate_up;
  const void* w_down;
  const float* s_gate_up;
  const float* s_down;
  const uint8_t* b_gate_up;  // nvfp4 block scales
  const uint8_t* b_down;
  const int* offsets;
  const int* sorted_src;
  const float* topk_w;
  uint16_t* y;               // [Tk][H] fp16 expert outputs in sorted order, unweighted
  // dense MLP (problem 1 when experts are present, else problem 0), may be absent
  bool dense;
  const uint16_t* xn_dense;  // [T][H]
  const uint16_t* w_dgu;     // [2D][H]
  const uint16_t* w_dd;      // [H][D]
  void* dense_out;           // [T][H], bf16 or (dense_f32) fp32
  int dense_f32;
};

// Records ev[i] on s when a stage-event array was given.
bool mark(void* const* ev, int i, cudaStream_t s) {
  return ev == nullptr || cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s) == cudaSuccess;
}

// The routed tokens' rows in sorted order for the gate_up matmul: bf16 copies, fp16 copies
// (int8 experts) or per-row E4M3 codes and scales (fp8 experts).
moe_status_t gather_tokens(const Dims& d, const Layout& L, void* ws, const int* sorted,
                           const int* inv, const uint16_t* xn_moe, cudaStream_t s, bool pdl) {
  const int Tk = d.T * d.k;
  if (d.fp8)
    return cuda_status(launch_gather_quant_fp8(Tk, d.k, d.H, d.T, sorted, xn_moe,
                                               at<uint8_t>(ws, L.aperm), at<float>(ws, L.sx),
                                               s, pdl));
  return cuda_status(launch_gather_rows(Tk, d.k, d.H, d.T, sorted, inv, xn_moe,
                                        at<uint16_t>(ws, L.aperm), d.int8 || d.nvfp4, s, pdl));
}

// The two GEMM launches on the weight-streaming kernel.
moe_status_t run_stream_gemms(const Dims& d, const Layout& L, void* ws, const GemmJob& j,
                              cudaStream_t s, bool first_kernel, void* const* ev) {
  const int Tk = d.T * d.k;
  const int sms = sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  uint16_t* h = at<uint16_t>(ws, L.h);
  uint16_t* hd = at<uint16_t>(ws, L.hd);
  StreamParams gu{}, dn{};
  for (StreamParams* P : {&gu, &dn}) {
    P->partials = at<float>(ws, L.partials);
    P->counters = at<unsigned>(ws, L.counters);
  }
  int np = 0;
  if (j.experts) {
    const int wt = d.nvfp4 ? kStreamNvfp4 : kStreamInt8;
    StreamProblem& a = gu.prob[np];
    a.kind = 0; a.wtype = wt; a.groups = d.E; a.offsets = j.offsets; a.n_tokens = Tk;
    a.K = d.H; a.rows = 2 * d.I; a.F = d.I; a.w = j.w_gate_up; a.wscale = j.s_gate_up;
    a.bscale = j.b_gate_up;
    a.b = static_cast<const uint16_t*>(j.a_rows); a.out = h; a.out_type = kOutF16; a.out_ld = d.I;
    a.split = L.ss.gu_e; a.nt = L.ss.nt_e;
    StreamProblem& b = dn.prob[np];
    b.kind = 1; b.wtype = wt; b.groups = d.E; b.offsets = j.offsets; b.n_tokens = Tk;
    b.K = d.I; b.rows = d.H; b.F = d.H; b.w = j.w_down; b.wscale = j.s_down; b.bscale = j.b_down;
    b.b = h; b.out = j.y; b.out_type = kOutF16; b.out_ld = d.H;
    b.split = L.ss.dn_e; b.nt = L.ss.nt_e;
    ++np;
  }
  if (j.dense) {
    StreamProblem& a = gu.prob[np];
    a.kind = 0; a.wtype = kStreamBf16; a.groups = 1; a.offsets = nullptr; a.n_tokens = d.T;
    a.K = d.H; a.rows = 2 * d.D; a.F = d.D; a.w = j.w_dgu; a.b = j.xn_dense; a.out = hd;
    a.out_type = kOutBf16; a.out_ld = d.D; a.split = L.ss.gu_d; a.nt = L.ss.nt_d;
    StreamProblem& b = dn.prob[np];
    b.kind = 1; b.wtype = kStreamBf16; b.groups = 1; b.offsets = nullptr; b.n_tokens = d.T;
    b.K = d.D; b.rows = d.H; b.F = d.H; b.w = j.w_dd; b.b = hd; b.out = j.dense_out;
    b.out_type = j.dense_f32 ? kOutF32 : kOutBf16; b.out_ld = d.H; b.split = L.ss.dn_d;
    b.nt = L.ss.nt_d;
    ++np;
  }
  gu.nprob = dn.nprob = np;
  moe_status_t st = cuda_status(launch_stream_gemm(gu, sms, s, !first_kernel));
  if (st != MOE_OK) return st;
  if (!mark(ev, 4, s)) return MOE_ERR_CUDA;
  st = cuda_status(launch_stream_gemm(dn, sms, s, true));
  if (st != MOE_OK) return st;
  return mark(ev, 5, s) ? MOE_OK : MOE_ERR_CUDA;
}

// The counters in the workspace start at zero (the caller zeroes a new workspace once)
// and every kernel that uses one returns it to zero, so no call clears them.
// first_kernel: the gate_up launch is the entry point's first kernel (no dependent
// launch on whatever the stream ran before).
moe_status_t run_gemms(const Dims& d, const Layout& L, void* ws, const GemmJob& j,
                       cudaStream_t s, bool first_kernel, void* const* ev = nullptr) {
  if (stream_path(d)) return run_stream_gemms(d, L, ws, j, s, first_kernel, ev);
  const int64_t Tk = static_cast<int64_t>(d.T) * d.k;
  const int grid = sm_count();
  if (grid <= 0) return MOE_ERR_CUDA;
  uint16_t* h = at<uint16_t>(ws, L.h);
  uint16_t* hd = at<uint16_t>(ws, L.hd);

  GemmParams gu{}, dn{};
  GemmMaps mgu{}, mdn{};
  // int8 experts: the launches take the converter-warp variant (int8 A tiles are turned
  // into fp16 in tensor memory; the bf16 dense MLP in the same launch reads its A tiles
  // from shared memory as usual).
  const bool w8 = j.experts && d.int8;
  gu.sched = at<unsigned>(ws, L.sched);
  dn.sched = at<unsigned>(ws, L.sched) + 2;  // the down launch may start before gate_up ends
  for (GemmParams* P : {&gu, &dn}) {
    P->partials = at<float>(ws, L.partials);
    P->counters = at<unsigned>(ws, L.counters);
    P->status = at<unsigned>(ws, L.status);
    P->timeout_ns = kWaitTimeoutNs;
    P->int8_weights = w8 ? 1 : 0;
  }
  auto encode_a = [&](CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows,
                      bool int8) {
    return int8 ? encode_i8(m, base, rows, cols, box_rows)
                : encode_bf16(m, base, rows, cols, box_rows);
  };
  // CTA pairs load half of each token tile.  A pair takes two M tiles; with an odd count
  // the last pair's second tile is idle, which costs more than pairs save when the tiles
  // are full (tensor-bound), and less when most tiles are partly filled (weight-stream
  // bound: mean tokens per expert below the tile width).
  const bool pairs_ok = gemm_pairs_allowed(L.bn, w8);
  const bool streaming = static_cast<double>(d.T) * d.k / d.E < L.bn;
  const bool gu_pairs = pairs_ok && (streaming || ((!j.experts || (d.I / 64) % 2 == 0) &&
                                                   (!j.dense || (d.D / 64) % 2 == 0)));
  const bool dn_pairs = pairs_ok && (streaming || (d.H / 128) % 2 == 0);
  gu.pairs = gu_pairs ? 1 : 0;
  dn.pairs = dn_pairs ? 1 : 0;
  const int bbox_gu = gu_pairs ? L.bn / 2 : L.bn;
  const int bbox_dn = dn_pairs ? L.bn / 2 : L.bn;
  int np = 0;
  if (j.experts) {
    GemmProblem& a = gu.prob[np];
    a = GemmProblem{};
    // int8 and fp8 steps cover 128 K (a ragged last step reads zeros past K through the
    // maps)
    const int kw = (d.int8 || d.fp8) ? 128 : 64;
    a.kind = 0; a.groups = d.E; a.offsets = j.offsets; a.n_tokens = static_cast<int>(Tk);
    a.k_steps = (d.H + kw - 1) / kw; a.m_tiles = d.I / 64; a.w_rows_per_group = 2 * d.I; a.nw = d.I;
    a.split = std::min(L.split_gu, a.k_steps); a.map = np; a.out = h; a.out_ld = d.I;
    a.wscale = j.s_gate_up;
    a.w8 = d.int8;
    a.f16 = d.int8;  // int8 codes become fp16 (exact); the gathered rows and h are fp16
    a.fp8 = d.fp8;   // E4M3 weights times E4M3 token rows, each row with its scale
    a.xscale = d.fp8 ? j.a_scales : nullptr;
    GemmProblem& b = dn.prob[np];
    b = GemmProblem{};
    b.kind = 1; b.groups = d.E; b.offsets = j.offsets; b.n_tokens = static_cast<int>(Tk);
    b.k_steps = (d.I + kw - 1) / kw; b.m_tiles = d.H / 128; b.w_rows_per_group = d.H; b.nw = 0;
    b.split = std::min(L.split_d, b.k_steps); b.map = np; b.out = j.y; b.out_type = kOutF16;
    b.out_ld = d.H;
    b.wscale = j.s_down; b.w8 = d.int8; b.f16 = d.int8;
    b.fp8 = d.fp8;
    b.xscale = d.fp8 ? at<float>(ws, L.sh) : nullptr;
    // 8-bit weights (int8, E4M3) are byte tiles of 128 K; E4M3 token rows likewise
    const bool w1 = d.int8 || d.fp8;
    if (!encode_gate_up(&mgu.a[np], j.w_gate_up, d.E, d.I, d.H, w1) ||
        !(d.fp8 ? encode_i8(&mgu.b[np], j.a_rows, Tk, d.H, bbox_gu)
                : encode_bf16(&mgu.b[np], j.a_rows, Tk, d.H, bbox_gu)) ||
        !encode_a(&mdn.a[np], j.w_down, static_cast<int64_t>(d.E) * d.H, d.I, 128, w1) ||
        !(d.fp8 ? encode_i8(&mdn.b[np], at<uint8_t>(ws, L.h8), Tk, d.I, bbox_dn)
                : encode_bf16(&mdn.b[np], h, Tk, d.I, bbox_dn)))
      return MOE_ERR_CUDA;
    ++np;
  }
  if (j.dense) {
    GemmProblem& a = gu.prob[np];
    a = GemmProblem{};
    a.kind = 0; a.groups = 1; a.offsets = nullptr; a.n_tokens = d.T;
    a.k_steps = d.H / 64; a.m_tiles = d.D / 64; a.w_rows_per_group = 2 * d.D; a.nw = d.D;
    a.split = L.split_dgu; a.map = np; a.out = hd; a.out_ld = d.D;
    GemmProblem& b = dn.prob[np];
    b = GemmProblem{};
    b.kind = 1; b.groups = 1; b.offsets = nullptr; b.n_tokens = d.T;
    b.k_steps = d.D / 64; b.m_tiles = d.H / 128; b.w_rows_per_group = d.H;
    b.split = L.split_dd; b.map = np; b.out = j.dense_out;
    b.out_type = j.dense_f32 ? kOutF32 : kOutBf16;
    b.out_ld = d.H;
    if (!encode_gate_up(&mgu.a[np], j.w_dgu, 1, d.D, d.H, false) ||
        !encode_bf16(&mgu.b[np], j.xn_dense, d.T, d.H, bbox_gu) ||
        !encode_a(&mdn.a[np], j.w_dd, d.H, d.D, 128, false) ||
        !encode_bf16(&mdn.b[np], hd, d.T, d.D, bbox_dn))
      return MOE_ERR_CUDA;
    ++np;
  }
  gu.nprob = dn.nprob = np;
  if (np == 1) {  // unused second set: a valid copy of the first
    mgu.a[1] = mgu.a[0]; mgu.b[1] = mgu.b[0];
    mdn.a[1] = mdn.a[0]; mdn.b[1] = mdn.b[0];
  }
  // after a kernel of the same entry point the gate_up launch overlaps that kernel's tail
  // (programmatic dependent launch)
  moe_status_t st = cuda_status(launch_grouped_gemm(L.bn, mgu, gu, grid, s, !first_kernel));
  if (st != MOE_OK) return st;
  // fp8 experts: h (bf16, sorted order) quantised per row for the down matmul
  if (j.experts && d.fp8 &&
      (st = cuda_status(launch_gather_quant_fp8(static_cast<int>(Tk), 1, d.I, static_cast<int>(Tk),
                                                nullptr, h, at<uint8_t>(ws, L.h8),
                                                at<float>(ws, L.sh), s, true))) != MOE_OK)
    return st;
  if (!mark(ev, 4, s)) return MOE_ERR_CUDA;
  st = cuda_status(launch_grouped_gemm(L.bn, mdn, dn, grid, s, true));
  if (st != MOE_OK) return st;
  return mark(ev, 5, s) ? MOE_OK : MOE_ERR_CUDA;
}

// Inputs and outputs of the router step.
struct RouteJob {
  const uint16_t* x;
  const uint16_t* router_scale;
  const uint16_t* w_router;
  const float* logit_bias;
  const uint16_t* per_expert_scale;
  const uint16_t* g_pre_moe;
  const uint16_t* g_pre_dense;
  int* topk_idx;
  float* topk_w;
  uint16_t* xn_moe;
  uint16_t* xn_dense;
  int* offsets;  // with sorted_src and inv_pos: sort the pairs in the same launch; or NULL
  int* sorted_src;
  int* inv_pos;
  uint16_t* aperm;  // with the sort: gather the routed rows there too (router_gathers); or NULL
  bool aperm_f16;
};

// The router step, launched as the first kernel of the entry point: the tensor-core
// router for large batches, the small-batch one (router.cu) for small ones.  Only the
// small-batch router sorts the pairs in the same launch (r.offsets); the caller asks for
// it for batches of the small-batch router.
moe_status_t run_router(const Dims& d, const Layout& L, void* ws, const RouteJob& r,
                        cudaStream_t s) {
  unsigned* counters = at<unsigned>(ws, L.rcounters);
  unsigned* status = at<unsigned>(ws, L.status);
  if (!router_uses_tc(d.T))
    return cuda_status(launch_router(d.T, d.H, d.E, d.k, d.eps, r.x, r.router_scale, r.w_router,
                                     r.logit_bias, r.per_expert_scale, r.g_pre_moe,
                                     r.g_pre_dense, r.xn_moe, r.xn_dense,
                                     at<float>(ws, L.logits), r.topk_idx, r.topk_w, counters,
                                     status, r.offsets, r.sorted_src, r.inv_pos, r.aperm,
                                     r.aperm_f16, s));
  uint16_t* whi = at<uint16_t>(ws, L.wr_hi);
  uint16_t* wlo = at<uint16_t>(ws, L.wr_lo);
  const int ne = (d.E + 15) / 16 * 16 / router_tc_slices(d.T, d.E);  // experts per CTA
  if (r.offsets != nullptr || r.aperm != nullptr) return MOE_ERR_INVALID_ARG;  // not on this path
  RouterTcMaps m;
  if (!encode_bf16(&m.x, r.x, d.T, d.H, 128) || !encode_bf16(&m.whi, whi, d.E, d.H, ne) ||
      !encode_bf16(&m.wlo, wlo, d.E, d.H, ne))
    return MOE_ERR_CUDA;
  return cuda_status(launch_router_tc(m, d.T, d.H, d.E, d.k, d.eps, r.w_router, r.router_scale,
                                      whi, wlo, r.logit_bias, r.per_expert_scale, r.g_pre_moe,
                                      r.g_pre_dense, r.xn_moe, r.xn_dense, r.topk_idx, r.topk_w,
                                      at<float>(ws, L.logits), counters, status, kWaitTimeoutNs,
                                      s));
}

bool w_ok(const moe_expert_weights_t* w, const Dims& d) {
  if (w == nullptr || w->w_gate_up == nullptr || w->w_down == nullptr) return false;
  if (!aligned16(w->w_gate_up) || !aligned16(w->w_down)) return false;
  if (d.nvfp4) {
    // block scales are copied four bytes at a time, the matrix scales read one by one
    return w->s_gate_up != nullptr && w->s_down != nullptr && w->b_gate_up != nullptr &&
           w->b_down != nullptr && (reinterpret_cast<uintptr_t>(w->b_gate_up) & 3u) == 0 &&
           (reinterpret_cast<uintptr_t>(w->b_down) & 3u) == 0;
  }
  if (w->b_gate_up != nullptr || w->b_down != nullptr) return false;
  if (d.int8 || d.fp8) return w->s_gate_up != nullptr && w->s_down != nullptr;
  return w->s_gate_up == nullptr && w->s_down == nullptr;
}

}  // namespace

// ================================================================ the C interface

extern "C" {

int32_t moe_abi_version(void) { return 7; }

int32_t moe_block_launch_count(const moe_config_t* cfg, int32_t T) {
  Dims d;
  if (check_cfg(cfg, T, &d) != MOE_OK) return -1;
  if (T == 0) return 0;
  const int Tk = d.T * d.k;
  // the same decisions as moe_block_forward
  const bool tc = router_uses_tc(d.T);
  const bool fused_sort = !tc && permute_blocks(Tk) == 0;
  int n = tc ? 2 : 1;                                     // router (prep + router)
  if (!fused_sort) n += permute_blocks(Tk) == 0 ? 1 : 3;  // permutation
  if (d.fp8) n += 1;                                      // h quantised for the down matmul
  if (!(fused_sort && router_gathers(d))) n += 1;         // gather
  return n + 3;                                           // gate_up, down, combine
}

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported size";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "CUDA call failed";
    case MOE_ERR_DEVICE_TIMEOUT: return "a bounded device wait ran out";
  }
  return "unknown status";
}

size_t moe_workspace_size(const moe_config_t* cfg, int32_t T) {
  Dims d;
  if (check_cfg(cfg, T, &d) != MOE_OK) return 0;
  return layout_of(d).total;
}

moe_status_t moe_router(const moe_config_t* cfg, int32_t T, const moe_bf16_t* x,
                        const moe_bf16_t* router_scale, const moe_bf16_t* w_router,
                        const float* logit_bias, const moe_bf16_t* per_expert_scale,
                        const moe_bf16_t* g_pre_moe, const moe_bf16_t* g_pre_dense,
                        int32_t* topk_idx, float* topk_w, moe_bf16_t* xn_moe,
                        moe_bf16_t* xn_dense, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  moe_status_t st = check_cfg(cfg, T, &d);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  for (const void* p : {(const void*)x, (const void*)router_scale, (const void*)w_router,
                        (const void*)per_expert_scale, (const void*)g_pre_moe,
                        (const void*)g_pre_dense, (const void*)topk_idx, (const void*)topk_w,
                        (const void*)xn_moe, (const void*)xn_dense})
    if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (logit_bias != nullptr && !aligned16(logit_bias)) return MOE_ERR_INVALID_ARG;
  Layout L;
  if ((st = check_ws(d, ws, ws_bytes, &L)) != MOE_OK) return st;
  const RouteJob r{x, router_scale, w_router, logit_bias, per_expert_scale, g_pre_moe,
                   g_pre_dense, topk_idx, topk_w, xn_moe, xn_dense, nullptr, nullptr, nullptr};
  return run_router(d, L, ws, r, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_permute(const moe_config_t* cfg, int32_t T, const int32_t* topk_idx,
                         int32_t* expert_offsets, int32_t* sorted_src, int32_t* inv_pos,
                         void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  moe_status_t st = check_cfg(cfg, T, &d);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  for (const void* p : {(const void*)topk_idx, (const void*)expert_offsets,
                        (const void*)sorted_src, (const void*)inv_pos})
    if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  Layout L;
  if ((st = check_ws(d, ws, ws_bytes, &L)) != MOE_OK) return st;
  return cuda_status(launch_permute(d.T * d.k, d.E, topk_idx, expert_offsets, sorted_src, inv_pos,
                                    at<int>(ws, L.bhist), at<int>(ws, L.bbase),
                                    static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ffn_forward(const moe_config_t* cfg, int32_t T, const moe_bf16_t* xn_moe,
                             const float* topk_w, const int32_t* expert_offsets,
                             const int32_t* sorted_src, const int32_t* inv_pos,
                             const moe_expert_weights_t* experts, moe_bf16_t* moe_out,
                             void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  moe_status_t st = check_cfg(cfg, T, &d);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  for (const void* p : {(const void*)xn_moe, (const void*)topk_w, (const void*)expert_offsets,
                        (const void*)sorted_src, (const void*)inv_pos, (const void*)moe_out})
    if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (!w_ok(experts, d)) return MOE_ERR_INVALID_ARG;
  Layout L;
  if ((st = check_ws(d, ws, ws_bytes, &L)) != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint16_t* y = at<uint16_t>(ws, L.y);
  if ((st = gather_tokens(d, L, ws, sorted_src, inv_pos, xn_moe, s, false)) != MOE_OK) return st;
  GemmJob j{};
  j.experts = true;
  j.a_rows = at<uint8_t>(ws, L.aperm);
  j.a_scales = at<float>(ws, L.sx);
  j.w_gate_up = experts->w_gate_up;
  j.w_down = experts->w_down;
  j.s_gate_up = experts->s_gate_up;
  j.s_down = experts->s_down;
  j.b_gate_up = experts->b_gate_up;
  j.b_down = experts->b_down;
  j.offsets = expert_offsets;
  j.sorted_src = sorted_src;
  j.topk_w = topk_w;
  j.y = y;
  if ((st = run_gemms(d, L, ws, j, s, false)) != MOE_OK) return st;
  return cuda_status(launch_combine_moe(d.T, d.H, d.k, y, inv_pos, sorted_src, topk_w, moe_out,
                                        s, true));
}

moe_status_t dense_mlp_forward(const moe_config_t* cfg, int32_t T, const moe_bf16_t* xn_dense,
                               const moe_bf16_t* w_gate_up, const moe_bf16_t* w_down,
                               moe_bf16_t* dense_out, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  moe_status_t st = check_cfg(cfg, T, &d);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  for (const void* p : {(const void*)xn_dense, (const void*)w_gate_up, (const void*)w_down,
                        (const void*)dense_out})
    if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  Layout L;
  if ((st = check_ws(d, ws, ws_bytes, &L)) != MOE_OK) return st;
  GemmJob j{};
  j.dense = true;
  j.xn_dense = xn_dense;
  j.w_dgu = w_gate_up;
  j.w_dd = w_down;
  j.dense_out = dense_out;
  return run_gemms(d, L, ws, j, static_cast<cudaStream_t>(stream), true);
}

moe_status_t moe_block_forward(const moe_config_t* cfg, int32_t T, const moe_bf16_t* x,
                               const moe_block_weights_t* w, moe_bf16_t* out,
                               moe_bf16_t* moe_out, void* ws, size_t ws_bytes, void* stream,
                               void* const* ev) {
  Dims d;
  moe_status_t st = check_cfg(cfg, T, &d);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (w == nullptr) return MOE_ERR_INVALID_ARG;
  for (const void* p : {(const void*)x, (const void*)out, (const void*)w->router_scale,
                        (const void*)w->w_router, (const void*)w->per_expert_scale,
                        (const void*)w->g_pre_moe, (const void*)w->g_pre_dense,
                        (const void*)w->g_post_ff, (const void*)w->w_dense_gate_up,
                        (const void*)w->w_dense_down})
    if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  for (const void* p : {(const void*)moe_out, (const void*)w->logit_bias,
                        (const void*)w->g_post_moe, (const void*)w->g_post_dense})
    if (p != nullptr && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (!w_ok(&w->experts, d)) return MOE_ERR_INVALID_ARG;
  Layout L;
  if ((st = check_ws(d, ws, ws_bytes, &L)) != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int Tk = d.T * d.k;
  int* topk_idx = at<int>(ws, L.topk_idx);
  float* topk_w = at<float>(ws, L.topk_w);
  int* offsets = at<int>(ws, L.offsets);
  int* sorted = at<int>(ws, L.sorted);
  int* inv = at<int>(ws, L.inv);
  uint16_t* xn_moe = at<uint16_t>(ws, L.xn_moe);
  uint16_t* xn_dense = at<uint16_t>(ws, L.xn_dense);
  uint16_t* aperm = at<uint16_t>(ws, L.aperm);
  uint16_t* y = at<uint16_t>(ws, L.y);
  float* dense = at<float>(ws, L.dense);

  if (ev != nullptr)
    for (int i = 0; i < MOE_BLOCK_EVENTS; ++i)
      if (ev[i] == nullptr) return MOE_ERR_INVALID_ARG;
  if (!mark(ev, 0, s)) return MOE_ERR_CUDA;
  const bool fused_sort = !router_uses_tc(d.T) && permute_blocks(Tk) == 0;
  const bool rgather = fused_sort && router_gathers(d);
  const RouteJob r{x, w->router_scale, w->w_router, w->logit_bias, w->per_expert_scale,
                   w->g_pre_moe, w->g_pre_dense, topk_idx, topk_w, xn_moe, xn_dense,
                   fused_sort ? offsets : nullptr, sorted, inv,
                   rgather ? aperm : nullptr, false};
  if ((st = run_router(d, L, ws, r, s)) != MOE_OK) return st;
  if (!mark(ev, 1, s)) return MOE_ERR_CUDA;
  if (!fused_sort &&
      (st = cuda_status(launch_permute(Tk, d.E, topk_idx, offsets, sorted, inv, at<int>(ws, L.bhist),
                                       at<int>(ws, L.bbase), s, true))) != MOE_OK)
    return st;
  if (!mark(ev, 2, s)) return MOE_ERR_CUDA;
  if (!rgather && (st = gather_tokens(d, L, ws, sorted, inv, xn_moe, s, true)) != MOE_OK)
    return st;
  if (!mark(ev, 3, s)) return MOE_ERR_CUDA;
  GemmJob j{};
  j.experts = true;
  j.a_rows = aperm;
  j.a_scales = at<float>(ws, L.sx);
  j.w_gate_up = w->experts.w_gate_up;
  j.w_down = w->experts.w_down;
  j.s_gate_up = w->experts.s_gate_up;
  j.s_down = w->experts.s_down;
  j.b_gate_up = w->experts.b_gate_up;
  j.b_down = w->experts.b_down;
  j.offsets = offsets;
  j.sorted_src = sorted;
  j.topk_w = topk_w;
  j.y = y;
  j.dense = true;
  j.xn_dense = xn_dense;
  j.w_dgu = w->w_dense_gate_up;
  j.w_dd = w->w_dense_down;
  j.dense_out = dense;
  j.dense_f32 = 1;
  if ((st = run_gemms(d, L, ws, j, s, false, ev)) != MOE_OK) return st;
  if ((st = cuda_status(launch_combine_block(d.T, d.H, d.k, d.eps, x, y, inv, nullptr, topk_w,
                                             dense, w->g_post_moe,
                                             w->g_post_dense, w->g_post_ff, out, moe_out, s,
                                             true))) != MOE_OK)
    return st;
  return mark(ev, 6, s) ? MOE_OK : MOE_ERR_CUDA;
}

int32_t moe_stack_chunk_tokens(int32_t chunk_tokens) {
  constexpr int32_t kSnap = 1024, kMax = 32768;
  const int32_t c = chunk_tokens / kSnap * kSnap;
  return std::min(kMax, std::max(kSnap, c));
}

size_t moe_stack_workspace_size(const moe_config_t* cfg, int32_t chunk_tokens) {
  Dims d;
  const int32_t c = moe_stack_chunk_tokens(chunk_tokens);
  if (check_cfg(cfg, c, &d) != MOE_OK) return 0;
  // the block's workspace, then two [chunk][H] bf16 buffers for the residual chain
  const size_t block = align_up(layout_of(d).total, kAlign);
  return block + 2 * align_up(static_cast<size_t>(c) * d.H * 2, kAlign);
}

moe_status_t moe_stack_forward(const moe_config_t* cfg, int32_t T, const moe_bf16_t* x,
                               const moe_block_weights_t* layers, int32_t n_layers,
                               moe_bf16_t* out, int32_t chunk_tokens, void* ws,
                               size_t ws_bytes, void* stream) {
  Dims d;
  const int32_t c = moe_stack_chunk_tokens(chunk_tokens);
  moe_status_t st = check_cfg(cfg, c, &d);
  if (st != MOE_OK) return st;
  if (T < 0 || n_layers < 1 || layers == nullptr) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (x == nullptr || out == nullptr || !aligned16(x) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 ||
      ws_bytes < moe_stack_workspace_size(cfg, chunk_tokens))
    return MOE_ERR_WORKSPACE;
  const size_t block = align_up(layout_of(d).total, kAlign);
  const size_t buf = align_up(static_cast<size_t>(c) * d.H * 2, kAlign);
  moe_bf16_t* ping[2] = {at<moe_bf16_t>(ws, block), at<moe_bf16_t>(ws, block + buf)};
  for (int32_t t0 = 0; t0 < T; t0 += c) {
    const int32_t n = std::min(c, T - t0);
    const size_t row0 = static_cast<size_t>(t0) * d.H;
    const moe_bf16_t* in = x + row0;
    for (int32_t l = 0; l < n_layers; ++l) {
      moe_bf16_t* dst = l == n_layers - 1 ? out + row0 : ping[l & 1];
      // the block's own checks run on every call; its workspace is the first part of ws
      st = moe_block_forward(cfg, n, in, &layers[l], dst, nullptr, ws, block, stream, nullptr);
      if (st != MOE_OK) return st;
      in = dst;
    }
  }
  return MOE_OK;
}

moe_status_t moe_quantize_int8(const moe_bf16_t* w, int64_t rows, int32_t cols, int8_t* q,
                               float* scales, void* stream) {
  if (rows < 0 || cols < 8 || cols > 65536 || cols % 8) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (rows > (int64_t(1) << 34)) return MOE_ERR_UNSUPPORTED;
  if (w == nullptr || q == nullptr || scales == nullptr || !aligned16(w) || !aligned16(q))
    return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(scales) & 3u) != 0) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_quantize_int8(w, rows, cols, q, scales, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_quantize_fp8(const moe_bf16_t* w, int64_t rows, int32_t cols, uint8_t* q,
                              float* scales, void* stream) {
  if (rows < 0 || cols < 8 || cols > 65536 || cols % 8) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (rows > (int64_t(1) << 34)) return MOE_ERR_UNSUPPORTED;
  if (w == nullptr || q == nullptr || scales == nullptr || !aligned16(w) || !aligned16(q))
    return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(scales) & 3u) != 0) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_quantize_fp8(w, rows, cols, q, scales, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_quantize_nvfp4(const moe_bf16_t* w, int64_t matrices, int64_t rows,
                                int32_t cols, uint8_t* q, uint8_t* block_scales,
                                float* tensor_scales, void* stream) {
  if (matrices < 0 || rows < 1 || cols < 16 || cols > 65536 || cols % 16) return MOE_ERR_INVALID_ARG;
  if (matrices == 0) return MOE_OK;
  if (matrices > (int64_t(1) << 24) || matrices * rows > (int64_t(1) << 34)) return MOE_ERR_UNSUPPORTED;
  if (w == nullptr || q == nullptr || block_scales == nullptr || tensor_scales == nullptr ||
      !aligned16(w) || (reinterpret_cast<uintptr_t>(q) & 7u) != 0 ||
      (reinterpret_cast<uintptr_t>(tensor_scales) & 3u) != 0)
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_quantize_nvfp4(w, matrices, rows, cols, q, block_scales, tensor_scales,
                                           static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_wait_selftest(void* ws, size_t ws_bytes, uint64_t timeout_ns, void* stream) {
  if (ws == nullptr || ws_bytes < 256 || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return MOE_ERR_WORKSPACE;
  if (timeout_ns < 1000ull || timeout_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;
  return cuda_status(
      launch_wait_selftest(static_cast<unsigned*>(ws), timeout_ns, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_check_device_status(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < 256 || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned host = 0;
  if (cudaMemcpyAsync(&host, ws, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (host == 0) return MOE_OK;
  if (cudaMemsetAsync(ws, 0, sizeof(unsigned), s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  return host == static_cast<unsigned>(MOE_ERR_DEVICE_TIMEOUT) ? MOE_ERR_DEVICE_TIMEOUT : MOE_ERR_CUDA;
}

}  // extern "C"

// ================================================================ no-workspace permutation
//
// For callers that can hand the library no scratch memory (see moe_permute_noalloc in
// include/moe_ffn.h).  The multi-block counting sort needs per-block histograms and
// per-block bases (2 x 256 blocks x 256 experts ints); they live in this fixed device
// array instead of a caller workspace.  Its host-side name is only a handle: the device
// address is looked up on every call with cudaGetSymbolAddress (an allocation-free
// lookup), in the context current at the call, so that no address outlives a device
// reset or belongs to another context of the same device.

namespace {

constexpr int kNoAllocMaxBlocks = 256;  // the multi-block sort uses at most 256 blocks
constexpr int kNoAllocInts = 2 * kNoAllocMaxBlocks * 256;
static_assert(kNoAllocInts * 4 == MOE_PERMUTE_NOALLOC_SCRATCH_BYTES, "scratch size");

static __device__ __align__(256) int g_permute_scratch[kNoAllocInts];

// Device address of the scratch array in the current context (NULL on failure).
int* permute_scratch() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

}  // namespace

extern "C" moe_status_t moe_permute_noalloc(const moe_config_t* cfg, int32_t T,
                                            const int32_t* topk_idx, int32_t* expert_offsets,
                                            int32_t* sorted_src, int32_t* inv_pos,
                                            void* stream) {
  Dims d;
  moe_status_t st = check_cfg(cfg, T, &d);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  for (const void* p : {(const void*)topk_idx, (const void*)expert_offsets,
                        (const void*)sorted_src, (const void*)inv_pos})
    if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const int64_t n = static_cast<int64_t>(d.T) * d.k;
  if (n > MOE_PERMUTE_NOALLOC_MAX_PAIRS) return MOE_ERR_UNSUPPORTED;
  int* scratch = permute_scratch();
  if (scratch == nullptr) return MOE_ERR_CUDA;
  // block histograms in the first half, block bases in the second (nb * E <= 256 * 256)
  return cuda_status(launch_permute(static_cast<int>(n), d.E, topk_idx, expert_offsets,
                                    sorted_src, inv_pos, scratch,
                                    scratch + kNoAllocMaxBlocks * 256,
                                    static_cast<cudaStream_t>(stream)));
}
