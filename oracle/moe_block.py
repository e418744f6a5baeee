"""Plain fp64 CPU oracle of the hybrid MoE feed-forward block (Gemma-4-26B-A4B shape).

TEST INFRASTRUCTURE ONLY.  The test suite, the package smoke check and the benchmark's
CPU-baseline leg may call this module; the product path never does, and this module
shares no code with the CUDA path.  It imports only numpy.

It computes the block as the model pages define it, one definition per function, in
float64.  Inputs are the same bf16 / int8 / fp32 tensors the GPU receives: bf16 is
passed as uint16 bit patterns and widened exactly.

Sources (page title, section):
  [P1] "Gemma-4 26B-A4B (MoE) on AWS Inferentia2", sections "The architecture (a
       dual-path FFN)" and "How it works (the recipe)".
  [P2] "Gemma-4 26B-A4B (MoE, int8 experts) on AWS Inferentia2", opening paragraph
       and "How it works".
  [P5] "Gemma-4 26B-A4B-it - ONNX MoE text decoder", table "Truthful graph
       contracts" (rows "Mixture of Experts", "MoE topology", "Router").
  [P6] "Gemma 4 26B-A4B IT" (inference recipe), section "Quantized Variants" and its
       variant list: FP8 (E4M3) weights with dynamic per-token activation quantization.

Readings taken where the pages leave a step open:
  R1  RMSNorm multiplies by the stored gain as-is, eps inside the square root.
  R2  "four feed-forward layernorms" = a pre and a post norm on each branch, followed
      by the post_ff norm of the sum; a post norm given as None is skipped.
  R3  The router reads the un-normed block input x and applies its own scale-free norm.
  R4  The router's learned scale is a per-channel vector [H]; hidden_size^-0.5 a scalar.
  R5  An optional fp32 logit offset b[E] stands in for the synthetic router bias.
  R6  Top-k is taken on the logits (softmax is monotone), ties to the lower index, and
      the selected experts are ordered by (logit descending, index ascending).
  R7  per_expert_scale multiplies the renormalised weight of its expert.
  R8  gate_up rows 0..I-1 are the gate projection and rows I..2I-1 the up projection.
  R9  int8 experts: per output row s = max|w| / 127 (fp32), q = round-half-even(w / s)
      clamped to [-127, 127]; an all-zero row takes s = 1.
  R18 NVFP4 experts ([P6] variant list: "NVFP4 (4-bit) quantized weights", the format
      named, not defined): weight-only; E2M1 values (1 sign, 2 exponent bits of bias 1,
      1 mantissa bit: 0, 0.5, 1, 1.5, 2, 3, 4, 6) with one E4M3 scale per 16 consecutive
      weights of a row and one fp32 scale per weight matrix.  Quantiser (a reading):
      t = max|W| / (448 * 6) in fp32 (1 for an all-zero matrix); block scale
      b = E4M3(max|block| / 6 / t); codes E2M1(w / (b t)), nearest, ties to even,
      saturating at +-6 (a block whose scale rounds to zero gets zero codes).  The weight
      is q * b * t.
  R17 fp8 experts ([P6]): E4M3 as the OCP 8-bit format defines it (1 sign, 4 exponent
      bits of bias 7, 3 mantissa bits, subnormals, no infinities, largest finite 448).
      Weights per output row and activations per token row (the rows entering each
      expert matmul: the routed token's xn_moe, and h) take s = max|v| / 448 (fp32, an
      all-zero row s = 1) and codes e4m3(v / s): the fp32 quotient rounded to nearest
      even on the E4M3 grid, saturating at +-448.  The activations are quantised from
      the bf16 values the expert matmuls receive (xn_moe and h are bf16 tensors), so both
      sides take each rounding decision from the same number.
"""
from __future__ import annotations

import numpy as np

SQRT_2_OVER_PI = np.sqrt(2.0 / np.pi)
GELU_CUBIC = 0.044715


# ----------------------------------------------------------------------------- formats

def bf16(u16) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float64, exactly."""
    u = np.asarray(u16, dtype=np.uint16)
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------- pieces

def rms_norm(v: np.ndarray, gain, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: v / sqrt(mean(v^2) + eps), times gain (R1).

    gain=None gives the scale-free form the router uses ([P5] Router row).
    """
    v = np.asarray(v, dtype=np.float64)
    r = v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    return r if gain is None else r * np.asarray(gain, dtype=np.float64)


def gelu_tanh(a: np.ndarray) -> np.ndarray:
    """gelu_pytorch_tanh ([P5] Mixture of Experts row): 0.5 a (1 + tanh(sqrt(2/pi)(a + 0.044715 a^3)))."""
    a = np.asarray(a, dtype=np.float64)
    return 0.5 * a * (1.0 + np.tanh(SQRT_2_OVER_PI * (a + GELU_CUBIC * a * a * a)))


def softmax(l: np.ndarray) -> np.ndarray:
    """Softmax over the last axis (max subtracted first)."""
    m = np.max(l, axis=-1, keepdims=True)
    e = np.exp(l - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def router(x, router_scale, w_router, logit_bias, per_expert_scale, top_k: int, eps: float) -> dict:
    """The router, in the order of [P5] Router row.

    scale-free RMSNorm -> x learned scale x hidden_size^-0.5 -> linear to E logits
    -> softmax -> top-k -> renormalise over the selected -> x per_expert_scale.

    Returns logits [T,E], probs [T,E], topk_idx [T,k] (int32), topk_w [T,k] (final
    routing weights) and topk_w_renorm [T,k] (before per_expert_scale).
    """
    x = np.asarray(x, dtype=np.float64)
    H = x.shape[-1]
    xhat = rms_norm(x, None, eps)                                   # R3
    z = xhat * np.asarray(router_scale, dtype=np.float64) * (H ** -0.5)   # R4
    logits = z @ np.asarray(w_router, dtype=np.float64).T           # linear to E logits
    if logit_bias is not None:                                       # R5
        logits = logits + np.asarray(logit_bias, dtype=np.float64)
    probs = softmax(logits)
    T, E = logits.shape
    idx = np.empty((T, top_k), dtype=np.int32)
    for t in range(T):
        # R6: order by (logit desc, index asc); a stable sort of -logit keeps equal
        # logits in index order.
        order = np.argsort(-logits[t], kind="stable")
        idx[t] = order[:top_k]
    psel = np.take_along_axis(probs, idx.astype(np.int64), axis=1)
    w_renorm = psel / np.sum(psel, axis=1, keepdims=True)            # renormalise
    pes = np.asarray(per_expert_scale, dtype=np.float64)
    w = w_renorm * pes[idx]                                          # R7
    return {"logits": logits, "probs": probs, "topk_idx": idx,
            "topk_w": w, "topk_w_renorm": w_renorm, "xhat": xhat}


def permute(topk_idx: np.ndarray, num_experts: int):
    """Token-to-expert permutation: a stable sort of the flat (token, slot) pairs by expert.

    The flat pair index is p = t*k + j.  sorted_src lists the pairs grouped by expert,
    each group in increasing p; expert_offsets[e] is where expert e's group starts
    (expert_offsets[E] = T*k); inv_pos[p] is the position of pair p in sorted_src.
    """
    flat = np.asarray(topk_idx, dtype=np.int64).reshape(-1)
    sorted_src = np.argsort(flat, kind="stable").astype(np.int32)
    counts = np.bincount(flat, minlength=num_experts)
    offsets = np.zeros(num_experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    inv_pos = np.empty_like(sorted_src)
    inv_pos[sorted_src] = np.arange(flat.size, dtype=np.int32)
    return offsets, sorted_src, inv_pos


def gated_mlp(u: np.ndarray, w_gate_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """One gated-GELU MLP ([P5] Mixture of Experts row; [P1] fused gate_up naming).

    w_gate_up is [2I][H] with the gate rows first (R8); w_down is [H][I].
      g = u W_gate^T, v = u W_up^T, h = gelu_tanh(g) * v, y = h W_down^T
    """
    I = w_gate_up.shape[0] // 2
    g = u @ w_gate_up[:I].T
    v = u @ w_gate_up[I:].T
    h = gelu_tanh(g) * v
    return h @ w_down.T


class Experts:
    """Access to expert weights as float64, from bf16 bits or int8 codes + fp32 scales.

    bf16: w_gate_up [E][2I][H] uint16, w_down [E][H][I] uint16.
    int8: q_gate_up int8 + s_gate_up [E][2I] fp32; q_down int8 + s_down [E][H] fp32;
          the weight is q * s ([P2]: per-channel symmetric int8).
    """

    def __init__(self, w_gate_up=None, w_down=None, q_gate_up=None, s_gate_up=None,
                 q_down=None, s_down=None, fp8: bool = False, nvfp4=None):
        self.fp8 = fp8                     # q_* are E4M3 codes (uint8) and the activations
        self.int8 = q_gate_up is not None and not fp8   # of both matmuls are quantised
        # NVFP4 (R18): {"gate_up": [(codes, block scales, tensor scale)] per expert,
        # "down": [...]}, weight-only
        self.nvfp4 = nvfp4
        self.w_gate_up, self.w_down = w_gate_up, w_down
        self.q_gate_up, self.s_gate_up = q_gate_up, s_gate_up
        self.q_down, self.s_down = q_down, s_down

    def gate_up(self, e: int) -> np.ndarray:
        if self.nvfp4 is not None:
            return dequantize_nvfp4(*self.nvfp4["gate_up"][e])
        if self.fp8:
            return dequantize_fp8(self.q_gate_up[e], self.s_gate_up[e])
        if self.int8:
            return dequantize(self.q_gate_up[e], self.s_gate_up[e])
        return bf16(self.w_gate_up[e])

    def down(self, e: int) -> np.ndarray:
        if self.nvfp4 is not None:
            return dequantize_nvfp4(*self.nvfp4["down"][e])
        if self.fp8:
            return dequantize_fp8(self.q_down[e], self.s_down[e])
        if self.int8:
            return dequantize(self.q_down[e], self.s_down[e])
        return bf16(self.w_down[e])



def expert_mlp(experts, u: np.ndarray, e: int) -> np.ndarray:
    """Expert e's gated MLP on rows u; fp8 experts run it on quantised activations (R17).
    `experts` is anything with gate_up(e) and down(e) (and optionally fp8)."""
    f = gated_mlp_fp8 if getattr(experts, "fp8", False) else gated_mlp
    return f(u, experts.gate_up(e), experts.down(e))


def moe_sparse(xn_moe: np.ndarray, topk_idx: np.ndarray, topk_w: np.ndarray,
               experts: Experts) -> np.ndarray:
    """Routed experts, sparse form: moe[t] = sum_j w[t,j] * MLP_{idx[t,j]}(xn_moe[t]).

    Each expert runs once on the rows routed to it (one matmul per expert), then the
    weighted outputs are summed per token in slot order j = 0..k-1 ([P1] "How it works").
    """
    xn = np.asarray(xn_moe, dtype=np.float64)
    T, k = topk_idx.shape
    y = np.zeros((T, k, xn.shape[1]), dtype=np.float64)
    for e in np.unique(topk_idx):
        tt, jj = np.nonzero(topk_idx == e)
        y[tt, jj] = expert_mlp(experts, xn[tt], int(e))
    moe = np.zeros((T, xn.shape[1]), dtype=np.float64)
    for j in range(k):
        moe += topk_w[:, j:j + 1] * y[:, j]
    return moe


def moe_all_experts_dense(xn_moe: np.ndarray, route: np.ndarray, experts: Experts) -> np.ndarray:
    """All-experts-dense form ([P1] "How it works"): every token runs every expert and the
    outputs are weighted by a dense [T,E] routing vector that is 0 for unselected experts."""
    xn = np.asarray(xn_moe, dtype=np.float64)
    moe = np.zeros_like(xn)
    for e in range(route.shape[1]):
        moe += route[:, e:e + 1] * expert_mlp(experts, xn, e)
    return moe


def dense_route(topk_idx: np.ndarray, topk_w: np.ndarray, num_experts: int) -> np.ndarray:
    """Scatter the top-k weights into a dense [T,E] routing vector (0 elsewhere)."""
    T, k = topk_idx.shape
    r = np.zeros((T, num_experts), dtype=np.float64)
    for j in range(k):
        r[np.arange(T), topk_idx[:, j]] += topk_w[:, j]
    return r


def block_forward(x_bits, p: dict, experts: Experts, top_k: int, eps: float,
                  logit_bias=None, all_experts_dense: bool = False) -> dict:
    """One hybrid MoE feed-forward block ([P5] MoE topology row; [P1] architecture).

    out = x + post_ff_norm( post_dense_norm(dense(pre_dense_norm(x)))
                            + post_moe_norm(moe(pre_moe_norm(x))) )

    p holds bf16 bit patterns: router_scale, w_router, per_expert_scale, g_pre_moe,
    g_pre_dense, g_post_moe (or None), g_post_dense (or None), g_post_ff,
    w_dense_gate_up [2D][H], w_dense_down [H][D].
    """
    x = bf16(x_bits)
    E = p["w_router"].shape[0]
    r = router(x, bf16(p["router_scale"]), bf16(p["w_router"]), logit_bias,
               bf16(p["per_expert_scale"]), top_k, eps)
    xhat = r["xhat"]                                      # the same rms(x) serves every pre norm
    xn_moe = xhat * bf16(p["g_pre_moe"])
    xn_dense = xhat * bf16(p["g_pre_dense"])
    if all_experts_dense:
        moe = moe_all_experts_dense(xn_moe, dense_route(r["topk_idx"], r["topk_w"], E), experts)
    else:
        moe = moe_sparse(xn_moe, r["topk_idx"], r["topk_w"], experts)
    dense = gated_mlp(xn_dense, bf16(p["w_dense_gate_up"]), bf16(p["w_dense_down"]))
    gpm = p.get("g_post_moe")
    gpd = p.get("g_post_dense")
    a = dense if gpd is None else rms_norm(dense, bf16(gpd), eps)
    b = moe if gpm is None else rms_norm(moe, bf16(gpm), eps)
    out = x + rms_norm(a + b, bf16(p["g_post_ff"]), eps)
    return {"out": out, "moe": moe, "dense": dense, "xn_moe": xn_moe, "xn_dense": xn_dense,
            **{k: v for k, v in r.items() if k != "xhat"}}


# ----------------------------------------------------------------------------- int8

def quantize_int8_per_channel(w_bits: np.ndarray):
    """Per-output-row symmetric int8 quantisation of bf16 weights ([P2]; reading R9).

    Works in fp32, the precision the GPU quantiser uses, so that both sides take the
    same rounding decisions: s = max|w| / 127, q = rint(w / s) clamped to +-127.
    Rows are the last-but-one axis; returns (q int8 same shape, s fp32 shape[:-1]).
    """
    u = np.asarray(w_bits, dtype=np.uint16)
    w = (u.astype(np.uint32) << np.uint32(16)).view(np.float32)
    amax = np.max(np.abs(w), axis=-1)
    s = np.where(amax > 0, amax / np.float32(127.0), np.float32(1.0)).astype(np.float32)
    q = np.rint(w / s[..., None])
    q = np.clip(q, -127, 127).astype(np.int8)
    return q, s


def dequantize(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """q * s per row, in float64."""
    return np.asarray(q, dtype=np.float64) * np.asarray(s, dtype=np.float64)[..., None]


# ----------------------------------------------------------------------------- fp8 (E4M3)

E4M3_MAX = 448.0


def e4m3_decode_table() -> np.ndarray:
    """Value of every E4M3 code 0..255, from the format's definition (R17): sign bit 7,
    exponent bits 6..3 (bias 7), mantissa bits 2..0; exponent 0 is subnormal
    (m/8 * 2^-6); code S.1111.111 is NaN."""
    c = np.arange(256)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    mag = np.where((e == 15) & ((c & 7) == 7), np.nan, mag)
    return sign * mag


def e4m3_round(v) -> np.ndarray:
    """Round to the nearest E4M3 value, ties to even, saturating at +-448 (R17).

    Normal binade [2^e, 2^(e+1)) has spacing 2^(e-3); below 2^-6 the spacing is 2^-9
    (subnormals).  np.rint rounds half to even on the integer multiple of the spacing,
    which is the even-mantissa rule of the format."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))       # a = f * 2^ex, f in [0.5, 1)
    spacing = np.where(a < 2.0 ** -6, 2.0 ** -9, 2.0 ** (ex - 1 - 3.0))
    q = np.rint(a / spacing) * spacing
    return np.copysign(np.minimum(q, E4M3_MAX), v)   # keeps the sign of a rounded zero


def e4m3_encode(v) -> np.ndarray:
    """Code (uint8) of E4M3 grid values (already rounded).  The format has a signed zero:
    a negative value that rounded to zero is -0, code 0x80."""
    tab = e4m3_decode_table()
    pos = tab[:127]                                   # codes 0..126: 0 .. 448, increasing
    v = np.asarray(v, dtype=np.float64)
    idx = np.searchsorted(pos, np.abs(v))
    assert np.all(pos[np.minimum(idx, 126)] == np.abs(v)), "not an E4M3 value"
    return (idx + np.where(np.signbit(v), 128, 0)).astype(np.uint8)


def quantize_fp8_rows(v32: np.ndarray):
    """Per-row E4M3 quantisation (R17) of fp32 values (rows = all axes but the last):
    s = max|v| / 448 in fp32 (1 for an all-zero row), codes of e4m3(fp32(v / s)).
    Returns (codes uint8, s fp32)."""
    v = np.asarray(v32, dtype=np.float32)
    amax = np.max(np.abs(v), axis=-1)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    quot = (v / s[..., None]).astype(np.float32)      # the fp32 quotient the kernels round
    return e4m3_encode(e4m3_round(quot)), s


def quantize_fp8_per_channel(w_bits: np.ndarray):
    """Per-output-row E4M3 quantisation of bf16 weights ([P6]; R17)."""
    u = np.asarray(w_bits, dtype=np.uint16)
    return quantize_fp8_rows((u.astype(np.uint32) << np.uint32(16)).view(np.float32))


def dequantize_fp8(codes: np.ndarray, s: np.ndarray) -> np.ndarray:
    """E4M3 value times the row scale, in float64."""
    return e4m3_decode_table()[np.asarray(codes, dtype=np.uint8)] * \
        np.asarray(s, dtype=np.float64)[..., None]


def bf16_round(v) -> np.ndarray:
    """float64 -> fp32 (nearest) -> bf16 (nearest, ties to even), back as float64: the
    value of an activation stored as bf16."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint32) << np.uint32(16)
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def fp8_activation(v) -> np.ndarray:
    """An expert matmul's activation rows as the fp8 path uses them (R17): stored as
    bf16, quantised per row to E4M3, dequantised (float64)."""
    q, s = quantize_fp8_rows(bf16_round(v).astype(np.float32))
    return dequantize_fp8(q, s)


def gated_mlp_fp8(u: np.ndarray, w_gate_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """gated_mlp with both expert matmuls on fp8 activations (R17): the input rows and h
    are quantised per row; the weights arrive already dequantised."""
    I = w_gate_up.shape[0] // 2
    uq = fp8_activation(u)
    h = gelu_tanh(uq @ w_gate_up[:I].T) * (uq @ w_gate_up[I:].T)
    return fp8_activation(h) @ w_down.T


# ----------------------------------------------------------------------------- NVFP4

E2M1_MAX = 6.0
NVFP4_BLOCK = 16


def e2m1_decode_table() -> np.ndarray:
    """Value of every E2M1 code 0..15 (R18): sign bit 3, exponent bits 2..1 (bias 1),
    mantissa bit 0; exponent 0 is subnormal (m/2)."""
    c = np.arange(16)
    sign = np.where(c & 8, -1.0, 1.0)
    e = (c >> 1) & 3
    m = (c & 1).astype(np.float64)
    mag = np.where(e == 0, m / 2.0, (1.0 + m / 2.0) * 2.0 ** (e - 1.0))
    return sign * mag


def e2m1_round(v) -> np.ndarray:
    """Round to the nearest E2M1 value, ties to the even mantissa, saturating at +-6: the
    binade [2^e, 2^(e+1)) has spacing 2^(e-1), below 1 the spacing is 0.5."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    spacing = np.where(a < 1.0, 0.5, 2.0 ** (ex - 1 - 1.0))
    q = np.rint(a / spacing) * spacing
    return np.copysign(np.minimum(q, E2M1_MAX), v)


def e2m1_encode(v) -> np.ndarray:
    """Code (uint8, low 4 bits) of E2M1 values; -0 is code 8."""
    pos = e2m1_decode_table()[:8]
    v = np.asarray(v, dtype=np.float64)
    idx = np.searchsorted(pos, np.abs(v))
    assert np.all(pos[np.minimum(idx, 7)] == np.abs(v)), "not an E2M1 value"
    return (idx + np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def quantize_nvfp4(w_bits: np.ndarray):
    """R18 quantiser of one bf16 weight matrix [rows][K] (K a multiple of 16), in fp32:
    returns (E2M1 codes uint8 [rows][K], E4M3 block-scale codes uint8 [rows][K/16],
    fp32 tensor scale)."""
    u = np.asarray(w_bits, dtype=np.uint16)
    w = (u.astype(np.uint32) << np.uint32(16)).view(np.float32)
    amax = np.float32(np.max(np.abs(w)))
    t = np.float32(amax / np.float32(E4M3_MAX * E2M1_MAX)) if amax > 0 else np.float32(1.0)
    blocks = w.reshape(*w.shape[:-1], -1, NVFP4_BLOCK)
    bmax = np.max(np.abs(blocks), axis=-1)
    b = e4m3_round((bmax / np.float32(E2M1_MAX) / t).astype(np.float32).astype(np.float64))
    bs = (b.astype(np.float32) * t).astype(np.float32)            # fp32 b * t
    with np.errstate(divide="ignore", invalid="ignore"):
        quot = np.where(bs[..., None] > 0, blocks / bs[..., None], 0.0).astype(np.float32)
    q = e2m1_encode(e2m1_round(quot.astype(np.float64))).reshape(w.shape)
    return q, e4m3_encode(b), t


def dequantize_nvfp4(q: np.ndarray, bcodes: np.ndarray, t) -> np.ndarray:
    """q * b * t in float64 (R18)."""
    vals = e2m1_decode_table()[np.asarray(q, dtype=np.uint8)]
    b = e4m3_decode_table()[np.asarray(bcodes, dtype=np.uint8)]
    blocks = vals.reshape(*vals.shape[:-1], -1, NVFP4_BLOCK) * b[..., None]
    return blocks.reshape(vals.shape) * float(t)


# ----------------------------------------------------------------------------- gaps

def topk_gaps(logits: np.ndarray, top_k: int) -> np.ndarray:
    """Smallest gap between adjacent sorted logits among the top k+1 of each row.

    A row whose gap is at least g has a unique, ordered top-k under any rounding of the
    logits smaller than g/2.
    """
    s = -np.sort(-np.asarray(logits, dtype=np.float64), axis=-1)
    kk = min(top_k + 1, s.shape[-1])
    return np.min(s[:, :kk - 1] - s[:, 1:kk], axis=-1)
