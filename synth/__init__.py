"""Seeded synthetic inputs for the hybrid MoE feed-forward block.

This module only draws random numbers and stores them in the formats the block's
interface uses (bf16 bit patterns, fp32). It holds none of the block's arithmetic,
so both the CUDA path's tests and the oracle can take their inputs from here.

Every tensor gets its own Philox stream, keyed by (seed, tensor id, layer, ...).
Large tensors are drawn in fixed-size chunks, each with its own key, so a tensor's
values do not depend on how many threads draw it.

Distributions follow the workloads that the model pages describe (Gemma-4-26B-A4B
card, "The architecture"; ONNX export card, "Truthful graph contracts"):
  - weights N(0, 0.02), rounded to bf16 (round to nearest even);
  - activations N(0, 1) in bf16;
  - norm gains, the router scale and per_expert_scale U(0.5, 1.5) in bf16;
  - an optional Zipf-ranked per-expert router-logit offset (fp32).
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os

import numpy as np

# Tensor ids.  Each id has its own key space, so no two tensors share draws.
X = 1
W_ROUTER = 2
ROUTER_SCALE = 3
PER_EXPERT_SCALE = 4
G_PRE_MOE = 5
G_PRE_DENSE = 6
G_POST_MOE = 7
G_POST_DENSE = 8
G_POST_FF = 9
W_GATE_UP = 10
W_DOWN = 11
W_DENSE_GATE_UP = 12
W_DENSE_DOWN = 13
BIAS_RANKS = 14

_CHUNK = 1 << 22  # elements per independently keyed chunk


@dataclasses.dataclass(frozen=True)
class Shape:
    """Sizes of one MoE feed-forward layer and of one batch of tokens."""
    T: int      # tokens
    H: int      # hidden size
    E: int      # routed experts
    k: int      # experts per token
    I: int      # expert intermediate size
    D: int      # shared dense MLP intermediate size
    eps: float = 1e-6


# The workloads.  Sizes of the full layer come from the Gemma-4-26B-A4B card
# ("The architecture": 128 experts, top 8, moe_intermediate_size 704,
# intermediate_size 2112, hidden_size 2816).
TINY = Shape(T=8, H=512, E=16, k=4, I=128, D=384)
DECODE = Shape(T=8, H=2816, E=128, k=8, I=704, D=2112)
PREFILL = Shape(T=2048, H=2816, E=128, k=8, I=704, D=2112)
STACK_T = 16384
STACK_LAYERS = 30


def _key(seed: int, *ids: int) -> np.random.Generator:
    ss = np.random.SeedSequence([int(seed) & 0xFFFFFFFF, *[int(i) for i in ids]])
    return np.random.Generator(np.random.Philox(ss))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return the uint16 bit patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _fill_chunked(shape, draw, seed, ids, threads=None) -> np.ndarray:
    """Draw a tensor chunk by chunk; chunk c uses key (seed, *ids, c)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    nchunks = max(1, (n + _CHUNK - 1) // _CHUNK)

    def work(c):
        lo = c * _CHUNK
        hi = min(n, lo + _CHUNK)
        out[lo:hi] = f32_to_bf16_bits(draw(_key(seed, *ids, c), hi - lo))

    if nchunks == 1:
        work(0)
    else:
        threads = threads or min(32, os.cpu_count() or 1)
        with _cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(work, range(nchunks)))
    return out.reshape(shape)


def normal_bf16(seed: int, ids: tuple, shape, std: float) -> np.ndarray:
    """N(0, std^2) draws rounded to bf16 (uint16 bit patterns)."""
    return _fill_chunked(
        shape, lambda g, m: g.standard_normal(m, dtype=np.float32) * np.float32(std), seed, ids)


def uniform_bf16(seed: int, ids: tuple, shape, lo: float, hi: float) -> np.ndarray:
    """U(lo, hi) draws rounded to bf16 (uint16 bit patterns)."""
    return _fill_chunked(
        shape, lambda g, m: (g.random(m, dtype=np.float32) * np.float32(hi - lo) + np.float32(lo)),
        seed, ids)


def x_row(seed: int, H: int, t: int, attempt: int = 0, layer: int = 0) -> np.ndarray:
    """One activation row N(0, 1) in bf16; (t, attempt) pick an independent stream."""
    return f32_to_bf16_bits(_key(seed, X, layer, t, attempt).standard_normal(H, dtype=np.float32))


def x_rows(seed: int, H: int, T: int, attempts=None, layer: int = 0) -> np.ndarray:
    """T activation rows; row t uses draw number attempts[t] (default 0)."""
    out = np.empty((T, H), dtype=np.uint16)
    for t in range(T):
        out[t] = x_row(seed, H, t, 0 if attempts is None else int(attempts[t]), layer)
    return out


def zipf_bias(seed: int, E: int, alpha: float, s: float = 1.1) -> np.ndarray:
    """Per-expert logit offset b_e = -alpha * s * ln(rank_e), ranks a seeded permutation of 1..E."""
    ranks = _key(seed, BIAS_RANKS).permutation(E) + 1
    return (-alpha * s * np.log(ranks.astype(np.float64))).astype(np.float32)


def make_router(seed: int, shape: Shape, layer: int = 0, std: float = 0.02,
                gains=(0.5, 1.5), router_std=None) -> dict:
    """The router's tensors of one layer (the same draws make_layer returns).
    router_std (default: std) sets the spread of the router weights alone."""
    lo, hi = gains
    return {
        "w_router": normal_bf16(seed, (W_ROUTER, layer), (shape.E, shape.H),
                                std if router_std is None else router_std),
        "router_scale": uniform_bf16(seed, (ROUTER_SCALE, layer), (shape.H,), lo, hi),
        "per_expert_scale": uniform_bf16(seed, (PER_EXPERT_SCALE, layer), (shape.E,), lo, hi),
    }


def make_layer(seed: int, shape: Shape, layer: int = 0, std: float = 0.02,
               gains=(0.5, 1.5), router_std=None) -> dict:
    """All weights of one layer as bf16 bit patterns (numpy uint16).

    Layout (row-major, K contiguous):
      w_router      [E][H]
      w_gate_up     [E][2I][H]   rows 0..I-1 gate, I..2I-1 up
      w_down        [E][H][I]
      w_dense_gate_up [2D][H]    rows 0..D-1 gate, D..2D-1 up
      w_dense_down  [H][D]
      router_scale, g_pre_moe, g_pre_dense, g_post_moe, g_post_dense, g_post_ff [H]
      per_expert_scale [E]
    """
    H, E, I, D = shape.H, shape.E, shape.I, shape.D
    lo, hi = gains
    L = layer
    return {
        **make_router(seed, shape, layer, std, gains, router_std),
        "w_gate_up": normal_bf16(seed, (W_GATE_UP, L), (E, 2 * I, H), std),
        "w_down": normal_bf16(seed, (W_DOWN, L), (E, H, I), std),
        "w_dense_gate_up": normal_bf16(seed, (W_DENSE_GATE_UP, L), (2 * D, H), std),
        "w_dense_down": normal_bf16(seed, (W_DENSE_DOWN, L), (H, D), std),
        "g_pre_moe": uniform_bf16(seed, (G_PRE_MOE, L), (H,), lo, hi),
        "g_pre_dense": uniform_bf16(seed, (G_PRE_DENSE, L), (H,), lo, hi),
        "g_post_moe": uniform_bf16(seed, (G_POST_MOE, L), (H,), lo, hi),
        "g_post_dense": uniform_bf16(seed, (G_POST_DENSE, L), (H,), lo, hi),
        "g_post_ff": uniform_bf16(seed, (G_POST_FF, L), (H,), lo, hi),
    }


def torch_layer(shape: Shape, seed: int, layer: int, device, std: float = 0.02,
                gains=(0.5, 1.5)) -> dict:
    """Same distributions as make_layer, drawn on a torch device (for large timing runs).

    The values differ from make_layer's (another generator); the distributions and
    layout are the same.
    """
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1000003 + 7919 * int(layer) + 17) & 0x7FFFFFFFFFFFFFFF)
    H, E, I, D = shape.H, shape.E, shape.I, shape.D
    lo, hi = gains

    def nrm(*s):
        return (torch.randn(*s, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)

    def uni(*s):
        return (torch.rand(*s, generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo).to(torch.bfloat16)

    return {
        "w_router": nrm(E, H),
        "w_gate_up": nrm(E, 2 * I, H),
        "w_down": nrm(E, H, I),
        "w_dense_gate_up": nrm(2 * D, H),
        "w_dense_down": nrm(H, D),
        "router_scale": uni(H),
        "per_expert_scale": uni(E),
        "g_pre_moe": uni(H),
        "g_pre_dense": uni(H),
        "g_post_moe": uni(H),
        "g_post_dense": uni(H),
        "g_post_ff": uni(H),
    }


def torch_x(shape: Shape, seed: int, step: int, device):
    """Activations N(0, 1) in bf16 on a torch device."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 7777777 + 31 * int(step) + 5) & 0x7FFFFFFFFFFFFFFF)
    return torch.randn(shape.T, shape.H, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def cosine_rows(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Per-row cosine similarity (a comparison helper; not part of the block)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    num = (a * b).sum(-1)
    den = np.sqrt((a * a).sum(-1) * (b * b).sum(-1))
    return np.where(den > 0, num / np.where(den > 0, den, 1.0), 1.0)

