"""Shared test inputs and the parity bar.

Inputs come from `synth` (seeded draws only).  The top-k gap filter uses the oracle's
router, so it lives here with the tests and never in the product path.
"""
from __future__ import annotations

import dataclasses
import json
import os

import numpy as np

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# The accuracy bar: per-row cosine >= 0.9999 and max-abs error <= frac * rms(row of
# the oracle output), frac 2e-2 for bf16 experts and 4e-2 for int8 experts.  The ABI
# returns bf16, so half a bf16 ulp of the oracle value is added to each element's
# allowance: that is the rounding the output format itself imposes.
COS_MIN = 0.9999
FRAC_BF16 = 2e-2
FRAC_INT8 = 4e-2
# fp8 experts: the oracle takes every E4M3 rounding decision from the same bf16 activation
# the kernels quantise (xn_moe, h) in the same fp32 arithmetic, so the two sides differ by
# fp32-vs-fp64 accumulation and the rare code that this moves across a rounding boundary
# (one E4M3 step, 2^-3 relative, on one element of a 704- or 2816-long dot product): the
# int8 bar holds with margin.
FRAC_FP8 = 4e-2
# NVFP4 experts (weight-only, R18): the oracle multiplies the same dequantised weights
# (q * b * t, exact in fp16 before t) as the kernels; the two sides differ by the fp16
# activations and fp32-vs-fp64 accumulation, as for int8, so the bar of 8-bit weights holds.
FRAC_NVFP4 = 4e-2
MIN_GAP = 1e-3


def half_ulp_bf16(v: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 1e-38)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)


def check_bar(got: np.ndarray, ref: np.ndarray, frac: float, what: str = "") -> dict:
    """Assert the bar row by row; return the worst figures."""
    got = np.asarray(got, dtype=np.float64).reshape(ref.shape[0], -1)
    ref = np.asarray(ref, dtype=np.float64).reshape(ref.shape[0], -1)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    cos = synth.cosine_rows(got, ref)
    rms = np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
    err = np.abs(got - ref)
    allow = frac * rms + half_ulp_bf16(ref)
    ratio = err / np.maximum(allow, 1e-300)
    # the same error against the bare bar (frac * rms, without the output format's half
    # ulp), reported so that the margin to it stays visible
    bare = err / np.maximum(frac * rms, 1e-300)
    worst = {"min_cos": float(cos.min()), "max_err_over_allow": float(ratio.max()),
             "max_err_over_bare_bar": float(bare.max()), "max_abs_err": float(err.max())}
    assert cos.min() >= COS_MIN, f"{what}: cosine {cos.min():.7f} < {COS_MIN} ({worst})"
    assert ratio.max() <= 1.0, f"{what}: max-abs error over the bar ({worst})"
    return worst


@dataclasses.dataclass
class Case:
    shape: synth.Shape
    x: np.ndarray              # [T][H] bf16 bits
    p: dict                    # layer weights, bf16 bits
    bias: np.ndarray | None    # [E] fp32 or None
    seed: int


def zipf_alpha() -> float:
    with open(os.path.join(GOLDEN, "zipf_alpha.json")) as f:
        return float(json.load(f)["alpha"])


def gap_filtered_x(seed: int, shape: synth.Shape, p: dict, bias, min_gap: float = MIN_GAP,
                   max_attempts: int = 20000, layer: int = 0) -> np.ndarray:
    """Draw x row by row, redrawing a row until its oracle logits have top-(k+1)
    adjacent gaps >= min_gap.  Returns bf16 bits [T][H]."""
    T, H = shape.T, shape.H
    rs = oracle.bf16(p["router_scale"])
    wr = oracle.bf16(p["w_router"])
    pes = oracle.bf16(p["per_expert_scale"])
    attempts = np.zeros(T, dtype=np.int64)
    x = synth.x_rows(seed, H, T, attempts, layer)
    pending = np.arange(T)
    while pending.size:
        r = oracle.router(oracle.bf16(x[pending]), rs, wr, bias, pes, shape.k, shape.eps)
        ok = oracle.topk_gaps(r["logits"], shape.k) >= min_gap
        pending = pending[~ok]
        if pending.size == 0:
            break
        attempts[pending] += 1
        if attempts.max() > max_attempts:
            raise RuntimeError("gap filter: too many redraws")
        for t in pending:
            x[t] = synth.x_row(seed, H, int(t), int(attempts[t]), layer)
    return x


class _Lru(dict):
    def __init__(self, n):
        super().__init__()
        self.n = n

    def put(self, key, value):
        if key in self:
            del self[key]
        while len(self) >= self.n:
            del self[next(iter(self))]
        self[key] = value
        return value


_LAYER_CACHE = _Lru(3)
_CASE_CACHE = _Lru(16)


def make_case(shape: synth.Shape, seed: int = 1234, zipf: bool = False, layer: int = 0,
              gap: bool = True, router_std=None) -> Case:
    ckey = (shape, seed, zipf, layer, gap, router_std)
    if ckey in _CASE_CACHE:
        return _CASE_CACHE[ckey]
    key = (shape.H, shape.E, shape.I, shape.D, seed, layer, router_std)
    p = _LAYER_CACHE[key] if key in _LAYER_CACHE else _LAYER_CACHE.put(
        key, synth.make_layer(seed, shape, layer, router_std=router_std))
    bias = synth.zipf_bias(seed, shape.E, zipf_alpha()) if zipf else None
    if gap:
        x = gap_filtered_x(seed + 1, shape, p, bias, layer=layer)
    else:
        x = synth.x_rows(seed + 1, shape.H, shape.T, layer=layer)
    return _CASE_CACHE.put(ckey, Case(shape, x, p, bias, seed))


def bf16_experts(p: dict) -> oracle.Experts:
    return oracle.Experts(w_gate_up=p["w_gate_up"], w_down=p["w_down"])
