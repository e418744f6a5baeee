"""Pins for the oracle: each check ties it to something other than itself.

Library routines (torch's rms_norm, gelu, softmax, topk, linear), closed forms,
brute force on tiny inputs and the identities the model pages state.  Every test here
runs on the CPU.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth
from tests import cases

RNG = np.random.default_rng(7)


def _rand(*s, scale=1.0):
    return RNG.standard_normal(s) * scale


# ------------------------------------------------------------------ pieces vs library

def test_rms_norm_matches_torch():
    v = _rand(5, 48, scale=3.0)
    g = RNG.uniform(0.5, 1.5, 48)
    eps = 1e-6
    ref = F.rms_norm(torch.from_numpy(v), (48,), torch.from_numpy(g), eps).numpy()
    np.testing.assert_allclose(oracle.rms_norm(v, g, eps), ref, rtol=1e-13, atol=0)
    ref0 = F.rms_norm(torch.from_numpy(v), (48,), None, eps).numpy()
    np.testing.assert_allclose(oracle.rms_norm(v, None, eps), ref0, rtol=1e-13, atol=0)


def test_rms_norm_closed_form():
    # A constant row c has mean square c^2, so the norm is c / sqrt(c^2 + eps).
    c, eps = -2.5, 1e-6
    got = oracle.rms_norm(np.full((1, 7), c), None, eps)
    np.testing.assert_allclose(got, np.full((1, 7), c / math.sqrt(c * c + eps)), rtol=1e-15)


def test_gelu_tanh_matches_torch_and_limits():
    a = np.linspace(-9, 9, 1001)
    ref = F.gelu(torch.from_numpy(a), approximate="tanh").numpy()
    np.testing.assert_allclose(oracle.gelu_tanh(a), ref, rtol=1e-13, atol=1e-15)
    assert oracle.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert abs(oracle.gelu_tanh(np.array([30.0]))[0] - 30.0) < 1e-12
    assert abs(oracle.gelu_tanh(np.array([-30.0]))[0]) < 1e-12


def test_softmax_matches_torch():
    l = _rand(4, 128, scale=0.05)
    ref = torch.softmax(torch.from_numpy(l), dim=-1).numpy()
    np.testing.assert_allclose(oracle.softmax(l), ref, rtol=1e-14)


# ------------------------------------------------------------------ router

def _tiny_router_inputs(T=6, H=16, E=7):
    x = _rand(T, H)
    rs = RNG.uniform(0.5, 1.5, H)
    wr = _rand(E, H, scale=0.3)
    pes = RNG.uniform(0.5, 1.5, E)
    return x, rs, wr, pes


def test_router_topk_brute_force():
    """P4: the top-k set is the k-subset with the largest logit sum (ties: smallest indices)."""
    for k in (1, 2, 3, 7):
        x, rs, wr, pes = _tiny_router_inputs()
        r = oracle.router(x, rs, wr, None, pes, k, 1e-6)
        for t in range(x.shape[0]):
            l = r["logits"][t]
            best = max(itertools.combinations(range(len(l)), k),
                       key=lambda S: (sum(l[i] for i in S), [-i for i in S]))
            assert sorted(best) == sorted(r["topk_idx"][t].tolist())
            # ordered by logit descending
            sel = l[r["topk_idx"][t]]
            assert np.all(np.diff(sel) <= 0)


def test_router_ties_go_to_lower_index():
    # Equal rows of W_r give equal logits: the lower expert index must come first.
    x, rs, wr, pes = _tiny_router_inputs(T=3, E=6)
    wr[4] = wr[1]
    wr[5] = wr[1]
    r = oracle.router(x, rs, wr, np.array([0, 9.0, 0, 0, 9.0, 9.0]), pes, 3, 1e-6)
    assert r["topk_idx"].tolist() == [[1, 4, 5]] * 3


def test_router_matches_torch_topk():
    x, rs, wr, pes = _tiny_router_inputs(T=20, H=32, E=16)
    r = oracle.router(x, rs, wr, None, pes, 4, 1e-6)
    v, i = torch.topk(torch.from_numpy(r["logits"]), 4, dim=-1, sorted=True)
    assert np.array_equal(i.numpy(), r["topk_idx"])


def test_router_closed_form_logits():
    """A constant x, a constant learned scale s and constant W_r rows a_e give
    logit_e = a_e * s * sqrt(H) * sign(c) / sqrt(1 + eps / c^2)."""
    H, E, c, s, eps = 64, 5, -1.7, 1.25, 1e-6
    a = np.array([0.3, -0.2, 0.1, 0.5, -0.05])
    x = np.full((1, H), c)
    r = oracle.router(x, np.full(H, s), np.repeat(a[:, None], H, axis=1), None, np.ones(E), 2, eps)
    want = a * s * math.sqrt(H) * math.copysign(1.0, c) / math.sqrt(1 + eps / (c * c))
    np.testing.assert_allclose(r["logits"][0], want, rtol=1e-13)
    # the bias is added to the logits
    b = np.arange(E, dtype=np.float64)
    rb = oracle.router(x, np.full(H, s), np.repeat(a[:, None], H, axis=1), b, np.ones(E), 2, eps)
    np.testing.assert_allclose(rb["logits"][0], want + b, rtol=1e-13)


def test_routing_weights_renormalised():
    """P2: the weights sum to 1 before per_expert_scale, are positive, and
    per_expert_scale multiplies each selected expert's weight."""
    x, rs, wr, pes = _tiny_router_inputs(T=30, H=24, E=9)
    r = oracle.router(x, rs, wr, None, pes, 3, 1e-6)
    np.testing.assert_allclose(r["topk_w_renorm"].sum(1), 1.0, atol=1e-15)
    assert np.all(r["topk_w_renorm"] > 0)
    np.testing.assert_allclose(r["topk_w"], r["topk_w_renorm"] * pes[r["topk_idx"]], rtol=1e-15)
    # renormalised softmax = exp(l_j) / sum over the selected of exp(l_i)
    l = np.take_along_axis(r["logits"], r["topk_idx"].astype(np.int64), 1)
    e = np.exp(l - l.max(1, keepdims=True))
    np.testing.assert_allclose(r["topk_w_renorm"], e / e.sum(1, keepdims=True), rtol=1e-13)


# ------------------------------------------------------------------ permutation

def _permute_brute(idx, E):
    pairs = [(int(e), p) for p, e in enumerate(np.asarray(idx).reshape(-1))]
    src = [p for e in range(E) for (ee, p) in pairs if ee == e]
    counts = [sum(1 for (ee, _) in pairs if ee == e) for e in range(E)]
    offs = [0]
    for c in counts:
        offs.append(offs[-1] + c)
    inv = [0] * len(src)
    for q, p in enumerate(src):
        inv[p] = q
    return offs, src, inv


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (5, 2, 4), (33, 4, 16), (64, 8, 128), (0, 8, 128)])
def test_permute_brute_force(T, k, E):
    """P6: counting sort by expert, stable by flat index t*k+j."""
    idx = RNG.integers(0, E, size=(T, k)).astype(np.int32)
    offs, src, inv = oracle.permute(idx, E)
    bo, bs, bi = _permute_brute(idx, E)
    assert offs.tolist() == bo and src.tolist() == bs and inv.tolist() == bi


# ------------------------------------------------------------------ expert MLP

def test_gated_mlp_matches_torch_linear():
    H, I = 24, 10
    u = _rand(3, H)
    wgu = _rand(2 * I, H, scale=0.2)
    wd = _rand(H, I, scale=0.2)
    tu = torch.from_numpy(u)
    g = F.linear(tu, torch.from_numpy(wgu[:I]))
    v = F.linear(tu, torch.from_numpy(wgu[I:]))
    ref = F.linear(F.gelu(g, approximate="tanh") * v, torch.from_numpy(wd)).numpy()
    np.testing.assert_allclose(oracle.gated_mlp(u, wgu, wd), ref, rtol=1e-12, atol=1e-14)


def test_gated_mlp_permutation_closed_form():
    """With permutation matrices P (gate), Q (up), R (down):
    y = R (gelu(P u) * (Q u)); a transposed operand would use P^T, Q^T or R^T."""
    n = 6
    P = np.eye(n)[[1, 2, 3, 4, 5, 0]]
    Q = np.eye(n)[[3, 0, 4, 1, 5, 2]]
    R = np.eye(n)[[2, 5, 1, 0, 3, 4]]
    u = np.arange(1.0, n + 1.0) * np.array([1, -1, 1, -1, 1, -1]) * 0.7
    want = np.empty(n)
    for i in range(n):
        gi = u[[1, 2, 3, 4, 5, 0][i]]
        vi = u[[3, 0, 4, 1, 5, 2][i]]
        want[i] = 0.5 * gi * (1 + math.tanh(math.sqrt(2 / math.pi) * (gi + 0.044715 * gi ** 3))) * vi
    want = want[[2, 5, 1, 0, 3, 4]]
    got = oracle.gated_mlp(u[None], np.vstack([P, Q]), R)[0]
    np.testing.assert_allclose(got, want, rtol=1e-14)


# ------------------------------------------------------------------ block identities

def _tiny_block(T=6, H=16, E=6, k=2, I=4, D=8, seed=3, bias=None):
    shape = synth.Shape(T=T, H=H, E=E, k=k, I=I, D=D)
    p = synth.make_layer(seed, shape, std=0.3)
    x = synth.x_rows(seed + 1, H, T)
    return shape, p, x


def test_all_experts_dense_equals_sparse():
    """P1: the all-experts-dense form (weight 0 for unselected experts) equals sparse top-k."""
    shape, p, x = _tiny_block(T=9, H=32, E=8, k=3, I=8, D=8)
    ex = cases.bf16_experts(p)
    a = oracle.block_forward(x, p, ex, shape.k, shape.eps)
    b = oracle.block_forward(x, p, ex, shape.k, shape.eps, all_experts_dense=True)
    np.testing.assert_allclose(a["moe"], b["moe"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(a["out"], b["out"], rtol=1e-12, atol=1e-15)


def test_k_equals_E_is_dense_softmax_mixture():
    """P3: with k = E the renormalisation is the full softmax, so
    moe = sum_e p_e * pes_e * MLP_e(xn)."""
    shape, p, x = _tiny_block(T=5, H=16, E=5, k=5, I=4, D=4)
    ex = cases.bf16_experts(p)
    o = oracle.block_forward(x, p, ex, shape.k, shape.eps)
    pes = oracle.bf16(p["per_expert_scale"])
    want = np.zeros_like(o["moe"])
    for e in range(shape.E):
        want += (o["probs"][:, e] * pes[e])[:, None] * oracle.gated_mlp(o["xn_moe"], ex.gate_up(e), ex.down(e))
    np.testing.assert_allclose(o["moe"], want, rtol=1e-12, atol=1e-15)


def test_single_expert_is_plain_gated_mlp():
    """P5: E = k = 1 gives moe = per_expert_scale * MLP(xn_moe); a zero down projection
    gives moe = 0 and out = x + post_ff(post_dense(dense))."""
    shape, p, x = _tiny_block(T=4, H=16, E=1, k=1, I=4, D=4)
    ex = cases.bf16_experts(p)
    o = oracle.block_forward(x, p, ex, 1, shape.eps)
    pes = oracle.bf16(p["per_expert_scale"])[0]
    np.testing.assert_allclose(o["topk_w"], pes, rtol=1e-15)
    np.testing.assert_allclose(o["moe"], pes * oracle.gated_mlp(o["xn_moe"], ex.gate_up(0), ex.down(0)),
                               rtol=1e-13)
    p0 = dict(p, w_down=np.zeros_like(p["w_down"]))
    o0 = oracle.block_forward(x, p0, cases.bf16_experts(p0), 1, shape.eps)
    assert np.all(o0["moe"] == 0)
    eps = shape.eps
    want = oracle.bf16(x) + oracle.rms_norm(oracle.rms_norm(o0["dense"], oracle.bf16(p["g_post_dense"]), eps),
                                            oracle.bf16(p["g_post_ff"]), eps)
    np.testing.assert_allclose(o0["out"], want, rtol=1e-13)


def test_rows_are_independent():
    """P7: permuting the tokens permutes the outputs (no capacity limit, no cross-token term)."""
    shape, p, x = _tiny_block(T=7, H=16, E=6, k=2, I=4, D=4)
    ex = cases.bf16_experts(p)
    perm = np.array([3, 0, 6, 1, 5, 2, 4])
    a = oracle.block_forward(x, p, ex, shape.k, shape.eps)
    b = oracle.block_forward(x[perm], p, ex, shape.k, shape.eps)
    np.testing.assert_allclose(b["out"], a["out"][perm], rtol=1e-14)
    assert np.array_equal(b["topk_idx"], a["topk_idx"][perm])


def _block_brute(x, p, k, eps):
    """The block with plain Python loops and math.* only, from the definitions."""
    X = oracle.bf16(x)
    T, H = X.shape
    E = p["w_router"].shape[0]
    f = {n: oracle.bf16(p[n]) for n in p if p[n] is not None}
    I = f["w_gate_up"].shape[1] // 2
    D = f["w_dense_gate_up"].shape[0] // 2

    def gelu(a):
        return 0.5 * a * (1 + math.tanh(math.sqrt(2 / math.pi) * (a + 0.044715 * a ** 3)))

    def norm(v, g):
        r = math.sqrt(sum(t * t for t in v) / len(v) + eps)
        return [v[i] / r * (1.0 if g is None else g[i]) for i in range(len(v))]

    def mlp(u, wgu, wd, n):
        h = []
        for i in range(n):
            g = sum(u[c] * wgu[i][c] for c in range(H))
            v = sum(u[c] * wgu[n + i][c] for c in range(H))
            h.append(gelu(g) * v)
        return [sum(h[i] * wd[o][i] for i in range(n)) for o in range(H)]

    outs = []
    for t in range(T):
        xh = norm(list(X[t]), None)
        z = [xh[c] * f["router_scale"][c] / math.sqrt(H) for c in range(H)]
        l = [sum(z[c] * f["w_router"][e][c] for c in range(H)) for e in range(E)]
        S = max(itertools.combinations(range(E), k), key=lambda S: (sum(l[i] for i in S), [-i for i in S]))
        m = max(l)
        ex = [math.exp(v - m) for v in l]
        tot = sum(ex)
        pr = [v / tot for v in ex]
        ssum = sum(pr[i] for i in S)
        moe = [0.0] * H
        um = [xh[c] * f["g_pre_moe"][c] for c in range(H)]
        for e in S:
            y = mlp(um, f["w_gate_up"][e], f["w_down"][e], I)
            w = pr[e] / ssum * f["per_expert_scale"][e]
            moe = [moe[c] + w * y[c] for c in range(H)]
        ud = [xh[c] * f["g_pre_dense"][c] for c in range(H)]
        dense = mlp(ud, f["w_dense_gate_up"], f["w_dense_down"], D)
        a = norm(dense, f["g_post_dense"])
        b = norm(moe, f["g_post_moe"])
        c = norm([a[i] + b[i] for i in range(H)], f["g_post_ff"])
        outs.append([X[t][i] + c[i] for i in range(H)])
    return np.array(outs)


def test_block_brute_force_tiny():
    """P4: the whole block against plain loops (subset search for the top-k)."""
    shape, p, x = _tiny_block(T=3, H=8, E=5, k=2, I=3, D=4)
    got = oracle.block_forward(x, p, cases.bf16_experts(p), shape.k, shape.eps)["out"]
    np.testing.assert_allclose(got, _block_brute(x, p, shape.k, shape.eps), rtol=1e-11, atol=1e-13)


# ------------------------------------------------------------------ int8

def test_int8_quantiser_pins():
    """P8 and R9: |q s - w| <= s/2, the largest |q| of a non-zero row is 127, an
    all-zero row takes s = 1 and q = 0, and halves round to even."""
    w = synth.normal_bf16(5, (99,), (6, 40), 0.02)
    w[3] = 0
    q, s = oracle.quantize_int8_per_channel(w)
    wf = synth.bf16_bits_to_f32(w).astype(np.float64)
    assert q.dtype == np.int8 and s.dtype == np.float32
    assert np.all(np.abs(q.astype(np.float64) * s[:, None] - wf) <= s[:, None] / 2 * (1 + 1e-6))
    nz = [i for i in range(6) if i != 3]
    assert np.all(np.abs(q[nz]).max(1) == 127)
    assert s[3] == 1.0 and np.all(q[3] == 0)
    # amax = 127/128 makes s = 2^-7 exactly; 2.5 s, 3.5 s, -2.5 s, -0.5 s -> 2, 4, -2, 0
    row = np.array([127 / 128, 2.5 / 128, 3.5 / 128, -2.5 / 128, -0.5 / 128], dtype=np.float32)
    qq, ss = oracle.quantize_int8_per_channel(synth.f32_to_bf16_bits(row)[None])
    assert ss[0] == np.float32(2.0 ** -7)
    assert qq[0].tolist() == [127, 2, 4, -2, 0]


# ------------------------------------------------------------------ fp8 (E4M3)

def test_e4m3_decode_table_matches_torch():
    """R17: the format written out (sign, 4 exponent bits of bias 7, 3 mantissa bits,
    subnormals, NaN at S.1111.111) equals the library's float8_e4m3fn decoding."""
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    tab = oracle.e4m3_decode_table()
    assert np.array_equal(np.isnan(tab), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(tab[ok], ref[ok])
    assert tab[0x7E] == 448.0 and tab[0x01] == 2.0 ** -9 and tab[0x08] == 2.0 ** -6
    # every code but the two NaNs decodes and encodes back to itself (0x80 is -0)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(oracle.e4m3_encode(tab[codes]), codes)


def test_e4m3_rounding_matches_torch_and_closed_forms():
    """Round-to-nearest-even onto the E4M3 grid equals the library's fp32 -> float8_e4m3fn
    conversion inside the finite range; ties, the subnormal floor and the saturation at
    448 (the kernels' satfinite rounding, which the library conversion does not do) by
    closed forms."""
    tab = oracle.e4m3_decode_table()
    fin = tab[np.isfinite(tab)]
    assert np.array_equal(oracle.e4m3_round(fin), fin)           # grid values stay put
    pos = np.unique(np.abs(fin))
    mids = (pos[:-1] + pos[1:]) / 2                                # every exact tie
    v = np.concatenate([RNG.uniform(-440, 440, 4000), RNG.uniform(-0.05, 0.05, 4000),
                        mids, -mids, [0.0]]).astype(np.float32)
    ref8 = torch.from_numpy(v).to(torch.float8_e4m3fn)
    ref = ref8.to(torch.float64).numpy()
    got = oracle.e4m3_round(v.astype(np.float64))
    assert np.array_equal(got, ref)
    # codes too, which also fixes the sign of values that round to zero (signed zero)
    assert np.array_equal(oracle.e4m3_encode(got), ref8.view(torch.uint8).numpy())
    tiny = np.array([-1e-9, -2.0 ** -11, 2.0 ** -11, -0.0, 0.0], dtype=np.float32)
    t8 = torch.from_numpy(tiny).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert t8.tolist() == [0x80, 0x80, 0x00, 0x80, 0x00]
    assert oracle.e4m3_encode(oracle.e4m3_round(tiny.astype(np.float64))).tolist() == t8.tolist()
    got = oracle.e4m3_round([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, 449.0, 1e6, -1e6])
    assert got.tolist() == [1.0, 1.25, 0.0, 2.0 ** -8, 448.0, 448.0, -448.0]
    assert oracle.e4m3_encode(got[:4]).tolist() == [0x38, 0x3A, 0x00, 0x02]


def test_fp8_quantiser_pins():
    """R17: s = max|w| / 448; each value lands within half an E4M3 step (relative 2^-4,
    or 2^-10 s absolute below the normal range) of w; the largest |w| of a row becomes
    +-448 exactly; an all-zero row takes s = 1 and code 0."""
    w = synth.normal_bf16(5, (98,), (6, 40), 0.02)
    w[3] = 0
    q, s = oracle.quantize_fp8_per_channel(w)
    wf = synth.bf16_bits_to_f32(w).astype(np.float64)
    assert q.dtype == np.uint8 and s.dtype == np.float32
    deq = oracle.dequantize_fp8(q, s)
    err = np.abs(deq - wf)
    bound = np.maximum(np.abs(wf) * 2.0 ** -4, s[:, None] * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound)
    tab = oracle.e4m3_decode_table()
    nz = [i for i in range(6) if i != 3]
    assert np.all(np.abs(tab[q[nz]]).max(1) == 448.0)
    assert s[3] == 1.0 and np.all(q[3] == 0)


def test_fp8_activation_scale_is_per_token():
    """R17 and [P6] (dynamic per-token activation scales): the all-experts-dense form runs
    every token through every expert, the sparse form only the routed rows; the two agree
    only if a token's quantisation does not depend on which other rows share the matmul."""
    E, k, H, I, T = 6, 2, 32, 16, 9
    wgu = synth.normal_bf16(21, (1,), (E, 2 * I, H), 0.2)
    wd = synth.normal_bf16(21, (2,), (E, H, I), 0.2)
    qg, sg = oracle.quantize_fp8_per_channel(wgu)
    qd, sd = oracle.quantize_fp8_per_channel(wd)
    ex = oracle.Experts(q_gate_up=qg, s_gate_up=sg, q_down=qd, s_down=sd, fp8=True)
    xn = RNG.standard_normal((T, H))
    idx = np.stack([RNG.permutation(E)[:k] for _ in range(T)])
    tw = RNG.uniform(0.1, 1.0, (T, k))
    sparse = oracle.moe_sparse(xn, idx, tw, ex)
    dense = oracle.moe_all_experts_dense(xn, oracle.dense_route(idx, tw, E), ex)
    np.testing.assert_allclose(sparse, dense, rtol=1e-12, atol=1e-12)
    # and the quantisation is really there: the bf16-weight reading differs by ~ 2^-4
    bfx = oracle.Experts(w_gate_up=wgu, w_down=wd)
    rel = np.abs(sparse - oracle.moe_sparse(xn, idx, tw, bfx)).max() / np.abs(sparse).max()
    assert 1e-3 < rel < 0.2


def _bf16_truncating(v):
    """A deliberately wrong bf16 rounding (drops the low 16 bits), to show the pin below
    tells it apart."""
    u = np.asarray(v, dtype=np.float64).astype(np.float32).view(np.uint32)
    return (u & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)


def _bf16_ties_away(v):
    """A deliberately wrong bf16 rounding (nearest, ties away from zero)."""
    u = np.asarray(v, dtype=np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x8000) >> 16).astype(np.uint32) << np.uint32(16)
    return r.view(np.float32).astype(np.float64)


def test_bf16_round_matches_torch():
    """The bf16 storage of an activation (R10, R17) equals the library's fp32 -> bfloat16
    conversion (round to nearest, ties to even) on random values of every magnitude,
    exact ties with an even and with an odd kept bit, fp32 subnormals, values next to
    the largest finite bf16 (which round up to infinity past it) and signed zeros.  The
    inputs tell a truncating and a ties-away rounding apart from the right one."""
    mant = RNG.integers(0, 1 << 23, 3000, dtype=np.uint32)
    expo = RNG.integers(1, 254, 3000, dtype=np.uint32)
    sign = RNG.integers(0, 2, 3000, dtype=np.uint32) << np.uint32(31)
    rnd = (sign | (expo << np.uint32(23)) | mant).view(np.float32)
    hi = RNG.integers(0, 1 << 16, 200, dtype=np.uint32) << np.uint32(16)
    ties = (hi | np.uint32(0x8000)) & np.uint32(0x7F7FFFFF)      # low half exactly 0x8000
    ties = ties[(ties >> np.uint32(23)) > 0].view(np.float32)
    sub = (RNG.integers(1, 1 << 23, 200, dtype=np.uint32)).view(np.float32)   # subnormals
    big = np.array([0x7F7F0000, 0x7F7F7FFF, 0x7F7F8000, 0x7F7FFFFF, 0x7F7E8000,
                    0xFF7F8000], dtype=np.uint32).view(np.float32)
    special = np.array([0.0, -0.0, 1.0, -1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8],
                       dtype=np.float32)
    v = np.concatenate([rnd, ties, -ties, sub, -sub, big, special])
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.bf16_round(v.astype(np.float64))
    assert np.array_equal(got, ref) and np.array_equal(np.signbit(got), np.signbit(ref))
    # closed forms: 1 + 2^-8 is the tie between 1 and 1 + 2^-7 (even: 1); 1 + 3 * 2^-8
    # is the tie between 1 + 2^-7 and 1 + 2^-6 (even: 1 + 2^-6)
    assert oracle.bf16_round([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8]).tolist() == \
        [1.0, 1.0 + 2.0 ** -6]
    assert np.isinf(oracle.bf16_round([3.4e38])[0])
    # the pin discriminates: both wrong roundings differ from the library somewhere
    for wrong in (_bf16_truncating, _bf16_ties_away):
        assert not np.array_equal(wrong(v.astype(np.float64)), ref)


def test_fp8_activation_closed_form_rows():
    """R17 on hand-built rows whose scales and E4M3 codes are known: row 0 has max 7, so
    s = 7/448 = 2^-6 and the quotients are v * 64; row 1 has max 14 (s = 2^-5, v * 32),
    so a per-row scale gives each row its own grid.  Expected values, worked by hand:
      row 0: 7 -> 448 (code 0x7E); 3.5 -> 224; -1.75 -> -112; 17/64 -> 17 is the tie
      between 16 and 18 on the spacing-2 binade [16, 32), even mantissa: 16 (code 0x58:
      exponent field 4 + 7, mantissa 0) -> 0.25;
      19/64 -> tie between 18 and 20, even: 20 -> 20/64; 3 * 2^-16 -> 3 * 2^-10 is the
      tie between the subnormals 2^-9 and 2 * 2^-9, even: 2^-8 -> 2^-14;
      1 + 2^-9 -> stored as bf16 first: the tie between 1 and 1 + 2^-7 rounds to 1,
      then 64 -> 1.0; 0 -> 0.
      row 1: 14 -> 448; -14 -> -448; 0.5 -> 16 -> 0.5; 5/32 -> 5 (exact in [4, 8) with
      spacing 0.5) -> 5/32."""
    r0 = [7.0, 3.5, -1.75, 17 / 64, 19 / 64, 3 * 2.0 ** -16, 1.0 + 2.0 ** -9, 0.0]
    r1 = [14.0, -14.0, 0.5, 5 / 32, 0.0, 0.0, 0.0, 0.0]
    got = oracle.fp8_activation(np.array([r0, r1]))
    want0 = [7.0, 3.5, -1.75, 0.25, 20 / 64, 2.0 ** -14, 1.0, 0.0]
    want1 = [14.0, -14.0, 0.5, 5 / 32, 0.0, 0.0, 0.0, 0.0]
    assert got.tolist() == [want0, want1]
    q, s = oracle.quantize_fp8_rows(oracle.bf16_round(np.array([r0, r1])).astype(np.float32))
    assert s.tolist() == [2.0 ** -6, 2.0 ** -5]
    assert q[0, 0] == 0x7E and q[1, 1] == 0xFE and q[0, 3] == 0x58 and q[0, 5] == 0x02


def test_gated_mlp_fp8_matches_torch_float8():
    """R17: the fp8 gated MLP against the same steps written with the library's own
    pieces: bfloat16 storage, per-row scales max|row| / 448 in fp32, float8_e4m3fn
    rounding, float64 matmuls and torch's gelu(tanh).  The rows' quotients never exceed
    448 (where the library's conversion, unlike the kernels', does not saturate)."""
    T, H, I = 7, 48, 24
    u = RNG.standard_normal((T, H)) * 1.3
    wgu = RNG.standard_normal((2 * I, H)) * 0.2
    wd = RNG.standard_normal((H, I)) * 0.2

    def q8(v):
        b = torch.from_numpy(v).to(torch.bfloat16).to(torch.float32)
        s = b.abs().amax(dim=1, keepdim=True) / 448.0
        s = torch.where(s > 0, s, torch.ones_like(s))
        return (b / s).to(torch.float8_e4m3fn).to(torch.float64) * s.to(torch.float64)

    uq = q8(u)
    g = uq @ torch.from_numpy(wgu[:I]).T
    v = uq @ torch.from_numpy(wgu[I:]).T
    h = F.gelu(g, approximate="tanh") * v
    ref = (q8(h.numpy()) @ torch.from_numpy(wd).T).numpy()
    got = oracle.gated_mlp_fp8(u, wgu, wd)
    np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-12)


def test_topk_gaps_hand_computed():
    """The gap filter's measure on hand-computed rows: the smallest adjacent gap among the
    k + 1 largest logits, the (k+1)-th included and everything past it ignored.
      [0.5, 0.1, 0.9, 0.45, -1.0], k = 2: sorted 0.9, 0.5, 0.45 -> gaps 0.4, 0.05 -> 0.05
        (the gap between the k-th and the (k+1)-th, which decides the selected set);
      [1.0, 0.8, 0.5, 0.49], k = 2: top three 1.0, 0.8, 0.5 -> 0.2 (0.01 lies past them);
      [0.3, 0.3, 0.1, 0.0], k = 1: a tie at the top -> 0;
      [2.0, -1.0, 0.5], k = 3 (k = E): all three -> min(1.5, 1.5) = 1.5."""
    g = oracle.topk_gaps(np.array([[0.5, 0.1, 0.9, 0.45, -1.0], [1.0, 0.8, 0.5, 0.49, -5.0]]), 2)
    np.testing.assert_allclose(g, [0.05, 0.2], rtol=0, atol=1e-15)
    assert oracle.topk_gaps(np.array([[0.3, 0.3, 0.1, 0.0]]), 1).tolist() == [0.0]
    assert oracle.topk_gaps(np.array([[2.0, -1.0, 0.5]]), 3).tolist() == [1.5]


# ------------------------------------------------------------------ NVFP4 (E2M1 + E4M3 blocks)

def test_e2m1_table_and_rounding_by_brute_force():
    """R18: the E2M1 values written out from the format (0, 0.5, 1, 1.5, 2, 3, 4, 6 and
    their negatives), and rounding equal to a brute-force nearest-value search that breaks
    ties towards the code with an even mantissa bit, saturating at 6."""
    tab = oracle.e2m1_decode_table()
    assert tab[:8].tolist() == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert np.array_equal(tab[8:], -tab[:8])
    grid = tab[:8]

    def brute(v):
        a = min(abs(v), 6.0)
        d = np.abs(grid - a)
        best = np.flatnonzero(d == d.min())
        pick = best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]
        return np.copysign(grid[pick], v)

    pos = grid
    v = np.concatenate([RNG.uniform(-8, 8, 3000), (pos[:-1] + pos[1:]) / 2,
                        -(pos[:-1] + pos[1:]) / 2, [0.0, 6.0, 6.5, 1e9]])
    assert np.array_equal(oracle.e2m1_round(v), np.array([brute(x) for x in v]))
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(oracle.e2m1_encode(tab[codes]), codes)


def test_nvfp4_quantiser_pins():
    """R18: the tensor scale maps the matrix max to 448 * 6; every block scale is an E4M3
    value and makes the block's max land within rounding of 6; each weight is within half
    an E2M1 step (times b t) of its dequantised value; zero blocks and an all-zero matrix
    give zero codes."""
    w = synth.normal_bf16(9, (5,), (6, 64), 0.02)
    w[2, :16] = 0                                    # one all-zero block
    q, bc, t = oracle.quantize_nvfp4(w)
    wf = synth.bf16_bits_to_f32(w).astype(np.float64)
    assert t == np.float32(np.abs(wf).max() / (448 * 6))
    b = oracle.e4m3_decode_table()[bc]
    assert np.all(np.isfinite(b)) and np.all(b >= 0)
    deq = oracle.dequantize_nvfp4(q, bc, t)
    bt = np.repeat(b, 16, axis=-1) * float(t)
    # half the E2M1 step at |w| (0.25 below 2, else 2^(floor(log2)-2)), scaled, plus
    # the saturation excess where rounding the block scale down pushed w / (b t) above 6
    a = np.abs(wf) / np.where(bt > 0, bt, 1)
    step = np.where(a < 1, 0.5, 2.0 ** (np.floor(np.log2(np.maximum(a, 1))) - 1))
    bound = step / 2 * bt + np.maximum(np.abs(wf) - 6 * bt, 0)
    assert np.all(np.abs(deq - wf) <= bound * (1 + 1e-6) + 1e-30)
    assert np.all(q[2, :16] == 0) and bc[2, 0] == 0
    z = np.zeros((2, 32), dtype=np.uint16)
    qz, bz, tz = oracle.quantize_nvfp4(z)
    assert tz == 1.0 and np.all(qz == 0) and np.all(bz == 0)


def test_nvfp4_experts_in_the_block():
    """R18 through the whole block: each expert matrix carries its own tensor scale; the
    block runs on the dequantised weights (activations untouched), so its MoE branch stays
    close to the bf16 one (4-bit weights: a few percent) and the all-experts-dense
    identity holds exactly."""
    c = cases.make_case(synth.TINY, seed=1234)
    p, E = c.p, c.shape.E
    nv = {"gate_up": [oracle.quantize_nvfp4(p["w_gate_up"][e]) for e in range(E)],
          "down": [oracle.quantize_nvfp4(p["w_down"][e]) for e in range(E)]}
    ex = oracle.Experts(nvfp4=nv)
    o4 = oracle.block_forward(c.x, p, ex, c.shape.k, c.shape.eps, c.bias)
    o16 = oracle.block_forward(c.x, p, cases.bf16_experts(p), c.shape.k, c.shape.eps, c.bias)
    rel = np.abs(o4["moe"] - o16["moe"]).max() / np.abs(o16["moe"]).max()
    assert 1e-3 < rel < 0.3
    assert np.array_equal(o4["topk_idx"], o16["topk_idx"])      # the router is untouched
    dense = oracle.block_forward(c.x, p, ex, c.shape.k, c.shape.eps, c.bias,
                                 all_experts_dense=True)
    np.testing.assert_allclose(dense["moe"], o4["moe"], rtol=1e-10, atol=1e-12)


# ------------------------------------------------------------------ the bar discriminates

def test_fp16_accumulation_fails_the_bar():
    """P9 (negative control): expert GEMMs that accumulate in fp16 at H = 2816 miss the
    bar (on these synthetic weights by the max-abs term; the page's cosine ~0.97 was
    seen on the real checkpoint and is not asserted), while fp32 accumulation with bf16 storage of xn and h meets it
    (ONNX export card, "MoE dispatch": fp16-accumulated expert GEMMs lose accuracy at
    this hidden size)."""
    H, I, n = 2816, 704, 6
    wgu = synth.normal_bf16(11, (1,), (2 * I, H), 0.02)
    wd = synth.normal_bf16(11, (2,), (H, I), 0.02)
    u = oracle.bf16(synth.x_rows(12, H, n))
    W1, W2 = oracle.bf16(wgu), oracle.bf16(wd)
    ref = oracle.gated_mlp(u, W1, W2)

    def dot_fp16(a, B):  # sequential fp16 accumulation of fp16-rounded products
        prod = (a[:, None, :] * B[None, :, :]).astype(np.float16)
        return np.cumsum(prod, axis=-1, dtype=np.float16)[..., -1].astype(np.float64)

    u16 = u.astype(np.float16).astype(np.float64)
    g = dot_fp16(u16, W1[:I])
    v = dot_fp16(u16, W1[I:])
    h = (oracle.gelu_tanh(g) * v).astype(np.float16).astype(np.float64)
    y16 = dot_fp16(h, W2)
    with pytest.raises(AssertionError, match="max-abs"):
        cases.check_bar(y16, ref, cases.FRAC_BF16, "fp16-accumulate model")

    def to_bf16(a):
        return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(a.astype(np.float32))).astype(np.float64)

    ub = to_bf16(u)
    g32 = (ub.astype(np.float32) @ W1[:I].T.astype(np.float32)).astype(np.float64)
    v32 = (ub.astype(np.float32) @ W1[I:].T.astype(np.float32)).astype(np.float64)
    h32 = to_bf16(oracle.gelu_tanh(g32) * v32)
    y32 = (h32.astype(np.float32) @ W2.T.astype(np.float32)).astype(np.float64)
    cases.check_bar(to_bf16(y32), ref, cases.FRAC_BF16, "fp32-accumulate model")


# ------------------------------------------------------------------ workloads

def test_layer_shape_matches_the_pages():
    with open(os.path.join(cases.GOLDEN, "gemma4_26b_a4b_moe.json")) as f:
        g = json.load(f)
    s = synth.DECODE
    assert (s.H, s.E, s.k, s.I, s.D) == (g["hidden_size"], g["num_experts"], g["top_k"],
                                         g["moe_intermediate_size"], g["intermediate_size"])
    assert synth.STACK_LAYERS == g["num_layers"]
    assert synth.PREFILL.H == s.H and synth.PREFILL.T == 2048


def test_gap_filter_gives_unique_topk():
    c = cases.make_case(synth.TINY, seed=42)
    r = oracle.router(oracle.bf16(c.x), oracle.bf16(c.p["router_scale"]), oracle.bf16(c.p["w_router"]),
                      None, oracle.bf16(c.p["per_expert_scale"]), c.shape.k, c.shape.eps)
    assert oracle.topk_gaps(r["logits"], c.shape.k).min() >= cases.MIN_GAP


def test_zipf_workload_is_skewed():
    """The calibrated offset leaves some experts near or above ten times the mean load
    and at least one expert empty."""
    shape = synth.PREFILL
    p = synth.make_router(1234, shape)
    x = synth.x_rows(1235, shape.H, shape.T)
    b = synth.zipf_bias(1234, shape.E, cases.zipf_alpha())
    r = oracle.router(oracle.bf16(x), oracle.bf16(p["router_scale"]), oracle.bf16(p["w_router"]),
                      b, oracle.bf16(p["per_expert_scale"]), shape.k, shape.eps)
    c = np.bincount(r["topk_idx"].reshape(-1), minlength=shape.E)
    mean = shape.T * shape.k / shape.E
    assert (c == 0).sum() >= 1
    assert (c >= 8 * mean).sum() >= 2
