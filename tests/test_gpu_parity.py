"""Parity of the CUDA path with the oracle, through the C interface, on a B200.

Indices and the permutation are compared bit for bit; floating-point outputs at the
accuracy bar (per-row cosine >= 0.9999, max-abs error <= 2e-2 * rms of the oracle row,
plus half a bf16 ulp for the bf16 output format).
"""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_05_b200 as mf
import oracle
import synth
from tests import cases
from tests.gpu_util import (bf16_np, config, device_layer, oracle_block, run_block, run_permute,
                            run_router, to_dev)

pytestmark = pytest.mark.gpu

# name -> (shape, zipf offset).  The "limits" case (largest H, E and k the interface
# takes) draws its router weights with std 0.3 so that its 16-of-256 top-k has gaps of
# at least 1e-3 often enough to draw inputs.
ROUTER_STD = {"limits": 0.3, "limits_T300": 0.3}
SHAPES = {
    "tiny": (synth.TINY, False),
    "tiny_T37": (synth.Shape(T=37, H=512, E=16, k=4, I=128, D=384), False),
    "tiny_T1": (synth.Shape(T=1, H=512, E=16, k=4, I=128, D=384), False),
    "decode_T8": (synth.DECODE, False),
    "decode_T1": (synth.Shape(T=1, H=2816, E=128, k=8, I=704, D=2112), False),
    "decode_T64": (synth.Shape(T=64, H=2816, E=128, k=8, I=704, D=2112), False),
    # the largest batch of the small-batch router (16 token blocks, the multi-block sort)
    "decode_T128": (synth.Shape(T=128, H=2816, E=128, k=8, I=704, D=2112), False),
    "prefill_T2048_zipf": (synth.PREFILL, True),
    "limits": (synth.Shape(T=5, H=6144, E=256, k=16, I=128, D=128), False),
    # batches above 128 tokens take the tensor-core router: ragged last token tile,
    # the smallest expert count (N = 16), and the largest H, E and k
    "tiny_T200": (synth.Shape(T=200, H=512, E=16, k=4, I=128, D=384), False),
    "decode_T160": (synth.Shape(T=160, H=2816, E=128, k=8, I=704, D=2112), False),
    "limits_T300": (synth.Shape(T=300, H=6144, E=256, k=16, I=128, D=128), False),
}
FAST = ["tiny", "tiny_T37", "tiny_T1", "decode_T8", "decode_T1", "decode_T64"]


def _case(name):
    shape, zipf = SHAPES[name]
    return cases.make_case(shape, seed=1234, zipf=zipf, router_std=ROUTER_STD.get(name))


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    mf.lib()


# ------------------------------------------------------------------ router

@pytest.mark.parametrize("name", list(SHAPES))
def test_router(name):
    c = _case(name)
    cfg = config(c.shape)
    layer = device_layer(c)
    r = run_router(cfg, c, layer)
    o = oracle_block(c)
    assert np.array_equal(r["topk_idx"].cpu().numpy(), o["topk_idx"])
    got_w = r["topk_w"].cpu().numpy().astype(np.float64)
    # Both routers take the logits from tensor-core sums of the two-term split of W'
    # (2H/16 products of 16 terms, added into fp32 accumulators: one, or one per term and
    # then the two sums); each addition may lose up to one unit in the last place of the
    # accumulator (nothing promises round-to-nearest inside the tensor core), so a logit
    # may be off by steps * 2^-23 * max|l - b| and a weight, exp(l_j - l_0) / sum, by four
    # times that, relatively.
    lraw = np.abs(o["logits"] - (0.0 if c.bias is None else c.bias[None, :]))
    steps = 2 * c.shape.H / 16
    rtol = 2e-6 + 4 * steps * 2.0 ** -23 * lraw.max(axis=1, keepdims=True)
    err = np.abs(got_w - o["topk_w"]) / np.abs(o["topk_w"])
    assert np.all(err <= rtol), f"topk_w: worst {err.max():.3g} over {rtol.max():.3g}"
    for nm in ("xn_moe", "xn_dense"):
        got = bf16_np(r[nm])
        ref = o[nm]
        allow = cases.half_ulp_bf16(ref) * (1 + 1e-5) + 2e-6 * np.abs(ref)
        assert np.all(np.abs(got - ref) <= allow), nm


# ------------------------------------------------------------------ permutation

@pytest.mark.parametrize("T,k,E", [(8, 4, 16), (37, 8, 128), (1, 8, 128), (2048, 8, 128),
                                   (1025, 8, 128), (3000, 16, 256), (16384, 8, 128)])
def test_permute_bit_exact(T, k, E):
    rng = np.random.default_rng(T * 131 + k)
    # skewed ids: some experts empty, some hot
    p = rng.zipf(1.3, size=(T, k)) % E
    idx = p.astype(np.int32)
    cfg = mf.Config(512, E, k, 128, 128)
    got = run_permute(cfg, to_dev(idx, torch.int32))
    offs, src, inv = oracle.permute(idx, E)
    n = T * k
    assert np.array_equal(got["offsets"].cpu().numpy(), offs)
    assert np.array_equal(got["sorted_src"].cpu().numpy()[:n], src)
    assert np.array_equal(got["inv_pos"].cpu().numpy()[:n], inv)


def test_permute_drops_invalid_ids():
    idx = np.array([[3, -1], [16, 3], [0, 2]], dtype=np.int32)  # E = 16: -1 and 16 invalid
    cfg = mf.Config(512, 16, 2, 128, 128)
    got = run_permute(cfg, to_dev(idx, torch.int32))
    flat = idx.reshape(-1)
    valid = np.nonzero((flat >= 0) & (flat < 16))[0]
    order = valid[np.argsort(flat[valid], kind="stable")]
    offs = got["offsets"].cpu().numpy()
    assert offs[-1] == len(valid)
    assert np.array_equal(got["sorted_src"].cpu().numpy()[:len(valid)], order)


# ------------------------------------------------------------------ branches

@pytest.mark.parametrize("name", FAST + ["prefill_T2048_zipf", "limits"])
def test_expert_branch(name):
    """moe_ffn_forward: the routed experts before their post norm."""
    c = _case(name)
    cfg = config(c.shape)
    layer = device_layer(c)
    r = run_router(cfg, c, layer)
    p = run_permute(cfg, r["topk_idx"])
    moe = torch.empty(c.shape.T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    ws = mf.workspace(cfg, c.shape.T)
    mf.moe_ffn_forward(cfg, r["xn_moe"], r["topk_w"], p["offsets"], p["sorted_src"], p["inv_pos"],
                       layer, moe, ws)
    assert mf.moe_check_device_status(ws) == mf.MOE_OK
    cases.check_bar(bf16_np(moe), oracle_block(c)["moe"], cases.FRAC_BF16, f"moe {name}")


@pytest.mark.parametrize("name", FAST + ["prefill_T2048_zipf", "limits"])
def test_dense_branch(name):
    c = _case(name)
    cfg = config(c.shape)
    layer = device_layer(c)
    r = run_router(cfg, c, layer)
    out = torch.empty(c.shape.T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    ws = mf.workspace(cfg, c.shape.T)
    mf.dense_mlp_forward(cfg, r["xn_dense"], layer["w_dense_gate_up"], layer["w_dense_down"], out, ws)
    assert mf.moe_check_device_status(ws) == mf.MOE_OK
    cases.check_bar(bf16_np(out), oracle_block(c)["dense"], cases.FRAC_BF16, f"dense {name}")


# ------------------------------------------------------------------ the block

@pytest.mark.parametrize("name", list(SHAPES))
def test_block(name):
    c = _case(name)
    cfg = config(c.shape)
    out, moe = run_block(cfg, c, device_layer(c))
    o = oracle_block(c)
    cases.check_bar(bf16_np(out), o["out"], cases.FRAC_BF16, f"out {name}")
    cases.check_bar(bf16_np(moe), o["moe"], cases.FRAC_BF16, f"moe_out {name}")


@pytest.mark.parametrize("seed", [99, 7, 11])
def test_block_at_the_limits_over_seeds(seed):
    """The interface limits (H = 6144, E = 256, k = 16, I = D = 128, T = 300) meet the bar
    for other seeds than the fixed one as well: the bf16 rounding of the GEMM operands is
    the whole error budget there (an emulation of the pipeline over six seeds reached at
    most 0.93 of the bar on `out`; with D = 64 it reached 1.15, which is why I and D start
    at 128)."""
    shape, _ = SHAPES["limits_T300"]
    c = cases.make_case(shape, seed=seed, router_std=ROUTER_STD["limits_T300"])
    cfg = config(c.shape)
    out, moe = run_block(cfg, c, device_layer(c))
    o = oracle_block(c)
    w1 = cases.check_bar(bf16_np(out), o["out"], cases.FRAC_BF16, f"out limits seed {seed}")
    w2 = cases.check_bar(bf16_np(moe), o["moe"], cases.FRAC_BF16, f"moe_out limits seed {seed}")
    print("limits seed", seed, w1, w2)


def test_block_extreme_skew_T16384():
    """Every token of a 16384-token batch routed to the same 8 experts (a logit offset of
    43..50 on experts 0..7, far above the logits' spread): 16384 tokens per expert, 64
    tiles of 256 tokens each, 120 experts with no token.  The ids must be exactly 0..7 in
    offset order for every token, and sampled rows (first, last, and spread over the
    batch) must meet the bar against the oracle block."""
    shape = synth.Shape(T=16384, H=2816, E=128, k=8, I=704, D=2112)
    base = cases.make_case(synth.DECODE, seed=1234)          # the layer's weights
    bias = np.zeros(shape.E, dtype=np.float32)
    bias[:8] = 50.0 - np.arange(8, dtype=np.float32)
    x = synth.x_rows(4242, shape.H, shape.T)
    c = cases.Case(shape, x, base.p, bias, 4242)
    cfg = config(shape)
    layer = device_layer(c)
    T = shape.T
    xd = to_dev(x)
    r = run_router(cfg, c, layer, x=xd)
    assert torch.equal(r["topk_idx"].cpu(), torch.arange(8, dtype=torch.int32).repeat(T, 1))
    out, moe = run_block(cfg, c, layer, x=xd)
    rows = np.unique(np.concatenate([[0, 1, T - 1], np.linspace(0, T - 1, 61).astype(int)]))
    o = oracle.block_forward(x[rows], c.p, cases.bf16_experts(c.p), shape.k, shape.eps, bias)
    cases.check_bar(bf16_np(out)[rows], o["out"], cases.FRAC_BF16, "out, extreme skew")
    cases.check_bar(bf16_np(moe)[rows], o["moe"], cases.FRAC_BF16, "moe_out, extreme skew")


def test_block_without_branch_post_norms():
    """g_post_moe / g_post_dense given as NULL skip those norms."""
    c = _case("tiny_T37")
    cfg = config(c.shape)
    layer = device_layer(c)
    layer.pop("g_post_moe")
    layer.pop("g_post_dense")
    out, _ = run_block(cfg, c, layer)
    p = dict(c.p, g_post_moe=None, g_post_dense=None)
    o = oracle.block_forward(c.x, p, cases.bf16_experts(c.p), c.shape.k, c.shape.eps, c.bias)
    cases.check_bar(bf16_np(out), o["out"], cases.FRAC_BF16, "out without branch post norms")


@pytest.mark.parametrize("name", ["decode_T8", "prefill_T2048_zipf"])
def test_block_is_deterministic(name):
    c = _case(name)
    cfg = config(c.shape)
    layer = device_layer(c)
    a, ma = run_block(cfg, c, layer)
    b, mb = run_block(cfg, c, layer)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(ma.view(torch.int16), mb.view(torch.int16))


@pytest.mark.parametrize("name", ["tiny_T37", "decode_T64", "tiny_T200"])
def test_block_rows_are_independent(name):
    """Shuffling the tokens shuffles the outputs the same way, bit for bit."""
    c = _case(name)
    cfg = config(c.shape)
    layer = device_layer(c)
    a, _ = run_block(cfg, c, layer)
    perm = np.random.default_rng(5).permutation(c.shape.T)
    c2 = cases.Case(c.shape, c.x[perm], c.p, c.bias, c.seed)
    b, _ = run_block(cfg, c2, layer)
    assert torch.equal(b.view(torch.int16), a[torch.from_numpy(perm).cuda()].view(torch.int16))


def test_block_zero_tokens():
    c = _case("tiny")
    cfg = config(c.shape)
    bw = mf.BlockWeights(cfg, device_layer(c))
    x = torch.empty(0, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(0, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    ws = mf.workspace(cfg, 0)
    mf.moe_block_forward(cfg, x, bw, out, ws)


def test_zipf_case_has_empty_and_hot_experts():
    c = _case("prefill_T2048_zipf")
    idx = oracle_block(c)["topk_idx"]
    cnt = np.bincount(idx.reshape(-1), minlength=c.shape.E)
    assert (cnt == 0).sum() >= 1 and cnt.max() >= 8 * c.shape.T * c.shape.k / c.shape.E


# ------------------------------------------------------------------ int8 quantiser

def test_quantize_int8_bit_exact():
    w = synth.normal_bf16(77, (1,), (300, 2816), 0.02)
    w[5] = 0                                              # all-zero row
    row = np.zeros(2816, dtype=np.float32)
    row[:5] = [127 / 128, 2.5 / 128, 3.5 / 128, -2.5 / 128, -0.5 / 128]   # halves to even
    w[7] = synth.f32_to_bf16_bits(row)
    q = torch.empty(w.shape, dtype=torch.int8, device="cuda")
    s = torch.empty(w.shape[0], dtype=torch.float32, device="cuda")
    mf.moe_quantize_int8(to_dev(w), q, s)
    qo, so = oracle.quantize_int8_per_channel(w)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
