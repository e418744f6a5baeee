"""FP8 experts (E4M3 weights with per-output-row scales and dynamic per-token E4M3
activations, the FP8-dynamic variant of the "Gemma 4 26B-A4B IT" recipe page) through
the C interface: the GPU quantiser must produce the oracle's codes and scales bit for
bit, and the block must meet the fp8 bar (per-row cosine >= 0.9999, max-abs <= 4e-2 *
rms) against the oracle, which quantises the same bf16 activations per token."""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_05_b200 as mf
import oracle
import synth
from tests import cases
from tests.gpu_util import (bf16_np, config, device_layer, fp8_experts, run_permute, run_router,
                            to_dev)

pytestmark = pytest.mark.gpu

SHAPES = {
    "tiny": synth.TINY,
    "tiny_T37": synth.Shape(T=37, H=512, E=16, k=4, I=128, D=384),
    "fp8_T1": synth.Shape(T=1, H=2816, E=128, k=8, I=704, D=2112),
    "fp8_T64": synth.Shape(T=64, H=2816, E=128, k=8, I=704, D=2112),
    "fp8_T1024": synth.Shape(T=1024, H=2816, E=128, k=8, I=704, D=2112),
    # the interface limits: H = 6144, E = 256, k = 16, and the smallest I = D = 128
    "limits_T300": synth.Shape(T=300, H=6144, E=256, k=16, I=128, D=128),
}
ROUTER_STD = {"limits_T300": 0.3}  # wider router weights, so the gap filter finds rows


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    mf.lib()


def _setup(name):
    c = cases.make_case(SHAPES[name], seed=1234, router_std=ROUTER_STD.get(name))
    dev8, ex8, same = fp8_experts(c)
    layer = dict(device_layer(c))
    layer.update(dev8)
    return c, config(c.shape, fp8=True), layer, ex8, same


_ORC: dict = {}


def _oracle(c, ex8):
    key = (id(c.p), hash(c.x.tobytes()))
    if key not in _ORC or _ORC[key][0] is not c.p:
        _ORC.clear()
        _ORC[key] = (c.p, oracle.block_forward(c.x, c.p, ex8, c.shape.k, c.shape.eps, c.bias))
    return _ORC[key][1]


@pytest.mark.parametrize("name", list(SHAPES))
def test_fp8_quantiser_matches_oracle(name):
    *_, same = _setup(name)
    assert same


def test_fp8_quantiser_edge_rows():
    """Saturation, ties and an all-zero row through the GPU quantiser, against the
    oracle's codes: rows whose max is 448 s make every other value an exact multiple of
    the scale, so E4M3 ties (x.5 steps) and the subnormal range are hit on purpose."""
    steps = np.array([448.0, 1.0625, 1.1875, -3 * 2.0 ** -10, 2.0 ** -10, 300.0, -448.0, 0.5],
                     dtype=np.float32)
    rows = np.stack([steps, steps * np.float32(2.0 ** -20), np.zeros(8, np.float32),
                     steps[::-1] * np.float32(7.0)])
    w = synth.f32_to_bf16_bits(rows)
    q = torch.empty(rows.shape, dtype=torch.uint8, device="cuda")
    s = torch.empty(rows.shape[0], dtype=torch.float32, device="cuda")
    mf.moe_quantize_fp8(to_dev(w), q, s)
    qo, so = oracle.quantize_fp8_per_channel(w)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


@pytest.mark.parametrize("name", list(SHAPES))
def test_fp8_expert_branch(name):
    c, cfg, layer, ex8, _ = _setup(name)
    r = run_router(cfg, c, layer)
    p = run_permute(cfg, r["topk_idx"])
    moe = torch.empty(c.shape.T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    ws = mf.workspace(cfg, c.shape.T)
    mf.moe_ffn_forward(cfg, r["xn_moe"], r["topk_w"], p["offsets"], p["sorted_src"], p["inv_pos"],
                       layer, moe, ws)
    assert mf.moe_check_device_status(ws) == mf.MOE_OK
    cases.check_bar(bf16_np(moe), _oracle(c, ex8)["moe"], cases.FRAC_FP8, f"fp8 moe {name}")


@pytest.mark.parametrize("name", list(SHAPES))
def test_fp8_block(name):
    c, cfg, layer, ex8, _ = _setup(name)
    T = c.shape.T
    out = torch.empty(T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    moe = torch.empty(T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    ws = mf.workspace(cfg, T)
    mf.moe_block_forward(cfg, to_dev(c.x), mf.BlockWeights(cfg, layer), out, ws, moe_out=moe)
    assert mf.moe_check_device_status(ws) == mf.MOE_OK
    o = _oracle(c, ex8)
    cases.check_bar(bf16_np(out), o["out"], cases.FRAC_FP8, f"fp8 out {name}")
    cases.check_bar(bf16_np(moe), o["moe"], cases.FRAC_FP8, f"fp8 moe_out {name}")


def test_fp8_block_is_deterministic():
    c, cfg, layer, _, _ = _setup("fp8_T64")
    bw = mf.BlockWeights(cfg, layer)
    outs = []
    for _ in range(2):
        out = torch.empty(c.shape.T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
        ws = mf.workspace(cfg, c.shape.T)
        mf.moe_block_forward(cfg, to_dev(c.x), bw, out, ws)
        outs.append(out)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
