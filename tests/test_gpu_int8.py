"""int8 expert weights (per-output-channel symmetric int8, the int8 build of the
Inferentia2 card) through the C interface: the GPU quantiser must produce the oracle's
codes and scales bit for bit, and the block with int8 experts must meet the int8 bar
(per-row cosine >= 0.9999, max-abs <= 4e-2 * rms) against the oracle run on the
oracle's own dequantised weights."""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_05_b200 as mf
import oracle
import synth
from tests import cases
from tests.gpu_util import (bf16_np, config, device_layer, int8_experts, run_permute, run_router,
                            to_dev)

pytestmark = pytest.mark.gpu

SHAPES = {
    "tiny": synth.TINY,
    "tiny_T37": synth.Shape(T=37, H=512, E=16, k=4, I=128, D=384),
    "int8_T1": synth.Shape(T=1, H=2816, E=128, k=8, I=704, D=2112),
    "int8_T64": synth.Shape(T=64, H=2816, E=128, k=8, I=704, D=2112),
    "int8_T1024": synth.Shape(T=1024, H=2816, E=128, k=8, I=704, D=2112),
    # the interface limits: H = 6144, E = 256, k = 16, and the smallest I = D = 128
    "limits_T300": synth.Shape(T=300, H=6144, E=256, k=16, I=128, D=128),
    # the same limits on the weight-streaming kernel of small batches
    "limits_T48": synth.Shape(T=48, H=6144, E=256, k=16, I=128, D=128),
    # Zipf-skewed routing on the weight-streaming kernel: the busiest experts hold more than
    # one 32-token chunk, and the dense MLP's 256 tokens are eight chunks
    "int8_T256_zipf": synth.Shape(T=256, H=2816, E=128, k=8, I=704, D=2112),
}
ROUTER_STD = {"limits_T300": 0.3, "limits_T48": 0.3}  # wider router weights (gap filter)
ZIPF = {"int8_T256_zipf"}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    mf.lib()


def _setup(name):
    c = cases.make_case(SHAPES[name], seed=1234, zipf=name in ZIPF, router_std=ROUTER_STD.get(name))
    dev8, ex8, same = int8_experts(c)
    layer = dict(device_layer(c))
    layer.update(dev8)
    return c, config(c.shape, int8=True), layer, ex8, same


_ORC: dict = {}


def _oracle(c, ex8):
    key = (id(c.p), hash(c.x.tobytes()))
    if key not in _ORC or _ORC[key][0] is not c.p:
        _ORC.clear()
        _ORC[key] = (c.p, oracle.block_forward(c.x, c.p, ex8, c.shape.k, c.shape.eps, c.bias))
    return _ORC[key][1]


@pytest.mark.parametrize("name", list(SHAPES))
def test_int8_quantiser_matches_oracle(name):
    *_, same = _setup(name)
    assert same


@pytest.mark.parametrize("name", list(SHAPES))
def test_int8_expert_branch(name):
    c, cfg, layer, ex8, _ = _setup(name)
    r = run_router(cfg, c, layer)
    p = run_permute(cfg, r["topk_idx"])
    moe = torch.empty(c.shape.T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    ws = mf.workspace(cfg, c.shape.T)
    mf.moe_ffn_forward(cfg, r["xn_moe"], r["topk_w"], p["offsets"], p["sorted_src"], p["inv_pos"],
                       layer, moe, ws)
    assert mf.moe_check_device_status(ws) == mf.MOE_OK
    cases.check_bar(bf16_np(moe), _oracle(c, ex8)["moe"], cases.FRAC_INT8, f"int8 moe {name}")


@pytest.mark.parametrize("name", list(SHAPES))
def test_int8_block(name):
    c, cfg, layer, ex8, _ = _setup(name)
    T = c.shape.T
    out = torch.empty(T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    moe = torch.empty(T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    ws = mf.workspace(cfg, T)
    mf.moe_block_forward(cfg, to_dev(c.x), mf.BlockWeights(cfg, layer), out, ws, moe_out=moe)
    assert mf.moe_check_device_status(ws) == mf.MOE_OK
    o = _oracle(c, ex8)
    cases.check_bar(bf16_np(out), o["out"], cases.FRAC_INT8, f"int8 out {name}")
    cases.check_bar(bf16_np(moe), o["moe"], cases.FRAC_INT8, f"int8 moe_out {name}")


def test_int8_block_is_deterministic():
    c, cfg, layer, _, _ = _setup("int8_T64")
    bw = mf.BlockWeights(cfg, layer)
    outs = []
    for _ in range(2):
        out = torch.empty(c.shape.T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
        ws = mf.workspace(cfg, c.shape.T)
        mf.moe_block_forward(cfg, to_dev(c.x), bw, out, ws)
        outs.append(out)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
