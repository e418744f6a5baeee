"""NVFP4 expert weights (the "NVFP4 (4-bit) quantized weights" of the "Gemma 4 26B-A4B IT"
recipe page's variant list; weight-only, reading R18) through the C interface: the GPU
quantiser must produce the oracle's E2M1 codes, E4M3 block scales and fp32 matrix scales
bit for bit, and the block with NVFP4 experts must meet the bar of 8-bit weights (per-row
cosine >= 0.9999, max-abs <= 4e-2 * rms) against the oracle run on the oracle's own
dequantised weights.  Every batch size runs on the weight-streaming kernel."""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_05_b200 as mf
import oracle
import synth
from tests import cases
from tests.gpu_util import (bf16_np, config, device_layer, nvfp4_experts, run_permute,
                            run_router, to_dev, unpack_nvfp4)

pytestmark = pytest.mark.gpu

SHAPES = {
    "tiny": synth.TINY,
    "tiny_T37": synth.Shape(T=37, H=512, E=16, k=4, I=128, D=384),
    "nvfp4_T1": synth.Shape(T=1, H=2816, E=128, k=8, I=704, D=2112),
    "nvfp4_T64": synth.Shape(T=64, H=2816, E=128, k=8, I=704, D=2112),
    "nvfp4_T1024": synth.Shape(T=1024, H=2816, E=128, k=8, I=704, D=2112),
    # the interface limits (H = 6144, E = 256, k = 16, the smallest I = D = 128: the down
    # matmul's K is half of one 256-wide NVFP4 item)
    "limits_T48": synth.Shape(T=48, H=6144, E=256, k=16, I=128, D=128),
    "nvfp4_T256_zipf": synth.Shape(T=256, H=2816, E=128, k=8, I=704, D=2112),
}
ROUTER_STD = {"limits_T48": 0.3}
ZIPF = {"nvfp4_T256_zipf"}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    mf.lib()


def _cfg(shape):
    c = config(shape)
    return mf.Config(c.hidden, c.num_experts, c.top_k, c.expert_inter, c.dense_inter, c.eps,
                     nvfp4=True)


def _setup(name):
    c = cases.make_case(SHAPES[name], seed=1234, zipf=name in ZIPF, router_std=ROUTER_STD.get(name))
    dev4, ex4, same = nvfp4_experts(c)
    layer = dict(device_layer(c))
    layer.update(dev4)
    return c, _cfg(c.shape), layer, ex4, same


_ORC: dict = {}


def _oracle(c, ex4):
    key = (id(c.p), hash(c.x.tobytes()))
    if key not in _ORC or _ORC[key][0] is not c.p:
        _ORC.clear()
        _ORC[key] = (c.p, oracle.block_forward(c.x, c.p, ex4, c.shape.k, c.shape.eps, c.bias))
    return _ORC[key][1]


def test_unpack_layout_round_trip():
    """The packed layout read back by the test helper: element e of each group of 8 sits in
    nibble 2e (e < 4) ... written out by hand for one word."""
    codes = np.arange(8, dtype=np.uint8)             # elements 0..7 carry codes 0..7
    word = 0
    for e, c in enumerate(codes):
        nib = e // 2 if e % 2 == 0 else 4 + e // 2
        word |= int(c) << (4 * nib)
    packed = np.array([word], dtype=np.uint32).view(np.uint8)
    assert unpack_nvfp4(packed[None, :])[0].tolist() == codes.tolist()


@pytest.mark.parametrize("name", ["tiny", "nvfp4_T1", "limits_T48"])
def test_nvfp4_quantiser_matches_oracle(name):
    *_, same = _setup(name)
    assert same


def test_nvfp4_quantiser_edge_matrices():
    """An all-zero matrix (t = 1, all codes and scales 0), a matrix with one non-zero
    element (every other block's scale rounds to zero), and negative zeros."""
    w = np.zeros((3, 4, 64), dtype=np.float32)
    w[1, 2, 17] = -0.75
    w[2] = -0.0
    w[2, 0, 0] = 3.0
    bits = synth.f32_to_bf16_bits(w)
    q = torch.empty(3, 4, 32, dtype=torch.uint8, device="cuda")
    b = torch.empty(3, 4, 4, dtype=torch.uint8, device="cuda")
    t = torch.empty(3, dtype=torch.float32, device="cuda")
    mf.moe_quantize_nvfp4(to_dev(bits), q, b, t)
    qg, bg, tg = unpack_nvfp4(q.cpu().numpy()), b.cpu().numpy(), t.cpu().numpy()
    for m in range(3):
        qo, bo, to = oracle.quantize_nvfp4(bits[m])
        assert np.array_equal(qg[m], qo) and np.array_equal(bg[m], bo), m
        assert np.float32(tg[m]).view(np.uint32) == np.float32(to).view(np.uint32), m
    assert tg[0] == 1.0 and not qg[0].any() and not bg[0].any()


@pytest.mark.parametrize("name", list(SHAPES))
def test_nvfp4_expert_branch(name):
    c, cfg, layer, ex4, same = _setup(name)
    assert same
    r = run_router(cfg, c, layer)
    p = run_permute(cfg, r["topk_idx"])
    moe = torch.empty(c.shape.T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    ws = mf.workspace(cfg, c.shape.T)
    mf.moe_ffn_forward(cfg, r["xn_moe"], r["topk_w"], p["offsets"], p["sorted_src"], p["inv_pos"],
                       layer, moe, ws)
    assert mf.moe_check_device_status(ws) == mf.MOE_OK
    cases.check_bar(bf16_np(moe), _oracle(c, ex4)["moe"], cases.FRAC_NVFP4, f"nvfp4 moe {name}")


@pytest.mark.parametrize("name", list(SHAPES))
def test_nvfp4_block(name):
    c, cfg, layer, ex4, _ = _setup(name)
    T = c.shape.T
    out = torch.empty(T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    moe = torch.empty(T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    ws = mf.workspace(cfg, T)
    mf.moe_block_forward(cfg, to_dev(c.x), mf.BlockWeights(cfg, layer), out, ws, moe_out=moe)
    assert mf.moe_check_device_status(ws) == mf.MOE_OK
    o = _oracle(c, ex4)
    cases.check_bar(bf16_np(out), o["out"], cases.FRAC_NVFP4, f"nvfp4 out {name}")
    cases.check_bar(bf16_np(moe), o["moe"], cases.FRAC_NVFP4, f"nvfp4 moe_out {name}")


def test_nvfp4_block_is_deterministic():
    c, cfg, layer, _, _ = _setup("nvfp4_T64")
    bw = mf.BlockWeights(cfg, layer)
    outs = []
    for _ in range(2):
        out = torch.empty(c.shape.T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
        ws = mf.workspace(cfg, c.shape.T)
        mf.moe_block_forward(cfg, to_dev(c.x), bw, out, ws)
        outs.append(out)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
