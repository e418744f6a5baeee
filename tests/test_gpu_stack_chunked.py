"""The chunked prefill driver (moe_stack_forward): a prompt longer than one chunk runs
chunk after chunk through every layer of a residual-chained stack.  The block is
row-independent, so the driver's result must equal, bit for bit, the same chunks chained
layer by layer through moe_block_forward by hand; a ragged last chunk is included.  The
first layer's rows of the first chunk are also checked against the oracle at the bar."""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_05_b200 as mf
import oracle
import synth
from tests import cases
from tests.gpu_util import bf16_np, config, device_layer, oracle_block, to_dev

pytestmark = pytest.mark.gpu

SHAPE = synth.Shape(T=2500, H=512, E=16, k=4, I=128, D=384)
LAYERS = 3
CHUNK = 1024  # three chunks: 1024, 1024 and 452 tokens


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    mf.lib()


def _layers(cfg):
    ls = []
    for l in range(LAYERS):
        c = cases.make_case(synth.Shape(T=8, H=SHAPE.H, E=SHAPE.E, k=SHAPE.k, I=SHAPE.I, D=SHAPE.D),
                            seed=4321 + l, gap=False)
        ls.append(mf.BlockWeights(cfg, device_layer(c)))
    return ls


def test_chunked_stack_equals_chunks_chained_by_hand():
    cfg = config(SHAPE)
    layers = _layers(cfg)
    x = to_dev(synth.x_rows(99, SHAPE.H, SHAPE.T))
    out = torch.empty_like(x)
    ws = mf.stack_workspace(cfg, CHUNK)
    mf.moe_stack_forward(cfg, x, layers, out, ws, chunk_tokens=CHUNK)
    assert mf.moe_check_device_status(ws) == mf.MOE_OK
    ref = torch.empty_like(x)
    for t0 in range(0, SHAPE.T, CHUNK):
        n = min(CHUNK, SHAPE.T - t0)
        cur = x[t0:t0 + n].contiguous()
        wsb = mf.workspace(cfg, n)
        for l in range(LAYERS):
            nxt = torch.empty_like(cur)
            mf.moe_block_forward(cfg, cur, layers[l], nxt, wsb)
            cur = nxt
        ref[t0:t0 + n] = cur
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_one_layer_chunked_matches_the_oracle():
    """One layer, two chunks (1024 + 476 tokens of a gap-filtered batch): every row at the
    accuracy bar against the oracle block."""
    shape = synth.Shape(T=1500, H=SHAPE.H, E=SHAPE.E, k=SHAPE.k, I=SHAPE.I, D=SHAPE.D)
    c = cases.make_case(shape, seed=777)
    cfg = config(shape)
    layer = mf.BlockWeights(cfg, device_layer(c))
    x = to_dev(c.x)
    out = torch.empty_like(x)
    ws = mf.stack_workspace(cfg, CHUNK)
    mf.moe_stack_forward(cfg, x, [layer], out, ws, chunk_tokens=CHUNK)
    assert mf.moe_check_device_status(ws) == mf.MOE_OK
    o = oracle_block(c)
    cases.check_bar(bf16_np(out), o["out"], cases.FRAC_BF16, "chunked one layer")
