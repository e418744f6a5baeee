"""Parity at full size: the residual-chained stack of 30 distinct layers at T = 16384.

This is the largest workload the benchmark times, run here in the same launch
configuration (one moe_block_forward per layer, one workspace reused by every layer,
the current stream).  The oracle cannot run 16384 tokens through 30 layers, and the
layer inputs after the first come from the GPU itself, so each layer is checked on
sampled rows, with the oracle fed the GPU's own input rows for that layer:

  * top-k ids, bit for bit, on every sampled row whose oracle logits have adjacent gaps
    of at least MIN_GAP among the top k+1 (about 3% of the rows of these layers: the
    inputs cannot be redrawn once they come from the previous layer);
  * on every other sampled row, that the ids are a valid top-k of the oracle's logits
    up to LOGIT_TOL: distinct, in non-increasing logit order, none below the k-th
    largest logit (where two logits are within LOGIT_TOL either order is correct);
  * out and moe_out at the accuracy bar on the first rows of the sample that pass the
    gap rule.

The oracle reads back from the device only the expert matrices those rows use.
"""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_05_b200 as mf
import oracle
import synth
from tests import cases
from tests.gpu_util import bf16_np, config

pytestmark = pytest.mark.gpu

SHAPE = synth.Shape(T=synth.STACK_T, H=2816, E=128, k=8, I=704, D=2112)
LAYERS = synth.STACK_LAYERS
SEED = 1234          # the benchmark's seed on its first rank
CANDIDATES = 512     # rows sampled per layer for the top-k check
FULL_ROWS = 3        # of those, rows run through the whole oracle block per layer
LOGIT_TOL = 1e-5     # far above the router's logit error, far below MIN_GAP


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    mf.lib()


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class _DeviceExperts:
    """The oracle's expert accessor over device-resident bf16 weights: each matrix is
    copied to the host when the oracle asks for it, and only then."""

    def __init__(self, layer):
        self.w_gate_up, self.w_down = layer["w_gate_up"], layer["w_down"]

    def gate_up(self, e: int) -> np.ndarray:
        return bf16_np(self.w_gate_up[e])

    def down(self, e: int) -> np.ndarray:
        return bf16_np(self.w_down[e])


def _sample_rows(layer_idx: int) -> np.ndarray:
    """The first and last rows (ragged ends of every tile walk) plus a seeded sample."""
    rng = np.random.default_rng(7 + layer_idx)
    mid = rng.choice(np.arange(1, SHAPE.T - 1), size=CANDIDATES - 2, replace=False)
    return np.concatenate([[0, SHAPE.T - 1], np.sort(mid)]).astype(np.int64)


def test_stack_30_layers_T16384_sampled_rows():
    dev = torch.device("cuda")
    cfg = config(SHAPE)
    T, k = SHAPE.T, SHAPE.k
    layers = [synth.torch_layer(SHAPE, SEED, l, dev) for l in range(LAYERS)]
    x = synth.torch_x(SHAPE, SEED, 0, dev)
    ws = mf.workspace(cfg, T)
    ws_r = mf.workspace(cfg, T)
    bufs = [torch.empty_like(x), torch.empty_like(x)]
    moe = torch.empty_like(x)
    ti = torch.empty(T, k, dtype=torch.int32, device=dev)
    tw = torch.empty(T, k, dtype=torch.float32, device=dev)
    xa, xb = torch.empty_like(x), torch.empty_like(x)

    compared = excluded = checked_rows = 0
    for l, L in enumerate(layers):
        out = bufs[l % 2]
        mf.moe_block_forward(cfg, x, mf.BlockWeights(cfg, L), out, ws, moe_out=moe)
        mf.moe_router(cfg, x, L["router_scale"], L["w_router"], None, L["per_expert_scale"],
                      L["g_pre_moe"], L["g_pre_dense"], ti, tw, xa, xb, ws_r)
        for w in (ws, ws_r):
            st = mf.moe_check_device_status(w)
            assert st == mf.MOE_OK, (l, mf.status_string(st))

        rows = _sample_rows(l)
        ridx = torch.from_numpy(rows).to(dev)
        xr = _bits(x.index_select(0, ridx))
        p = {n: _bits(t) for n, t in L.items() if n not in ("w_gate_up", "w_down")}
        r = oracle.router(oracle.bf16(xr), oracle.bf16(p["router_scale"]),
                          oracle.bf16(p["w_router"]), None, oracle.bf16(p["per_expert_scale"]),
                          k, SHAPE.eps)
        ok = oracle.topk_gaps(r["logits"], k) >= cases.MIN_GAP
        got_idx = ti.index_select(0, ridx).cpu().numpy()
        assert np.array_equal(got_idx[ok], r["topk_idx"][ok]), f"layer {l}: top-k ids"
        compared += int(ok.sum())
        excluded += int((~ok).sum())
        lg = np.take_along_axis(r["logits"], got_idx.astype(np.int64), axis=1)
        kth = -np.sort(-r["logits"], axis=1)[:, k - 1]
        assert all(len(set(row)) == k for row in got_idx.tolist()), f"layer {l}: repeated id"
        assert np.all(lg[:, :-1] >= lg[:, 1:] - LOGIT_TOL), f"layer {l}: top-k order"
        assert np.all(lg.min(axis=1) >= kth - LOGIT_TOL), f"layer {l}: not a top-k"

        sel = np.nonzero(ok)[0][:FULL_ROWS]
        assert sel.size > 0, f"layer {l}: no sampled row passes the gap rule"
        o = oracle.block_forward(xr[sel], p, _DeviceExperts(L), k, SHAPE.eps)
        sidx = torch.from_numpy(rows[sel]).to(dev)
        cases.check_bar(bf16_np(out.index_select(0, sidx)), o["out"], cases.FRAC_BF16,
                        f"layer {l} out")
        cases.check_bar(bf16_np(moe.index_select(0, sidx)), o["moe"], cases.FRAC_BF16,
                        f"layer {l} moe_out")
        checked_rows += sel.size
        x = out

    # the gap rule keeps a useful share of the sampled rows
    assert compared >= LAYERS * CANDIDATES // 100, (compared, excluded)
    assert checked_rows >= LAYERS
