"""The synthetic inputs follow the stated recipe: weights N(0, 0.02) and activations
N(0, 1) rounded to bf16, gains and scales U(0.5, 1.5), each tensor its own reproducible
stream (same seed and ids, same bits; another tensor id or layer, other bits)."""
import numpy as np

import synth

SHAPE = synth.Shape(T=64, H=512, E=16, k=4, I=128, D=384)


def _f(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def test_layer_distributions_follow_the_recipe():
    L = synth.make_layer(99, SHAPE)
    for name in ("w_router", "w_gate_up", "w_down", "w_dense_gate_up", "w_dense_down"):
        w = _f(L[name])
        n = w.size
        assert abs(w.mean()) < 5 * 0.02 / np.sqrt(n), name
        assert abs(w.std() / 0.02 - 1) < 5 / np.sqrt(2 * n) + 4e-3, name
    for name in ("router_scale", "per_expert_scale", "g_pre_moe", "g_pre_dense",
                 "g_post_moe", "g_post_dense", "g_post_ff"):
        g = _f(L[name])
        assert g.min() >= 0.5 - 2 ** -8 and g.max() <= 1.5 + 2 ** -7, name
        assert abs(g.mean() - 1.0) < 5 * (1 / np.sqrt(12)) / np.sqrt(g.size), name
    x = _f(synth.x_rows(99, SHAPE.H, SHAPE.T))
    assert abs(x.mean()) < 5 / np.sqrt(x.size) and abs(x.std() - 1) < 0.02


def test_streams_are_reproducible_and_independent():
    a = synth.make_layer(5, SHAPE, layer=0)
    b = synth.make_layer(5, SHAPE, layer=0)
    c = synth.make_layer(5, SHAPE, layer=1)
    for name in a:
        assert np.array_equal(a[name], b[name]), name
        assert not np.array_equal(a[name], c[name]), name
    # different tensors of one layer are different draws
    assert not np.array_equal(a["g_pre_moe"], a["g_pre_dense"])
    assert not np.array_equal(a["g_post_moe"], a["g_post_ff"])
