"""Helpers of the GPU tests: move seeded inputs to the device, call the library through
its binding, and fetch results back as numpy."""
from __future__ import annotations

import numpy as np
import torch

import mixture_experts_ffn_05_b200 as mf
import oracle
import synth
from tests import cases


def to_dev(a: np.ndarray, dtype=torch.bfloat16) -> torch.Tensor:
    if dtype is torch.bfloat16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).cuda()


def bf16_np(t: torch.Tensor) -> np.ndarray:
    """A bf16 device tensor as float64 numpy values."""
    return oracle.bf16(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def config(shape: synth.Shape, int8: bool = False, fp8: bool = False) -> mf.Config:
    return mf.Config(shape.H, shape.E, shape.k, shape.I, shape.D, shape.eps, int8, fp8)


_DEV_CACHE = cases._Lru(3)


def device_layer(case: cases.Case) -> dict:
    key = id(case.p)
    if key not in _DEV_CACHE or _DEV_CACHE[key][0] is not case.p:
        _DEV_CACHE.put(key, (case.p, {n: to_dev(v) for n, v in case.p.items()}))
    d = dict(_DEV_CACHE[key][1])
    if case.bias is not None:
        d["logit_bias"] = to_dev(case.bias, torch.float32)
    return d


_ORACLE_CACHE = cases._Lru(12)


def oracle_block(case: cases.Case) -> dict:
    key = (id(case.p), hash(case.x.tobytes()), None if case.bias is None else case.bias.tobytes())
    if key not in _ORACLE_CACHE or _ORACLE_CACHE[key][0] is not case.p:
        _ORACLE_CACHE.put(key, (case.p, oracle.block_forward(
            case.x, case.p, cases.bf16_experts(case.p), case.shape.k, case.shape.eps, case.bias)))
    return _ORACLE_CACHE[key][1]


def run_router(cfg, case, layer, x=None):
    T = case.shape.T
    x = to_dev(case.x) if x is None else x
    r = {
        "topk_idx": torch.empty(T, cfg.top_k, dtype=torch.int32, device="cuda"),
        "topk_w": torch.empty(T, cfg.top_k, dtype=torch.float32, device="cuda"),
        "xn_moe": torch.empty(T, cfg.hidden, dtype=torch.bfloat16, device="cuda"),
        "xn_dense": torch.empty(T, cfg.hidden, dtype=torch.bfloat16, device="cuda"),
    }
    ws = mf.workspace(cfg, T)
    mf.moe_router(cfg, x, layer["router_scale"], layer["w_router"], layer.get("logit_bias"),
                  layer["per_expert_scale"], layer["g_pre_moe"], layer["g_pre_dense"],
                  r["topk_idx"], r["topk_w"], r["xn_moe"], r["xn_dense"], ws)
    return r


def run_permute(cfg, topk_idx: torch.Tensor):
    T, k = topk_idx.shape
    n = T * k
    p = {
        "offsets": torch.empty(cfg.num_experts + 1, dtype=torch.int32, device="cuda"),
        "sorted_src": torch.empty(max(n, 1), dtype=torch.int32, device="cuda"),
        "inv_pos": torch.empty(max(n, 1), dtype=torch.int32, device="cuda"),
    }
    ws = mf.workspace(cfg, T)
    mf.moe_permute(cfg, topk_idx, p["offsets"], p["sorted_src"], p["inv_pos"], ws)
    return p


def run_block(cfg, case, layer, want_moe=True, ws=None, x=None):
    T = case.shape.T
    x = to_dev(case.x) if x is None else x
    out = torch.empty(T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    moe = torch.empty(T, cfg.hidden, dtype=torch.bfloat16, device="cuda") if want_moe else None
    ws = mf.workspace(cfg, T) if ws is None else ws
    bw = mf.BlockWeights(cfg, layer)
    mf.moe_block_forward(cfg, x, bw, out, ws, moe_out=moe)
    st = mf.moe_check_device_status(ws)
    assert st == mf.MOE_OK, mf.status_string(st)
    return out, moe


_INT8_CACHE = cases._Lru(2)


def int8_experts(case: cases.Case):
    """Quantise the case's expert weights on the GPU (moe_quantize_int8) and with the
    oracle; return (device tensors for the library, oracle.Experts built from the
    oracle's own codes and scales, whether the two quantisations are identical)."""
    key = id(case.p)
    if key in _INT8_CACHE and _INT8_CACHE[key][0] is case.p:
        return _INT8_CACHE[key][1]
    dev = {}
    host = {}
    same = True
    for name, sname in (("w_gate_up", "s_gate_up"), ("w_down", "s_down")):
        w = case.p[name]
        rows, cols = int(np.prod(w.shape[:-1])), w.shape[-1]
        q = torch.empty(w.shape, dtype=torch.int8, device="cuda")
        s = torch.empty(w.shape[:-1], dtype=torch.float32, device="cuda")
        mf.moe_quantize_int8(to_dev(w).view(rows, cols), q.view(rows, cols), s.view(rows))
        qo, so = oracle.quantize_int8_per_channel(w)
        same = same and np.array_equal(q.cpu().numpy(), qo) and \
            np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
        dev[name], dev[sname] = q, s
        host[name], host[sname] = qo, so
    ex = oracle.Experts(q_gate_up=host["w_gate_up"], s_gate_up=host["s_gate_up"],
                        q_down=host["w_down"], s_down=host["s_down"])
    res = (dev, ex, same)
    _INT8_CACHE.put(key, (case.p, res))
    return res


_FP8_CACHE = cases._Lru(2)


def fp8_experts(case: cases.Case):
    """Quantise the case's expert weights to E4M3 on the GPU (moe_quantize_fp8) and with
    the oracle; return (device tensors, oracle.Experts in fp8 mode built from the oracle's
    own codes and scales, whether the two quantisations are identical)."""
    key = id(case.p)
    if key in _FP8_CACHE and _FP8_CACHE[key][0] is case.p:
        return _FP8_CACHE[key][1]
    dev, host, same = {}, {}, True
    for name, sname in (("w_gate_up", "s_gate_up"), ("w_down", "s_down")):
        w = case.p[name]
        rows, cols = int(np.prod(w.shape[:-1])), w.shape[-1]
        q = torch.empty(w.shape, dtype=torch.uint8, device="cuda")
        s = torch.empty(w.shape[:-1], dtype=torch.float32, device="cuda")
        mf.moe_quantize_fp8(to_dev(w).view(rows, cols), q.view(rows, cols), s.view(rows))
        qo, so = oracle.quantize_fp8_per_channel(w)
        same = same and np.array_equal(q.cpu().numpy(), qo) and \
            np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
        dev[name], dev[sname] = q, s
        host[name], host[sname] = qo, so
    ex = oracle.Experts(q_gate_up=host["w_gate_up"], s_gate_up=host["s_gate_up"],
                        q_down=host["w_down"], s_down=host["s_down"], fp8=True)
    res = (dev, ex, same)
    _FP8_CACHE.put(key, (case.p, res))
    return res


def unpack_nvfp4(q: np.ndarray) -> np.ndarray:
    """E2M1 codes (one per uint8, natural element order) from the library's packed layout:
    each little-endian 32-bit word holds 8 consecutive elements, nibbles 0-3 elements 0, 2,
    4, 6 and nibbles 4-7 elements 1, 3, 5, 7."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    words = q.reshape(*q.shape[:-1], -1, 4).view(np.uint32)[..., 0]   # [..., cols / 8]
    nib = np.stack([(words >> np.uint32(4 * n)) & np.uint32(0xF) for n in range(8)], axis=-1)
    order = [0, 4, 1, 5, 2, 6, 3, 7]  # element e sits in nibble order[e]
    out = nib[..., order].astype(np.uint8)
    return out.reshape(*q.shape[:-1], q.shape[-1] * 2)


_NVFP4_CACHE = cases._Lru(2)


def nvfp4_experts(case: cases.Case):
    """Quantise the case's expert weights to NVFP4 on the GPU (moe_quantize_nvfp4, one
    matrix per expert) and with the oracle; return (device tensors, oracle.Experts built
    from the oracle's own codes and scales, whether the two quantisations are identical)."""
    key = id(case.p)
    if key in _NVFP4_CACHE and _NVFP4_CACHE[key][0] is case.p:
        return _NVFP4_CACHE[key][1]
    dev, host, same = {}, {}, True
    for name, bname, sname, part in (("w_gate_up", "b_gate_up", "s_gate_up", "gate_up"),
                                     ("w_down", "b_down", "s_down", "down")):
        w = case.p[name]
        E, rows, cols = w.shape
        q = torch.empty(E, rows, cols // 2, dtype=torch.uint8, device="cuda")
        b = torch.empty(E, rows, cols // 16, dtype=torch.uint8, device="cuda")
        t = torch.empty(E, dtype=torch.float32, device="cuda")
        mf.moe_quantize_nvfp4(to_dev(w), q, b, t)
        qg, bg, tg = unpack_nvfp4(q.cpu().numpy()), b.cpu().numpy(), t.cpu().numpy()
        ref = [oracle.quantize_nvfp4(w[e]) for e in range(E)]
        for e in range(E):
            qo, bo, to = ref[e]
            same = same and np.array_equal(qg[e], qo) and np.array_equal(bg[e], bo) and \
                np.float32(tg[e]).view(np.uint32) == np.float32(to).view(np.uint32)
        dev[name], dev[bname], dev[sname] = q, b, t
        host[part] = ref
    ex = oracle.Experts(nvfp4=host)
    res = (dev, ex, same)
    _NVFP4_CACHE.put(key, (case.p, res))
    return res
