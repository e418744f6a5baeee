"""Hybrid MoE feed-forward block (Gemma-4-26B-A4B shape) on B200: Python binding.

A thin ctypes layer over the C interface in include/moe_ffn.h (libmoeffn.so, built by
`python -m mixture_experts_ffn_05_b200.build`).  Every function here only checks and
marshals its torch tensors into pointers and calls the library entry point of the
same name; all computation runs in the library's CUDA kernels.  torch supplies device
memory and the current stream.  Without the built library every call raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoeffn.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_TIMEOUT = 5

MOE_W_BF16 = 0
MOE_W_INT8 = 1
MOE_W_FP8 = 2
MOE_W_NVFP4 = 3

# Entry points of include/moe_ffn.h (the CPU tests check the header declares exactly these).
ENTRY_POINTS = ("moe_workspace_size", "moe_router", "moe_permute", "moe_permute_noalloc",
                "moe_ffn_forward", "dense_mlp_forward", "moe_block_forward",
                "moe_quantize_int8", "moe_quantize_fp8", "moe_quantize_nvfp4",
                "moe_check_device_status",
                "moe_wait_selftest", "moe_stack_chunk_tokens", "moe_stack_workspace_size",
                "moe_stack_forward",
                "moe_block_launch_count", "moe_status_string", "moe_abi_version")
PERMUTE_NOALLOC_MAX_PAIRS = 1 << 20


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} (status {status})")


class CConfig(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("num_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("expert_inter", ctypes.c_int32),
                ("dense_inter", ctypes.c_int32), ("eps", ctypes.c_float),
                ("expert_wdtype", ctypes.c_int32)]


class CExpertWeights(ctypes.Structure):
    _fields_ = [("w_gate_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("s_gate_up", ctypes.c_void_p), ("s_down", ctypes.c_void_p),
                ("b_gate_up", ctypes.c_void_p), ("b_down", ctypes.c_void_p)]


class CBlockWeights(ctypes.Structure):
    _fields_ = [("router_scale", ctypes.c_void_p), ("w_router", ctypes.c_void_p),
                ("logit_bias", ctypes.c_void_p), ("per_expert_scale", ctypes.c_void_p),
                ("g_pre_moe", ctypes.c_void_p), ("g_pre_dense", ctypes.c_void_p),
                ("g_post_moe", ctypes.c_void_p), ("g_post_dense", ctypes.c_void_p),
                ("g_post_ff", ctypes.c_void_p), ("experts", CExpertWeights),
                ("w_dense_gate_up", ctypes.c_void_p), ("w_dense_down", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_SIG = {
    "moe_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(CConfig), _I32]),
    "moe_router": (_I32, [ctypes.POINTER(CConfig), _I32] + [_P] * 12 + [ctypes.c_size_t, _P]),
    "moe_permute": (_I32, [ctypes.POINTER(CConfig), _I32] + [_P] * 5 + [ctypes.c_size_t, _P]),
    "moe_permute_noalloc": (_I32, [ctypes.POINTER(CConfig), _I32] + [_P] * 4 + [_P]),
    "moe_ffn_forward": (_I32, [ctypes.POINTER(CConfig), _I32, _P, _P, _P, _P, _P,
                               ctypes.POINTER(CExpertWeights), _P, _P, ctypes.c_size_t, _P]),
    "dense_mlp_forward": (_I32, [ctypes.POINTER(CConfig), _I32] + [_P] * 5 + [ctypes.c_size_t, _P]),
    "moe_block_forward": (_I32, [ctypes.POINTER(CConfig), _I32, _P, ctypes.POINTER(CBlockWeights),
                                 _P, _P, _P, ctypes.c_size_t, _P, ctypes.POINTER(_P)]),
    "moe_quantize_int8": (_I32, [_P, ctypes.c_int64, _I32, _P, _P, _P]),
    "moe_quantize_fp8": (_I32, [_P, ctypes.c_int64, _I32, _P, _P, _P]),
    "moe_quantize_nvfp4": (_I32, [_P, ctypes.c_int64, ctypes.c_int64, _I32, _P, _P, _P, _P]),
    "moe_check_device_status": (_I32, [_P, ctypes.c_size_t, _P]),
    "moe_wait_selftest": (_I32, [_P, ctypes.c_size_t, ctypes.c_uint64, _P]),
    "moe_block_launch_count": (_I32, [ctypes.POINTER(CConfig), _I32]),
    "moe_stack_chunk_tokens": (_I32, [_I32]),
    "moe_stack_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(CConfig), _I32]),
    "moe_stack_forward": (_I32, [ctypes.POINTER(CConfig), _I32, _P, ctypes.POINTER(CBlockWeights),
                                 _I32, _P, _I32, _P, ctypes.c_size_t, _P]),
    "moe_status_string": (ctypes.c_char_p, [_I32]),
    "moe_abi_version": (_I32, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m mixture_experts_ffn_05_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIG.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != MOE_OK:
        raise MoeError(fn, status)


@dataclasses.dataclass(frozen=True)
class Config:
    hidden: int
    num_experts: int
    top_k: int
    expert_inter: int
    dense_inter: int
    eps: float = 1e-6
    int8: bool = False
    fp8: bool = False   # E4M3 expert weights, per-token E4M3 activations
    nvfp4: bool = False  # NVFP4 expert weights (packed E2M1 codes, E4M3 block scales)

    def c(self) -> CConfig:
        wd = (MOE_W_NVFP4 if self.nvfp4 else MOE_W_FP8 if self.fp8 else
              (MOE_W_INT8 if self.int8 else MOE_W_BF16))
        return CConfig(self.hidden, self.num_experts, self.top_k, self.expert_inter,
                       self.dense_inter, self.eps, wd)


def _ptr(t, dtype=None, name="tensor", nullable=False):
    if t is None:
        if nullable:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    return t.data_ptr()


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def workspace_size(cfg: Config, T: int) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(cfg.c()), int(T)))


def workspace(cfg: Config, T: int, device=None) -> torch.Tensor:
    """A zeroed device buffer of moe_workspace_size bytes, ready for its first use
    (torch allocations are 512-byte aligned)."""
    n = workspace_size(cfg, T)
    if n == 0:
        raise MoeError("moe_workspace_size", MOE_ERR_INVALID_ARG)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


BF16 = torch.bfloat16


def moe_router(cfg, x, router_scale, w_router, logit_bias, per_expert_scale, g_pre_moe,
               g_pre_dense, topk_idx, topk_w, xn_moe, xn_dense, ws, stream=None):
    T = x.shape[0]
    st = lib().moe_router(ctypes.byref(cfg.c()), T, _ptr(x, BF16, "x"),
                          _ptr(router_scale, BF16, "router_scale"), _ptr(w_router, BF16, "w_router"),
                          _ptr(logit_bias, torch.float32, "logit_bias", True),
                          _ptr(per_expert_scale, BF16, "per_expert_scale"),
                          _ptr(g_pre_moe, BF16, "g_pre_moe"), _ptr(g_pre_dense, BF16, "g_pre_dense"),
                          _ptr(topk_idx, torch.int32, "topk_idx"), _ptr(topk_w, torch.float32, "topk_w"),
                          _ptr(xn_moe, BF16, "xn_moe"), _ptr(xn_dense, BF16, "xn_dense"),
                          _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check("moe_router", st)


def moe_permute(cfg, topk_idx, expert_offsets, sorted_src, inv_pos, ws, stream=None):
    T = topk_idx.shape[0]
    st = lib().moe_permute(ctypes.byref(cfg.c()), T, _ptr(topk_idx, torch.int32, "topk_idx"),
                           _ptr(expert_offsets, torch.int32, "expert_offsets"),
                           _ptr(sorted_src, torch.int32, "sorted_src"),
                           _ptr(inv_pos, torch.int32, "inv_pos"), _ptr(ws, torch.uint8, "ws"),
                           ws.numel(), _stream(stream))
    _check("moe_permute", st)


def moe_permute_noalloc(cfg, topk_idx, expert_offsets, sorted_src, inv_pos, stream=None):
    """moe_permute without a workspace, for callers that cannot provide scratch memory:
    the library's own fixed device array (512 KiB, up to 2^20 pairs) is used instead.
    Calls that overlap on the GPU share that array and must be serialised."""
    T = topk_idx.shape[0]
    st = lib().moe_permute_noalloc(ctypes.byref(cfg.c()), T, _ptr(topk_idx, torch.int32, "topk_idx"),
                                   _ptr(expert_offsets, torch.int32, "expert_offsets"),
                                   _ptr(sorted_src, torch.int32, "sorted_src"),
                                   _ptr(inv_pos, torch.int32, "inv_pos"), _stream(stream))
    _check("moe_permute_noalloc", st)


def _experts(cfg, e: dict) -> CExpertWeights:
    wt = torch.uint8 if (cfg.fp8 or cfg.nvfp4) else (torch.int8 if cfg.int8 else BF16)
    return CExpertWeights(_ptr(e["w_gate_up"], wt, "w_gate_up"), _ptr(e["w_down"], wt, "w_down"),
                          _ptr(e.get("s_gate_up"), torch.float32, "s_gate_up", True),
                          _ptr(e.get("s_down"), torch.float32, "s_down", True),
                          _ptr(e.get("b_gate_up"), torch.uint8, "b_gate_up", True),
                          _ptr(e.get("b_down"), torch.uint8, "b_down", True))


def moe_ffn_forward(cfg, xn_moe, topk_w, expert_offsets, sorted_src, inv_pos, experts: dict,
                    moe_out, ws, stream=None):
    T = xn_moe.shape[0]
    ew = _experts(cfg, experts)
    st = lib().moe_ffn_forward(ctypes.byref(cfg.c()), T, _ptr(xn_moe, BF16, "xn_moe"),
                               _ptr(topk_w, torch.float32, "topk_w"),
                               _ptr(expert_offsets, torch.int32, "expert_offsets"),
                               _ptr(sorted_src, torch.int32, "sorted_src"),
                               _ptr(inv_pos, torch.int32, "inv_pos"), ctypes.byref(ew),
                               _ptr(moe_out, BF16, "moe_out"), _ptr(ws, torch.uint8, "ws"),
                               ws.numel(), _stream(stream))
    _check("moe_ffn_forward", st)


def dense_mlp_forward(cfg, xn_dense, w_gate_up, w_down, dense_out, ws, stream=None):
    T = xn_dense.shape[0]
    st = lib().dense_mlp_forward(ctypes.byref(cfg.c()), T, _ptr(xn_dense, BF16, "xn_dense"),
                                 _ptr(w_gate_up, BF16, "w_gate_up"), _ptr(w_down, BF16, "w_down"),
                                 _ptr(dense_out, BF16, "dense_out"), _ptr(ws, torch.uint8, "ws"),
                                 ws.numel(), _stream(stream))
    _check("dense_mlp_forward", st)


class BlockWeights:
    """Holds one layer's device tensors and their C struct (keeps the tensors alive)."""

    NAMES = ("router_scale", "w_router", "logit_bias", "per_expert_scale", "g_pre_moe",
             "g_pre_dense", "g_post_moe", "g_post_dense", "g_post_ff", "w_dense_gate_up",
             "w_dense_down")
    NULLABLE = ("logit_bias", "g_post_moe", "g_post_dense")

    def __init__(self, cfg: Config, tensors: dict):
        self.cfg = cfg
        self.tensors = dict(tensors)
        vals = {}
        for n in self.NAMES:
            dt = torch.float32 if n == "logit_bias" else BF16
            vals[n] = _ptr(self.tensors.get(n), dt, n, n in self.NULLABLE)
        self.c = CBlockWeights(
            vals["router_scale"], vals["w_router"], vals["logit_bias"], vals["per_expert_scale"],
            vals["g_pre_moe"], vals["g_pre_dense"], vals["g_post_moe"], vals["g_post_dense"],
            vals["g_post_ff"], _experts(cfg, self.tensors), vals["w_dense_gate_up"],
            vals["w_dense_down"])


MOE_BLOCK_EVENTS = 7


def moe_block_forward(cfg, x, weights: BlockWeights, out, ws, moe_out=None, stream=None,
                      stage_events=None):
    """stage_events: None or MOE_BLOCK_EVENTS torch.cuda.Event(enable_timing=True) objects,
    recorded at the block's stage boundaries (see include/moe_ffn.h)."""
    T = x.shape[0]
    ev = None
    if stage_events is not None:
        if len(stage_events) != MOE_BLOCK_EVENTS:
            raise ValueError(f"stage_events needs {MOE_BLOCK_EVENTS} events")
        for e in stage_events:
            if e.cuda_event == 0:  # torch creates the CUDA event on its first record
                e.record(torch.cuda.current_stream() if stream is None else stream)
        ev = (_P * MOE_BLOCK_EVENTS)(*[e.cuda_event for e in stage_events])
    st = lib().moe_block_forward(ctypes.byref(cfg.c()), T, _ptr(x, BF16, "x"),
                                 ctypes.byref(weights.c), _ptr(out, BF16, "out"),
                                 _ptr(moe_out, BF16, "moe_out", True), _ptr(ws, torch.uint8, "ws"),
                                 ws.numel(), _stream(stream), ev)
    _check("moe_block_forward", st)


def moe_stack_chunk_tokens(chunk_tokens: int) -> int:
    """The chunk length moe_stack_forward uses for a requested one (host only)."""
    return int(lib().moe_stack_chunk_tokens(int(chunk_tokens)))


def stack_workspace(cfg: Config, chunk_tokens: int, device=None) -> torch.Tensor:
    """A zeroed workspace for moe_stack_forward with chunks of chunk_tokens tokens."""
    n = int(lib().moe_stack_workspace_size(ctypes.byref(cfg.c()), int(chunk_tokens)))
    if n == 0:
        raise MoeError("moe_stack_workspace_size", MOE_ERR_INVALID_ARG)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def moe_stack_forward(cfg, x, layers, out, ws, chunk_tokens: int = 16384, stream=None):
    """x [T][H] through every BlockWeights of `layers` (residual chain), chunk by chunk."""
    T = x.shape[0]
    arr = (CBlockWeights * len(layers))(*[l.c for l in layers])
    st = lib().moe_stack_forward(ctypes.byref(cfg.c()), T, _ptr(x, BF16, "x"), arr, len(layers),
                                 _ptr(out, BF16, "out"), int(chunk_tokens),
                                 _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check("moe_stack_forward", st)


def moe_quantize_int8(w, q, scales, stream=None):
    cols = w.shape[-1]
    rows = w.numel() // cols
    st = lib().moe_quantize_int8(_ptr(w, BF16, "w"), rows, cols, _ptr(q, torch.int8, "q"),
                                 _ptr(scales, torch.float32, "scales"), _stream(stream))
    _check("moe_quantize_int8", st)


def moe_quantize_fp8(w, q, scales, stream=None):
    """Per-output-row E4M3 codes (uint8) and fp32 scales of bf16 weights."""
    cols = w.shape[-1]
    rows = w.numel() // cols
    st = lib().moe_quantize_fp8(_ptr(w, BF16, "w"), rows, cols, _ptr(q, torch.uint8, "q"),
                                _ptr(scales, torch.float32, "scales"), _stream(stream))
    _check("moe_quantize_fp8", st)


def moe_quantize_nvfp4(w, q, block_scales, tensor_scales, stream=None):
    """NVFP4 codes of bf16 weight matrices w [matrices][rows][cols] (or [rows][cols]):
    q [.., rows, cols // 2] uint8 packed codes, block_scales [.., rows, cols // 16] uint8
    E4M3 codes, tensor_scales [matrices] fp32."""
    cols = w.shape[-1]
    rows = w.shape[-2]
    matrices = w.numel() // (rows * cols)
    st = lib().moe_quantize_nvfp4(_ptr(w, BF16, "w"), matrices, rows, cols,
                                  _ptr(q, torch.uint8, "q"),
                                  _ptr(block_scales, torch.uint8, "block_scales"),
                                  _ptr(tensor_scales, torch.float32, "tensor_scales"),
                                  _stream(stream))
    _check("moe_quantize_nvfp4", st)


def moe_wait_selftest(ws, timeout_ns: int, stream=None) -> None:
    """Run one bounded device wait that is bound to run out (the failure path of every
    kernel's waits); afterwards moe_check_device_status reports MOE_ERR_DEVICE_TIMEOUT."""
    _check("moe_wait_selftest", lib().moe_wait_selftest(_ptr(ws, torch.uint8, "ws"), ws.numel(),
                                                         int(timeout_ns), _stream(stream)))


def moe_block_launch_count(cfg, T: int) -> int:
    """Kernels one moe_block_forward launches for this config and T (-1: invalid)."""
    return int(lib().moe_block_launch_count(ctypes.byref(cfg.c()), int(T)))


def moe_check_device_status(ws, stream=None) -> int:
    """Waits for the stream; returns the status recorded by the last call's kernels."""
    return int(lib().moe_check_device_status(_ptr(ws, torch.uint8, "ws"), ws.numel(),
                                             _stream(stream)))
