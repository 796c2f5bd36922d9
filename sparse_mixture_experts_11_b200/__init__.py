"""Python binding of ``libmoe.so``, the sparse MoE layer forward pass on B200 (sm_100a).

The functions mirror the C ABI in ``include/moe.h`` name for name (without the ``moe_``
prefix). They only marshal arguments: they check torch tensors' dtype, shape, device and
contiguity, then pass raw device pointers and the current CUDA stream to the library. Every
step of the layer runs in the library's CUDA kernels. There is no fallback: importing this
package fails if the library is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python sparse_mixture_experts_11_b200/build.py` "
        "(the MoE layer has no implementation other than this CUDA library)")
_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE, ERR_TIMEOUT, ERR_BOUNDS = 0, -1, -2, -3, -4, -5, -6
ACT_SWIGLU, ACT_GELU = 0, 1
_ACTS = {"swiglu": ACT_SWIGLU, "gelu": ACT_GELU}


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class Dims(ctypes.Structure):
    """``moe_dims``: T, d_model, n_experts, top_k, d_ff, act, capacity."""
    _fields_ = [("T", ctypes.c_int32), ("d_model", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("act", ctypes.c_int32),
                ("capacity", ctypes.c_int32)]

    def __repr__(self):
        return ("Dims(T={0.T}, d_model={0.d_model}, n_experts={0.n_experts}, top_k={0.top_k}, "
                "d_ff={0.d_ff}, act={0.act}, capacity={0.capacity})".format(self))


class ForwardBuffers(ctypes.Structure):
    """``moe_forward_buffers``: device pointers into a moe_forward workspace."""
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "logits", "topk_idx", "topk_w", "slot", "expert_count", "expert_offset", "row_of_pair",
        "pair_of_row", "x_perm", "h", "y_perm", "stage_ws")] + [("stage_ws_bytes", ctypes.c_size_t)]


WFMT_BF16, WFMT_MXFP8, WFMT_MXFP4, WFMT_MXFP8_BS, WFMT_MXFP4_BS = 0, 1, 2, 3, 4
# "_bs": the same weights on the block-scaled MMA, with MXFP8-quantised token rows and h
_WFMT = {"mxfp8": WFMT_MXFP8, "mxfp4": WFMT_MXFP4, "mxfp8_bs": WFMT_MXFP8_BS,
         "mxfp4_bs": WFMT_MXFP4_BS}


class MxWeights(ctypes.Structure):
    """``moe_mx_weights``: expert weights in an MX format (device pointers)."""
    _fields_ = [("fmt", ctypes.c_int32), ("gate_up", ctypes.c_void_p),
                ("gate_up_scales", ctypes.c_void_p), ("down", ctypes.c_void_p),
                ("down_scales", ctypes.c_void_p)]


_P = ctypes.c_void_p
_DIMS = ctypes.POINTER(Dims)
_MXW = ctypes.POINTER(MxWeights)
_SIGS = {
    "moe_capacity": (ctypes.c_int32, [ctypes.c_double, ctypes.c_int32, ctypes.c_int32]),
    "moe_max_rows": (ctypes.c_int64, [_DIMS]),
    "moe_workspace_bytes": (ctypes.c_int, [_DIMS, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_workspace_init": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
    "moe_route": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_route_from_logits": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_route_with_stats": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_float,
                                            _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_redirect_overflow": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_permute": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_grouped_ffn": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_unpermute_combine": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, ctypes.c_int32, _P,
                                             ctypes.c_size_t, _P]),
    "moe_forward_workspace_bytes": (ctypes.c_int, [_DIMS, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_mx_act_workspace_bytes": (ctypes.c_int, [_DIMS, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_forward_layout": (ctypes.c_int, [_DIMS, _P, ctypes.c_size_t, ctypes.POINTER(ForwardBuffers)]),
    "moe_forward": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_route_noalloc": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_grouped_ffn_mx": (ctypes.c_int, [_DIMS, _P, _P, _MXW, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_forward_mx": (ctypes.c_int, [_DIMS, _P, _P, _P, _MXW, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_router_stats": (ctypes.c_int, [_DIMS, _P, _P, _P, ctypes.c_float, _P, _P, _P, _P, _P,
                                        ctypes.c_size_t, _P]),
    "moe_backward_workspace_bytes": (ctypes.c_int, [_DIMS, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_backward": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P, _P, _P,
                                    _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_read_device_error": (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_int)]),
    "moe_debug_set_wait_timeout_ns": (ctypes.c_uint64, [ctypes.c_uint64]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


# ----------------------------------------------------------------------------- marshalling
def _check(status: int, where: str) -> None:
    if status != OK:
        raise MoeError(status, where)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, shape=None, allow_none=False):
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _nbytes(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.numel() * t.element_size()


# ----------------------------------------------------------------------------- host helpers
def debug_set_wait_timeout_ns(ns: int) -> int:
    """Limit of the kernels' bounded waits for later calls (0 = default 2 s); returns the old one."""
    return int(_lib.moe_debug_set_wait_timeout_ns(int(ns)))


def status_string(status: int) -> str:
    return _lib.moe_status_string(int(status)).decode()


def capacity(capacity_factor: Optional[float], T: int, n_experts: int) -> int:
    """ceil(capacity_factor * T / n_experts); None / <=0 / inf means no limit (T)."""
    cf = 0.0 if capacity_factor is None else float(capacity_factor)
    return int(_lib.moe_capacity(cf, int(T), int(n_experts)))


def make_dims(T: int, d_model: int, n_experts: int, top_k: int, d_ff: int, act="swiglu",
              capacity: Optional[int] = None) -> Dims:
    a = _ACTS[act] if isinstance(act, str) else int(act)
    return Dims(int(T), int(d_model), int(n_experts), int(top_k), int(d_ff), a,
                int(T if capacity is None else capacity))


def max_rows(dims: Dims) -> int:
    r = int(_lib.moe_max_rows(ctypes.byref(dims)))
    if r < 0:
        raise MoeError(ERR_INVALID, "moe_max_rows")
    return r


def workspace_bytes(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.moe_workspace_bytes(ctypes.byref(dims), ctypes.byref(n)), "moe_workspace_bytes")
    return int(n.value)


def forward_workspace_bytes(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.moe_forward_workspace_bytes(ctypes.byref(dims), ctypes.byref(n)),
           "moe_forward_workspace_bytes")
    return int(n.value)


def mx_act_workspace_bytes(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.moe_mx_act_workspace_bytes(ctypes.byref(dims), ctypes.byref(n)),
           "moe_mx_act_workspace_bytes")
    return int(n.value)


def new_workspace(dims: Dims, device=None, forward: bool = False,
                  block_scaled: bool = False) -> torch.Tensor:
    """A zeroed uint8 workspace tensor for the per-stage calls (or for moe_forward); with
    block_scaled, room for the block-scaled MX formats' quantised activations after it."""
    n = forward_workspace_bytes(dims) if forward else workspace_bytes(dims)
    if block_scaled:
        n = (n + 255) // 256 * 256 + mx_act_workspace_bytes(dims)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def forward_layout(dims: Dims, ws: torch.Tensor) -> ForwardBuffers:
    b = ForwardBuffers()
    _check(_lib.moe_forward_layout(ctypes.byref(dims), _ptr(ws, "ws", torch.uint8), _nbytes(ws),
                                   ctypes.byref(b)), "moe_forward_layout")
    return b


def read_device_error(ws: torch.Tensor, stream=None, offset_bytes: int = 0) -> int:
    err = ctypes.c_int(0)
    p = ctypes.c_void_p(ws.data_ptr() + offset_bytes)
    _check(_lib.moe_read_device_error(p, _stream(stream), ctypes.byref(err)), "moe_read_device_error")
    return int(err.value)


# ----------------------------------------------------------------------------- stages
def route(dims: Dims, x, w_router, logit_bias, logits, topk_idx, topk_w, slot, expert_count,
          ws, stream=None) -> None:
    T, d, N, k = dims.T, dims.d_model, dims.n_experts, dims.top_k
    _check(_lib.moe_route(
        ctypes.byref(dims), _ptr(x, "x", torch.bfloat16, (T, d)),
        _ptr(w_router, "w_router", torch.float32, (N, d)),
        _ptr(logit_bias, "logit_bias", torch.float32, (N,), allow_none=True),
        _ptr(logits, "logits", torch.float32, (T, N)), _ptr(topk_idx, "topk_idx", torch.int32, (T, k)),
        _ptr(topk_w, "topk_w", torch.float32, (T, k)), _ptr(slot, "slot", torch.int32, (T, k)),
        _ptr(expert_count, "expert_count", torch.int32, (N,)), _ptr(ws, "ws", torch.uint8),
        _nbytes(ws), _stream(stream)), "moe_route")


def route_noalloc(dims: Dims, x, w_router, logit_bias, logits, topk_idx, topk_w, slot,
                  expert_count, stream=None) -> None:
    """moe_route without a workspace argument: for callers that cannot allocate device memory.
    Its scratch is a fixed array inside the library, shared by all calls. Calls that overlap
    on the GPU race on it, and shapes beyond its size are rejected (MOE_ERR_WORKSPACE)."""
    T, d, N, k = dims.T, dims.d_model, dims.n_experts, dims.top_k
    _check(_lib.moe_route_noalloc(
        ctypes.byref(dims), _ptr(x, "x", torch.bfloat16, (T, d)),
        _ptr(w_router, "w_router", torch.float32, (N, d)),
        _ptr(logit_bias, "logit_bias", torch.float32, (N,), allow_none=True),
        _ptr(logits, "logits", torch.float32, (T, N)), _ptr(topk_idx, "topk_idx", torch.int32, (T, k)),
        _ptr(topk_w, "topk_w", torch.float32, (T, k)), _ptr(slot, "slot", torch.int32, (T, k)),
        _ptr(expert_count, "expert_count", torch.int32, (N,)), _stream(stream)), "moe_route_noalloc")


def route_with_stats(dims: Dims, x, w_router, logit_bias, logits, topk_idx, topk_w, slot,
                     expert_count, picks, prob_mean, aux_loss, dropped, ws, alpha=0.01,
                     stream=None) -> None:
    """moe_route with the router statistics emitted by the routing launches."""
    T, d, N, k = dims.T, dims.d_model, dims.n_experts, dims.top_k
    _check(_lib.moe_route_with_stats(
        ctypes.byref(dims), _ptr(x, "x", torch.bfloat16, (T, d)),
        _ptr(w_router, "w_router", torch.float32, (N, d)),
        _ptr(logit_bias, "logit_bias", torch.float32, (N,), allow_none=True),
        _ptr(logits, "logits", torch.float32, (T, N)), _ptr(topk_idx, "topk_idx", torch.int32, (T, k)),
        _ptr(topk_w, "topk_w", torch.float32, (T, k)), _ptr(slot, "slot", torch.int32, (T, k)),
        _ptr(expert_count, "expert_count", torch.int32, (N,)), ctypes.c_float(alpha),
        _ptr(picks, "picks", torch.int32, (N,)), _ptr(prob_mean, "prob_mean", torch.float32, (N,)),
        _ptr(aux_loss, "aux_loss", torch.float32, (1,)), _ptr(dropped, "dropped", torch.int32, (1,)),
        _ptr(ws, "ws", torch.uint8), _nbytes(ws), _stream(stream)), "moe_route_with_stats")


def route_from_logits(dims: Dims, logits, topk_idx, topk_w, slot, expert_count, ws,
                      stream=None) -> None:
    T, N, k = dims.T, dims.n_experts, dims.top_k
    _check(_lib.moe_route_from_logits(
        ctypes.byref(dims), _ptr(logits, "logits", torch.float32, (T, N)),
        _ptr(topk_idx, "topk_idx", torch.int32, (T, k)), _ptr(topk_w, "topk_w", torch.float32, (T, k)),
        _ptr(slot, "slot", torch.int32, (T, k)), _ptr(expert_count, "expert_count", torch.int32, (N,)),
        _ptr(ws, "ws", torch.uint8), _nbytes(ws), _stream(stream)), "moe_route_from_logits")


REDIRECT_MAX_PAIRS = 163840  # T * k limit of moe_redirect_overflow


def redirect_overflow(dims: Dims, logits, topk_idx, slot, expert_count, ws, stream=None) -> None:
    """Overflow policy "redirect" after route(): topk_idx is rewritten with the serving expert."""
    T, N, k = dims.T, dims.n_experts, dims.top_k
    _check(_lib.moe_redirect_overflow(
        ctypes.byref(dims), _ptr(logits, "logits", torch.float32, (T, N)),
        _ptr(topk_idx, "topk_idx", torch.int32, (T, k)), _ptr(slot, "slot", torch.int32, (T, k)),
        _ptr(expert_count, "expert_count", torch.int32, (N,)),
        _ptr(ws, "ws", torch.uint8), _nbytes(ws), _stream(stream)), "moe_redirect_overflow")


def permute(dims: Dims, x, topk_idx, slot, expert_count, expert_offset, row_of_pair,
            pair_of_row, x_perm, ws, stream=None) -> None:
    T, d, N, k = dims.T, dims.d_model, dims.n_experts, dims.top_k
    R = max_rows(dims)
    _check(_lib.moe_permute(
        ctypes.byref(dims), _ptr(x, "x", torch.bfloat16, (T, d)),
        _ptr(topk_idx, "topk_idx", torch.int32, (T, k)), _ptr(slot, "slot", torch.int32, (T, k)),
        _ptr(expert_count, "expert_count", torch.int32, (N,)),
        _ptr(expert_offset, "expert_offset", torch.int32, (N + 1,)),
        _ptr(row_of_pair, "row_of_pair", torch.int32, (T, k)),
        _ptr(pair_of_row, "pair_of_row", torch.int32, (R,)),
        _ptr(x_perm, "x_perm", torch.bfloat16, (R, d)), _ptr(ws, "ws", torch.uint8), _nbytes(ws),
        _stream(stream)), "moe_permute")


def grouped_ffn(dims: Dims, x_perm, expert_offset, w_gate_up, w_down, h, y_perm, ws,
                stream=None) -> None:
    d, N, F = dims.d_model, dims.n_experts, dims.d_ff
    R = max_rows(dims)
    rows = 2 * F if dims.act == ACT_SWIGLU else F
    _check(_lib.moe_grouped_ffn(
        ctypes.byref(dims), _ptr(x_perm, "x_perm", torch.bfloat16, (R, d)),
        _ptr(expert_offset, "expert_offset", torch.int32, (N + 1,)),
        _ptr(w_gate_up, "w_gate_up", torch.bfloat16, (N, rows, d)),
        _ptr(w_down, "w_down", torch.bfloat16, (N, d, F)), _ptr(h, "h", torch.bfloat16, (R, F)),
        _ptr(y_perm, "y_perm", torch.float32, (R, d)), _ptr(ws, "ws", torch.uint8), _nbytes(ws),
        _stream(stream)), "moe_grouped_ffn")


def mx_weights(dims: Dims, fmt: str, gate_up, gate_up_scales, down, down_scales) -> MxWeights:
    """Check shapes and dtypes of MX expert weights and describe them for the C ABI.
    gate_up [N, rows, d_model or d_model/2] uint8, gate_up_scales [N, d_model/32, rows] uint8,
    down [N, d_model, d_ff or d_ff/2] uint8, down_scales [N, d_ff/32, d_model] uint8."""
    d, N, F = dims.d_model, dims.n_experts, dims.d_ff
    rows = 2 * F if dims.act == ACT_SWIGLU else F
    per = 1 if fmt.startswith("mxfp8") else 2
    return MxWeights(_WFMT[fmt],
                     _ptr(gate_up, "gate_up", torch.uint8, (N, rows, d // per)),
                     _ptr(gate_up_scales, "gate_up_scales", torch.uint8, (N, d // 32, rows)),
                     _ptr(down, "down", torch.uint8, (N, d, F // per)),
                     _ptr(down_scales, "down_scales", torch.uint8, (N, F // 32, d)))


def grouped_ffn_mx(dims: Dims, x_perm, expert_offset, w: MxWeights, h, y_perm, ws,
                   stream=None) -> None:
    d, N, F = dims.d_model, dims.n_experts, dims.d_ff
    R = max_rows(dims)
    _check(_lib.moe_grouped_ffn_mx(
        ctypes.byref(dims), _ptr(x_perm, "x_perm", torch.bfloat16, (R, d)),
        _ptr(expert_offset, "expert_offset", torch.int32, (N + 1,)), ctypes.byref(w),
        _ptr(h, "h", torch.bfloat16, (R, F)), _ptr(y_perm, "y_perm", torch.float32, (R, d)),
        _ptr(ws, "ws", torch.uint8), _nbytes(ws), _stream(stream)), "moe_grouped_ffn_mx")


def forward_mx_into(dims: Dims, x, w_router, logit_bias, w: MxWeights, residual, out, ws,
                    stream=None) -> None:
    """moe_forward_mx with caller-provided output and workspace (no allocation)."""
    T, d, N = dims.T, dims.d_model, dims.n_experts
    _check(_lib.moe_forward_mx(
        ctypes.byref(dims), _ptr(x, "x", torch.bfloat16, (T, d)),
        _ptr(w_router, "w_router", torch.float32, (N, d)),
        _ptr(logit_bias, "logit_bias", torch.float32, (N,), allow_none=True), ctypes.byref(w),
        _ptr(residual, "residual", torch.bfloat16, (T, d), allow_none=True),
        _ptr(out, "out", torch.bfloat16, (T, d)), _ptr(ws, "ws", torch.uint8), _nbytes(ws),
        _stream(stream)), "moe_forward_mx")


def unpermute_combine(dims: Dims, y_perm, row_of_pair, topk_w, residual, out, ws=None,
                      stream=None) -> None:
    T, d, k = dims.T, dims.d_model, dims.top_k
    R = max_rows(dims)
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out must be bf16 or fp32")
    _check(_lib.moe_unpermute_combine(
        ctypes.byref(dims), _ptr(y_perm, "y_perm", torch.float32, (R, d)),
        _ptr(row_of_pair, "row_of_pair", torch.int32, (T, k)),
        _ptr(topk_w, "topk_w", torch.float32, (T, k)),
        _ptr(residual, "residual", torch.bfloat16, (T, d), allow_none=True),
        _ptr(out, "out", None, (T, d)), 1 if out.dtype == torch.float32 else 0,
        _ptr(ws, "ws", torch.uint8, allow_none=True), _nbytes(ws), _stream(stream)),
        "moe_unpermute_combine")


def router_stats(dims: Dims, logits, topk_idx, slot, picks, prob_mean, aux_loss, dropped, ws,
                 alpha: float = 1e-2, stream=None) -> None:
    """Per-expert picks and mean router probability, dropped pairs, and the auxiliary loss
    alpha * N * sum_e (picks_e / T) * P_e."""
    T, N, k = dims.T, dims.n_experts, dims.top_k
    _check(_lib.moe_router_stats(
        ctypes.byref(dims), _ptr(logits, "logits", torch.float32, (T, N)),
        _ptr(topk_idx, "topk_idx", torch.int32, (T, k)), _ptr(slot, "slot", torch.int32, (T, k)),
        float(alpha), _ptr(picks, "picks", torch.int32, (N,)),
        _ptr(prob_mean, "prob_mean", torch.float32, (N,)),
        _ptr(aux_loss, "aux_loss", torch.float32, (1,)), _ptr(dropped, "dropped", torch.int32, (1,)),
        _ptr(ws, "ws", torch.uint8), _nbytes(ws), _stream(stream)), "moe_router_stats")


def forward_into(dims: Dims, x, w_router, logit_bias, w_gate_up, w_down, residual, out, ws,
                 stream=None) -> None:
    """moe_forward with caller-provided output and workspace (no allocation)."""
    T, d, N, F = dims.T, dims.d_model, dims.n_experts, dims.d_ff
    rows = 2 * F if dims.act == ACT_SWIGLU else F
    _check(_lib.moe_forward(
        ctypes.byref(dims), _ptr(x, "x", torch.bfloat16, (T, d)),
        _ptr(w_router, "w_router", torch.float32, (N, d)),
        _ptr(logit_bias, "logit_bias", torch.float32, (N,), allow_none=True),
        _ptr(w_gate_up, "w_gate_up", torch.bfloat16, (N, rows, d)),
        _ptr(w_down, "w_down", torch.bfloat16, (N, d, F)),
        _ptr(residual, "residual", torch.bfloat16, (T, d), allow_none=True),
        _ptr(out, "out", torch.bfloat16, (T, d)), _ptr(ws, "ws", torch.uint8), _nbytes(ws),
        _stream(stream)), "moe_forward")


def forward(x: torch.Tensor, w_router: torch.Tensor, w_gate_up: torch.Tensor,
            w_down: torch.Tensor, *, top_k: int, act: str = "swiglu",
            capacity_factor: Optional[float] = None, logit_bias: Optional[torch.Tensor] = None,
            residual: Optional[torch.Tensor] = None, use_residual: bool = True,
            workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The whole layer; allocates the output (and a workspace unless one is given).

    ``residual`` defaults to ``x`` (the layer returns x + MoE(x)); pass use_residual=False for
    the MoE part alone.
    """
    T, d = x.shape
    N = w_router.shape[0]
    F = w_down.shape[2]
    dims = make_dims(T, d, N, top_k, F, act, capacity(capacity_factor, T, N))
    if workspace is None:
        workspace = new_workspace(dims, x.device, forward=True)
    out = torch.empty((T, d), dtype=torch.bfloat16, device=x.device)
    res = (x if residual is None else residual) if use_residual else None
    forward_into(dims, x, w_router, logit_bias, w_gate_up, w_down, res, out, workspace)
    return out


def exported_symbols() -> list:
    """Names of the functions include/moe.h declares (parsed from the header)."""
    import re
    hdr = os.path.join(os.path.dirname(_HERE), "include", "moe.h")
    with open(hdr) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(moe_\w+)\s*\(", text, flags=re.M)))


# ----------------------------------------------------------------------------- backward
def backward_workspace_bytes(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.moe_backward_workspace_bytes(ctypes.byref(dims), ctypes.byref(n)),
           "moe_backward_workspace_bytes")
    return int(n.value)


def new_backward_workspace(dims: Dims, device=None) -> torch.Tensor:
    return torch.zeros(backward_workspace_bytes(dims), dtype=torch.uint8, device=device or "cuda")


def backward_into(dims: Dims, x, w_router, w_gate_up, w_down, fwd_ws, d_out, d_x, d_w_router,
                  d_logit_bias, d_w_gate_up, d_w_down, ws, stream=None) -> None:
    """moe_backward after moe_forward (whose workspace is fwd_ws) on the same inputs."""
    T, d, N, F = dims.T, dims.d_model, dims.n_experts, dims.d_ff
    rows = 2 * F if dims.act == ACT_SWIGLU else F
    _check(_lib.moe_backward(
        ctypes.byref(dims), _ptr(x, "x", torch.bfloat16, (T, d)),
        _ptr(w_router, "w_router", torch.float32, (N, d)),
        _ptr(w_gate_up, "w_gate_up", torch.bfloat16, (N, rows, d)),
        _ptr(w_down, "w_down", torch.bfloat16, (N, d, F)),
        _ptr(fwd_ws, "fwd_ws", torch.uint8), _nbytes(fwd_ws),
        _ptr(d_out, "d_out", torch.bfloat16, (T, d)), _ptr(d_x, "d_x", torch.float32, (T, d)),
        _ptr(d_w_router, "d_w_router", torch.float32, (N, d)),
        _ptr(d_logit_bias, "d_logit_bias", torch.float32, (N,), allow_none=True),
        _ptr(d_w_gate_up, "d_w_gate_up", torch.float32, (N, rows, d)),
        _ptr(d_w_down, "d_w_down", torch.float32, (N, d, F)),
        _ptr(ws, "ws", torch.uint8), _nbytes(ws), _stream(stream)), "moe_backward")
