"""Seeded synthetic inputs for the sparse MoE layer forward pass.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It draws random tensors and nothing else: it holds none of the
layer's arithmetic (no routing, no capacity, no expert math).

Layer shapes follow the five synthetic workloads the build is measured on:

* ``tiny_top2``        T=64,    d=128,  N=8,   k=2, SwiGLU d_ff=256,   capacity factor 1.25
* ``switch_top1``      T=4096,  d=1024, N=64,  k=1, GELU   d_ff=4096,  capacity factor 1.0
* ``mixtral``          T in {1,16,512,8192}, d=4096, N=8, k=2, SwiGLU d_ff=14336, no capacity limit
* ``gpt_oss``          T in {1,8,64,16384},  d=2880, N=32, k=4, SwiGLU d_ff=2880, no capacity limit
* ``fine_grained``     T=16384, d=7168, N=256, k=8, SwiGLU d_ff=2048,  capacity factor 1.25,
                       Zipf(s=1.1) additive router-logit bias

Value distributions (one reading of the ``N(0, s)`` notation, stated once):

* hidden states x ~ N(0, 1), rounded to bf16 (round-to-nearest-even);
* router weight W_r ~ N(0, variance 1/d_model), kept in fp32, so that logits are ~N(0, 1);
* expert weights ~ N(0, std 0.02), rounded to bf16;
* the residual stream is x itself;
* ``fine_grained`` adds b_e = ln(p_{e+1}) to expert e's logit, where
  p_r = r^-s / sum_{r'=1..N} r'^-s (expert 0 hottest).

Every tensor is drawn from its own torch generator whose seed is derived from
(seed, tensor id, expert id), so tensors do not depend on generation order and
large expert stacks can be drawn one expert at a time on the device.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Tuple

import torch


@dataclass(frozen=True)
class LayerShape:
    name: str
    d_model: int
    n_experts: int
    top_k: int
    d_ff: int
    act: str                      # "swiglu" or "gelu"
    capacity_factor: Optional[float]  # None = no capacity limit
    token_counts: Tuple[int, ...]
    zipf_s: Optional[float] = None

    def gate_up_rows(self) -> int:
        return 2 * self.d_ff if self.act == "swiglu" else self.d_ff

    def describe(self, T: int) -> str:
        cf = "none" if self.capacity_factor is None else f"{self.capacity_factor:g}"
        z = "" if self.zipf_s is None else f" zipf_bias={self.zipf_s:g}"
        return (f"{self.name} T={T} d_model={self.d_model} N={self.n_experts} "
                f"k={self.top_k} d_ff={self.d_ff} {self.act} capacity_factor={cf}{z}")


SHAPES = {
    "tiny_top2": LayerShape("tiny_top2", 128, 8, 2, 256, "swiglu", 1.25, (64,)),
    "switch_top1": LayerShape("switch_top1", 1024, 64, 1, 4096, "gelu", 1.0, (4096,)),
    "mixtral": LayerShape("mixtral", 4096, 8, 2, 14336, "swiglu", None, (1, 16, 512, 8192)),
    "gpt_oss": LayerShape("gpt_oss", 2880, 32, 4, 2880, "swiglu", None, (1, 8, 64, 16384)),
    "fine_grained": LayerShape("fine_grained", 7168, 256, 8, 2048, "swiglu", 1.25, (16384,), zipf_s=1.1),
}

# tensor ids for per-tensor generator streams
_X, _WR, _WGU, _WD = 1, 2, 3, 4
_WGU_Q, _WGU_S, _WD_Q, _WD_S = 5, 6, 7, 8
_DOUT = 9


def _gen(device: torch.device, seed: int, tensor_id: int, sub: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    # distinct, order-independent 63-bit seeds per (seed, tensor, expert)
    s = (seed * 1_000_003 + tensor_id * 65_537 + sub * 257 + 12345) & ((1 << 63) - 1)
    g.manual_seed(s)
    return g


def _normal(shape, std: float, device, seed, tensor_id, sub=0) -> torch.Tensor:
    g = _gen(device, seed, tensor_id, sub)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def zipf_logit_bias(n_experts: int, s: float) -> torch.Tensor:
    """b_e = ln(p_{e+1}) with p_r proportional to r^-s, normalised over r = 1..N (fp32)."""
    ranks = torch.arange(1, n_experts + 1, dtype=torch.float64)
    w = ranks.pow(-s)
    p = w / w.sum()
    return torch.log(p).to(torch.float32)


def make_hidden(T: int, d_model: int, *, seed: int = 0, device="cpu") -> torch.Tensor:
    """x ~ N(0,1) rounded to bf16, shape [T, d_model]."""
    return _normal((T, d_model), 1.0, torch.device(device), seed, _X).to(torch.bfloat16)


def make_grad_output(T: int, d_model: int, *, seed: int = 0, device="cpu") -> torch.Tensor:
    """Gradient of the layer output for the backward pass: N(0,1) rounded to bf16, [T, d_model]."""
    return _normal((T, d_model), 1.0, torch.device(device), seed, _DOUT).to(torch.bfloat16)


def make_layer_weights(shape: LayerShape, *, seed: int = 0, device="cpu",
                       expert_std: float = 0.02) -> dict:
    """Router and packed expert weights for one layer shape.

    w_router  [N, d]            fp32, N(0, 1/d)
    logit_bias [N] fp32 or None  Zipf bias for skewed shapes
    w_gate_up [N, 2F, d] bf16    (SwiGLU: rows 0..F-1 gate, F..2F-1 up) or [N, F, d] (GELU)
    w_down    [N, d, F] bf16
    """
    dev = torch.device(device)
    N, d, F = shape.n_experts, shape.d_model, shape.d_ff
    rows = shape.gate_up_rows()
    w_gate_up = torch.empty((N, rows, d), dtype=torch.bfloat16, device=dev)
    w_down = torch.empty((N, d, F), dtype=torch.bfloat16, device=dev)
    for e in range(N):  # one expert at a time keeps the fp32 temporaries small
        gu, dn = make_expert_weights(shape, e, seed=seed, device=dev, expert_std=expert_std)
        w_gate_up[e].copy_(gu)
        w_down[e].copy_(dn)
    return {**make_router_weights(shape, seed=seed, device=dev), "w_gate_up": w_gate_up,
            "w_down": w_down}


def make_router_weights(shape: LayerShape, *, seed: int = 0, device="cpu") -> dict:
    """w_router [N, d] fp32 N(0, 1/d) and the logit bias ([N] fp32 for skewed shapes, else None)."""
    dev = torch.device(device)
    N, d = shape.n_experts, shape.d_model
    w_router = _normal((N, d), 1.0 / math.sqrt(d), dev, seed, _WR)
    bias = zipf_logit_bias(N, shape.zipf_s).to(dev) if shape.zipf_s is not None else None
    return {"w_router": w_router, "logit_bias": bias}


def make_expert_weights(shape: LayerShape, e: int, *, seed: int = 0, device="cpu",
                        expert_std: float = 0.02) -> Tuple[torch.Tensor, torch.Tensor]:
    """Expert e's packed weights alone, bf16: gate_up [2F or F, d] and down [d, F]. The same
    values as expert e of make_layer_weights on the same device type."""
    dev = torch.device(device)
    d, F = shape.d_model, shape.d_ff
    gu = _normal((shape.gate_up_rows(), d), expert_std, dev, seed, _WGU, e).to(torch.bfloat16)
    dn = _normal((d, F), expert_std, dev, seed, _WD, e).to(torch.bfloat16)
    return gu, dn


def make_layer_inputs(shape: LayerShape, T: int, *, seed: int = 0, device="cpu",
                      expert_std: float = 0.02) -> dict:
    d = make_layer_weights(shape, seed=seed, device=device, expert_std=expert_std)
    d["x"] = make_hidden(T, shape.d_model, seed=seed, device=device)
    return d


def make_custom_inputs(T: int, d_model: int, n_experts: int, d_ff: int, act: str, *,
                       seed: int = 0, device="cpu", expert_std: float = 0.02,
                       router_std: Optional[float] = None, zipf_s: Optional[float] = None) -> dict:
    """Inputs for an arbitrary (small) layer shape, same recipe as the named shapes."""
    shape = LayerShape("custom", d_model, n_experts, 1, d_ff, act, None, (T,), zipf_s)
    out = make_layer_inputs(shape, T, seed=seed, device=device, expert_std=expert_std)
    if router_std is not None:
        out["w_router"] = _normal((n_experts, d_model), router_std, torch.device(device), seed, _WR)
    return out


# ---------------------------------------------------------------- MX-format expert weights
# Expert weights stored in an MX format are drawn as codes directly (no quantisation step):
#   element codes: "mxfp8" E4M3 codes uniform over the 254 non-NaN codes; "mxfp4" E2M1 codes
#                  uniform over all 16 codes, two per byte;
#   scale codes:   E8M0 codes 127 + scale_exp + U{-1, 0, 1} per block of 32 elements.
# scale_exp is chosen so that the decoded weights have magnitudes like the bf16 recipe's
# (E4M3 codes reach 448, E2M1 codes 6).
MX_SCALE_EXP = {"mxfp8": -13, "mxfp4": -8}


def _mx_codes(shape, fmt: str, g: torch.Generator, device) -> torch.Tensor:
    if fmt == "mxfp8":
        c = torch.randint(0, 254, shape, generator=g, device=device, dtype=torch.int32)
        c = c + (c >= 127).to(torch.int32)  # skip 0x7F; 0xFF is never drawn
        return c.to(torch.uint8)
    if fmt == "mxfp4":
        packed = shape[:-1] + (shape[-1] // 2,)
        return torch.randint(0, 256, packed, generator=g, device=device, dtype=torch.int32).to(torch.uint8)
    raise ValueError(fmt)


def make_mx_matrix_stack(n_experts: int, rows: int, K: int, fmt: str, *, seed: int, tensor_id: int,
                         scale_tensor_id: int, device="cpu") -> Tuple[torch.Tensor, torch.Tensor]:
    """elements [N, rows, K] (mxfp8) or [N, rows, K/2] (mxfp4) uint8, scales [N, K/32, rows] uint8."""
    dev = torch.device(device)
    kb = K if fmt == "mxfp8" else K // 2
    el = torch.empty((n_experts, rows, kb), dtype=torch.uint8, device=dev)
    sc = torch.empty((n_experts, K // 32, rows), dtype=torch.uint8, device=dev)
    for e in range(n_experts):
        el[e].copy_(_mx_codes((rows, K), fmt, _gen(dev, seed, tensor_id, e), dev))
        j = torch.randint(-1, 2, (K // 32, rows), generator=_gen(dev, seed, scale_tensor_id, e),
                          device=dev, dtype=torch.int32)
        sc[e].copy_((127 + MX_SCALE_EXP[fmt] + j).to(torch.uint8))
    return el, sc


def make_mx_layer_inputs(shape: LayerShape, T: int, fmt: str, *, seed: int = 0, device="cpu") -> dict:
    """Hidden states and router as in make_layer_inputs; expert weights in an MX format:
    w_gate_up_q/_s for the packed gate_up rows ([N, 2F or F, d]) and w_down_q/_s ([N, d, F]).
    fmt "mxfp8_bs" / "mxfp4_bs" (block-scaled path) draws the same weights as "mxfp8" / "mxfp4"."""
    dev = torch.device(device)
    N, d, F = shape.n_experts, shape.d_model, shape.d_ff
    wfmt, fmt = fmt, fmt[:-3] if fmt.endswith("_bs") else fmt
    w_router = _normal((N, d), 1.0 / math.sqrt(d), dev, seed, _WR)
    bias = zipf_logit_bias(N, shape.zipf_s).to(dev) if shape.zipf_s is not None else None
    gq, gs = make_mx_matrix_stack(N, shape.gate_up_rows(), d, fmt, seed=seed, tensor_id=_WGU_Q,
                                  scale_tensor_id=_WGU_S, device=dev)
    dq, ds = make_mx_matrix_stack(N, d, F, fmt, seed=seed, tensor_id=_WD_Q, scale_tensor_id=_WD_S,
                                  device=dev)
    return {"x": make_hidden(T, d, seed=seed, device=dev), "w_router": w_router, "logit_bias": bias,
            "wfmt": wfmt, "w_gate_up_q": gq, "w_gate_up_s": gs, "w_down_q": dq, "w_down_s": ds}


def make_mx_custom_inputs(T: int, d_model: int, n_experts: int, d_ff: int, act: str, fmt: str, *,
                          seed: int = 0, device="cpu", zipf_s: Optional[float] = None) -> dict:
    shape = LayerShape("custom", d_model, n_experts, 1, d_ff, act, None, (T,), zipf_s)
    return make_mx_layer_inputs(shape, T, fmt, seed=seed, device=device)
