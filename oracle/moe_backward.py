"""CPU oracle for the backward pass of the sparse Mixture-of-Experts layer.

TEST INFRASTRUCTURE. Only the test suite and the benchmark's CPU legs may import or run
this module; the CUDA library never calls it and shares no code with it.

The pages discuss training MoE layers (page «Что такое Mixture of Experts (MoE) в
трансформерах: архитектура и параллелизм», section «Обучение MoE с помощью Transformers»:
grouped-GEMM kernels for training) but print no gradient formulas. The backward pass here
is the derivative of the forward pass the oracle defines (``moe_oracle``), written out by
the chain rule in float64, one step per function, in reverse order of the forward:

  out[t] = residual[t] + sum over kept j of w[t, j] * y[row(t, j)]
  y[r]   = h[r] W_d^T,          h = silu(x W_g^T) * (x W_u^T)   (SwiGLU)
                                h = gelu(x W_1^T)               (GELU)
  w[t]   = softmax of the chosen logits L[t, idx[t, :]]
  L      = x W_r^T (+ b)

Reading: the choice of experts (top-k) and the capacity slots are piecewise constant in
the inputs and pass no gradient; dropped pairs contribute nothing to out, so their weight
gets a zero gradient, but it still takes part in the softmax over the chosen logits. The
residual's gradient is d_out itself and is not part of the returned dx.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np
from scipy.special import erf as _erf

from .moe_oracle import (expert_permutation, router_logits, route_from_logits, silu, gelu)


def logistic(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def silu_derivative(z: np.ndarray) -> np.ndarray:
    """d/dz [z * s(z)] = s(z) + z * s(z) * (1 - s(z)), s the logistic function."""
    s = logistic(z)
    return s + z * s * (1.0 - s)


def gelu_derivative(z: np.ndarray) -> np.ndarray:
    """d/dz [z * Phi(z)] = Phi(z) + z * phi(z) (exact erf GELU)."""
    Phi = 0.5 * (1.0 + _erf(z / math.sqrt(2.0)))
    phi = np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)
    return Phi + z * phi


def combine_backward(d_out: np.ndarray, y_rows: np.ndarray, topk_w: np.ndarray,
                     row_of_pair: np.ndarray):
    """Gradients of out[t] = sum_j w[t, j] y[row(t, j)] with respect to y and w.

    dy[row(t, j)] = w[t, j] * d_out[t];  dw[t, j] = <d_out[t], y[row(t, j)]>; dropped pairs
    have no row and get dw = 0.
    """
    T, k = topk_w.shape
    dy = np.zeros_like(y_rows)
    dw = np.zeros((T, k))
    for t in range(T):
        for j in range(k):
            r = row_of_pair[t, j]
            if r < 0:
                continue
            dy[r] = topk_w[t, j] * d_out[t]
            dw[t, j] = float(d_out[t] @ y_rows[r])
    return dy, dw


def renormalise_backward(topk_w: np.ndarray, dw: np.ndarray, topk_idx: np.ndarray,
                         n_experts: int) -> np.ndarray:
    """Gradient of the chosen logits through w = softmax(L[idx]) (the renormalised top-k).

    dw_j/dL_i = w_j (delta_ij - w_i) for chosen i, so dL_i = w_i (dw_i - sum_j w_j dw_j);
    experts not chosen get zero.
    """
    T, k = topk_w.shape
    dL = np.zeros((T, n_experts))
    for t in range(T):
        s = float(topk_w[t] @ dw[t])
        for i in range(k):
            dL[t, topk_idx[t, i]] += topk_w[t, i] * (dw[t, i] - s)
    return dL


def aux_loss_backward(logits: np.ndarray, topk_idx: np.ndarray, alpha: float = 1e-2,
                      d_aux: float = 1.0) -> np.ndarray:
    """Gradient of the auxiliary loss with respect to the logits (page «Sparse
    Mixture-of-Experts», section «Маршрутизация токена и auxiliary loss»: aux =
    alpha * N * sum_e f_e * P_e, f_e the fraction of the batch's tokens sent to expert e, P_e
    the batch mean of the router probability).

    f comes from the choice of experts and passes no gradient. P_e = (1/T) sum_t p_te and
    dp_te/dL_ti = p_te (delta_ei - p_ti), so
    dL_ti = d_aux * alpha * N / T * p_ti * (f_i - sum_e f_e p_te).
    """
    T, N = logits.shape
    z = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    f = np.zeros(N)
    for t in range(T):
        for e in topk_idx[t]:
            f[int(e)] += 1.0 / T
    return d_aux * alpha * N / T * p * (f[None, :] - (p * f[None, :]).sum(axis=1, keepdims=True))


def expert_backward(rows: np.ndarray, dy: np.ndarray, w_gate_up: np.ndarray,
                    w_down: np.ndarray, act: str):
    """One expert's rows: y = act-FFN(rows). Returns (d_rows, d_w_gate_up, d_w_down, pre, h).

    dh = dy W_d;  dW_d = dy^T h.
    SwiGLU: pre = [g | u] = rows [W_g | W_u]^T, h = silu(g) u;
            dg = dh u silu'(g), du = dh silu(g), d_pre = [dg | du].
    GELU:   pre = rows W_1^T, h = gelu(pre), d_pre = dh gelu'(pre).
    d_rows = d_pre W_gu;  dW_gu = d_pre^T rows.
    """
    pre = rows @ w_gate_up.T
    if act == "swiglu":
        F = w_gate_up.shape[0] // 2
        g, u = pre[:, :F], pre[:, F:]
        h = silu(g) * u
    elif act == "gelu":
        h = gelu(pre)
    else:
        raise ValueError(f"unknown activation {act!r}")
    dh = dy @ w_down
    d_w_down = dy.T @ h
    if act == "swiglu":
        d_pre = np.concatenate([dh * u * silu_derivative(g), dh * silu(g)], axis=1)
    else:
        d_pre = dh * gelu_derivative(pre)
    d_rows = d_pre @ w_gate_up
    d_w_gate_up = d_pre.T @ rows
    return d_rows, d_w_gate_up, d_w_down, pre, h


def moe_layer_backward(x: np.ndarray, w_router: np.ndarray, w_gate_up: np.ndarray,
                       w_down: np.ndarray, d_out: np.ndarray, *, top_k: int, act: str,
                       capacity: int, logit_bias: Optional[np.ndarray] = None,
                       logits: Optional[np.ndarray] = None) -> dict:
    """Gradients of the whole layer (without the residual's identity term).

    ``logits`` lets a caller route on given logits (the GPU's own, so that the routing is
    the same); by default they are computed from x, w_router and logit_bias.
    Returns dx [T, d], d_w_router [N, d], d_logit_bias [N], d_w_gate_up, d_w_down (the
    weights' shapes) and the intermediates of each step.
    """
    T, d = x.shape
    N = w_router.shape[0]
    if logits is None:
        logits = router_logits(x, w_router, logit_bias)
    r = route_from_logits(logits, top_k, capacity)
    off, rop, por = expert_permutation(r["topk_idx"], r["slot"], r["expert_count"])
    R = int(off[-1])
    x_rows = np.zeros((R, d))
    for row in range(R):
        x_rows[row] = x[por[row] // top_k]
    # forward outputs of each expert's rows
    y_rows = np.zeros((R, d))
    for e in range(N):
        a, b = int(off[e]), int(off[e + 1])
        if b > a:
            pre = x_rows[a:b] @ w_gate_up[e].T
            if act == "swiglu":
                F = w_gate_up.shape[1] // 2
                h = silu(pre[:, :F]) * pre[:, F:]
            else:
                h = gelu(pre)
            y_rows[a:b] = h @ w_down[e].T
    dy, dw = combine_backward(d_out, y_rows, r["topk_w"], rop)
    dx_rows = np.zeros((R, d))
    d_w_gate_up = np.zeros_like(w_gate_up, dtype=np.float64)
    d_w_down = np.zeros_like(w_down, dtype=np.float64)
    pre_rows = np.zeros((R, w_gate_up.shape[1]))
    h_rows = np.zeros((R, w_down.shape[2]))
    for e in range(N):
        a, b = int(off[e]), int(off[e + 1])
        if b == a:
            continue
        dxr, dgu, dd, pre, h = expert_backward(x_rows[a:b], dy[a:b], w_gate_up[e], w_down[e], act)
        dx_rows[a:b] = dxr
        d_w_gate_up[e] = dgu
        d_w_down[e] = dd
        pre_rows[a:b] = pre
        h_rows[a:b] = h
    dL = renormalise_backward(r["topk_w"], dw, r["topk_idx"], N)
    dx = dL @ w_router
    for row in range(R):
        dx[por[row] // top_k] += dx_rows[row]
    return {"dx": dx, "d_w_router": dL.T @ x, "d_logit_bias": dL.sum(axis=0),
            "d_w_gate_up": d_w_gate_up, "d_w_down": d_w_down,
            "dw": dw, "d_logits": dL, "dy_rows": dy, "dx_rows": dx_rows,
            "pre_rows": pre_rows, "h_rows": h_rows, "y_rows": y_rows,
            "expert_offset": off, "row_of_pair": rop, "pair_of_row": por, **r}
