"""Pins of the backward oracle: values it does not produce itself.

* central finite differences of the forward oracle (itself pinned to the pages) for every
  input element, on small batches whose routing does not change under the perturbation;
* special cases that reduce to a library routine: one expert with k = 1 and no capacity
  limit is a plain FFN, and k = N with no limit is a softmax-gated dense mixture; both are
  differentiated by torch.autograd in float64.

Each pin takes the backward module (``oracle.moe_backward``) so that tests can plant
mistakes in it.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle.moe_oracle as fwd


def _problem(seed, T, d, N, F, act, bias):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(T, d))
    wr = rng.normal(size=(N, d)) / math.sqrt(d)
    rows = 2 * F if act == "swiglu" else F
    wgu = rng.normal(size=(N, rows, d)) * 0.4
    wd = rng.normal(size=(N, d, F)) * 0.4
    b = rng.normal(size=N) * 0.3 if bias else None
    g = rng.normal(size=(T, d))
    return x, wr, wgu, wd, b, g


def _margin(logits, k):
    """Smallest gap between the k-th and (k+1)-th logit of any token, and between chosen
    logits, so that a perturbation below it keeps the routing."""
    s = np.sort(logits, axis=1)[:, ::-1]
    gaps = np.diff(-s, axis=1)
    return float(gaps.min()) if gaps.size else 1.0


def _loss(x, wr, wgu, wd, b, g, k, act, cap):
    out = fwd.moe_layer_forward(x, wr, wgu, wd, top_k=k, act=act, capacity=cap,
                                logit_bias=b)["out"]
    return float((g * out).sum())


def _fd_check(bwd, seed, T, d, N, F, k, act, cap, bias):
    x, wr, wgu, wd, b, g = _problem(seed, T, d, N, F, act, bias)
    L = fwd.router_logits(x, wr, b)
    assert _margin(L, k) > 1e-3, "pick another seed: logits too close for finite differences"
    got = bwd.moe_layer_backward(x, wr, wgu, wd, g, top_k=k, act=act, capacity=cap, logit_bias=b)
    base = fwd.route_from_logits(L, k, cap)
    eps = 1e-6
    params = {"dx": x, "d_w_router": wr, "d_w_gate_up": wgu, "d_w_down": wd}
    if bias:
        params["d_logit_bias"] = b
    for name, arr in params.items():
        num = np.zeros_like(arr)
        flat = arr.reshape(-1)
        nflat = num.reshape(-1)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + eps
            lp = _loss(x, wr, wgu, wd, b, g, k, act, cap)
            flat[i] = keep - eps
            lm = _loss(x, wr, wgu, wd, b, g, k, act, cap)
            flat[i] = keep
            nflat[i] = (lp - lm) / (2 * eps)
        # the routing is unchanged by the perturbations (margin check above)
        r2 = fwd.route_from_logits(fwd.router_logits(x, wr, b), k, cap)
        assert np.array_equal(r2["slot"], base["slot"])
        err = np.abs(got[name] - num).max()
        scale = max(1.0, np.abs(num).max())
        assert err <= 1e-6 * scale, f"{name}: finite differences differ by {err}"
    return base


def pin_fd_swiglu_top2_drops(bwd):
    # capacity 2 with 6 tokens, 4 experts, top-2: some pairs are dropped
    base = _fd_check(bwd, 3, 6, 5, 4, 3, 2, "swiglu", 2, bias=True)
    assert (base["slot"] < 0).any()


def pin_fd_gelu_top1(bwd):
    base = _fd_check(bwd, 8, 7, 4, 3, 5, 1, "gelu", 2, bias=False)
    assert (base["slot"] < 0).any()


def pin_fd_swiglu_top3_no_limit(bwd):
    _fd_check(bwd, 12, 4, 4, 5, 3, 3, "swiglu", 4, bias=False)


def _torch_ffn(X, wgu, wd, act):
    pre = X @ wgu.T
    if act == "swiglu":
        F = wgu.shape[0] // 2
        h = torch.nn.functional.silu(pre[:, :F]) * pre[:, F:]
    else:
        h = torch.nn.functional.gelu(pre)  # exact erf form
    return h @ wd.T


def pin_single_expert_is_plain_ffn(bwd):
    for act in ("swiglu", "gelu"):
        x, wr, wgu, wd, _, g = _problem(21, 9, 6, 1, 5, act, False)
        got = bwd.moe_layer_backward(x, wr, wgu, wd, g, top_k=1, act=act, capacity=9)
        X = torch.tensor(x, requires_grad=True)
        Wgu = torch.tensor(wgu[0], requires_grad=True)
        Wd = torch.tensor(wd[0], requires_grad=True)
        (torch.from_numpy(g) * _torch_ffn(X, Wgu, Wd, act)).sum().backward()
        np.testing.assert_allclose(got["dx"], X.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(got["d_w_gate_up"][0], Wgu.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(got["d_w_down"][0], Wd.grad.numpy(), rtol=1e-10, atol=1e-12)
        # one expert: its weight is 1 whatever the logit, so the router gets no gradient
        assert np.abs(got["d_w_router"]).max() == 0.0


def pin_dense_mixture(bwd):
    # k = N, no capacity: out = sum_e softmax(x W_r^T)_e FFN_e(x)
    x, wr, wgu, wd, b, g = _problem(34, 5, 4, 3, 3, "swiglu", True)
    got = bwd.moe_layer_backward(x, wr, wgu, wd, g, top_k=3, act="swiglu", capacity=5,
                                 logit_bias=b)
    X = torch.tensor(x, requires_grad=True)
    Wr = torch.tensor(wr, requires_grad=True)
    B = torch.tensor(b, requires_grad=True)
    Wgu = torch.tensor(wgu, requires_grad=True)
    Wd = torch.tensor(wd, requires_grad=True)
    p = torch.softmax(X @ Wr.T + B, dim=-1)
    out = sum(p[:, e:e + 1] * _torch_ffn(X, Wgu[e], Wd[e], "swiglu") for e in range(3))
    (torch.from_numpy(g) * out).sum().backward()
    for name, ref in (("dx", X.grad), ("d_w_router", Wr.grad), ("d_logit_bias", B.grad),
                      ("d_w_gate_up", Wgu.grad), ("d_w_down", Wd.grad)):
        np.testing.assert_allclose(got[name], ref.numpy(), rtol=1e-10, atol=1e-12, err_msg=name)


def pin_aux_loss_gradient(bwd):
    """Finite differences of the forward oracle's auxiliary loss (routing held fixed by a
    margin check), and two closed forms: a batch that loads every expert equally, and a single
    expert, both have a zero gradient (sum_e p_te = 1)."""
    rng = np.random.default_rng(41)
    for T, N, k in ((9, 5, 2), (12, 4, 1)):
        L = rng.normal(size=(T, N)) * 2.0
        assert _margin(L, k) > 1e-3
        idx = fwd.select_top_k(L, k)
        got = bwd.aux_loss_backward(L, idx, alpha=0.01)
        slot = np.zeros_like(idx)
        eps = 1e-6
        num = np.zeros_like(L)
        for t in range(T):
            for i in range(N):
                keep = L[t, i]
                L[t, i] = keep + eps
                lp = fwd.router_statistics(L, idx, slot, alpha=0.01)["aux_loss"]
                L[t, i] = keep - eps
                lm = fwd.router_statistics(L, idx, slot, alpha=0.01)["aux_loss"]
                L[t, i] = keep
                num[t, i] = (lp - lm) / (2 * eps)
        assert np.abs(got - num).max() <= 1e-8 * max(1.0, np.abs(num).max())
    # every expert picked equally often: f_e = k / N, and the gradient vanishes
    T, N, k = 8, 4, 2
    idx = np.array([[t % N, (t + 1) % N] for t in range(T)])
    g = bwd.aux_loss_backward(rng.normal(size=(T, N)), idx, alpha=0.5)
    assert np.abs(g).max() < 1e-15
    g1 = bwd.aux_loss_backward(rng.normal(size=(5, 1)), np.zeros((5, 1), dtype=np.int64))
    assert np.abs(g1).max() == 0.0


BACKWARD_PINS = [pin_fd_swiglu_top2_drops, pin_fd_gelu_top1, pin_fd_swiglu_top3_no_limit,
                 pin_single_expert_is_plain_ffn, pin_dense_mixture, pin_aux_loss_gradient]
