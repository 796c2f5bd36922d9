"""The backward oracle against its pins, and planted mistakes that some pin must catch
(CPU only; the mistakes are planted in the oracle module with monkeypatch)."""
import math

import numpy as np
import pytest

import oracle.moe_backward as bwd
from tests import oracle_backward_pins as pins


@pytest.mark.parametrize("pin", pins.BACKWARD_PINS, ids=lambda f: f.__name__)
def test_backward_pin(pin):
    pin(bwd)


def _silu_derivative_no_second_term(z):
    return bwd.logistic(z)


def _gelu_derivative_cdf_only(z):
    from scipy.special import erf
    return 0.5 * (1.0 + erf(z / math.sqrt(2.0)))


def _renormalise_backward_plain_softmax_missing_sum(topk_w, dw, topk_idx, n_experts):
    T, k = topk_w.shape
    dL = np.zeros((T, n_experts))
    for t in range(T):
        for i in range(k):
            dL[t, topk_idx[t, i]] += topk_w[t, i] * dw[t, i]
    return dL


def _renormalise_backward_sign(topk_w, dw, topk_idx, n_experts):
    return -bwd.__dict__["_orig_renormalise_backward"](topk_w, dw, topk_idx, n_experts)


def _combine_backward_unscaled(d_out, y_rows, topk_w, row_of_pair):
    dy, dw = bwd.__dict__["_orig_combine_backward"](d_out, y_rows, topk_w, row_of_pair)
    T, k = topk_w.shape
    for t in range(T):
        for j in range(k):
            if row_of_pair[t, j] >= 0:
                dy[row_of_pair[t, j]] = d_out[t]
    return dy, dw


def _expert_backward_transposed_dw_down(rows, dy, wgu, wd, act):
    d_rows, dgu, dd, pre, h = bwd.__dict__["_orig_expert_backward"](rows, dy, wgu, wd, act)
    return d_rows, dgu, (dd.T if dd.shape[0] == dd.shape[1] else dd[::-1]), pre, h


def _expert_backward_swapped_gate_up(rows, dy, wgu, wd, act):
    d_rows, dgu, dd, pre, h = bwd.__dict__["_orig_expert_backward"](rows, dy, wgu, wd, act)
    if act == "swiglu":
        F = wgu.shape[0] // 2
        dgu = np.concatenate([dgu[F:], dgu[:F]], axis=0)
    return d_rows, dgu, dd, pre, h


def _aux_backward_without_mean_term(logits, topk_idx, alpha=1e-2, d_aux=1.0):
    T, N = logits.shape
    z = np.exp(logits - logits.max(axis=1, keepdims=True))
    p = z / z.sum(axis=1, keepdims=True)
    f = np.zeros(N)
    for t in range(T):
        for e in topk_idx[t]:
            f[int(e)] += 1.0 / T
    return d_aux * alpha * N / T * p * f[None, :]


def _aux_backward_per_pair_f(logits, topk_idx, alpha=1e-2, d_aux=1.0):
    k = topk_idx.shape[1]
    return bwd.__dict__["_orig_aux_loss_backward"](logits, topk_idx, alpha, d_aux) / k


MUTANTS = {
    "aux_backward_without_mean_term": ("aux_loss_backward", _aux_backward_without_mean_term),
    "aux_backward_f_over_pairs": ("aux_loss_backward", _aux_backward_per_pair_f),
    "silu_derivative_without_z_term": ("silu_derivative", _silu_derivative_no_second_term),
    "gelu_derivative_without_z_phi": ("gelu_derivative", _gelu_derivative_cdf_only),
    "renormalise_backward_missing_sum": ("renormalise_backward",
                                         _renormalise_backward_plain_softmax_missing_sum),
    "renormalise_backward_sign": ("renormalise_backward", _renormalise_backward_sign),
    "combine_backward_dy_not_weighted": ("combine_backward", _combine_backward_unscaled),
    "expert_backward_wrong_w_down_layout": ("expert_backward", _expert_backward_transposed_dw_down),
    "expert_backward_gate_up_swapped": ("expert_backward", _expert_backward_swapped_gate_up),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_some_backward_pin_catches(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setitem(bwd.__dict__, "_orig_" + attr, getattr(bwd, attr))
    monkeypatch.setattr(bwd, attr, fn)
    caught = []
    for pin in pins.BACKWARD_PINS:
        try:
            pin(bwd)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
