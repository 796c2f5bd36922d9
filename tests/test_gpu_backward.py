"""Backward pass on the GPU against the float64 backward oracle (GPU).

The oracle routes on the GPU's own logits, so both sides take the same experts and slots.
Bars, per gradient tensor g against the oracle's o:
  mean-rel  sum |g - o| / sum |o| <= 1e-2;
  max-abs   max |g - o| <= 3e-2 * max |o|.
They come from the arithmetic: the expert GEMMs take bf16 operands (d_out * w and the
activation's gradient are rounded once to bf16, relative error 2^-9 each, and the forward's
h and y carry the same bf16 roundings), accumulate in fp32, and add at most a few thousand
terms; the router's gradients are fp32 throughout but inherit y's rounding through
dw = <d_out, y>.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import sparse_mixture_experts_11_b200 as moe
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

MEAN_REL = 1e-2
MAX_ABS_FRAC = 3e-2

# (name, T, d, N, k, F, act, capacity_factor, zipf)
CASES = [
    ("swiglu_top2_drops_bias", 200, 128, 8, 2, 128, "swiglu", 1.0, 1.1),
    ("gelu_top1_ragged_tiles", 300, 192, 4, 1, 320, "gelu", 1.25, None),
    ("swiglu_many_experts_k4", 96, 128, 64, 4, 128, "swiglu", 1.25, 1.1),
    ("gpt_oss_dims_two_experts", 24, 2880, 2, 1, 2880, "swiglu", None, None),
    ("multi_m_tile_experts", 700, 256, 4, 2, 256, "swiglu", None, None),
    ("single_token", 1, 256, 8, 2, 256, "gelu", None, None),
]


def _run(T, d, N, k, F, act, cap, zipf, seed=7):
    inp = synthetic.make_custom_inputs(T, d, N, F, act, seed=seed, device="cuda", zipf_s=zipf)
    dims = moe.make_dims(T, d, N, k, F, act, cap)
    fws = moe.new_workspace(dims, forward=True)
    out = torch.empty_like(inp["x"])
    moe.forward_into(dims, inp["x"], inp["w_router"], inp["logit_bias"], inp["w_gate_up"],
                     inp["w_down"], inp["x"], out, fws)
    g = synthetic.make_grad_output(T, d, seed=seed, device="cuda")
    rows = 2 * F if act == "swiglu" else F
    grads = {"dx": torch.empty((T, d), dtype=torch.float32, device="cuda"),
             "d_w_router": torch.empty((N, d), dtype=torch.float32, device="cuda"),
             "d_logit_bias": torch.empty((N,), dtype=torch.float32, device="cuda"),
             "d_w_gate_up": torch.full((N, rows, d), float("nan"), dtype=torch.float32, device="cuda"),
             "d_w_down": torch.full((N, d, F), float("nan"), dtype=torch.float32, device="cuda")}
    bws = moe.new_backward_workspace(dims)
    moe.backward_into(dims, inp["x"], inp["w_router"], inp["w_gate_up"], inp["w_down"], fws, g,
                      grads["dx"], grads["d_w_router"], grads["d_logit_bias"], grads["d_w_gate_up"],
                      grads["d_w_down"], bws)
    torch.cuda.synchronize()
    assert moe.read_device_error(bws) == 0
    b = moe.forward_layout(dims, fws)
    logits = fws[b.logits - fws.data_ptr():][: T * N * 4].view(torch.float32).view(T, N)
    return inp, dims, g, grads, logits


def _compare(name, got, want):
    g = H.f64(got)
    err = np.abs(g - want)
    den = np.abs(want).sum()
    mean_rel = err.sum() / den if den > 0 else err.sum()
    scale = np.abs(want).max()
    assert np.isfinite(g).all(), f"{name}: non-finite values"
    assert mean_rel <= MEAN_REL, f"{name}: mean-rel {mean_rel}"
    assert err.max() <= MAX_ABS_FRAC * scale + 1e-12, f"{name}: max-abs {err.max()} vs scale {scale}"
    return float(mean_rel)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_backward_matches_oracle(case):
    name, T, d, N, k, F, act, cf, zipf = case
    cap = oracle.capacity_from_factor(cf, T, N)
    inp, dims, g, grads, logits = _run(T, d, N, k, F, act, cap, zipf)
    bias = inp["logit_bias"]
    want = oracle.moe_layer_backward(
        H.f64(inp["x"]), H.f64(inp["w_router"]), H.f64(inp["w_gate_up"]), H.f64(inp["w_down"]),
        H.f64(g), top_k=k, act=act, capacity=cap,
        logit_bias=None if bias is None else H.f64(bias), logits=H.f64(logits))
    for key in ("dx", "d_w_router", "d_logit_bias", "d_w_gate_up", "d_w_down"):
        _compare(key, grads[key], want[key])
    # experts with no kept rows get exact zeros
    counts = np.diff(want["expert_offset"])
    for e in np.nonzero(counts == 0)[0]:
        assert torch.count_nonzero(grads["d_w_gate_up"][int(e)]) == 0
        assert torch.count_nonzero(grads["d_w_down"][int(e)]) == 0


def test_backward_zero_capacity_gives_zero_gradients():
    T, d, N, k, F = 32, 128, 8, 2, 128
    inp, dims, g, grads, logits = _run(T, d, N, k, F, "swiglu", 0, None)
    for key, t in grads.items():
        assert torch.count_nonzero(t) == 0, key


def test_backward_is_deterministic():
    T, d, N, k, F = 300, 192, 8, 2, 256
    cap = oracle.capacity_from_factor(1.25, T, N)
    _, _, _, a, _ = _run(T, d, N, k, F, "swiglu", cap, 1.1, seed=3)
    _, _, _, b, _ = _run(T, d, N, k, F, "swiglu", cap, 1.1, seed=3)
    for key in a:
        assert torch.equal(a[key], b[key]), key
