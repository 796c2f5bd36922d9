"""The CPU oracle against values it does not produce itself (CPU only)."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle)


def test_active_params_page_numbers():
    oracle_pins.pin_active_params_demo()


def test_against_torch_eager_loop_float64():
    """Independent cross-check: torch float64 softmax/topk and the pages' eager
    per-choice, per-expert loop, on tie-free inputs with no capacity limit."""
    rng = np.random.default_rng(11)
    for act in ("swiglu", "gelu"):
        T, d, N, F, k = 13, 8, 5, 6, 2
        x = rng.normal(size=(T, d))
        wr = rng.normal(size=(N, d)) / math.sqrt(d)
        rows = 2 * F if act == "swiglu" else F
        wgu = rng.normal(size=(N, rows, d)) * 0.2
        wd = rng.normal(size=(N, d, F)) * 0.2
        got = oracle.moe_layer_forward(x, wr, wgu, wd, top_k=k, act=act, capacity=T, residual=x)

        X = torch.from_numpy(x)
        probs = torch.softmax(X @ torch.from_numpy(wr).T, dim=-1)
        top_p, top_i = torch.topk(probs, k, dim=-1)
        top_p = top_p / top_p.sum(dim=-1, keepdim=True)
        out = X.clone()
        for j in range(k):
            for e in range(N):
                m = top_i[:, j] == e
                if not m.any():
                    continue
                W = torch.from_numpy(wgu[e])
                if act == "swiglu":
                    hh = torch.nn.functional.silu(X[m] @ W[:F].T) * (X[m] @ W[F:].T)
                else:
                    hh = torch.nn.functional.gelu(X[m] @ W.T)
                out[m] += top_p[m, j:j + 1] * (hh @ torch.from_numpy(wd[e]).T)
        assert got["topk_idx"].tolist() == top_i.tolist()
        np.testing.assert_allclose(got["topk_w"], top_p.numpy(), rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(got["out"], out.numpy(), rtol=1e-12, atol=1e-12)


def test_token_subset_matches_full():
    rng = np.random.default_rng(8)
    T, d, N, F = 30, 6, 4, 5
    x = rng.normal(size=(T, d))
    wr = rng.normal(size=(N, d))
    wgu = rng.normal(size=(N, 2 * F, d)) * 0.3
    wd = rng.normal(size=(N, d, F)) * 0.3
    full = oracle.moe_layer_forward(x, wr, wgu, wd, top_k=2, act="swiglu", capacity=9, residual=x)
    sub = np.array([29, 0, 17, 3])
    part = oracle.moe_layer_forward(x, wr, wgu, wd, top_k=2, act="swiglu", capacity=9,
                                    residual=x, tokens=sub)
    np.testing.assert_allclose(part["out"], full["out"][sub], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("pin", oracle_pins.MX_PINS, ids=lambda f: f.__name__)
def test_mx_pin(pin):
    pin(oracle.mx_oracle)
