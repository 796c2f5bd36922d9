"""Parity of the CUDA path with the CPU oracle on small and ragged shapes (GPU)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

# (name, T, d, N, k, F, act, capacity_factor, zipf)
SMALL_CASES = [
    ("tiny_top2_cfg", 64, 128, 8, 2, 256, "swiglu", 1.25, None),
    ("ragged_multi_mtile", 600, 192, 4, 2, 320, "swiglu", None, None),
    ("gelu_switch_small", 512, 256, 16, 1, 512, "gelu", 1.0, None),
    ("gelu_ragged_n", 300, 320, 5, 3, 192, "gelu", 1.25, None),
    ("many_experts_k8", 96, 128, 256, 8, 128, "swiglu", 1.25, 1.1),
    ("gpt_oss_dims_small_T", 64, 2880, 32, 4, 2880, "swiglu", None, None),
    ("single_token", 1, 256, 8, 2, 256, "swiglu", None, None),
    ("k_equals_n", 40, 64, 4, 4, 64, "swiglu", None, None),
    ("heavy_drop", 200, 128, 8, 2, 128, "swiglu", 0.25, 1.1),
    # decode-sized batches whose GEMMs split K across CTAs (last split adds the partials)
    ("splitk_decode_swiglu", 3, 512, 8, 2, 1024, "swiglu", None, None),
    ("splitk_decode_gelu", 5, 256, 16, 1, 2048, "gelu", None, None),
    ("splitk_decode_deep_k", 2, 4096, 8, 2, 2048, "swiglu", None, None),
    ("splitk_decode_ragged_n", 7, 2880, 32, 4, 2880, "swiglu", None, None),
    # at most two rows per expert, GELU and both tokens in both experts
    ("gemv_decode_gelu", 2, 384, 16, 2, 1088, "gelu", None, None),
    ("gemv_two_rows_per_expert", 2, 576, 2, 2, 768, "swiglu", None, None),
    # large enough that the router runs on tensor cores (T*N*d*4 bytes > 256 MiB);
    # expert counts padded to 16, 32, 64, 128 (N=100) and 256 tensor-core columns
    ("tc_router_n8_bias", 20000, 512, 8, 2, 128, "swiglu", 1.25, 1.1),
    ("tc_router_n32_ragged_T", 2200, 1024, 32, 4, 128, "swiglu", None, None),
    ("tc_router_n64_gelu", 3000, 512, 64, 2, 256, "gelu", 1.0, None),
    ("tc_router_n100", 2700, 256, 100, 3, 128, "swiglu", 1.25, None),
    ("tc_router_n256_k8", 1100, 256, 256, 8, 64, "swiglu", 1.25, 1.1),
]


def _inputs(T, d, N, F, act, zipf, seed=0):
    inp = synthetic.make_custom_inputs(T, d, N, F, act, seed=seed, device="cuda", zipf_s=zipf)
    return inp


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: c[0])
def test_stage_parity(case):
    name, T, d, N, k, F, act, cf, zipf = case
    inp = _inputs(T, d, N, F, act, zipf)
    cap = oracle.capacity_from_factor(cf, T, N)
    run = H.StageRun(inp, k, act, cap).run()
    H.check_logits(H.f64(run.logits), H.f64(inp["x"]), H.f64(inp["w_router"]),
                   None if inp["logit_bias"] is None else H.f64(inp["logit_bias"]))
    routing, off, rop = H.check_routing(run, cap)
    H.check_x_perm(run, rop)
    R = int(off[-1])
    if R:
        H.check_expert_rows(run, routing, act, np.unique(np.linspace(0, R - 1, min(R, 24)).astype(np.int64)))
    H.check_outputs(run, routing, act)
    H.check_dropped_tokens_pass_through(run, routing["slot"])


def test_no_residual_and_zero_capacity():
    T, d, N, k, F = 48, 128, 8, 2, 128
    inp = _inputs(T, d, N, F, "swiglu", None, seed=3)
    run = H.StageRun(inp, k, "swiglu", 0).run(residual=True)
    routing, off, _ = H.check_routing(run, 0)
    assert int(off[-1]) == 0
    assert torch.equal(run.out.view(torch.int16), inp["x"].view(torch.int16))
    run = H.StageRun(inp, k, "swiglu", T).run(residual=False)
    routing, _, _ = H.check_routing(run, T)
    H.check_outputs(run, routing, "swiglu", residual=False)


def _route_logits(L, k, cap):
    import sparse_mixture_experts_11_b200 as moe
    T, N = L.shape
    dims = moe.make_dims(T, 64, N, k, 64, "swiglu", cap)
    ws = moe.new_workspace(dims)
    lg = torch.from_numpy(L).cuda()
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    slot = torch.empty((T, k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((N,), dtype=torch.int32, device="cuda")
    moe.route_from_logits(dims, lg, idx, w, slot, cnt, ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy(), slot.cpu().numpy(), cnt.cpu().numpy()


def test_route_from_logits_hand_case():
    """The hand-worked case (a tie, drops at capacity 1) straight against its written values."""
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_case_top2_cap1.json")))
    idx, w, slot, cnt = _route_logits(np.array(g["logits"], np.float32), g["top_k"], g["capacity"])
    assert idx.tolist() == g["topk_idx"]
    assert slot.tolist() == g["slot"]
    assert cnt.tolist() == g["expert_count"]
    np.testing.assert_allclose(w, np.array(g["topk_w"]), atol=H.WEIGHT_ATOL, rtol=0)


@pytest.mark.parametrize("T,N,k", [(50, 8, 2), (33, 64, 4), (70, 256, 8), (9000, 16, 3), (20000, 8, 8)])
def test_route_from_logits_ties(T, N, k):
    """Crafted logits with many exact ties; several capacity-scan chunks for the large cases."""
    rng = np.random.default_rng(T + N + k)
    L = rng.integers(-3, 4, size=(T, N)).astype(np.float32) * 0.5
    cap = int(np.ceil(1.0 * T / N))
    idx, w, slot, cnt = _route_logits(L, k, cap)
    r = oracle.route_from_logits(L.astype(np.float64), k, cap)
    assert np.array_equal(idx, r["topk_idx"])
    assert np.array_equal(slot, r["slot"])
    assert np.array_equal(cnt, r["expert_count"])
    np.testing.assert_allclose(w, r["topk_w"], atol=H.WEIGHT_ATOL, rtol=0)


def test_forward_matches_stages_bitwise():
    """moe_forward (one call) and the four stage calls produce identical bits."""
    import sparse_mixture_experts_11_b200 as moe
    T, d, N, k, F = 300, 192, 8, 2, 320
    inp = _inputs(T, d, N, F, "swiglu", None, seed=5)
    cap = oracle.capacity_from_factor(1.25, T, N)
    run = H.StageRun(inp, k, "swiglu", cap).run()
    dims = run.dims
    ws = moe.new_workspace(dims, forward=True)
    out = torch.empty_like(inp["x"])
    for _ in range(2):
        moe.forward_into(dims, inp["x"], inp["w_router"], None, inp["w_gate_up"], inp["w_down"],
                         inp["x"], out, ws)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), run.out.view(torch.int16))


def test_repeat_runs_are_bitwise_identical():
    T, d, N, k, F = 700, 256, 16, 2, 256
    inp = _inputs(T, d, N, F, "swiglu", 1.1, seed=9)
    cap = oracle.capacity_from_factor(1.0, T, N)
    a = H.StageRun(inp, k, "swiglu", cap).run()
    o1 = a.out.clone()
    y1 = a.y_perm.clone()
    a.run()
    assert torch.equal(o1.view(torch.int16), a.out.view(torch.int16))
    assert torch.equal(y1, a.y_perm)


def test_empty_batch_is_a_no_op():
    import sparse_mixture_experts_11_b200 as moe
    dims = moe.make_dims(0, 128, 8, 2, 128, "swiglu", 0)
    ws = moe.new_workspace(dims, forward=True)
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros((8, 128), dtype=torch.float32, device="cuda")
    wgu = torch.zeros((8, 256, 128), dtype=torch.bfloat16, device="cuda")
    wd = torch.zeros((8, 128, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    moe.forward_into(dims, x, wr, None, wgu, wd, x, out, ws)
    torch.cuda.synchronize()


def test_k_scaled_capacity():
    """Overflow-policy variant: capacity scaled by k, ceil(cf * k * T / N), passed through the
    capacity field (fine-grained-like shape: N=256, k=8, Zipf-skewed loads)."""
    import math
    T, d, N, k, F = 600, 256, 256, 8, 128
    inp = _inputs(T, d, N, F, "swiglu", 1.1, seed=21)
    cap = int(math.ceil(1.25 * k * T / N))
    run = H.StageRun(inp, k, "swiglu", cap).run()
    routing, off, rop = H.check_routing(run, cap)
    H.check_x_perm(run, rop)
    H.check_outputs(run, routing, "swiglu")
    H.check_dropped_tokens_pass_through(run, routing["slot"])
    assert int((routing["slot"] < 0).sum()) > 0  # the Zipf skew still overflows hot experts


# Decode-sized batches route in one launch (router split over d across CTAs; the last CTA
# adds the partial dot products, takes top-k and the capacity slots) and, in moe_forward,
# also sort by expert while x_perm is at most 512 KB.
# (T, d, N, k, F, act, capacity_factor, zipf)
DECODE_CASES = [
    (1, 2880, 32, 4, 256, "swiglu", None, None),
    (16, 512, 256, 8, 128, "swiglu", 1.25, 1.1),
    (16, 7168, 8, 2, 128, "gelu", None, None),
    (12, 4096, 64, 8, 128, "swiglu", 0.5, 1.1),  # x_perm 768 KB: separate permute launch
    (5, 320, 100, 3, 192, "gelu", 1.0, None),
    (2, 64, 4, 4, 64, "swiglu", None, None),     # one d slice, k = N
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: f"T{c[0]}_d{c[1]}_N{c[2]}_k{c[3]}")
def test_decode_route_and_forward(case):
    import sparse_mixture_experts_11_b200 as moe
    T, d, N, k, F, act, cf, zipf = case
    inp = _inputs(T, d, N, F, act, zipf, seed=31)
    cap = oracle.capacity_from_factor(cf, T, N)
    run = H.StageRun(inp, k, act, cap).run()
    H.check_logits(H.f64(run.logits), H.f64(inp["x"]), H.f64(inp["w_router"]),
                   None if inp["logit_bias"] is None else H.f64(inp["logit_bias"]))
    routing, off, rop = H.check_routing(run, cap)
    H.check_x_perm(run, rop)
    H.check_outputs(run, routing, act)
    H.check_dropped_tokens_pass_through(run, routing["slot"])
    ws = moe.new_workspace(run.dims, forward=True)
    out = torch.empty_like(inp["x"])
    for _ in range(2):  # the arrival counter is back at zero after each call
        out.fill_(0)
        moe.forward_into(run.dims, inp["x"], inp["w_router"], inp["logit_bias"], inp["w_gate_up"],
                         inp["w_down"], inp["x"], out, ws)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), run.out.view(torch.int16))


# Overflow policy "redirect": pairs at a full expert go to the token's next most suitable
# expert with a free slot (the oracle re-run on the GPU's own logits decides every pair).
def _redirect_logits(L, k, cap):
    import sparse_mixture_experts_11_b200 as moe
    T, N = L.shape
    dims = moe.make_dims(T, 64, N, k, 64, "swiglu", cap)
    ws = moe.new_workspace(dims)
    lg = torch.from_numpy(L).cuda()
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    slot = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    moe.route_from_logits(dims, lg, idx, w, slot, cnt, ws)
    moe.redirect_overflow(dims, lg, idx, slot, cnt, ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy(), slot.cpu().numpy(), cnt.cpu().numpy()


def test_redirect_hand_case():
    """Worked by hand: one slot per expert, top-1. Token 0 keeps expert 0; token 1 prefers 0
    (full), then 2 (logit 2 > 1); token 2 prefers 0 (full), then 1 (2 > 1, expert 2 full)."""
    L = np.array([[3, 1, 2], [3, 1, 2], [3, 2, 1]], np.float32)
    idx, w, slot, cnt = _redirect_logits(L, 1, 1)
    assert idx.tolist() == [[0], [2], [1]]
    assert slot.tolist() == [[0], [0], [0]]
    assert cnt.tolist() == [1, 1, 1]
    np.testing.assert_allclose(w, np.ones((3, 1)), atol=H.WEIGHT_ATOL, rtol=0)


@pytest.mark.parametrize("T,N,k,cf", [(50, 8, 2, 1.0), (33, 64, 4, 0.5), (70, 256, 8, 1.0),
                                      (2000, 16, 3, 1.0), (4096, 256, 8, 0.75), (4096, 256, 8, 8.0),
                                      (300, 4, 4, 0.5),
                                      (64, 8, 2, 0.0),
                                      (16384, 256, 8, 1.25), (20480, 256, 8, 40.0)])
def test_redirect_ties(T, N, k, cf):
    """Crafted logits with many exact ties. (16384, 256, 8): the fine-grained layer's 131072
    pairs; (20480, 256, 8) with room for every pair: 163840 pairs, the largest supported batch,
    walked to its end."""
    rng = np.random.default_rng(7 * T + N + k)
    L = rng.integers(-3, 4, size=(T, N)).astype(np.float32) * 0.5
    cap = oracle.capacity_from_factor(cf, T, N) if cf > 0 else 0
    idx, w, slot, cnt = _redirect_logits(L, k, cap)
    r = oracle.route_from_logits(L.astype(np.float64), k, cap, reroute=True)
    assert np.array_equal(idx, r["topk_idx"])
    assert np.array_equal(slot, r["slot"])
    assert np.array_equal(cnt, r["expert_count"])
    np.testing.assert_allclose(w, r["topk_w"], atol=H.WEIGHT_ATOL, rtol=0)


@pytest.mark.parametrize("T,d,N,k,F,act,cf,zipf", [
    (600, 256, 16, 2, 256, "swiglu", 1.0, 1.1),
    (200, 128, 8, 2, 128, "gelu", 0.5, 1.1),
    (96, 128, 256, 8, 128, "swiglu", 1.25, 1.1),
], ids=["switchlike_zipf", "gelu_heavy_overflow", "fine_grained_k8"])
def test_redirect_full_pipeline(T, d, N, k, F, act, cf, zipf):
    """route -> redirect -> permute -> grouped FFN -> combine against the oracle."""
    inp = _inputs(T, d, N, F, act, zipf, seed=41)
    cap = oracle.capacity_from_factor(cf, T, N)
    run = H.StageRun(inp, k, act, cap).run(redirect=True)
    routing, off, rop = H.check_routing(run, cap, reroute=True)
    H.check_x_perm(run, rop)
    H.check_outputs(run, routing, act)
    H.check_dropped_tokens_pass_through(run, routing["slot"])
    drop = oracle.route_from_logits(H.f64(run.logits), k, cap)
    # the policy keeps pairs that dropping loses
    assert int((routing["slot"] >= 0).sum()) > int((drop["slot"] >= 0).sum())


def test_redirect_switch_size_gaussian_logits():
    """The default switch-like batch (T=4096, N=64, top-1, capacity factor 1.0) with Gaussian
    logits skewed towards a few experts, as the router produces them."""
    rng = np.random.default_rng(11)
    T, N, k = 4096, 64, 1
    L = (rng.standard_normal((T, N)) + np.linspace(0.0, 1.5, N)[None, :]).astype(np.float32)
    cap = oracle.capacity_from_factor(1.0, T, N)
    idx, w, slot, cnt = _redirect_logits(L, k, cap)
    r = oracle.route_from_logits(L.astype(np.float64), k, cap, reroute=True)
    assert np.array_equal(idx, r["topk_idx"])
    assert np.array_equal(slot, r["slot"])
    assert np.array_equal(cnt, r["expert_count"])
    assert int((slot >= 0).sum()) == min(T * k, N * cap)  # nothing is dropped while room is left
