"""moe_route_noalloc: routing for callers that cannot allocate device memory (GPU).

Some callers cannot call cudaMalloc. Examples: an engine that owns all device memory through
its own arena; a real-time loop where an allocation could synchronise the device or fail
mid-run; a plugin whose host framework controls every allocation. For them the library
offers moe_route_noalloc. It works like moe_route, but it takes its scratch from a fixed
array inside the library instead of a caller workspace.

This file checks the call through the C ABI against moe_route, the existing entry point.
It makes several calls in a row, with shapes of different sizes, because every call reuses
the same scratch and keeps the last call's contents. It also checks that a shape too large
for the scratch is refused before anything runs. The file is named so that pytest collects
it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import synthetic
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _buffers(T, N, k):
    dev = "cuda"
    return {"logits": torch.full((T, N), float("nan"), dtype=torch.float32, device=dev),
            "topk_idx": torch.full((T, k), -7, dtype=torch.int32, device=dev),
            "topk_w": torch.full((T, k), float("nan"), dtype=torch.float32, device=dev),
            "slot": torch.full((T, k), -7, dtype=torch.int32, device=dev),
            "expert_count": torch.full((N,), -7, dtype=torch.int32, device=dev)}


def _route_both(T, d, N, k, cap, seed, zipf=None):
    import sparse_mixture_experts_11_b200 as moe
    inp = synthetic.make_custom_inputs(T, d, N, 64, "swiglu", seed=seed, device="cuda", zipf_s=zipf)
    dims = moe.make_dims(T, d, N, k, 64, "swiglu", cap)
    ref = _buffers(T, N, k)
    ws = moe.new_workspace(dims)
    moe.route(dims, inp["x"], inp["w_router"], inp["logit_bias"], ref["logits"], ref["topk_idx"],
              ref["topk_w"], ref["slot"], ref["expert_count"], ws)
    got = _buffers(T, N, k)
    moe.route_noalloc(dims, inp["x"], inp["w_router"], inp["logit_bias"], got["logits"],
                      got["topk_idx"], got["topk_w"], got["slot"], got["expert_count"])
    torch.cuda.synchronize()
    return ref, got


def _assert_same_routing(ref, got):
    lr, lg = H.f64(ref["logits"]), H.f64(got["logits"])
    assert (np.abs(lg - lr) <= H.LOGIT_RTOL * np.maximum(1.0, np.abs(lr))).all()
    for key in ("topk_idx", "slot", "expert_count"):
        assert torch.equal(ref[key], got[key]), key
    np.testing.assert_allclose(H.f64(got["topk_w"]), H.f64(ref["topk_w"]), rtol=0, atol=H.WEIGHT_ATOL)


def test_noalloc_matches_route_on_consecutive_calls():
    # several capacity chunks each, so the built-in scratch is really used; the second shape
    # needs more scratch than the first, the third less than the second
    shapes = [(9000, 256, 64, 2, 160, 1, None),
              (4000, 128, 256, 8, 130, 2, 1.1),
              (9000, 256, 64, 2, 160, 1, None)]
    for T, d, N, k, cap, seed, zipf in shapes:
        ref, got = _route_both(T, d, N, k, cap, seed, zipf)
        _assert_same_routing(ref, got)
        assert int((ref["slot"] < 0).sum()) > 0  # drops happened, so the scan mattered


def test_noalloc_twice_in_a_row_small():
    for _ in range(2):
        ref, got = _route_both(64, 128, 8, 2, 10, 0)
        _assert_same_routing(ref, got)


def test_noalloc_refuses_shapes_beyond_its_scratch():
    import sparse_mixture_experts_11_b200 as moe
    # N = 256, T * k = 262145 pairs -> 65 chunks * 256 ints > 16384 ints of scratch
    dims = moe.make_dims(262145, 64, 256, 1, 64, "swiglu", 262145)
    P = ctypes.c_void_p
    r = moe._lib.moe_route_noalloc(ctypes.byref(dims), P(16), P(16), None, P(16), P(16), P(16),
                                   P(16), P(16), None)
    assert r == moe.ERR_WORKSPACE
    dims = moe.make_dims(262144, 64, 256, 1, 64, "swiglu", 262144)
    # the largest shape that fits passes the size check (and then fails on the null pointer)
    r = moe._lib.moe_route_noalloc(ctypes.byref(dims), None, P(16), None, P(16), P(16), P(16),
                                   P(16), P(16), None)
    assert r == moe.ERR_INVALID


@pytest.mark.parametrize("T,d,N,k,cap", [(1, 2880, 32, 4, 1), (16, 512, 256, 8, 1), (7, 4096, 8, 2, 2)])
def test_noalloc_matches_route_decode_sized(T, d, N, k, cap):
    """Decode-sized batches take the one-launch router in both calls (same partial sums)."""
    for _ in range(2):  # the static arrival counter is back at zero after each call
        ref, got = _route_both(T, d, N, k, cap, 3, 1.1)
        _assert_same_routing(ref, got)
        assert torch.equal(ref["logits"], got["logits"])


def test_noalloc_survives_a_timed_out_call():
    """This call has no status word, so a wait that runs out is not reported. With a limit far
    below the default, the tensor-core router (this shape's path) stops early; the context
    stays usable and the next call, with the default limit, matches moe_route again."""
    import sparse_mixture_experts_11_b200 as moe
    T, d, N, k, cap = 9000, 256, 64, 2, 160
    inp = synthetic.make_custom_inputs(T, d, N, 64, "swiglu", seed=1, device="cuda")
    dims = moe.make_dims(T, d, N, k, 64, "swiglu", cap)
    got = _buffers(T, N, k)
    old = moe.debug_set_wait_timeout_ns(1)
    try:
        moe.route_noalloc(dims, inp["x"], inp["w_router"], inp["logit_bias"], got["logits"],
                          got["topk_idx"], got["topk_w"], got["slot"], got["expert_count"])
        torch.cuda.synchronize()  # raises if the early stop had faulted
    finally:
        moe.debug_set_wait_timeout_ns(0)
    assert old == 2_000_000_000
    for _ in range(2):
        ref, got = _route_both(T, d, N, k, cap, 1)
        _assert_same_routing(ref, got)
