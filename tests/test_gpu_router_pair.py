"""The tensor-core router on CTA pairs (GPU).

With a workspace, when every 128-token tile has a CTA of its own, the tiles pair up and the
router has at least 128 padded expert columns, moe_route runs the router kernel on CTA pairs:
the even CTA of a pair issues M = 256 MMAs over both CTAs' token tiles, and each CTA holds
half of the rows of every weight term tile. moe_route_noalloc (terms split in the kernel)
never pairs. Both use the same three bf16 terms in the same MMA order, so the logits must be
identical bit for bit. Against the oracle: fp64 logits on sampled tokens (first and last
tile included) and the routing re-run on the GPU's own logits.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests import gpu_helpers as H
from tests.test_zz_no_alloc import _route_both

pytestmark = pytest.mark.gpu

# T, d, N, k, capacity, zipf: 76 tiles (the last one ragged), 96 tiles; padded N = 256 with
# N = 256 and N = 200 (the odd CTA's term rows past N are zero), padded N = 128
CASES = [(9700, 512, 256, 8, 380, 1.1),
         (9728, 384, 200, 4, 240, None),
         (12288, 256, 128, 4, 400, 1.1)]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"T{c[0]}_N{c[2]}")
def test_pair_router_matches_unpaired_and_oracle(case):
    T, d, N, k, cap, zipf = case
    assert (T + 127) // 128 % 2 == 0 and (T + 127) // 128 * 2 > 148  # the paired shape
    ref, got = _route_both(T, d, N, k, cap, 5, zipf)
    assert torch.equal(ref["logits"].view(torch.int32), got["logits"].view(torch.int32))
    for key in ("topk_idx", "topk_w", "slot", "expert_count"):
        assert torch.equal(ref[key], got[key]), key

    inp = synthetic.make_custom_inputs(T, d, N, 64, "swiglu", seed=5, device="cuda", zipf_s=zipf)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([np.arange(4), np.arange(T - 4, T), np.arange(124, 132),
                                     rng.choice(T, 48, replace=False)]))
    bias = inp.get("logit_bias")
    H.check_logits(H.f64(ref["logits"]), H.f64(inp["x"]), H.f64(inp["w_router"]),
                   None if bias is None else H.f64(bias), rows=rows)
    r = oracle.route_from_logits(H.f64(ref["logits"]), k, cap)
    assert np.array_equal(ref["topk_idx"].cpu().numpy(), r["topk_idx"])
    np.testing.assert_allclose(H.f64(ref["topk_w"]), r["topk_w"], rtol=0, atol=H.WEIGHT_ATOL)
    assert np.array_equal(ref["slot"].cpu().numpy(), r["slot"])
    assert np.array_equal(ref["expert_count"].cpu().numpy(), r["expert_count"])
