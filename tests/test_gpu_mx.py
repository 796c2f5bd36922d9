"""Parity of the grouped FFN with expert weights in the MX formats (MXFP8 E4M3, MXFP4 E2M1;
E8M0 block scales) against the oracle's float64 layer on the weights the oracle decodes from
the same bytes (GPU). The decode on the GPU is exact, so the bars are the bf16 path's."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

# (name, T, d, N, k, F, act, capacity_factor, fmt)
MX_CASES = [
    # decode-sized: stream-K over short partial tiles; ragged last gate/up n-tile (F = 320)
    ("decode_swiglu_fp4", 1, 512, 8, 2, 320, "swiglu", None, "mxfp4"),
    ("decode_swiglu_fp8", 3, 512, 8, 2, 320, "swiglu", None, "mxfp8"),
    ("decode_gelu_fp8", 5, 256, 16, 1, 512, "gelu", None, "mxfp8"),
    ("decode_gelu_fp4_deep_k", 2, 2048, 4, 2, 256, "gelu", None, "mxfp4"),
    # whole tiles, 64-row and 128-row tiles, several m-tiles per expert, drops
    ("prefill_swiglu_fp8", 300, 256, 4, 2, 320, "swiglu", 1.25, "mxfp8"),
    ("prefill_swiglu_fp4", 300, 256, 4, 2, 320, "swiglu", 1.25, "mxfp4"),
    ("prefill_gelu_fp4_bm64", 256, 192, 8, 1, 256, "gelu", 2.0, "mxfp4"),
    ("gpt_oss_dims_fp4", 4, 2880, 32, 4, 2880, "swiglu", None, "mxfp4"),
]


def _run(case, seed=0):
    name, T, d, N, k, F, act, cf, fmt = case
    inp = synthetic.make_mx_custom_inputs(T, d, N, F, act, fmt, seed=seed, device="cuda")
    cap = oracle.capacity_from_factor(cf, T, N)
    return H.StageRun(inp, k, act, cap).run(), cap, act


@pytest.mark.parametrize("case", MX_CASES, ids=lambda c: c[0])
def test_mx_stage_parity(case):
    run, cap, act = _run(case)
    routing, off, rop = H.check_routing(run, cap)
    H.check_x_perm(run, rop)
    R = int(off[-1])
    if R:
        H.check_expert_rows(run, routing, act, np.unique(np.linspace(0, R - 1, min(R, 16)).astype(np.int64)))
    H.check_outputs(run, routing, act)
    H.check_dropped_tokens_pass_through(run, routing["slot"])


@pytest.mark.parametrize("case", [MX_CASES[0], MX_CASES[4]], ids=lambda c: c[0])
def test_mx_forward_matches_stages_bitwise(case):
    import sparse_mixture_experts_11_b200 as moe
    run, cap, act = _run(case, seed=3)
    i = run.inp
    ws = moe.new_workspace(run.dims, forward=True)
    out = torch.empty_like(i["x"])
    for _ in range(2):
        out.fill_(0)
        moe.forward_mx_into(run.dims, i["x"], i["w_router"], i["logit_bias"], run.mx, i["x"], out, ws)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), run.out.view(torch.int16))


def test_mx_repeat_runs_are_bitwise_identical():
    run, cap, act = _run(MX_CASES[4], seed=5)
    y1, o1 = run.y_perm.clone(), run.out.clone()
    run.run()
    assert torch.equal(y1, run.y_perm)
    assert torch.equal(o1.view(torch.int16), run.out.view(torch.int16))


def test_mx_rejects_bad_format():
    import sparse_mixture_experts_11_b200 as moe
    run, cap, act = _run(MX_CASES[0])
    bad = moe.MxWeights(7, run.mx.gate_up, run.mx.gate_up_scales, run.mx.down, run.mx.down_scales)
    with pytest.raises(moe.MoeError):
        moe.grouped_ffn_mx(run.dims, run.x_perm, run.expert_offset, bad, run.h, run.y_perm, run.ws)
