"""Parity of the block-scaled MX formats (GPU): the MXFP8 / MXFP4 expert weights read by the
tcgen05 block-scaled MMA (kind::mxf8f6f4, E8M0 scale factors in TMEM), with the token rows
and h quantised to MXFP8 per 32 along K. Checked against the oracle's layer with the same
quantisation (oracle.expert_ffn_mxfp8_act) on the weights it decodes from the same bytes.

The rows' quantisation is exact on both sides (bf16 inputs); h is computed in fp32 on the GPU
and in float64 by the oracle, so an h element whose value sits at an E4M3 rounding boundary can
round the other way (one E4M3 step, at most 1/8 of the element): rare, and far inside the
bars below, which are the bf16 path's."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

# (name, T, d, N, k, F, act, capacity_factor, fmt)
BS_CASES = [
    # decode-sized: stream-K over short partial tiles; F = 320: a ragged last n-tile and a half k block
    ("bs8_decode_swiglu", 1, 512, 8, 2, 320, "swiglu", None, "mxfp8_bs"),
    ("bs4_decode_swiglu", 3, 512, 8, 2, 256, "swiglu", None, "mxfp4_bs"),
    ("bs8_decode_gelu", 5, 256, 16, 1, 512, "gelu", None, "mxfp8_bs"),
    # whole tiles, several m-tiles per expert, drops
    ("bs8_prefill_swiglu", 300, 256, 4, 2, 320, "swiglu", 1.25, "mxfp8_bs"),
    ("bs4_prefill_gelu", 256, 256, 8, 1, 256, "gelu", 2.0, "mxfp4_bs"),
    ("bs4_prefill_swiglu_deep_k", 200, 1024, 4, 2, 384, "swiglu", None, "mxfp4_bs"),
    # gpt_oss widths: d = F = 2880 is 22.5 k blocks of 128 in both GEMMs
    ("bs8_gpt_oss_dims", 4, 2880, 32, 4, 2880, "swiglu", None, "mxfp8_bs"),
]


def _run(case, seed=0):
    name, T, d, N, k, F, act, cf, fmt = case
    inp = synthetic.make_mx_custom_inputs(T, d, N, F, act, fmt, seed=seed, device="cuda")
    cap = oracle.capacity_from_factor(cf, T, N)
    return H.StageRun(inp, k, act, cap).run(), cap, act


@pytest.mark.parametrize("case", BS_CASES, ids=lambda c: c[0])
def test_block_scaled_stage_parity(case):
    run, cap, act = _run(case)
    routing, off, rop = H.check_routing(run, cap)
    H.check_x_perm(run, rop)
    R = int(off[-1])
    if R:
        H.check_expert_rows(run, routing, act, np.unique(np.linspace(0, R - 1, min(R, 16)).astype(np.int64)))
    H.check_outputs(run, routing, act)
    H.check_dropped_tokens_pass_through(run, routing["slot"])


def test_block_scaled_h_codes_match_oracle():
    """h as stored (E4M3 codes, bytes of the h buffer) against the oracle's quantisation of the
    rows' h: equal codes except at rare rounding boundaries (fp32 vs float64 activation)."""
    case = BS_CASES[3]
    run, cap, act = _run(case, seed=2)
    routing, off, rop = H.check_routing(run, cap)
    R, F = int(off[-1]), run.dims.d_ff
    por = run.pair_of_row.cpu().numpy()
    k = run.dims.top_k
    rows = np.unique(np.linspace(0, R - 1, min(R, 12)).astype(np.int64))
    hq = run.h.view(torch.uint8).view(-1)[: run.R_max * F].view(run.R_max, F)
    x = H.f64(run.inp["x"])
    mism = 0
    for r in rows:
        e = int(np.searchsorted(off, r, side="right") - 1)
        t = int(por[r]) // k
        xq = oracle.mxfp8_round_trip(x[t:t + 1])
        gu = run.gu(e)
        Fh = gu.shape[0] // 2
        h = oracle.silu(xq @ gu[:Fh].T) * (xq @ gu[Fh:].T)
        want, _ = oracle.quantize_mxfp8(h)
        got = hq[int(r)].cpu().numpy()
        mism += int((got != want[0]).sum())
    assert mism <= max(2, rows.size * F // 2000), f"{mism} h codes differ"


def test_block_scaled_forward_matches_stages_bitwise():
    import sparse_mixture_experts_11_b200 as moe
    run, cap, act = _run(BS_CASES[0], seed=3)
    i = run.inp
    ws = moe.new_workspace(run.dims, forward=True, block_scaled=True)
    out = torch.empty_like(i["x"])
    for _ in range(2):
        out.fill_(0)
        moe.forward_mx_into(run.dims, i["x"], i["w_router"], i["logit_bias"], run.mx, i["x"], out, ws)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), run.out.view(torch.int16))


def test_block_scaled_needs_its_workspace():
    import sparse_mixture_experts_11_b200 as moe
    run, cap, act = _run(BS_CASES[0])
    small = moe.new_workspace(run.dims)  # without the activation region
    with pytest.raises(moe.MoeError):
        moe.grouped_ffn_mx(run.dims, run.x_perm, run.expert_offset, run.mx, run.h, run.y_perm, small)
