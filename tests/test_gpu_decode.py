"""The decode path (at most 8 tokens, SwiGLU): the one-launch decode router with the sort by
expert, the grouped FFN with every expert's weights cut along d_ff over all SMs (stream-K, fp32
partials added in a fixed order), the combine (GPU).

Checked against the CPU oracle on the GPU's own logits, and moe_forward against the four stage
calls bit for bit (routing, permutation, h, y_perm and the output)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

# (T, d, N, k, F, capacity (None: no limit), zipf, residual)
CASES = [
    (1, 2880, 32, 4, 2880, None, None, True),     # gpt-oss-shaped token, d not a multiple of 128
    (8, 512, 2, 2, 512, None, None, True),        # both experts hold exactly 8 rows
    (8, 256, 8, 2, 320, 1, 1.1, True),            # capacity 1: most pairs dropped, skewed loads
    (6, 320, 6, 3, 64, 2, None, False),           # d_ff of one k block, no residual
    (4, 1024, 64, 8, 2048, None, 1.1, True),      # many experts
    (7, 192, 5, 5, 128, None, None, True),        # k = N: every expert active
]


def _ids(c):
    return f"T{c[0]}_d{c[1]}_N{c[2]}_k{c[3]}_F{c[4]}_cap{c[5]}_res{int(c[7])}"


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_decode_stage_parity(case):
    T, d, N, k, F, cap, zipf, residual = case
    inp = synthetic.make_custom_inputs(T, d, N, F, "swiglu", seed=13, device="cuda", zipf_s=zipf)
    cap = T if cap is None else cap
    run = H.StageRun(inp, k, "swiglu", cap).run(residual=residual)
    routing, off, rop = H.check_routing(run, cap)
    H.check_x_perm(run, rop)
    R = int(off[-1])
    if R:
        H.check_expert_rows(run, routing, "swiglu", np.arange(R))  # every row
    H.check_outputs(run, routing, "swiglu", residual=residual)
    H.check_dropped_tokens_pass_through(run, routing["slot"], residual=residual)
    # h: the activation of every kept row, rounded once to bf16
    x = H.f64(inp["x"])
    por = run.pair_of_row.cpu().numpy()
    h = H.f64(run.h[:R]) if R else np.zeros((0, F))
    for r in range(R):
        e = int(np.searchsorted(off, r, side="right") - 1)
        w = H.f64(inp["w_gate_up"][e])
        xr = x[int(por[r]) // k][None, :]
        want = (oracle.silu(xr @ w[:F].T) * (xr @ w[F:].T))[0]
        # one bf16 ulp: fp32 rounding of g and u can move the value across a rounding midpoint
        bound = 1e-3 + H.bf16_half_ulp(want) * 2.02
        assert (np.abs(h[r] - want) <= bound).all(), (r, float(np.abs(h[r] - want).max()))


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_decode_forward_matches_stages(case):
    """Every buffer moe_forward writes equals the stage calls' bit for bit, on two calls in a row
    (the counters return to zero)."""
    import sparse_mixture_experts_11_b200 as moe
    T, d, N, k, F, cap, zipf, residual = case
    inp = synthetic.make_custom_inputs(T, d, N, F, "swiglu", seed=17, device="cuda", zipf_s=zipf)
    cap = T if cap is None else cap
    run = H.StageRun(inp, k, "swiglu", cap).run(residual=residual)
    ws = moe.new_workspace(run.dims, forward=True)
    b = moe.forward_layout(run.dims, ws)
    out = torch.empty_like(inp["x"])
    R = int(run.expert_offset[-1].item())
    view = lambda ptr, n, dt: ws[ptr - ws.data_ptr():][: n * torch.empty((), dtype=dt).element_size()].view(dt)
    for _ in range(2):
        out.fill_(0)
        moe.forward_into(run.dims, inp["x"], inp["w_router"], inp["logit_bias"], inp["w_gate_up"],
                         inp["w_down"], inp["x"] if residual else None, out, ws)
        torch.cuda.synchronize()
        assert moe.read_device_error(ws, offset_bytes=b.stage_ws - ws.data_ptr()) == moe.OK
        assert torch.equal(out.view(torch.int16), run.out.view(torch.int16))
        assert torch.equal(view(b.topk_idx, T * k, torch.int32), run.topk_idx.flatten())
        assert torch.equal(view(b.slot, T * k, torch.int32), run.slot.flatten())
        assert torch.equal(view(b.row_of_pair, T * k, torch.int32), run.row_of_pair.flatten())
        assert torch.equal(view(b.y_perm, R * d, torch.float32), run.y_perm[:R].flatten())
        assert torch.equal(view(b.h, R * F, torch.bfloat16).view(torch.int16),
                           run.h[:R].flatten().view(torch.int16))
