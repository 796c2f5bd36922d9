"""Parity at the benchmark's full sizes, in the launch configuration bench.py times (each
stage captured as a CUDA graph and replayed). Routing is checked in full against the oracle
re-run on the GPU's own logits. Outputs are checked on sampled tokens: a token's output
depends only on its own kept pairs. Expert rows are checked on sampled rows, logits on
sampled tokens. Fully dropped tokens must pass the residual through bit for bit (GPU)."""
import numpy as np
import pytest
import torch

import bench
import oracle
import synthetic
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

WORKLOADS = ["tiny_top2:64", "switch_top1:4096", "mixtral:1", "mixtral:16", "mixtral:512",
             "mixtral:8192", "gpt_oss:1", "gpt_oss:8", "gpt_oss:64", "gpt_oss:16384",
             "fine_grained:16384"]


def _replay_forward(spec):
    shape, T = bench.parse_workload(spec)
    layer = bench.Layer(shape, T, torch.device("cuda"))
    for call in layer.stage_calls():
        call()
    torch.cuda.synchronize()
    layer.capture_stage_graphs()
    # the whole-forward graph (moe_forward) and the stage graphs give the same bits
    layer.out.fill_(0)
    layer.graph_full.replay()
    torch.cuda.synchronize()
    full = layer.out.clone()
    layer.out.fill_(0)
    for g in layer.graphs:
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(full.view(torch.int16), layer.out.view(torch.int16))
    return shape, T, layer


@pytest.mark.parametrize("spec", WORKLOADS)
def test_full_size_parity(spec):
    import sparse_mixture_experts_11_b200 as moe
    shape, T, layer = _replay_forward(spec)
    v = layer.views()
    err = moe.read_device_error(v["stage_ws"])
    assert err == 0, moe.status_string(err)
    inp = layer.inp
    cap = layer.dims.capacity
    rng = np.random.default_rng(1)

    # logits on sampled tokens (fp64 oracle on exactly the GPU's inputs)
    rows = np.unique(rng.integers(0, T, size=min(T, 256)))
    L = H.f64(v["logits"])
    bias = None if inp["logit_bias"] is None else H.f64(inp["logit_bias"])
    want_L = oracle.router_logits(H.f64(inp["x"][torch.from_numpy(rows).cuda()]), H.f64(inp["w_router"]), bias)
    bad = np.abs(L[rows] - want_L) > H.LOGIT_RTOL * np.maximum(1.0, np.abs(want_L))
    assert not bad.any(), f"{bad.sum()} logits off"

    # routing in full, bit-exact against the oracle re-run on the GPU's logits
    r = oracle.route_from_logits(L, shape.top_k, cap)
    assert np.array_equal(v["topk_idx"].cpu().numpy(), r["topk_idx"])
    np.testing.assert_allclose(H.f64(v["topk_w"]), r["topk_w"], rtol=0, atol=H.WEIGHT_ATOL)
    assert np.array_equal(v["slot"].cpu().numpy(), r["slot"])
    assert np.array_equal(v["expert_count"].cpu().numpy(), r["expert_count"])
    off, rop, por = oracle.expert_permutation(r["topk_idx"], r["slot"], r["expert_count"])
    assert np.array_equal(v["expert_offset"].cpu().numpy(), off)
    assert np.array_equal(v["row_of_pair"].cpu().numpy(), rop)
    R = int(off[-1])
    assert np.array_equal(v["pair_of_row"][:R].cpu().numpy(), por)

    # x_perm rows are bit copies of their tokens
    kept = rop >= 0
    tok = np.repeat(np.arange(T), shape.top_k).reshape(T, shape.top_k)
    a = v["x_perm"].index_select(0, torch.from_numpy(rop[kept]).long().cuda()).view(torch.int16)
    b = inp["x"].index_select(0, torch.from_numpy(tok[kept]).long().cuda()).view(torch.int16)
    assert torch.equal(a, b)

    # tokens with every choice dropped keep the residual's bits
    all_dropped = np.all(r["slot"] < 0, axis=1)
    if all_dropped.any():
        idx = torch.from_numpy(np.nonzero(all_dropped)[0]).long().cuda()
        assert torch.equal(layer.out.index_select(0, idx).view(torch.int16),
                           inp["x"].index_select(0, idx).view(torch.int16))

    # sampled tokens' outputs, touching a bounded number of experts (host fp64 copies)
    params = bench.expert_params(shape.d_model, shape.d_ff, shape.act)
    max_experts = int(max(2, min(16, 4e9 // (params * 8))))
    toks = H.sample_tokens(r, n=32, max_experts=max_experts)
    gu = H.expert_weights_f64(inp["w_gate_up"])
    dn = H.expert_weights_f64(inp["w_down"])
    x = H.f64(inp["x"])
    want = oracle.combine(x, r, gu, dn, shape.act, x, toks)
    got = H.f64(layer.out[torch.from_numpy(toks).cuda()])
    bound = H.OUT_MAX_ABS + H.bf16_half_ulp(want)
    assert (np.abs(got - want) <= bound).all(), float((np.abs(got - want) - bound).max())
    assert H.mean_rel(got, want) <= H.OUT_MEAN_REL

    # expert rows of the sampled tokens (fp32 y_perm against the oracle's expert FFN)
    y = H.f64(v["y_perm"])
    checked = 0
    for t in toks[:8]:
        for j in range(shape.top_k):
            row = rop[t, j]
            if row < 0:
                continue
            e = r["topk_idx"][t, j]
            want_y = oracle.expert_ffn(x[t:t + 1], gu(e), dn(e), shape.act)[0]
            assert np.abs(y[row] - want_y).max() <= H.OUT_MAX_ABS
            assert H.mean_rel(y[row], want_y) <= H.OUT_MEAN_REL
            checked += 1
    assert checked > 0 or R == 0
