"""Parity at the benchmark's full sizes, in the launch configuration bench.py times (each
stage captured as a CUDA graph and replayed) (GPU).

* Routing is checked in full against the oracle re-run on the GPU's own logits; logits on
  sampled tokens against the oracle's router.
* Every expert with kept rows is checked: its weights are read back in float64 one expert at
  a time, and at least 8 of its y_perm rows (all of them when it has fewer) are compared with
  the oracle's expert FFN. The rows include the first and the last rows of the first two
  m-tiles at both tile heights the kernel uses (64 and 128 rows) and the expert's last rows,
  which lie in its partial last m-tile, the tile stream-K splits.
* Token outputs are checked on sampled tokens (a token's output depends only on its own kept
  pairs): the oracle's combine runs once per expert on the routing restricted to that expert,
  and the per-expert sums are added to the residual. The bf16 output (the product) and the
  fp32-output mode of moe_unpermute_combine (strict bar) are both compared, and so is the MoE
  contribution alone, out - residual, relative to its own size.
* Fully dropped tokens must pass the residual through bit for bit.
"""
import numpy as np
import pytest
import torch

import bench
import oracle
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

WORKLOADS = ["tiny_top2:64", "switch_top1:4096", "mixtral:1", "mixtral:16", "mixtral:512",
             "mixtral:8192", "gpt_oss:1", "gpt_oss:8", "gpt_oss:64", "gpt_oss:16384",
             "fine_grained:16384"]
SAMPLED_TOKENS = 48


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


def _rows_to_check(n: int, rng) -> list:
    """Local rows of an expert with n rows: both ends of the first two m-tiles at 64 and 128
    rows per tile, the middle, the expert's last rows (its partial last tile), two random."""
    if n <= 8:
        return list(range(n))
    cand = {0, 1, 63, 64, 127, 128, 191, 255, 256, n // 2, n - 33, n - 32, n - 2, n - 1}
    cand = {c for c in cand if 0 <= c < n}
    cand |= {int(v) for v in rng.integers(0, n, size=2)}
    while len(cand) < 8:
        cand.add(int(rng.integers(0, n)))
    return sorted(cand)


def _only_expert(r: dict, e: int) -> dict:
    """The routing with every pair not served by expert e marked dropped."""
    out = dict(r)
    out["slot"] = np.where(r["topk_idx"] == e, r["slot"], -1)
    return out


@pytest.mark.parametrize("spec", WORKLOADS)
def test_full_size_parity(spec):
    import sparse_mixture_experts_11_b200 as moe
    shape, T, layer = _replay_forward(spec)
    v = layer.views()
    err = moe.read_device_error(v["stage_ws"])
    assert err == 0, moe.status_string(err)
    inp = layer.inp
    cap = layer.dims.capacity
    k = shape.top_k
    rng = np.random.default_rng(1)

    # logits on sampled tokens (fp64 oracle on exactly the GPU's inputs)
    rows = np.unique(rng.integers(0, T, size=min(T, 256)))
    L = H.f64(v["logits"])
    bias = None if inp["logit_bias"] is None else H.f64(inp["logit_bias"])
    want_L = oracle.router_logits(H.f64(inp["x"][torch.from_numpy(rows).cuda()]), H.f64(inp["w_router"]), bias)
    bad = np.abs(L[rows] - want_L) > H.LOGIT_RTOL * np.maximum(1.0, np.abs(want_L))
    assert not bad.any(), f"{bad.sum()} logits off"

    # routing in full, bit-exact against the oracle re-run on the GPU's logits
    r = oracle.route_from_logits(L, k, cap)
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
    tok = np.repeat(np.arange(T), k).reshape(T, k)
    a = v["x_perm"].index_select(0, torch.from_numpy(rop[kept]).long().cuda()).view(torch.int16)
    b = inp["x"].index_select(0, torch.from_numpy(tok[kept]).long().cuda()).view(torch.int16)
    assert torch.equal(a, b)

    # tokens with every choice dropped keep the residual's bits
    all_dropped = np.all(r["slot"] < 0, axis=1)
    if all_dropped.any():
        idx = torch.from_numpy(np.nonzero(all_dropped)[0]).long().cuda()
        assert torch.equal(layer.out.index_select(0, idx).view(torch.int16),
                           inp["x"].index_select(0, idx).view(torch.int16))

    # fp32-output mode of the combine on the same expert rows (the verification mode)
    out32 = torch.empty((T, shape.d_model), dtype=torch.float32, device="cuda")
    moe.unpermute_combine(layer.dims, v["y_perm"], v["row_of_pair"], v["topk_w"], inp["x"], out32,
                          v["stage_ws"])
    torch.cuda.synchronize()

    # sampled tokens: random ones, plus partly dropped ones when there are any
    toks = set(int(t) for t in rng.choice(T, size=min(T, SAMPLED_TOKENS), replace=False))
    partly = np.nonzero(np.any(r["slot"] < 0, axis=1) & ~all_dropped)[0]
    toks |= set(int(t) for t in partly[:8])
    toks = np.array(sorted(toks), dtype=np.int64)

    # every expert with kept rows: sampled y_perm rows, and its share of the sampled outputs
    x = H.f64(inp["x"])
    contrib = np.zeros((toks.shape[0], shape.d_model))
    checked_rows = 0
    experts_checked = 0
    rows_required = 0
    for e in range(shape.n_experts):
        n = int(off[e + 1] - off[e])
        if n == 0:
            continue
        gu = H.f64(inp["w_gate_up"][e])
        dn = H.f64(inp["w_down"][e])
        local = _rows_to_check(n, rng)
        glob = [int(off[e]) + i for i in local]
        y = H.f64(v["y_perm"][torch.tensor(glob, dtype=torch.long, device="cuda")])
        src = [int(por[g]) // k for g in glob]
        want_y = oracle.expert_ffn(x[src], gu, dn, shape.act)
        for m, g in enumerate(glob):
            err_row = np.abs(y[m] - want_y[m])
            assert err_row.max() <= H.y_row_max_abs(want_y[m]), \
                f"expert {e} row {g - int(off[e])} of {n}: max-abs {err_row.max()}"
            assert H.mean_rel(y[m], want_y[m]) <= H.OUT_MEAN_REL, f"expert {e} row {g - int(off[e])}"
        checked_rows += len(glob)
        rows_required += min(n, 8)
        experts_checked += 1
        contrib += oracle.combine(x, _only_expert(r, e), lambda _: gu, lambda _: dn, shape.act,
                                  None, toks)
        del gu, dn
    assert experts_checked == int((r["expert_count"] > 0).sum())
    assert checked_rows >= rows_required

    want = x[toks] + contrib
    sel = torch.from_numpy(toks).cuda()
    g16 = H.f64(layer.out[sel])
    bound = H.OUT_MAX_ABS + H.bf16_half_ulp(want)
    assert (np.abs(g16 - want) <= bound).all(), float((np.abs(g16 - want) - bound).max())
    assert H.mean_rel(g16, want) <= H.OUT_MEAN_REL
    g32 = H.f64(out32[sel])
    assert np.abs(g32 - want).max() <= H.OUT_MAX_ABS, float(np.abs(g32 - want).max())
    assert H.mean_rel(g32, want) <= H.OUT_MEAN_REL
    if np.abs(contrib).sum() > 0:
        assert H.mean_rel(g32 - x[toks], contrib) <= H.OUT_MEAN_REL, \
            f"contribution mean-rel {H.mean_rel(g32 - x[toks], contrib)}"
