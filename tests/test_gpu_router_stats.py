"""Router statistics and the auxiliary load-balancing loss on the GPU against the oracle (GPU).

The statistics are computed from the GPU's own logits and routing: integer counts must match
exactly, the mean probabilities and the loss to within fp32 summation error."""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_11_b200 as moe
import synthetic
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,N,k,cf,zipf", [(64, 8, 2, 1.25, None), (4096, 64, 1, 1.0, None),
                                           (16384, 256, 8, 1.25, 1.1), (1000, 100, 3, 0.5, None),
                                           (3, 4, 4, 1.0, None), (1, 8, 2, None, None)])
def test_router_stats_match_oracle(T, N, k, cf, zipf):
    g = torch.Generator(device="cuda")
    g.manual_seed(T * 7 + N)
    L = torch.randn((T, N), generator=g, device="cuda")
    if zipf is not None:
        L += synthetic.zipf_logit_bias(N, zipf).cuda()
    cap = oracle.capacity_from_factor(cf, T, N)
    dims = moe.make_dims(T, 64, N, k, 64, "swiglu", cap)
    ws = moe.new_workspace(dims)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    slot = torch.empty((T, k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((N,), dtype=torch.int32, device="cuda")
    moe.route_from_logits(dims, L, idx, w, slot, cnt, ws)
    picks = torch.full((N,), -1, dtype=torch.int32, device="cuda")
    pm = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
    aux = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    dropped = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for _ in range(2):  # twice: identical bits (deterministic sums)
        moe.router_stats(dims, L, idx, slot, picks, pm, aux, dropped, ws, alpha=0.01)
        torch.cuda.synchronize()
        first = (pm.clone(), aux.clone())
    assert torch.equal(first[0], pm) and torch.equal(first[1], aux)
    want = oracle.router_statistics(H.f64(L), idx.cpu().numpy(), slot.cpu().numpy(), 0.01)
    assert np.array_equal(picks.cpu().numpy(), want["picks"])
    assert int(dropped.item()) == want["dropped"]
    np.testing.assert_allclose(H.f64(pm), want["prob_mean"], rtol=2e-5, atol=1e-7)
    assert abs(float(aux.item()) - want["aux_loss"]) <= 2e-5 * abs(want["aux_loss"]) + 1e-9


# (T, d, N, k, capacity factor, zipf): the routing path each takes
#   tensor-core router, one CTA per tile (T*N*d*4 > 256 MiB, many tiles)
#   tensor-core router, tiles split over a cluster (few tiles)
#   per-token router; decode-sized router (one launch)
FUSED_CASES = [
    (16384, 512, 256, 8, 1.25, 1.1),   # 128 tiles, one CTA each; several capacity chunks
    (4096, 1024, 64, 1, 1.0, None),    # 32 tiles of 128 tokens, each split over 4 CTAs
    (2200, 1024, 32, 4, None, None),   # 18 tiles, split over 4 CTAs, ragged last tile
    (300, 256, 100, 3, 0.5, None),     # per-token router
    (5, 2880, 32, 4, 1.0, None),       # decode-sized: statistics formed in the one launch
]


@pytest.mark.parametrize("T,d,N,k,cf,zipf", FUSED_CASES,
                         ids=lambda v: str(v) if not isinstance(v, float) else f"{v:g}")
def test_route_with_stats_matches_oracle(T, d, N, k, cf, zipf):
    """moe_route_with_stats: the routing equals moe_route's bit for bit, and the statistics the
    routing launches emit match the oracle on the GPU's own logits and routing."""
    inp = synthetic.make_custom_inputs(T, d, N, 64, "swiglu", seed=T + N, device="cuda", zipf_s=zipf)
    cap = oracle.capacity_from_factor(cf, T, N)
    dims = moe.make_dims(T, d, N, k, 64, "swiglu", cap)
    ws = moe.new_workspace(dims)
    z = lambda shape, dt: torch.full(shape, -7, dtype=dt, device="cuda")
    ref = {n: z(s, dt) for n, s, dt in [("logits", (T, N), torch.float32), ("idx", (T, k), torch.int32),
                                         ("w", (T, k), torch.float32), ("slot", (T, k), torch.int32),
                                         ("cnt", (N,), torch.int32)]}
    moe.route(dims, inp["x"], inp["w_router"], inp["logit_bias"], ref["logits"], ref["idx"], ref["w"],
              ref["slot"], ref["cnt"], ws)
    got = {n: torch.empty_like(t) for n, t in ref.items()}
    picks = torch.full((N,), -1, dtype=torch.int32, device="cuda")
    pm = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
    aux = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    dropped = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    firsts = []
    for _ in range(2):  # twice: identical bits (deterministic sums)
        moe.route_with_stats(dims, inp["x"], inp["w_router"], inp["logit_bias"], got["logits"],
                             got["idx"], got["w"], got["slot"], got["cnt"], picks, pm, aux, dropped,
                             ws, alpha=0.01)
        torch.cuda.synchronize()
        firsts.append((pm.clone(), aux.clone()))
    assert moe.read_device_error(ws) == moe.OK
    assert torch.equal(firsts[0][0], firsts[1][0]) and torch.equal(firsts[0][1], firsts[1][1])
    for n in ref:
        assert torch.equal(ref[n], got[n]), n
    want = oracle.router_statistics(H.f64(got["logits"]), got["idx"].cpu().numpy(),
                                    got["slot"].cpu().numpy(), 0.01)
    assert np.array_equal(picks.cpu().numpy(), want["picks"])
    assert int(dropped.item()) == want["dropped"]
    np.testing.assert_allclose(H.f64(pm), want["prob_mean"], rtol=2e-5, atol=1e-7)
    assert abs(float(aux.item()) - want["aux_loss"]) <= 2e-5 * abs(want["aux_loss"]) + 1e-9
