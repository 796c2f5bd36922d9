"""The grouped FFN on CTA pairs (GPU).

With bf16 weights and experts that average at least eight 128-row m-tiles (R_max >= 1024 N),
the grouped FFN runs as clusters of two CTAs: the even CTA issues M = 256 MMAs over two
neighbouring m-tiles of one expert, each CTA holding half of the 256 weight rows. Shapes here
give experts odd and even m-tile counts (so some pairs have an empty odd m-tile) and ragged
last tiles; y rows of every expert and the layer output are checked against the oracle."""
import numpy as np
import pytest

import oracle
import synthetic
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

# name, T, d, N, k, F, act, capacity factor, zipf
PAIR_CASES = [
    ("swiglu_even", 4096, 512, 4, 2, 640, "swiglu", None, None),
    ("swiglu_skewed", 3000, 256, 4, 2, 384, "swiglu", None, 1.2),
    ("gelu_skewed_capacity", 3200, 384, 3, 1, 512, "gelu", 1.1, 1.5),
]


@pytest.mark.parametrize("case", PAIR_CASES, ids=lambda c: c[0])
def test_pair_ffn_parity(case):
    name, T, d, N, k, F, act, cf, zipf = case
    inp = synthetic.make_custom_inputs(T, d, N, F, act, seed=9, device="cuda", zipf_s=zipf)
    cap = oracle.capacity_from_factor(cf, T, N)
    run = H.StageRun(inp, k, act, cap).run()
    assert run.R_max >= 1024 * N and min(cap, T) > 64  # the paired shape
    routing, off, rop = H.check_routing(run, cap)
    counts = np.diff(off)
    assert any((c + 127) // 128 % 2 == 1 for c in counts if c)  # some pair has an empty half
    rows = []
    for e in range(N):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi > lo:
            rows += [lo, min(lo + 127, hi - 1), min(lo + 128, hi - 1), min(lo + 300, hi - 1), hi - 1]
    H.check_expert_rows(run, routing, act, np.unique(np.array(rows, dtype=np.int64)))
    tokens = np.unique(np.linspace(0, T - 1, 64).astype(np.int64))
    H.check_outputs(run, routing, act, tokens=tokens)
    H.check_dropped_tokens_pass_through(run, routing["slot"])
