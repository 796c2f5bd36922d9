"""The bounded-wait error path on the GPU: a wait limit far too short for the work makes the
tensor-core kernels give up, record MOE_ERR_TIMEOUT in the workspace status word and exit
(after draining their own copies and MMAs); the context stays usable and the next forward,
with the default limit and a re-zeroed workspace, is bit-identical to a clean one (GPU).

No fault is injected: the only change is the limit the library passes to its own waits."""
import pytest
import torch

import sparse_mixture_experts_11_b200 as moe
import synthetic

pytestmark = pytest.mark.gpu


def _forward(dims, inp, ws, out):
    moe.forward_into(dims, inp["x"], inp["w_router"], inp["logit_bias"], inp["w_gate_up"],
                     inp["w_down"], inp["x"], out, ws)
    torch.cuda.synchronize()


# per-token router, decode-sized one-launch router, tensor-core router (T * N * d * 4 > 256 MiB),
# the tensor-core router on CTA pairs (76 tiles, 256 experts), the grouped FFN on CTA pairs
# (R_max >= 1024 N), and a single token (one-launch router, stream-K grouped FFN)
@pytest.mark.parametrize("T,d,N,k,F", [(512, 1024, 8, 2, 2048), (3, 512, 8, 2, 1024),
                                       (4096, 1024, 64, 1, 1024), (9728, 512, 256, 8, 256),
                                       (4096, 512, 4, 2, 512), (1, 512, 8, 2, 1024)])
def test_wait_timeout_reported_and_context_survives(T, d, N, k, F):
    inp = synthetic.make_custom_inputs(T, d, N, F, "swiglu", seed=4, device="cuda")
    dims = moe.make_dims(T, d, N, k, F, "swiglu", T)
    ws = moe.new_workspace(dims, forward=True)
    b = moe.forward_layout(dims, ws)
    status_off = b.stage_ws - ws.data_ptr()
    clean = torch.empty_like(inp["x"])
    _forward(dims, inp, ws, clean)
    assert moe.read_device_error(ws, offset_bytes=status_off) == moe.OK

    out = torch.empty_like(inp["x"])
    old = moe.debug_set_wait_timeout_ns(1)
    try:
        _forward(dims, inp, ws, out)
    finally:
        moe.debug_set_wait_timeout_ns(0)
    assert moe.read_device_error(ws, offset_bytes=status_off) == moe.ERR_TIMEOUT
    assert old == 2_000_000_000

    ws.zero_()  # split-K counters may have been left mid-count
    _forward(dims, inp, ws, out)
    assert moe.read_device_error(ws, offset_bytes=status_off) == moe.OK
    assert torch.equal(out.view(torch.int16), clean.view(torch.int16))
