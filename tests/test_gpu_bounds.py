"""The device-side bounds check (GPU): a row index computed from device data that falls outside
its buffer is skipped and recorded as MOE_ERR_BOUNDS, without a fault.

moe_unpermute_combine gets a row_of_pair entry at or past R_max. The y_perm allocation has
padding rows past R_max, so even an unchecked read of that row would stay inside the
allocation: the test cannot fault the GPU whatever the kernel does."""
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu


def test_combine_row_past_r_max_is_skipped_and_reported():
    import sparse_mixture_experts_11_b200 as moe
    T, d, N, k, F = 6, 256, 8, 2, 128
    dims = moe.make_dims(T, d, N, k, F, "swiglu", T)
    R = moe.max_rows(dims)
    pad = 16
    g = torch.Generator(device="cuda").manual_seed(3)
    y_big = torch.randn((R + pad, d), generator=g, device="cuda", dtype=torch.float32)
    y = y_big[:R]  # the call sees R rows; the allocation holds R + pad
    x = synthetic.make_hidden(T, d, seed=2, device="cuda")
    rows = torch.arange(T * k, dtype=torch.int32, device="cuda").view(T, k)
    w = torch.full((T, k), 0.5, dtype=torch.float32, device="cuda")
    ws = moe.new_workspace(dims)
    clean = torch.empty_like(x)
    moe.unpermute_combine(dims, y, rows, w, x, clean, ws)
    torch.cuda.synchronize()
    assert moe.read_device_error(ws) == moe.OK

    # token 2's first choice points past R_max (into the padding)
    bad_rows = rows.clone()
    bad_rows[2, 0] = R + 3
    out = torch.empty_like(x)
    moe.unpermute_combine(dims, y, bad_rows, w, x, out, ws)
    torch.cuda.synchronize()
    assert moe.read_device_error(ws) == moe.ERR_BOUNDS
    # every other token is unchanged; token 2 gets its valid pair only, as if the bad one
    # had been dropped
    others = [t for t in range(T) if t != 2]
    assert torch.equal(out[others].view(torch.int16), clean[others].view(torch.int16))
    dropped_rows = rows.clone()
    dropped_rows[2, 0] = -1
    want = torch.empty_like(x)
    moe.unpermute_combine(dims, y, dropped_rows, w, x, want, ws)
    torch.cuda.synchronize()
    assert moe.read_device_error(ws) == moe.OK
    assert torch.equal(out[2].view(torch.int16), want[2].view(torch.int16))
