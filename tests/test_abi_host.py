"""The C-ABI library on the host (no GPU): it loads, exports every declared symbol, and its
host-only helpers and argument validation behave as include/moe.h states."""
import ctypes
import math
import re
import subprocess

import pytest

import oracle
import sparse_mixture_experts_11_b200 as moe


def test_every_declared_symbol_is_exported():
    declared = moe.exported_symbols()
    assert len(declared) >= 14
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (moe_\w+)$", out, flags=re.M))
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    for s in declared:
        getattr(moe._lib, s)


@pytest.mark.parametrize("cf,T,N", [(1.0, 32, 8), (1.25, 32, 8), (1.25, 64, 8), (1.0, 4096, 64),
                                    (1.25, 16384, 256), (1.0, 3, 4), (0.1, 7, 3), (2.0, 5, 1),
                                    (None, 17, 4), (float("inf"), 9, 2), (1.1, 1000, 7)])
def test_capacity_matches_oracle(cf, T, N):
    assert moe.capacity(cf, T, N) == oracle.capacity_from_factor(cf, T, N)


def test_capacity_page_values():
    assert moe.capacity(1.0, 32, 8) == 4
    assert moe.capacity(1.25, 32, 8) == 5


def test_max_rows():
    d = moe.make_dims(64, 128, 8, 2, 256, "swiglu", 10)
    assert moe.max_rows(d) == 80
    d = moe.make_dims(16384, 7168, 256, 8, 2048, "swiglu", 80)
    assert moe.max_rows(d) == 20480
    d = moe.make_dims(8192, 4096, 8, 2, 14336, "swiglu", 8192)
    assert moe.max_rows(d) == 16384
    d = moe.make_dims(5, 64, 4, 2, 64, "gelu", 0)
    assert moe.max_rows(d) == 0


def test_workspace_sizes():
    def counters(m_tiles, tiles1, tiles2):
        # FFN counters: finished gate/up tiles per m-tile, CTAs done, stream-K arrival
        # counters of both GEMMs' tiles; rounded to 256 B
        return -(-((m_tiles + 1 + tiles1 + tiles2) * 4) // 256) * 256

    small = moe.make_dims(64, 128, 8, 2, 256, "swiglu", 10)
    # status word + counters (at most 10 m-tiles of 64 rows: 20 gate/up and 10 down tiles) +
    # two partial slots of 10 rows x 256 fp32 columns for each CTA that can hold a stream-K
    # range of either GEMM (20 and 10)
    assert moe.workspace_bytes(small) == 256 + counters(10, 20, 10) + (20 + 10) * 2 * 10 * 256 * 4
    big = moe.make_dims(16384, 7168, 256, 8, 2048, "swiglu", 80)
    # 80-row partial tiles: whole tiles only; status word + per-m-tile counters (at most
    # 160 + 256 m-tiles) + the routing scratch: capacity-scan chunk totals + the bf16
    # three-term split of W_r that the tensor-core router reads + the router's probability sums
    # for moe_route_with_stats (one row of 256 per 128-token tile)
    assert moe.workspace_bytes(big) == (256 + counters(416, 0, 0) + 32 * 256 * 4
                                        + 3 * 256 * 7168 * 2 + 128 * 256 * 4)
    decode = moe.make_dims(4, 2880, 32, 4, 2880, "swiglu", 4)
    # status word (+ the decode router's arrival counter) + counters (at most 1 + 16 m-tiles:
    # 17 x 23 gate/up and 17 x 12 down tiles) + the larger of the decode router's partial dot
    # products (23 slices x 4 tokens x 32 experts) and two 4-row partial slots per CTA for each
    # GEMM (148 + 148 CTAs)
    assert moe.workspace_bytes(decode) == (256 + counters(17, 17 * 23, 17 * 12)
                                           + max(23 * 4 * 32 * 4, 296 * 2 * 4 * 256 * 4))
    fb = moe.forward_workspace_bytes(big)
    assert fb > 20480 * 7168 * 6


@pytest.mark.parametrize("kw,status", [
    (dict(top_k=9, n_experts=16), moe.ERR_UNSUPPORTED),
    (dict(top_k=3, n_experts=2), moe.ERR_INVALID),
    (dict(n_experts=300), moe.ERR_UNSUPPORTED),
    (dict(d_model=100), moe.ERR_UNSUPPORTED),
    (dict(d_ff=96), moe.ERR_UNSUPPORTED),
    (dict(T=-1), moe.ERR_INVALID),
    (dict(capacity=-2), moe.ERR_INVALID),
    (dict(act=7), moe.ERR_INVALID),
])
def test_validation_before_any_launch(kw, status):
    base = dict(T=16, d_model=128, n_experts=8, top_k=2, d_ff=128, act=0, capacity=16)
    base.update(kw)
    d = moe.Dims(**base)
    n = ctypes.c_size_t(0)
    assert moe._lib.moe_workspace_bytes(ctypes.byref(d), ctypes.byref(n)) == status
    # a compute call with these dims fails validation before touching any device
    P = ctypes.c_void_p
    r = moe._lib.moe_route(ctypes.byref(d), P(16), P(16), None, P(16), P(16), P(16), P(16), P(16),
                           P(16), 1 << 20, None)
    assert r == status


def test_null_and_alignment_checks_precede_device_use():
    d = moe.make_dims(16, 128, 8, 2, 128, "swiglu", 16)
    P = ctypes.c_void_p
    lib = moe._lib
    assert lib.moe_route(ctypes.byref(d), None, P(16), None, P(16), P(16), P(16), P(16), P(16),
                         P(16), 1 << 20, None) == moe.ERR_INVALID
    assert lib.moe_route(ctypes.byref(d), P(24), P(16), None, P(16), P(16), P(16), P(16), P(16),
                         P(16), 1 << 20, None) == moe.ERR_UNSUPPORTED
    assert lib.moe_route(ctypes.byref(d), P(16), P(16), None, P(16), P(16), P(16), P(16), P(16),
                         P(16), 8, None) == moe.ERR_WORKSPACE


def test_empty_batch_returns_ok_without_device():
    d = moe.make_dims(0, 128, 8, 2, 128, "swiglu", 0)
    assert moe._lib.moe_route(ctypes.byref(d), None, None, None, None, None, None, None, None,
                              None, 0, None) == moe.OK


def test_forward_layout_is_disjoint_and_aligned():
    d = moe.make_dims(300, 192, 8, 2, 320, "swiglu", 75)
    n = moe.forward_workspace_bytes(d)
    b = moe.ForwardBuffers()
    base = 1 << 20
    assert moe._lib.moe_forward_layout(ctypes.byref(d), ctypes.c_void_p(base), n, ctypes.byref(b)) == 0
    R = moe.max_rows(d)
    regions = [(b.logits, 300 * 8 * 4), (b.topk_idx, 600 * 4), (b.topk_w, 600 * 4), (b.slot, 600 * 4),
               (b.expert_count, 8 * 4), (b.expert_offset, 9 * 4), (b.row_of_pair, 600 * 4),
               (b.pair_of_row, R * 4), (b.x_perm, R * 192 * 2), (b.h, R * 320 * 2),
               (b.y_perm, R * 192 * 4), (b.stage_ws, b.stage_ws_bytes)]
    regions.sort()
    for (a, la), (c, _) in zip(regions, regions[1:]):
        assert a + la <= c
    assert all(p % 256 == 0 for p, _ in regions)
    assert regions[-1][0] + regions[-1][1] <= base + n


def test_status_strings():
    for s in (0, -1, -2, -3, -4, -5, -6):
        assert moe.status_string(s)


def _r256(n):
    return (n + 255) // 256 * 256


def test_backward_workspace_bytes():
    """Regions: status word, dL, dy, pre, dh, d_pre, h, dx_rows, router partial sums."""
    for T, d, N, k, F, act, cap in [(300, 192, 8, 2, 320, "swiglu", 75), (4096, 1024, 64, 1, 4096, "gelu", 64),
                                    (40000, 128, 4, 2, 64, "gelu", 40000)]:
        dims = moe.make_dims(T, d, N, k, F, act, cap)
        R = moe.max_rows(dims)
        n_gu = 2 * F if act == "swiglu" else F
        chunk = max(256, (T + 15) // 16)
        chunks = (T + chunk - 1) // chunk
        sizes = [256, T * N * 4, R * d * 2, R * n_gu * 4, R * F * 4, R * n_gu * 2, R * F * 2,
                 R * d * 4, chunks * N * d * 4]
        assert moe.backward_workspace_bytes(dims) == sum(_r256(s) for s in sizes)


def test_backward_validation_precedes_device_use():
    d = moe.make_dims(16, 128, 8, 2, 128, "swiglu", 16)
    P = ctypes.c_void_p
    lib = moe._lib
    big = 1 << 30
    fw = moe.forward_workspace_bytes(d)
    args = lambda x=P(16), ws_bytes=big, fwd_bytes=fw, d_bias=None: (
        ctypes.byref(d), x, P(16), P(16), P(16), P(16), fwd_bytes, P(16), P(16), P(16), d_bias,
        P(16), P(16), P(16), ws_bytes, None)
    assert lib.moe_backward(*args(x=None)) == moe.ERR_INVALID
    assert lib.moe_backward(*args(x=P(24))) == moe.ERR_UNSUPPORTED
    assert lib.moe_backward(*args(d_bias=P(8))) == moe.ERR_UNSUPPORTED
    assert lib.moe_backward(*args(ws_bytes=64)) == moe.ERR_WORKSPACE
    assert lib.moe_backward(*args(fwd_bytes=64)) == moe.ERR_WORKSPACE
    e = moe.make_dims(0, 128, 8, 2, 128, "swiglu", 0)
    assert lib.moe_backward(ctypes.byref(e), None, None, None, None, None, 0, None, None, None,
                            None, None, None, None, 0, None) == moe.OK


def test_redirect_validation_precedes_device_use():
    P = ctypes.c_void_p
    lib = moe._lib
    d = moe.make_dims(16, 128, 8, 2, 128, "swiglu", 4)
    assert lib.moe_redirect_overflow(ctypes.byref(d), None, P(16), P(16), P(16), P(16), 1 << 20,
                                     None) == moe.ERR_INVALID
    assert lib.moe_redirect_overflow(ctypes.byref(d), P(16), P(20), P(16), P(16), P(16), 1 << 20,
                                     None) == moe.ERR_UNSUPPORTED
    assert lib.moe_redirect_overflow(ctypes.byref(d), P(16), P(16), P(16), P(16), P(16), 8,
                                     None) == moe.ERR_WORKSPACE
    big = moe.make_dims(20481, 128, 256, 8, 128, "swiglu", 4)  # T * k = 163848 pairs
    assert lib.moe_redirect_overflow(ctypes.byref(big), P(16), P(16), P(16), P(16), P(16), 1 << 30,
                                     None) == moe.ERR_UNSUPPORTED
    assert moe.REDIRECT_MAX_PAIRS == 163840
