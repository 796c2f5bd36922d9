"""Plant plausible mistakes in the CPU oracle and check that some pin catches each.

The mistakes are planted in the oracle module on the CPU, for the duration of one
test, with monkeypatch; nothing here touches the CUDA path.
"""
import math

import numpy as np
import pytest

import oracle.moe_oracle as om
from tests import oracle_pins


def _silu_sign(z):
    return z / (1.0 + np.exp(z))


def _gelu_tanh(z):
    return 0.5 * z * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)))


def _ffn_transposed_down(rows, wgu, wd, act):
    if act == "swiglu":
        F = wgu.shape[0] // 2
        h = om.silu(rows @ wgu[:F].T) * (rows @ wgu[F:].T)
    else:
        h = om.gelu(rows @ wgu.T)
    return h @ wd if wd.shape[0] == wd.shape[1] else h @ wd.T  # transposed when square


def _ffn_gate_up_swapped(rows, wgu, wd, act):
    if act == "swiglu":
        F = wgu.shape[0] // 2
        h = om.silu(rows @ wgu[F:].T) * (rows @ wgu[:F].T)
    else:
        h = om.gelu(rows @ wgu.T)
    return h @ wd.T


def _select_ties_high(logits, k):
    T, N = logits.shape
    idx = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        order = np.lexsort((-np.arange(N), -logits[t]))
        idx[t] = order[:k]
    return idx


def _no_renormalise(probs, idx):
    return np.take_along_axis(probs, idx, axis=1)


def _slots_token_major(idx, cap, n):
    T, k = idx.shape
    filled = np.zeros(n, dtype=np.int64)
    slot = np.full((T, k), -1, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            if filled[e] < cap:
                slot[t, j] = filled[e]
                filled[e] += 1
    return slot, filled


def _capacity_floor(cf, T, n):
    if cf is None or not math.isfinite(cf) or cf <= 0:
        return T
    return int(math.floor(cf * T / n))


def _capacity_times_k(cf, T, n):
    if cf is None or not math.isfinite(cf) or cf <= 0:
        return T
    return int(math.ceil(2 * cf * T / n))


def _router_transposed_bias_sign(x, wr, b=None):
    L = x @ wr.T
    return L if b is None else L - b[None, :]


def _router_bias_ignored(x, wr, b=None):
    return x @ wr.T


def _router_bias_per_token(x, wr, b=None):
    L = x @ wr.T
    return L if b is None else L + b[:L.shape[0], None]


def _softmax_no_shift_wrong_axis(logits):
    ez = np.exp(logits)
    return ez / ez.sum(axis=0, keepdims=True)


def _combine_drops_residual(x, routing, wgu, wd, act, residual, tokens=None):
    return _orig_combine(x, routing, wgu, wd, act, None, tokens)


def _aux_without_n(logits, topk_idx, slot, alpha=1e-2):
    st = _orig_stats(logits, topk_idx, slot, alpha)
    st["aux_loss"] /= logits.shape[1]
    return st


def _aux_f_over_tk(logits, topk_idx, slot, alpha=1e-2):
    st = _orig_stats(logits, topk_idx, slot, alpha)
    st["aux_loss"] /= topk_idx.shape[1]
    st["picks"] = st["picks"] // topk_idx.shape[1]
    return st


_orig_stats = om.router_statistics


_orig_combine = om.combine

MUTANTS = {
    "silu_sign": ("silu", _silu_sign),
    "gelu_tanh_approx": ("gelu", _gelu_tanh),
    "down_transposed": ("expert_ffn", _ffn_transposed_down),
    "gate_up_swapped": ("expert_ffn", _ffn_gate_up_swapped),
    "ties_to_high_index": ("select_top_k", _select_ties_high),
    "no_renormalise": ("renormalise", _no_renormalise),
    "token_major_slots": ("assign_capacity_slots", _slots_token_major),
    "capacity_floor": ("capacity_from_factor", _capacity_floor),
    "capacity_times_k": ("capacity_from_factor", _capacity_times_k),
    "softmax_wrong_axis": ("softmax_over_experts", _softmax_no_shift_wrong_axis),
    "residual_dropped": ("combine", _combine_drops_residual),
    "aux_without_N": ("router_statistics", _aux_without_n),
    "aux_f_over_Tk": ("router_statistics", _aux_f_over_tk),
    "bias_sign": ("router_logits", _router_transposed_bias_sign),
    "bias_ignored": ("router_logits", _router_bias_ignored),
    "bias_per_token": ("router_logits", _router_bias_per_token),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_some_pin_catches(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(om, attr, fn)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(om)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"



# ---------------------------------------------------------------- MX decoding mutants
import oracle.mx_oracle as mxo  # noqa: E402


def _unpack_high_first(packed):
    b = np.asarray(packed, dtype=np.int64)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int64)
    out[..., 0::2] = b >> 4
    out[..., 1::2] = b & 15
    return out


def _e4m3_bias8(codes):
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e, mm = (c >> 3) & 15, c & 7
    v = sign * np.where(e == 0, np.ldexp(mm / 8.0, -7), np.ldexp(1.0 + mm / 8.0, e - 8))
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


def _e2m1_no_subnormal(codes):
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where((c >> 3) & 1, -1.0, 1.0)
    e, mm = (c >> 1) & 3, c & 1
    return sign * np.ldexp(1.0 + mm / 2.0, e - 1)


def _e8m0_bias128(codes):
    c = np.asarray(codes, dtype=np.int64)
    return np.where(c == 255, np.nan, np.ldexp(1.0, c - 128))


def _dequant_scales_not_transposed(elements, scales, fmt):
    vals = mxo.decode_e4m3(elements) if fmt == "mxfp8" else mxo.decode_e2m1(mxo.unpack_fp4(elements))
    x = mxo.decode_e8m0(scales)  # read as [rows, K/32]
    return vals * np.repeat(x, mxo.MX_BLOCK, axis=1)


def _quantize_scale_ceil(x):
    x = np.asarray(x, dtype=np.float64)
    blocks = x.reshape(x.shape[:-1] + (x.shape[-1] // 32, 32))
    amax = np.abs(blocks).max(axis=-1)
    e = np.where(amax > 0, np.ceil(np.log2(np.where(amax > 0, amax, 1.0))) - 8, -127)
    e = np.clip(e, -127, 127).astype(np.int64)
    codes = mxo.encode_e4m3(blocks * np.ldexp(1.0, -e)[..., None])
    return codes.reshape(x.shape), (e + 127).astype(np.uint8)


def _quantize_emax_7(x):
    x = np.asarray(x, dtype=np.float64)
    blocks = x.reshape(x.shape[:-1] + (x.shape[-1] // 32, 32))
    amax = np.abs(blocks).max(axis=-1)
    _, ex = np.frexp(amax)
    e = np.clip(np.where(amax > 0, ex - 1 - 7, -127), -127, 127).astype(np.int64)
    codes = mxo.encode_e4m3(blocks * np.ldexp(1.0, -e)[..., None])
    return codes.reshape(x.shape), (e + 127).astype(np.uint8)


def _encode_truncating(v):
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), 448.0)
    code = np.clip(np.searchsorted(mxo._E4M3_POS, a, side="right") - 1, 0, 126).astype(np.int64)
    return np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)


def _encode_no_saturation(v):
    v = np.asarray(v, dtype=np.float64)
    out = mxo.__dict__["_encode_ref"](v).astype(np.int64)
    return np.where(np.abs(v) > 448.0, out | 0x7F, out).astype(np.uint8)  # NaN code


def _ffn_h_not_quantised(rows, wgu, wd, act):
    xq = mxo.mxfp8_round_trip(rows)
    F = wgu.shape[0] // 2
    h = om.silu(xq @ wgu[:F].T) * (xq @ wgu[F:].T) if act == "swiglu" else om.gelu(xq @ wgu.T)
    return h @ wd.T


def _ffn_x_not_quantised(rows, wgu, wd, act):
    F = wgu.shape[0] // 2
    h = om.silu(rows @ wgu[:F].T) * (rows @ wgu[F:].T) if act == "swiglu" else om.gelu(rows @ wgu.T)
    return mxo.mxfp8_round_trip(h) @ wd.T


MX_MUTANTS = {
    "mxfp8_scale_from_ceil": ("quantize_mxfp8", _quantize_scale_ceil),
    "mxfp8_emax_7": ("quantize_mxfp8", _quantize_emax_7),
    "e4m3_encode_truncates": ("encode_e4m3", _encode_truncating),
    "e4m3_encode_no_saturation": ("encode_e4m3", _encode_no_saturation),
    "act_ffn_h_not_quantised": ("expert_ffn_mxfp8_act", _ffn_h_not_quantised),
    "act_ffn_x_not_quantised": ("expert_ffn_mxfp8_act", _ffn_x_not_quantised),
    "fp4_high_nibble_first": ("unpack_fp4", _unpack_high_first),
    "e4m3_bias_8": ("decode_e4m3", _e4m3_bias8),
    "e2m1_no_subnormal": ("decode_e2m1", _e2m1_no_subnormal),
    "e8m0_bias_128": ("decode_e8m0", _e8m0_bias128),
    "scales_not_transposed": ("dequantize_mx", _dequant_scales_not_transposed),
}


@pytest.mark.parametrize("name", sorted(MX_MUTANTS))
def test_some_mx_pin_catches(name, monkeypatch):
    attr, fn = MX_MUTANTS[name]
    monkeypatch.setitem(mxo.__dict__, "_encode_ref", mxo.encode_e4m3)
    monkeypatch.setattr(mxo, attr, fn)
    caught = []
    for pin in oracle_pins.MX_PINS:
        try:
            pin(mxo)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"


# ---------------------------------------------------------------- reroute policy mutants
def _reroute_allows_reuse(topk_idx, logits, capacity):
    T, k = topk_idx.shape
    N = logits.shape[1]
    expert = np.array(topk_idx, dtype=np.int64, copy=True)
    filled = np.zeros(N, dtype=np.int64)
    slot = np.full((T, k), -1, dtype=np.int64)
    for j in range(k):
        for t in range(T):
            e = int(expert[t, j])
            if filled[e] < capacity:
                slot[t, j] = filled[e]
                filled[e] += 1
                continue
            for c in sorted(range(N), key=lambda c: (-logits[t, c], c)):
                if filled[c] < capacity:  # mistake: may pick an expert the token already uses
                    expert[t, j], slot[t, j] = c, filled[c]
                    filled[c] += 1
                    break
    return expert, slot, filled


def _reroute_token_major(topk_idx, logits, capacity):
    T, k = topk_idx.shape
    N = logits.shape[1]
    expert = np.array(topk_idx, dtype=np.int64, copy=True)
    filled = np.zeros(N, dtype=np.int64)
    slot = np.full((T, k), -1, dtype=np.int64)
    for t in range(T):  # mistake: token-major arrivals
        for j in range(k):
            e = int(expert[t, j])
            if filled[e] < capacity:
                slot[t, j] = filled[e]
                filled[e] += 1
                continue
            used = set(expert[t].tolist())
            for c in sorted(range(N), key=lambda c: (-logits[t, c], c)):
                if c not in used and filled[c] < capacity:
                    expert[t, j], slot[t, j] = c, filled[c]
                    filled[c] += 1
                    break
    return expert, slot, filled


def _reroute_worst_first(topk_idx, logits, capacity):
    T, k = topk_idx.shape
    N = logits.shape[1]
    expert = np.array(topk_idx, dtype=np.int64, copy=True)
    filled = np.zeros(N, dtype=np.int64)
    slot = np.full((T, k), -1, dtype=np.int64)
    for j in range(k):
        for t in range(T):
            e = int(expert[t, j])
            if filled[e] < capacity:
                slot[t, j] = filled[e]
                filled[e] += 1
                continue
            used = set(expert[t].tolist())
            for c in sorted(range(N), key=lambda c: (logits[t, c], c)):  # mistake: least suitable
                if c not in used and filled[c] < capacity:
                    expert[t, j], slot[t, j] = c, filled[c]
                    filled[c] += 1
                    break
    return expert, slot, filled


REROUTE_MUTANTS = {
    "reroute_reuses_own_expert": ("assign_capacity_slots_reroute", _reroute_allows_reuse),
    "reroute_token_major": ("assign_capacity_slots_reroute", _reroute_token_major),
    "reroute_least_suitable": ("assign_capacity_slots_reroute", _reroute_worst_first),
}


@pytest.mark.parametrize("name", sorted(REROUTE_MUTANTS))
def test_some_reroute_pin_catches(name, monkeypatch):
    attr, fn = REROUTE_MUTANTS[name]
    monkeypatch.setattr(om, attr, fn)
    caught = []
    for pin in oracle_pins.REROUTE_PINS:
        try:
            pin(om)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
