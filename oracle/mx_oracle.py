"""CPU oracle for expert weights stored in the MX (microscaling) formats.

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only the test suite, the smoke check and
the benchmark's CPU-baseline leg may use it, and it shares no code with the CUDA library.

The pages name the format only: page «Что такое Mixture of Experts (MoE) в трансформерах:
архитектура и параллелизм» (aglamov.biz), introduction, remarks that gpt-oss's decode
speed would be higher with kernels for its native mxfp4 quantisation. The format itself is
the published OCP Microscaling Formats (MX) Specification v1.0:

* a block of 32 consecutive elements along the reduction axis shares one scale X;
* the scale type is E8M0: an unsigned 8-bit exponent, X = 2^(s - 127); s = 255 is NaN;
* element type FP8 E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 holds
  the subnormals m/8 * 2^-6; S.1111.111 is NaN (no infinities); largest value 448;
* element type FP4 E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 holds
  0 and 0.5; the magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6;
* the value of element i of a block is X * element_i.

Storage (this library's layout, written down in include/moe.h):

* elements [rows, K] uint8 (E4M3), or [rows, K/2] uint8 (E2M1, element 2i in the low
  nibble of byte i, element 2i+1 in the high nibble);
* scales [K/32, rows] uint8: scale block b of row r at [b, r].

Everything is float64; every decoded value is exact.
"""
from __future__ import annotations

import numpy as np

MX_BLOCK = 32


def decode_e8m0(codes: np.ndarray) -> np.ndarray:
    """Scale codes -> 2^(s - 127) (NaN for s = 255)."""
    c = np.asarray(codes, dtype=np.int64)
    out = np.ldexp(1.0, c - 127).astype(np.float64)
    return np.where(c == 255, np.nan, out)


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """FP8 E4M3 codes -> values: (-1)^S * 2^(E-7) * (1 + M/8), or 2^-6 * M/8 when E = 0."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 15
    m = c & 7
    normal = np.ldexp(1.0 + m / 8.0, e - 7)
    sub = np.ldexp(m / 8.0, -6)
    v = sign * np.where(e == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


def decode_e2m1(codes: np.ndarray) -> np.ndarray:
    """FP4 E2M1 codes -> values: (-1)^S * 2^(E-1) * (1 + M/2), or M/2 when E = 0."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where((c >> 3) & 1, -1.0, 1.0)
    e = (c >> 1) & 3
    m = c & 1
    normal = np.ldexp(1.0 + m / 2.0, e - 1)
    sub = m / 2.0
    return sign * np.where(e == 0, sub, normal)


def unpack_fp4(packed: np.ndarray) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] E2M1 codes; element 2i is the low nibble of byte i."""
    b = np.asarray(packed, dtype=np.int64)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int64)
    out[..., 0::2] = b & 15
    out[..., 1::2] = b >> 4
    return out


def dequantize_mx(elements: np.ndarray, scales: np.ndarray, fmt: str) -> np.ndarray:
    """One expert's weight matrix [rows, K] in float64 from its MX storage.

    elements  [rows, K] (fmt "mxfp8") or [rows, K/2] (fmt "mxfp4") uint8
    scales    [K/32, rows] uint8 (E8M0)
    """
    if fmt == "mxfp8":
        vals = decode_e4m3(elements)
    elif fmt == "mxfp4":
        vals = decode_e2m1(unpack_fp4(elements))
    else:
        raise ValueError(fmt)
    rows, K = vals.shape
    if K % MX_BLOCK or scales.shape != (K // MX_BLOCK, rows):
        raise ValueError("scales must be [K/32, rows]")
    x = decode_e8m0(scales).T  # [rows, K/32]
    return vals * np.repeat(x, MX_BLOCK, axis=1)


# --------------------------------------------------------------------------
# MXFP8 activations (the block-scaled tensor-core variant)
# --------------------------------------------------------------------------
# Reading (the pages fix no activation format): with the block-scaled formats the token rows
# and h are quantised to MXFP8 along the reduction axis, following the OCP MX v1.0
# conversion: per block of 32 the shared scale is X = 2^(floor(log2(amax)) - 8), 8 being the
# exponent of E4M3's largest power of two (256), clamped to E8M0's range [-127, 127] (an
# all-zero block takes 2^-127); each element is v / X rounded to the nearest E4M3 value,
# ties to the even code, magnitudes above 448 saturating to 448.

E4M3_EMAX = 8
_E4M3_POS = decode_e4m3(np.arange(0x7F))  # codes 0x00..0x7E: 0 .. 448, increasing


def encode_e4m3(v: np.ndarray) -> np.ndarray:
    """Finite values -> E4M3 codes: nearest value (ties to the even code), |v| > 448 -> 448.

    The sign bit is the value's (so -0.0 and negatives that round to zero give 0x80)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), 448.0)
    hi = np.clip(np.searchsorted(_E4M3_POS, a, side="left"), 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(take_hi, hi, lo).astype(np.int64)
    return np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)


def quantize_mxfp8(x: np.ndarray):
    """[..., K] values (K a multiple of 32) -> (codes [..., K] uint8 E4M3,
    scales [..., K/32] uint8 E8M0), per block of 32 along the last axis."""
    x = np.asarray(x, dtype=np.float64)
    K = x.shape[-1]
    if K % MX_BLOCK:
        raise ValueError("K must be a multiple of 32")
    blocks = x.reshape(x.shape[:-1] + (K // MX_BLOCK, MX_BLOCK))
    amax = np.abs(blocks).max(axis=-1)
    _, ex = np.frexp(amax)  # amax = m * 2^ex with m in [0.5, 1): floor(log2(amax)) = ex - 1
    e = np.where(amax > 0, ex - 1 - E4M3_EMAX, -127)
    e = np.clip(e, -127, 127).astype(np.int64)
    codes = encode_e4m3(blocks * np.ldexp(1.0, -e)[..., None])
    return codes.reshape(x.shape), (e + 127).astype(np.uint8)


def dequantize_mxfp8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Inverse of quantize_mxfp8's storage: codes [..., K], scales [..., K/32] -> float64."""
    vals = decode_e4m3(codes)
    x = decode_e8m0(scales)
    return vals * np.repeat(x, MX_BLOCK, axis=-1)


def mxfp8_round_trip(x: np.ndarray) -> np.ndarray:
    """x as the block-scaled tensor cores see it: quantised to MXFP8 and read back."""
    return dequantize_mxfp8(*quantize_mxfp8(x))


def expert_ffn_mxfp8_act(rows: np.ndarray, w_gate_up: np.ndarray, w_down: np.ndarray,
                         act: str) -> np.ndarray:
    """One expert with MXFP8 activations: the rows quantised along d, h (computed from the
    quantised rows, then the activation) quantised along F, both products exact in float64.

    SwiGLU: w_gate_up [2F, d] (gate rows, then up rows); GELU: w_gate_up [F, d]; w_down [d, F].
    """
    from .moe_oracle import gelu, silu
    xq = mxfp8_round_trip(rows)
    if act == "swiglu":
        F = w_gate_up.shape[0] // 2
        h = silu(xq @ w_gate_up[:F].T) * (xq @ w_gate_up[F:].T)
    elif act == "gelu":
        h = gelu(xq @ w_gate_up.T)
    else:
        raise ValueError(f"unknown activation {act!r}")
    return mxfp8_round_trip(h) @ w_down.T
