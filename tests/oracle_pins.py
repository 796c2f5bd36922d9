"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each ``pin_*`` function takes the oracle module and raises AssertionError when
the oracle disagrees with:

* values printed on the pages (capacity limits and drop counts of the second
  demo script, active-parameter counts of the first);
* routing worked out by hand (a tie, renormalised weights, drops, row order);
* expert outputs worked out by hand from textbook constants;
* brute force on tiny inputs (all k-subsets; capacity slots by their rank
  definition rather than the oracle's running counter);
* the dense special case k = N with no capacity limit, which must equal the
  softmax-weighted mixture of all experts;
* invariants (weights sum to one, no expert above capacity, kept pairs precede
  dropped pairs, a fully dropped token leaves the residual unchanged).

They live in a plain module so ``test_oracle_mutations.py`` can plant mistakes
in the oracle and check that some pin catches each one.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- capacity / drops
def pin_capacity_demo(o):
    g = _golden("capacity_demo.json")
    T, N = g["tokens"], g["experts"]
    loads = g["collapsed_tokens_per_expert"]
    assert sum(loads) == T
    # a top-1 routing with exactly those per-expert loads, tokens interleaved
    idx = []
    remaining = list(loads)
    while any(remaining):
        for e in range(N):
            if remaining[e]:
                idx.append(e)
                remaining[e] -= 1
    topk_idx = np.array(idx, dtype=np.int64)[:, None]
    for case in g["cases"]:
        cap = o.capacity_from_factor(case["capacity_factor"], T, N)
        assert cap == case["capacity"], (cap, case)
        slot, kept = o.assign_capacity_slots(topk_idx, cap, N)
        assert int((slot < 0).sum()) == case["dropped"], (int((slot < 0).sum()), case)
        assert list(kept) == [min(c, cap) for c in loads]


def pin_capacity_formula(o):
    assert o.capacity_from_factor(1.25, 64, 8) == 10
    assert o.capacity_from_factor(1.0, 4096, 64) == 64
    assert o.capacity_from_factor(1.25, 16384, 256) == 80
    assert o.capacity_from_factor(1.0, 3, 4) == 1          # rounds up
    assert o.capacity_from_factor(1.0, 33, 8) == 5
    assert o.capacity_from_factor(None, 17, 4) == 17      # unlimited
    assert o.capacity_from_factor(float("inf"), 17, 4) == 17


# ----------------------------------------------------------------- hand routing case
def pin_hand_routing(o):
    g = _golden("hand_case_top2_cap1.json")
    L = np.array(g["logits"], dtype=np.float64)
    T, N = L.shape
    cap = o.capacity_from_factor(g["capacity_factor"], T, N)
    assert cap == g["capacity"]
    r = o.route_from_logits(L, g["top_k"], cap)
    assert r["topk_idx"].tolist() == g["topk_idx"]
    np.testing.assert_allclose(r["topk_w"], np.array(g["topk_w"]), rtol=0, atol=1e-15)
    assert r["slot"].tolist() == g["slot"]
    assert r["expert_count"].tolist() == g["expert_count"]
    off, rop, por = o.expert_permutation(r["topk_idx"], r["slot"], r["expert_count"])
    assert off.tolist() == g["expert_offset"]
    assert rop.tolist() == g["row_of_pair"]
    assert por.tolist() == g["pair_of_row"]
    u = g["unlimited"]
    r = o.route_from_logits(L, g["top_k"], u["capacity"])
    assert r["slot"].tolist() == u["slot"]
    assert r["expert_count"].tolist() == u["expert_count"]
    off, rop, por = o.expert_permutation(r["topk_idx"], r["slot"], r["expert_count"])
    assert off.tolist() == u["expert_offset"]
    assert rop.tolist() == u["row_of_pair"]
    assert por.tolist() == u["pair_of_row"]


def pin_logit_bias_hand_case(o):
    """The per-expert logit bias, worked by hand: it enters every token's logits per expert
    (not per token), with a plus sign, before selection and before the weights."""
    g = _golden("hand_case_logit_bias.json")
    x = np.array(g["x"], dtype=np.float64)
    wr = np.array(g["w_router"], dtype=np.float64)
    b = np.array(g["logit_bias"], dtype=np.float64)
    L = o.router_logits(x, wr, b)
    assert L.tolist() == g["logits"], L.tolist()
    T, N = L.shape
    r = o.route_from_logits(L, g["top_k"], T)
    assert r["topk_idx"].tolist() == g["topk_idx"]
    np.testing.assert_allclose(r["topk_w"], np.array(g["topk_w"]), rtol=0, atol=1e-15)
    assert o.route_from_logits(L, 1, T)["topk_idx"].tolist() == g["top1_idx"]
    c1 = g["capacity_1"]
    r = o.route_from_logits(L, g["top_k"], 1)
    assert r["slot"].tolist() == c1["slot"] and r["expert_count"].tolist() == c1["expert_count"]
    # the whole layer routes on the biased logits as well
    out = o.moe_layer_forward(x, wr, np.zeros((N, 2, 2)), np.zeros((N, 2, 1)), top_k=g["top_k"],
                              act="swiglu", capacity=T, logit_bias=b, residual=x)
    assert out["topk_idx"].tolist() == g["topk_idx"]


def pin_top1_weight_is_one(o):
    rng = np.random.default_rng(7)
    L = rng.normal(size=(20, 6))
    r = o.route_from_logits(L, 1, 20)
    assert np.all(r["topk_w"] == 1.0)
    assert r["topk_idx"][:, 0].tolist() == np.argmax(L, axis=1).tolist()


def pin_two_way_weights(o):
    # k=2: w0 = logistic(a - b) for the two chosen logits a > b
    L = np.array([[0.0, 1.0, -3.0, 0.5], [2.0, 2.0, 0.0, 1.0]])
    r = o.route_from_logits(L, 2, 2)
    assert r["topk_idx"].tolist() == [[1, 3], [0, 1]]
    np.testing.assert_allclose(r["topk_w"][0], [0.6224593312018546, 0.3775406687981454], atol=1e-15)
    np.testing.assert_allclose(r["topk_w"][1], [0.5, 0.5], atol=0)


# ----------------------------------------------------------------- brute force
def _brute_topk(row, k):
    """The k-subset whose sorted logits are lexicographically largest; among equal
    ones the lexicographically smallest sorted index tuple; best first."""
    N = len(row)
    best = None
    for S in itertools.combinations(range(N), k):
        vals = tuple(sorted((row[e] for e in S), reverse=True))
        key = (vals, tuple(-e for e in S))
        if best is None or key > best[0]:
            best = (key, S)
    S = best[1]
    return sorted(S, key=lambda e: (-row[e], e))


def _brute_slots(idx, cap):
    """slot(t, j) = number of earlier pairs (in (choice, token) order) with the same expert."""
    T, k = idx.shape
    slot = np.full((T, k), -1)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            rank = sum(1 for jj in range(k) for tt in range(T)
                       if (jj, tt) < (j, t) and idx[tt, jj] == e)
            slot[t, j] = rank if rank < cap else -1
    return slot


def pin_brute_force_routing(o):
    rng = np.random.default_rng(1234)
    for trial in range(60):
        T = int(rng.integers(1, 9))
        N = int(rng.integers(2, 7))
        k = int(rng.integers(1, N + 1))
        # small integers force many exact ties
        L = rng.integers(-2, 3, size=(T, N)).astype(np.float64)
        cap = int(rng.integers(0, T + 1))
        r = o.route_from_logits(L, k, cap)
        for t in range(T):
            assert r["topk_idx"][t].tolist() == _brute_topk(L[t].tolist(), k), (L[t], k)
        assert r["slot"].tolist() == _brute_slots(r["topk_idx"], cap).tolist()
        for e in range(N):
            c_e = int((r["topk_idx"] == e).sum())
            assert r["expert_count"][e] == min(c_e, cap)
        # weights: softmax of the chosen logits, computed directly
        for t in range(T):
            sel = L[t, r["topk_idx"][t]]
            ex = [math.exp(v - sel.max()) for v in sel]
            np.testing.assert_allclose(r["topk_w"][t], [v / sum(ex) for v in ex], rtol=1e-13, atol=0)


# ----------------------------------------------------------------- expert FFN
def pin_ffn_hand_cases(o):
    g = _golden("ffn_hand_cases.json")
    for act in ("swiglu", "gelu"):
        c = g[act]
        y = o.expert_ffn(np.array(c["x"], float), np.array(c["w_gate_up"], float),
                         np.array(c["w_down"], float), act)
        np.testing.assert_allclose(y, np.array(c["y"]), rtol=0, atol=2e-15)


def pin_activation_limits(o):
    z = np.array([0.0, 30.0, -30.0, 1.0, -1.0])
    s = o.silu(z)
    assert s[0] == 0.0 and abs(s[1] - 30.0) < 1e-11 and abs(s[2]) < 1e-11
    np.testing.assert_allclose(s[3] - s[4], 1.0, atol=1e-15)        # silu(z) - silu(-z) = z
    gl = o.gelu(z)
    assert gl[0] == 0.0 and abs(gl[1] - 30.0) < 1e-12 and abs(gl[2]) < 1e-12
    np.testing.assert_allclose(gl[3] - gl[4], 1.0, atol=1e-15)      # gelu(z) - gelu(-z) = z


# ----------------------------------------------------------------- whole layer
def _small_layer(rng, T, d, N, F, act):
    x = rng.normal(size=(T, d))
    wr = rng.normal(size=(N, d)) / math.sqrt(d)
    rows = 2 * F if act == "swiglu" else F
    wgu = rng.normal(size=(N, rows, d)) * 0.3
    wd = rng.normal(size=(N, d, F)) * 0.3
    return x, wr, wgu, wd


def pin_dense_special_case(o):
    """k = N with no capacity limit: sum_e softmax(L)_e * E_e(x) over every expert."""
    rng = np.random.default_rng(99)
    for act in ("swiglu", "gelu"):
        T, d, N, F = 7, 5, 4, 3
        x, wr, wgu, wd = _small_layer(rng, T, d, N, F, act)
        res = rng.normal(size=(T, d))
        got = o.moe_layer_forward(x, wr, wgu, wd, top_k=N, act=act, capacity=T, residual=res)["out"]
        L = x @ wr.T
        want = res.copy()
        for t in range(T):
            ex = np.array([math.exp(v - L[t].max()) for v in L[t]])
            p = ex / ex.sum()
            for e in range(N):
                want[t] += p[e] * o.expert_ffn(x[t:t + 1], wgu[e], wd[e], act)[0]
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def pin_dense_with_logit_bias(o):
    """k = N, no limit, with a per-expert logit bias b: out = r + sum_e softmax(L + b)_e E_e(x),
    the softmax written out term by term from the logits and the bias."""
    rng = np.random.default_rng(41)
    T, d, N, F = 5, 4, 3, 2
    x, wr, wgu, wd = _small_layer(rng, T, d, N, F, "swiglu")
    b = np.array([1.5, -0.75, 0.25])
    got = o.moe_layer_forward(x, wr, wgu, wd, top_k=N, act="swiglu", capacity=T,
                              logit_bias=b, residual=x)["out"]
    want = x.copy()
    for t in range(T):
        z = [sum(x[t, i] * wr[e, i] for i in range(d)) + b[e] for e in range(N)]
        ex = [math.exp(v - max(z)) for v in z]
        for e in range(N):
            want[t] += ex[e] / sum(ex) * o.expert_ffn(x[t:t + 1], wgu[e], wd[e], "swiglu")[0]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def pin_single_expert_layer(o):
    """k = 1 with no limit: out[t] = res[t] + E_argmax(x[t]); token order irrelevant."""
    rng = np.random.default_rng(5)
    T, d, N, F = 9, 4, 3, 2
    x, wr, wgu, wd = _small_layer(rng, T, d, N, F, "swiglu")
    got = o.moe_layer_forward(x, wr, wgu, wd, top_k=1, act="swiglu", capacity=T, residual=x)["out"]
    L = x @ wr.T
    for t in range(T):
        e = int(np.argmax(L[t]))
        want = x[t] + o.expert_ffn(x[t:t + 1], wgu[e], wd[e], "swiglu")[0]
        np.testing.assert_allclose(got[t], want, rtol=1e-13, atol=1e-13)


def pin_invariants(o):
    rng = np.random.default_rng(2024)
    for trial in range(12):
        T = int(rng.integers(4, 40))
        N = int(rng.integers(2, 9))
        k = int(rng.integers(1, min(N, 4) + 1))
        d, F = 6, 4
        x, wr, wgu, wd = _small_layer(rng, T, d, N, F, "swiglu")
        cap = o.capacity_from_factor(float(rng.choice([0.5, 1.0, 1.25])), T, N)
        r = o.moe_layer_forward(x, wr, wgu, wd, top_k=k, act="swiglu", capacity=cap, residual=x)
        np.testing.assert_allclose(r["topk_w"].sum(axis=1), 1.0, rtol=0, atol=1e-14)
        assert np.all(r["expert_count"] <= cap)
        # per expert: kept pairs come before dropped pairs in (choice, token) order
        for e in range(N):
            seen_drop = False
            for j in range(k):
                for t in range(T):
                    if r["topk_idx"][t, j] != e:
                        continue
                    if r["slot"][t, j] < 0:
                        seen_drop = True
                    else:
                        assert not seen_drop
        # a token with every choice dropped leaves the residual unchanged, bit for bit
        all_dropped = np.all(r["slot"] < 0, axis=1)
        assert np.array_equal(r["out"][all_dropped], x[all_dropped])
        # the dropped-pair count obeys sum_e max(0, c_e - cap)
        c = [int((r["topk_idx"] == e).sum()) for e in range(N)]
        assert int((r["slot"] < 0).sum()) == sum(max(0, ce - cap) for ce in c)


def pin_zero_down_weights(o):
    rng = np.random.default_rng(3)
    T, d, N, F = 6, 4, 3, 5
    x, wr, wgu, wd = _small_layer(rng, T, d, N, F, "gelu")
    out = o.moe_layer_forward(x, wr, wgu, np.zeros_like(wd), top_k=2, act="gelu",
                              capacity=T, residual=x)["out"]
    assert np.array_equal(out, x)


def pin_active_params_demo(o_unused=None):
    """The page's active/total parameter arithmetic (router + k experts; router + N experts)."""
    g = _golden("active_params_demo.json")
    d, h, N = g["d_model"], g["hidden"], g["experts"]
    expert = d * h + h + h * d + d
    router = d * N
    assert router + 1 * expert == g["top1_active"]
    assert router + 2 * expert == g["top2_active"]
    assert router + N * expert == g["total"]


# ----------------------------------------------------------------- router statistics
def pin_aux_loss_closed_forms(o):
    alpha = 0.01
    # equal logits and a round-robin top-1 routing: f_i = P_i = 1/N, so the loss is alpha
    T, N = 16, 8
    L = np.zeros((T, N))
    idx = (np.arange(T) % N)[:, None]
    st = o.router_statistics(L, idx, np.zeros((T, 1)), alpha)
    assert abs(st["aux_loss"] - alpha) < 1e-15
    np.testing.assert_allclose(st["prob_mean"], 1.0 / N, atol=1e-15)
    assert st["picks"].tolist() == [2] * N and st["dropped"] == 0
    # collapse: every token sends to expert 0 with probability ~1: the loss tends to alpha * N
    L = np.zeros((T, N))
    L[:, 0] = 60.0
    st = o.router_statistics(L, np.zeros((T, 1), dtype=np.int64), np.full((T, 1), -1), alpha)
    assert abs(st["aux_loss"] - alpha * N) < 1e-12
    assert st["dropped"] == T
    # by hand: t0 = (0, 0) -> p = (1/2, 1/2); t1 = (ln 3, 0) -> p = (3/4, 1/4); both pick
    # expert 0, so f = (1, 0), P = (5/8, 3/8) and the loss is alpha * 2 * 5/8 = 1.25 alpha
    L = np.array([[0.0, 0.0], [math.log(3.0), 0.0]])
    st = o.router_statistics(L, np.array([[0], [0]]), np.array([[0], [1]]), alpha)
    np.testing.assert_allclose(st["prob_mean"], [0.625, 0.375], atol=1e-15)
    assert abs(st["aux_loss"] - 1.25 * alpha) < 1e-15
    # top-2 counts each chosen expert once per token
    st = o.router_statistics(np.zeros((3, 4)), np.array([[0, 1], [1, 2], [3, 0]]),
                             np.array([[0, -1], [0, 0], [0, -1]]), alpha)
    assert st["picks"].tolist() == [2, 2, 1, 1] and st["dropped"] == 2


ALL_PINS = [pin_capacity_demo, pin_capacity_formula, pin_hand_routing, pin_logit_bias_hand_case,
            pin_top1_weight_is_one,
            pin_two_way_weights, pin_brute_force_routing, pin_ffn_hand_cases,
            pin_activation_limits, pin_dense_special_case, pin_dense_with_logit_bias,
            pin_single_expert_layer,
            pin_invariants, pin_zero_down_weights, pin_aux_loss_closed_forms]


# ---------------------------------------------------------------- MX weight formats
# Pins of oracle/mx_oracle.py against the OCP Microscaling (MX) v1.0 definitions (closed
# forms of the scale and element encodings) and against torch's own float8_e4m3fn cast.
def pin_e8m0_closed_forms(m):
    v = m.decode_e8m0(np.array([127, 128, 126, 0, 254, 255]))
    assert v[:5].tolist() == [1.0, 2.0, 0.5, 2.0 ** -127, 2.0 ** 127]
    assert math.isnan(v[5])


def pin_e4m3_closed_forms(m):
    codes = np.array([0x00, 0x80, 0x38, 0xB8, 0x40, 0x7E, 0xFE, 0x08, 0x01, 0x07, 0x3C])
    want = [0.0, -0.0, 1.0, -1.0, 2.0, 448.0, -448.0, 2.0 ** -6, 2.0 ** -9, 7 / 8 * 2.0 ** -6, 1.5]
    assert m.decode_e4m3(codes).tolist() == want
    assert np.isnan(m.decode_e4m3(np.array([0x7F, 0xFF]))).all()


def pin_e4m3_against_torch(m):
    import torch
    codes = np.arange(256)
    got = m.decode_e4m3(codes)
    ref = torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def pin_e2m1_table(m):
    # the spec's FP4 E2M1 magnitudes for codes 0..7; codes 8..15 are their negatives
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    v = m.decode_e2m1(np.arange(16))
    assert v[:8].tolist() == mags
    assert (-v[8:]).tolist() == mags and np.signbit(v[8])


def pin_fp4_nibble_order(m):
    # element 2i is the low nibble of byte i
    assert m.unpack_fp4(np.array([[0x21, 0xF0]])).tolist() == [[1, 2, 0, 15]]


def pin_dequantize_blocks(m):
    # scales are [K/32, rows]: row 0 gets 2^0 then 2^3, row 1 gets 2^2 then 2^-1
    scales = np.array([[127, 129], [130, 126]], dtype=np.uint8)
    w8 = m.dequantize_mx(np.full((2, 64), 0x38, dtype=np.uint8), scales, "mxfp8")  # all 1.0
    assert w8[0].tolist() == [1.0] * 32 + [8.0] * 32
    assert w8[1].tolist() == [4.0] * 32 + [0.5] * 32
    # FP4: byte 0x72 holds codes 2 (1.0, low nibble) and 7 (6.0, high nibble)
    w4 = m.dequantize_mx(np.full((2, 32), 0x72, dtype=np.uint8), scales, "mxfp4")
    assert w4[0].tolist() == [1.0, 6.0] * 16 + [8.0, 48.0] * 16
    assert w4[1].tolist() == [4.0, 24.0] * 16 + [0.5, 3.0] * 16


# MXFP8 activations (block-scaled variant): OCP MX v1.0 conversion, X = 2^(floor(log2 amax) - 8)
def pin_mxfp8_quantize_closed_forms(m):
    def q(block):
        b = np.zeros(32)
        b[:len(block)] = block
        codes, scales = m.quantize_mxfp8(b[None, :])
        return codes[0, :len(block)].tolist(), int(scales[0, 0])
    assert q([1.0] * 32) == ([0x78] * 32, 119)          # amax 1: X = 2^-8, 256 = 1.0 * 2^8
    assert q([448.0, 1.0]) == ([0x7E, 0x38], 127)        # amax 448: X = 1
    assert q([480.0, -511.0]) == ([0x7E, 0xFE], 127)     # (448, 512) saturates to 448
    assert q([256.0, 1.0625, 1.1875, -1.0625]) == ([0x78, 0x38, 0x3A, 0xB8], 127)  # ties to even
    assert q([256.0, 3 / 512, 2.0 ** -10]) == ([0x78, 0x03, 0x00], 127)  # subnormal; half of 2^-9
    assert q([0.0, 0.0]) == ([0, 0], 0)                  # all-zero block: X = 2^-127
    assert q([2.0 ** -130]) == ([0x20], 0)               # X clamped to 2^-127: 2^-3 remains
    assert q([2.0 ** 140]) == ([0x7E], 254)              # X clamped to 2^127: 2^13 saturates
    assert q([20.0, 0.0])[1] == 123                      # floor(log2 20) = 4: X = 2^-4


def pin_mxfp8_encode_against_torch(m):
    import torch
    rng = np.random.default_rng(7)
    mags = np.ldexp(rng.uniform(1.0, 2.0, 4000), rng.integers(-12, 9, 4000))
    v = (np.where(rng.random(4000) < 0.5, -1.0, 1.0) * mags).astype(np.float32)
    v = v[np.abs(v) <= 448.0]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(m.encode_e4m3(v.astype(np.float64)), ref)


def pin_mxfp8_round_trip(m):
    # blocks whose largest element lies in E4M3's top binade [256, 448] come back unchanged
    rng = np.random.default_rng(11)
    codes = rng.integers(0, 0x7F, size=(6, 64)) | (rng.integers(0, 2, size=(6, 64)) << 7)
    codes[:, 0] = 0x7A
    codes[:, 32] = 0xFC
    scales = rng.integers(100, 150, size=(6, 2)).astype(np.uint8)
    c2, s2 = m.quantize_mxfp8(m.dequantize_mxfp8(codes.astype(np.uint8), scales))
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)


def pin_mxfp8_act_ffn_hand_case(m):
    # x = 1.0625 (a tie between 1.0 and 1.125 at X = 2^-8: 1.0 stays); SwiGLU gate 20 x, up x;
    # h = silu(20) = 19.99999996 (X = 2^-4: 319.9999993 -> 320, so 20); y = [1, 0.5] h
    d = F = 32
    x = np.zeros((1, d))
    x[0, 0] = 1.0625
    wgu = np.zeros((2 * F, d))
    wgu[0, 0], wgu[F, 0] = 20.0, 1.0
    wd = np.zeros((d, F))
    wd[0, 0], wd[1, 0] = 1.0, 0.5
    y = m.expert_ffn_mxfp8_act(x, wgu, wd, "swiglu")
    assert y[0, :2].tolist() == [20.0, 10.0] and not y[0, 2:].any()
    # GELU: z = 4 x = 4.0, gelu(4) = 3.99987... (X = 2^-7: 511.98 saturates to 448 -> 3.5)
    wg = np.zeros((F, d))
    wg[0, 0] = 4.0
    y = m.expert_ffn_mxfp8_act(x, wg, wd, "gelu")
    assert y[0, :2].tolist() == [3.5, 1.75]


MX_PINS = [pin_e8m0_closed_forms, pin_e4m3_closed_forms, pin_e4m3_against_torch, pin_e2m1_table,
           pin_fp4_nibble_order, pin_dequantize_blocks, pin_mxfp8_quantize_closed_forms,
           pin_mxfp8_encode_against_torch, pin_mxfp8_round_trip, pin_mxfp8_act_ffn_hand_case]


# ---------------------------------------------------------------- reroute overflow policy
def pin_reroute_hand_case(o):
    # N = 3, k = 1, capacity 1. Token 0 takes expert 0; token 1 overflows expert 0 and goes to
    # its next best expert 2; token 2 overflows expert 0, its next best (1) has room.
    logits = np.array([[3.0, 1.0, 2.0], [3.0, 1.0, 2.0], [3.0, 2.0, 1.0]])
    top = o.select_top_k(logits, 1)
    expert, slot, kept = o.assign_capacity_slots_reroute(top, logits, 1)
    assert expert.tolist() == [[0], [2], [1]]
    assert slot.tolist() == [[0], [0], [0]] and kept.tolist() == [1, 1, 1]
    # a fourth token finds every expert full: dropped, and keeps its own choice
    logits4 = np.vstack([logits, [[0.0, 5.0, 4.0]]])
    expert, slot, kept = o.assign_capacity_slots_reroute(o.select_top_k(logits4, 1), logits4, 1)
    assert expert[3].tolist() == [1] and slot[3].tolist() == [-1]


def pin_reroute_skips_own_choices(o):
    # k = 2, capacity 1, N = 4: token 1's choices are experts 0 and 1 (both taken by token 0
    # in choice order); its redirects skip its own choices and each other: experts 2, then 3.
    logits = np.array([[9.0, 8.0, 1.0, 0.0], [9.0, 8.0, 2.0, 3.0]])
    top = o.select_top_k(logits, 2)
    expert, slot, kept = o.assign_capacity_slots_reroute(top, logits, 1)
    # arrivals: (t0, j0)->0, (t1, j0)->0 full->best free not used {3 (3.0), 2 (2.0)} = 3,
    # (t0, j1)->1, (t1, j1)->1 full-> free and unused: 2
    assert expert.tolist() == [[0, 1], [3, 2]]
    assert slot.tolist() == [[0, 0], [0, 0]] and kept.tolist() == [1, 1, 1, 1]


def pin_reroute_properties(o):
    rng = np.random.default_rng(5)
    for trial in range(40):
        T, N = int(rng.integers(1, 12)), int(rng.integers(2, 7))
        k = int(rng.integers(1, N + 1))
        cap = int(rng.integers(0, 4))
        logits = rng.integers(-3, 4, size=(T, N)).astype(np.float64)  # many ties
        top = o.select_top_k(logits, k)
        expert, slot, kept = o.assign_capacity_slots_reroute(top, logits, cap)
        # without overflow the policy equals dropping
        s0, k0 = o.assign_capacity_slots(top, max(cap, T), N)
        e1, s1, k1 = o.assign_capacity_slots_reroute(top, logits, max(cap, T))
        assert np.array_equal(e1, top) and np.array_equal(s1, s0) and np.array_equal(k1, k0)
        for t in range(T):
            assert len(set(expert[t].tolist())) == k, "a token's pairs use distinct experts"
        assert (kept <= cap).all()
        for e in range(N):  # slots of each expert are 0..kept-1 exactly once
            got = sorted(int(slot[t, j]) for t in range(T) for j in range(k)
                         if expert[t, j] == e and slot[t, j] >= 0)
            assert got == list(range(kept[e]))
        # a dropped pair's token already uses every expert that still has room at the end
        for t in range(T):
            for j in range(k):
                if slot[t, j] < 0:
                    free = {e for e in range(N) if kept[e] < cap}
                    assert free <= set(expert[t].tolist())
        # brute force: replay the arrivals with the "best free unused expert" rule written as
        # an argmax (equal logits to the lower index) instead of a sorted scan
        ex = top.copy()
        cnt = np.zeros(N, dtype=np.int64)
        for j in range(k):
            for t in range(T):
                e = ex[t, j]
                if cnt[e] < cap:
                    cnt[e] += 1
                    continue
                cands = [c for c in range(N) if cnt[c] < cap and c not in set(ex[t].tolist())]
                if cands:
                    best = max(cands, key=lambda c: (logits[t, c], -c))
                    ex[t, j] = best
                    cnt[best] += 1
        assert np.array_equal(ex, expert) and np.array_equal(cnt, kept)


REROUTE_PINS = [pin_reroute_hand_case, pin_reroute_skips_own_choices, pin_reroute_properties]
ALL_PINS = ALL_PINS + REROUTE_PINS
