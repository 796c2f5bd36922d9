"""CPU model of how the redirect kernel decides arrivals, against the oracle's sequential rule.

The kernel (moe_redirect_overflow) does not walk the arrivals one by one. It takes 32 at a
time and decides each from the counts at the window's start:
  * a pair whose expert has room targets it;
  * otherwise the pair targets the first qualifying entry of its token's list of the 16
    experts ranked after its top-k (free slot, not already the token's), or, if every entry
    fails and the list does not hold all the token's other experts, it needs a full scan.
Lanes on the same target take consecutive slots in lane order. The window commits every lane
before the first whose slot passed the capacity, that needs the scan, or whose token already
has an earlier lane in the window; a window's first lane always commits (scanning if it must).
This test replays that procedure in Python on random batches with many ties and checks that
it gives exactly the oracle's sequential result: the claim the kernel's design rests on.
"""
import numpy as np
import pytest

import oracle

LIST = 16
WINDOW = 32


def _lists(logits, k):
    T, N = logits.shape
    out = []
    for t in range(T):
        order = sorted(range(N), key=lambda c: (-logits[t, c], c))
        out.append(order[k:k + LIST])
    return out


def _windowed(logits, topk, cap):
    T, N = logits.shape
    k = topk.shape[1]
    P = T * k
    lists = _lists(logits, k)
    whole = N - k <= LIST
    ex = topk.reshape(-1).copy()
    cnt = np.zeros(N, dtype=np.int64)
    slot = np.full(P, -9, dtype=np.int64)
    room = N if cap > 0 else 0
    a0 = 0
    windows = 0
    while a0 < P:
        windows += 1
        if room == 0:
            for a in range(a0, P):
                j, t = divmod(a, T)
                slot[t * k + j] = -1
            break
        n = min(WINDOW, P - a0)
        lanes = []
        for l in range(n):
            j, t = divmod(a0 + l, T)
            lanes.append((t, t * k + j))
        target, scan = [], []
        for t, q in lanes:
            e = int(ex[q])
            if cnt[e] < cap:
                target.append(e)
                scan.append(False)
                continue
            used = set(int(u) for u in ex[t * k:(t + 1) * k])
            pick = next((c for c in lists[t] if cnt[c] < cap and c not in used), -1)
            target.append(pick)
            scan.append(pick < 0 and not whole)
        first = n
        seen = {}
        tokens = set()
        for l, (t, q) in enumerate(lanes):
            c = cnt[target[l]] + seen.get(target[l], 0) if target[l] >= 0 else -1
            if (target[l] >= 0 and c >= cap) or scan[l] or t in tokens:
                first = l
                break
            if target[l] >= 0:
                seen[target[l]] = seen.get(target[l], 0) + 1
            tokens.add(t)
        if first == 0:  # the first lane needs the full scan
            t, q = lanes[0]
            used = set(int(u) for u in ex[t * k:(t + 1) * k])
            cands = [c for c in range(N) if cnt[c] < cap and c not in used]
            if cands:
                best = min(cands, key=lambda c: (-logits[t, c], c))
                slot[q] = cnt[best]
                cnt[best] += 1
                ex[q] = best
                room -= int(cnt[best] == cap)
            else:
                slot[q] = -1
            a0 += 1
            continue
        for l in range(first):
            t, q = lanes[l]
            e = target[l]
            if e < 0:
                slot[q] = -1
                continue
            slot[q] = cnt[e]
            cnt[e] += 1
            ex[q] = e
            room -= int(cnt[e] == cap)
        a0 += first
    return ex.reshape(T, k), slot.reshape(T, k), cnt, windows


@pytest.mark.parametrize("seed", range(6))
def test_window_procedure_equals_sequential_rule(seed):
    rng = np.random.default_rng(seed)
    for _ in range(40):
        T = int(rng.integers(1, 120))
        N = int(rng.integers(1, 60))
        k = int(rng.integers(1, min(8, N) + 1))
        if rng.random() < 0.5:
            logits = rng.integers(-3, 4, size=(T, N)).astype(np.float64) * 0.5  # many ties
        else:
            logits = rng.normal(size=(T, N)) + np.linspace(0.0, 2.0, N)      # skewed load
        cap = min(int(rng.integers(0, 2 * T * k // N + 2)), T)
        want = oracle.route_from_logits(logits, k, cap, reroute=True)
        ex, slot, cnt, _ = _windowed(logits, oracle.select_top_k(logits, k), cap)
        assert np.array_equal(ex, want["topk_idx"])
        assert np.array_equal(slot, want["slot"])
        assert np.array_equal(cnt, want["expert_count"])


def test_windows_are_fewer_than_arrivals_on_a_switch_like_batch():
    """4096 top-1 pairs over 64 experts at capacity factor 1: most windows commit many lanes."""
    rng = np.random.default_rng(11)
    T, N, k = 4096, 64, 1
    logits = rng.normal(size=(T, N)) + np.linspace(0.0, 1.5, N)
    cap = oracle.capacity_from_factor(1.0, T, N)
    want = oracle.route_from_logits(logits, k, cap, reroute=True)
    ex, slot, cnt, windows = _windowed(logits, oracle.select_top_k(logits, k), cap)
    assert np.array_equal(slot, want["slot"])
    assert windows < T // 8
