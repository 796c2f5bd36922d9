"""CPU oracle for the forward pass of a sparse Mixture-of-Experts layer.

TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
CPU-baseline leg may import or run this module. The product (the CUDA library
and its Python binding) never calls it, and it shares no code with the product:
no kernels, helpers, tables or constants. Both sides get their inputs from the
seeded generators in ``synthetic.py``, which hold none of the layer's arithmetic.

Everything here is deliberately plain: float64 numpy, one step per function, in
the order the pages give them, with a library matmul as the only building block.
Sources (cited by page title and section):

* page «Sparse Mixture-of-Experts» (bigdataschool wiki), sections
  «Роутер и top-k gating» (router, softmax, top-k, renormalisation, weighted sum),
  «Expert capacity и capacity factor» (capacity formula, dropping, residual pass-through),
  «Подводные камни collapse экспертов и token dropping» (first-come-first-served fill),
  «Демо top-k router на PyTorch» (the eager per-slot / per-expert loop, the
  token-order slot loop, the parameter arithmetic);
* page «Что такое Mixture of Experts (MoE) в трансформерах: архитектура и
  параллелизм» (aglamov.biz), sections «Динамическая загрузка весов с
  WeightConverter» (packed gate_up_proj / down_proj layout) and «Бэкенд для
  экспертов» (eager loop as the correctness reference; grouped_mm sorts tokens by
  expert id).

Readings where the pages are silent (each listed in the design notes):

* selection is made on the logits (softmax is strictly increasing, so this picks
  the same experts as selecting on probabilities); equal logits go to the lower
  expert index;
* the capacity is ceil(capacity_factor * T / N) slots per expert, not scaled by k;
  "no capacity limit" means capacity T;
* with k > 1, slots are filled choice by choice: every token's first choice in
  token order, then every token's second choice, and so on;
* a dropped (token, choice) pair contributes nothing and the surviving weights
  are not renormalised again;
* the layer returns residual + sum of weighted expert outputs;
* experts are bias-free; SwiGLU is silu(x W_g^T) * (x W_u^T) then W_d; GELU is the
  exact erf form.

Array conventions: every floating-point array is float64 holding the exact
values the GPU used (bf16 or fp32 values widen to float64 exactly).
"""
from __future__ import annotations

import math
from typing import Callable, Optional, Sequence, Union

import numpy as np
from scipy.special import erf as _erf

UNLIMITED = None


# --------------------------------------------------------------------------
# capacity  (page «Sparse Mixture-of-Experts», «Expert capacity и capacity factor»)
# --------------------------------------------------------------------------
def capacity_from_factor(capacity_factor: Optional[float], T: int, n_experts: int) -> int:
    """Slots per expert: capacity_factor * tokens_in_batch / experts, rounded up.

    ``None``, a non-positive or an infinite factor means no limit, which is T slots:
    a token picks each expert at most once, so T slots can never overflow.
    """
    if capacity_factor is None or not math.isfinite(capacity_factor) or capacity_factor <= 0:
        return T
    return int(math.ceil(capacity_factor * T / n_experts))


# --------------------------------------------------------------------------
# router  (page «Sparse Mixture-of-Experts», «Роутер и top-k gating»)
# --------------------------------------------------------------------------
def router_logits(x: np.ndarray, w_router: np.ndarray,
                  logit_bias: Optional[np.ndarray] = None) -> np.ndarray:
    """Linear router without bias term: logits[t, e] = sum_i x[t, i] * W_r[e, i].

    ``logit_bias`` is an optional per-expert additive term on the logits (used
    only to skew the synthetic load); it enters both selection and weights.
    """
    logits = x @ w_router.T
    if logit_bias is not None:
        logits = logits + logit_bias[None, :]
    return logits


def softmax_over_experts(logits: np.ndarray) -> np.ndarray:
    """p[t, e] = exp(logit[t, e]) / sum_e' exp(logit[t, e']), max-shifted for range."""
    z = logits - logits.max(axis=1, keepdims=True)
    ez = np.exp(z)
    return ez / ez.sum(axis=1, keepdims=True)


def select_top_k(logits: np.ndarray, k: int) -> np.ndarray:
    """The k experts with the largest scores per token, best first.

    Order: larger logit first; equal logits ordered by lower expert index.
    """
    T, N = logits.shape
    idx = np.empty((T, k), dtype=np.int64)
    experts = np.arange(N)
    for t in range(T):
        order = np.lexsort((experts, -logits[t]))  # primary key: -logit; then index
        idx[t] = order[:k]
    return idx


def renormalise(probs: np.ndarray, topk_idx: np.ndarray) -> np.ndarray:
    """Weights of the chosen experts rescaled to sum to one: p_j / sum_selected p."""
    sel = np.take_along_axis(probs, topk_idx, axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


# --------------------------------------------------------------------------
# capacity slots and dropping
# (page «Sparse Mixture-of-Experts», «Expert capacity и capacity factor»; the
#  first-come-first-served token loop of the second demo script)
# --------------------------------------------------------------------------
def assign_capacity_slots(topk_idx: np.ndarray, capacity: int, n_experts: int):
    """Give each (token, choice) pair a slot in its expert's buffer, in arrival order.

    Arrival order: all tokens' choice 0 in token order, then all tokens' choice 1,
    and so on. A pair that arrives at a full expert is dropped (slot -1).
    Returns (slot [T, k], kept_count [N]).
    """
    T, k = topk_idx.shape
    filled = np.zeros(n_experts, dtype=np.int64)
    slot = np.full((T, k), -1, dtype=np.int64)
    for j in range(k):
        for t in range(T):
            e = int(topk_idx[t, j])
            if filled[e] < capacity:
                slot[t, j] = filled[e]
                filled[e] += 1
    return slot, filled


def assign_capacity_slots_reroute(topk_idx: np.ndarray, logits: np.ndarray, capacity: int):
    """Overflow policy "redirect to the next most suitable expert" (page «Архитектура MoE в
    больших языковых моделях — кто такие «эксперты»?» (gerwin.io), section «Как работает MoE:
    принцип маршрутизации», the load-balancing list: exceeding an expert's capacity may drop
    tokens or redirect them to the next most suitable expert).

    Reading (the page names the policy only): pairs arrive in the same order as for
    dropping (choice 0 of every token in token order, then choice 1, ...). A pair whose
    expert is full goes instead to the token's most probable expert (largest logit, equal
    logits to the lower index) that has a free slot and that the token does not already
    use: neither another of its top-k choices nor an earlier redirect. If no expert
    qualifies, the pair is dropped. A redirected pair keeps its router weight.
    Returns (expert [T, k] serving each pair, slot [T, k], kept_count [N]).
    """
    T, k = topk_idx.shape
    n_experts = logits.shape[1]
    expert = np.array(topk_idx, dtype=np.int64, copy=True)
    filled = np.zeros(n_experts, dtype=np.int64)
    slot = np.full((T, k), -1, dtype=np.int64)
    for j in range(k):
        for t in range(T):
            e = int(expert[t, j])
            if filled[e] < capacity:
                slot[t, j] = filled[e]
                filled[e] += 1
                continue
            used = {int(u) for u in expert[t]}
            # candidates in the token's order of preference
            order = sorted(range(n_experts), key=lambda c: (-logits[t, c], c))
            for c in order:
                if c not in used and filled[c] < capacity:
                    expert[t, j] = c
                    slot[t, j] = filled[c]
                    filled[c] += 1
                    break
    return expert, slot, filled


def route_from_logits(logits: np.ndarray, k: int, capacity: int, reroute: bool = False) -> dict:
    """Softmax, top-k, renormalise and capacity assignment for given logits. With reroute,
    overflowing pairs go to the next most suitable expert (topk_idx then holds the expert
    serving each pair; the weights are the router's)."""
    n_experts = logits.shape[1]
    probs = softmax_over_experts(logits)
    topk_idx = select_top_k(logits, k)
    topk_w = renormalise(probs, topk_idx)
    if reroute:
        topk_idx, slot, kept = assign_capacity_slots_reroute(topk_idx, logits, capacity)
    else:
        slot, kept = assign_capacity_slots(topk_idx, capacity, n_experts)
    return {"topk_idx": topk_idx, "topk_w": topk_w, "slot": slot, "expert_count": kept}


# --------------------------------------------------------------------------
# sort by expert id  (page «Что такое Mixture of Experts (MoE) в трансформерах»,
# «Бэкенд для экспертов», grouped_mm: tokens sorted by expert id and grouped)
# --------------------------------------------------------------------------
def expert_permutation(topk_idx: np.ndarray, slot: np.ndarray, expert_count: np.ndarray):
    """Expert-contiguous row order of the kept pairs.

    expert_offset[e] = number of kept pairs of experts < e; a kept pair (t, j) of
    expert e with slot s lives in row expert_offset[e] + s. Dropped pairs get -1.
    pair_of_row[row] = t * k + j is the inverse map.
    """
    T, k = topk_idx.shape
    n_experts = expert_count.shape[0]
    expert_offset = np.zeros(n_experts + 1, dtype=np.int64)
    for e in range(n_experts):
        expert_offset[e + 1] = expert_offset[e] + expert_count[e]
    row_of_pair = np.full((T, k), -1, dtype=np.int64)
    pair_of_row = np.full(int(expert_offset[-1]), -1, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            if slot[t, j] >= 0:
                r = expert_offset[topk_idx[t, j]] + slot[t, j]
                row_of_pair[t, j] = r
                pair_of_row[r] = t * k + j
    return expert_offset, row_of_pair, pair_of_row


# --------------------------------------------------------------------------
# experts  (page «Sparse Mixture-of-Experts», «Архитектура и ключевые особенности»:
# an expert is an ordinary transformer FFN; packed layout from page «Что такое
# Mixture of Experts (MoE) в трансформерах», «Динамическая загрузка весов с
# WeightConverter»: gate_up_proj = experts' w1 then w3 stacked along the row axis)
# --------------------------------------------------------------------------
def silu(z: np.ndarray) -> np.ndarray:
    """z * logistic(z) = z / (1 + exp(-z))."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def gelu(z: np.ndarray) -> np.ndarray:
    """Exact GELU: z * Phi(z) = 0.5 * z * (1 + erf(z / sqrt(2)))."""
    return 0.5 * z * (1.0 + _erf(z / math.sqrt(2.0)))


def expert_ffn(rows: np.ndarray, w_gate_up: np.ndarray, w_down: np.ndarray, act: str) -> np.ndarray:
    """One expert applied to the rows routed to it.

    SwiGLU: w_gate_up is [2F, d] (gate rows first, then up rows), w_down is [d, F];
            y = (silu(rows W_g^T) * (rows W_u^T)) W_d^T.
    GELU:   w_gate_up is [F, d], w_down is [d, F]; y = gelu(rows W_1^T) W_2^T.
    """
    if act == "swiglu":
        F = w_gate_up.shape[0] // 2
        g = rows @ w_gate_up[:F].T
        u = rows @ w_gate_up[F:].T
        h = silu(g) * u
    elif act == "gelu":
        h = gelu(rows @ w_gate_up.T)
    else:
        raise ValueError(f"unknown activation {act!r}")
    return h @ w_down.T


ExpertWeights = Union[np.ndarray, Sequence[np.ndarray], Callable[[int], np.ndarray]]


def _expert(weights: ExpertWeights, e: int) -> np.ndarray:
    return weights(e) if callable(weights) else weights[e]


# --------------------------------------------------------------------------
# the layer: eager per-choice / per-expert loop
# (page «Sparse Mixture-of-Experts», «Демо top-k router на PyTorch», run_moe;
#  residual pass-through from «Expert capacity и capacity factor»)
# --------------------------------------------------------------------------
def combine(x: np.ndarray, routing: dict, w_gate_up: ExpertWeights, w_down: ExpertWeights,
            act: str, residual: Optional[np.ndarray], tokens: Optional[np.ndarray] = None,
            ffn: Callable = None) -> np.ndarray:
    """out[t] = residual[t] + sum over kept choices j of w[t, j] * E_{idx[t, j]}(x[t]).

    The loop runs over choices j, then experts e, as in the pages' eager loop;
    dropped pairs are skipped. ``tokens`` restricts the output to a subset of
    token indices (a token's output depends only on its own kept pairs). ``ffn`` is the
    expert (expert_ffn unless given; the MXFP8-activation variant passes its own).
    """
    if ffn is None:
        ffn = expert_ffn
    topk_idx, topk_w, slot = routing["topk_idx"], routing["topk_w"], routing["slot"]
    T, k = topk_idx.shape
    if tokens is None:
        tokens = np.arange(T)
    tokens = np.asarray(tokens, dtype=np.int64)
    d = x.shape[1]
    out = np.zeros((tokens.shape[0], d)) if residual is None else residual[tokens].astype(np.float64).copy()
    idx_sub, w_sub, slot_sub = topk_idx[tokens], topk_w[tokens], slot[tokens]
    n_experts = int(routing["expert_count"].shape[0])
    for j in range(k):
        for e in range(n_experts):
            mask = (idx_sub[:, j] == e) & (slot_sub[:, j] >= 0)
            if not mask.any():
                continue
            y = ffn(x[tokens[mask]], _expert(w_gate_up, e), _expert(w_down, e), act)
            out[mask] += w_sub[mask, j][:, None] * y
    return out


def moe_layer_forward(x: np.ndarray, w_router: np.ndarray, w_gate_up: ExpertWeights,
                      w_down: ExpertWeights, *, top_k: int, act: str, capacity: int,
                      logit_bias: Optional[np.ndarray] = None,
                      residual: Optional[np.ndarray] = None,
                      tokens: Optional[np.ndarray] = None) -> dict:
    """Whole layer: router -> softmax -> top-k -> renormalise -> capacity -> experts -> sum."""
    logits = router_logits(x, w_router, logit_bias)
    routing = route_from_logits(logits, top_k, capacity)
    out = combine(x, routing, w_gate_up, w_down, act, residual, tokens)
    return {"logits": logits, "out": out, **routing}


# --------------------------------------------------------------------------
# router statistics and the auxiliary load-balancing loss
# (page «Sparse Mixture-of-Experts», section «Маршрутизация токена и auxiliary loss»;
#  the auxiliary_loss function of the second demo script)
# --------------------------------------------------------------------------
def router_statistics(logits: np.ndarray, topk_idx: np.ndarray, slot: np.ndarray,
                      alpha: float = 1e-2) -> dict:
    """Per-expert load and router confidence over the batch, and the auxiliary loss.

    picks[e]     number of (token, choice) pairs that chose expert e, before the capacity
    prob_mean[e] P_e: mean over the batch of the router's softmax probability of expert e
    f[e]         fraction of the batch's tokens sent to expert e: picks[e] / T
    aux_loss     alpha * N * sum_e f[e] * P_e
    dropped      number of pairs that found their expert full
    """
    T, N = logits.shape
    probs = softmax_over_experts(logits)
    picks = np.zeros(N, dtype=np.int64)
    for t in range(T):
        for e in topk_idx[t]:
            picks[int(e)] += 1
    prob_mean = probs.mean(axis=0)
    f = picks / T
    aux = alpha * N * float((f * prob_mean).sum())
    return {"picks": picks, "prob_mean": prob_mean, "aux_loss": aux,
            "dropped": int((np.asarray(slot) < 0).sum())}
