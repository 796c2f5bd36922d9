"""Shared helpers of the GPU parity tests: run the CUDA path stage by stage or as one
moe_forward call, and compare what it produced with the CPU oracle.

Matching rules (tolerances are written here once and used by every parity test):

* logits: |gpu - oracle| <= 1e-4 * max(1, |oracle|) element-wise;
* routing (expert ids, slots, kept counts, offsets, rows, permutation): bit-exact against the
  oracle re-run on the GPU's own fp32 logits; weights within 2e-6 absolute;
* x_perm rows: bit-exact copies of x;
* outputs: fp32-output mode within max-abs 2e-2 and mean-rel 1e-2 of the fp64 oracle; the
  bf16 output within 2e-2 + half a bf16 ulp of the oracle value (the bf16 rounding of the exact
  answer alone can exceed 2e-2 once |out| >= 8) and mean-rel 1e-2; the MoE contribution
  (out - residual, fp32 mode) within mean-rel 1e-2 of the oracle's;
* tokens with every choice dropped: output bits equal to the residual's bits;
* expert rows (y_perm, an fp32 intermediate the target states no bar for): max-abs within
  2e-2 * max(1, rms of the oracle's row) and mean-rel 1e-2. The kernels round h to bf16 once
  (2^-9 relative); summed over d_ff terms that leaves an error of about 0.17 % of the row's rms
  (Mixtral-shaped expert, d_ff = 14336: rms(y) 2.4, largest error per 4096-element row 0.013 to
  0.017 in a float64 simulation of that rounding alone), which a fixed 2e-2 does not cover
  once rms(y) > 1.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import sparse_mixture_experts_11_b200 as moe

LOGIT_RTOL = 1e-4
WEIGHT_ATOL = 2e-6
OUT_MAX_ABS = 2e-2
OUT_MEAN_REL = 1e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def y_row_max_abs(want_row: np.ndarray) -> float:
    """Max-abs bar of one expert output row (see the module notes)."""
    return OUT_MAX_ABS * max(1.0, float(np.sqrt(np.mean(np.square(want_row)))))


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |v| (8 significand bits)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 0.5 * 2.0 ** (e - 7)


def mean_rel(g: np.ndarray, o: np.ndarray) -> float:
    den = np.abs(o).sum()
    return float(np.abs(g - o).sum() / den) if den > 0 else float(np.abs(g - o).sum())


class StageRun:
    """Runs route -> permute -> grouped_ffn -> combine through the C ABI on fresh buffers."""

    def __init__(self, inp: dict, top_k: int, act: str, cap: int, device="cuda"):
        x = inp["x"]
        T, d = x.shape
        N = inp["w_router"].shape[0]
        # MX weights: [N, F/32, d] down-projection scales give F
        F = inp["w_down"].shape[2] if "w_down" in inp else 32 * inp["w_down_s"].shape[1]
        self.dims = moe.make_dims(T, d, N, top_k, F, act, cap)
        R = moe.max_rows(self.dims)
        self.R_max = R
        dev = device
        # block-scaled MX formats: quantised activations, room for them after the workspace
        self.block_scaled = str(inp.get("wfmt", "")).endswith("_bs")
        self.ws = moe.new_workspace(self.dims, dev, block_scaled=self.block_scaled)
        z = lambda shape, dt: torch.full(shape, -7, dtype=dt, device=dev) if dt == torch.int32 \
            else torch.full(shape, float("nan"), dtype=dt, device=dev)
        self.logits = z((T, N), torch.float32)
        self.topk_idx = z((T, top_k), torch.int32)
        self.topk_w = z((T, top_k), torch.float32)
        self.slot = z((T, top_k), torch.int32)
        self.expert_count = z((N,), torch.int32)
        self.expert_offset = z((N + 1,), torch.int32)
        self.row_of_pair = z((T, top_k), torch.int32)
        self.pair_of_row = z((R,), torch.int32)
        self.x_perm = torch.zeros((R, d), dtype=torch.bfloat16, device=dev)
        self.h = torch.zeros((R, F), dtype=torch.bfloat16, device=dev)
        self.y_perm = torch.zeros((R, d), dtype=torch.float32, device=dev)
        self.out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
        self.out32 = torch.empty((T, d), dtype=torch.float32, device=dev)
        self.inp = inp
        if "wfmt" in inp:
            self.mx = moe.mx_weights(self.dims, inp["wfmt"], inp["w_gate_up_q"], inp["w_gate_up_s"],
                                     inp["w_down_q"], inp["w_down_s"])
            self.gu, self.dn = mx_weight_getters(inp)
        else:
            self.mx = None
            self.gu, self.dn = expert_weights_f64(inp["w_gate_up"]), expert_weights_f64(inp["w_down"])

    def run(self, residual=True, redirect=False):
        i = self.inp
        res = i["x"] if residual else None
        moe.route(self.dims, i["x"], i["w_router"], i.get("logit_bias"), self.logits, self.topk_idx,
                  self.topk_w, self.slot, self.expert_count, self.ws)
        if redirect:
            moe.redirect_overflow(self.dims, self.logits, self.topk_idx, self.slot,
                                  self.expert_count, self.ws)
        moe.permute(self.dims, i["x"], self.topk_idx, self.slot, self.expert_count,
                    self.expert_offset, self.row_of_pair, self.pair_of_row, self.x_perm, self.ws)
        if self.mx is not None:
            moe.grouped_ffn_mx(self.dims, self.x_perm, self.expert_offset, self.mx, self.h,
                               self.y_perm, self.ws)
        else:
            moe.grouped_ffn(self.dims, self.x_perm, self.expert_offset, i["w_gate_up"],
                            i["w_down"], self.h, self.y_perm, self.ws)
        moe.unpermute_combine(self.dims, self.y_perm, self.row_of_pair, self.topk_w, res, self.out,
                              self.ws)
        moe.unpermute_combine(self.dims, self.y_perm, self.row_of_pair, self.topk_w, res, self.out32,
                              self.ws)
        torch.cuda.synchronize()
        err = moe.read_device_error(self.ws)
        assert err == 0, f"device status {err}: {moe.status_string(err)}"
        return self


def check_logits(gpu_logits: np.ndarray, x: np.ndarray, w_router: np.ndarray, bias, rows=None):
    xs = x if rows is None else x[rows]
    want = oracle.router_logits(xs, w_router, bias)
    got = gpu_logits if rows is None else gpu_logits[rows]
    bad = np.abs(got - want) > LOGIT_RTOL * np.maximum(1.0, np.abs(want))
    assert not bad.any(), f"{bad.sum()} logits off; worst {np.abs(got - want).max()}"


def check_routing(run: StageRun, cap: int, reroute=False):
    """Routing bit-exact against the oracle re-run on the GPU's own logits."""
    L = f64(run.logits)
    k = run.dims.top_k
    r = oracle.route_from_logits(L, k, cap, reroute=reroute)
    g_idx = run.topk_idx.cpu().numpy()
    assert np.array_equal(g_idx, r["topk_idx"]), "expert ids differ"
    np.testing.assert_allclose(f64(run.topk_w), r["topk_w"], rtol=0, atol=WEIGHT_ATOL)
    assert np.array_equal(run.slot.cpu().numpy(), r["slot"]), "slots differ"
    assert np.array_equal(run.expert_count.cpu().numpy(), r["expert_count"]), "kept counts differ"
    off, rop, por = oracle.expert_permutation(r["topk_idx"], r["slot"], r["expert_count"])
    assert np.array_equal(run.expert_offset.cpu().numpy(), off), "expert offsets differ"
    assert np.array_equal(run.row_of_pair.cpu().numpy(), rop), "row_of_pair differs"
    R = int(off[-1])
    assert np.array_equal(run.pair_of_row[:R].cpu().numpy(), por), "pair_of_row differs"
    return r, off, rop


def check_x_perm(run: StageRun, rop: np.ndarray):
    T, k = rop.shape
    tok = np.repeat(np.arange(T), k).reshape(T, k)
    kept = rop >= 0
    rows = torch.from_numpy(rop[kept]).long().cuda()
    toks = torch.from_numpy(tok[kept]).long().cuda()
    a = run.x_perm.index_select(0, rows).view(torch.int16)
    b = run.inp["x"].index_select(0, toks).view(torch.int16)
    assert torch.equal(a, b), "x_perm rows are not bit copies of x"


def expert_weights_f64(w: torch.Tensor):
    """Lazy per-expert float64 view of a packed expert tensor (read back one expert at a time)."""
    cache = {}

    def get(e):
        if e not in cache:
            cache[e] = f64(w[e])
        return cache[e]
    return get


def mx_weight_getters(inp):
    """Lazy per-expert float64 weights decoded from MX storage by the oracle."""
    fmt = inp["wfmt"]
    fmt = fmt[:-3] if fmt.endswith("_bs") else fmt

    def make(q, sc):
        cache = {}

        def get(e):
            if e not in cache:
                cache[e] = oracle.dequantize_mx(q[e].cpu().numpy(), sc[e].cpu().numpy(), fmt)
            return cache[e]
        return get
    return make(inp["w_gate_up_q"], inp["w_gate_up_s"]), make(inp["w_down_q"], inp["w_down_s"])


def expert_ffn_of(run: StageRun):
    """The oracle's expert for this run: MXFP8-quantised activations on the block-scaled path."""
    return oracle.expert_ffn_mxfp8_act if getattr(run, "block_scaled", False) else oracle.expert_ffn


def check_outputs(run: StageRun, routing: dict, act: str, tokens=None, residual=True):
    i = run.inp
    x = f64(i["x"])
    res = x if residual else None
    want = oracle.combine(x, routing, run.gu, run.dn, act, res, tokens, ffn=expert_ffn_of(run))
    sel = slice(None) if tokens is None else torch.from_numpy(np.asarray(tokens)).long().cuda()
    g32 = f64(run.out32[sel])
    g16 = f64(run.out[sel])
    # fp32-output mode: the plain bar
    err32 = np.abs(g32 - want)
    assert err32.max() <= OUT_MAX_ABS, f"fp32 out max-abs {err32.max()}"
    assert mean_rel(g32, want) <= OUT_MEAN_REL, f"fp32 out mean-rel {mean_rel(g32, want)}"
    # bf16 output
    err16 = np.abs(g16 - want)
    bound = OUT_MAX_ABS + bf16_half_ulp(want)
    assert (err16 <= bound).all(), f"bf16 out off by {(err16 - bound).max()} beyond bound"
    assert mean_rel(g16, want) <= OUT_MEAN_REL
    # the MoE contribution alone, relative to its own size
    if residual:
        xs = x if tokens is None else x[np.asarray(tokens)]
        c_g, c_o = g32 - xs, want - xs
        if np.abs(c_o).sum() > 0:
            assert mean_rel(c_g, c_o) <= OUT_MEAN_REL, f"contribution mean-rel {mean_rel(c_g, c_o)}"
    return float(err32.max()), float(mean_rel(g32, want))


def check_dropped_tokens_pass_through(run: StageRun, slot: np.ndarray, residual=True):
    all_dropped = np.all(slot < 0, axis=1)
    if not all_dropped.any():
        return 0
    idx = torch.from_numpy(np.nonzero(all_dropped)[0]).long().cuda()
    got = run.out.index_select(0, idx).view(torch.int16)
    if residual:
        want = run.inp["x"].index_select(0, idx).view(torch.int16)
        assert torch.equal(got, want), "a fully dropped token changed"
    else:
        assert torch.all(got == 0)
    return int(all_dropped.sum())


def check_expert_rows(run: StageRun, routing: dict, act: str, rows: np.ndarray):
    """y_perm rows against the oracle expert FFN applied to the token the row came from."""
    off = run.expert_offset.cpu().numpy()
    por = run.pair_of_row.cpu().numpy()
    k = run.dims.top_k
    x = run.inp["x"]
    gu, dn = run.gu, run.dn
    y = f64(run.y_perm[torch.from_numpy(rows).long().cuda()])
    for n, r in enumerate(rows):
        e = int(np.searchsorted(off, r, side="right") - 1)
        t = int(por[r]) // k
        want = expert_ffn_of(run)(f64(x[t:t + 1]), gu(e), dn(e), act)[0]
        err = np.abs(y[n] - want)
        assert err.max() <= y_row_max_abs(want), f"row {r} (expert {e}, token {t}) max-abs {err.max()}"
        assert mean_rel(y[n], want) <= OUT_MEAN_REL


def sample_tokens(routing: dict, n: int, max_experts: int, seed: int = 0) -> np.ndarray:
    """Up to n tokens whose kept pairs touch at most max_experts distinct experts."""
    rng = np.random.default_rng(seed)
    T = routing["topk_idx"].shape[0]
    chosen, experts = [], set()
    for t in rng.permutation(T):
        kept = {int(e) for e, s in zip(routing["topk_idx"][t], routing["slot"][t]) if s >= 0}
        if len(experts | kept) <= max_experts:
            chosen.append(int(t))
            experts |= kept
        if len(chosen) >= n:
            break
    return np.array(sorted(chosen), dtype=np.int64)
