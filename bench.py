#!/usr/bin/env python
"""Benchmark: sparse MoE layer forward tokens/s on B200 (one JSON line on rank 0).

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME[:T]] [--impl ours|reference]

A step is one whole forward pass of the layer (route, permute, grouped expert FFN, combine)
over one batch of synthetic tokens whose inputs already sit in HBM. The forward (moe_forward)
is captured once as a CUDA graph; a timed step replays it between two CUDA events on the
launching stream. Steps are timed one by one; before each step, outside the timed events, L2
is flushed: a 256 MB write, then a 256 MB read of a second buffer that takes the write's
write-back. A second pass replays the stages as separate graphs with events between them for
the per-stage breakdown and the grouped FFN's roofline. The end-to-end figure (e2e) calls
moe_forward eagerly, with the H2D copy of the tokens and the D2H copy of the output of every
step inside its timed region; the copies run on their own streams and overlap the
neighbouring steps' compute. Its `copies_only` entry times the same copies with no forward
between them, the host link's floor under the end-to-end figure. Under torchrun every rank runs its own replica of the workload
(weak scaling, no collective on the data path). Rank 0 prints the line, with the time taken
as the max over ranks.

--impl reference times the CPU oracle (the plain float64 definition of the layer) on a bounded
token sample of the same workload, on the host cores, as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

DEFAULT_WORKLOAD = "fine_grained:16384"   # the largest workload that fits one GPU
# every workload point of the five layer shapes, measured in one run (the "sweep" key)
SWEEP = ("tiny_top2:64", "switch_top1:4096", "mixtral:1", "mixtral:16", "mixtral:512",
         "mixtral:8192", "gpt_oss:1", "gpt_oss:8", "gpt_oss:64", "gpt_oss:16384",
         "fine_grained:16384")
DECODE_MIN_STEPS = 100  # sweep points with T <= 64 time at least this many steps
SWEEP_SETTLE_S = 2.0    # idle seconds before each sweep point
METRIC = "MoE-layer fwd tokens/s on 1 B200; % of bf16 tensor peak / % of HBM BW"
MEASURED_PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SLOT_CHUNK = 4096  # (token, choice) pairs per block in the library's capacity pass


# ----------------------------------------------------------------------------- workload model
def parse_workload(spec: str):
    name, _, t = spec.partition(":")
    shape = synthetic.SHAPES[name]
    T = int(t) if t else shape.token_counts[-1]
    return shape, T


def capacity_of(shape, T):
    import sparse_mixture_experts_11_b200 as moe
    return moe.capacity(shape.capacity_factor, T, shape.n_experts)


def expert_params(d_model: int, d_ff: int, act: str, bias: bool = False) -> int:
    """Parameters of one expert FFN: SwiGLU has gate, up and down projections; GELU up and down.
    With bias=True each projection also carries a bias vector (the pages' demo expert)."""
    if act == "swiglu":
        n = 3 * d_model * d_ff
        return n + (2 * d_ff + d_model if bias else 0)
    n = 2 * d_model * d_ff
    return n + (d_ff + d_model if bias else 0)


def active_params(d_model: int, d_ff: int, n_experts: int, k: int, act: str, bias: bool) -> int:
    """Parameters touched per token: the bias-free router plus k experts."""
    return d_model * n_experts + k * expert_params(d_model, d_ff, act, bias)


def weight_bytes(params: int, wfmt: str = "bf16") -> int:
    """Bytes of `params` expert weights in storage: bf16 2 B each; MX formats one E8M0 scale
    byte per 32 elements plus 1 B (MXFP8) or 1/2 B (MXFP4) per element."""
    if wfmt == "bf16":
        return params * 2
    return (params if wfmt.startswith("mxfp8") else params // 2) + params // 32


def algorithmic_bytes(shape, T: int, active_experts: int, R: int, wfmt: str = "bf16") -> dict:
    """Bytes the layer must move (counting rules in the design notes).

    weights: every expert with at least one kept row, read once (idle experts cost nothing).
             This is the grouped FFN's algorithmic traffic: its intermediates (x_perm, h,
             y_perm) are implementation overhead and are measured by ncu, not counted.
    layer:   the same expert weights; router weight (fp32); x read (bf16); out written (bf16).
             The residual is x itself.
    rows:    the FFN's intermediate rows, for reference: x_perm read (bf16), y_perm written (fp32).
    """
    d, F, N = shape.d_model, shape.d_ff, shape.n_experts
    w = active_experts * weight_bytes(expert_params(d, F, shape.act), wfmt)
    layer = w + N * d * 4 + T * d * 2 + T * d * 2
    return {"layer": layer, "weights": w, "rows": R * d * (2 + 4)}


def backward_model(shape, T: int, R: int, active_experts: int):
    """(FLOPs, algorithmic bytes) of one backward pass with R kept rows.

    FLOPs: the five expert GEMMs, pre = x W_gu^T (recomputed) and dx_rows = d_pre W_gu and
    dW_gu = d_pre^T x (2 R d n_gu each), dh = dy W_d and dW_d = dy^T h (2 R d F each).
    Bytes: the active experts' bf16 weights read once, every expert's fp32 weight gradients
    written, x_perm (bf16) and y_perm (fp32) read, d_out and x read (bf16), dx written
    (fp32), and the router's fp32 gradient written.
    """
    d, N, F = shape.d_model, shape.n_experts, shape.d_ff
    n_gu = 2 * F if shape.act == "swiglu" else F
    flops = 6 * R * d * n_gu + 4 * R * d * F
    per_expert = n_gu * d + d * F
    nbytes = (active_experts * per_expert * 2 + N * per_expert * 4 + R * d * (2 + 4)
              + T * d * (2 + 2 + 4) + N * d * 4)
    return flops, nbytes


def ffn_flops(shape, R: int) -> int:
    d, F = shape.d_model, shape.d_ff
    return 2 * R * d * F * (3 if shape.act == "swiglu" else 2)


def roofline_of(shape, T: int, R: int, active: int, ffn_ms: float, step_ms: float, peaks: dict,
                wfmt: str = "bf16", traffic=None) -> dict:
    """Roofline of the grouped FFN (the dominant kernel) and of the whole layer.

    The FFN is tensor-bound when its FLOPs (measured R) per algorithmic byte (active expert
    weights) exceed the machine ridge, measured bf16 burst TFLOP/s over measured copy GB/s.
    Its fraction is taken against the burst bf16 peak (the FFN stage is timed alone, between
    L2 flushes) or the copy peak. The layer's fraction is its algorithmic bytes (weights, W_r,
    x, out) over the whole step time against the copy peak; it is the figure the decode
    targets are stated on. Tensor-bound points also report the layer's TFLOP/s."""
    ab = algorithmic_bytes(shape, T, active, R, wfmt)
    flops = ffn_flops(shape, R)
    # the block-scaled formats run FP8 MMAs: their tensor peak is the bf16 one times the
    # nominal FP8 / bf16 ratio (4.5 / 2.25 PFLOP/s dense)
    fp8 = wfmt.endswith("_bs")
    t_peak = peaks["bf16_tflops"] * (2.0 if fp8 else 1.0)
    ridge = (t_peak * 1e12) / (peaks["hbm_gbs"] * 1e9)
    tensor = ab["weights"] > 0 and flops / ab["weights"] > ridge
    ffn_s, step_s = ffn_ms * 1e-3, step_ms * 1e-3
    if tensor:
        ach, peak, unit = flops / ffn_s / 1e12, t_peak, "TFLOP/s"
        per_launch = f"{flops} FLOP"
        src = peaks["source"] + (" bf16 burst x 2 (fp8)" if fp8 else " bf16 burst")
    else:
        ach, peak, unit = ab["weights"] / ffn_s / 1e9, peaks["hbm_gbs"], "GB/s"
        per_launch, src = f"{ab['weights']} B", peaks["source"] + " copy"
    ffn = {"bound": "tensor" if tensor else "hbm", "achieved": round(ach, 1), "peak": peak,
           "unit": unit, "frac": round(ach / peak, 4), "per_launch": per_launch,
           "peak_source": src, "traffic": int(traffic) if traffic else None,
           # over the weights, each read once: HBM-bound points show re-reads; tensor-bound
           # points add the activations (x_perm, h, y_perm) that spill out of L2
           "traffic_over_weights": round(traffic / ab["weights"], 3) if traffic else None}
    layer_gbs = ab["layer"] / step_s / 1e9
    layer = {"achieved_gbs": round(layer_gbs, 1), "frac_hbm": round(layer_gbs / peaks["hbm_gbs"], 4),
             "algorithmic_bytes": ab["layer"]}
    if tensor:
        layer["achieved_tflops"] = round((flops + 2 * T * shape.d_model * shape.n_experts)
                                         / step_s / 1e12, 1)
    return {"ffn": ffn, "layer": layer, "weights_bytes": ab["weights"], "ffn_flops": flops}


def router_on_tensor_cores(T: int, n_experts: int, d_model: int) -> bool:
    """The library's router path choice: tensor cores once the per-token path's re-reads of
    W_r (T * N * d * 4 bytes) would pass 256 MiB."""
    return T * n_experts * d_model * 4 > 268435456


DECODE_ROUTE_MAX_T = 16           # batches routed (and, when small, sorted) in one launch
DECODE_ROUTE_MAX_SCRATCH = 1 << 20  # ... while their partial dot products fit this
DECODE_PERMUTE_MAX_BYTES = 512 * 1024


def decode_route(T: int, n_experts: int, d_model: int) -> bool:
    """The library's rule for the one-launch routing of decode-sized batches."""
    return 1 <= T <= DECODE_ROUTE_MAX_T and \
        math.ceil(d_model / 128) * T * n_experts * 4 <= DECODE_ROUTE_MAX_SCRATCH


def launches_per_step(T: int, k: int, R_max: int, n_experts: int = 1, d_model: int = 1) -> int:
    """Kernels one forward (moe_forward) launches. Decode-sized batches (decode_route): one routing
    launch (router, top-k and slots), which also sorts by expert while x_perm is at most
    512 KB, else a permute launch. Larger batches: router + top-k (plus the W_r split kernel
    on the tensor-core path), capacity slots (1 pass, or 3 when the arrivals span several
    chunks), permute. Then the grouped FFN (both GEMMs in one launch, when rows can exist)
    and the combine."""
    ffn = (1 if R_max > 0 else 0) + 1
    if decode_route(T, n_experts, d_model):
        return 1 + (0 if R_max * d_model * 2 <= DECODE_PERMUTE_MAX_BYTES else 1) + ffn
    chunks = max(1, math.ceil(T * k / SLOT_CHUNK))
    router = 2 if router_on_tensor_cores(T, n_experts, d_model) else 1
    return router + (1 if chunks == 1 else 3) + 1 + ffn


# DRAM traffic of the grouped-FFN stage per forward (dram__bytes_read.sum +
# dram__bytes_write.sum of one launch, as ncu prints them: three significant digits) from one
# capture per workload of the current kernel; workloads without one report null.
MEASURED_FFN_TRAFFIC = {
    ("tiny_top2", 64): 1.67e6,
    ("switch_top1", 4096): 1.09e9 + 10.68e6,
    ("mixtral", 1): 709.46e6 + 3.15e6,
    ("mixtral", 16): 2.82e9 + 4.78e6,
    ("mixtral", 512): 2.86e9 + 45.51e6,
    ("mixtral", 8192): 5.83e9 + 726.43e6,  # the CTA-pair kernel
    ("gpt_oss", 1): 201.80e6 + 3.36e6,
    ("gpt_oss", 8): 958.33e6 + 3.38e6,
    ("gpt_oss", 64): 1.61e9 + 5.67e6,
    ("gpt_oss", 16384): 2.64e9 + 1.10e9,  # the CTA-pair kernel
    ("fine_grained", 16384): 19.44e9 + 181.11e6,
}


def load_peaks():
    if os.path.exists(MEASURED_PEAKS):
        with open(MEASURED_PEAKS) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock, power and clock-event reasons of one GPU through NVML every ~1 ms
    on a background thread while the timed region runs (the main thread spends that time in
    CUDA synchronisation, which releases the GIL)."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, torch_device_index: int, interval_s: float = 0.0002):
        self.interval = interval_s
        self.samples = []
        self.reasons = set()
        self.err = None
        self.nv = None
        self.handle = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.handle = nv.nvmlDeviceGetHandleByUUID(uuid)
            self.nv = nv
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = f"nvml unavailable: {e}"

    def _poll(self):
        import threading  # noqa: F401
        nv, h = self.nv, self.handle
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                rs = get_reasons(h)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0 if len(self.samples) % 8 == 0 else \
                    (self.samples[-1][1] if self.samples else 0.0)
                self.samples.append((sm, pw))
                for name, const in self.REASONS.items():
                    if rs & getattr(nv, const, 0):
                        self.reasons.add(name)
            except Exception as e:
                self.err = str(e)
                return
            self._stop.wait(self.interval)

    def start(self):
        if self.nv is None:
            return
        import threading
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._poll, daemon=True)
        self._t.start()
        t0 = time.perf_counter()
        while not self.samples and self.err is None and time.perf_counter() - t0 < 2.0:
            time.sleep(0.0005)  # the timed region starts once the sampler is running

    def stop(self) -> dict:
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": self.err}
        self._stop.set()
        self._t.join(timeout=5)
        sm = [a for a, _ in self.samples]
        pw = [b for _, b in self.samples]
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
               "power_w_max": max(pw) if pw else None, "samples": len(sm),
               "reasons": sorted(self.reasons), "source": "nvml"}
        if self.err:
            out["note"] = self.err
        return out


# ----------------------------------------------------------------------------- GPU arm
class Layer:
    """Device buffers of one layer invocation; stages called through the C ABI."""

    def __init__(self, shape, T, device, seed=0, wfmt="bf16", weights=None):
        """weights: the weights (and router) of an earlier Layer of the same shape to reuse;
        only the tokens are drawn then."""
        import sparse_mixture_experts_11_b200 as moe
        self.moe = moe
        self.shape, self.T, self.wfmt = shape, T, wfmt
        if weights is not None:
            self.inp = {k: v for k, v in weights.items() if k != "x"}
            self.inp["x"] = synthetic.make_hidden(T, shape.d_model, seed=seed, device=device)
        elif wfmt == "bf16":
            self.inp = synthetic.make_layer_inputs(shape, T, seed=seed, device=device)
        else:
            self.inp = synthetic.make_mx_layer_inputs(shape, T, wfmt, seed=seed, device=device)
        cap = capacity_of(shape, T)
        self.dims = moe.make_dims(T, shape.d_model, shape.n_experts, shape.top_k, shape.d_ff,
                                  shape.act, cap)
        i = self.inp
        self.mx = None if wfmt == "bf16" else moe.mx_weights(
            self.dims, wfmt, i["w_gate_up_q"], i["w_gate_up_s"], i["w_down_q"], i["w_down_s"])
        self.R_max = moe.max_rows(self.dims)
        # block-scaled formats ("_bs"): the quantised activations follow the forward workspace
        self.block_scaled = wfmt.endswith("_bs")
        self.fws = moe.new_workspace(self.dims, device, forward=True, block_scaled=self.block_scaled)
        self.b = moe.forward_layout(self.dims, self.fws)
        self.out = torch.empty((T, shape.d_model), dtype=torch.bfloat16, device=device)

    def _view(self, ptr, n, dtype):
        off = ptr - self.fws.data_ptr()
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return self.fws[off:off + nbytes].view(dtype)

    def views(self):
        """Tensor views of the intermediates inside the forward workspace."""
        s = self.shape
        T, k, N, d, F, R = self.T, s.top_k, s.n_experts, s.d_model, s.d_ff, self.R_max
        b = self.b
        return {"logits": self._view(b.logits, T * N, torch.float32).view(T, N),
                "topk_idx": self._view(b.topk_idx, T * k, torch.int32).view(T, k),
                "topk_w": self._view(b.topk_w, T * k, torch.float32).view(T, k),
                "slot": self._view(b.slot, T * k, torch.int32).view(T, k),
                "expert_count": self._view(b.expert_count, N, torch.int32),
                "expert_offset": self._view(b.expert_offset, N + 1, torch.int32),
                "row_of_pair": self._view(b.row_of_pair, T * k, torch.int32).view(T, k),
                "pair_of_row": self._view(b.pair_of_row, R, torch.int32),
                "x_perm": self._view(b.x_perm, R * d, torch.bfloat16).view(R, d),
                "y_perm": self._view(b.y_perm, R * d, torch.float32).view(R, d),
                "stage_ws": self._view(b.stage_ws, b.stage_ws_bytes, torch.uint8)}

    def stats_timing(self, steps: int, flush) -> dict:
        """moe_router_stats on the step's logits and routing: mean ms per call and its
        algorithmic bandwidth (logits, indices and slots read once)."""
        moe, v = self.moe, self.views()
        N, k, T = self.shape.n_experts, self.shape.top_k, self.T
        picks = torch.empty((N,), dtype=torch.int32, device=v["logits"].device)
        pm = torch.empty((N,), dtype=torch.float32, device=picks.device)
        aux = torch.empty((1,), dtype=torch.float32, device=picks.device)
        dropped = torch.empty((1,), dtype=torch.int32, device=picks.device)
        call = lambda: moe.router_stats(self.dims, v["logits"], v["topk_idx"], v["slot"], picks, pm,
                                        aux, dropped, v["stage_ws"], alpha=0.01)
        call()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for e0, e1 in evs:
            flush_l2(flush)
            e0.record()
            g.replay()
            e1.record()
        torch.cuda.synchronize()
        ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs)
        nbytes = T * N * 4 + 2 * T * k * 4
        return {"ms": round(ms, 4), "aux_loss": round(float(aux.item()), 6),
                "dropped_pairs": int(dropped.item()), "algorithmic_bytes": nbytes,
                "achieved_gbs": round(nbytes / (ms * 1e-3) / 1e9, 1)}

    def route_stats_timing(self, steps: int, flush) -> dict:
        """The route stage alone (moe_route) and with the router statistics emitted by the
        routing launches (moe_route_with_stats), each a captured graph replayed between events
        with L2 flushed before every call: mean ms of each and the difference."""
        moe, i, b, v = self.moe, self.inp, self.b, self.views()
        N = self.shape.n_experts
        dev = i["x"].device
        picks = torch.empty((N,), dtype=torch.int32, device=dev)
        pm = torch.empty((N,), dtype=torch.float32, device=dev)
        aux = torch.empty((1,), dtype=torch.float32, device=dev)
        dropped = torch.empty((1,), dtype=torch.int32, device=dev)
        plain = self.stage_calls()[0]

        def fused():
            moe.route_with_stats(self.dims, i["x"], i["w_router"], i["logit_bias"], v["logits"],
                                 v["topk_idx"], v["topk_w"], v["slot"], v["expert_count"], picks,
                                 pm, aux, dropped, v["stage_ws"], alpha=0.01)
        out = {}
        for name, call in (("route_ms", plain), ("route_with_stats_ms", fused)):
            call()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                call()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(steps)]
            for e0, e1 in evs:
                flush_l2(flush)
                e0.record()
                g.replay()
                e1.record()
            torch.cuda.synchronize()
            out[name] = round(statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs), 4)
        out["added_us"] = round((out["route_with_stats_ms"] - out["route_ms"]) * 1e3, 2)
        out["aux_loss"] = round(float(aux.item()), 6)
        return out

    def backward_timing(self, steps: int, flush, peaks: dict) -> dict:
        """moe_backward after this layer's forward (bf16 weights): mean ms per call of the
        captured backward between events, with L2 flushed before each call. FLOPs are the five
        expert GEMMs (pre recomputed, dh, dx_rows, dW_d, dW_gu); algorithmic bytes are the
        expert weights read once, the fp32 weight gradients written, the saved rows read
        (x_perm, y_perm), d_out and x read, dx and the router's gradient written."""
        moe, i, s = self.moe, self.inp, self.shape
        T, d, N, F = self.T, s.d_model, s.n_experts, s.d_ff
        dev = i["x"].device
        n_gu = 2 * F if s.act == "swiglu" else F
        g = synthetic.make_grad_output(T, d, seed=1, device=dev)
        out = {"dx": torch.empty((T, d), dtype=torch.float32, device=dev),
               "d_w_router": torch.empty((N, d), dtype=torch.float32, device=dev),
               "d_logit_bias": torch.empty((N,), dtype=torch.float32, device=dev),
               "d_w_gate_up": torch.empty((N, n_gu, d), dtype=torch.float32, device=dev),
               "d_w_down": torch.empty((N, d, F), dtype=torch.float32, device=dev)}
        bws = moe.new_backward_workspace(self.dims, dev)

        def call():
            moe.backward_into(self.dims, i["x"], i["w_router"], i["w_gate_up"], i["w_down"],
                              self.fws, g, out["dx"], out["d_w_router"], out["d_logit_bias"],
                              out["d_w_gate_up"], out["d_w_down"], bws)
        self.forward_call()
        call()
        torch.cuda.synchronize()
        err = moe.read_device_error(bws)
        if err != 0:
            raise RuntimeError(f"backward device status: {moe.status_string(err)}")
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            call()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for e0, e1 in evs:
            flush_l2(flush)
            e0.record()
            gr.replay()
            e1.record()
        torch.cuda.synchronize()
        ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs)
        counts = self.views()["expert_count"].cpu()
        R, active = int(counts.sum()), int((counts > 0).sum())
        flops, nbytes = backward_model(s, T, R, active)
        tensor = flops / nbytes > (peaks["bf16_tflops"] * 1e12) / (peaks["hbm_gbs"] * 1e9)
        if tensor:
            ach, peak, unit = flops / (ms * 1e-3) / 1e12, peaks["bf16_tflops_sustained"], "TFLOP/s"
        else:
            ach, peak, unit = nbytes / (ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s"
        return {"ms": round(ms, 4), "tokens_per_s": round(T / (ms * 1e-3), 1),
                "flops": flops, "algorithmic_bytes": nbytes,
                "bound": "tensor" if tensor else "hbm", "achieved": round(ach, 1), "peak": peak,
                "unit": unit, "frac": round(ach / peak, 4),
                "launches": 11 if R > 0 else 5}

    def redirect_timing(self, steps: int, flush) -> dict:
        """moe_redirect_overflow (overflow policy "redirect") on the step's logits and top-k,
        into separate buffers: mean ms per call of a graph that restores the router's top-k
        (a T*k*4-byte device copy) and redirects. Pairs kept and redirected, against dropping."""
        moe, v = self.moe, self.views()
        N, k, T = self.shape.n_experts, self.shape.top_k, self.T
        dev = v["logits"].device
        idx0 = v["topk_idx"].clone()
        idx = torch.empty_like(idx0)
        slot = torch.empty((T, k), dtype=torch.int32, device=dev)
        cnt = torch.empty((N,), dtype=torch.int32, device=dev)

        def call():
            idx.copy_(idx0)
            moe.redirect_overflow(self.dims, v["logits"], idx, slot, cnt, v["stage_ws"])
        call()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for e0, e1 in evs:
            flush_l2(flush)
            e0.record()
            g.replay()
            e1.record()
        torch.cuda.synchronize()
        ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs)
        kept = int((slot >= 0).sum())
        return {"ms": round(ms, 4), "pairs": T * k, "kept_pairs": kept,
                "kept_pairs_drop_policy": int((v["slot"] >= 0).sum()),
                "redirected_pairs": int((idx != idx0).sum()),
                "ns_per_pair": round(ms * 1e6 / (T * k), 2)}

    def stage_calls(self):
        """The four stage calls of one forward (the calls moe_forward makes), as closures."""
        moe, i, b, dims = self.moe, self.inp, self.b, self.dims
        lib = moe._lib
        d = moe.ctypes.byref(dims)
        P = moe.ctypes.c_void_p
        ptr = lambda t: P(t.data_ptr()) if t is not None else None

        def route():
            moe._check(lib.moe_route(d, ptr(i["x"]), ptr(i["w_router"]), ptr(i["logit_bias"]),
                                     P(b.logits), P(b.topk_idx), P(b.topk_w), P(b.slot),
                                     P(b.expert_count), P(b.stage_ws), b.stage_ws_bytes,
                                     moe._stream(None)), "route")

        def permute():
            moe._check(lib.moe_permute(d, ptr(i["x"]), P(b.topk_idx), P(b.slot), P(b.expert_count),
                                       P(b.expert_offset), P(b.row_of_pair), P(b.pair_of_row),
                                       P(b.x_perm), P(b.stage_ws), b.stage_ws_bytes,
                                       moe._stream(None)), "permute")

        # the per-stage workspace is the forward layout's last region; the block-scaled formats
        # find their activation region right after it
        stage_ws_avail = self.fws.numel() - (b.stage_ws - self.fws.data_ptr())

        def ffn():
            if self.mx is not None:
                moe._check(lib.moe_grouped_ffn_mx(d, P(b.x_perm), P(b.expert_offset),
                                                  moe.ctypes.byref(self.mx), P(b.h), P(b.y_perm),
                                                  P(b.stage_ws), stage_ws_avail,
                                                  moe._stream(None)), "grouped_ffn_mx")
                return
            moe._check(lib.moe_grouped_ffn(d, P(b.x_perm), P(b.expert_offset), ptr(i["w_gate_up"]),
                                           ptr(i["w_down"]), P(b.h), P(b.y_perm), P(b.stage_ws),
                                           b.stage_ws_bytes, moe._stream(None)), "grouped_ffn")

        def combine():
            moe._check(lib.moe_unpermute_combine(d, P(b.y_perm), P(b.row_of_pair), P(b.topk_w),
                                                 ptr(i["x"]), ptr(self.out), 0, P(b.stage_ws),
                                                 b.stage_ws_bytes, moe._stream(None)), "combine")
        return [route, permute, ffn, combine]

    def forward_call(self):
        """moe_forward on the layer's inputs (the public call; decode-sized batches route and
        sort in one launch there, which the stage calls do not)."""
        self.forward_on(self.inp["x"], self.out)

    def forward_on(self, x, out, stream=None):
        """moe_forward (bf16 or MX weights) of tokens x into out, residual x."""
        i = self.inp
        if self.mx is not None:
            self.moe.forward_mx_into(self.dims, x, i["w_router"], i["logit_bias"], self.mx, x, out,
                                     self.fws, stream=stream)
        else:
            self.moe.forward_into(self.dims, x, i["w_router"], i["logit_bias"], i["w_gate_up"],
                                  i["w_down"], x, out, self.fws, stream=stream)

    def capture_stage_graphs(self):
        """The forward captured as CUDA graphs: once whole (moe_forward; its kernels overlap
        through programmatic dependent launch) and once per stage (the four stage calls, for
        the stage breakdown)."""
        self.graphs = []
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for call in self.stage_calls():  # one eager pass on the capture stream first
                call()
            self.forward_call()
        torch.cuda.current_stream().wait_stream(s)
        self.graph_full = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph_full):
            self.forward_call()
        for call in self.stage_calls():
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                call()
            self.graphs.append(g)

    def step_full(self, ev):
        """One forward: the whole-forward graph between two events."""
        ev[0].record()
        self.graph_full.replay()
        ev[1].record()

    def step_stages(self, ev):
        """One forward: the four stage graphs replayed with events between them (5 events)."""
        ev[0].record()
        for n, g in enumerate(self.graphs):
            g.replay()
            ev[n + 1].record()

    def e2e_copies(self, steps: int, warmup: int):
        """The copies of e2e_pipeline alone: per step the H2D of the tokens and the D2H of an
        output buffer, on the same two copy streams and pinned buffers, with no forward between
        them. Returns the elapsed ms of `steps` steps, first H2D to last D2H on the device: the
        floor under the end-to-end figure that the host link sets."""
        i = self.inp
        T, d = self.T, self.shape.d_model
        x_host = [i["x"].cpu().pin_memory() for _ in range(2)]
        out_host = [torch.empty((T, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        x_dev = [torch.empty_like(i["x"]) for _ in range(2)]
        out_dev = [torch.zeros_like(i["x"]) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        s_in.wait_stream(torch.cuda.current_stream())
        s_out.wait_stream(torch.cuda.current_stream())
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for n in range(warmup + steps):
            b = n % 2
            if n == warmup:
                s_in.wait_stream(s_out)
                s_out.wait_stream(s_in)
                t0.record(s_in)
            with torch.cuda.stream(s_in):
                x_dev[b].copy_(x_host[b], non_blocking=True)
            with torch.cuda.stream(s_out):
                out_host[b].copy_(out_dev[b], non_blocking=True)
        s_in.wait_stream(s_out)
        t1.record(s_in)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    def e2e_pipeline(self, steps: int, warmup: int):
        """End to end through the public call, as a serving loop would run it: every step
        copies its tokens from pinned host memory (H2D), runs moe_forward, and copies the
        output back (D2H). H2D, compute and D2H use three streams and two device buffers, so
        the copies of neighbouring steps overlap the compute. Returns the elapsed ms of
        `steps` steps (after `warmup` untimed ones), measured from the first H2D to the last
        D2H on the device."""
        moe, i = self.moe, self.inp
        T, d = self.T, self.shape.d_model
        x_host = [i["x"].cpu().pin_memory() for _ in range(2)]
        out_host = [torch.empty((T, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        x_dev = [torch.empty_like(i["x"]) for _ in range(2)]
        out_dev = [torch.empty_like(i["x"]) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        s_comp = torch.cuda.current_stream()
        ev = lambda: torch.cuda.Event()
        h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        for e in comp_done + d2h_done:
            e.record(s_comp)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for n in range(warmup + steps):
            b = n % 2
            if n == warmup:
                s_in.wait_stream(s_comp)
                s_in.wait_stream(s_out)
                t0.record(s_in)
            with torch.cuda.stream(s_in):
                s_in.wait_event(comp_done[b])        # step n-2 no longer reads x_dev[b]
                x_dev[b].copy_(x_host[b], non_blocking=True)
                h2d_done[b].record(s_in)
            s_comp.wait_event(h2d_done[b])
            s_comp.wait_event(d2h_done[b])           # step n-2's output has left out_dev[b]
            self.forward_on(x_dev[b], out_dev[b], stream=s_comp)
            comp_done[b].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[b])
                out_host[b].copy_(out_dev[b], non_blocking=True)
                d2h_done[b].record(s_out)
        s_comp.wait_stream(s_out)
        t1.record(s_comp)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)


def e2e_entry(T: int, d: int, steps: int, world: int, e2e_ms: float, copies_ms: float) -> dict:
    """The end-to-end figure and its bound: the same steps' host copies alone (H2D of x and
    D2H of out, both directions at once), as tokens/s and as the copies' rate in GB/s."""
    nbytes = T * d * 2
    e2e = tokens_per_second(T, steps, world, e2e_ms)
    floor = tokens_per_second(T, steps, world, copies_ms)
    return {"value": round(e2e, 1), "unit": "tokens/s", "h2d_bytes_per_step": nbytes,
            "d2h_bytes_per_step": nbytes,
            "copies_only": {"value": round(floor, 1), "unit": "tokens/s",
                            "gbs_per_direction": round(nbytes * steps / (copies_ms * 1e-3) / 1e9, 1),
                            "frac": round(e2e / floor, 4)}}


def reduce_max(values, world: int, device) -> list:
    """Max over ranks of each timed duration (a no-op on one rank). Every rank calls it at the
    same point, so the collective sequence is identical on all ranks."""
    if world <= 1:
        return list(values)
    t = torch.tensor(values, dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def tokens_per_second(tokens_per_rank: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * steps * world / (max_ms * 1e-3)


def flush_l2(buf):
    """Evict L2 before a step: a 256 MB write (larger than the 126 MB L2), then a 256 MB read
    of a second buffer, so the write's dirty lines go back to HBM here, outside the timed
    region, instead of during the step, and the step starts with no line of its own data
    in L2."""
    w, r = buf
    w.add_(1)
    torch.sum(r, dtype=torch.float32)


def measure_forward(layer, steps: int, warmup: int, flush, world: int = 1, clocks=None):
    """Warm-up, then `steps` timed whole-forward steps (one captured graph each, L2 flushed
    before every step outside the events) and `steps` stage-by-stage steps for the breakdown.
    Returns (per-step ms of the whole forward, mean ms per stage)."""
    moe = layer.moe
    for call in layer.stage_calls():  # first calls set kernel attributes outside any capture
        call()
    torch.cuda.synchronize()
    layer.capture_stage_graphs()
    wev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    for _ in range(warmup):
        flush_l2(flush)
        layer.step_full(wev)
        flush_l2(flush)
        layer.step_stages(wev)
    torch.cuda.synchronize()
    err = moe.read_device_error(layer.fws, offset_bytes=layer.b.stage_ws - layer.fws.data_ptr())
    if err != 0:
        raise RuntimeError(f"device status after warm-up: {moe.status_string(err)}")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.start()
    for k in range(steps):
        flush_l2(flush)
        layer.step_full(evs[k])
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop() if clocks is not None else None
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    # stage breakdown: the same number of steps replayed stage by stage, events between stages
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for k in range(steps):
        flush_l2(flush)
        layer.step_stages(sev[k])
    torch.cuda.synchronize()
    stage_ms = {n: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in sev)
                for i, n in enumerate(["route", "permute", "grouped_ffn", "combine"])}
    err = moe.read_device_error(layer.fws, offset_bytes=layer.b.stage_ws - layer.fws.data_ptr())
    if err != 0:
        raise RuntimeError(f"device status after the timed steps: {moe.status_string(err)}")
    return step_ms, stage_ms, clk


def routing_counts(layer):
    counts = layer.views()["expert_count"].cpu()
    return int(counts.sum()), int((counts > 0).sum())


def sweep_entry(layer, spec: str, step_ms: list, stage_ms: dict, peaks: dict) -> dict:
    shape, T = layer.shape, layer.T
    R, active = routing_counts(layer)
    mean_ms = statistics.mean(step_ms)
    roof = roofline_of(shape, T, R, active, stage_ms["grouped_ffn"], mean_ms, peaks, layer.wfmt,
                       MEASURED_FFN_TRAFFIC.get((shape.name, T)) if layer.wfmt == "bf16" else None)
    return {"workload": spec, "T": T, "steps": len(step_ms), "ms_per_step": round(mean_ms, 4),
            "ms_median": round(statistics.median(step_ms), 4),
            "tokens_per_s": round(T / (mean_ms * 1e-3), 1),
            "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
            "kept_rows": R, "active_experts": active, "capacity": layer.dims.capacity,
            "ffn": roof["ffn"], "layer": roof["layer"],
            "gpu_launches_per_step": launches_per_step(T, shape.top_k, layer.R_max,
                                                       shape.n_experts, shape.d_model)}


def run_sweep(args, device, flush, peaks, headline=None) -> dict:
    """Every workload point of the five shapes (bf16 or the --wfmt expert weights), each timed
    like the headline line; points of one shape share its weights. The headline's own entry is
    reused. Clocks are sampled over the whole sweep."""
    specs = SWEEP if args.sweep == "all" else tuple(x for x in args.sweep.split(",") if x)
    out = []
    cache = {}
    for spec in specs:
        shape, T = parse_workload(spec)
        if headline is not None and (shape.name, T) == (headline[0].shape.name, headline[0].T):
            out.append(headline[1])
            continue
        if cache.get("name") != shape.name:
            cache.clear()
            torch.cuda.empty_cache()
            cache["name"] = shape.name
        steps = max(args.steps, DECODE_MIN_STEPS) if T <= 64 else args.steps
        layer = Layer(shape, T, device, wfmt=args.wfmt, weights=cache.get("weights"))
        cache["weights"] = layer.inp
        # an idle pause first: a point timed right after a power-capped one (the large prefill
        # GEMMs hold a 1 kW part at its power limit) otherwise starts at the capped clock
        torch.cuda.synchronize()
        time.sleep(SWEEP_SETTLE_S)
        clocks = ClockSampler(torch.cuda.current_device())
        step_ms, stage_ms, clk = measure_forward(layer, steps, args.warmup, flush, clocks=clocks)
        entry = sweep_entry(layer, spec, step_ms, stage_ms, peaks)
        entry["clocks"] = {key: clk.get(key) for key in ("sm_mhz", "sm_max_mhz", "reasons", "samples")}
        out.append(entry)
        del layer
    cache.clear()
    torch.cuda.empty_cache()
    return {"points": out,
            "timing": "per point, after a 2 s idle pause: the whole forward as one captured graph, L2 flushed before "
                      "every step; mean (and median) of the timed steps; grouped FFN from the "
                      "stage-by-stage pass; clocks sampled over each point's timed steps"}


def run_gpu(args, rank, world, local_rank):
    import sparse_mixture_experts_11_b200 as moe  # fails loudly without the CUDA library
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    shape, T = parse_workload(args.workload)
    peaks = load_peaks()
    layer = Layer(shape, T, device, wfmt=args.wfmt)
    flush = (torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=device),
             torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=device))
    clocks = ClockSampler(torch.cuda.current_device())
    step_ms, stage_ms, clk = measure_forward(layer, args.steps, args.warmup, flush, world, clocks)
    total_ms = sum(step_ms)
    ffn_ms = stage_ms["grouped_ffn"]

    extras = not args.no_extras
    # router statistics and the auxiliary loss over this step's routing (a "next" row),
    # replayed as a graph K times between events
    stats = layer.stats_timing(args.steps, flush) if extras else None
    # the same statistics emitted by the routing launches themselves
    fused_stats = layer.route_stats_timing(args.steps, flush) if extras else None
    # backward pass after this forward (a "next" row); bf16 expert weights only
    backward = (layer.backward_timing(args.steps, flush, peaks)
                if extras and args.wfmt == "bf16" else None)
    # overflow policy "redirect" on the same routing (a "next" row), where the batch allows it
    redirect = (layer.redirect_timing(args.steps, flush)
                if extras and T * shape.top_k <= moe.REDIRECT_MAX_PAIRS else None)

    # end to end through the public call with host buffers (copies overlap neighbouring steps)
    if world > 1:
        torch.distributed.barrier()
    e2e_ms = layer.e2e_pipeline(args.steps, args.warmup)
    copies_ms = layer.e2e_copies(args.steps, args.warmup)

    total_ms, e2e_ms, copies_ms = reduce_max([total_ms, e2e_ms, copies_ms], world, device)

    R, active = routing_counts(layer)
    traffic = MEASURED_FFN_TRAFFIC.get((shape.name, T)) if args.wfmt == "bf16" else None
    roof_all = roofline_of(shape, T, R, active, ffn_ms, total_ms / args.steps, peaks, args.wfmt,
                           traffic)
    roof = dict(roof_all["ffn"])
    roof["kernel"] = "grouped_ffn_kernel (gate/up and down GEMMs in one launch)"
    headline_entry = sweep_entry(layer, f"{shape.name}:{T}", step_ms, stage_ms, peaks)
    headline_entry["clocks"] = {key: clk.get(key) for key in ("sm_mhz", "sm_max_mhz", "reasons", "samples")}

    value = tokens_per_second(T, args.steps, world, total_ms)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": ("synthetic (seeded; x~N(0,1) bf16, router W~N(0,1/d) fp32, expert W~N(0,0.02) bf16)"
                 if args.wfmt == "bf16" else
                 f"synthetic (seeded; x~N(0,1) bf16, router W~N(0,1/d) fp32, expert weights "
                 f"{args.wfmt}: random element codes, E8M0 scales per 32 elements)"),
        "config": {"workload": shape.describe(T) + ("" if args.wfmt == "bf16" else f" weights={args.wfmt}"),
                   "T": T, "d_model": shape.d_model, "expert_weights": args.wfmt,
                   "n_experts": shape.n_experts, "top_k": shape.top_k, "d_ff": shape.d_ff,
                   "act": shape.act, "capacity": layer.dims.capacity, "kept_rows": R,
                   "active_experts": active,
                   "l2": "flushed before every step (256 MB write, then 256 MB read of another buffer, outside the timed events); "
                         "expert weights also exceed L2",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "launch": "value: the whole forward as one captured CUDA graph (kernels chained "
                             "by programmatic dependent launch); stages_ms and roofline: the same "
                             "steps replayed as one graph per stage with events between stages"},
        "stages_ms": {k: round(v_, 4) for k, v_ in stage_ms.items()},
        "router_stats": stats,
        "route_with_stats": fused_stats,
        "overflow_redirect": redirect,
        "backward": backward,
        "roofline": roof,
        "layer": roof_all["layer"],
        "e2e": e2e_entry(T, shape.d_model, args.steps, world, e2e_ms, copies_ms),
        "gpu_launches": launches_per_step(T, shape.top_k, layer.R_max, shape.n_experts,
                                          shape.d_model) * args.steps,
        "clocks": clk,
    }
    if args.sweep != "none" and world == 1:
        line["sweep"] = run_sweep(args, device, flush, peaks, headline=(layer, headline_entry))
    return line, layer


# ----------------------------------------------------------------------------- CPU oracle arm
def oracle_sample(shape, T, layer_inputs_cpu, n_tokens: int):
    """Time the oracle's layer forward on the first n_tokens of the batch (routing over all T)."""
    import numpy as np
    import oracle
    x = layer_inputs_cpu["x"]
    cap = oracle.capacity_from_factor(shape.capacity_factor, T, shape.n_experts)
    toks = np.arange(min(n_tokens, T))
    t0 = time.perf_counter()
    oracle.moe_layer_forward(x, layer_inputs_cpu["w_router"], layer_inputs_cpu["w_gate_up"],
                             layer_inputs_cpu["w_down"], top_k=shape.top_k, act=shape.act,
                             capacity=cap, logit_bias=layer_inputs_cpu["logit_bias"],
                             residual=x, tokens=toks)
    return time.perf_counter() - t0, len(toks)


def cpu_inputs(shape, T, source: dict):
    """float64 host copies of the inputs; expert weights converted one expert at a time, on
    first use. source holds x, w_router, logit_bias and either the stacked expert weights
    (w_gate_up, w_down: device or host tensors) or `expert`, a function e -> (gate_up, down)."""
    f = lambda t: None if t is None else t.detach().to("cpu", torch.float64).numpy()
    cache = {}

    def get(e):
        if e not in cache:
            if "expert" in source:
                gu, dn = source["expert"](e)
            else:
                gu, dn = source["w_gate_up"][e], source["w_down"][e]
            cache[e] = (f(gu), f(dn))
        return cache[e]
    return {"x": f(source["x"]), "w_router": f(source["w_router"]), "logit_bias": f(source["logit_bias"]),
            "w_gate_up": lambda e: get(e)[0], "w_down": lambda e: get(e)[1], "_cache": cache}


def sample_tokens_for(shape, T) -> int:
    """Tokens per oracle sample: a few seconds of float64 CPU work, and at most ~6 GB of
    float64 expert weights touched (each token touches up to k experts)."""
    p = expert_params(shape.d_model, shape.d_ff, shape.act)
    by_flops = 4e10 // max(2 * shape.top_k * p, 1)
    if min(shape.n_experts, T * shape.top_k) * p * 8 <= 6e9:
        by_mem = T
    else:
        by_mem = 6e9 // (shape.top_k * p * 8)
    return int(max(1, min(T, by_flops, by_mem)))


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(shape, T, source: dict) -> dict:
    inp = cpu_inputs(shape, T, source)
    n = sample_tokens_for(shape, T)
    oracle_sample(shape, T, inp, n)   # converts the touched experts' weights to float64 once
    dt, used = oracle_sample(shape, T, inp, n)
    return {"value": round(used / dt, 2), "unit": "tokens/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"float64 oracle layer forward on the first {used} of {T} tokens "
                      f"(routing and capacity over all {T}); {dt:.2f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    shape, T = parse_workload(args.workload)
    # tokens and router drawn whole; each expert's weights drawn when the sample first uses it
    src = dict(synthetic.make_router_weights(shape, seed=0, device="cpu"),
               x=synthetic.make_hidden(T, shape.d_model, seed=0, device="cpu"),
               expert=lambda e: synthetic.make_expert_weights(shape, e, seed=0, device="cpu"))
    inp = cpu_inputs(shape, T, src)
    n = sample_tokens_for(shape, T)
    for _ in range(args.warmup):
        oracle_sample(shape, T, inp, n)
    dts = []
    for _ in range(args.steps):
        dt, used = oracle_sample(shape, T, inp, n)
        dts.append(dt)
    total = sum(dts)
    value = used * args.steps / total
    cores = blas_threads()
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": shape.describe(T), "T": T, "sample_tokens": used},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"float64 oracle layer forward on the first {used} of {T} tokens "
                                   f"per step (routing and capacity over all {T})"},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- main
def run_route_only(args) -> dict:
    """moe_route on the workload's tokens and router (synthetic, as in the layer), timed as a
    captured graph between L2 flushes."""
    import sparse_mixture_experts_11_b200 as moe
    device = torch.device("cuda")
    shape, T = parse_workload(args.workload)
    r = synthetic.make_router_weights(shape, device=device)
    x = synthetic.make_hidden(T, shape.d_model, device=device)
    N, k = shape.n_experts, shape.top_k
    dims = moe.make_dims(T, shape.d_model, N, k, shape.d_ff, shape.act, capacity_of(shape, T))
    ws = moe.new_workspace(dims, device)
    logits = torch.empty(T, N, device=device)
    idx = torch.empty(T, k, dtype=torch.int32, device=device)
    tw = torch.empty(T, k, device=device)
    slot = torch.empty(T, k, dtype=torch.int32, device=device)
    cnt = torch.empty(N, dtype=torch.int32, device=device)
    call = lambda: moe.route(dims, x, r["w_router"], r.get("logit_bias"), logits, idx, tw, slot, cnt, ws)
    flush = (torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=device),
             torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=device))
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    ts = []
    for _ in range(args.steps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    del g
    return {"metric": "route_ms", "value": round(statistics.median(ts), 4), "unit": "ms",
            "workload": shape.describe(T), "steps": args.steps, "warmup": args.warmup}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="shape[:T], shapes: " + ", ".join(synthetic.SHAPES))
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--wfmt", choices=["bf16", "mxfp8", "mxfp4", "mxfp8_bs", "mxfp4_bs"], default="bf16",
                    help="expert weight storage (MX formats: OCP microscaling, E8M0 block scales; "
                         "_bs: on the block-scaled MMA with MXFP8-quantised activations)")
    ap.add_argument("--sweep", default="all",
                    help="'all' (every workload point), 'none', or a comma list of shape:T")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the router-statistics, backward and redirect timings")
    ap.add_argument("--route-only", action="store_true",
                    help="time moe_route alone on the workload's tokens (no expert weights on "
                         "the device; for profiling the routing kernels)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0

    if args.route_only:
        print(json.dumps(run_route_only(args)), flush=True)
        return 0

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line, layer = run_gpu(args, rank, world, local_rank)
        if rank == 0 and not args.no_cpu_baseline and args.wfmt == "bf16":
            line["cpu_baseline"] = cpu_baseline(layer.shape, layer.T, layer.inp)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
