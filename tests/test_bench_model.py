"""The benchmark's counting model (CPU): parameter counts pinned to the pages' printed numbers,
and the launch count and byte counts for the workloads."""
import json
import os

import bench
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_active_params_reproduce_page_numbers():
    g = json.load(open(os.path.join(GOLDEN, "active_params_demo.json")))
    d, h, N = g["d_model"], g["hidden"], g["experts"]
    # the demo expert is fc1 (d->h) and fc2 (h->d), each with bias: the GELU-shaped two-matrix FFN
    assert bench.active_params(d, h, N, 1, "gelu", bias=True) == g["top1_active"]
    assert bench.active_params(d, h, N, 2, "gelu", bias=True) == g["top2_active"]
    assert N * bench.expert_params(d, h, "gelu", bias=True) + d * N == g["total"]


def test_bandwidth_estimate_of_page():
    # 800 GB/s over 3.6 B active params at 2 bytes each is about 111 tokens/s
    assert round(800e9 / (3.6e9 * 2)) == 111


def test_bytes_model_switch():
    s = synthetic.SHAPES["switch_top1"]
    b = bench.algorithmic_bytes(s, 4096, 64, 4096)
    assert b["weights"] == 64 * 2 * 1024 * 4096 * 2
    assert b["layer"] == b["weights"] + 64 * 1024 * 4 + 2 * 4096 * 1024 * 2
    assert b["rows"] == 4096 * 1024 * 6


def test_roofline_counting():
    """The FFN's numerator is the active experts' weights (HBM-bound points) or the FLOPs of
    the kept rows (tensor-bound points), against the burst bf16 peak or the copy peak."""
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1300.0,
             "source": "test"}
    s = synthetic.SHAPES["gpt_oss"]
    w = 4 * 3 * 2880 * 2880 * 2
    r = bench.roofline_of(s, 1, 4, 4, 0.05, 0.06, peaks)
    assert r["ffn"]["bound"] == "hbm" and r["ffn"]["per_launch"] == f"{w} B"
    assert abs(r["ffn"]["frac"] - w / 0.05e-3 / 6000e9) < 1e-4
    lb = w + 32 * 2880 * 4 + 2 * 2880 * 2
    assert abs(r["layer"]["frac_hbm"] - lb / 0.06e-3 / 6000e9) < 1e-4
    m = synthetic.SHAPES["mixtral"]
    fl = 2 * 16384 * 4096 * 14336 * 3
    r = bench.roofline_of(m, 8192, 16384, 8, 5.0, 5.5, peaks)
    assert r["ffn"]["bound"] == "tensor" and r["ffn"]["peak"] == 1500.0
    assert abs(r["ffn"]["frac"] - fl / 5e-3 / 1500e12) < 1e-4


def test_launch_counts():
    # switch: W_r split + tensor-core router, one slot pass, permute, grouped FFN, combine
    assert bench.launches_per_step(4096, 1, 4096, 64, 1024) == 6
    # fine-grained: tensor-core router (2), three slot passes, permute, grouped FFN, combine
    assert bench.launches_per_step(16384, 8, 20480, 256, 7168) == 8
    # mid-size: per-token router, one slot pass, permute, grouped FFN, combine
    assert bench.launches_per_step(64, 4, 256, 32, 2880) == 5
    # decode: one launch routes and sorts, grouped FFN, combine
    assert bench.launches_per_step(1, 2, 2, 8, 4096) == 3
    assert bench.launches_per_step(8, 4, 32, 32, 2880) == 3
    # ... a separate permute when x_perm exceeds 512 KB (8 tokens x 8 choices x 7168)
    assert bench.launches_per_step(8, 8, 64, 256, 7168) == 4
    # decode with an x_perm above 512 KB (16 tokens x 8 choices x 7168): separate permute
    assert bench.launches_per_step(16, 8, 128, 256, 7168) == 4
    # no rows can be kept: routing (and sort) and the combine only
    assert bench.launches_per_step(5, 2, 0) == 2
    # 16 tokens, N = 256, d = 16384: partial dot products above 1 MiB, so per-token router,
    # slot pass, permute, grouped FFN, combine
    assert bench.launches_per_step(16, 8, 128, 256, 16384) == 5


def test_workload_parsing():
    s, T = bench.parse_workload("mixtral:512")
    assert s.d_model == 4096 and T == 512
    s, T = bench.parse_workload("switch_top1")
    assert T == 4096


def test_mx_weight_bytes():
    # one E8M0 scale byte per 32 elements; 1 byte (MXFP8) or half a byte (MXFP4) per element
    assert bench.weight_bytes(1024, "bf16") == 2048
    assert bench.weight_bytes(1024, "mxfp8") == 1024 + 32
    assert bench.weight_bytes(1024, "mxfp4") == 512 + 32
    s = synthetic.SHAPES["gpt_oss"]
    b = bench.algorithmic_bytes(s, 1, 4, 4, "mxfp4")
    params = 3 * 2880 * 2880
    assert b["weights"] == 4 * (params // 2 + params // 32)


def test_backward_model_hand_numbers():
    """Backward FLOPs and bytes for a hand-sized GELU and SwiGLU layer."""
    import synthetic
    gelu = synthetic.LayerShape("t", 8, 2, 1, 4, "gelu", None, (3,))
    flops, nbytes = bench.backward_model(gelu, T=3, R=3, active_experts=2)
    assert flops == 10 * 3 * 8 * 4                        # 6 R d F + 4 R d F
    per = 4 * 8 + 8 * 4                                    # W_1 and W_2 of one expert
    assert nbytes == 2 * per * 2 + 2 * per * 4 + 3 * 8 * 6 + 3 * 8 * 8 + 2 * 8 * 4
    swiglu = synthetic.LayerShape("t", 8, 2, 1, 4, "swiglu", None, (3,))
    flops, _ = bench.backward_model(swiglu, T=3, R=3, active_experts=2)
    assert flops == 6 * 3 * 8 * 8 + 4 * 3 * 8 * 4
