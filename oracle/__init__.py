"""CPU oracle of the sparse MoE layer forward and backward passes (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
use this package. The CUDA library never imports it.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import (capacity_from_factor, router_logits, softmax_over_experts,  # noqa: F401
                         select_top_k, renormalise, assign_capacity_slots,
                         assign_capacity_slots_reroute, route_from_logits,
                         expert_permutation, silu, gelu, expert_ffn, combine,
                         moe_layer_forward, router_statistics)
from .mx_oracle import (MX_BLOCK, decode_e8m0, decode_e4m3, decode_e2m1,  # noqa: F401
                        unpack_fp4, dequantize_mx, encode_e4m3, quantize_mxfp8,
                        dequantize_mxfp8, mxfp8_round_trip, expert_ffn_mxfp8_act)
from .moe_backward import (logistic, silu_derivative, gelu_derivative,  # noqa: F401
                           combine_backward, renormalise_backward, expert_backward, aux_loss_backward,
                           moe_layer_backward)
