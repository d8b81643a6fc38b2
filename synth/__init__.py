"""Seeded synthetic workloads for the routed MoE FFN forward pass.

This package holds the five workload shapes and the seeded generators that
draw their inputs.  It holds none of the layer's arithmetic: no routing, no
grouping, no expert FFN, no quantisation.  Both the CUDA path (tests, bench)
and the float64 oracle (tests) receive the tensors it draws.
"""

from .workloads import (ACT_GEGLU, ACT_SWIGLU, WFMT_BF16, WFMT_INT4_G128, WORKLOADS, Workload, draw_groups,
                        draw_logits, draw_topk_idx, draw_tree_router, expert_weights_f32, get_workload,
                        make_inputs)

__all__ = ["ACT_SWIGLU", "ACT_GEGLU", "WFMT_BF16", "WFMT_INT4_G128", "WORKLOADS", "Workload", "get_workload", "make_inputs", "expert_weights_f32",
           "draw_topk_idx", "draw_logits", "draw_groups", "draw_tree_router"]
