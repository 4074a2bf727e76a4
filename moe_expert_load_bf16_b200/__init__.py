"""B200-native (sm_100a) MoE expert-parallel load-balancing decision path.

The five steps (lookahead gate + top-k, per-rank histograms, locality-aware
replica planning, Relief split, destinations + stable permutation) run in
hand-written CUDA kernels behind the C ABI of liblb.so (include/lb.h).  This
package is the thin Python binding over that library; `pipeline` strings the
steps together for one layer, `workloads` draws seeded synthetic inputs.
"""
from ._lib import (LBError, decode_plan, lb_assign, lb_assign_workspace_bytes, lb_count, lb_gate_tuning,
                   lb_get_status, lb_plan_bytes, lb_plan_replicas, lb_plan_swaps, lb_predict_topk,
                   lb_predict_topk_chain, lb_solve, lb_split, lb_version,
                   plan_layout)

__all__ = ["LBError", "decode_plan", "lb_assign", "lb_assign_workspace_bytes", "lb_count", "lb_gate_tuning",
           "lb_get_status", "lb_plan_bytes", "lb_plan_replicas", "lb_plan_swaps", "lb_predict_topk", "lb_predict_topk_chain", "lb_solve", "lb_split",
           "lb_version",
           "plan_layout"]
