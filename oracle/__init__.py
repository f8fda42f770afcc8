"""CPU oracle for the multi-round dropless MoE layer (forward, and backward with recompute).

TEST INFRASTRUCTURE: imported only by tests/, the smoke check in
__graft_entry__.py and the CPU-baseline leg of bench.py. The library never
imports it and shares no code with it.
"""
from .moe_oracle import (bf16_to_f64, router_logits, select_topk, gates, plan, plan_borrow,  # noqa: F401
                         round_rows, silu, expert_hidden, expert_ffn, forward,
                         forward_rounds, layer)
from .moe_backward import (silu_grad, expert_backward, gates_backward, router_backward,  # noqa: F401
                           backward, backward_sampled, backward_rounds)
from .moe_ep import owner, ep_plan, ep_forward  # noqa: F401
