"""CPU oracle for the MoE layer forward pass (test infrastructure only).

Only tests/, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
import this package.  The CUDA library never links, imports or calls it.
"""
from .moe_oracle import (  # noqa: F401
    ACT_RELU, ACT_SWIGLU, GATE_RENORM, GATE_SWITCH,
    aux_and_z, assign_slots, balance_losses, expert_capacity, expert_ffn, gates, moe_forward,
    router_logits, softmax_lse, top_k,
)
