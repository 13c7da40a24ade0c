"""CPU oracles for the MoE layer forward pass (test infrastructure only).

Two independent restatements of the layer: ``moe_oracle`` (float64 NumPy,
re-exported here) and the plain C++ loops of ``moe_oracle.cpp`` (bound by
``oracle.cpp``; built with g++).  The backward-pass oracle is
``oracle.moe_backward``.  Only tests/, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline and reference legs import this package.  The CUDA
library never links, imports or calls it.
"""
from .moe_oracle import (  # noqa: F401
    ACT_RELU, ACT_SWIGLU, GATE_RENORM, GATE_SWITCH,
    aux_and_z, assign_slots, balance_losses, expert_capacity, expert_ffn, gates, moe_forward,
    router_logits, softmax_lse, top_k,
)
