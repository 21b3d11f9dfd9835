"""fp64 CPU oracle of the Switch-layer forward pass (test infrastructure only).

This package is the reference the CUDA path is checked against.  It is plain
numpy in float64, step by step as the pages define the layer, with no blocking,
fusion or reordering beyond the definitions.  It shares no code with the CUDA
path.  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it; the product path never does.
"""
from .switch_layer import (  # noqa: F401
    capacity, router_logits, router_probs, top1, positions, expert_ffn,
    load_balance_stats, aux_loss, switch_forward, switch_forward_sampled,
    logit_gap, capacity_k, top2, positions_top2, switch_forward_top2, gelu, expert_ffn_geglu,
    switch_backward, positions_ntlb, switch_forward_ntlb,
)
