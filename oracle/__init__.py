"""fp64 CPU oracle of the fine-grained MoE layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
reference legs may import this package; the product path never does.
"""
from .moe_oracle import (  # noqa: F401
    router_logits, selection_scores, select_topk, expert_counts, expert_offsets,
    dispatch, gelu_erf, expert_ffn, grouped_ffn, combine, moe_layer_forward, capacity,
    capacity_page_float, gini_exact, gini_page_form, load_stats, bias_update,
)
