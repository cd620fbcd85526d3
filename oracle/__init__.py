"""CPU oracle for GQE prefill, decode and the attention layer around them (test infrastructure, not product code).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library under
``moe_routed_grouped_b200`` never calls it and shares no code with it.
"""
from .gqe_oracle import (  # noqa: F401
    bf16_to_f64,
    f64_to_bf16_bits,
    router_logits,
    route,
    topk_exact_order,
    bucket,
    causal_attention,
    gqe_prefill,
    gqe_prefill_rows,
    gqe_decode_step,
    gqe_append_step,
    exact_logits,
    dense_gqa,
    dense_gqa_repeat,
    kv_cache_bytes,
    gqe_layer_prefill,
    causal_attention_backward,
    gqe_prefill_values,
    gqe_prefill_backward,
    router_values,
    router_backward,
    load_balance_loss,
)
