"""GQE (Grouped Query Experts) causal prefill, decode and the attention layer
around them (projections, W_O) for B200 (sm_100a).

The compute lives in ``libgqe.so`` (CUDA kernels behind the C ABI of
``include/gqe.h``); this package only loads it (``_lib``) and offers a thin
torch-facing layer (``layer``) that allocates device buffers and calls the ABI.
"""
from ._lib import (  # noqa: F401
    EXPORTS, GqeDims, GqeError, LIB, LIB_PATH, STATUS, dims, gqe_append_workspace_size,
    gqe_attention_append, gqe_attention_decode, gqe_attention_prefill, gqe_decode_workspace_size,
    gqe_attention_prefill_static, gqe_bucket,
    gqe_dense_gqa_prefill, gqe_get_device_status, gqe_kv_cache_bytes, gqe_route,
    gqe_selftest_bounded_wait, gqe_set_pair_threshold, gqe_set_profile_events, gqe_set_router_resident, gqe_status_string,
    gqe_workspace_size, gqe_static_device_status, gqe_linear, gqe_routed_q_project,
    gqe_layer_prefill, gqe_dense_layer_prefill, gqe_prefill_chunk_workspace_size,
    gqe_attention_prefill_chunk, gqe_attention_prefill_train, gqe_prefill_backward_workspace_size,
    gqe_prefill_backward,
)
