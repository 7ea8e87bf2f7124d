"""B200-native (sm_100a) SeerAttention prefill library.

The compute lives in libseer.so (C ABI, include/seer.h); this package is its
thin Python binding plus the seeded synthetic-input recipe.
"""
from ._lib import (  # noqa: F401
    SELECT_FORCE_DIAGONAL, SELECT_THRESHOLD, SELECT_TOPK_DENSITY, SELECT_TOPK_K, gate_varlen_workspace_size,
    seer_gate_varlen, seer_sparse_attn_tf32, sparse_attn_tf32_workspace_size, SeerError, attn_forward_map_workspace_size,
    blockmax_workspace_size, seer_attn_forward_map,
    gate_kl_backward_workspace_size, gate_required_cap, gate_workspace_size, lib, seer_attn_blockmax, seer_gate,
    seer_gate_kl_backward, seer_gate_noalloc, seer_gate_select, seer_sparse_attn, seer_workspace_status,
    sparse_attn_workspace_size, decode_blockmax_workspace_size, decode_gate_required_cap,
    decode_gate_workspace_size, seer_decode_blockmax,
    seer_decode_gate, seer_decode_kcache_update, seer_sparse_decode_attn, sparse_decode_attn_workspace_size,
    prefill_host_buffer_size, seer_prefill_host,
)
