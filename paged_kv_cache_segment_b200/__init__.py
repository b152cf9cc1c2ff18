"""Multi-stream attention over a paged bf16 KV cache, as a C-ABI CUDA library
for B200 (sm_100a), with a thin ctypes binding.

    from paged_kv_cache_segment_b200 import binding as tf
    tf.tf_paged_attn_decode(...); tf.tf_attn_merge(...)

The computation runs only in libtfpaged.so's kernels; the binding checks and
marshals arguments.
"""
from .binding import (  # noqa: F401
    EXPORTS,
    TfError,
    load,
    tf_abi_version,
    tf_argmax_rows,
    tf_attn_merge,
    tf_kv_append,
    tf_paged_attn_block,
    tf_paged_attn_decode,
    tf_paged_attn_prompt,
    tf_ring_attn,
    tf_ring_attn_noalloc,
    tf_ring_tree_attn,
    tf_ring_tree_workspace_bytes,
    tf_ring_workspace_bytes,
    tf_choose_split_keys,
    tf_status_str,
    tf_verify_round,
    tf_wait_limit_test,
)
