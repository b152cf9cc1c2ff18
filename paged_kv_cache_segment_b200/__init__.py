"""Multi-stream attention over a paged bf16 KV cache, as a C-ABI CUDA library for B200 (sm_100a)."""
