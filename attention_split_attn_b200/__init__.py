"""attention_split_attn_b200 -- attention over a KV cache on B200 (sm_100a).

The CUDA library and its Python binding are added next to this file; the
seeded input generators live in ``workloads``.
"""
