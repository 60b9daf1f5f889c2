"""token_sparse_attention_sm_b200: shared-routing token-sparse decode
attention for NVIDIA B200 (sm_100a)."""
