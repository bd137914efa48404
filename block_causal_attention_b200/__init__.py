"""block_causal_attention_b200: block-causal GQA attention for B200 (sm_100a)."""
