"""block_hybrid_linear_b200 -- block-hybrid attention on B200 (placeholder)."""
