"""expert_warp_top_b200: an Occult-style MoE layer hot path for B200 (sm_100a)."""
