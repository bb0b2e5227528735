"""Prefix-aware batched decode attention for B200 (sm_100a)."""
