"""Sliding-window causal attention for B200 (sm_100a)."""
