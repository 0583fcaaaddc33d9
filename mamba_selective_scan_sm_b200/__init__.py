"""Mamba selective-scan forward and decode state update for B200 (sm_100a)."""
