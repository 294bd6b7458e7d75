"""Verified sparse attention (vAttention) decode step for B200 (sm_100a)."""
