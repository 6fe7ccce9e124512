"""Exact attention forward for NVIDIA B200 (sm_100a)."""
