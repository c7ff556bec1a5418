"""Chunked causal linear attention prefill for NVIDIA B200 (sm_100a)."""
