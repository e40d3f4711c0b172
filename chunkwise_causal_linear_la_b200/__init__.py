"""Chunkwise causal linear attention on NVIDIA B200 (sm_100a)."""
