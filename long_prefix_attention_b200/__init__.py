"""Attention State Memory (ASM) hot path for NVIDIA B200 (sm_100a)."""
