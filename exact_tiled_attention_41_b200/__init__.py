"""Exact tiled attention for NVIDIA B200 (sm_100a)."""
