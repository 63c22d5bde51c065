"""NVFP4 W4A4 routed mixture-of-experts feed-forward layer for NVIDIA B200 (sm_100a)."""
