"""NVFP4 W4A4 linear for B200 (sm_100a)."""
