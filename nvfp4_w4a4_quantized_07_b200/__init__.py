"""NVFP4 W4A4 linear layers for B200 (sm_100a): Python binding of libnvfp4."""
