"""NVFP4 two-level quantization and block-scaled FP4 GEMMs for B200 (sm_100a)."""
