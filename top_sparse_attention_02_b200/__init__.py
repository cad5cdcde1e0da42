"""Top-k context-sparse attention at decode, for NVIDIA B200 (sm_100a)."""
