"""AQLM weight-only additive-quantised linear layer for NVIDIA B200 (sm_100a)."""
