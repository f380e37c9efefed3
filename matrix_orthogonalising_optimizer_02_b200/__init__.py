"""Muon optimizer step for NVIDIA B200 (sm_100a): C-ABI library + thin binding."""
