"""Reduced cross-entropy (RECE / SCE) loss on B200 (sm_100a)."""
