"""Batched speculative-sampling verification on B200 (sm_100a)."""
