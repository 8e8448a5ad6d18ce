"""DiT attention hot path for B200 (sm_100a)."""
