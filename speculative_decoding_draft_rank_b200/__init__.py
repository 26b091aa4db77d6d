"""DSpark per-round token path on B200 (sm_100a)."""
