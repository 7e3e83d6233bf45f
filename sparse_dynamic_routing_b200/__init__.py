"""Graph Machine sparse layer (SER + SEA) for B200 (sm_100a)."""
