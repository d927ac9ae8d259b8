"""q8-KV single-query decode attention for B200 (sm_100a)."""
