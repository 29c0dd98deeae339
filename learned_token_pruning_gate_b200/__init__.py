"""TokenGate gated-prefill hot path for B200 (sm_100a)."""
