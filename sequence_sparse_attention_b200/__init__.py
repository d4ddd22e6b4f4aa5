"""B200-native APB-V / Spava approximate-attention prefill (sm_100a)."""
