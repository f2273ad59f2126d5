"""B200-native fused Mixture-of-Experts layer (sm_100a CUDA behind a C ABI)."""
