"""B200-native flow-matching action-expert denoise loop (sm_100a CUDA, C-ABI)."""
