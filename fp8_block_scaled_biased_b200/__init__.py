"""B200-native FP8 block-scaled biased MoE layer (sm_100a CUDA kernels behind a C ABI)."""
