"""B200-native MoE routing hot path: a C-ABI CUDA library and its thin binding."""
