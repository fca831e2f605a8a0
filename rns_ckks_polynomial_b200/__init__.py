"""B200-native RNS-CKKS hot path: a C-ABI CUDA library plus a thin binding."""
