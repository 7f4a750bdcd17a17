"""B200-native 2-D convolution forward (sm_100a CUDA behind a C ABI)."""
