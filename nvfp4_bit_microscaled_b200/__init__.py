"""B200-native NVFP4 quantized linear layer (sm_100a CUDA kernels behind a C ABI)."""
