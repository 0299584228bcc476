"""B200-native NVFP4 quantized linear layer (sm_100a CUDA kernels behind a C ABI).

``api`` holds the PyTorch-facing calls (amax, quantize, gemm, linear_fwd/bwd);
``dp`` the data-parallel linear layer over torch.distributed; ``synth`` the
seeded synthetic inputs; ``build`` compiles libnvfp4.so in-tree.
The library is loaded on first use and there is no fallback path.
"""
