"""B200-native H-BitLinear forward (BitNet v2): CUDA kernels behind a C ABI."""
