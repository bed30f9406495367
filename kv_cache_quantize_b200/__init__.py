"""B200-native per-token KV-cache epilogue (sm_100a CUDA kernels behind a C ABI)."""
