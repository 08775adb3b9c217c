"""B200-native batched multi-LoRA delta path (C-ABI CUDA library + thin binding)."""
