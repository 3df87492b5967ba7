"""B200-native MXFP8 / per-group FP8 quantization for MoE expert-parallel training."""
