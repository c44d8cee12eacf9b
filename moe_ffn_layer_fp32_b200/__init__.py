"""Fused MoE feed-forward layer (INT4 weights, INT8 activations, FP32 router) for B200."""
