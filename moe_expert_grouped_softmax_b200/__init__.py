"""B200-native MoE split-LoRA expert block (route, permute, grouped GEMMs with
fused LoRA and SwiGLU, weighted unpermute, backward) behind a C ABI.

The ops live in :mod:`moe_expert_grouped_softmax_b200.ops`; they call the
sm_100a library ``libmoe_lora.so`` and raise if it is missing.
"""
__all__ = ["ops", "synthetic", "workload"]
