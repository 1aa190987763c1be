"""B200-native group-scaled quantized linear layer y = x . dequant(W)^T and its
MoE gate_up use (sm_100a CUDA behind a C ABI, ``libqlinear.so``).

The binding lives in :mod:`moe_hadamard128_act_b200.qlinear`; it loads the
compiled library on first use and raises if it is missing.
"""
__all__ = ["qlinear", "synth"]
