"""B200-native QLoRA NF4 linear path: quantize, double-quantize, dequantize,
dequant-GEMV and the fused LoRA linear forward/backward, as hand-written
sm_100a CUDA behind a C ABI (``include/qlora_nf4.h``).

Importing the package loads nothing native; ``bit_nf4_quantized_blk_b200.binding``
loads the shared library and raises if it is missing.
"""

__all__ = ["binding", "workloads"]
