"""B200-native DeepSeekMoE FP8 layer forward pass (sm_100a kernels behind a C ABI).

    from fine_grained_fp8_sigmoid_b200 import binding, MoELayerFP8

`binding` mirrors include/moe_fp8.h call by call; `MoELayerFP8` owns the
buffers of one layer and runs route -> quant -> permute -> grouped FP8 GEMM
-> combine -> bias update.
"""
from .layer import MoELayerFP8  # noqa: F401

__all__ = ["MoELayerFP8"]
