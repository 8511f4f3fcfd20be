"""B200-native frozen-NF4 linear layer with a bf16 LoRA adapter.

The computation lives in libqlora_nf4.so (CUDA, sm_100a); this package is its
ctypes binding (``_lib``), the in-tree build script (``build``) and the seeded
synthetic workload generator (``synthetic``).
"""
from ._lib import (  # noqa: F401
    EXPORTED,
    QLORA_SCALES_E4M3,
    QLORA_SCALES_E5M2,
    QLORA_SCALES_FP32,
    QLORA_SCALES_U8,
    Adam8State,
    Format,
    MLP,
    adamw8_state,
    NF4Tensor,
    QloraError,
    device_error_word,
    empty_nf4,
    lib,
    mlp_workspace,
    nf4_build_codebook,
    qlora_adamw8_step,
    qlora_dequantize,
    qlora_dequantize_fmt,
    qlora_format_sizes,
    qlora_linear_backward,
    qlora_linear_forward,
    qlora_linear_workspace_size,
    qlora_merge,
    qlora_merge_many,
    qlora_mlp_backward,
    qlora_mlp_forward,
    qlora_mlp_workspace_size,
    qlora_quantize,
    qlora_quantize_bf16,
    qlora_quantize_fmt,
    qlora_quantize_many,
    qlora_quantized_sizes,
    status_string,
    workspace,
)
