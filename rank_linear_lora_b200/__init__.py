"""B200-native fused LoRA linear layer (forward and backward, optional 4-bit frozen W).

The compute path is liblora_linear.so (hand-written sm_100a kernels behind a C ABI,
include/lora_linear.h); ``lora_linear`` is its ctypes binding.
"""
from . import lora_linear  # noqa: F401
from .lora_linear import (  # noqa: F401
    LoraError,
    lora_linear_bwd,
    lora_linear_bwd_q4,
    lora_linear_check,
    lora_linear_fwd,
    lora_linear_fwd_q4,
    lora_linear_workspace_size,
    lora_status_string,
)
