"""NF4 + double-quantisation + LoRA linear layer for B200 (sm_100a).

The computation lives in ``libqlora_nf4.so`` (C ABI: ``include/qlora_nf4.h``); the
``binding`` module marshals torch tensors into it. Importing the package does not load
the library; the first call does, and fails loudly if it is missing.
"""
from .binding import (NF4Weight, QNError, linear_workspace_size, launch_count, load, new_workspace, nf4_dequantize,
                      nf4_quantize, nf4_quantize_static_ws, qlora_linear_bwd_x, qlora_linear_fwd,
                      qlora_lora_grads, qlora_merge_bf16, quantize_workspace_size, sizes, weight_sizes, workspace_check)

__all__ = ["NF4Weight", "QNError", "linear_workspace_size", "launch_count", "load", "new_workspace", "nf4_dequantize",
           "nf4_quantize", "nf4_quantize_static_ws", "qlora_linear_bwd_x", "qlora_linear_fwd",
           "qlora_lora_grads", "qlora_merge_bf16", "quantize_workspace_size", "sizes", "weight_sizes",
           "workspace_check"]
