"""QLoRA frozen-base linear layer with NF4 + double-quantized weights on B200.

Python binding of libqlora.so (the C ABI in include/qlora.h): NF4 blockwise
quantization, double quantization, dequantization and the fused
dequant-GEMM forward / backward of Y = X W' + s X L1 L2.  All arithmetic runs
in hand-written sm_100a CUDA kernels; this package only marshals arguments.
"""
from ._lib import (  # noqa: F401
    EXPORTS,
    LIB_PATH,
    NF4Weight,
    QLoRAError,
    lib,
    qlora_check_status,
    qlora_launch_count,
    qlora_trace_enable,
    qlora_trace_read,
    qlora_dequant,
    qlora_double_quant,
    qlora_linear_bwd,
    qlora_linear_fwd,
    qlora_linear_fwd_noalloc,
    qlora_merge_bf16,
    qlora_nf4_boundaries,
    qlora_nf4_codebook,
    qlora_quantize_nf4,
    quantize_weight,
)

__version__ = "1.0.0"
