"""NF4 blockwise quantization with double quantization, and the QLoRA linear layer, as
hand-written CUDA for NVIDIA B200 (sm_100a) behind a small C ABI (include/qlora_nf4.h).

The Python layer only marshals arguments; the library is loaded lazily on first use and
every call raises if it is missing (there is no CPU fallback).
"""

from .binding import (  # noqa: F401
    NF4Tensor,
    QNF4Error,
    check_device_error,
    e4m3_encode,
    lib,
    library_path,
    linear_plan,
    merge_requantize,
    nf4_dequant,
    nf4_quantize_dq,
    qlora_linear_bwd,
    qlora_linear_fwd,
    quantize,
    set_timing_events,
)
from .paged import PagedAdamW  # noqa: F401

__all__ = [
    "NF4Tensor", "PagedAdamW", "QNF4Error", "check_device_error", "e4m3_encode", "lib", "library_path", "linear_plan", "merge_requantize", "set_timing_events",
    "nf4_dequant", "nf4_quantize_dq", "qlora_linear_bwd", "qlora_linear_fwd", "quantize",
]
