"""Block-scaled FP4 (NVFP4 / MXFP4 / uniform-grid UFP4) quantization for rollout-guided FP4 QAT on B200.

The quantization path runs in the CUDA library ``libtrace_fp4.so`` (C ABI
declared in include/trace_fp4.h); :mod:`.binding` marshals torch tensors
into it, :mod:`.ste` wraps it in straight-through autograd functions,
:mod:`.workloads` draws the seeded synthetic inputs.
"""
from .binding import (  # noqa: F401
    MXFP4, NVFP4, UFP4, Desc, Quantized, Tf4Error, capture_layers, lib, read_status, sizes,
    tf4_dequantize, tf4_guided_fake_quant, tf4_mismatch_stats, tf4_pack_guidance, tf4_quantize_capture,
    tf4_quantize_capture_batched, tf4_quantize_guided, tf4_quantize_rtn, tf4_quantize_sr, tf4_segment_amax,
    tf4_swizzle_scales, tf4_unpack_guidance,
)
