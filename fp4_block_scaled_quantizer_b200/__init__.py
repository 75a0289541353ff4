"""Block-scaled FP4 (NVFP4 / MXFP4) quantization for rollout-guided FP4 QAT on B200."""
