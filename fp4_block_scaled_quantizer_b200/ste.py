"""Straight-through fake quantization for the trainer's forward pass.

The trainer's forward uses the quantized value (guided by the rollout's
record, or plain nearest rounding); the backward passes the incoming
gradient through unchanged (straight-through estimator) -- TRACE summary
(ai-papers.net), section "TRACEの仕組み": the gradient flows through the
chosen quantized value as if rounding were the identity.

Forward = one kernel of the CUDA library (guided: the fused
quantize-dequantize pass; nearest / stochastic: quantize + dequantize);
backward = no kernel (the same gradient tensor is returned when its dtype
matches the input's).
"""
from __future__ import annotations

import torch

from . import binding as B


def _through(grad: torch.Tensor, dtype: torch.dtype) -> torch.Tensor:
    return grad if grad.dtype == dtype else grad.to(dtype)


class GuidedFakeQuant(torch.autograd.Function):
    """y = dequantize(guided_quantize(x, record)); dy/dx := identity."""

    @staticmethod
    def forward(ctx, x: torch.Tensor, rec: B.Quantized, out_dtype=torch.float32):
        ctx.in_dtype = x.dtype
        if out_dtype in (torch.float32, torch.bfloat16):
            y, _ = B.tf4_guided_fake_quant(x, rec, out_dtype=out_dtype)
            return y.reshape(x.shape)
        y, _ = B.tf4_guided_fake_quant(x, rec)
        return y.reshape(x.shape).to(out_dtype)

    @staticmethod
    def backward(ctx, grad_out):
        return _through(grad_out, ctx.in_dtype), None, None


class RTNFakeQuant(torch.autograd.Function):
    """y = dequantize(rtn_quantize(x)); dy/dx := identity (plain QAT)."""

    @staticmethod
    def forward(ctx, x: torch.Tensor, fmt=B.NVFP4, seg_off=None, out_dtype=torch.float32):
        ctx.in_dtype = x.dtype
        q = B.tf4_quantize_rtn(x, fmt=fmt, seg_off=seg_off)
        return B.tf4_dequantize(q).reshape(x.shape).to(out_dtype)

    @staticmethod
    def backward(ctx, grad_out):
        return _through(grad_out, ctx.in_dtype), None, None, None


class SRFakeQuant(torch.autograd.Function):
    """y = dequantize(sr_quantize(x, seed)); dy/dx := identity."""

    @staticmethod
    def forward(ctx, x: torch.Tensor, seed: int, fmt=B.NVFP4, out_dtype=torch.float32):
        ctx.in_dtype = x.dtype
        q = B.tf4_quantize_sr(x, seed, fmt=fmt)
        return B.tf4_dequantize(q).reshape(x.shape).to(out_dtype)

    @staticmethod
    def backward(ctx, grad_out):
        return _through(grad_out, ctx.in_dtype), None, None, None


def guided_fake_quant(x, rec, out_dtype=torch.float32):
    return GuidedFakeQuant.apply(x, rec, out_dtype)


def rtn_fake_quant(x, fmt=B.NVFP4, seg_off=None, out_dtype=torch.float32):
    return RTNFakeQuant.apply(x, fmt, seg_off, out_dtype)


def sr_fake_quant(x, seed, fmt=B.NVFP4, out_dtype=torch.float32):
    return SRFakeQuant.apply(x, seed, fmt, out_dtype)
