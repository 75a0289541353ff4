"""Usage of the library from Python on one GPU (every call is asynchronous
on the current stream).  The GPU tests run this module as written."""
import torch

import fp4_block_scaled_quantizer_b200 as tf4
from fp4_block_scaled_quantizer_b200.ste import guided_fake_quant


def bf16(*shape):
    return torch.randn(*shape, device="cuda").to(torch.bfloat16)


def main():
    x = bf16(4096, 2048)                                          # rollout-side activations
    x_train = (x.float() * (1 + 1e-3 * torch.randn_like(x.float()))).to(torch.bfloat16)  # trainer's recompute
    rec = tf4.tf4_quantize_capture(x)                             # codes, scales, s_t, guidance bits
    codes = tf4.tf4_quantize_guided(x_train, rec)                 # train side: the rollout's neighbours
    y = guided_fake_quant(x_train.requires_grad_(), rec)          # forward value; backward = identity
    stack = tf4.tf4_quantize_capture_batched([bf16(4096, 2048) for _ in range(40)], keep=20)  # info cache
    assert tf4.read_status(x.device) == 0                         # no non-finite input was seen
    return dict(x_train=x_train, codes=codes, y=y, stack=stack)


if __name__ == "__main__":
    main()
