"""The usage example (tests/usage_example.py) runs as written, and its
straight-through backward returns the incoming gradient."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_usage_example_runs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_block_scaled_quantizer_b200 import build as libbuild

    libbuild.build()
    import usage_example

    env = usage_example.main()
    y, x_train = env["y"], env["x_train"]
    y.sum().backward()
    assert torch.equal(x_train.grad, torch.ones_like(x_train))
    assert env["codes"].numel() == x_train.numel() // 2
    assert env["stack"].info_bits.shape == (20, 4096 * 2048 // 8)
