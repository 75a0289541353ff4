"""The README's usage example runs as written (extracted from README.md and
executed), and its straight-through backward returns the incoming gradient."""
import os
import re

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_example_runs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_block_scaled_quantizer_b200 import build as libbuild

    libbuild.build()
    text = open(os.path.join(ROOT, "README.md")).read()
    (code,) = re.findall(r"```python\n(.*?)```", text, flags=re.S)
    env = {}
    exec(compile(code, "README.md", "exec"), env)
    y, x_train = env["y"], env["x_train"]
    y.sum().backward()
    assert torch.equal(x_train.grad, torch.ones_like(x_train))
    assert env["codes"].numel() == x_train.numel() // 2
    assert env["stack"].info_bits.shape == (20, 4096 * 2048 // 8)
