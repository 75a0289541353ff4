"""The multi-process oracle runner used by the CPU baseline does the same
work as the oracle called directly (no GPU)."""
import numpy as np

import oracle as O
from oracle.pool import OraclePool, _layer_task


def test_pool_matches_direct_calls():
    rng = np.random.default_rng(0)
    xs = [(rng.standard_normal((16, 256)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
          for _ in range(4)]
    xts = [(x.astype(np.uint32) ^ 1).astype(np.uint16) for x in xs[2:]]
    pool = OraclePool(2)
    try:
        got = pool.run(xs, xts, 2)
    finally:
        pool.close()
    want = [_layer_task((x, xts[i - 2] if i >= 2 else None)) for i, x in enumerate(xs)]
    assert got == want
    r = O.quantize(xs[0], O.NVFP4)
    assert got[0] == [int(r["codes"].sum()), int(r["scales"].sum())]
