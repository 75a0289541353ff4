"""The single-launch capture of tensors up to 2^25 elements (one segment):
its results equal the oracle's and the two-launch path's, and its bounded
grid-wide wait gives up with TF4_DEV_TIMEOUT, leaving the GPU usable, when
the wait cannot end (a workspace whose arrival counter was not zero)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from fp4_block_scaled_quantizer_b200 import binding as B
from fp4_block_scaled_quantizer_b200 import build as libbuild
from fp4_block_scaled_quantizer_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"
FUSED_MAX = 1 << 25
TIMEOUT = 6  # TF4_ERR_TIMEOUT


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    libbuild.build()
    B.lib()
    O.lib()


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("fmt", [B.NVFP4, B.UFP4])
@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (257, 2048), (4096, 2048), (8192, 4096)])
def test_single_launch_equals_oracle_and_two_launch_path(fmt, shape):
    rows, cols = shape
    assert rows * cols <= FUSED_MAX
    x = W.random_bf16(shape, seed=rows + cols, device=DEV, outlier_frac=0.002)
    q = B.tf4_quantize_capture(x, fmt=fmt)            # single launch
    amax = B.tf4_segment_amax(x)
    q2 = B.tf4_quantize_capture(x, fmt=fmt, amax_in=amax)  # amax pass, then the quantize launch
    qr = B.tf4_quantize_rtn(x, fmt=fmt)
    assert B.read_status(x.device) == 0
    for name in ("codes", "scales", "s_t", "bits"):
        assert torch.equal(getattr(q, name), getattr(q2, name)), name
    assert torch.equal(q.codes, qr.codes) and torch.equal(q.scales, qr.scales)
    if rows * cols <= 1 << 21:
        r = O.quantize(W.bf16_bits(x), fmt, O.RTN, bits=True)
        assert np.array_equal(q.codes.cpu().numpy(), r["codes"])
        assert np.array_equal(q.scales.cpu().numpy().reshape(-1), r["scales"])
        assert np.array_equal(q.bits.cpu().numpy(), r["bits"])
        assert np.array_equal(q.s_t.cpu().numpy().view(np.uint32), r["s_t"].view(np.uint32))


def test_just_above_the_single_launch_size_takes_two_launches():
    x = W.random_bf16((8193, 4096), seed=3, device=DEV)
    assert x.numel() > FUSED_MAX
    q = B.tf4_quantize_capture(x)
    q2 = B.tf4_quantize_capture(x, amax_in=B.tf4_segment_amax(x))
    assert torch.equal(q.codes, q2.codes) and torch.equal(q.bits, q2.bits)


def test_single_launch_wait_times_out_and_recovers():
    """A workspace whose arrival counter (word 1) is not zero: no CTA sees
    the count it waits for, every wait gives up after its bound, the call
    reports TF4_ERR_TIMEOUT, and after the workspace is zero-filled again the
    same call gives the right result."""
    L = B.lib()
    rows, cols = 512, 1024
    x = W.random_bf16((rows, cols), seed=5, device=DEV)
    ref = B.tf4_quantize_capture(x)
    d = B.Desc(B.NVFP4, rows, cols)
    ws = torch.zeros(64, dtype=torch.int32, device=DEV)
    ws[1] = 1 << 30
    codes = torch.empty(rows * cols // 2, dtype=torch.uint8, device=DEV)
    scales = torch.empty(rows * cols // 16, dtype=torch.uint8, device=DEV)
    s_t = torch.empty(1, dtype=torch.float32, device=DEV)
    bits = torch.empty(rows * cols // 8, dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert L.tf4_quantize_capture(d.ptr, _p(x), None, _p(codes), _p(scales), _p(s_t), _p(bits), _p(ws), 256,
                                  _p(st), s) == 0
    assert L.tf4_read_status(_p(st), s) == TIMEOUT
    ws.zero_()
    assert L.tf4_quantize_capture(d.ptr, _p(x), None, _p(codes), _p(scales), _p(s_t), _p(bits), _p(ws), 256,
                                  _p(st), s) == 0
    assert L.tf4_read_status(_p(st), s) == 0
    assert torch.equal(codes, ref.codes) and torch.equal(bits, ref.bits)
    assert int(ws.count_nonzero()) == 0  # left zero-filled by the call


def test_binding_zero_fills_its_workspace_after_a_timeout():
    x = W.random_bf16((64, 512), seed=6, device=DEV)
    ref = B.tf4_quantize_capture(x)
    torch.cuda.synchronize()
    ws = B.workspace(B.Desc(B.NVFP4, 64, 512), x.device)
    ws.view(torch.int32)[1] = 1 << 30  # the state a timed-out call leaves behind
    B.tf4_quantize_capture(x)
    assert B.read_status(x.device) == TIMEOUT
    q = B.tf4_quantize_capture(x)
    assert B.read_status(x.device) == 0
    assert torch.equal(q.codes, ref.codes)
