"""The allocation-free capture entry point.

Some callers cannot allocate device memory or provide a workspace (for
example a plug-in inside an engine that owns all device memory), so the
library offers tf4_quantize_capture_noalloc, whose amax scratch lives in a
fixed device array inside the library.  This checks, through the C ABI,
that it produces exactly what tf4_quantize_capture produces, on two calls
in a row (the second call reuses the scratch the first one left behind),
and that it refuses more segments than its scratch holds.

This file is named to be collected last, so that a run that stops at the
first failure has already run every other test.
"""
import ctypes

import pytest
import torch

from fp4_block_scaled_quantizer_b200 import binding as B
from fp4_block_scaled_quantizer_b200 import build as libbuild
from fp4_block_scaled_quantizer_b200 import workloads as W

pytestmark = pytest.mark.gpu

MAX_SEGMENTS = 256  # TF4_NOALLOC_MAX_SEGMENTS in include/trace_fp4.h


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc_capture(L, x, seg, with_bits=True, fmt=B.NVFP4, stream=None):
    rows, cols = x.shape
    d = B.Desc(fmt, rows, cols, seg)
    codes = torch.empty(rows * cols // 2, dtype=torch.uint8, device=x.device)
    scales = torch.empty((rows, cols // B.BLOCK[fmt]), dtype=torch.uint8, device=x.device)
    s_t = torch.empty(d.num_segments, dtype=torch.float32, device=x.device) if B.HAS_TENSOR_SCALE[fmt] else None
    bits = torch.empty(rows * cols // 8, dtype=torch.uint8, device=x.device) if with_bits else None
    s = stream if stream is not None else torch.cuda.current_stream(x.device)
    st = L.tf4_quantize_capture_noalloc(d.ptr, _p(x), _p(codes), _p(scales), _p(s_t), _p(bits),
                                        _p(B.status_word(x.device, stream)), ctypes.c_void_p(s.cuda_stream))
    return st, codes, scales, s_t, bits


@pytest.mark.parametrize("fmt", [B.NVFP4, B.UFP4, B.MXFP4])
def test_noalloc_capture_matches_workspace_capture(fmt):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    libbuild.build()
    L = B.lib()
    cases = [
        ((300, 1024), [0, 120, 120, 300]),   # ragged segments, one empty
        ((257, 2048), None),                 # one segment, several CTAs
    ]
    for call, ((rows, cols), seg) in enumerate(cases):
        if seg is not None and not B.HAS_TENSOR_SCALE[fmt]:
            continue  # MXFP4 has no tensor scale, hence no segments
        x = W.random_bf16((rows, cols), seed=100 + call, device="cuda", outlier_frac=0.01)
        ref = B.tf4_quantize_capture(x, fmt=fmt, seg_off=seg)
        st, codes, scales, s_t, bits = _noalloc_capture(L, x, seg, fmt=fmt)
        assert st == 0, B.STATUS.get(st, st)
        assert B.read_status(x.device) == 0
        assert torch.equal(codes, ref.codes)
        assert torch.equal(scales.view(-1), ref.scales.view(-1))
        if B.HAS_TENSOR_SCALE[fmt]:
            assert torch.equal(s_t.view(torch.int32), ref.s_t.view(torch.int32))
        assert torch.equal(bits, ref.bits)


def test_noalloc_capture_rejects_too_many_segments():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    libbuild.build()
    L = B.lib()
    rows = MAX_SEGMENTS + 1
    x = W.random_bf16((rows, 32), seed=7, device="cuda")
    seg = list(range(rows + 1))  # one row per segment: MAX_SEGMENTS + 1 segments
    st, *_ = _noalloc_capture(L, x, seg)
    assert st == 4  # TF4_ERR_WORKSPACE: more segments than the static scratch holds
    st, codes, *_ = _noalloc_capture(L, x[:MAX_SEGMENTS], list(range(MAX_SEGMENTS + 1)))
    assert st == 0
    ref = B.tf4_quantize_capture(x[:MAX_SEGMENTS].contiguous(), seg_off=list(range(MAX_SEGMENTS + 1)))
    assert torch.equal(codes, ref.codes)


def test_noalloc_capture_on_a_created_stream():
    """A stream the caller created on the current device is accepted (the
    call checks that the stream belongs to the current device, whose copy
    of the scratch array it uses)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    libbuild.build()
    L = B.lib()
    x = W.random_bf16((130, 512), seed=9, device="cuda", outlier_frac=0.01)
    ref = B.tf4_quantize_capture(x, seg_off=[0, 64, 130])
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    for _ in range(2):
        st, codes, scales, s_t, bits = _noalloc_capture(L, x, [0, 64, 130], stream=s)
        assert st == 0, B.STATUS.get(st, st)
        s.synchronize()
        assert torch.equal(codes, ref.codes) and torch.equal(bits, ref.bits)
        assert torch.equal(s_t.view(torch.int32), ref.s_t.view(torch.int32))
