"""Host-side tests of the C ABI (no GPU): the library loads, exports every
symbol the header declares, sizes its records, and rejects bad arguments
synchronously -- before any CUDA call, so these run on a CPU-only host."""
import ctypes
import os
import re
from fractions import Fraction as F

import pytest

import fp4_block_scaled_quantizer_b200 as tf4
from fp4_block_scaled_quantizer_b200 import binding as B
from fp4_block_scaled_quantizer_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "trace_fp4.h")


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return B.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tf4_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    want = {"tf4_quantize_rtn", "tf4_quantize_sr", "tf4_quantize_capture", "tf4_quantize_guided",
            "tf4_dequantize", "tf4_pack_guidance", "tf4_unpack_guidance"}
    assert want <= set(declared_functions())


def test_library_exports_every_declared_symbol(L):
    names = declared_functions()
    assert set(names) == set(B.EXPORTS)
    for n in names:
        assert hasattr(L, n), n
    assert L.tf4_version() >= 1


def test_status_strings(L):
    for code in range(8):
        assert L.tf4_status_string(code)


def test_sizes_and_one_sixth(L):
    """Record sizes; the 40-layer activation stack keeping the deepest 20
    layers' compact record retains 1/6 of the full information (NVFP4,
    ignoring the 4-byte tensor scale)."""
    rows, cols = 65536, 4096
    s = B.sizes(B.NVFP4, rows, cols)
    n = rows * cols
    assert s["codes"] == n // 2 and s["scales"] == n // 16 and s["guidance"] == n // 8
    assert s["record_full"] == n // 2 + n // 16 + 4
    assert s["record_compact"] == n // 8 + n // 16 + 4
    keep = B.capture_layers(40, 20)
    assert keep == list(range(20, 40))
    ratio = F(len(keep) * (s["record_compact"] - 4), 40 * (s["record_full"] - 4))
    assert ratio == F(1, 6)
    m = B.sizes(B.MXFP4, 8192, 28672)
    assert m["scales"] == 8192 * 28672 // 32 and m["workspace"] == 0
    seg = [0, 3, 3, 10]
    assert B.sizes(B.NVFP4, 10, 64, seg)["record_full"] == 320 + 40 + 12


BAD = ctypes.c_void_p(0x1001)   # misaligned, never dereferenced
GOOD = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced (rejected first)


def _rtn(L, d, x=GOOD, codes=GOOD, scales=GOOD, s_t=GOOD, ws=GOOD, wsb=4096, amax=None):
    return L.tf4_quantize_rtn(d.ptr if d is not None else None, x, amax, codes, scales, s_t, ws, wsb, None, None)


def test_rejects_bad_shapes(L):
    assert _rtn(L, B.Desc(B.NVFP4, 4, 24)) == 2           # cols % 16
    assert _rtn(L, B.Desc(B.MXFP4, 4, 48)) == 2           # cols % 32
    assert _rtn(L, B.Desc(B.NVFP4, -1, 16)) == 2
    assert _rtn(L, B.Desc(B.NVFP4, 4, 0)) == 2
    assert _rtn(L, B.Desc(B.NVFP4, 2**40, 2**40)) == 2    # overflow
    assert _rtn(L, None) == 1
    assert _rtn(L, B.Desc(7, 4, 16)) == 1                 # unknown format


def test_rejects_bad_segments(L):
    assert _rtn(L, B.Desc(B.NVFP4, 10, 16, [0, 5, 4, 10])) == 1   # decreasing
    assert _rtn(L, B.Desc(B.NVFP4, 10, 16, [1, 5, 10])) == 1      # not starting at 0
    assert _rtn(L, B.Desc(B.NVFP4, 10, 16, [0, 5, 9])) == 1       # not ending at rows
    assert _rtn(L, B.Desc(B.MXFP4, 10, 32, [0, 5, 10])) == 1      # MXFP4 has no segments
    d = B.Desc(B.NVFP4, 10, 16)
    d.c.num_segments = 3                                           # offsets missing
    assert _rtn(L, d) == 1
    d.c.num_segments = B.MAX_SEGMENTS + 1
    assert _rtn(L, d) == 1


def test_rejects_misaligned_pointers(L):
    d = B.Desc(B.NVFP4, 4, 32)
    assert _rtn(L, d, x=BAD) == 3
    assert _rtn(L, d, codes=BAD) == 3
    assert _rtn(L, d, s_t=ctypes.c_void_p(0x10002)) == 3
    assert L.tf4_dequantize(d.ptr, GOOD, GOOD, GOOD, BAD, None) == 3
    assert L.tf4_unpack_guidance(d.ptr, GOOD, BAD, None) == 3
    assert L.tf4_quantize_guided(d.ptr, GOOD, GOOD, GOOD, ctypes.c_void_p(0x10002), GOOD, None, None) == 3


def test_rejects_missing_pointers_and_workspace(L):
    d = B.Desc(B.NVFP4, 4, 32)
    assert _rtn(L, d, x=None) == 1
    assert _rtn(L, d, s_t=None) == 1
    assert _rtn(L, d, ws=None) == 4
    assert _rtn(L, d, wsb=4) == 4
    assert L.tf4_quantize_guided(d.ptr, GOOD, GOOD, None, GOOD, GOOD, None, None) == 1
    assert L.tf4_segment_amax(B.Desc(B.MXFP4, 4, 32).ptr, GOOD, GOOD, GOOD, 4096, None, None) == 1
    assert L.tf4_read_status(None, None) == 1
    assert L.tf4_workspace_bytes(d.ptr) >= 8
    assert L.tf4_workspace_bytes(B.Desc(B.NVFP4, 4, 24).ptr) == 0


def test_product_path_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB_PATH", "/nonexistent/libtrace_fp4.so")
    with pytest.raises(ImportError):
        B.lib()


def test_package_exports_entry_points():
    for n in ("tf4_quantize_rtn", "tf4_quantize_sr", "tf4_quantize_capture", "tf4_quantize_guided",
              "tf4_dequantize", "tf4_pack_guidance", "tf4_unpack_guidance", "tf4_segment_amax"):
        assert callable(getattr(tf4, n))


def test_batched_capture_rejects_bad_arguments(L):
    d = B.Desc(B.NVFP4, 4, 32)
    ptrs = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    call = lambda desc, nl, x, keep, info, ws=GOOD, wsb=4096, s_t=GOOD: L.tf4_quantize_capture_batched(
        desc.ptr, nl, x, GOOD, GOOD, s_t, keep, info, ws, wsb, None, None)
    assert call(d, 0, ptrs, 0, None) == 1                       # no layers
    assert call(d, 65, ptrs, 0, None) == 1                      # more than TF4_MAX_BATCH
    assert call(d, 2, None, 0, None) == 1                       # no pointer array
    assert call(d, 2, ptrs, 3, GOOD) == 1                       # keep > num_layers
    assert call(d, 2, ptrs, 1, None) == 1                       # keep > 0 without a buffer
    assert call(d, 2, ptrs, 0, GOOD) == 1                       # buffer without keep
    assert call(B.Desc(B.NVFP4, 4, 32, [0, 2, 4]), 2, ptrs, 0, None) == 1  # segmented layers
    assert call(d, 2, (ctypes.c_void_p * 2)(0x10000, 0x20001), 0, None) == 3  # misaligned layer
    assert call(d, 2, ptrs, 0, None, wsb=4) == 4                # workspace too small
    assert call(d, 2, ptrs, 0, None, s_t=None) == 1
    assert L.tf4_workspace_bytes_batched(3) == 256 and L.tf4_workspace_bytes_batched(0) == 0


def test_uniform_grid_format_arguments(L):
    """UFP4 uses NVFP4's container: 16-element blocks, segments and a
    workspace; unknown format numbers are refused."""
    assert _rtn(L, B.Desc(B.UFP4, 4, 24)) == 2                       # cols % 16
    assert L.tf4_workspace_bytes(B.Desc(B.UFP4, 4, 32).ptr) >= 8
    assert L.tf4_workspace_bytes(B.Desc(B.UFP4, 10, 32, [0, 5, 10]).ptr) >= 12
    assert _rtn(L, B.Desc(B.UFP4, 10, 16, [0, 5, 4, 10])) == 1       # decreasing offsets
    assert _rtn(L, B.Desc(B.UFP4, 4, 32), s_t=None) == 1             # tensor scale required
    assert _rtn(L, B.Desc(3, 4, 32)) == 1
    s = B.sizes(B.UFP4, 64, 128)
    assert s["scales"] == 64 * 128 // 16 and s["record_full"] == 64 * 128 // 2 + 64 * 128 // 16 + 4


def test_binding_rejects_bad_tensors_before_the_library():
    """The binding checks dtype, device and layout of its inputs and the
    size of caller-supplied buffers (the C ABI sees only pointers); on a
    CPU-only host every such call is refused before any pointer is passed."""
    import torch

    with pytest.raises(TypeError):
        B.tf4_quantize_capture(torch.zeros(4, 16, dtype=torch.float32))
    with pytest.raises(ValueError):
        B.tf4_quantize_capture(torch.zeros(4, 16, dtype=torch.bfloat16))  # host tensor
    with pytest.raises(ValueError):
        B.tf4_quantize_capture(torch.zeros(16, 4, dtype=torch.bfloat16).t())  # not contiguous
    with pytest.raises(ValueError):
        B._buf(torch.zeros(8, dtype=torch.uint8), "out", 8, torch.uint8, torch.device("cuda", 0))
    with pytest.raises(TypeError):
        B._buf(None, "out", 8, torch.uint8, torch.device("cuda", 0))
    with pytest.raises(ValueError):
        B.tf4_quantize_capture_batched([])
    with pytest.raises(ValueError):
        B.tf4_pack_guidance(torch.zeros(8, dtype=torch.uint8), 1, 16)


def test_debug_bounds_entry_points(L):
    """The release library reports no bounds checking; the checked build
    (if present) reports it; a NULL count is refused before any CUDA call."""
    assert L.tf4_debug_bounds_enabled() == 0
    assert L.tf4_debug_bounds_violations(None, None) == 1
    if os.path.exists(B.DEBUG_LIB_PATH):
        D = ctypes.CDLL(B.DEBUG_LIB_PATH)
        assert D.tf4_debug_bounds_enabled() == 1
