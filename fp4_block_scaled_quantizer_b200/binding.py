"""Python binding of the trace_fp4 C ABI (argument marshalling only).

Every step of the quantization path runs in the CUDA library
``libtrace_fp4.so`` built in-tree from ``csrc/``; this module only turns
torch tensors into pointers, allocates outputs with torch, and checks the
returned status.  There is no CPU fallback: if the library is missing the
first call raises.

The C entry points keep their names (``tf4_quantize_rtn``,
``tf4_quantize_sr``, ``tf4_quantize_capture``, ``tf4_quantize_guided``,
``tf4_dequantize``, ``tf4_pack_guidance``, ``tf4_unpack_guidance``,
``tf4_segment_amax``) as attributes of :func:`lib`; the Python functions of
the same names take tensors.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtrace_fp4.so")

NVFP4, MXFP4, UFP4 = 0, 1, 2
BLOCK = {NVFP4: 16, MXFP4: 32, UFP4: 16}
# formats with an fp32 per-segment tensor scale (and segments, a workspace)
HAS_TENSOR_SCALE = {NVFP4: True, MXFP4: False, UFP4: True}
MAX_SEGMENTS = 1024
DEV_NONFINITE, DEV_TIMEOUT = 1, 2

STATUS = {
    0: "TF4_OK", 1: "TF4_ERR_INVALID_ARG", 2: "TF4_ERR_SHAPE", 3: "TF4_ERR_ALIGN",
    4: "TF4_ERR_WORKSPACE", 5: "TF4_ERR_NONFINITE", 6: "TF4_ERR_TIMEOUT", 7: "TF4_ERR_CUDA",
}

# symbols declared in include/trace_fp4.h
EXPORTS = (
    "tf4_workspace_bytes", "tf4_codes_bytes", "tf4_scales_bytes", "tf4_guidance_bytes",
    "tf4_record_bytes", "tf4_segment_amax", "tf4_quantize_rtn", "tf4_quantize_sr",
    "tf4_quantize_capture", "tf4_quantize_guided", "tf4_dequantize", "tf4_pack_guidance",
    "tf4_unpack_guidance", "tf4_guided_fake_quant", "tf4_mismatch_stats", "tf4_workspace_bytes_batched",
    "tf4_quantize_capture_batched", "tf4_blocked_scales_bytes", "tf4_swizzle_scales", "tf4_quantize_capture_noalloc", "tf4_read_status", "tf4_status_string",
    "tf4_version",
)


class Tf4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


class tf4_desc(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32),
        ("num_segments", ctypes.c_int32),
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
        ("seg_row_offsets", ctypes.POINTER(ctypes.c_int64)),
    ]


_lib = None
_lock = threading.Lock()


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise ImportError(
                        f"trace_fp4 CUDA library not built ({LIB_PATH}); run "
                        "`python -m fp4_block_scaled_quantizer_b200.build`")
                L = ctypes.CDLL(LIB_PATH)
                vp, sz, st, i32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p
                dp = ctypes.POINTER(tf4_desc)
                sig = {
                    "tf4_workspace_bytes": (sz, [dp]),
                    "tf4_codes_bytes": (sz, [dp]),
                    "tf4_scales_bytes": (sz, [dp]),
                    "tf4_guidance_bytes": (sz, [dp]),
                    "tf4_record_bytes": (sz, [dp, ctypes.c_int]),
                    "tf4_segment_amax": (st, [dp, vp, vp, vp, sz, i32p, vp]),
                    "tf4_quantize_rtn": (st, [dp, vp, vp, vp, vp, vp, vp, sz, i32p, vp]),
                    "tf4_quantize_sr": (st, [dp, vp, ctypes.c_uint64, vp, vp, vp, vp, vp, sz, i32p, vp]),
                    "tf4_quantize_capture": (st, [dp, vp, vp, vp, vp, vp, vp, vp, sz, i32p, vp]),
                    "tf4_quantize_guided": (st, [dp, vp, vp, vp, vp, vp, i32p, vp]),
                    "tf4_dequantize": (st, [dp, vp, vp, vp, vp, vp]),
                    "tf4_pack_guidance": (st, [dp, vp, vp, vp]),
                    "tf4_unpack_guidance": (st, [dp, vp, vp, vp]),
                    "tf4_quantize_capture_noalloc": (st, [dp, vp, vp, vp, vp, vp, i32p, vp]),
                    "tf4_guided_fake_quant": (st, [dp, vp, vp, vp, vp, vp, vp, ctypes.c_int, i32p, vp]),
                    "tf4_mismatch_stats": (st, [dp, vp, vp, vp, vp, vp, i32p, vp]),
                    "tf4_workspace_bytes_batched": (sz, [ctypes.c_int32]),
                    "tf4_blocked_scales_bytes": (sz, [dp]),
                    "tf4_swizzle_scales": (st, [dp, vp, vp, vp]),
                    "tf4_quantize_capture_batched": (st, [dp, ctypes.c_int32, vp, vp, vp, vp, ctypes.c_int32, vp,
                                                          vp, sz, i32p, vp]),
                    "tf4_read_status": (st, [i32p, vp]),
                    "tf4_status_string": (ctypes.c_char_p, [st]),
                    "tf4_version": (ctypes.c_int, []),
                }
                for name, (res, args) in sig.items():
                    fn = getattr(L, name)
                    fn.restype = res
                    fn.argtypes = args
                _lib = L
    return _lib


# ------------------------------------------------------------------ helpers
@dataclass
class Desc:
    """Owns a tf4_desc and the host copy of its segment offsets."""
    fmt: int
    rows: int
    cols: int
    seg_off: Optional[Sequence[int]] = None

    def __post_init__(self):
        self._off = None
        nseg = 1
        if self.seg_off is not None:
            self._off = (ctypes.c_int64 * len(self.seg_off))(*[int(v) for v in self.seg_off])
            nseg = len(self.seg_off) - 1
        self.c = tf4_desc(self.fmt, nseg, self.rows, self.cols,
                          ctypes.cast(self._off, ctypes.POINTER(ctypes.c_int64)) if self._off else None)

    @property
    def num_segments(self) -> int:
        return self.c.num_segments

    @property
    def ptr(self):
        return ctypes.byref(self.c)

    @property
    def n(self) -> int:
        return self.rows * self.cols


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "expected a contiguous CUDA tensor"
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream], device) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != 0:
        raise Tf4Error(status, what)


def _as_2d(x: torch.Tensor):
    assert x.dtype == torch.bfloat16, "input must be bf16"
    assert x.is_cuda and x.is_contiguous()
    return x.reshape(-1, x.shape[-1]) if x.dim() != 2 else x


_ws_cache: dict = {}
_status_cache: dict = {}


def workspace(desc: Desc, device, stream=None) -> torch.Tensor:
    """A zero-filled workspace for this device/stream (reused: every call
    returns it to zero when it completes)."""
    return _workspace_bytes(lib().tf4_workspace_bytes(desc.ptr), device, stream)


def _workspace_bytes(need: int, device, stream=None) -> torch.Tensor:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    key = (torch.device(device).index, s.cuda_stream)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def status_word(device) -> torch.Tensor:
    key = torch.device(device).index
    t = _status_cache.get(key)
    if t is None:
        t = torch.zeros(1, dtype=torch.int32, device=device)
        _status_cache[key] = t
    return t


def read_status(device, stream=None) -> int:
    """Synchronize and return (and clear) the device status code."""
    t = status_word(device)
    return int(lib().tf4_read_status(_ptr(t), _stream(stream, t.device)))


def sizes(fmt: int, rows: int, cols: int, seg_off=None) -> dict:
    d = Desc(fmt, rows, cols, seg_off)
    L = lib()
    return dict(codes=L.tf4_codes_bytes(d.ptr), scales=L.tf4_scales_bytes(d.ptr),
                guidance=L.tf4_guidance_bytes(d.ptr), workspace=L.tf4_workspace_bytes(d.ptr),
                record_full=L.tf4_record_bytes(d.ptr, 1), record_compact=L.tf4_record_bytes(d.ptr, 0))


# --------------------------------------------------------------- entry points
@dataclass
class Quantized:
    codes: torch.Tensor                  # uint8 [rows*cols/2]
    scales: torch.Tensor                 # uint8 [rows, cols/block]
    s_t: Optional[torch.Tensor]          # float [num_segments] (NVFP4, UFP4)
    bits: Optional[torch.Tensor] = None  # uint8 [rows*cols/8] (capture)
    fmt: int = NVFP4
    rows: int = 0
    cols: int = 0
    seg_off: Optional[Sequence[int]] = None


def _outputs(desc: Desc, device, want_bits: bool, out: Optional[Quantized]):
    if out is not None:
        return out
    codes = torch.empty(desc.n // 2, dtype=torch.uint8, device=device)
    scales = torch.empty((desc.rows, desc.cols // BLOCK[desc.fmt]), dtype=torch.uint8, device=device)
    s_t = (torch.empty(desc.num_segments, dtype=torch.float32, device=device) if HAS_TENSOR_SCALE[desc.fmt]
           else None)
    bits = torch.empty(desc.n // 8, dtype=torch.uint8, device=device) if want_bits else None
    return Quantized(codes, scales, s_t, bits, desc.fmt, desc.rows, desc.cols, desc.seg_off)


def tf4_segment_amax(x: torch.Tensor, seg_off=None, stream=None, out=None) -> torch.Tensor:
    x2 = _as_2d(x)
    d = Desc(NVFP4, x2.shape[0], x2.shape[1], seg_off)
    amax = out if out is not None else torch.empty(d.num_segments, dtype=torch.float32, device=x.device)
    ws = workspace(d, x.device, stream)
    _check(lib().tf4_segment_amax(d.ptr, _ptr(x2), _ptr(amax), _ptr(ws), ws.numel(),
                                  _ptr(status_word(x.device)), _stream(stream, x.device)), "tf4_segment_amax")
    return amax


def tf4_quantize_rtn(x, fmt=NVFP4, seg_off=None, amax_in=None, stream=None, out=None) -> Quantized:
    x2 = _as_2d(x)
    d = Desc(fmt, x2.shape[0], x2.shape[1], seg_off)
    q = _outputs(d, x.device, False, out)
    ws = workspace(d, x.device, stream)
    _check(lib().tf4_quantize_rtn(d.ptr, _ptr(x2), _ptr(amax_in), _ptr(q.codes), _ptr(q.scales), _ptr(q.s_t),
                                  _ptr(ws), ws.numel(), _ptr(status_word(x.device)), _stream(stream, x.device)),
           "tf4_quantize_rtn")
    return q


def tf4_quantize_sr(x, seed: int, fmt=NVFP4, seg_off=None, amax_in=None, stream=None, out=None) -> Quantized:
    x2 = _as_2d(x)
    d = Desc(fmt, x2.shape[0], x2.shape[1], seg_off)
    q = _outputs(d, x.device, False, out)
    ws = workspace(d, x.device, stream)
    _check(lib().tf4_quantize_sr(d.ptr, _ptr(x2), ctypes.c_uint64(seed & (2**64 - 1)), _ptr(amax_in),
                                 _ptr(q.codes), _ptr(q.scales), _ptr(q.s_t), _ptr(ws), ws.numel(),
                                 _ptr(status_word(x.device)), _stream(stream, x.device)), "tf4_quantize_sr")
    return q


def tf4_quantize_capture(x, fmt=NVFP4, seg_off=None, guidance=True, amax_in=None, stream=None,
                         out=None) -> Quantized:
    """Rollout-side capture; ``guidance=False`` for layers whose guidance is
    not kept (codes/scales/s_t are then those of round-to-nearest)."""
    x2 = _as_2d(x)
    d = Desc(fmt, x2.shape[0], x2.shape[1], seg_off)
    q = _outputs(d, x.device, guidance, out)
    ws = workspace(d, x.device, stream)
    _check(lib().tf4_quantize_capture(d.ptr, _ptr(x2), _ptr(amax_in), _ptr(q.codes), _ptr(q.scales),
                                      _ptr(q.s_t), _ptr(q.bits if guidance else None), _ptr(ws), ws.numel(),
                                      _ptr(status_word(x.device)), _stream(stream, x.device)),
           "tf4_quantize_capture")
    return q


@dataclass
class BatchedCapture:
    codes: torch.Tensor            # uint8 [L, rows*cols/2]
    scales: torch.Tensor           # uint8 [L, rows, cols/block]
    s_t: Optional[torch.Tensor]    # float [L] (NVFP4, UFP4)
    info_bits: Optional[torch.Tensor]  # uint8 [keep, rows*cols/8]: the info cache
    fmt: int
    rows: int
    cols: int
    keep: int

    def layer(self, i: int) -> Quantized:
        """Layer i as a record usable by tf4_quantize_guided / tf4_dequantize."""
        L = self.codes.shape[0]
        bits = self.info_bits[i - (L - self.keep)] if i >= L - self.keep else None
        s_t = self.s_t[i:i + 1] if self.s_t is not None else None
        return Quantized(self.codes[i], self.scales[i], s_t, bits, self.fmt, self.rows, self.cols, None)


def tf4_quantize_capture_batched(xs, fmt=NVFP4, keep=0, stream=None, out: Optional[BatchedCapture] = None):
    """Capture a list of same-shaped bf16 tensors (layers) in two launches;
    guidance is kept for the last `keep` layers, in one contiguous buffer."""
    L = len(xs)
    x2 = [_as_2d(x) for x in xs]
    rows, cols = x2[0].shape
    assert all(t.shape == (rows, cols) for t in x2)
    dev = x2[0].device
    d = Desc(fmt, rows, cols)
    if out is None:
        n = rows * cols
        out = BatchedCapture(torch.empty((L, n // 2), dtype=torch.uint8, device=dev),
                             torch.empty((L, rows, cols // BLOCK[fmt]), dtype=torch.uint8, device=dev),
                             torch.empty(L, dtype=torch.float32, device=dev) if HAS_TENSOR_SCALE[fmt] else None,
                             torch.empty((keep, n // 8), dtype=torch.uint8, device=dev) if keep else None,
                             fmt, rows, cols, keep)
    ptrs = (ctypes.c_void_p * L)(*[t.data_ptr() for t in x2])
    ws = _workspace_bytes(lib().tf4_workspace_bytes_batched(L), dev, stream)
    _check(lib().tf4_quantize_capture_batched(d.ptr, L, ptrs, _ptr(out.codes), _ptr(out.scales), _ptr(out.s_t),
                                              keep, _ptr(out.info_bits), _ptr(ws), ws.numel(),
                                              _ptr(status_word(dev)), _stream(stream, dev)),
           "tf4_quantize_capture_batched")
    return out


def tf4_quantize_guided(x, rec: Quantized, stream=None, out=None, rec_bits=None) -> torch.Tensor:
    """Train-side guided quantization of x against a rollout record."""
    x2 = _as_2d(x)
    d = Desc(rec.fmt, x2.shape[0], x2.shape[1], rec.seg_off)
    bits = rec_bits if rec_bits is not None else rec.bits
    assert bits is not None, "the record holds no guidance bits"
    codes = out if out is not None else torch.empty(d.n // 2, dtype=torch.uint8, device=x.device)
    _check(lib().tf4_quantize_guided(d.ptr, _ptr(x2), _ptr(rec.scales), _ptr(rec.s_t), _ptr(bits), _ptr(codes),
                                     _ptr(status_word(x.device)), _stream(stream, x.device)), "tf4_quantize_guided")
    return codes


def tf4_guided_fake_quant(x, rec: Quantized, out_dtype=torch.float32, want_codes=False, stream=None,
                          out=None, codes=None, rec_bits=None):
    """Guided quantization + dequantization in one pass.  Returns (values,
    codes): values [rows, cols] in out_dtype (float32, or bfloat16 = RNE of
    the fp32 value); codes only if want_codes (else None)."""
    assert out_dtype in (torch.float32, torch.bfloat16)
    x2 = _as_2d(x)
    d = Desc(rec.fmt, x2.shape[0], x2.shape[1], rec.seg_off)
    bits = rec_bits if rec_bits is not None else rec.bits
    assert bits is not None, "the record holds no guidance bits"
    o = out if out is not None else torch.empty(x2.shape, dtype=out_dtype, device=x.device)
    c = codes if codes is not None else (
        torch.empty(d.n // 2, dtype=torch.uint8, device=x.device) if want_codes else None)
    _check(lib().tf4_guided_fake_quant(d.ptr, _ptr(x2), _ptr(rec.scales), _ptr(rec.s_t), _ptr(bits), _ptr(c),
                                       _ptr(o), 1 if o.dtype == torch.bfloat16 else 0,
                                       _ptr(status_word(x.device)), _stream(stream, x.device)),
           "tf4_guided_fake_quant")
    return o, c


def tf4_mismatch_stats(x, rec: Quantized, counts=None, stream=None) -> torch.Tensor:
    """Mismatch diagnostics of train values x against a rollout record
    (codes + scales): adds [#mismatch, #adjacent, #far, #after-guidance] to
    `counts` (int64 [4], zero-initialised if not given) and returns it."""
    x2 = _as_2d(x)
    d = Desc(rec.fmt, x2.shape[0], x2.shape[1], rec.seg_off)
    c = counts if counts is not None else torch.zeros(4, dtype=torch.int64, device=x.device)
    _check(lib().tf4_mismatch_stats(d.ptr, _ptr(x2), _ptr(rec.scales), _ptr(rec.s_t), _ptr(rec.codes), _ptr(c),
                                    _ptr(status_word(x.device)), _stream(stream, x.device)), "tf4_mismatch_stats")
    return c


def tf4_dequantize(q: Quantized, codes=None, stream=None, out=None) -> torch.Tensor:
    d = Desc(q.fmt, q.rows, q.cols, q.seg_off)
    c = codes if codes is not None else q.codes
    o = out if out is not None else torch.empty((q.rows, q.cols), dtype=torch.float32, device=c.device)
    _check(lib().tf4_dequantize(d.ptr, _ptr(c), _ptr(q.scales), _ptr(q.s_t), _ptr(o), _stream(stream, c.device)),
           "tf4_dequantize")
    return o


def tf4_swizzle_scales(q: Quantized, stream=None, out=None) -> torch.Tensor:
    """The record's block scales in the tiled layout block-scaled FP4 GEMMs
    read (uint8 [ceil(rows/128)*128, ceil(nb/4)*4] as laid out in memory)."""
    d = Desc(q.fmt, q.rows, q.cols, q.seg_off)
    nb = q.cols // BLOCK[q.fmt]
    shape = ((q.rows + 127) // 128 * 128, (nb + 3) // 4 * 4)
    assert lib().tf4_blocked_scales_bytes(d.ptr) == shape[0] * shape[1]
    o = out if out is not None else torch.empty(shape, dtype=torch.uint8, device=q.scales.device)
    _check(lib().tf4_swizzle_scales(d.ptr, _ptr(q.scales), _ptr(o), _stream(stream, q.scales.device)),
           "tf4_swizzle_scales")
    return o


def tf4_pack_guidance(codes: torch.Tensor, rows: int, cols: int, fmt=NVFP4, stream=None, out=None):
    d = Desc(fmt, rows, cols)
    o = out if out is not None else torch.empty(d.n // 8, dtype=torch.uint8, device=codes.device)
    _check(lib().tf4_pack_guidance(d.ptr, _ptr(codes), _ptr(o), _stream(stream, codes.device)),
           "tf4_pack_guidance")
    return o


def tf4_unpack_guidance(bits: torch.Tensor, rows: int, cols: int, fmt=NVFP4, stream=None, out=None):
    d = Desc(fmt, rows, cols)
    o = out if out is not None else torch.empty(d.n, dtype=torch.uint8, device=bits.device)
    _check(lib().tf4_unpack_guidance(d.ptr, _ptr(bits), _ptr(o), _stream(stream, bits.device)),
           "tf4_unpack_guidance")
    return o


def capture_layers(num_layers: int, keep: int) -> list:
    """Layer indices whose guidance is kept: the deepest `keep` of
    `num_layers` (the highest indices)."""
    keep = max(0, min(keep, num_layers))
    return list(range(num_layers - keep, num_layers))
