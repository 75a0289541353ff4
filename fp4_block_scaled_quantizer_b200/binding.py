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

import contextlib
import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtrace_fp4.so")
DEBUG_LIB_PATH = os.path.join(HERE, "libtrace_fp4_debug.so")  # built with --debug-bounds

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
    "tf4_workspace_bytes", "tf4_codes_bytes", "tf4_scales_bytes", "tf4_guidance_bytes", "tf4_record_bytes",
    "tf4_segment_amax", "tf4_quantize_rtn", "tf4_quantize_sr", "tf4_quantize_capture", "tf4_quantize_guided",
    "tf4_dequantize", "tf4_pack_guidance", "tf4_unpack_guidance", "tf4_guided_fake_quant", "tf4_mismatch_stats",
    "tf4_workspace_bytes_batched", "tf4_quantize_capture_batched", "tf4_blocked_scales_bytes", "tf4_swizzle_scales",
    "tf4_quantize_capture_noalloc", "tf4_read_status", "tf4_status_string", "tf4_version",
    "tf4_debug_bounds_enabled", "tf4_debug_bounds_violations",
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
                    "tf4_debug_bounds_enabled": (ctypes.c_int, []),
                    "tf4_debug_bounds_violations": (st, [ctypes.POINTER(ctypes.c_uint64), vp]),
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
    if not (t.is_cuda and t.is_contiguous()):
        raise ValueError(f"expected a contiguous CUDA tensor, got one on {t.device}"
                         f"{'' if t.is_contiguous() else ' (not contiguous)'}")
    return ctypes.c_void_p(t.data_ptr())


def _buf(t: Optional[torch.Tensor], name: str, numel: int, dtype: torch.dtype, device: torch.device):
    """Check a caller-supplied buffer before its pointer is handed to the
    library, which cannot see sizes: a CUDA tensor on `device`, contiguous,
    of `dtype`, with at least `numel` elements (the kernels read or write
    exactly `numel`; a shorter buffer would be overrun)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name}: expected a CUDA tensor on {device}, got one on {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected dtype {dtype}, got {t.dtype}")
    if t.numel() < numel:
        raise ValueError(f"{name}: needs {numel} elements, has {t.numel()}")
    return t


def _stream(stream: Optional[torch.cuda.Stream], device) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != 0:
        raise Tf4Error(status, what)


def _as_2d(x: torch.Tensor):
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"expected a torch.Tensor, got {type(x).__name__}")
    if x.dtype != torch.bfloat16:
        raise TypeError(f"input must be bf16, got {x.dtype}")
    if not (x.is_cuda and x.is_contiguous()):
        raise ValueError(f"input must be a contiguous CUDA tensor (got one on {x.device})")
    if x.dim() == 0:
        raise ValueError("input must have at least one dimension")
    return x.reshape(-1, x.shape[-1]) if x.dim() != 2 else x


def _check_record(rec, desc: "Desc", device, name: str, bits=None, codes=False):
    """Sizes of a rollout record's buffers against the shape they are used with."""
    nb = desc.n // BLOCK[desc.fmt]
    _buf(rec.scales, f"{name}: record scales", nb, torch.uint8, device)
    if HAS_TENSOR_SCALE[desc.fmt]:
        _buf(rec.s_t, f"{name}: record s_t", desc.num_segments, torch.float32, device)
    if bits is not None:
        _buf(bits, f"{name}: guidance bits", desc.n // 8, torch.uint8, device)
    if codes:
        _buf(rec.codes, f"{name}: record codes", desc.n // 2, torch.uint8, device)


_ws_cache: dict = {}
_status_cache: dict = {}


def _on(stream):
    """Context in which torch allocates and fills on `stream` (the stream
    the library call will launch on), so that a new output, workspace or
    status word is ordered before the call's kernels; no-op for None (the
    current stream)."""
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def _stream_key(device, stream=None):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return (torch.device(device).index, s.cuda_stream), s


def workspace(desc: Desc, device, stream=None) -> torch.Tensor:
    """A zero-filled workspace for this device/stream (reused: every call
    returns it to zero when it completes)."""
    return _workspace_bytes(lib().tf4_workspace_bytes(desc.ptr), device, stream)


def _workspace_bytes(need: int, device, stream=None) -> torch.Tensor:
    key, s = _stream_key(device, stream)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < need:
        with torch.cuda.stream(s):  # zero-filled on the stream that will use it
            ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def status_word(device, stream=None) -> torch.Tensor:
    """The device status word the library's calls on (device, stream) OR
    their data-dependent errors into: one per stream, so that reading it
    (read_status synchronizes that stream only) never races with kernels
    still running on another stream."""
    key, s = _stream_key(device, stream)
    t = _status_cache.get(key)
    if t is None:
        with torch.cuda.stream(s):
            t = torch.zeros(1, dtype=torch.int32, device=device)
        _status_cache[key] = t
    return t


@contextlib.contextmanager
def use_library(path: str):
    """Route this module's calls through the library at `path` (for example
    the bounds-checking build, DEBUG_LIB_PATH) inside the `with` block."""
    global _lib, LIB_PATH
    with _lock:
        saved = (_lib, LIB_PATH)
        _lib, LIB_PATH = None, path
    try:
        yield lib()
    finally:
        with _lock:
            _lib, LIB_PATH = saved


def debug_bounds_violations(device=None, stream=None) -> int:
    """Synchronize and return (and reset) the number of work units the
    kernels skipped as out of range; always 0 unless the loaded library is
    the bounds-checking build."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    n = ctypes.c_uint64(0)
    _check(lib().tf4_debug_bounds_violations(ctypes.byref(n), _stream(stream, dev)), "tf4_debug_bounds_violations")
    return int(n.value)


def read_status(device, stream=None) -> int:
    """Synchronize `stream` (default: the current stream) and return (and
    clear) the status code of the calls issued on it.  After a timed-out
    wait (status 6) the stream's cached workspace is zero-filled again, as
    the library requires before its reuse."""
    t = status_word(device, stream)
    st = int(lib().tf4_read_status(_ptr(t), _stream(stream, t.device)))
    if st == 6:
        key, s = _stream_key(t.device, stream)
        ws = _ws_cache.get(key)
        if ws is not None:
            with torch.cuda.stream(s):
                ws.zero_()
    return st


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
        _buf(out.codes, "out.codes", desc.n // 2, torch.uint8, device)
        _buf(out.scales, "out.scales", desc.n // BLOCK[desc.fmt], torch.uint8, device)
        if HAS_TENSOR_SCALE[desc.fmt]:
            _buf(out.s_t, "out.s_t", desc.num_segments, torch.float32, device)
        if want_bits:
            _buf(out.bits, "out.bits", desc.n // 8, torch.uint8, device)
        # the record describes what this call wrote
        out.fmt, out.rows, out.cols, out.seg_off = desc.fmt, desc.rows, desc.cols, desc.seg_off
        return out
    codes = torch.empty(desc.n // 2, dtype=torch.uint8, device=device)
    scales = torch.empty((desc.rows, desc.cols // BLOCK[desc.fmt]), dtype=torch.uint8, device=device)
    s_t = (torch.empty(desc.num_segments, dtype=torch.float32, device=device) if HAS_TENSOR_SCALE[desc.fmt]
           else None)
    bits = torch.empty(desc.n // 8, dtype=torch.uint8, device=device) if want_bits else None
    return Quantized(codes, scales, s_t, bits, desc.fmt, desc.rows, desc.cols, desc.seg_off)


def _amax_in(amax_in, desc: Desc, device):
    if amax_in is not None:
        _buf(amax_in, "amax_in", desc.num_segments, torch.float32, device)


def tf4_segment_amax(x: torch.Tensor, seg_off=None, stream=None, out=None) -> torch.Tensor:
    with _on(stream):
        x2 = _as_2d(x)
        d = Desc(NVFP4, x2.shape[0], x2.shape[1], seg_off)
        amax = (_buf(out, "out", d.num_segments, torch.float32, x.device) if out is not None
                else torch.empty(d.num_segments, dtype=torch.float32, device=x.device))
        ws = workspace(d, x.device, stream)
        _check(lib().tf4_segment_amax(d.ptr, _ptr(x2), _ptr(amax), _ptr(ws), ws.numel(),
                                      _ptr(status_word(x.device, stream)), _stream(stream, x.device)),
               "tf4_segment_amax")
        return amax


def tf4_quantize_rtn(x, fmt=NVFP4, seg_off=None, amax_in=None, stream=None, out=None) -> Quantized:
    with _on(stream):
        x2 = _as_2d(x)
        d = Desc(fmt, x2.shape[0], x2.shape[1], seg_off)
        q = _outputs(d, x.device, False, out)
        _amax_in(amax_in, d, x.device)
        ws = workspace(d, x.device, stream)
        _check(lib().tf4_quantize_rtn(d.ptr, _ptr(x2), _ptr(amax_in), _ptr(q.codes), _ptr(q.scales), _ptr(q.s_t),
                                      _ptr(ws), ws.numel(), _ptr(status_word(x.device, stream)),
                                      _stream(stream, x.device)),
               "tf4_quantize_rtn")
        return q


def tf4_quantize_sr(x, seed: int, fmt=NVFP4, seg_off=None, amax_in=None, stream=None, out=None) -> Quantized:
    with _on(stream):
        x2 = _as_2d(x)
        d = Desc(fmt, x2.shape[0], x2.shape[1], seg_off)
        q = _outputs(d, x.device, False, out)
        _amax_in(amax_in, d, x.device)
        ws = workspace(d, x.device, stream)
        _check(lib().tf4_quantize_sr(d.ptr, _ptr(x2), ctypes.c_uint64(seed & (2**64 - 1)), _ptr(amax_in),
                                     _ptr(q.codes), _ptr(q.scales), _ptr(q.s_t), _ptr(ws), ws.numel(),
                                     _ptr(status_word(x.device, stream)), _stream(stream, x.device)), "tf4_quantize_sr")
        return q


def tf4_quantize_capture(x, fmt=NVFP4, seg_off=None, guidance=True, amax_in=None, stream=None,
                         out=None) -> Quantized:
    """Rollout-side capture; ``guidance=False`` for layers whose guidance is
    not kept (codes/scales/s_t are then those of round-to-nearest)."""
    with _on(stream):
        x2 = _as_2d(x)
        d = Desc(fmt, x2.shape[0], x2.shape[1], seg_off)
        q = _outputs(d, x.device, guidance, out)
        _amax_in(amax_in, d, x.device)
        ws = workspace(d, x.device, stream)
        _check(lib().tf4_quantize_capture(d.ptr, _ptr(x2), _ptr(amax_in), _ptr(q.codes), _ptr(q.scales),
                                          _ptr(q.s_t), _ptr(q.bits if guidance else None), _ptr(ws), ws.numel(),
                                          _ptr(status_word(x.device, stream)), _stream(stream, x.device)),
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
    with _on(stream):
        L = len(xs)
        if L == 0:
            raise ValueError("tf4_quantize_capture_batched: no layers")
        x2 = [_as_2d(x) for x in xs]
        rows, cols = x2[0].shape
        dev = x2[0].device
        if any(t.shape != (rows, cols) or t.device != dev for t in x2):
            raise ValueError("tf4_quantize_capture_batched: layers must share one shape and one device")
        if not 0 <= keep <= L:
            raise ValueError(f"tf4_quantize_capture_batched: keep={keep} outside [0, {L}]")
        d = Desc(fmt, rows, cols)
        if out is not None:
            n = rows * cols
            _buf(out.codes, "out.codes", L * (n // 2), torch.uint8, dev)
            _buf(out.scales, "out.scales", L * (n // BLOCK[fmt]), torch.uint8, dev)
            if HAS_TENSOR_SCALE[fmt]:
                _buf(out.s_t, "out.s_t", L, torch.float32, dev)
            if keep:
                _buf(out.info_bits, "out.info_bits", keep * (n // 8), torch.uint8, dev)
        else:
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
                                                  _ptr(status_word(dev, stream)), _stream(stream, dev)),
               "tf4_quantize_capture_batched")
        return out


def tf4_quantize_guided(x, rec: Quantized, stream=None, out=None, rec_bits=None) -> torch.Tensor:
    """Train-side guided quantization of x against a rollout record."""
    with _on(stream):
        x2 = _as_2d(x)
        d = Desc(rec.fmt, x2.shape[0], x2.shape[1], rec.seg_off)
        bits = rec_bits if rec_bits is not None else rec.bits
        if bits is None:
            raise ValueError("tf4_quantize_guided: the record holds no guidance bits")
        _check_record(rec, d, x.device, "tf4_quantize_guided", bits=bits)
        codes = (_buf(out, "out", d.n // 2, torch.uint8, x.device) if out is not None
                 else torch.empty(d.n // 2, dtype=torch.uint8, device=x.device))
        _check(lib().tf4_quantize_guided(d.ptr, _ptr(x2), _ptr(rec.scales), _ptr(rec.s_t), _ptr(bits), _ptr(codes),
                                         _ptr(status_word(x.device, stream)), _stream(stream, x.device)),
               "tf4_quantize_guided")
        return codes


def tf4_guided_fake_quant(x, rec: Quantized, out_dtype=torch.float32, want_codes=False, stream=None,
                          out=None, codes=None, rec_bits=None):
    """Guided quantization + dequantization in one pass.  Returns (values,
    codes): values [rows, cols] in out_dtype (float32, or bfloat16 = RNE of
    the fp32 value); codes only if want_codes (else None)."""
    with _on(stream):
        if out_dtype not in (torch.float32, torch.bfloat16):
            raise TypeError(f"tf4_guided_fake_quant: out_dtype must be float32 or bfloat16, got {out_dtype}")
        x2 = _as_2d(x)
        d = Desc(rec.fmt, x2.shape[0], x2.shape[1], rec.seg_off)
        bits = rec_bits if rec_bits is not None else rec.bits
        if bits is None:
            raise ValueError("tf4_guided_fake_quant: the record holds no guidance bits")
        _check_record(rec, d, x.device, "tf4_guided_fake_quant", bits=bits)
        if out is not None:
            if not isinstance(out, torch.Tensor) or out.dtype not in (torch.float32, torch.bfloat16):
                raise TypeError("tf4_guided_fake_quant: out must be a float32 or bfloat16 tensor")
            o = _buf(out, "out", d.n, out.dtype, x.device)
        else:
            o = torch.empty(x2.shape, dtype=out_dtype, device=x.device)
        if codes is not None:
            c = _buf(codes, "codes", d.n // 2, torch.uint8, x.device)
        else:
            c = torch.empty(d.n // 2, dtype=torch.uint8, device=x.device) if want_codes else None
        _check(lib().tf4_guided_fake_quant(d.ptr, _ptr(x2), _ptr(rec.scales), _ptr(rec.s_t), _ptr(bits), _ptr(c),
                                           _ptr(o), 1 if o.dtype == torch.bfloat16 else 0,
                                           _ptr(status_word(x.device, stream)), _stream(stream, x.device)),
               "tf4_guided_fake_quant")
        return o, c


MISMATCH_COUNTS = 6


def tf4_mismatch_stats(x, rec: Quantized, counts=None, stream=None) -> torch.Tensor:
    """Mismatch diagnostics of train values x against a rollout record
    (codes + scales): adds [#mismatch, #adjacent, #far, #after-guidance,
    #toward-smaller, #toward-larger] to `counts` (int64 [6], zero-initialised
    if not given) and returns it."""
    with _on(stream):
        x2 = _as_2d(x)
        d = Desc(rec.fmt, x2.shape[0], x2.shape[1], rec.seg_off)
        _check_record(rec, d, x.device, "tf4_mismatch_stats", codes=True)
        c = (_buf(counts, "counts", MISMATCH_COUNTS, torch.int64, x.device) if counts is not None
             else torch.zeros(MISMATCH_COUNTS, dtype=torch.int64, device=x.device))
        _check(lib().tf4_mismatch_stats(d.ptr, _ptr(x2), _ptr(rec.scales), _ptr(rec.s_t), _ptr(rec.codes), _ptr(c),
                                        _ptr(status_word(x.device, stream)), _stream(stream, x.device)),
               "tf4_mismatch_stats")
        return c


def tf4_dequantize(q: Quantized, codes=None, stream=None, out=None) -> torch.Tensor:
    with _on(stream):
        d = Desc(q.fmt, q.rows, q.cols, q.seg_off)
        c = codes if codes is not None else q.codes
        if not isinstance(c, torch.Tensor) or not c.is_cuda:
            raise ValueError("tf4_dequantize: codes must be a CUDA tensor")
        _buf(c, "codes", d.n // 2, torch.uint8, c.device)
        _check_record(q, d, c.device, "tf4_dequantize")
        o = (_buf(out, "out", d.n, torch.float32, c.device) if out is not None
             else torch.empty((q.rows, q.cols), dtype=torch.float32, device=c.device))
        _check(lib().tf4_dequantize(d.ptr, _ptr(c), _ptr(q.scales), _ptr(q.s_t), _ptr(o), _stream(stream, c.device)),
               "tf4_dequantize")
        return o


def tf4_swizzle_scales(q: Quantized, stream=None, out=None) -> torch.Tensor:
    """The record's block scales in the tiled layout block-scaled FP4 GEMMs
    read (uint8 [ceil(rows/128)*128, ceil(nb/4)*4] as laid out in memory)."""
    with _on(stream):
        d = Desc(q.fmt, q.rows, q.cols, q.seg_off)
        nb = q.cols // BLOCK[q.fmt]
        shape = ((q.rows + 127) // 128 * 128, (nb + 3) // 4 * 4)
        if not isinstance(q.scales, torch.Tensor) or not q.scales.is_cuda:
            raise ValueError("tf4_swizzle_scales: the record's scales must be a CUDA tensor")
        dev = q.scales.device
        _buf(q.scales, "record scales", q.rows * nb, torch.uint8, dev)
        o = (_buf(out, "out", shape[0] * shape[1], torch.uint8, dev) if out is not None
             else torch.empty(shape, dtype=torch.uint8, device=dev))
        _check(lib().tf4_swizzle_scales(d.ptr, _ptr(q.scales), _ptr(o), _stream(stream, q.scales.device)),
               "tf4_swizzle_scales")
        return o


def tf4_pack_guidance(codes: torch.Tensor, rows: int, cols: int, fmt=NVFP4, stream=None, out=None):
    with _on(stream):
        d = Desc(fmt, rows, cols)
        if not isinstance(codes, torch.Tensor) or not codes.is_cuda:
            raise ValueError("tf4_pack_guidance: codes must be a CUDA tensor")
        _buf(codes, "codes", d.n // 2, torch.uint8, codes.device)
        o = (_buf(out, "out", d.n // 8, torch.uint8, codes.device) if out is not None
             else torch.empty(d.n // 8, dtype=torch.uint8, device=codes.device))
        _check(lib().tf4_pack_guidance(d.ptr, _ptr(codes), _ptr(o), _stream(stream, codes.device)),
               "tf4_pack_guidance")
        return o


def tf4_unpack_guidance(bits: torch.Tensor, rows: int, cols: int, fmt=NVFP4, stream=None, out=None):
    with _on(stream):
        d = Desc(fmt, rows, cols)
        if not isinstance(bits, torch.Tensor) or not bits.is_cuda:
            raise ValueError("tf4_unpack_guidance: bits must be a CUDA tensor")
        _buf(bits, "bits", d.n // 8, torch.uint8, bits.device)
        o = (_buf(out, "out", d.n, torch.uint8, bits.device) if out is not None
             else torch.empty(d.n, dtype=torch.uint8, device=bits.device))
        _check(lib().tf4_unpack_guidance(d.ptr, _ptr(bits), _ptr(o), _stream(stream, bits.device)),
               "tf4_unpack_guidance")
        return o


def capture_layers(num_layers: int, keep: int) -> list:
    """Layer indices whose guidance is kept: the deepest `keep` of
    `num_layers` (the highest indices)."""
    keep = max(0, min(keep, num_layers))
    return list(range(num_layers - keep, num_layers))
