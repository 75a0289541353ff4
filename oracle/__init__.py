"""CPU oracle for block-scaled FP4 quantization -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and the cpu_baseline / reference
leg of ``bench.py`` may import this package.  The product path (the CUDA
library and its Python binding) never imports or calls it.

This module is a ctypes + numpy wrapper over ``tf4_oracle.c``; every
definition (and the page it follows) is documented there.  Inputs are bf16
bit patterns as ``np.uint16`` arrays of shape [rows, cols].
"""
import ctypes
import os

import numpy as np

from . import build as _build

NVFP4, MXFP4, UFP4 = 0, 1, 2
RTN, SR = 0, 1
NONFINITE = 1
BLOCK = {NVFP4: 16, MXFP4: 32, UFP4: 16}
HAS_TENSOR_SCALE = {NVFP4: True, MXFP4: False, UFP4: True}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u8p, u16p, f32p, i64p, u32p = (
            ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(ctypes.c_uint16),
            ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int64),
            ctypes.POINTER(ctypes.c_uint32),
        )
        i64, i32, u64, d = ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64, ctypes.c_double
        sig = {
            "orc_bf16_to_float": (ctypes.c_float, [ctypes.c_uint16]),
            "orc_e2m1_value": (d, [ctypes.c_int]),
            "orc_grid_value": (d, [ctypes.c_int, ctypes.c_int]),
            "orc_e4m3_value": (d, [ctypes.c_uint8]),
            "orc_e4m3_encode": (ctypes.c_uint8, [ctypes.c_float]),
            "orc_e8m0_exponent": (ctypes.c_int, [ctypes.c_float]),
            "orc_tensor_scale": (ctypes.c_float, [ctypes.c_int, ctypes.c_float]),
            "orc_nvfp4_tensor_scale": (ctypes.c_float, [ctypes.c_float]),
            "orc_block_scale_code": (ctypes.c_uint8, [ctypes.c_int, ctypes.c_float, ctypes.c_float]),
            "orc_nvfp4_block_scale_code": (ctypes.c_uint8, [ctypes.c_float, ctypes.c_float]),
            "orc_nvfp4_block_scale": (ctypes.c_float, [ctypes.c_uint8, ctypes.c_float]),
            "orc_mxfp4_block_scale": (ctypes.c_float, [ctypes.c_uint8]),
            "orc_rtn_m3": (ctypes.c_int, [d, d]),
            "orc_sr_m3": (ctypes.c_int, [d, d, ctypes.c_uint32]),
            "orc_guided_m3": (ctypes.c_int, [d, d, ctypes.c_int]),
            "orc_rtn_code": (ctypes.c_int, [ctypes.c_int, d, d]),
            "orc_sr_code": (ctypes.c_int, [ctypes.c_int, d, d, ctypes.c_uint32]),
            "orc_guided_code": (ctypes.c_int, [ctypes.c_int, d, d, ctypes.c_int]),
            "orc_philox4x32_10": (None, [u32p, u32p, u32p]),
            "orc_sr_uniform24": (ctypes.c_uint32, [u64, u64]),
            "orc_segment_amax": (ctypes.c_int, [u16p, i64, i64, i32, i64p, f32p]),
            "orc_segment_scales": (ctypes.c_int, [ctypes.c_int, u16p, i64, i64, i32, i64p, f32p]),
            "orc_quantize_rows": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, u16p, i64, i64, i32, i64p,
                                                 f32p, u64, i64, i64, u8p, u8p, u8p]),
            "orc_quantize_guided_rows": (ctypes.c_int, [ctypes.c_int, u16p, i64, i64, i32, i64p, u8p,
                                                        f32p, u8p, i64, i64, u8p]),
            "orc_dequantize_rows": (None, [ctypes.c_int, u8p, u8p, f32p, i64, i64, i32, i64p, i64, i64,
                                           f32p]),
            "orc_pack_guidance": (None, [u8p, i64, u8p]),
            "orc_unpack_guidance": (None, [u8p, i64, u8p]),
            "orc_rtn_with_scales_rows": (None, [ctypes.c_int, u16p, i64, i64, i32, i64p, u8p, f32p, i64, i64,
                                                u8p]),
            "orc_swizzle_scales": (None, [u8p, i64, i64, u8p]),
            "orc_f32_to_bf16": (ctypes.c_uint16, [ctypes.c_float]),
            "orc_f32_to_bf16_array": (None, [f32p, i64, u16p]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a, ctype):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _seg(seg_off, rows):
    if seg_off is None:
        return 1, None
    so = np.ascontiguousarray(np.asarray(seg_off, dtype=np.int64))
    assert so[0] == 0 and so[-1] == rows and np.all(np.diff(so) >= 0)
    return len(so) - 1, so


# ----------------------------------------------------------------- scalars
def e4m3_encode(r: float) -> int:
    return int(lib().orc_e4m3_encode(float(r)))


def e4m3_value(code: int) -> float:
    return float(lib().orc_e4m3_value(int(code)))


def e8m0_exponent(bamax: float) -> int:
    return int(lib().orc_e8m0_exponent(float(bamax)))


def nvfp4_tensor_scale(amax: float) -> float:
    return float(lib().orc_nvfp4_tensor_scale(float(amax)))


def tensor_scale(fmt: int, amax: float) -> float:
    return float(lib().orc_tensor_scale(int(fmt), float(amax)))


def block_scale_code(fmt: int, bamax: float, s_t: float) -> int:
    return int(lib().orc_block_scale_code(int(fmt), float(bamax), float(s_t)))


def grid_value(fmt: int, m3: int) -> float:
    return float(lib().orc_grid_value(int(fmt), int(m3)))


def rtn_code(fmt: int, ax: float, S: float) -> int:
    return int(lib().orc_rtn_code(int(fmt), float(ax), float(S)))


def sr_code(fmt: int, ax: float, S: float, r24: int) -> int:
    return int(lib().orc_sr_code(int(fmt), float(ax), float(S), int(r24)))


def guided_code(fmt: int, ax: float, S: float, g: int) -> int:
    return int(lib().orc_guided_code(int(fmt), float(ax), float(S), int(g)))


def rtn_m3(ax: float, S: float) -> int:
    return int(lib().orc_rtn_m3(float(ax), float(S)))


def sr_m3(ax: float, S: float, r24: int) -> int:
    return int(lib().orc_sr_m3(float(ax), float(S), int(r24)))


def guided_m3(ax: float, S: float, g: int) -> int:
    return int(lib().orc_guided_m3(float(ax), float(S), int(g)))


def philox4x32_10(ctr, key):
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_p(c, ctypes.c_uint32), _p(k, ctypes.c_uint32), _p(out, ctypes.c_uint32))
    return out


def sr_uniform24(idx: int, seed: int) -> int:
    return int(lib().orc_sr_uniform24(int(idx), int(seed)))


# ------------------------------------------------------------------ tensors
def segment_amax(x, seg_off=None):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows, cols = x.shape
    nseg, so = _seg(seg_off, rows)
    out = np.zeros(nseg, dtype=np.float32)
    st = lib().orc_segment_amax(_p(x, ctypes.c_uint16), rows, cols, nseg, _p(so, ctypes.c_int64),
                                _p(out, ctypes.c_float))
    return out, st


def segment_scales(x, seg_off=None, fmt=NVFP4):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows, cols = x.shape
    nseg, so = _seg(seg_off, rows)
    out = np.zeros(nseg, dtype=np.float32)
    st = lib().orc_segment_scales(int(fmt), _p(x, ctypes.c_uint16), rows, cols, nseg, _p(so, ctypes.c_int64),
                                  _p(out, ctypes.c_float))
    return out, st


def quantize(x, fmt=NVFP4, mode=RTN, seg_off=None, seed=0, bits=False, s_t=None, row_range=None):
    """Returns dict(codes, scales, s_t, bits, status).  ``s_t`` may be given
    (NVFP4 / UFP4) to quantize a row range of a larger tensor without a full
    pass."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows, cols = x.shape
    blk = BLOCK[fmt]
    assert cols % blk == 0
    nseg, so = _seg(seg_off, rows)
    status = 0
    if HAS_TENSOR_SCALE[fmt]:
        if s_t is None:
            s_t, status = segment_scales(x, seg_off, fmt)
        s_t = np.ascontiguousarray(s_t, dtype=np.float32)
    else:
        s_t = None
    rb, re = (0, rows) if row_range is None else row_range
    codes = np.zeros(rows * cols // 2, dtype=np.uint8)
    scales = np.zeros(rows * cols // blk, dtype=np.uint8)
    gb = np.zeros((rows * cols + 7) // 8, dtype=np.uint8) if bits else None
    status |= lib().orc_quantize_rows(fmt, mode, _p(x, ctypes.c_uint16), rows, cols, nseg,
                                      _p(so, ctypes.c_int64), _p(s_t, ctypes.c_float), seed, rb, re,
                                      _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8),
                                      _p(gb, ctypes.c_uint8))
    return dict(codes=codes, scales=scales, s_t=s_t, bits=gb, status=status)


def quantize_guided(x, rec_scales, rec_bits, fmt=NVFP4, rec_s_t=None, seg_off=None, row_range=None):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows, cols = x.shape
    nseg, so = _seg(seg_off, rows)
    rs = np.ascontiguousarray(rec_scales, dtype=np.uint8)
    rbits = np.ascontiguousarray(rec_bits, dtype=np.uint8)
    st = None if rec_s_t is None else np.ascontiguousarray(rec_s_t, dtype=np.float32)
    rb, re = (0, rows) if row_range is None else row_range
    codes = np.zeros(rows * cols // 2, dtype=np.uint8)
    status = lib().orc_quantize_guided_rows(fmt, _p(x, ctypes.c_uint16), rows, cols, nseg,
                                            _p(so, ctypes.c_int64), _p(rs, ctypes.c_uint8),
                                            _p(st, ctypes.c_float), _p(rbits, ctypes.c_uint8), rb, re,
                                            _p(codes, ctypes.c_uint8))
    return codes, status


def dequantize(codes, scales, rows, cols, fmt=NVFP4, s_t=None, seg_off=None, row_range=None):
    nseg, so = _seg(seg_off, rows)
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    st = None if s_t is None else np.ascontiguousarray(s_t, dtype=np.float32)
    rb, re = (0, rows) if row_range is None else row_range
    out = np.zeros(rows * cols, dtype=np.float32)
    lib().orc_dequantize_rows(fmt, _p(c, ctypes.c_uint8), _p(s, ctypes.c_uint8), _p(st, ctypes.c_float),
                              rows, cols, nseg, _p(so, ctypes.c_int64), rb, re, _p(out, ctypes.c_float))
    return out.reshape(rows, cols)


def pack_guidance(codes, n):
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.zeros((n + 7) // 8, dtype=np.uint8)
    lib().orc_pack_guidance(_p(c, ctypes.c_uint8), n, _p(out, ctypes.c_uint8))
    return out


def unpack_guidance(bits, n):
    b = np.ascontiguousarray(bits, dtype=np.uint8)
    out = np.zeros(n, dtype=np.uint8)
    lib().orc_unpack_guidance(_p(b, ctypes.c_uint8), n, _p(out, ctypes.c_uint8))
    return out


def unpack_codes(codes, n):
    """Nibble array (one uint8 per element) from packed codes (layout helper)."""
    c = np.asarray(codes, dtype=np.uint8)
    out = np.empty(2 * len(c), dtype=np.uint8)
    out[0::2] = c & 0xF
    out[1::2] = c >> 4
    return out[:n]


def swizzle_scales(scales2d):
    """The [rows, nb] scale bytes in the 128 x 4 tiled layout of block-scaled
    GEMMs (flat uint8 array, zero-padded)."""
    sc = np.ascontiguousarray(scales2d, dtype=np.uint8)
    rows, nb = sc.shape
    out = np.zeros(((rows + 127) // 128 * 128) * ((nb + 3) // 4 * 4), dtype=np.uint8)
    lib().orc_swizzle_scales(_p(sc, ctypes.c_uint8), rows, nb, _p(out, ctypes.c_uint8))
    return out


def f32_to_bf16(v):
    """bf16 bit patterns (RNE) of an fp32 array."""
    a = np.ascontiguousarray(v, dtype=np.float32).reshape(-1)
    out = np.zeros(a.size, dtype=np.uint16)
    lib().orc_f32_to_bf16_array(_p(a, ctypes.c_float), a.size, _p(out, ctypes.c_uint16))
    return out.reshape(np.shape(v))


def guided_fake_quant(x, rec_scales, rec_bits, fmt=NVFP4, rec_s_t=None, seg_off=None):
    """Train-side fake quantization: guided codes, then their fp32 values."""
    rows, cols = np.shape(x)
    codes, status = quantize_guided(x, rec_scales, rec_bits, fmt, rec_s_t=rec_s_t, seg_off=seg_off)
    return codes, dequantize(codes, rec_scales, rows, cols, fmt, s_t=rec_s_t, seg_off=seg_off), status


def rtn_with_scales(x, scales, fmt=NVFP4, s_t=None, seg_off=None):
    """Nearest rounding of x on a given (recorded) grid of scales."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows, cols = x.shape
    nseg, so = _seg(seg_off, rows)
    sc = np.ascontiguousarray(scales, dtype=np.uint8)
    st = None if s_t is None else np.ascontiguousarray(s_t, dtype=np.float32)
    codes = np.zeros(rows * cols // 2, dtype=np.uint8)
    lib().orc_rtn_with_scales_rows(fmt, _p(x, ctypes.c_uint16), rows, cols, nseg, _p(so, ctypes.c_int64),
                                   _p(sc, ctypes.c_uint8), _p(st, ctypes.c_float), 0, rows,
                                   _p(codes, ctypes.c_uint8))
    return codes


def grid_index(codes, n):
    """Signed grid index of each code (sign ? -m3 : m3)."""
    nib = unpack_codes(codes, n).astype(np.int64)
    m = nib & 7
    return np.where(nib & 8, -m, m)


def mismatch_stats(x, rec_scales, rec_codes, fmt=NVFP4, rec_s_t=None, seg_off=None):
    """[#(n_r != n_o), #(|n_r - n_o| == 1), #(|n_r - n_o| >= 2), #(n_g != n_o),
    #(n_r != n_o, |n_o| < |n_r|), #(n_r != n_o, |n_o| > |n_r|)] with n_r the
    train value's nearest rounding on the recorded grid, n_o the rollout
    code, n_g the guided code, |.| the codeword magnitude: the last two split
    the corrections guidance makes by direction, toward the smaller or the
    larger codeword (TRACE summary, section 量子化情報キャッシュ)."""
    rows, cols = np.shape(x)
    n = rows * cols
    nr = rtn_with_scales(x, rec_scales, fmt, rec_s_t, seg_off)
    bits = pack_guidance(rec_codes, n)
    ng, _ = quantize_guided(x, rec_scales, bits, fmt, rec_s_t=rec_s_t, seg_off=seg_off)
    io, ir, ig = grid_index(rec_codes, n), grid_index(nr, n), grid_index(ng, n)
    d = np.abs(ir - io)
    smaller = (d != 0) & (np.abs(io) < np.abs(ir))
    larger = (d != 0) & (np.abs(io) > np.abs(ir))
    return np.array([(d != 0).sum(), (d == 1).sum(), (d >= 2).sum(), (ig != io).sum(), smaller.sum(),
                     larger.sum()], dtype=np.int64)
