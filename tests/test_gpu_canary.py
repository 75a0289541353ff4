"""Out-of-bounds write detection without a sanitizer: every output buffer of
every call sits between two 64 KiB guard bands of 0xA5 bytes, and after the
call both bands must be intact.  Shapes are the odd ones: a single row,
one or two blocks per row, ragged block counts, empty segments and a last
segment of one row.  (Values are checked against the oracle elsewhere.)"""
import pytest
import torch

from fp4_block_scaled_quantizer_b200 import binding as B
from fp4_block_scaled_quantizer_b200 import build as libbuild
from fp4_block_scaled_quantizer_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"
GUARD = 64 << 10
CANARY = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    libbuild.build()
    B.lib()


class Guarded:
    """Byte buffers with guard bands; views of the requested sizes."""

    def __init__(self):
        self.bufs = []

    def __call__(self, shape, dtype):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        buf = torch.full((GUARD + nbytes + GUARD,), CANARY, dtype=torch.uint8, device=DEV)
        self.bufs.append((buf, nbytes))
        return buf[GUARD:GUARD + nbytes].view(dtype).view(shape)

    def check(self, what):
        torch.cuda.synchronize()
        for buf, nbytes in self.bufs:
            lo, hi = buf[:GUARD], buf[GUARD + nbytes:]
            assert bool((lo == CANARY).all()), f"{what}: write before a buffer of {nbytes} bytes"
            assert bool((hi == CANARY).all()), f"{what}: write past a buffer of {nbytes} bytes"


def record(g, fmt, rows, cols, nseg, bits=True):
    blk = B.BLOCK[fmt]
    return B.Quantized(g((rows * cols // 2,), torch.uint8), g((rows, cols // blk), torch.uint8),
                       g((nseg,), torch.float32) if B.HAS_TENSOR_SCALE[fmt] else None,
                       g((rows * cols // 8,), torch.uint8) if bits else None, fmt, rows, cols, None)


CASES = [
    (B.NVFP4, 1, 16, None), (B.NVFP4, 3, 48, [0, 0, 2, 3]), (B.NVFP4, 129, 80, [0, 64, 64, 128, 129]),
    (B.MXFP4, 1, 32, None), (B.MXFP4, 5, 96, None), (B.UFP4, 2, 16, None), (B.UFP4, 37, 144, [0, 36, 37]),
]


@pytest.mark.parametrize("fmt,rows,cols,seg", CASES)
def test_outputs_stay_inside_their_buffers(fmt, rows, cols, seg):
    x = W.random_bf16((rows, cols), seed=rows + cols, device=DEV, outlier_frac=0.05)
    xt = W.perturb(x, 3, rel=0.05)
    nseg = 1 if seg is None else len(seg) - 1
    g = Guarded()
    q = record(g, fmt, rows, cols, nseg)
    q.seg_off = seg
    B.tf4_quantize_capture(x, fmt=fmt, seg_off=seg, out=q)
    B.tf4_quantize_rtn(x, fmt=fmt, seg_off=seg, out=record(g, fmt, rows, cols, nseg, bits=False))
    B.tf4_quantize_sr(x, 7, fmt=fmt, seg_off=seg, out=record(g, fmt, rows, cols, nseg, bits=False))
    if B.HAS_TENSOR_SCALE[fmt]:
        B.tf4_segment_amax(x, seg, out=g((nseg,), torch.float32))
    B.tf4_quantize_guided(xt, q, out=g((rows * cols // 2,), torch.uint8))
    B.tf4_dequantize(q, out=g((rows, cols), torch.float32))
    f32_16 = g((rows * cols + 4,), torch.float32)[4:].view(rows, cols)  # 16-B but not 32-B aligned
    B.tf4_dequantize(q, out=f32_16)
    B.tf4_guided_fake_quant(xt, q, out=g((rows, cols), torch.float32), codes=g((rows * cols // 2,), torch.uint8))
    B.tf4_guided_fake_quant(xt, q, out=g((rows, cols), torch.bfloat16))
    B.tf4_guided_fake_quant(xt, q, out=f32_16)
    B.tf4_mismatch_stats(xt, q, counts=g((B.MISMATCH_COUNTS,), torch.int64).zero_())
    B.tf4_pack_guidance(q.codes, rows, cols, fmt, out=g((rows * cols // 8,), torch.uint8))
    B.tf4_unpack_guidance(q.bits, rows, cols, fmt, out=g((rows * cols,), torch.uint8))
    nb = cols // B.BLOCK[fmt]
    B.tf4_swizzle_scales(q, out=g(((rows + 127) // 128 * 128, (nb + 3) // 4 * 4), torch.uint8))
    assert B.read_status(x.device) == 0
    g.check(f"fmt {fmt} {rows}x{cols}")


@pytest.mark.parametrize("fmt", [B.NVFP4, B.MXFP4, B.UFP4])
def test_batched_capture_outputs_stay_inside(fmt):
    rows, cols, L, keep = 5, 16 * B.BLOCK[fmt] // 16 * 3, 3, 2
    xs = [W.random_bf16((rows, cols), seed=40 + i, device=DEV) for i in range(L)]
    g = Guarded()
    n = rows * cols
    out = B.BatchedCapture(g((L, n // 2), torch.uint8), g((L, rows, cols // B.BLOCK[fmt]), torch.uint8),
                           g((L,), torch.float32) if B.HAS_TENSOR_SCALE[fmt] else None,
                           g((keep, n // 8), torch.uint8), fmt, rows, cols, keep)
    B.tf4_quantize_capture_batched(xs, fmt=fmt, keep=keep, out=out)
    assert B.read_status(xs[0].device) == 0
    g.check(f"batched fmt {fmt}")


def test_short_or_mistyped_buffers_are_refused_before_launch():
    """Buffers the library would overrun (or misread) are refused by the
    binding with nothing launched: the caller's buffer keeps its bytes."""
    rows, cols = 64, 256
    n = rows * cols
    x = W.random_bf16((rows, cols), seed=5, device=DEV)
    q = B.tf4_quantize_capture(x)
    short = torch.full((n // 2 - 1,), CANARY, dtype=torch.uint8, device=DEV)
    with pytest.raises(ValueError):
        B.tf4_quantize_guided(x, q, out=short)
    with pytest.raises(ValueError):
        B.tf4_quantize_guided(W.random_bf16((2 * rows, cols), seed=6, device=DEV), q)  # record too small
    with pytest.raises(ValueError):
        B.tf4_pack_guidance(q.codes, rows, cols, out=short[: n // 8 - 1])
    with pytest.raises(ValueError):
        B.tf4_unpack_guidance(q.bits, rows, cols, out=short)  # needs n bytes
    bad = B.Quantized(torch.empty(n // 2, dtype=torch.uint8, device=DEV), torch.empty(10, dtype=torch.uint8, device=DEV),
                      torch.empty(1, dtype=torch.float32, device=DEV), torch.empty(n // 8, dtype=torch.uint8, device=DEV))
    with pytest.raises(ValueError):
        B.tf4_quantize_capture(x, out=bad)
    with pytest.raises(ValueError):
        B.tf4_quantize_rtn(x, seg_off=[0, 32, 64], amax_in=torch.ones(1, device=DEV))
    with pytest.raises(TypeError):
        B.tf4_dequantize(q, out=torch.empty((rows, cols), dtype=torch.float16, device=DEV))
    with pytest.raises(TypeError):
        B.tf4_mismatch_stats(x, q, counts=torch.zeros(B.MISMATCH_COUNTS, dtype=torch.int32, device=DEV))
    with pytest.raises(ValueError):  # the four counts of library version 1 are too few
        B.tf4_mismatch_stats(x, q, counts=torch.zeros(4, dtype=torch.int64, device=DEV))
    with pytest.raises(TypeError):
        B.tf4_guided_fake_quant(x, q, out=torch.empty((rows, cols), dtype=torch.float16, device=DEV))
    torch.cuda.synchronize()
    assert bool((short == CANARY).all())
    assert B.read_status(x.device) == 0
