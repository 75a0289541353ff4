"""The bounds-checking build (TF4_DEBUG_BOUNDS, libtrace_fp4_debug.so):
every call on odd shapes (one row, one or two blocks, ragged block counts,
empty segments, a last segment of one row) and on a multi-wave layer gives
the release build's bytes, and its kernels count no work unit outside the
range a CTA owns or the buffers' extent."""
import pytest
import torch

from fp4_block_scaled_quantizer_b200 import binding as B
from fp4_block_scaled_quantizer_b200 import build as libbuild
from fp4_block_scaled_quantizer_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    libbuild.build()
    libbuild.build(debug_bounds=True)
    B.lib()


def run_all(fmt, rows, cols, seg):
    """Every call of the library on one input; returns the outputs."""
    x = W.random_bf16((rows, cols), seed=rows * 7 + cols, device=DEV, outlier_frac=0.05)
    xt = W.perturb(x, 3, rel=0.05)
    out = {}
    q = B.tf4_quantize_capture(x, fmt=fmt, seg_off=seg)
    out.update(codes=q.codes, scales=q.scales, bits=q.bits)
    if q.s_t is not None:
        out["s_t"] = q.s_t
    out["rtn"] = B.tf4_quantize_rtn(x, fmt=fmt, seg_off=seg).codes
    out["sr"] = B.tf4_quantize_sr(x, 11, fmt=fmt, seg_off=seg).codes
    if B.HAS_TENSOR_SCALE[fmt]:
        out["amax"] = B.tf4_segment_amax(x, seg)
    out["guided"] = B.tf4_quantize_guided(xt, q)
    out["dequant"] = B.tf4_dequantize(q)
    f16 = torch.empty(rows * cols + 4, dtype=torch.float32, device=DEV)[4:].view(rows, cols)
    out["dequant16"] = B.tf4_dequantize(q, out=f16).clone()
    out["fq32"], out["fq_codes"] = B.tf4_guided_fake_quant(xt, q, want_codes=True)
    out["fq16"] = B.tf4_guided_fake_quant(xt, q, out_dtype=torch.bfloat16)[0]
    out["mismatch"] = B.tf4_mismatch_stats(xt, q)
    out["pack"] = B.tf4_pack_guidance(q.codes, rows, cols, fmt)
    out["unpack"] = B.tf4_unpack_guidance(q.bits, rows, cols, fmt)
    out["swizzle"] = B.tf4_swizzle_scales(q)
    assert B.read_status(x.device) == 0
    return out


CASES = [
    (B.NVFP4, 1, 16, None), (B.NVFP4, 3, 48, [0, 0, 2, 3]), (B.NVFP4, 129, 80, [0, 64, 64, 128, 129]),
    (B.MXFP4, 1, 32, None), (B.MXFP4, 5, 96, None), (B.UFP4, 2, 16, None), (B.UFP4, 37, 144, [0, 36, 37]),
    (B.NVFP4, 4096, 2048, None), (B.MXFP4, 2048, 4096, None), (B.UFP4, 3000, 512, [0, 1000, 1000, 2999, 3000]),
]


@pytest.mark.parametrize("fmt,rows,cols,seg", CASES)
def test_debug_build_matches_release_with_no_violations(fmt, rows, cols, seg):
    want = run_all(fmt, rows, cols, seg)
    with B.use_library(B.DEBUG_LIB_PATH) as L:
        assert L.tf4_debug_bounds_enabled() == 1
        B.debug_bounds_violations()  # reset
        got = run_all(fmt, rows, cols, seg)
        assert B.debug_bounds_violations() == 0
    for k, v in want.items():
        assert torch.equal(got[k], v), k
    assert B.lib().tf4_debug_bounds_enabled() == 0


@pytest.mark.parametrize("fmt", [B.NVFP4, B.MXFP4])
def test_debug_build_batched_capture(fmt):
    xs = [W.random_bf16((33, 3 * B.BLOCK[fmt] * 4), seed=90 + i, device=DEV) for i in range(5)]
    want = B.tf4_quantize_capture_batched(xs, fmt=fmt, keep=2)
    with B.use_library(B.DEBUG_LIB_PATH):
        B.debug_bounds_violations()
        got = B.tf4_quantize_capture_batched(xs, fmt=fmt, keep=2)
        assert B.debug_bounds_violations() == 0
    for k in ("codes", "scales", "s_t", "info_bits"):
        if getattr(want, k) is not None:
            assert torch.equal(getattr(got, k), getattr(want, k)), k
