"""Every row of the full-size workloads against the oracle.

The sampled checks in test_gpu_parity.py compare a few dozen rows of each
full-size workload; these compare every element: one 65536 x 4096 layer of
the activation stack through exactly the calls the benchmark times (amax
pass, capture with the amax given, guided quantization of the perturbed
train copy the benchmark draws), plus dequantization, the fused fake-quant
and the mismatch counts; the 128-expert MoE dispatch; one K tensor of the KV
cache.  The oracle runs on row ranges spread over the host's cores (spawned
processes), with the tensor scales of its own full amax pass.
"""
import numpy as np
import pytest
import torch

import oracle as O
from fp4_block_scaled_quantizer_b200 import binding as B
from fp4_block_scaled_quantizer_b200 import build as libbuild
from fp4_block_scaled_quantizer_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"
CHUNKS = 128


@pytest.fixture(scope="module")
def pool():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from oracle.pool import OraclePool

    p = OraclePool()  # spawned workers: safe although this process uses the GPU
    libbuild.build()
    B.lib()
    O.lib()
    yield p
    p.close()


def host(t):
    return t.detach().cpu().numpy()


def f32_bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def assert_same(name, got, want):
    got, want = np.asarray(got).reshape(-1), np.asarray(want).reshape(-1)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{name}: {bad.size} mismatches, first at {bad[:8]}: got {got[bad[:8]]} want {want[bad[:8]]}"


def row_ranges(rows, seg=None):
    """About CHUNKS row ranges covering [0, rows), with the segment offsets
    of each made relative to it."""
    step = max(1, -(-rows // CHUNKS))
    out = []
    for a in range(0, rows, step):
        b = min(rows, a + step)
        rel = None if seg is None else [int(min(max(v - a, 0), b - a)) for v in seg]
        out.append((a, b, rel))
    return out


def oracle_full(pool, fmt, xs, xts, seg=None):
    """The oracle's capture of xs (all rows), guided quantization of xts
    against that record, dequantization, fused fake-quant values and the
    mismatch counts -- computed range by range on the pool."""
    rows, cols = xs.shape
    blk, n = O.BLOCK[fmt], rows * cols
    s_t = None
    if O.HAS_TENSOR_SCALE[fmt]:
        s_t, st = O.segment_scales(xs, seg, fmt)
        assert st == 0
    rr = row_ranges(rows, seg)
    cap = pool.map_rows("capture", [dict(fmt=fmt, seg=g, s_t=s_t, x=xs[a:b]) for a, b, g in rr])
    assert all(c[3] == 0 for c in cap)
    codes = np.concatenate([c[0] for c in cap])
    scales = np.concatenate([c[1] for c in cap])
    bits = np.concatenate([c[2] for c in cap])
    assert codes.size == n // 2 and scales.size == n // blk and bits.size == n // 8

    def cut(a, b):
        return dict(codes=codes[a * cols // 2:b * cols // 2], scales=scales[a * cols // blk:b * cols // blk],
                    bits=bits[a * cols // 8:b * cols // 8])

    gd = pool.map_rows("guided", [dict(fmt=fmt, seg=g, s_t=s_t, x=xts[a:b], scales=cut(a, b)["scales"],
                                       bits=cut(a, b)["bits"]) for a, b, g in rr])
    assert all(st == 0 for _, st in gd)
    guided = np.concatenate([c for c, _ in gd])
    dq = pool.map_rows("dequant", [dict(fmt=fmt, seg=g, s_t=s_t, shape=(b - a, cols), codes=cut(a, b)["codes"],
                                        scales=cut(a, b)["scales"]) for a, b, g in rr])
    fq = pool.map_rows("dequant", [dict(fmt=fmt, seg=g, s_t=s_t, shape=(b - a, cols),
                                        codes=guided[a * cols // 2:b * cols // 2], scales=cut(a, b)["scales"])
                                   for a, b, g in rr])
    mm = pool.map_rows("mismatch", [dict(fmt=fmt, seg=g, s_t=s_t, x=xts[a:b], scales=cut(a, b)["scales"],
                                         codes=cut(a, b)["codes"]) for a, b, g in rr])
    return dict(codes=codes, scales=scales, bits=bits, s_t=s_t, guided=guided,
                dequant=np.concatenate([d.reshape(-1) for d in dq]),
                fq=np.concatenate([d.reshape(-1) for d in fq]), counts=np.sum(mm, axis=0))


def check_all(pool, fmt, x, xt, seg=None, bench_path=False):
    """Library vs oracle on every element of x (capture) and xt (guided,
    fused fake-quant, diagnostics), and the dequantized record."""
    if bench_path:  # the benchmark's calls: amax pass, then capture with the amax given
        amax = B.tf4_segment_amax(x, seg)
        q = B.tf4_quantize_capture(x, fmt=fmt, seg_off=seg, amax_in=amax)
        q_self = B.tf4_quantize_capture(x, fmt=fmt, seg_off=seg)
        for name in ("codes", "scales", "s_t", "bits"):
            assert torch.equal(getattr(q, name), getattr(q_self, name)), name
        del q_self
    else:
        q = B.tf4_quantize_capture(x, fmt=fmt, seg_off=seg)
    g = B.tf4_quantize_guided(xt, q)
    d = B.tf4_dequantize(q)
    y, c = B.tf4_guided_fake_quant(xt, q, want_codes=True)
    yb, _ = B.tf4_guided_fake_quant(xt, q, out_dtype=torch.bfloat16)
    cnt = B.tf4_mismatch_stats(xt, q)
    assert B.read_status(x.device) == 0
    torch.cuda.synchronize()
    xs, xts = W.bf16_bits(x), W.bf16_bits(xt)
    want = oracle_full(pool, fmt, xs, xts, seg)
    assert_same("codes", host(q.codes), want["codes"])
    assert_same("scales", host(q.scales), want["scales"])
    assert_same("bits", host(q.bits), want["bits"])
    if O.HAS_TENSOR_SCALE[fmt]:
        assert_same("s_t", f32_bits(host(q.s_t)), f32_bits(want["s_t"]))
    assert_same("guided", host(g), want["guided"])
    assert_same("fake-quant codes", host(c), want["guided"])
    del g, c
    assert_same("dequant", f32_bits(host(d)), f32_bits(want["dequant"]))
    del d
    assert_same("fake-quant fp32", f32_bits(host(y)), f32_bits(want["fq"]))
    del y
    assert_same("fake-quant bf16", host(yb.view(torch.int16)).view(np.uint16), O.f32_to_bf16(want["fq"]))
    assert host(cnt).tolist() == want["counts"].tolist()
    return want["counts"]


@pytest.mark.parametrize("fmt", [O.NVFP4, O.UFP4, O.MXFP4])
def test_layer_stack_deep_layer_every_row(pool, fmt):
    """Layer 39 and the benchmark's own train copy of it (seed 1000 + layer,
    relative perturbation 1e-3)."""
    x = W.layer_stack_layer(39, DEV)
    xt = W.perturb(x, 1039)
    check_all(pool, fmt, x, xt, bench_path=O.HAS_TENSOR_SCALE[fmt])


@pytest.mark.parametrize("fmt", [O.NVFP4, O.UFP4, O.MXFP4])
def test_layer_stack_layer_every_row_at_5_percent_mismatch(pool, fmt):
    """A train copy 5% away (relative) from the rollout's values: about 5% of
    the train values round to another codeword than the rollout's, the case
    guided rounding exists for."""
    x = W.layer_stack_layer(20, DEV)
    xt = W.perturb(x, 1020, rel=5e-2)
    counts = check_all(pool, fmt, x, xt)
    assert counts[0] > 0.02 * x.numel()


@pytest.mark.parametrize("fmt", [O.NVFP4, O.UFP4])
def test_moe_dispatch_every_row(pool, fmt):
    w = W.moe_dispatch(DEV)
    check_all(pool, fmt, w["x"], w["x_train"], seg=w["seg_off"].tolist())


@pytest.mark.parametrize("fmt", [O.NVFP4, O.MXFP4])
def test_kv_cache_k_every_row(pool, fmt):
    w = W.kv_cache(DEV)
    check_all(pool, fmt, w["k"], w["k_train"])


@pytest.mark.parametrize("fmt", [O.NVFP4, O.UFP4, O.MXFP4])
def test_guided_phases_mixed_within_ranges(pool, fmt):
    """A 16384x4096 train copy perturbed (rel 5e-2) on every fourth band of 8
    rows and equal to the rollout tensor elsewhere.  Each CTA's range spans
    several iterations, some clean and some with mismatches, so warps run the
    nearest phase with and without fine-rounding calls and switch to the
    fine phase at different points of their ranges; every element of the
    guided codes, the fused pass and the counts equals the oracle's."""
    x = W.layer_stack_layer(27, DEV, rows=16384)
    hot = W.perturb(x, 1027, rel=5e-2)
    band = (torch.arange(x.shape[0], device=DEV) // 8) % 4 == 0
    xt = torch.where(band[:, None], hot, x)
    del hot
    counts = check_all(pool, fmt, x, xt)
    assert 0.002 * x.numel() < counts[0] < 0.03 * x.numel()
