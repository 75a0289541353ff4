"""Parity of the CUDA library (through its C ABI) with the CPU oracle.

Bit-exact on codes, scale bytes, s_t bits, guidance bits and dequantized
fp32 values.  Small cases are compared in full (several CTAs, ragged
tails, empty segments); the full-size workloads are compared on sampled
rows that the oracle computes one by one after its own full amax pass.
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


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    libbuild.build()
    B.lib()
    O.lib()


def host(t):
    return t.detach().cpu().numpy()


def f32_bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def assert_same(name, got, want):
    got, want = np.asarray(got).reshape(-1), np.asarray(want).reshape(-1)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{name}: {bad.size} mismatches, first at {bad[:8]}: got {got[bad[:8]]} want {want[bad[:8]]}"


def check_quant(xb, fmt, mode=O.RTN, seg=None, seed=0, bits=True):
    """Run the library on xb (bf16 CUDA tensor) and compare with the oracle."""
    if mode == O.SR:
        q = B.tf4_quantize_sr(xb, seed, fmt=fmt, seg_off=seg)
    else:
        q = B.tf4_quantize_capture(xb, fmt=fmt, seg_off=seg, guidance=bits)
    assert B.read_status(xb.device) == 0
    xs = W.bf16_bits(xb)
    r = O.quantize(xs, fmt, mode, seg_off=seg, seed=seed, bits=bits and mode != O.SR)
    assert r["status"] == 0
    assert_same("codes", host(q.codes), r["codes"])
    assert_same("scales", host(q.scales), r["scales"])
    if O.HAS_TENSOR_SCALE[fmt]:
        assert_same("s_t", f32_bits(host(q.s_t)), f32_bits(r["s_t"]))
    if bits and mode != O.SR:
        assert_same("bits", host(q.bits), r["bits"])
    return q, r


SHAPES_NV = [(1, 16), (1, 32), (3, 48), (5, 16 * 33), (37, 2048), (129, 4096), (1000, 80), (2, 16 * 3001)]
SHAPES_MX = [(1, 32), (3, 64), (5, 32 * 33), (37, 2048), (129, 4096), (1000, 96), (2, 32 * 3001)]


@pytest.mark.parametrize("shape", SHAPES_NV)
def test_nvfp4_capture_shapes(shape):
    xb = W.random_bf16(shape, seed=sum(shape), device=DEV, outlier_frac=0.003)
    check_quant(xb, O.NVFP4)


@pytest.mark.parametrize("shape", SHAPES_MX)
def test_mxfp4_capture_shapes(shape):
    xb = W.random_bf16(shape, seed=sum(shape) + 1, device=DEV, outlier_frac=0.003)
    check_quant(xb, O.MXFP4)


@pytest.mark.parametrize("shape", SHAPES_NV)
def test_ufp4_capture_shapes(shape):
    xb = W.random_bf16(shape, seed=sum(shape) + 2, device=DEV, outlier_frac=0.003)
    check_quant(xb, O.UFP4)


FMTS = [O.NVFP4, O.MXFP4, O.UFP4]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("seed", [0, 4, 2**40 + 3])
def test_sr_parity(fmt, seed):
    xb = W.random_bf16((67, 1024), seed=seed % 1000, device=DEV, outlier_frac=0.01)
    check_quant(xb, fmt, O.SR, seed=seed)


def _seed_with_zero_uniform(idx):
    """A seed < 2^32 whose Philox4x32-10 word 0 at counter idx has its top 24
    bits zero (about one seed in 2^24), found with a vectorised search and
    confirmed by the oracle's own Philox."""
    M0, M1, W0, W1 = 0xD2511F53, 0xCD9E8D57, 0x9E3779B9, 0xBB67AE85
    mask = np.uint64(0xFFFFFFFF)
    for base in range(0, 1 << 32, 1 << 24):
        k0 = np.arange(base, base + (1 << 24), dtype=np.uint64)
        k1 = np.zeros_like(k0)
        c0 = np.full_like(k0, idx)
        c1, c2, c3 = np.zeros_like(k0), np.zeros_like(k0), np.zeros_like(k0)
        for _ in range(10):
            p0, p1 = np.uint64(M0) * c0, np.uint64(M1) * c2
            c0, c1, c2, c3 = ((p1 >> np.uint64(32)) ^ c1 ^ k0) & mask, p1 & mask, \
                ((p0 >> np.uint64(32)) ^ c3 ^ k1) & mask, p0 & mask
            k0, k1 = (k0 + np.uint64(W0)) & mask, (k1 + np.uint64(W1)) & mask
        hit = np.nonzero((c0 >> np.uint64(8)) == 0)[0]
        if hit.size:
            seed = base + int(hit[0])
            assert O.sr_uniform24(idx, seed) == 0
            return seed
    raise AssertionError("no seed found")


def test_mxfp4_sr_quotient_underflow():
    """MXFP4 with block scale 2^118 and a subnormal element: |x| 2^-118
    underflows fp32 to 0, but the exact threshold is positive, so with the
    uniform 0 the element rounds up to 0.5 (times the scale)."""
    idx = 5
    seed = _seed_with_zero_uniform(idx)
    for tiny, want in ((0x0001, 0x1), (0x8003, 0x9)):  # +2^-133, -3 * 2^-133
        x = np.zeros((1, 64), np.uint16)
        x[0, 0] = 0x7B80        # 2^120: e = 118
        x[0, idx] = tiny        # the uniform at this index is 0
        x[0, 7] = 0x3F80        # 1.0: also far below the grid's first point
        q, r = check_quant(W.from_bits(x, DEV), O.MXFP4, O.SR, seed=seed)
        assert O.unpack_codes(r["codes"], x.size)[idx] == want  # rounded up, sign kept


@pytest.mark.parametrize("fmt", FMTS)
def test_sr_full_compare_16m(fmt):
    """Every element of a 16.8M-element SR call against the oracle: enough
    elements for ~80 uniforms to fall within the fast path's safety margin
    of their threshold, which then takes the exact comparison."""
    xb = W.random_bf16((4096, 4096), seed=77, device=DEV, outlier_frac=0.001)
    check_quant(xb, fmt, O.SR, seed=2**35 + 17)


def test_rtn_equals_capture_without_guidance():
    xb = W.random_bf16((64, 512), seed=3, device=DEV)
    a = B.tf4_quantize_rtn(xb)
    b = B.tf4_quantize_capture(xb, guidance=False)
    assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales) and torch.equal(a.s_t, b.s_t)


def test_e2m1_exhaustive_via_unit_scale():
    """MXFP4 blocks whose max is 4.0 have S = 1, so y = x: every bf16 value
    with |x| < 8 (both signs) goes through the device rounding as itself."""
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    v = ((b.astype(np.uint32) << 16).view(np.float32))
    sel = b[np.isfinite(v) & (np.abs(v) < 8.0)]
    per = 31
    nblk = (len(sel) + per - 1) // per
    pad = np.zeros(nblk * per, np.uint16)
    pad[: len(sel)] = sel
    blocks = np.concatenate([np.full((nblk, 1), 0x4080, np.uint16), pad.reshape(nblk, per)], axis=1)
    xb = W.from_bits(blocks, DEV)
    check_quant(xb, O.MXFP4)


def test_uniform_grid_exhaustive_via_unit_scale():
    """UFP4 with s_t = 1 (amax = 3136) and blocks whose max is 7.0 have
    S = 1, so y = x: every bf16 value with |x| < 8 (both signs) goes through
    the device's uniform-grid rounding as itself."""
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    v = ((b.astype(np.uint32) << 16).view(np.float32))
    sel = b[np.isfinite(v) & (np.abs(v) < 7.0)]
    per = 15
    nblk = (len(sel) + per - 1) // per
    pad = np.zeros(nblk * per, np.uint16)
    pad[: len(sel)] = sel
    blocks = np.concatenate([np.full((nblk, 1), 0x40E0, np.uint16), pad.reshape(nblk, per)], axis=1)  # 7.0
    blocks = np.concatenate([blocks, np.full((1, 16), 0x4544, np.uint16)], axis=0)  # 3136.0
    check_quant(W.from_bits(blocks, DEV), O.UFP4)


@pytest.mark.parametrize("fmt,amax_bits,amax", [(O.NVFP4, 0x4528, 2688.0), (O.UFP4, 0x4544, 3136.0)])
def test_e4m3_block_scale_sweep(fmt, amax_bits, amax):
    """s_t = 1 (amax = 448 * grid max): every positive bf16 block max up to
    amax gives r = bamax / grid max, sweeping the device E4M3 rounding."""
    b = np.arange(1, 0x7F80, dtype=np.uint32).astype(np.uint16)
    v = (b.astype(np.uint32) << 16).view(np.float32)
    b = b[v <= amax]
    x = np.zeros((len(b) + 1, 16), np.uint16)
    x[:-1, 0] = b
    x[:-1, 1] = 0x8000 | b  # negative copy
    x[:-1, 2:] = (b[:, None] >> 1) & 0x7F7F
    x[-1, 0] = amax_bits
    check_quant(W.from_bits(x, DEV), fmt)


def _near_tie_tensor(rng, s_mant, rows=256, fmt=O.NVFP4):
    """Rows whose per-tensor scale is 'nice' (amax = 448 * grid max * s), so
    that many midpoint * S are bf16 values; elements sit on and around those
    points."""
    if fmt == O.UFP4:
        mids, top = np.concatenate([np.arange(7) + 0.5, np.arange(1, 8)]), 7.0
    else:
        mids, top = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, 0.5, 1, 1.5, 2, 3, 4, 6]), 6.0
    out = np.zeros((rows, 16), np.float32)
    for r in range(rows):
        S = float(np.float32(rng.choice([0.5, 1.0, 1.25, 0.75, 1.5, 0.875]) * 2.0 ** rng.integers(-3, 3)))
        pts = rng.choice(mids, 15) * S
        out[r, 1:] = pts * (1 + rng.choice([-1, 0, 0, 1], 15) * 2.0 ** -8)
        out[r, 0] = top * S
    out[0, 0] = 448.0 * top * s_mant
    xb = torch.from_numpy(out).to(torch.bfloat16)
    return xb


@pytest.mark.parametrize("fmt", [O.NVFP4, O.UFP4])
@pytest.mark.parametrize("s_mant", [1.0, 0.5, 3.0])
def test_near_tie_blocks(fmt, s_mant):
    rng = np.random.default_rng(int(s_mant * 10))
    xb = _near_tie_tensor(rng, s_mant, fmt=fmt).to(DEV)
    check_quant(xb, fmt)
    check_quant(xb, fmt, O.SR, seed=11)


@pytest.mark.parametrize("fmt", FMTS)
def test_tiny_and_zero_scales(fmt):
    x = np.zeros((8, 64), np.uint16)
    x[1, :] = 0x0001          # smallest subnormals
    x[2, 3] = 0x8000          # -0
    x[3, :16] = np.arange(16) + 0x0080  # tiny normals
    x[4, 5] = 0x0C00          # ~1e-35
    xb = W.from_bits(x, DEV)
    check_quant(xb, fmt)
    check_quant(xb, fmt, O.SR, seed=3)  # E4M3-subnormal and zero scales take the exact SR path
    seg = [0, 2, 2, 4, 8]
    if O.HAS_TENSOR_SCALE[fmt]:
        check_quant(xb, fmt, seg=seg)
        check_quant(xb, fmt, O.SR, seg=seg, seed=4)


@pytest.mark.parametrize("fmt", [O.NVFP4, O.UFP4])
def test_segments_ragged_with_empties(fmt):
    xb = W.random_bf16((300, 256), seed=9, device=DEV, outlier_frac=0.01)
    seg = [0, 0, 1, 1, 50, 51, 51, 299, 300, 300]
    q, r = check_quant(xb, fmt, seg=seg)
    check_quant(xb, fmt, O.SR, seg=seg, seed=5)
    xt = W.perturb(xb, 7, rel=0.02)
    g = B.tf4_quantize_guided(xt, q)
    want, st = O.quantize_guided(W.bf16_bits(xt), r["scales"], r["bits"], fmt, rec_s_t=r["s_t"], seg_off=seg)
    assert_same("guided", host(g), want)


@pytest.mark.parametrize("fmt", [O.NVFP4, O.UFP4])
def test_maximum_segment_count(fmt):
    """TF4_MAX_SEGMENTS (1024) ragged segments, about a fifth of them empty,
    each with its own tensor scale (values scaled per segment over 2^-20 ..
    2^20): capture, SR, guided, dequantize and fused fake-quant = oracle."""
    rng = np.random.default_rng(21)
    rows, cols, nseg = 3000, 64, B.MAX_SEGMENTS
    cuts = np.sort(rng.integers(0, rows + 1, size=nseg - 1))
    cuts[rng.random(nseg - 1) < 0.2] = cuts[0]  # repeated offsets: empty segments
    seg = [0] + sorted(int(c) for c in cuts) + [rows]
    row_scale = np.ones(rows, np.float32)
    for s in range(nseg):
        row_scale[seg[s]:seg[s + 1]] = 2.0 ** rng.integers(-20, 21)
    x = W.random_bf16((rows, cols), seed=22, device=DEV, outlier_frac=0.01)
    xb = (x.float() * torch.from_numpy(row_scale).to(DEV)[:, None]).to(torch.bfloat16)
    q, r = check_quant(xb, fmt, seg=seg)
    check_quant(xb, fmt, O.SR, seg=seg, seed=23)
    xt = W.perturb(xb, 24, rel=0.02)
    xts = W.bf16_bits(xt)
    want, _ = O.quantize_guided(xts, r["scales"], r["bits"], fmt, rec_s_t=r["s_t"], seg_off=seg)
    assert_same("guided", host(B.tf4_quantize_guided(xt, q)), want)
    rd = O.dequantize(r["codes"], r["scales"], rows, cols, fmt, s_t=r["s_t"], seg_off=seg)
    assert_same("dequant", f32_bits(host(B.tf4_dequantize(q))), f32_bits(rd))
    y, _ = B.tf4_guided_fake_quant(xt, q)
    _, rv, _ = O.guided_fake_quant(xts, r["scales"], r["bits"], fmt, rec_s_t=r["s_t"], seg_off=seg)
    assert_same("fake-quant", f32_bits(host(y)), f32_bits(rv))
    assert B.read_status(xb.device) == 0


@pytest.mark.parametrize("fmt", [O.NVFP4, O.UFP4])
def test_segment_amax_and_amax_in(fmt):
    xb = W.random_bf16((200, 512), seed=12, device=DEV, outlier_frac=0.01)
    seg = [0, 20, 20, 150, 200]
    amax = B.tf4_segment_amax(xb, seg)
    want, _ = O.segment_amax(W.bf16_bits(xb), seg)
    assert_same("amax", f32_bits(host(amax)), f32_bits(want))
    a = B.tf4_quantize_capture(xb, fmt=fmt, seg_off=seg)
    b = B.tf4_quantize_capture(xb, fmt=fmt, seg_off=seg, amax_in=amax)
    for n in ("codes", "scales", "s_t", "bits"):
        assert torch.equal(getattr(a, n), getattr(b, n)), n
    check_quant(xb, fmt, seg=seg)


def test_workspace_returns_to_zero():
    xb = W.random_bf16((64, 1024), seed=13, device=DEV)
    seg = [0, 10, 64]
    B.tf4_quantize_rtn(xb, seg_off=seg)
    torch.cuda.synchronize()
    for ws in B._ws_cache.values():
        assert int(ws.count_nonzero()) == 0


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("perturb", [0.0, 1e-3, 0.05])
def test_guided_parity(fmt, perturb):
    xb = W.random_bf16((96, 1024), seed=17, device=DEV, outlier_frac=0.005)
    q, r = check_quant(xb, fmt)
    xt = W.perturb(xb, 23, rel=perturb) if perturb else xb
    g = B.tf4_quantize_guided(xt, q)
    assert B.read_status(xb.device) == 0
    want, st = O.quantize_guided(W.bf16_bits(xt), r["scales"], r["bits"], fmt, rec_s_t=r["s_t"])
    assert st == 0
    assert_same("guided", host(g), want)
    if perturb == 0.0:
        assert torch.equal(g, q.codes)


@pytest.mark.parametrize("fmt", FMTS)
def test_guided_unrelated_train_tensor(fmt):
    """Train-side values unrelated to the rollout's (about half the nibbles
    disagree with the recorded bit): every element still lands on the
    neighbour the oracle picks."""
    xb = W.random_bf16((80, 2048), seed=19, device=DEV, outlier_frac=0.005)
    q, r = check_quant(xb, fmt)
    xt = W.random_bf16((80, 2048), seed=20, device=DEV, outlier_frac=0.005)
    g = B.tf4_quantize_guided(xt, q)
    want, _ = O.quantize_guided(W.bf16_bits(xt), r["scales"], r["bits"], fmt, rec_s_t=r["s_t"])
    assert_same("guided", host(g), want)


@pytest.mark.parametrize("fmt", FMTS)
def test_guided_reproduces_sr_capture(fmt):
    xb = W.random_bf16((64, 512), seed=29, device=DEV)
    q = B.tf4_quantize_sr(xb, 77, fmt=fmt)
    q.bits = B.tf4_pack_guidance(q.codes, 64, 512, fmt)
    g = B.tf4_quantize_guided(xb, q)
    assert torch.equal(g, q.codes)


@pytest.mark.parametrize("fmt", [O.NVFP4, O.UFP4])
def test_guided_near_ties(fmt):
    rng = np.random.default_rng(5)
    xb = _near_tie_tensor(rng, 1.0, fmt=fmt).to(DEV)
    q, r = check_quant(xb, fmt)
    xt = _near_tie_tensor(np.random.default_rng(6), 1.0, fmt=fmt).to(DEV)
    g = B.tf4_quantize_guided(xt, q)
    want, _ = O.quantize_guided(W.bf16_bits(xt), r["scales"], r["bits"], fmt, rec_s_t=r["s_t"])
    assert_same("guided", host(g), want)


def _large_scale_with_tiny_train_values(fmt, rows=64, cols=1024):
    """Rollout values of order 2^20 (NVFP4, UFP4) or 2^115 (MXFP4), so that
    every block scale is large; the train copy replaces a quarter of the
    elements with zeros and bf16 subnormals of both signs.  A subnormal train
    value times the block's reciprocal scale underflows fp32 to zero, yet
    its exact quotient is positive and not a codeword: where the recorded bit
    is 1 the guided code is the smallest nonzero codeword, never zero."""
    big = 2.0 ** (115 if fmt == O.MXFP4 else 20)
    xb = W.random_bf16((rows, cols), seed=91, device=DEV, scale=big)
    bits = W.bf16_bits(xb).copy().reshape(-1)
    rng = np.random.default_rng(92)
    pos = rng.choice(bits.size, bits.size // 4, replace=False)
    tiny = rng.choice(np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x0003, 0x007F, 0x8040], dtype=np.uint16), pos.size)
    bits[pos] = tiny
    return xb, W.from_bits(bits.reshape(rows, cols), DEV)


@pytest.mark.parametrize("fmt", FMTS)
def test_guided_tiny_train_values_under_large_scales(fmt):
    xb, xt = _large_scale_with_tiny_train_values(fmt)
    q, r = check_quant(xb, fmt)
    want, _ = O.quantize_guided(W.bf16_bits(xt), r["scales"], r["bits"], fmt, rec_s_t=r["s_t"])
    # the case is live: nonzero train subnormals recorded with bit 1 must move off zero
    assert (O.unpack_codes(want, want.size * 2) & 7).astype(bool).any()
    assert_same("guided", host(B.tf4_quantize_guided(xt, q)), want)
    codes, vals, _ = O.guided_fake_quant(W.bf16_bits(xt), r["scales"], r["bits"], fmt, rec_s_t=r["s_t"])
    y, c = B.tf4_guided_fake_quant(xt, q, want_codes=True)
    assert_same("fake-quant codes", host(c), codes)
    assert_same("fake-quant values", f32_bits(host(y)), f32_bits(vals))
    counts = B.tf4_mismatch_stats(xt, q)
    assert host(counts).tolist() == O.mismatch_stats(W.bf16_bits(xt), r["scales"], r["codes"], fmt,
                                                     rec_s_t=r["s_t"]).tolist()
    assert B.read_status(xb.device) == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_dequant_parity(fmt):
    xb = W.random_bf16((77, 2048), seed=31, device=DEV, outlier_frac=0.01)
    seg = [0, 30, 77] if O.HAS_TENSOR_SCALE[fmt] else None
    q, r = check_quant(xb, fmt, seg=seg)
    d = B.tf4_dequantize(q)
    want = O.dequantize(r["codes"], r["scales"], 77, 2048, fmt, s_t=r["s_t"], seg_off=seg)
    assert_same("dequant", f32_bits(host(d)), f32_bits(want))


@pytest.mark.parametrize("fmt,seg", [(O.NVFP4, None), (O.NVFP4, [0, 25, 25, 77]), (O.MXFP4, None), (O.UFP4, None),
                                     (O.UFP4, [0, 25, 25, 77])])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_guided_fake_quant_parity(fmt, seg, dtype):
    """The fused train-side pass equals guided quantization followed by
    dequantization (and, for bf16, RNE of the fp32 value), codes included."""
    xb = W.random_bf16((77, 2048), seed=43, device=DEV, outlier_frac=0.01)
    q, r = check_quant(xb, fmt, seg=seg)
    xt = W.perturb(xb, 44, rel=0.05)
    y, c = B.tf4_guided_fake_quant(xt, q, out_dtype=dtype, want_codes=True)
    assert B.read_status(xb.device) == 0
    codes, vals, st = O.guided_fake_quant(W.bf16_bits(xt), r["scales"], r["bits"], fmt, rec_s_t=r["s_t"],
                                          seg_off=seg)
    assert_same("codes", host(c), codes)
    if dtype == torch.float32:
        assert_same("values", f32_bits(host(y)), f32_bits(vals))
    else:
        assert_same("values", host(y.view(torch.int16)).view(np.uint16), O.f32_to_bf16(vals))


@pytest.mark.parametrize("fmt", FMTS)
def test_fp32_outputs_only_16_byte_aligned(fmt):
    """Outputs 16-B but not 32-B aligned take the 16-byte-store kernels
    (dequantize, fused fp32 fake-quant): same values."""
    rows, cols = 37, 1024
    xb = W.random_bf16((rows, cols), seed=47, device=DEV, outlier_frac=0.01)
    q, r = check_quant(xb, fmt)
    buf = torch.empty(rows * cols + 8, dtype=torch.float32, device=DEV)
    view = buf[4:4 + rows * cols].view(rows, cols)
    assert view.data_ptr() % 32 == 16
    d = B.tf4_dequantize(q, out=view)
    want = O.dequantize(r["codes"], r["scales"], rows, cols, fmt, s_t=r["s_t"])
    assert_same("dequant", f32_bits(host(d)), f32_bits(want))
    xt = W.perturb(xb, 48, rel=0.05)
    y, _ = B.tf4_guided_fake_quant(xt, q, out=view)
    _, vals, _ = O.guided_fake_quant(W.bf16_bits(xt), r["scales"], r["bits"], fmt, rec_s_t=r["s_t"])
    assert_same("fake-quant", f32_bits(host(y)), f32_bits(vals))


@pytest.mark.parametrize("fmt,shape", [(O.NVFP4, (1, 16)), (O.NVFP4, (3, 48)), (O.UFP4, (5, 16 * 33)), (O.MXFP4, (3, 64)),
                                       (O.MXFP4, (1, 32))])
def test_guided_fake_quant_small_shapes(fmt, shape):
    """Single blocks and ragged block counts through the fused pass."""
    xb = W.random_bf16(shape, seed=sum(shape) + 5, device=DEV, outlier_frac=0.05)
    q, r = check_quant(xb, fmt)
    xt = W.perturb(xb, 45, rel=0.05)
    for dtype in (torch.float32, torch.bfloat16):
        y, c = B.tf4_guided_fake_quant(xt, q, out_dtype=dtype, want_codes=True)
        codes, vals, st = O.guided_fake_quant(W.bf16_bits(xt), r["scales"], r["bits"], fmt, rec_s_t=r["s_t"])
        assert_same("codes", host(c), codes)
        if dtype == torch.float32:
            assert_same("values", f32_bits(host(y)), f32_bits(vals))
        else:
            assert_same("values", host(y.view(torch.int16)).view(np.uint16), O.f32_to_bf16(vals))


@pytest.mark.parametrize("fmt,seg", [(O.NVFP4, None), (O.NVFP4, [0, 30, 30, 64]), (O.MXFP4, None), (O.UFP4, None),
                                     (O.UFP4, [0, 30, 30, 64])])
@pytest.mark.parametrize("rel", [1e-3, 0.05, None])
def test_mismatch_stats_parity(fmt, seg, rel):
    """Mismatch diagnostics equal the oracle's counts (None: unrelated train tensor)."""
    xb = W.random_bf16((64, 2048), seed=51, device=DEV, outlier_frac=0.005)
    q, r = check_quant(xb, fmt, seg=seg)
    xt = W.perturb(xb, 52, rel=rel) if rel else W.random_bf16((64, 2048), seed=53, device=DEV)
    c = B.tf4_mismatch_stats(xt, q)
    assert B.read_status(xb.device) == 0
    want = O.mismatch_stats(W.bf16_bits(xt), r["scales"], r["codes"], fmt, rec_s_t=r["s_t"], seg_off=seg)
    assert host(c).tolist() == want.tolist()
    if rel == 1e-3:
        assert want[0] == want[1] + want[2]


def test_bench_mismatch_by_layer_counts():
    """The bench's per-layer diagnostics mode (a few small layers of the
    stack) reports, for every layer, the oracle's counts of that layer's
    train copy against its capture."""
    import argparse

    import bench

    args = argparse.Namespace(layers=3, rows=512, cols=1024, train_rel=0.05)
    out = bench.run_mismatch_by_layer(args)
    assert [r["layer"] for r in out["rows"]] == [0, 1, 2]
    for r in out["rows"]:
        x = W.layer_stack_layer(r["layer"], DEV, rows=512, cols=1024)
        xs = W.bf16_bits(x)
        rec = O.quantize(xs, O.NVFP4, O.RTN, bits=True)
        xt = W.bf16_bits(W.perturb(x, 1000 + r["layer"], rel=0.05))
        want = O.mismatch_stats(xt, rec["scales"], rec["codes"], O.NVFP4, rec_s_t=rec["s_t"])
        got = [r[k] for k in ("mismatch", "adjacent", "far", "after_guidance", "toward_smaller", "toward_larger")]
        assert got == want.tolist(), (r["layer"], got, want.tolist())
        assert r["elements"] == x.numel()


@pytest.mark.parametrize("fmt", [O.NVFP4, O.UFP4])
def test_mismatch_stats_near_ties(fmt):
    """Train values on and around the recorded grid's midpoints and codewords:
    the fast nearest / guided paths of the diagnostics agree with the oracle."""
    xb = _near_tie_tensor(np.random.default_rng(15), 1.0, fmt=fmt).to(DEV)
    q, r = check_quant(xb, fmt)
    xt = _near_tie_tensor(np.random.default_rng(16), 1.0, fmt=fmt).to(DEV)
    c = B.tf4_mismatch_stats(xt, q)
    want = O.mismatch_stats(W.bf16_bits(xt), r["scales"], r["codes"], fmt, rec_s_t=r["s_t"])
    assert host(c).tolist() == want.tolist()


@pytest.mark.parametrize("fmt,L,keep", [(O.NVFP4, 5, 2), (O.NVFP4, 3, 3), (O.NVFP4, 1, 0), (O.MXFP4, 4, 1),
                                        (O.UFP4, 4, 2)])
def test_capture_batched_parity(fmt, L, keep):
    """One batched call = per-layer capture (oracle) for every layer; the
    deepest `keep` layers' guidance lands contiguously in the info cache."""
    xs = [W.random_bf16((96, 1024), seed=60 + i, device=DEV, outlier_frac=0.01 * (i % 2)) for i in range(L)]
    out = B.tf4_quantize_capture_batched(xs, fmt=fmt, keep=keep)
    assert B.read_status(xs[0].device) == 0
    for i, x in enumerate(xs):
        r = O.quantize(W.bf16_bits(x), fmt, O.RTN, bits=True)
        assert_same(f"codes {i}", host(out.codes[i]), r["codes"])
        assert_same(f"scales {i}", host(out.scales[i]), r["scales"])
        if O.HAS_TENSOR_SCALE[fmt]:
            assert_same(f"s_t {i}", f32_bits(host(out.s_t[i:i + 1])), f32_bits(r["s_t"]))
        if i >= L - keep:
            assert_same(f"bits {i}", host(out.info_bits[i - (L - keep)]), r["bits"])
    if keep:
        g = B.tf4_quantize_guided(xs[-1], out.layer(L - 1))
        assert torch.equal(g, out.codes[L - 1])


@pytest.mark.parametrize("fmt,keep", [(O.NVFP4, 64), (O.MXFP4, 1), (O.UFP4, 33)])
def test_capture_batched_maximum_layer_count(fmt, keep):
    """TF4_MAX_BATCH (64) layers in one call, each with its own scale range."""
    L = 64
    blk = O.BLOCK[fmt]
    xs = [(W.random_bf16((7, 3 * blk), seed=200 + i, device=DEV, outlier_frac=0.05).float() * 2.0 ** (i - 32)
           ).to(torch.bfloat16) for i in range(L)]
    out = B.tf4_quantize_capture_batched(xs, fmt=fmt, keep=keep)
    assert B.read_status(xs[0].device) == 0
    for i, x in enumerate(xs):
        r = O.quantize(W.bf16_bits(x), fmt, O.RTN, bits=True)
        assert_same(f"codes {i}", host(out.codes[i]), r["codes"])
        assert_same(f"scales {i}", host(out.scales[i]), r["scales"])
        if O.HAS_TENSOR_SCALE[fmt]:
            assert_same(f"s_t {i}", f32_bits(host(out.s_t[i:i + 1])), f32_bits(r["s_t"]))
        if i >= L - keep:
            assert_same(f"bits {i}", host(out.info_bits[i - (L - keep)]), r["bits"])


def test_capture_batched_large_layers_per_layer_path():
    """Layers of 2^27 elements take the per-layer launch path inside the
    batched call: per layer the same bytes as tf4_quantize_capture, and
    sampled rows of the middle layer against the oracle."""
    rows, cols, L, keep = 8192, 16384, 3, 2
    xs = [W.random_bf16((rows, cols), seed=70 + i, device=DEV, outlier_frac=0.001) for i in range(L)]
    out = B.tf4_quantize_capture_batched(xs, keep=keep)
    assert B.read_status(xs[0].device) == 0
    for i, x in enumerate(xs):
        ref = B.tf4_quantize_capture(x, guidance=i >= L - keep)
        assert torch.equal(out.codes[i], ref.codes) and torch.equal(out.scales[i].reshape(-1), ref.scales.reshape(-1))
        assert torch.equal(out.s_t[i:i + 1].view(torch.int32), ref.s_t.view(torch.int32))
        if i >= L - keep:
            assert torch.equal(out.info_bits[i - (L - keep)], ref.bits)
    x1 = W.bf16_bits(xs[1])
    for r0 in (0, 4093, rows - 3):
        r = O.quantize(x1, O.NVFP4, bits=True, s_t=host(out.s_t[1:2]), row_range=(r0, r0 + 3))
        lo, hi = r0 * cols, (r0 + 3) * cols
        assert_same("codes rows", host(out.codes[1])[lo // 2:hi // 2], r["codes"][lo // 2:hi // 2])
        assert_same("bits rows", host(out.info_bits[0])[lo // 8:hi // 8], r["bits"][lo // 8:hi // 8])


@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (64, 1024), (5, 16 * 33)])
def test_pack_unpack_parity(shape):
    rows, cols = shape
    codes = torch.randint(0, 256, (rows * cols // 2,), dtype=torch.uint8, device=DEV)
    bits = B.tf4_pack_guidance(codes, rows, cols)
    want = O.pack_guidance(host(codes), rows * cols)
    assert_same("pack", host(bits), want)
    mant = B.tf4_unpack_guidance(bits, rows, cols)
    assert_same("unpack", host(mant), O.unpack_guidance(want, rows * cols))


def test_nonfinite_reported():
    xb = W.random_bf16((40, 256), seed=37, device=DEV)
    x = W.bf16_bits(xb)
    x[25, 7] = 0x7F80
    seg = [0, 20, 40]
    xb = W.from_bits(x, DEV)
    q = B.tf4_quantize_capture(xb, seg_off=seg)
    assert B.read_status(xb.device) == 5
    assert B.read_status(xb.device) == 0  # cleared
    r = O.quantize(x[:20], O.NVFP4, bits=True)
    assert_same("clean segment", host(q.codes)[: 20 * 128], r["codes"])
    B.tf4_quantize_rtn(xb, fmt=B.MXFP4)
    assert B.read_status(xb.device) == 5
    x2 = W.bf16_bits(W.random_bf16((4, 64), seed=1, device=DEV))
    q2 = B.tf4_quantize_capture(W.from_bits(x2, DEV))
    x2[1, 1] = 0x7FC1
    B.tf4_quantize_guided(W.from_bits(x2, DEV), q2)
    assert B.read_status(xb.device) == 5


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("bad", [0x7F80, 0xFF80, 0x7FC1])  # +Inf, -Inf, NaN
def test_nonfinite_reported_by_every_call(fmt, bad):
    """Every call that reads bf16 values reports a non-finite input in the
    status word (and the word clears on reading); the same calls on the
    clean tensor report nothing."""
    rows, cols = 48, 256
    clean = W.random_bf16((rows, cols), seed=41, device=DEV)
    xb = W.bf16_bits(clean)
    xb[31, 77] = bad
    dirty = W.from_bits(xb, DEV)
    q = B.tf4_quantize_capture(clean, fmt=fmt)
    assert B.read_status(clean.device) == 0
    calls = {
        "capture": lambda x: B.tf4_quantize_capture(x, fmt=fmt),
        "rtn": lambda x: B.tf4_quantize_rtn(x, fmt=fmt),
        "sr": lambda x: B.tf4_quantize_sr(x, 3, fmt=fmt),
        "guided": lambda x: B.tf4_quantize_guided(x, q),
        "fake_quant": lambda x: B.tf4_guided_fake_quant(x, q),
        "fake_quant_bf16": lambda x: B.tf4_guided_fake_quant(x, q, out_dtype=torch.bfloat16),
        "mismatch": lambda x: B.tf4_mismatch_stats(x, q),
        "batched": lambda x: B.tf4_quantize_capture_batched([clean, x], fmt=fmt, keep=1),
    }
    if O.HAS_TENSOR_SCALE[fmt]:
        calls["amax"] = lambda x: B.tf4_segment_amax(x)
    for name, call in calls.items():
        call(clean)
        assert B.read_status(clean.device) == 0, name
        call(dirty)
        assert B.read_status(clean.device) == 5, name
        assert B.read_status(clean.device) == 0, name


def test_empty_tensor():
    xb = torch.zeros((0, 64), dtype=torch.bfloat16, device=DEV)
    q = B.tf4_quantize_capture(xb, seg_off=[0, 0, 0])
    assert q.s_t.shape == (2,) and not q.s_t.any()


@pytest.mark.parametrize("fmt,shape", [(O.NVFP4, (1, 16)), (O.NVFP4, (130, 80)), (O.MXFP4, (300, 2048)),
                                       (O.UFP4, (77, 48)), (O.NVFP4, (256, 4096))])
def test_swizzled_scales_parity(fmt, shape):
    """Scale bytes in the tiled layout of block-scaled GEMMs: the oracle's
    index map, zero padding included."""
    xb = W.random_bf16(shape, seed=sum(shape) + 9, device=DEV, outlier_frac=0.01)
    q, r = check_quant(xb, fmt)
    blk = B.tf4_swizzle_scales(q)
    want = O.swizzle_scales(r["scales"].reshape(shape[0], -1))
    assert_same("blocked scales", host(blk), want)


def test_block_scaled_gemm_consumes_the_record():
    """An NVFP4 record (codes + tiled E4M3 scales) fed to the block-scaled
    FP4 GEMM behind torch._scaled_mm gives the product of the dequantized
    matrices times the two tensor scales (which the GEMM leaves out), within
    the bf16 output's rounding.  (torch's FP4 GEMM takes E4M3 block scales
    only; the MXFP4 layout is checked against the oracle above.)"""
    fmt = O.NVFP4
    m, n, k = 256, 384, 1024
    a = W.random_bf16((m, k), seed=91, device=DEV, outlier_frac=0.01)
    b = W.random_bf16((n, k), seed=92, device=DEV, outlier_frac=0.01)
    qa, qb = B.tf4_quantize_capture(a, fmt=fmt), B.tf4_quantize_capture(b, fmt=fmt)
    sdt = torch.float8_e4m3fn
    sa, sb = B.tf4_swizzle_scales(qa).view(sdt).reshape(-1), B.tf4_swizzle_scales(qb).view(sdt).reshape(-1)
    fa = qa.codes.view(m, k // 2).view(torch.float4_e2m1fn_x2)
    fb = qb.codes.view(n, k // 2).view(torch.float4_e2m1fn_x2)
    c = torch._scaled_mm(fa, fb.t(), sa, sb, out_dtype=torch.bfloat16).float() * (qa.s_t * qb.s_t)
    ref = B.tf4_dequantize(qa) @ B.tf4_dequantize(qb).t()
    err = (c - ref).abs().max().item()
    assert err <= 2.0 ** -7 * ref.abs().max().item(), (err, ref.abs().max().item())


def test_cuda_graph_capture_and_replay():
    """The calls launch only kernels on the given stream (no allocation, no
    host synchronisation), so a rollout capture + train-side fake-quant step
    can be captured in a CUDA graph and replayed on new data in the same
    buffers, with the results of direct calls."""
    rows, cols = 96, 2048
    x = W.random_bf16((rows, cols), seed=81, device=DEV, outlier_frac=0.01)
    xt = W.perturb(x, 82, rel=0.01)
    y = torch.empty((rows, cols), dtype=torch.bfloat16, device=DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up on the capture stream: its workspace exists before capture
        q = B.tf4_quantize_capture(x)
        B.tf4_guided_fake_quant(xt, q, out=y)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        B.tf4_quantize_capture(x, out=q)
        B.tf4_guided_fake_quant(xt, q, out=y)
    for seed in (83, 84):
        x.copy_(W.random_bf16((rows, cols), seed=seed, device=DEV, outlier_frac=0.02))
        xt.copy_(W.perturb(x, seed + 10, rel=0.01))
        g.replay()
        torch.cuda.synchronize()
        q2 = B.tf4_quantize_capture(x)
        y2, _ = B.tf4_guided_fake_quant(xt, q2, out_dtype=torch.bfloat16)
        for name in ("codes", "scales", "s_t", "bits"):
            assert torch.equal(getattr(q, name), getattr(q2, name)), name
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    assert B.read_status(x.device) == 0 and B.read_status(x.device, s) == 0
    del g


def test_wrappers_on_a_stream_that_is_not_current():
    """Every wrapper called with stream= a stream other than the current
    one, while the current stream is still busy: the outputs, the fresh
    workspace and the status word the call creates are ordered on that
    stream, so the results equal the oracle's."""
    rows, cols, seg = 96, 2048, [0, 40, 40, 96]
    x = W.random_bf16((rows, cols), seed=85, device=DEV, outlier_frac=0.01)
    xt = W.perturb(x, 86, rel=0.05)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()  # a new stream: new workspace and status-word keys
    busy = torch.empty(1 << 28, dtype=torch.float32, device=DEV)
    for _ in range(4):
        busy.mul_(1.0001)  # ~4 GB of traffic left running on the current stream
    q = B.tf4_quantize_capture(x, seg_off=seg, stream=s)
    g = B.tf4_quantize_guided(xt, q, stream=s)
    d = B.tf4_dequantize(q, stream=s)
    y, c = B.tf4_guided_fake_quant(xt, q, want_codes=True, stream=s)
    sr = B.tf4_quantize_sr(x, 2**33 + 5, seg_off=seg, stream=s)
    am = B.tf4_segment_amax(x, seg_off=seg, stream=s)
    bits = B.tf4_pack_guidance(q.codes, rows, cols, stream=s)
    assert B.read_status(x.device, s) == 0
    torch.cuda.synchronize()
    xs, xts = W.bf16_bits(x), W.bf16_bits(xt)
    r = O.quantize(xs, O.NVFP4, O.RTN, seg_off=seg, bits=True)
    assert_same("codes", host(q.codes), r["codes"])
    assert_same("s_t", f32_bits(host(q.s_t)), f32_bits(r["s_t"]))
    assert_same("bits", host(q.bits), r["bits"])
    assert_same("packed bits", host(bits), r["bits"])
    rg, _ = O.quantize_guided(xts, r["scales"], r["bits"], O.NVFP4, rec_s_t=r["s_t"], seg_off=seg)
    assert_same("guided", host(g), rg)
    assert_same("fake-quant codes", host(c), rg)
    rd = O.dequantize(r["codes"], r["scales"], rows, cols, O.NVFP4, s_t=r["s_t"], seg_off=seg)
    assert_same("dequant", f32_bits(host(d)), f32_bits(rd))
    _, rfq, _ = O.guided_fake_quant(xts, r["scales"], r["bits"], O.NVFP4, rec_s_t=r["s_t"], seg_off=seg)
    assert_same("fake-quant", f32_bits(host(y)), f32_bits(rfq))
    rs = O.quantize(xs, O.NVFP4, O.SR, seg_off=seg, seed=2**33 + 5)
    assert_same("sr codes", host(sr.codes), rs["codes"])
    assert_same("amax", f32_bits(host(am)), f32_bits(O.segment_amax(xs, seg)[0]))
    del busy


@pytest.mark.parametrize("fmt", [O.NVFP4, O.UFP4])
@pytest.mark.parametrize("world", [2, 3])
def test_row_sharded_capture_on_one_gpu(fmt, world):
    """The row-sharded path with its real CUDA calls: each shard's amax pass
    (tf4_segment_amax on its rows, every segment kept), the MAX over shards
    (what the all-reduce computes), then each shard's capture with amax_in.
    The shards' codes, scales, bits and s_t are exactly the unsharded
    capture's, which equals the oracle's."""
    from fp4_block_scaled_quantizer_b200 import sharded

    rows, cols, seg = 203, 1024, [0, 50, 50, 130, 203]
    x = W.random_bf16((rows, cols), seed=97, device=DEV, outlier_frac=0.01)
    full, r = check_quant(x, fmt, seg=seg)
    parts = []
    for rank in range(world):
        b, e = sharded.shard_rows(rows, world, rank)
        parts.append((b, e, x[b:e].contiguous(), sharded.shard_segments(seg, b, e)))
    amax = [B.tf4_segment_amax(xs, so) for _, _, xs, so in parts]
    gmax = amax[0]
    for a in amax[1:]:
        gmax = torch.maximum(gmax, a)
    for b, e, xs, so in parts:
        q = B.tf4_quantize_capture(xs, fmt=fmt, seg_off=so, amax_in=gmax)
        assert torch.equal(q.codes, full.codes[b * cols // 2:e * cols // 2])
        assert torch.equal(q.scales.view(-1), full.scales.view(-1)[b * cols // 16:e * cols // 16])
        assert torch.equal(q.bits, full.bits[b * cols // 8:e * cols // 8])
        assert torch.equal(q.s_t.view(torch.int32), full.s_t.view(torch.int32))
    assert B.read_status(x.device) == 0


def test_ste_identity_backward():
    from fp4_block_scaled_quantizer_b200 import ste
    xb = W.random_bf16((16, 256), seed=41, device=DEV).requires_grad_(True)
    q = B.tf4_quantize_capture(xb.detach())
    y = ste.guided_fake_quant(xb, q, out_dtype=torch.bfloat16)
    g = torch.randn_like(y)
    y.backward(g)
    assert torch.equal(xb.grad, g)
    d = B.tf4_dequantize(q)
    assert torch.equal(y.float(), d.to(torch.bfloat16).float())


# ------------------------------------------------------ full-size workloads
def sample_rows(rows, seg=None, k=24, seed=0):
    rng = np.random.default_rng(seed)
    pick = {0, rows - 1, rows // 2}
    if seg is not None:
        for s in seg[1:-1]:
            if 0 < s < rows:
                pick |= {s - 1, s}
    pick |= set(int(v) for v in rng.integers(0, rows, k))
    return sorted(pick)


def check_sampled(xb, q, fmt, seg=None, mode=O.RTN, seed=0, guided_x=None, g_codes=None):
    rows, cols = xb.shape
    xs = W.bf16_bits(xb)
    s_t = None
    if O.HAS_TENSOR_SCALE[fmt]:
        s_t, st = O.segment_scales(xs, seg, fmt)
        assert st == 0
        assert_same("s_t", f32_bits(host(q.s_t)), f32_bits(s_t))
    blk = O.BLOCK[fmt]
    gcodes, gsc = host(q.codes), host(q.scales).reshape(-1)
    gbits = host(q.bits) if q.bits is not None else None
    xt = W.bf16_bits(guided_x) if guided_x is not None else None
    gg = host(g_codes) if g_codes is not None else None
    for r in sample_rows(rows, seg):
        rr = O.quantize(xs, fmt, mode, seg_off=seg, seed=seed, s_t=s_t, row_range=(r, r + 1),
                        bits=gbits is not None)
        c0, c1 = r * cols // 2, (r + 1) * cols // 2
        assert_same(f"codes row {r}", gcodes[c0:c1], rr["codes"][c0:c1])
        assert_same(f"scales row {r}", gsc[r * cols // blk:(r + 1) * cols // blk],
                    rr["scales"][r * cols // blk:(r + 1) * cols // blk])
        if gbits is not None:
            assert_same(f"bits row {r}", gbits[r * cols // 8:(r + 1) * cols // 8],
                        rr["bits"][r * cols // 8:(r + 1) * cols // 8])
        if xt is not None:
            wg, _ = O.quantize_guided(xt, rr["scales"], rr["bits"], fmt, rec_s_t=s_t, seg_off=seg,
                                      row_range=(r, r + 1))
            assert_same(f"guided row {r}", gg[c0:c1], wg[c0:c1])


def test_activation_outliers_full():
    w = W.activation_outliers(DEV)
    q, r = check_quant(w["x"], O.NVFP4)
    for xt in (w["x_train"], w["x"]):
        g = B.tf4_quantize_guided(xt, q)
        want, _ = O.quantize_guided(W.bf16_bits(xt), r["scales"], r["bits"], O.NVFP4, rec_s_t=r["s_t"])
        assert_same("guided", host(g), want)


@pytest.mark.parametrize("fmt,layer", [(O.NVFP4, 0), (O.NVFP4, 39), (O.UFP4, 39)])
def test_layer_stack_layer_sampled(fmt, layer):
    x = W.layer_stack_layer(layer, DEV)
    q = B.tf4_quantize_capture(x, fmt=fmt, guidance=layer >= 20)
    g = B.tf4_quantize_guided(x, q) if layer >= 20 else None
    assert B.read_status(x.device) == 0
    check_sampled(x, q, fmt, g_codes=g, guided_x=x if g is not None else None)
    if g is not None:
        assert torch.equal(g, q.codes)


@pytest.mark.parametrize("fmt", [O.NVFP4, O.UFP4])
def test_moe_dispatch_sampled(fmt):
    w = W.moe_dispatch(DEV)
    seg = w["seg_off"]
    q = B.tf4_quantize_capture(w["x"], fmt=fmt, seg_off=seg)
    g = B.tf4_quantize_guided(w["x_train"], q)
    assert B.read_status(w["x"].device) == 0
    check_sampled(w["x"], q, fmt, seg=seg, guided_x=w["x_train"], g_codes=g)


def test_weights_sampled():
    x = W.weights(DEV)
    q = B.tf4_quantize_sr(x, 0)
    check_sampled(x, q, O.NVFP4, mode=O.SR, seed=0)
    qm = B.tf4_quantize_rtn(x, fmt=B.MXFP4)
    check_sampled(x, qm, O.MXFP4)


def test_kv_cache_sampled():
    w = W.kv_cache(DEV)
    for name in ("k", "v"):
        x, xt = w[name], w[name + "_train"]
        q = B.tf4_quantize_capture(x)
        g = B.tf4_quantize_guided(xt, q)
        check_sampled(x, q, O.NVFP4, guided_x=xt, g_codes=g)
        assert torch.equal(B.tf4_quantize_guided(x, q), q.codes)


def test_sr_counter_beyond_2_32():
    """Element indices above 2^32 use the counter's high word: MXFP4 SR on a
    (2^32 + 2^20)-element tensor, rows sampled across the boundary."""
    cols = 4096
    rows = (2**32 + 2**20) // cols
    g = torch.Generator(device=DEV).manual_seed(8)
    x = (torch.rand((rows, cols), generator=g, device=DEV) * 2 - 1).to(torch.bfloat16)
    q = B.tf4_quantize_sr(x, 2**33 + 5, fmt=B.MXFP4)
    torch.cuda.synchronize()
    r0 = 2**32 // cols
    for r in (0, r0 - 1, r0, r0 + 1, rows - 1):
        want = _oracle_row_with_offset(W.bf16_bits(x[r:r + 1])[0], r * cols, 2**33 + 5)
        assert_same(f"row {r}", host(q.codes[r * cols // 2:(r + 1) * cols // 2]), want)
    del x, q
    torch.cuda.empty_cache()


def test_nvfp4_capture_beyond_2_32_elements():
    """NVFP4 capture + guided on a (2^32 + 2^20)-element tensor: 64-bit
    block indices through amax, quantize, guided and pack; the tensor scale
    against the oracle's full amax pass, sampled rows (across the 2^32
    boundary) against the oracle given that scale."""
    cols = 4096
    rows = (2**32 + 2**20) // cols
    g = torch.Generator(device=DEV).manual_seed(9)
    x = torch.randn((rows, cols), generator=g, device=DEV, dtype=torch.bfloat16)
    q = B.tf4_quantize_capture(x)
    gq = B.tf4_quantize_guided(x, q)
    assert B.read_status(x.device) == 0
    assert torch.equal(gq, q.codes)
    del gq
    bits = B.tf4_pack_guidance(q.codes, rows, cols)
    assert torch.equal(bits, q.bits)
    del bits
    xs = W.bf16_bits(x)
    st, status = O.segment_scales(xs)
    assert status == 0
    assert_same("s_t", f32_bits(host(q.s_t)), f32_bits(st))
    r0 = 2**32 // cols
    for r in (0, r0 - 1, r0, r0 + 1, rows - 1):
        want = O.quantize(xs[r:r + 1], O.NVFP4, s_t=st, bits=True)
        assert_same(f"codes row {r}", host(q.codes[r * cols // 2:(r + 1) * cols // 2]), want["codes"])
        assert_same(f"scales row {r}", host(q.scales[r]), want["scales"])
        assert_same(f"bits row {r}", host(q.bits[r * cols // 8:(r + 1) * cols // 8]), want["bits"])
    del x, q, xs
    torch.cuda.empty_cache()


def test_dequant_fake_quant_unpack_diagnostics_beyond_2_32_elements():
    """The other 64-bit paths on a (2^32 + 2^20)-element NVFP4 record:
    dequantize (32-byte stores), bf16 fused fake-quant, unpack and the
    mismatch diagnostics; rows across the 2^32 boundary against the oracle."""
    cols = 4096
    rows = (2**32 + 2**20) // cols
    g = torch.Generator(device=DEV).manual_seed(10)
    x = torch.randn((rows, cols), generator=g, device=DEV, dtype=torch.bfloat16)
    q = B.tf4_quantize_capture(x)
    cnt = B.tf4_mismatch_stats(x, q)
    assert cnt.tolist() == [0] * B.MISMATCH_COUNTS
    r0 = 2**32 // cols
    sample = (0, r0 - 1, r0, r0 + 1, rows - 1)
    st = host(q.s_t)
    got = {}
    d = B.tf4_dequantize(q)
    got["dequant"] = {r: host(d[r]) for r in sample}
    del d
    y, _ = B.tf4_guided_fake_quant(x, q, out_dtype=torch.bfloat16)
    got["fq"] = {r: host(y[r].view(torch.int16)).view(np.uint16) for r in sample}
    del y
    mant = B.tf4_unpack_guidance(q.bits, rows, cols)
    got["unpack"] = {r: host(mant[r * cols:(r + 1) * cols]) for r in sample}
    del mant
    assert B.read_status(x.device) == 0
    for r in sample:
        xs = W.bf16_bits(x[r:r + 1])
        codes = host(q.codes[r * cols // 2:(r + 1) * cols // 2])
        scales = host(q.scales[r])
        bits = host(q.bits[r * cols // 8:(r + 1) * cols // 8])
        rd = O.dequantize(codes, scales, 1, cols, O.NVFP4, s_t=st)
        assert_same(f"dequant row {r}", f32_bits(got["dequant"][r]), f32_bits(rd))
        _, rv, _ = O.guided_fake_quant(xs, scales, bits, O.NVFP4, rec_s_t=st)
        assert_same(f"fake-quant row {r}", got["fq"][r], O.f32_to_bf16(rv))
        assert_same(f"unpack row {r}", got["unpack"][r], O.unpack_guidance(bits, cols))
    del x, q
    torch.cuda.empty_cache()


def _oracle_row_with_offset(row_bits, base_index, seed):
    """Oracle SR codes of one MXFP4 row whose first element has flat index
    base_index (element-level oracle calls)."""
    cols = len(row_bits)
    out = np.zeros(cols // 2, np.uint8)
    xf = (row_bits.astype(np.uint32) << 16).view(np.float32)
    for b in range(cols // 32):
        blk = row_bits[32 * b:32 * b + 32]
        bamax = float(np.abs(xf[32 * b:32 * b + 32]).max())
        e = O.e8m0_exponent(bamax)
        S = 2.0 ** e
        for k in range(32):
            i = 32 * b + k
            m3 = O.sr_m3(abs(float(xf[i])), S, O.sr_uniform24(base_index + i, seed))
            nib = ((int(blk[k]) >> 15) << 3) | m3
            out[i >> 1] |= nib << (4 * (i & 1))
    return out
