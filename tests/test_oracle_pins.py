"""Pins of the CPU oracle against things other than itself.

Each test checks one oracle definition against an independent source:
library conversions (ml_dtypes, torch float8), Triton's Philox (run on the
CPU by its interpreter), exact rational brute force, closed forms and
invariants that the pages or the mathematics fix.  No GPU is needed.
"""
import json
import math
import os
import subprocess
import sys
from fractions import Fraction as F

import ml_dtypes
import numpy as np
import pytest
import torch

from fp4_block_scaled_quantizer_b200 import workloads as W

V = [F(0), F(1, 2), F(1), F(3, 2), F(2), F(3), F(4), F(6)]
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def all_bf16_finite():
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    return b[(b & 0x7F80) != 0x7F80]


def bf16_to_f32(b):
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32)


# ------------------------------------------------------- brute-force oracles
def bf_rtn(ax, S):
    y = F(ax) / F(S)
    d = [abs(y - v) for v in V]
    m = min(d)
    c = [j for j in range(8) if d[j] == m]
    return c[0] if len(c) == 1 else [j for j in c if j % 2 == 0][0]


def bf_neighbours(ax, S):
    y = F(ax) / F(S)
    if y >= 6:
        return 7, 7, True
    if y in V:
        j = V.index(y)
        return j, j, True
    lo = max(j for j in range(8) if V[j] < y)
    return lo, lo + 1, False


def bf_guided(ax, S, g):
    lo, hi, fixed = bf_neighbours(ax, S)
    if fixed:
        return lo
    return lo if lo % 2 == g else hi


def bf_sr(ax, S, r):
    lo, hi, fixed = bf_neighbours(ax, S)
    if fixed:
        return lo
    y = F(ax) / F(S)
    return hi if F(r) < (1 << 24) * (y - V[lo]) / (V[hi] - V[lo]) else lo


def bf16_around(v, k=2):
    """bf16 values near the real v: the bf16 just below/above and k ulps on each side."""
    b = int(np.float32(v).view(np.uint32)) >> 16
    out = []
    for d in range(-k, k + 2):
        bb = b + d
        if 0 < bb < 0x7F80:
            out.append(float(bf16_to_f32(np.array([bb], np.uint16))[0]))
    return out


def scales_for_test(rng, n):
    """fp32 scales of many magnitudes: random mantissas, a few powers of two and
    small-integer ratios (which make midpoints exactly bf16-representable)."""
    out = [1.0, 0.5, 2.0 ** -20, 2.0 ** 30, 0.75, 1.25, 3.0, 5.0 / 8.0, 7.0 / 4.0]
    for _ in range(n):
        e = int(rng.integers(-60, 60))
        m = 1.0 + rng.random()
        out.append(float(np.float32(m * 2.0 ** e)))
    return out


# ------------------------------------------------------------------- E2M1
@pytest.mark.parametrize("k", [0, -3, 5, 40, -40])
def test_rtn_exhaustive_bf16_vs_ml_dtypes(orc, k):
    """With S = 2^k the real quotient is x * 2^-k exactly; the oracle's code
    must equal ml_dtypes' float4_e2m1fn conversion (RNE, saturate at 6,
    signed zero) for every finite bf16 pattern."""
    b = all_bf16_finite()
    x = bf16_to_f32(b).astype(np.float64)
    y = x * 2.0 ** (-k)
    keep = np.isfinite(y) & (np.abs(y) < 3e38)
    b, x, y = b[keep], x[keep], y[keep]
    yf = y.astype(np.float32)
    exact = yf.astype(np.float64) == y  # exclude quotients that are not fp32 values
    b, x, yf = b[exact], x[exact], yf[exact]
    want = yf.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    S = 2.0 ** k
    got = np.array([(int(bb >> 15) << 3) | orc.rtn_m3(abs(xx), S) for bb, xx in zip(b, x)], dtype=np.uint8)
    assert np.array_equal(got, want), np.nonzero(got != want)[0][:10]


def test_rtn_guided_sr_fraction_bruteforce_near_boundaries(orc):
    """Exact rational search: for many scales S, every bf16 value within two
    ulps of every codeword*S and midpoint*S (ties included)."""
    rng = np.random.default_rng(1)
    points = [F(1, 4), F(3, 4), F(5, 4), F(7, 4), F(5, 2), F(7, 2), F(5)] + V[1:]
    n = 0
    for S in scales_for_test(rng, 60):
        for p in points:
            for ax in bf16_around(float(p * F(S))):
                assert orc.rtn_m3(ax, S) == bf_rtn(ax, S), (ax, S)
                for g in (0, 1):
                    assert orc.guided_m3(ax, S, g) == bf_guided(ax, S, g), (ax, S, g)
                for r in (0, 1, (1 << 23), (1 << 24) - 1, int(rng.integers(0, 1 << 24))):
                    assert orc.sr_m3(ax, S, r) == bf_sr(ax, S, r), (ax, S, r)
                n += 1
    assert n > 5000


def test_sr_threshold_exact_boundary(orc):
    """r exactly at the threshold 2^24 (y-lo)/(hi-lo) rounds down (strict <)."""
    S = 1.0
    ax = 1.25  # y = 1.25 between 1 and 1.5, fraction 1/2 -> threshold 2^23
    assert orc.sr_m3(ax, S, (1 << 23) - 1) == 3
    assert orc.sr_m3(ax, S, 1 << 23) == 2
    # a value on the grid never moves
    for j in range(8):
        for r in (0, (1 << 24) - 1):
            assert orc.sr_m3(float(V[j]) * 0.375, 0.375, r) == j


# ------------------------------------------------------------------- E4M3
def e4m3_torch(r):
    t = torch.from_numpy(np.asarray(r, np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def e4m3_test_values():
    vals = []
    for e in range(-16, 9):  # fp32 exponents covering E4M3 subnormals .. 448+
        for top in range(16):
            for low in (0, 1, 0x3FFFF, 0x40000, 0x40001, 0x7FFFF):
                bits = ((e + 127) << 23) | (top << 19) | low
                vals.append(np.uint32(bits).view(np.float32))
    for k in range(0, 130):  # the subnormal lattice of E4M3 and its ties
        for d in (-1, 0, 1):
            v = np.float32(k * 2.0 ** -10)
            vals.append(np.nextafter(v, np.float32(np.inf if d > 0 else -np.inf)) if d else v)
    rng = np.random.default_rng(2)
    vals += list(rng.uniform(0, 464, 100000).astype(np.float32))
    vals += list(np.exp2(rng.uniform(-16, np.log2(463.9), 100000)).astype(np.float32))
    v = np.array(vals, dtype=np.float32)
    return v[(v >= 0) & (v < 464)]


def test_e4m3_encode_vs_torch_and_ml_dtypes(orc):
    r = e4m3_test_values()
    want_t = e4m3_torch(r)
    want_m = r.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(want_t, want_m)
    got = np.array([orc.e4m3_encode(float(v)) for v in r], dtype=np.uint8)
    bad = np.nonzero(got != want_t)[0]
    assert bad.size == 0, [(float(r[i]), got[i], want_t[i]) for i in bad[:5]]


def test_e4m3_saturates_above_448(orc):
    for v in (448.0, 463.9, 464.0, 500.0, 1e30):
        assert orc.e4m3_encode(v) == 0x7E


def test_e4m3_decode_vs_torch(orc):
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    got = np.array([orc.e4m3_value(int(c)) for c in codes])
    assert np.array_equal(got.astype(np.float32), want)


# ------------------------------------------------------------------- E8M0
def test_e8m0_exponent_vs_bitfield(orc):
    """floor(log2 x) - 2 read from the bf16 bit field (leading-one position for
    subnormals), clamped to [-127, 127]; checked for every positive finite bf16."""
    b = all_bf16_finite()
    b = b[(b & 0x8000) == 0]
    b = b[b != 0]
    for bb in b:
        e_field = (int(bb) >> 7) & 0xFF
        m = int(bb) & 0x7F
        fl = e_field - 127 if e_field else (-133 + m.bit_length() - 1)
        want = min(max(fl - 2, -127), 127)
        x = float(bf16_to_f32(np.array([bb], np.uint16))[0])
        assert orc.e8m0_exponent(x) == want, hex(bb)
        if want > -127:
            assert 2.0 ** (want + 2) <= x < 2.0 ** (want + 3)
    assert orc.e8m0_exponent(0.0) == -127


# ----------------------------------------------------------------- Philox
_TRITON_PHILOX = r"""
import os, sys, json
os.environ["TRITON_INTERPRET"] = "1"
import numpy as np, torch, triton, triton.language as tl

@triton.jit
def k(out_ptr, lo_ptr, hi_ptr, seed_lo, seed_hi, N: tl.constexpr):
    i = tl.arange(0, N)
    c0 = tl.load(lo_ptr + i)
    c1 = tl.load(hi_ptr + i)
    z = c0 * 0
    seed = (seed_hi.to(tl.uint64) << 32) | seed_lo.to(tl.uint64)
    a, b, c, d = tl.philox(seed, c0, c1, z, z)
    tl.store(out_ptr + i * 4 + 0, a)
    tl.store(out_ptr + i * 4 + 1, b)
    tl.store(out_ptr + i * 4 + 2, c)
    tl.store(out_ptr + i * 4 + 3, d)

req = json.loads(sys.stdin.read())
res = []
for seed in req["seeds"]:
    idx = np.array(req["idx"], dtype=np.uint64)
    lo = torch.from_numpy((idx & 0xFFFFFFFF).astype(np.uint32).view(np.int32))
    hi = torch.from_numpy((idx >> 32).astype(np.uint32).view(np.int32))
    out = torch.zeros(4 * len(idx), dtype=torch.int32)
    k[(1,)](out, lo, hi, seed & 0xFFFFFFFF, seed >> 32, N=len(idx))
    res.append(out.numpy().view(np.uint32).reshape(-1, 4).tolist())
print(json.dumps(res))
"""


def test_philox_vs_triton_interpreter(orc):
    """Philox4x32-10 against Triton's own implementation (a library routine),
    executed on the CPU by Triton's interpreter."""
    rng = np.random.default_rng(3)
    idx = list(range(24)) + [2**32 - 1, 2**32, 2**32 + 5, 2**40 + 123, 2**63 + 7] + [
        int(v) for v in rng.integers(0, 2**63, 3, dtype=np.int64)]
    seeds = [0, 1, 4, 0xDEADBEEF, 2**32 + 7, 2**63 + 12345]
    env = dict(os.environ, TRITON_INTERPRET="1")
    p = subprocess.run([sys.executable, "-c", _TRITON_PHILOX], input=json.dumps(dict(idx=idx, seeds=seeds)),
                       capture_output=True, text=True, env=env, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    res = json.loads(p.stdout.strip().splitlines()[-1])
    for s, rows in zip(seeds, res):
        for i, want in zip(idx, rows):
            got = orc.philox4x32_10([i & 0xFFFFFFFF, i >> 32, 0, 0], [s & 0xFFFFFFFF, s >> 32])
            assert list(map(int, got)) == want, (s, i)
            assert orc.sr_uniform24(i, s) == want[0] >> 8


def test_sr_uniform_chi2(orc):
    """The 24-bit SR uniforms over consecutive element indices are uniform
    (chi-square over 64 bins, 2^16 draws)."""
    n, bins = 1 << 16, 64
    u = np.array([orc.sr_uniform24(i, 4) for i in range(n)], dtype=np.int64)
    h = np.bincount(u >> 18, minlength=bins)
    chi2 = float(((h - n / bins) ** 2 / (n / bins)).sum())
    assert chi2 < 120.0  # df = 63; p(chi2 > 120) ~ 2e-5


# --------------------------------------------------------- tensor level
def small_case(rows=48, cols=256, seed=0, outliers=0.01):
    return W.bf16_bits(W.random_bf16((rows, cols), seed=seed, outlier_frac=outliers))


def test_nvfp4_scales_vs_numpy_torch(orc):
    """s_t = fl32(amax / 2688) (numpy fp32 division) and every block scale
    byte = torch E4M3 of fl32(fl32(bamax / 6) / s_t)."""
    x = small_case(64, 512, seed=5)
    r = orc.quantize(x, orc.NVFP4)
    xf = bf16_to_f32(x.reshape(-1)).reshape(x.shape)
    amax = np.float32(np.abs(xf).max())
    assert r["s_t"][0] == np.float32(amax) / np.float32(2688.0)
    bamax = np.abs(xf).reshape(-1, 16).max(axis=1).astype(np.float32)
    q = (bamax / np.float32(6.0)).astype(np.float32)
    rr = (q / r["s_t"][0]).astype(np.float32)
    assert np.array_equal(r["scales"], e4m3_torch(rr))


def test_tensor_max_block_closed_form(orc):
    """The block holding the tensor amax gets r ~ 448 -> scale 0x7E, and the
    amax element lands on the top codeword 6 (m3 = 7)."""
    for seed in range(5):
        x = small_case(32, 256, seed=seed)
        r = orc.quantize(x, orc.NVFP4)
        xf = np.abs(bf16_to_f32(x.reshape(-1)))
        i = int(np.argmax(xf))
        assert r["scales"][i // 16] == 0x7E
        assert orc.unpack_codes(r["codes"], x.size)[i] & 7 == 7


@pytest.mark.parametrize("fmt", [0, 1])
def test_codes_vs_bruteforce_tensor(orc, fmt):
    """Whole-tensor codes equal Fraction brute force given the oracle's own
    scale bytes (decoded independently: torch E4M3 / powers of two)."""
    x = small_case(16, 128, seed=7)
    r = orc.quantize(x, fmt)
    nib = orc.unpack_codes(r["codes"], x.size)
    xf = bf16_to_f32(x.reshape(-1))
    blk = orc.BLOCK[fmt]
    for i in range(x.size):
        sc = r["scales"][i // blk]
        if fmt == orc.NVFP4:
            S = float(np.float32(r["s_t"][0]) * torch.tensor([sc], dtype=torch.uint8).view(
                torch.float8_e4m3fn).float().numpy()[0])
        else:
            S = 2.0 ** (int(sc) - 127)
        ax = abs(float(xf[i]))
        assert nib[i] & 7 == bf_rtn(ax, S)
        assert nib[i] >> 3 == int(x.reshape(-1)[i]) >> 15


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("mode", [0, 1])
def test_guided_reproduces_rollout_when_inputs_equal(orc, fmt, mode):
    """[TRACE-KO] key idea: the trainer reproduces the rollout's rounding.
    With x' = x, guided codes equal the captured codes bit for bit (RTN- and
    SR-captured), including a ragged multi-segment tensor."""
    x = small_case(40, 256, seed=11, outliers=0.02)
    seg = [0, 7, 7, 30, 40] if fmt == orc.NVFP4 else None
    r = orc.quantize(x, fmt, mode, seg_off=seg, seed=9, bits=True)
    g, st = orc.quantize_guided(x, r["scales"], r["bits"], fmt, rec_s_t=r["s_t"], seg_off=seg)
    assert st == 0
    assert np.array_equal(g, r["codes"])


def test_guided_always_a_neighbour(orc):
    """[TRACE-JA] mechanism: the train side only ever picks one of the two
    adjacent codewords of its own value."""
    x = small_case(32, 256, seed=13)
    r = orc.quantize(x, orc.NVFP4, bits=True)
    xt = W.bf16_bits(W.perturb(W.from_bits(x), seed=2, rel=0.05))
    g, _ = orc.quantize_guided(xt, r["scales"], r["bits"], orc.NVFP4, rec_s_t=r["s_t"])
    nib = orc.unpack_codes(g, x.size)
    bits = orc.unpack_guidance(r["bits"], x.size)
    xf = bf16_to_f32(xt.reshape(-1))
    for i in range(0, x.size, 3):
        S = float(orc.lib().orc_nvfp4_block_scale(int(r["scales"][i // 16]), float(r["s_t"][0])))
        lo, hi, fixed = bf_neighbours(abs(float(xf[i])), S) if S > 0 else (0, 0, True)
        assert nib[i] & 7 in (lo, hi)
        if not fixed:
            assert (nib[i] & 1) == bits[i]


def test_mismatch_example_golden(orc):
    """The pages' mismatch example (tests/golden/mismatch_example.json): two
    nearby values land on different codewords under nearest rounding, and
    guided rounding with the rollout's mantissa bit removes the mismatch.
    The page gives no block scale; S = 1 would send both to 2, so a scale in
    (2.40/2.5, 2.49/2.5] is used (the reading stored in the fixture)."""
    with open(os.path.join(GOLDEN, "mismatch_example.json")) as f:
        ex = json.load(f)
    S = float(np.float32(ex["scale"]))
    ax = [float(bf16_to_f32(W.bf16_bits(torch.tensor([v]).to(torch.bfloat16)))[0]) for v in ex["values"]]
    m = [orc.rtn_m3(a, S) for a in ax]
    assert [float(V[j]) for j in m] == ex["codewords"]
    assert [orc.rtn_m3(a, 1.0) for a in ax] == [4, 4]  # why the literal reading fails
    # rollout recorded the first value's bit; the train side sees the second value
    g = m[0] & 1
    assert float(V[orc.guided_m3(ax[1], S, g)]) == ex["codewords"][0]


def _rows_scaled(rows, cols, seed):
    """N(0,1) rows times 10^(0, -1, ..., -5) in turn, with 2% outliers x50:
    block scales from the E4M3 top down to its subnormals and zero."""
    x = W.random_bf16((rows, cols), seed=seed, outlier_frac=0.02).float()
    x *= torch.tensor([10.0 ** -(r % 6) for r in range(rows)])[:, None]
    x[rows // 2, :32] = 0.0
    return W.bf16_bits(x.to(torch.bfloat16))


@pytest.mark.parametrize("seg", [None, [0, 20, 20, 64]])
def test_nvfp4_dequant_vs_library_decodes(orc, seg):
    """NVFP4 dequantization (TRACE summary, section TRACEの仕組み: the forward
    carries the chosen quantized value): every element equals the numpy fp32
    product of the code's E2M1 value (ml_dtypes' float4_e2m1fn decode, signed)
    and fp32(s_t * E4M3 value) (torch's float8_e4m3fn decode of the scale
    byte, s_t of the row's segment)."""
    rows, cols = 64, 512
    x = _rows_scaled(rows, cols, seed=21)
    r = orc.quantize(x, orc.NVFP4, seg_off=seg)
    assert r["status"] == 0
    d = orc.dequantize(r["codes"], r["scales"], rows, cols, orc.NVFP4, s_t=r["s_t"], seg_off=seg)
    nib = orc.unpack_codes(r["codes"], rows * cols).astype(np.uint8)
    v = nib.view(ml_dtypes.float4_e2m1fn).astype(np.float32).reshape(rows, cols)
    dec = torch.from_numpy(r["scales"].copy()).view(torch.float8_e4m3fn).float().numpy().reshape(rows, -1)
    off = seg if seg is not None else [0, rows]
    row_seg = np.searchsorted(np.asarray(off), np.arange(rows), side="right") - 1
    st = np.asarray(r["s_t"], np.float32)[row_seg]
    S = (st[:, None] * dec).astype(np.float32)                 # one fp32 rounding
    want = (v * np.repeat(S, 16, axis=1)).astype(np.float32)   # one more
    assert (r["scales"] < 8).any() and (r["scales"] == 0).any() and (r["scales"] == 0x7E).any()
    assert np.array_equal(d.view(np.uint32), want.view(np.uint32))


def test_mxfp4_dequant_vs_library_decodes(orc):
    """MXFP4 dequantization: the code's E2M1 value (ml_dtypes) times 2^(byte - 127)."""
    rows, cols = 64, 512
    x = _rows_scaled(rows, cols, seed=22)
    r = orc.quantize(x, orc.MXFP4)
    d = orc.dequantize(r["codes"], r["scales"], rows, cols, orc.MXFP4)
    nib = orc.unpack_codes(r["codes"], rows * cols).astype(np.uint8)
    v = nib.view(ml_dtypes.float4_e2m1fn).astype(np.float64).reshape(rows, cols)
    e = np.repeat(r["scales"].astype(np.int64).reshape(rows, -1) - 127, 32, axis=1)
    want = np.ldexp(v, e).astype(np.float32)                    # exact: a power of two times an E2M1 value
    assert np.array_equal(d.view(np.uint32), want.view(np.uint32))


def test_mxfp4_dequant_quant_idempotent(orc):
    """MXFP4 dequantized values are bf16-representable; re-quantizing them
    gives the same codes and scale bytes, and the same values."""
    x = small_case(24, 256, seed=17, outliers=0.05)
    r = orc.quantize(x, orc.MXFP4)
    d = orc.dequantize(r["codes"], r["scales"], 24, 256, orc.MXFP4)
    xb = W.bf16_bits(torch.from_numpy(d).to(torch.bfloat16))
    assert np.array_equal(bf16_to_f32(xb.reshape(-1)).reshape(d.shape), d)
    r2 = orc.quantize(xb, orc.MXFP4)
    assert np.array_equal(r2["codes"], r["codes"]) and np.array_equal(r2["scales"], r["scales"])


def test_codeword_maps_to_itself(orc):
    rng = np.random.default_rng(4)
    for S in scales_for_test(rng, 40):
        for j in range(8):
            ax = float(V[j]) * S
            if ax == float(np.float32(ax)) and (int(np.float32(ax).view(np.uint32)) & 0xFFFF) == 0:
                assert orc.rtn_m3(ax, S) == j
                assert orc.guided_m3(ax, S, 0) == j and orc.guided_m3(ax, S, 1) == j


def test_sr_unbiased(orc):
    """[FQT] section 3: stochastic rounding removes rounding bias.  Rows
    [A, v, ..., v] share one block scale; the mean of the dequantized v
    converges to v within 4 sigma / sqrt(n) plus the 2^-24 resolution."""
    n_rows = 1 << 16
    A, v = 5.0, 0.8137
    row = np.array([A] + [v] * 15, dtype=np.float32)
    x = W.bf16_bits(torch.from_numpy(np.tile(row, (n_rows, 1))).to(torch.bfloat16))
    vb = float(bf16_to_f32(x[0, 1:2])[0])
    r = orc.quantize(x, orc.NVFP4, orc.SR, seed=123)
    d = orc.dequantize(r["codes"], r["scales"], n_rows, 16, orc.NVFP4, s_t=r["s_t"])
    S = float(orc.lib().orc_nvfp4_block_scale(int(r["scales"][0]), float(r["s_t"][0])))
    lo, hi, _ = bf_neighbours(vb, S)
    gap = float(V[hi] - V[lo]) * S
    samples = d[:, 1:].reshape(-1).astype(np.float64)
    sigma = gap / 2
    bound = 4 * sigma / math.sqrt(samples.size) + 2.0 ** -24 * gap
    assert abs(samples.mean() - vb) < bound
    assert set(np.unique(samples)) <= {float(V[lo]) * S, float(V[hi]) * S}


def test_segments_are_independent(orc):
    """A multi-segment NVFP4 call equals quantizing each segment on its own
    (per-segment tensor scale), including empty segments."""
    x = small_case(50, 128, seed=19, outliers=0.03)
    seg = [0, 0, 13, 13, 14, 50]
    r = orc.quantize(x, orc.NVFP4, seg_off=seg, bits=True)
    codes = orc.unpack_codes(r["codes"], x.size).reshape(50, 128)
    sc = r["scales"].reshape(50, 8)
    for s in range(len(seg) - 1):
        a, b = seg[s], seg[s + 1]
        if a == b:
            assert r["s_t"][s] == 0.0
            continue
        rs = orc.quantize(x[a:b], orc.NVFP4, bits=True)
        assert rs["s_t"][0] == r["s_t"][s]
        assert np.array_equal(orc.unpack_codes(rs["codes"], (b - a) * 128), codes[a:b].reshape(-1))
        assert np.array_equal(rs["scales"], sc[a:b].reshape(-1))


def test_zero_and_tiny_segments(orc):
    x = np.zeros((4, 32), np.uint16)
    x[1, 3] = 0x8000  # -0.0
    x[2, 5] = 0x0001  # smallest bf16 subnormal: amax/2688 underflows -> zero segment
    r = orc.quantize(x, orc.NVFP4, bits=True)
    assert r["s_t"][0] == 0.0 and not r["scales"].any()
    nib = orc.unpack_codes(r["codes"], x.size)
    assert nib[1 * 32 + 3] == 0x8 and np.all(nib[np.arange(x.size) != 35] == 0)
    rm = orc.quantize(x, orc.MXFP4)
    assert rm["scales"][0] == 0  # all-zero block -> exponent -127


def test_nonfinite_flagged_per_segment(orc):
    x = small_case(20, 64, seed=23)
    x[12, 5] = 0x7F80  # +inf in segment 1
    seg = [0, 10, 20]
    r = orc.quantize(x, orc.NVFP4, seg_off=seg)
    assert r["status"] & orc.NONFINITE
    ok = orc.quantize(x[:10], orc.NVFP4)
    assert np.array_equal(r["codes"][: 10 * 64 // 2], ok["codes"])
    x2 = small_case(4, 64, seed=1)
    x2[0, 0] = 0x7FC1  # NaN
    assert orc.quantize(x2, orc.MXFP4)["status"] & orc.NONFINITE
    _, st = orc.quantize_guided(x2, np.zeros(8, np.uint8), np.zeros(32, np.uint8), orc.MXFP4)
    assert st & orc.NONFINITE


def test_guidance_bit_layout_and_roundtrip(orc):
    """bit (i & 7) of byte (i >> 3) holds m3_i & 1; unpack(pack(c)) = m3 & 1."""
    x = small_case(8, 64, seed=29)
    r = orc.quantize(x, orc.NVFP4, bits=True)
    nib = orc.unpack_codes(r["codes"], x.size)
    want = np.packbits((nib & 1).astype(np.uint8), bitorder="little")
    assert np.array_equal(r["bits"], want)
    assert np.array_equal(orc.pack_guidance(r["codes"], x.size), want)
    assert np.array_equal(orc.unpack_guidance(want, x.size), nib & 1)


def test_retained_information_one_sixth():
    """[TRACE-JA] quantization-info cache: keeping the mantissa bit and the
    block scale, for the deeper half of the layers, retains about 1/6 of the
    full quantization information.  NVFP4: full = 4 + 8/16 bits per element,
    compact = 1 + 8/16; 20 of 40 layers -> exactly 1/6."""
    with open(os.path.join(GOLDEN, "retained_info.json")) as f:
        g = json.load(f)
    full = F(4) + F(8, 16)
    compact = F(1) + F(8, 16)
    ratio = compact / full * F(g["layers_kept"], g["layers_total"])
    assert ratio == F(1, 6) == F(g["retained_fraction"])
    # the closed form generalises: MXFP4 with a 32-block
    mx = (F(1) + F(8, 32)) / (F(4) + F(8, 32)) * F(1, 2)
    assert abs(float(mx) - 0.147) < 1e-3


def test_f32_to_bf16_vs_torch(orc):
    """The bf16 output rounding (RNE of the fp32 value) against torch's
    fp32 -> bf16 conversion, on random values and around every tie."""
    rng = np.random.default_rng(9)
    v = np.concatenate([rng.standard_normal(200000).astype(np.float32) * np.float32(1e3),
                        (np.arange(1 << 16, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
                        (np.arange(1 << 16, dtype=np.uint32) << 16 | 0x7FFF).view(np.float32),
                        (np.arange(1 << 16, dtype=np.uint32) << 16 | 0x8001).view(np.float32)])
    v = v[np.isfinite(v) & (np.abs(v) < 3e38)]
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.f32_to_bf16(v), want)


def test_mismatch_stats_closed_form(orc):
    """Mismatch counts on constructed cases: identical inputs -> all zero; a
    train value moved across one midpoint -> one adjacent mismatch that
    guidance removes; moved across two codewords -> one far mismatch."""
    x = np.zeros((1, 32), np.uint16)
    vals = np.array([4.0, 2.4, 1.0, 0.3] + [0.0] * 28, np.float32)
    x[0] = W.bf16_bits(torch.from_numpy(vals).to(torch.bfloat16).reshape(1, 32))[0]
    r = orc.quantize(x, orc.MXFP4, bits=True)  # block max 4 -> S = 1
    assert orc.mismatch_stats(x, r["scales"], r["codes"], orc.MXFP4).tolist() == [0] * 6
    xt = x.copy()
    vt = vals.copy()
    vt[1] = 2.6   # 2.4 -> 2 (rollout), 2.6 -> 3: adjacent; the rollout's codeword is the smaller
    vt[2] = 1.9   # 1.0 -> 1, 1.9 -> 2: two codewords apart (1 -> 1.5 -> 2); smaller
    vt[3] = 0.2   # 0.3 -> 0.5, 0.2 -> 0: adjacent; the rollout's codeword is the larger
    xt[0] = W.bf16_bits(torch.from_numpy(vt).to(torch.bfloat16).reshape(1, 32))[0]
    st = orc.mismatch_stats(xt, r["scales"], r["codes"], orc.MXFP4)
    assert st.tolist() == [3, 2, 1, 1, 2, 1]


def _torch_to_blocked():
    """torch's rearrangement helper, taken from its testing module by
    compiling just that function (the module itself needs packages this
    image lacks)."""
    import ast
    import torch.testing._internal as ti
    path = os.path.join(os.path.dirname(ti.__file__), "common_quantized.py")
    tree = ast.parse(open(path).read())
    keep = [n for n in tree.body if isinstance(n, ast.FunctionDef) and n.name in ("to_blocked", "ceil_div")]
    ns = {"torch": torch, "math": math}
    exec(compile(ast.Module(body=keep, type_ignores=[]), path, "exec"), ns)
    if "ceil_div" not in ns:
        ns["ceil_div"] = lambda a, b: (a + b - 1) // b
    return ns["to_blocked"]


def test_swizzled_scales_vs_torch_to_blocked(orc):
    """The tiled scale layout of block-scaled GEMMs: the oracle's index map
    against torch's own rearrangement helper (an independent implementation
    of the same documented layout), with ragged row and column counts."""
    to_blocked = _torch_to_blocked()
    rng = np.random.default_rng(21)
    for rows, nb in [(1, 1), (128, 4), (130, 5), (300, 64), (77, 3), (256, 896)]:
        sc = rng.integers(1, 255, size=(rows, nb), dtype=np.uint8)
        want = to_blocked(torch.from_numpy(sc)).reshape(-1).numpy()
        got = orc.swizzle_scales(sc)
        assert got.shape == want.shape and np.array_equal(got, want), (rows, nb)
        assert np.count_nonzero(got) == rows * nb  # a permutation of the entries, zero padding
