"""Pins of the oracle's uniform-grid variant (UFP4).

The UFP4 page ("FP4学習の「収縮バイアス」問題を解決するUFP4レシピ", section
"UFP4 の設計と実装指針") replaces E2M1's grid by a uniform 4-bit grid
(E1M2 / INT4).  Read here as magnitudes {0, 1, ..., 7} in NVFP4's container
(16-element blocks, E4M3 block scale, fp32 tensor scale amax / (7 * 448)).
Each test checks the oracle against something other than itself: numpy's
round-half-even, exact rational brute force, torch's E4M3 conversion, a
separate E1M2 restatement, closed forms.  No GPU is needed.
"""
import math
from fractions import Fraction as F

import numpy as np
import pytest
import torch

from fp4_block_scaled_quantizer_b200 import workloads as W

U = [F(k) for k in range(8)]


def all_bf16_finite():
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    return b[(b & 0x7F80) != 0x7F80]


def bf16_to_f32(b):
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32)


def e4m3_torch_decode(code):
    return float(torch.tensor([int(code)], dtype=torch.uint8).view(torch.float8_e4m3fn).float()[0])


def e4m3_torch(v):
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


# -------------------------------------------------- brute force on a grid
def bf_rtn(grid, ax, S):
    y = F(ax) / F(S)
    d = [abs(y - v) for v in grid]
    m = min(d)
    c = [j for j in range(8) if d[j] == m]
    return c[0] if len(c) == 1 else [j for j in c if j % 2 == 0][0]


def bf_neighbours(grid, ax, S):
    y = F(ax) / F(S)
    if y >= grid[7]:
        return 7, 7, True
    if y in grid:
        j = grid.index(y)
        return j, j, True
    lo = max(j for j in range(8) if grid[j] < y)
    return lo, lo + 1, False


def bf_guided(grid, ax, S, g):
    lo, hi, fixed = bf_neighbours(grid, ax, S)
    return lo if fixed or lo % 2 == g else hi


def bf_sr(grid, ax, S, r):
    lo, hi, fixed = bf_neighbours(grid, ax, S)
    if fixed:
        return lo
    y = F(ax) / F(S)
    return hi if F(r) < (1 << 24) * (y - grid[lo]) / (grid[hi] - grid[lo]) else lo


def bf16_around(v, k=2):
    b = int(np.float32(v).view(np.uint32)) >> 16
    out = []
    for d in range(-k, k + 2):
        bb = b + d
        if 0 < bb < 0x7F80:
            out.append(float(bf16_to_f32(np.array([bb], np.uint16))[0]))
    return out


def small_case(rows, cols, seed, outliers=0.01):
    return W.bf16_bits(W.random_bf16((rows, cols), seed=seed, outlier_frac=outliers))


# ------------------------------------------------------------------ tests
def test_uniform_grid_and_guidance_bit(orc):
    """The grid is 0..7 in unit steps, and neighbouring codes always differ
    in their lowest bit (the UFP4 page's grid keeps the guidance rule)."""
    g = [orc.grid_value(orc.UFP4, k) for k in range(8)]
    assert g == [float(k) for k in range(8)]
    assert all(((k & 1) != ((k + 1) & 1)) for k in range(7))


@pytest.mark.parametrize("k", [0, -3, 5, 40, -40])
def test_ufp4_rtn_exhaustive_vs_numpy_rint(orc, k):
    """With S = 2^k the real quotient is |x| * 2^-k exactly; the code must be
    numpy's round-half-even of it, clipped to 7, for every finite bf16."""
    b = all_bf16_finite()
    x = bf16_to_f32(b).astype(np.float64)
    y = np.abs(x) * 2.0 ** (-k)
    want = ((b >> 15).astype(np.uint8) << 3) | np.minimum(np.rint(y), 7).astype(np.uint8)
    S = 2.0 ** k
    got = np.array([(int(bb >> 15) << 3) | orc.rtn_code(orc.UFP4, abs(xx), S) for bb, xx in zip(b, x)],
                   dtype=np.uint8)
    assert np.array_equal(got, want), np.nonzero(got != want)[0][:10]


def test_ufp4_fraction_bruteforce_near_boundaries(orc):
    """Every bf16 value within two ulps of every codeword*S and midpoint*S,
    for many scales S (ties included): RTN, guided and SR equal exact
    rational search on the uniform grid."""
    rng = np.random.default_rng(3)
    scales = [1.0, 0.5, 3.0, 2.0 ** -20, 2.0 ** 30, 1.0 / 7.0, 0.75]
    for _ in range(50):
        scales.append(float(np.float32((1.0 + rng.random()) * 2.0 ** int(rng.integers(-60, 60)))))
    points = [F(2 * j + 1, 2) for j in range(7)] + U[1:]
    n = 0
    for S in scales:
        for p in points:
            for ax in bf16_around(float(p * F(S))):
                assert orc.rtn_code(orc.UFP4, ax, S) == bf_rtn(U, ax, S), (ax, S)
                for g in (0, 1):
                    assert orc.guided_code(orc.UFP4, ax, S, g) == bf_guided(U, ax, S, g), (ax, S, g)
                for r in (0, 1, 1 << 23, (1 << 24) - 1, int(rng.integers(0, 1 << 24))):
                    assert orc.sr_code(orc.UFP4, ax, S, r) == bf_sr(U, ax, S, r), (ax, S, r)
                n += 1
    assert n > 4000


def test_ufp4_rtn_error_bound(orc):
    """Below the grid maximum + 1/2 the nearest code is within half a step."""
    rng = np.random.default_rng(5)
    for _ in range(2000):
        S = float(np.float32((1 + rng.random()) * 2.0 ** int(rng.integers(-20, 20))))
        ax = float(bf16_to_f32(W.bf16_bits(torch.tensor([rng.random() * 7.5 * S]).to(torch.bfloat16)))[0])
        if F(ax) / F(S) > F(15, 2):  # bf16 rounding can step just past 7.5
            continue
        k = orc.rtn_code(orc.UFP4, ax, S)
        assert abs(F(ax) / F(S) - k) <= F(1, 2)


def test_ufp4_scales_vs_numpy_torch(orc):
    """s_t = fl32(amax / 3136) (numpy fp32 division) and every scale byte =
    torch E4M3 of fl32(fl32(bamax / 7) / s_t)."""
    x = small_case(64, 512, seed=5)
    r = orc.quantize(x, orc.UFP4)
    xf = bf16_to_f32(x.reshape(-1)).reshape(x.shape)
    amax = np.float32(np.abs(xf).max())
    assert r["s_t"][0] == np.float32(amax) / np.float32(3136.0)
    bamax = np.abs(xf).reshape(-1, 16).max(axis=1).astype(np.float32)
    q = (bamax / np.float32(7.0)).astype(np.float32)
    assert np.array_equal(r["scales"], e4m3_torch((q / r["s_t"][0]).astype(np.float32)))


def test_ufp4_tensor_max_block_closed_form(orc):
    """The block holding the tensor amax gets r ~ 448 -> scale 0x7E and the
    amax element lands on the top code 7."""
    for seed in range(5):
        x = small_case(32, 256, seed=seed)
        r = orc.quantize(x, orc.UFP4)
        xf = np.abs(bf16_to_f32(x.reshape(-1)))
        i = int(np.argmax(xf))
        assert r["scales"][i // 16] == 0x7E
        assert orc.unpack_codes(r["codes"], x.size)[i] & 7 == 7


def test_ufp4_codes_vs_bruteforce_tensor(orc):
    """Whole-tensor codes equal rational brute force given the oracle's scale
    bytes decoded by torch; dequantized values equal torch's fp32 k * S."""
    x = small_case(16, 128, seed=7, outliers=0.03)
    r = orc.quantize(x, orc.UFP4)
    nib = orc.unpack_codes(r["codes"], x.size)
    xf = bf16_to_f32(x.reshape(-1))
    st = np.float32(r["s_t"][0])
    S_blk = np.array([np.float32(st * np.float32(e4m3_torch_decode(c))) for c in r["scales"]], np.float32)
    for i in range(x.size):
        assert nib[i] & 7 == bf_rtn(U, abs(float(xf[i])), float(S_blk[i // 16]))
        assert nib[i] >> 3 == int(x.reshape(-1)[i]) >> 15
    d = orc.dequantize(r["codes"], r["scales"], 16, 128, orc.UFP4, s_t=r["s_t"]).reshape(-1)
    k = torch.from_numpy((nib & 7).astype(np.float32))
    want = (k * torch.from_numpy(np.repeat(S_blk, 16))).numpy()
    want = np.where(nib & 8, -want, want)
    assert np.array_equal(d.view(np.uint32), want.astype(np.float32).view(np.uint32))


def test_ufp4_e1m2_reading_gives_same_codes(orc):
    """E1M2's grid is {0, 1/4, ..., 7/4}: with its own tensor scale
    amax / (1.75 * 448) and block rule (bamax / 1.75) / s_t, a separate
    restatement here (fp32 numpy arithmetic + rational rounding) gives the
    oracle's codes and scale bytes, and values equal up to the factor 4 in
    s_t -- the two names of the grid agree."""
    x = small_case(8, 128, seed=31, outliers=0.05)
    r = orc.quantize(x, orc.UFP4)
    xf = bf16_to_f32(x.reshape(-1))
    grid = [F(k, 4) for k in range(8)]
    st = np.float32(np.abs(xf).max()) / np.float32(784.0)
    assert st == np.float32(4.0) * r["s_t"][0]
    bamax = np.abs(xf).reshape(-1, 16).max(axis=1).astype(np.float32)
    sc = e4m3_torch(((bamax / np.float32(1.75)).astype(np.float32) / st).astype(np.float32))
    assert np.array_equal(sc, r["scales"])
    nib = orc.unpack_codes(r["codes"], x.size)
    for i in range(x.size):
        S = float(np.float32(st * np.float32(e4m3_torch_decode(sc[i // 16]))))
        assert nib[i] & 7 == bf_rtn(grid, abs(float(xf[i])), S)


@pytest.mark.parametrize("mode", [0, 1])
def test_ufp4_guided_reproduces_rollout(orc, mode):
    """With x' = x the guided codes equal the captured ones (RTN- and
    SR-captured, ragged segments)."""
    x = small_case(40, 256, seed=11, outliers=0.02)
    seg = [0, 7, 7, 30, 40]
    r = orc.quantize(x, orc.UFP4, mode, seg_off=seg, seed=9, bits=True)
    g, st = orc.quantize_guided(x, r["scales"], r["bits"], orc.UFP4, rec_s_t=r["s_t"], seg_off=seg)
    assert st == 0
    assert np.array_equal(g, r["codes"])


def test_ufp4_guided_always_a_neighbour(orc):
    x = small_case(32, 256, seed=13)
    r = orc.quantize(x, orc.UFP4, bits=True)
    xt = W.bf16_bits(W.perturb(W.from_bits(x), seed=2, rel=0.05))
    g, _ = orc.quantize_guided(xt, r["scales"], r["bits"], orc.UFP4, rec_s_t=r["s_t"])
    nib = orc.unpack_codes(g, x.size)
    bits = orc.unpack_guidance(r["bits"], x.size)
    xf = bf16_to_f32(xt.reshape(-1))
    st = np.float32(r["s_t"][0])
    for i in range(0, x.size, 3):
        S = float(np.float32(st * np.float32(e4m3_torch_decode(r["scales"][i // 16]))))
        lo, hi, fixed = bf_neighbours(U, abs(float(xf[i])), S) if S > 0 else (0, 0, True)
        assert nib[i] & 7 in (lo, hi)
        if not fixed:
            assert (nib[i] & 1) == bits[i]


def test_ufp4_sr_unbiased(orc):
    """Rows [A, v, ..., v] share one block scale; the mean of the
    dequantized v converges to v (4 sigma / sqrt(n) + 2^-24 resolution)."""
    n_rows = 1 << 16
    A, v = 5.0, 2.3719
    row = np.array([A] + [v] * 15, dtype=np.float32)
    x = W.bf16_bits(torch.from_numpy(np.tile(row, (n_rows, 1))).to(torch.bfloat16))
    vb = float(bf16_to_f32(x[0, 1:2])[0])
    r = orc.quantize(x, orc.UFP4, orc.SR, seed=77)
    d = orc.dequantize(r["codes"], r["scales"], n_rows, 16, orc.UFP4, s_t=r["s_t"])
    S = float(np.float32(np.float32(r["s_t"][0]) * np.float32(e4m3_torch_decode(r["scales"][0]))))
    lo, hi, _ = bf_neighbours(U, vb, S)
    gap = float(U[hi] - U[lo]) * S
    samples = d[:, 1:].reshape(-1).astype(np.float64)
    bound = 4 * (gap / 2) / math.sqrt(samples.size) + 2.0 ** -24 * gap
    assert abs(samples.mean() - vb) < bound
    assert set(np.unique(samples)) <= {float(np.float32(float(U[lo]) * S)), float(np.float32(float(U[hi]) * S))}


def test_ufp4_zero_segment(orc):
    x = np.zeros((4, 32), np.uint16)
    x[1, 3] = 0x8000
    x[2, 5] = 0x0001  # amax / 3136 underflows -> zero segment
    r = orc.quantize(x, orc.UFP4, bits=True)
    assert r["s_t"][0] == 0.0 and not r["scales"].any()
    nib = orc.unpack_codes(r["codes"], x.size)
    assert nib[35] == 0x8 and np.all(nib[np.arange(x.size) != 35] == 0)
