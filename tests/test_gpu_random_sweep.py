"""Randomised parity sweep: many small calls with random formats, shapes,
segment splits and value distributions (normal, heavy-tailed, huge / tiny
exponents, exact zeros, repeated values), each compared with the oracle
element by element -- capture (codes, scales, s_t, bits), SR, guided on a
perturbed copy, dequantize and fused fake-quant.  Plus two streams running
calls concurrently with their own workspaces."""
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


def host(t):
    return t.detach().cpu().numpy()


def bits32(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def random_values(rng, rows, cols):
    kind = rng.integers(0, 5)
    if kind == 0:
        v = rng.standard_normal((rows, cols))
    elif kind == 1:
        v = rng.standard_t(2.5, (rows, cols)) * np.exp(rng.standard_normal((1, cols)))
    elif kind == 2:
        v = rng.standard_normal((rows, cols)) * 2.0 ** rng.integers(-120, 120)
    elif kind == 3:
        v = rng.standard_normal((rows, cols))
        v[rng.random((rows, cols)) < 0.3] = 0.0
    else:
        v = rng.choice([-3.0, -0.5, 0.25, 1.0, 6.0, 1e-3], size=(rows, cols)) * 2.0 ** rng.integers(-10, 10)
    return torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("case", range(160))
def test_random_case(case):
    rng = np.random.default_rng(1000 + case)
    fmt = int(rng.choice([O.NVFP4, O.MXFP4, O.UFP4]))
    blk = O.BLOCK[fmt]
    rows = int(rng.integers(1, 300))
    cols = blk * int(rng.integers(1, 40))
    seg = None
    if O.HAS_TENSOR_SCALE[fmt] and rng.random() < 0.6:
        cuts = sorted(int(c) for c in rng.integers(0, rows + 1, size=int(rng.integers(1, 6))))
        seg = [0] + cuts + [rows]
    x = random_values(rng, rows, cols).to(DEV)
    xt = W.perturb(x, 2000 + case, rel=float(rng.choice([1e-3, 0.05])))
    xs, xts = W.bf16_bits(x), W.bf16_bits(xt)

    q = B.tf4_quantize_capture(x, fmt=fmt, seg_off=seg)
    r = O.quantize(xs, fmt, O.RTN, seg_off=seg, bits=True)
    assert np.array_equal(host(q.codes), r["codes"])
    assert np.array_equal(host(q.scales).reshape(-1), r["scales"])
    assert np.array_equal(host(q.bits), r["bits"])
    if O.HAS_TENSOR_SCALE[fmt]:
        assert np.array_equal(bits32(host(q.s_t)), bits32(r["s_t"]))

    seed = int(rng.integers(0, 2**63))
    qs = B.tf4_quantize_sr(x, seed, fmt=fmt, seg_off=seg)
    rs = O.quantize(xs, fmt, O.SR, seg_off=seg, seed=seed)
    assert np.array_equal(host(qs.codes), rs["codes"])

    g = B.tf4_quantize_guided(xt, q)
    rg, _ = O.quantize_guided(xts, r["scales"], r["bits"], fmt, rec_s_t=r["s_t"], seg_off=seg)
    assert np.array_equal(host(g), rg)

    d = B.tf4_dequantize(q)
    rd = O.dequantize(r["codes"], r["scales"], rows, cols, fmt, s_t=r["s_t"], seg_off=seg)
    assert np.array_equal(bits32(host(d)), bits32(rd))

    y, c = B.tf4_guided_fake_quant(xt, q, out_dtype=torch.bfloat16, want_codes=True)
    _, rv, _ = O.guided_fake_quant(xts, r["scales"], r["bits"], fmt, rec_s_t=r["s_t"], seg_off=seg)
    assert np.array_equal(host(c), rg)
    assert np.array_equal(host(y.view(torch.int16)).view(np.uint16).reshape(-1), O.f32_to_bf16(rv).reshape(-1))
    assert B.read_status(x.device) == 0


def test_two_streams_with_their_own_workspaces():
    """Captures issued on two streams at once (each stream gets its own
    workspace) give the results of the same calls made one after another."""
    xs = [W.random_bf16((512, 4096), seed=70 + i, device=DEV, outlier_frac=0.01) for i in range(4)]
    seq = [B.tf4_quantize_capture(x) for x in xs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [None] * len(xs)
    for i, x in enumerate(xs):
        s = streams[i % 2]
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            outs[i] = B.tf4_quantize_capture(x)
    torch.cuda.synchronize()
    for a, b in zip(seq, outs):
        for name in ("codes", "scales", "s_t", "bits"):
            assert torch.equal(getattr(a, name), getattr(b, name)), name
