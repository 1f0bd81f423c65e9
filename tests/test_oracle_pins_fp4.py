"""Pins of the oracle's FP4 microscaling formats (MXFP4, NVFP4) against what
the pages and the format definitions fix: E2M1 decoded from its bit layout,
hand-derived ties, E4M3 against torch's float8_e4m3fn, the OCP power-of-two
scale rule, nearest-value searches in exact arithmetic, and the block
structure.  CPU only."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def _e2m1_from_bits(c: int) -> float:
    """E2M1 from its fields: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit;
    exponent field 0 is subnormal (m/2)."""
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
    return -mag if s else mag


def test_e2m1_table_matches_bit_layout_and_page_values():
    vals = [oracle.e2m1_to_f32(c) for c in range(16)]
    assert vals == [_e2m1_from_bits(c) for c in range(16)]
    # arganzheng.life section 九.1: {0, 0.5, 1, 1.5, 2, 3, 4, 6} x +-
    assert sorted({abs(v) for v in vals}) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_e2m1_rounding_ties_and_saturation():
    # midpoints go to the neighbour with mantissa bit 0
    cases = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0,
             0.2499: 0.0, 0.2501: 0.5, 4.99: 4.0, 5.01: 6.0, 6.0: 6.0, 7.9: 6.0, 1e30: 6.0,
             -0.75: -1.0, -5.01: -6.0, -1e30: -6.0}
    for v, want in cases.items():
        assert oracle.e2m1_to_f32(oracle.f32_to_e2m1(v)) == want, v
    assert oracle.f32_to_e2m1(-0.1) == 8          # rounds to -0, sign kept
    assert oracle.f32_to_e2m1(0.1) == 0


def test_e4m3_codec_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).float().numpy()
    ours = np.array([oracle.e4m3_to_f32(c) for c in range(256)], dtype=np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and np.array_equal(ours[~nan], ref[~nan])
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.uniform(0, 448, 3000), 2.0 ** rng.uniform(-12, 8.8, 3000),
                           [2.0 ** -10, 2.0 ** -9 * 1.5, 448.0, 447.9, 232.0, 240.0]]).astype(np.float32)
    vals = vals[vals <= 448]
    t = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.f32_to_e4m3_sat(v) for v in vals], dtype=np.uint8)
    assert np.array_equal(ours, t)
    assert oracle.f32_to_e4m3_sat(1e6) == 0x7E and oracle.e4m3_to_f32(0x7E) == 448.0


def _codes(packed: np.ndarray) -> np.ndarray:
    lo, hi = packed & 0xF, packed >> 4
    return np.stack([lo, hi], axis=-1).reshape(packed.shape[0], -1)


def _nearest_e2m1_ok(t: Fraction, code: int):
    """code is the nearest E2M1 value to the exact quotient t (ties to the
    even magnitude index), or 6 when |t| >= 6."""
    a = abs(t)
    mags = [Fraction(x) for x in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
    m = code & 7
    if a >= 6:
        assert m == 7
        return
    d = abs(a - mags[m])
    for j, x in enumerate(mags):
        dj = abs(a - x)
        assert d < dj or (d == dj and (m & 1) == 0) or j == m, (t, code)
    if t != 0 and m != 0:
        assert (code >> 3) == (1 if t < 0 else 0)


def test_mxfp4_worked_blocks():
    W = np.zeros((1, 96), dtype=np.float32)
    W[0, :4] = [6.0, -3.0, 0.75, 0.2]          # amax 6 -> e = floor(log2 6) - 2 = 0, X = 1
    W[0, 32:34] = [7.9, 1.0]                    # amax 7.9 -> e = 0: 7.9 clips to 6 (OCP rule)
    W[0, 64:66] = [1.0, -0.3]                   # amax 1 -> e = -2, X = 0.25: 4, -1.2 -> -1
    q, s = oracle.mxfp4_quantize(W)
    assert s[0].tolist() == [127, 127, 125]
    c = _codes(q)[0]
    vals = [oracle.e2m1_to_f32(x) for x in c]
    assert vals[:4] == [6.0, -3.0, 1.0, 0.0] and vals[32:34] == [6.0, 1.0]
    assert vals[64:66] == [4.0, -1.0]
    deq = oracle.mxfp4_dequant(q, s)
    assert deq[0, 64] == 1.0 and deq[0, 65] == -0.25 and deq[0, 33] == 1.0


def test_mxfp4_zero_block_and_scale_rule():
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((3, 128)) * np.array([[1e-3], [1.0], [300.0]])).astype(np.float32)
    W[1, 32:64] = 0.0
    q, s = oracle.mxfp4_quantize(W)
    assert s[1, 1] == 0 and not _codes(q)[1, 32:64].any()
    c = _codes(q)
    for r in range(3):
        for b in range(4):
            blk = W[r, 32 * b:32 * b + 32]
            a = np.abs(blk).max()
            if a == 0:
                continue
            m, e = np.frexp(a)                   # a = m 2^e, m in [0.5, 1)
            assert int(s[r, b]) - 127 == (e - 1) - 2
            X = Fraction(2) ** (int(s[r, b]) - 127)
            for k in range(32):
                _nearest_e2m1_ok(Fraction(float(blk[k])) / X, int(c[r, 32 * b + k]))
    deq = oracle.mxfp4_dequant(q, s)
    ref = np.array([[oracle.e2m1_to_f32(x) for x in row] for row in c], dtype=np.float64)
    ref = ref * np.ldexp(1.0, s.astype(np.int64).repeat(32, axis=1) - 127)
    assert np.array_equal(deq.astype(np.float64), ref)


def test_nvfp4_scales_and_codes():
    rng = np.random.default_rng(2)
    W = (rng.standard_normal((4, 64)) * 0.02).astype(np.float32)
    W[2, 5] = 0.9                                 # the tensor maximum
    W[3, 16:32] = 0.0                              # a zero block
    q, s, st = oracle.nvfp4_quantize(W)
    A = float(np.abs(W).max())
    assert st == pytest.approx(A / 2688, rel=1e-7)
    assert s[2, 0] == 0x7E                         # the largest block scale maps to 448
    assert s[3, 1] == 0
    c = _codes(q)
    for r in range(4):
        for b in range(4):
            blk = W[r, 16 * b:16 * b + 16]
            a = np.float32(np.abs(blk).max())
            target = np.float32(np.float32(a / np.float32(6)) / np.float32(st))
            t8 = torch.tensor([min(float(target), 448.0)]).to(torch.float8_e4m3fn).view(torch.uint8)
            assert int(s[r, b]) == int(t8.item())
            S = np.float32(np.float32(oracle.e4m3_to_f32(int(s[r, b]))) * np.float32(st))
            if S == 0:
                assert not c[r, 16 * b:16 * b + 16].any()
                continue
            for k in range(16):
                _nearest_e2m1_ok(Fraction(float(np.float32(blk[k] / S))), int(c[r, 16 * b + k]))
    deq = oracle.nvfp4_dequant(q, s, st)
    err = np.abs(deq - W)
    assert err.max() <= 1.0 * np.abs(W).max() / 6      # at most half the widest E2M1 gap (1 of 6)


def test_fp4_error_ordering_on_gaussian_weights():
    """Smaller blocks and finer scales: NVFP4 (16, E4M3) is more accurate than
    MXFP4 (32, power of two), as the pages state (section 九.1)."""
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((64, 1024)) * 0.02).astype(np.float32)
    q, s = oracle.mxfp4_quantize(W)
    e_mx = np.mean((oracle.mxfp4_dequant(q, s) - W) ** 2)
    q, s, st = oracle.nvfp4_quantize(W)
    e_nv = np.mean((oracle.nvfp4_dequant(q, s, st) - W) ** 2)
    assert e_nv < e_mx


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_fp4_gemm_equals_matmul_of_dequantised(fmt):
    """The W4A4 product equals numpy's matmul of the two dequantised
    operands (fp32 dequantizations, exact here) and, on a weight and an
    activation that are already FP4 grid values, the unquantised product."""
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((24, 96)) * 0.02).astype(np.float32)
    X = rng.standard_normal((3, 96)).astype(np.float32)
    if fmt == "mxfp4":
        wq, ws = oracle.mxfp4_quantize(W)
        xq, xs = oracle.mxfp4_quantize(X)
        wst = xst = None
        Wd, Xd = oracle.mxfp4_dequant(wq, ws), oracle.mxfp4_dequant(xq, xs)
    else:
        wq, ws, wst = oracle.nvfp4_quantize(W)
        xq, xs, xst = oracle.nvfp4_quantize(X)
        Wd, Xd = oracle.nvfp4_dequant(wq, ws, wst), oracle.nvfp4_dequant(xq, xs, xst)
    y = oracle.fp4_gemm(fmt, wq, ws, wst, xq, xs, xst)
    ref = Xd.astype(np.float64) @ Wd.astype(np.float64).T
    # NVFP4's dequantization rounds S_b = e4m3 * s_t to fp32 (relative 2^-24 per
    # term); the product takes the scales exactly
    assert np.allclose(y, ref, rtol=1e-6, atol=1e-6 * np.sqrt(np.mean(ref ** 2)))
    # grid values survive quantization: the product is then the plain one
    G = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -6, -4, -3, -2, -1.5, -1, -0.5, -0.0] * 2,
                 dtype=np.float32)[None, :].repeat(2, 0)
    H = np.roll(G, 5, axis=1)
    if fmt == "mxfp4":
        gq, gs = oracle.mxfp4_quantize(G)
        hq, hs = oracle.mxfp4_quantize(H)
        yg = oracle.fp4_gemm(fmt, gq, gs, None, hq, hs, None)
    else:
        gq, gs, gst = oracle.nvfp4_quantize(G)
        hq, hs, hst = oracle.nvfp4_quantize(H)
        yg = oracle.fp4_gemm(fmt, gq, gs, gst, hq, hs, hst)
    assert np.allclose(yg, H.astype(np.float64) @ G.astype(np.float64).T, rtol=1e-6)


def test_fp4_gemm_hand_block():
    """One MXFP4 block each: w = [6, 1, 0.5, ...0] at scale 2^0, x = [1, -2, 4,
    ...0] at scale 2^-1 -> y = 6*0.5 + 1*(-1) + 0.5*2 = 3."""
    W = np.zeros((1, 32), dtype=np.float32)
    W[0, :3] = [6.0, 1.0, 0.5]
    X = np.zeros((1, 32), dtype=np.float32)
    X[0, :3] = [0.5, -1.0, 2.0]                    # amax 2 -> e = -1, codes 1, -2, 4
    wq, ws = oracle.mxfp4_quantize(W)
    xq, xs = oracle.mxfp4_quantize(X)
    assert ws[0, 0] == 127 and xs[0, 0] == 126
    assert oracle.fp4_gemm("mxfp4", wq, ws, None, xq, xs, None)[0, 0] == 3.0
