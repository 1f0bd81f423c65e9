"""Pins of the oracle's per-channel INT8 weight quantizer, its W8A16 product
and the INT8 / INT4 KV-cache quantizers against what the pages and the
mathematics fix: hand-worked rows, exact rational nearest-code searches,
invariants of the scale, and library routines (numpy's IEEE binary16 and
binary32 arithmetic, torch's bfloat16 conversion, numpy matmul).  CPU only.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def _nearest_codes_ok(w: np.ndarray, s: float, codes: np.ndarray, lo: int, hi: int):
    """codes[i] is the integer in [lo, hi] nearest to w[i] / s in exact
    arithmetic, ties to even; where the exact quotient lies within 2^-16 of a
    half-integer either neighbour is accepted (the fp32 quotient the method
    rounds may fall on either side)."""
    S = Fraction(float(s))
    for wi, c in zip(w.tolist(), codes.tolist()):
        t = Fraction(float(wi)) / S
        ideal = max(lo, min(hi, round(t)))   # round(Fraction): half to even
        if c == ideal:
            continue
        frac = abs(t - int(t))
        near_tie = abs(frac - Fraction(1, 2)) < Fraction(1, 65536)
        assert near_tie and abs(c - t) <= Fraction(1, 2) + Fraction(1, 65536), (wi, s, c, ideal)


# ------------------------------------------------------ INT8 weights

def test_q8_worked_row_scale_one():
    """max |w| = 127 makes the scale exactly 1, so the codes are the values
    rounded half to even (charles2530.github.io section 13, torch.round)."""
    w = np.array([[127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, -127.0, 126.5, 100.49, -3.5, 0.0]],
                 dtype=np.float32)
    q, s = oracle.q8_quantize_per_channel(w)
    assert s[0] == 1.0
    assert q[0].tolist() == [127, 2, 4, -2, 0, 0, 2, -127, 126, 100, -4, 0]


def test_q8_eps_floor():
    """clamp_min(1e-6): a zero row gets scale 1e-6/127 and codes 0; a row of
    amax 1e-7 is quantized on that floor scale, not on its own."""
    w = np.zeros((2, 16), dtype=np.float32)
    w[1, 0] = 1e-7
    w[1, 1] = -5e-8
    q, s = oracle.q8_quantize_per_channel(w)
    assert s[0] == s[1] == pytest.approx(7.874015748e-9, rel=1e-7)
    assert not q[0].any()
    assert q[1, 0] == 13 and q[1, 1] == -6 and not q[1, 2:].any()  # 12.7 -> 13, -6.35 -> -6


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_q8_codes_are_nearest_and_max_maps_to_127(seed):
    rng = np.random.default_rng(seed)
    mags = np.array([1e-3, 0.02, 1.0, 37.0])
    w = (rng.standard_normal((4, 96)) * mags[:, None]).astype(np.float32)
    q, s = oracle.q8_quantize_per_channel(w)
    for r in range(4):
        _nearest_codes_ok(w[r], float(s[r]), q[r], -127, 127)
        amax = np.abs(w[r]).max()
        j = int(np.abs(w[r]).argmax())
        assert abs(int(q[r, j])) == 127 and np.abs(q[r]).max() == 127
        # s * 127 reproduces amax to one fp32 rounding
        assert abs(float(s[r]) * 127 - amax) <= np.spacing(np.float32(amax)) * 1.0
        err = np.abs(w[r].astype(np.float64) - q[r] * np.float64(s[r]))
        assert err.max() <= float(s[r]) / 2 * (1 + 1e-6)


def test_q8_dequant_is_one_fp32_product():
    rng = np.random.default_rng(3)
    w = rng.standard_normal((5, 48)).astype(np.float32)
    q, s = oracle.q8_quantize_per_channel(w)
    got = oracle.q8_dequant(q, s)
    assert np.array_equal(got, q.astype(np.float32) * s[:, None])   # numpy IEEE fp32


@pytest.mark.parametrize("B", [1, 3, 8])
def test_q8_gemv_equals_matmul_of_dequantised(B):
    rng = np.random.default_rng(B)
    w = rng.standard_normal((33, 160)).astype(np.float32)
    q, s = oracle.q8_quantize_per_channel(w)
    x = torch.randn(B, 160, generator=torch.Generator().manual_seed(B)).to(torch.bfloat16)
    xf = x.float().numpy().astype(np.float64)
    ref = xf @ (q.astype(np.float64) * s.astype(np.float64)[:, None]).T
    got = oracle.q8_gemv(q, s, xf)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)
    rows = np.array([32, 0, 7])
    assert np.array_equal(oracle.q8_gemv(q, s, xf, rows), got[:, rows])


# ------------------------------------------------------- INT8 KV cache

def test_kv8_worked_token_fp16():
    """One fp16 token: amax 2, s = fp16(2/127) = 0.0157470703125 (0x2408);
    the codes are x / s rounded: 127.008, 63.504, 31.752, 15.876, 95.256."""
    kv = np.array([[[[2.0, -2.0, 1.0, 0.0, 0.5, -1.0, 0.25, 1.5]]]], dtype=np.float32)
    codes, scales = oracle.kv_quantize_int8(kv, False)
    assert scales.shape == (1, 1, 1) and int(scales[0, 0, 0]) == 0x2408
    assert codes[0, 0, 0].tolist() == [127, -127, 64, 0, 32, -64, 16, 95]
    deq = oracle.kv_dequant_int8(codes, scales, False).view(np.float16).astype(np.float64)
    # 64 * 0.0157470703125 = 1.0078125, 95 * s = 1.4959716796875 -> fp16 1.49609375
    assert deq[0, 0, 0, 2] == 1.0078125 and deq[0, 0, 0, 7] == 1.49609375


def _bf16_value(bits: int) -> float:
    t = torch.tensor([bits & 0xFFFF], dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    return float(t.float().item())


@pytest.mark.parametrize("is_bf16", [False, True])
def test_kv8_scale_is_nearest_cache_value_and_codes_nearest(is_bf16):
    rng = np.random.default_rng(11 + is_bf16)
    # rows with a large spread of magnitudes (attention-sink tokens)
    kv = (rng.standard_normal((2, 3, 5, 64)) * rng.choice([0.01, 1.0, 30.0], (2, 3, 5, 1)))
    if is_bf16:
        kv = torch.from_numpy(kv.astype(np.float32)).to(torch.bfloat16).float().numpy()
    else:
        kv = kv.astype(np.float16).astype(np.float32)
    codes, scales = oracle.kv_quantize_int8(kv, is_bf16)
    flat = kv.reshape(-1, 64)
    c2 = codes.reshape(-1, 64)
    for r in range(flat.shape[0]):
        target = Fraction(float(np.abs(flat[r]).max())) / 127
        bits = int(scales.ravel()[r])
        if is_bf16:   # positive values: adjacent bit patterns are the neighbours
            s, lo, hi = _bf16_value(bits), _bf16_value(bits - 1), _bf16_value(bits + 1)
        else:
            s = float(np.uint16(bits).view(np.float16))
            lo = float(np.nextafter(np.float16(s), np.float16(-np.inf)))
            hi = float(np.nextafter(np.float16(s), np.float16(np.inf)))
        # no neighbour of the stored scale is nearer to amax / 127
        assert abs(Fraction(s) - target) <= abs(Fraction(lo) - target)
        assert abs(Fraction(s) - target) <= abs(Fraction(hi) - target)
        _nearest_codes_ok(flat[r], s, c2[r], -128, 127)


@pytest.mark.parametrize("is_bf16", [False, True])
def test_kv8_dequant_matches_library_rounding(is_bf16):
    rng = np.random.default_rng(5)
    kv = (rng.standard_normal((1, 2, 7, 32)) * 3).astype(np.float16).astype(np.float32)
    codes, scales = oracle.kv_quantize_int8(kv, is_bf16)
    deq = oracle.kv_dequant_int8(codes, scales, is_bf16)
    if is_bf16:
        s = torch.from_numpy(scales.astype(np.int32)).to(torch.int16).view(torch.bfloat16)
        ref = (torch.from_numpy(codes).float() * s.float()[..., None]).to(torch.bfloat16)
        assert np.array_equal(deq, ref.view(torch.int16).numpy().view(np.uint16))
    else:
        s = scales.view(np.float16).astype(np.float32)
        ref = (codes.astype(np.float32) * s[..., None]).astype(np.float16)
        assert np.array_equal(deq, ref.view(np.uint16))


def test_kv8_zero_token():
    kv = np.zeros((1, 1, 2, 16), dtype=np.float32)
    kv[0, 0, 1, 3] = 0.75
    codes, scales = oracle.kv_quantize_int8(kv, False)
    assert int(scales[0, 0, 0]) == 0 and not codes[0, 0, 0].any()
    assert codes[0, 0, 1, 3] == 127
    assert not oracle.kv_dequant_int8(codes, scales, False)[0, 0, 0].any()


# ------------------------------------------------------- INT4 KV cache

def test_kv4_is_the_group_quantizer_per_token():
    """Each (batch, head, token) row of head_dim values is quantized on its
    own, in groups of group_size along head_dim ("压缩算法" section 7.4.1.2)."""
    rng = np.random.default_rng(9)
    kv = rng.standard_normal((2, 2, 3, 64)).astype(np.float16).astype(np.float32)
    kv[1, 0, 2, 32:] = 0.0        # an all-zero group beside a live one
    packed, scales = oracle.kv_quantize_int4(kv, 32)
    assert packed.shape == (2, 2, 3, 32) and scales.shape == (2, 2, 3, 2)
    for b in range(2):
        for h in range(2):
            for t in range(3):
                q1, s1, _ = oracle.quantize_pack(kv[b, h, t][None, :], 32, True)
                assert np.array_equal(packed[b, h, t], q1[0]) and np.array_equal(scales[b, h, t], s1[0])
    assert scales[1, 0, 2, 1] == 0 and not packed[1, 0, 2, 16:].any() and scales[1, 0, 2, 0] != 0
    # the largest magnitude of every live group takes code +-7
    for row, srow, prow in zip(kv.reshape(-1, 64), scales.reshape(-1, 2), packed.reshape(-1, 32)):
        for g in range(2):
            if srow[g] == 0:
                continue
            j = g * 32 + int(np.abs(row[g * 32:(g + 1) * 32]).argmax())
            nib = (int(prow[j // 2]) >> (4 * (j % 2))) & 0xF
            code = nib - 16 if nib >= 8 else nib
            assert abs(code) == 7
