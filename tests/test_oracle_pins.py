"""Pins of the CPU oracle against what the pages and the mathematics fix.

Every function of ``oracle/`` is checked here against something other than
itself: values printed by the pages (``tests/golden``), exact rational
arithmetic on small inputs, closed-form statistics of uniform quantization,
invariants, and library routines (numpy's IEEE binary16 conversion, torch's
bfloat16 conversion, numpy matmul).  These run on the CPU only.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_group_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _f16(values) -> np.ndarray:
    """fp32 array holding the fp16-rounded values (numpy's IEEE conversion)."""
    return np.asarray(values, dtype=np.float16).astype(np.float32)


# ----------------------------------------------------------------- codecs

def test_f16_decode_exhaustive_vs_numpy():
    bits = np.arange(65536, dtype=np.uint16)
    ours = oracle.f16_bits_to_f32_array(bits)
    ref = bits.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f16_encode_vs_numpy():
    rng = np.random.default_rng(0)
    # every binary16 value, the midpoints between neighbours (ties), points
    # just beside them, and random fp32 bit patterns over the whole range
    h = np.arange(0, 0x7C00, dtype=np.uint16)
    vals = h.view(np.float16).astype(np.float64)
    mids = (vals[:-1] + vals[1:]) / 2.0                   # exact in fp32
    mids32 = mids.astype(np.float32)
    near = np.concatenate([np.nextafter(mids32, np.float32(np.inf)),
                           np.nextafter(mids32, np.float32(-np.inf))])
    rnd = rng.integers(0, 2**32, size=2_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    rnd = rnd[np.isfinite(rnd)]
    big = np.array([65504.0, 65519.99, 65520.0, 1e6, 5.96e-8, 2.98e-8, 2.99e-8, 1e-9, 0.0],
                   dtype=np.float32)
    allv = np.concatenate([vals.astype(np.float32), mids32, near, rnd, big])
    allv = np.concatenate([allv, -allv])
    ours = oracle.f32_to_f16_bits_array(allv)
    with np.errstate(over="ignore"):
        ref = allv.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_codecs_vs_torch():
    rng = np.random.default_rng(1)
    rnd = rng.integers(0, 2**32, size=1_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    rnd = rnd[np.isfinite(rnd)]
    ties = (np.arange(1, 20000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    allv = np.concatenate([rnd, ties, -ties])
    ours = oracle.f32_to_bf16_bits_array(allv)
    ref = torch.from_numpy(allv).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    b = np.arange(65536, dtype=np.uint16)
    dec = oracle.bf16_bits_to_f32_array(b)
    tref = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).float().numpy()
    nan = np.isnan(tref)
    assert np.array_equal(np.isnan(dec), nan)
    assert np.array_equal(dec[~nan].view(np.uint32), tref[~nan].view(np.uint32))


# ------------------------------------------------- worked examples (golden)

def test_rounding_and_clipping_examples():
    g = _golden("rounding_example.json")
    r = g["rounding"]
    q = oracle.quantize_value(r["w"], r["scale"], r["zero_point"], -(2**20), 2**20)
    assert q == r["q"]
    deq = np.float32(q) * np.float32(r["scale"])
    assert abs(float(deq) - r["dequant"]) < 1e-6
    assert abs(abs(r["w"] - float(deq)) - r["abs_error"]) < 1e-5
    c = g["clipping"]
    q = oracle.quantize_value(c["w"], c["scale"], c["zero_point"], c["qmin"], c["qmax"])
    assert q == c["q"]
    assert abs(c["w"] - q * c["scale"]) == c["abs_error"]


def test_int4_worked_row_rtn_and_awq():
    g = _golden("int4_rtn_row.json")
    x = np.asarray(g["x"], dtype=np.float64)
    w = np.asarray(g["w"], dtype=np.float64)
    assert abs(float(w @ x) - g["y"]) < 1e-9
    for key in ("rtn", "awq"):
        row = g[key]
        cs = np.asarray(row["channel_scale"], dtype=np.float64)
        W = _f16((w * cs)[None, :])
        q, s, z = oracle.quantize_pack(W, g["group_size"], True)
        assert z is None
        codes = [oracle.code_at(q, 4, 0, k, True) for k in range(4)]
        assert codes == row["codes"], key
        # packed layout: even element in the low nibble
        expect_bytes = [(row["codes"][0] & 0xF) | ((row["codes"][1] & 0xF) << 4),
                        (row["codes"][2] & 0xF) | ((row["codes"][3] & 0xF) << 4)]
        assert q[0].tolist() == expect_bytes
        W_hat = oracle.dequant(q, s, z, 1, 4, 4, True)[0].astype(np.float64)
        assert np.max(np.abs(W_hat - np.asarray(row["dequant"]))) < 5e-4, key
        xs = x / cs
        y_hat = oracle.gemv(q, s, z, 1, 4, 4, True, xs[None, :])[0, 0]
        assert abs(y_hat - row["y_hat"]) < 6e-4, key
        rel = abs(W_hat[1] - (w * cs)[1]) / (w * cs)[1]
        assert abs(rel - row["rel_error_w2"]) < 2e-3, key


# ----------------------------------------- exact nearest-grid (brute force)

def _nearest_grid_codes(w32: np.ndarray, sf: float, z: int, qmin: int, qmax: int):
    """Exact rational nearest grid point, ties to an even (code - z)."""
    S = Fraction(float(sf))
    out = []
    for v in w32.tolist():
        t = Fraction(v) / S
        fl = t.numerator // t.denominator
        frac = t - fl
        if frac > Fraction(1, 2):
            m = fl + 1
        elif frac < Fraction(1, 2):
            m = fl
        else:
            m = fl if fl % 2 == 0 else fl + 1
        out.append(min(max(m + z, qmin), qmax))
    return out


@pytest.mark.parametrize("symmetric", [True, False])
@pytest.mark.parametrize("seed", [1, 2, 3])
def test_codes_are_exact_nearest_grid_tiny(symmetric, seed):
    # the 4x8 group-4 case plus a 6x32 group-8 case with mixed signs / scales
    for out, inn, g in ((4, 8, 4), (6, 32, 8)):
        W = wl.normal_weight(out, inn, seed).float().numpy()
        W[0, :g] *= 40.0                    # one loud group
        W[1, g:2 * g] = np.abs(W[1, g:2 * g])  # one all-positive group
        W = _f16(W)
        q, s, z = oracle.quantize_pack(W, g, symmetric)
        for r in range(out):
            for j in range(inn // g):
                sf = float(oracle.f16_to_f32(int(s[r, j])))
                zz = 0 if symmetric else int(oracle.f16_to_f32(int(z[r, j])))
                qmin, qmax = (-8, 7) if symmetric else (0, 15)
                grp = W[r, j * g:(j + 1) * g]
                got = [oracle.code_at(q, inn, r, j * g + k, symmetric) for k in range(g)]
                if sf == 0.0:
                    assert got == [0] * g
                    continue
                assert got == _nearest_grid_codes(grp, sf, zz, qmin, qmax)


@pytest.mark.parametrize("scale_bits", [0x2C5A, 0x1F00, 0x3C00, 0x0003])
def test_rounding_window_exhaustive(scale_bits):
    """All fp16 values in [-8.6 s, 8.6 s] at a fixed fp16 scale: the fp32
    division + round-half-even step equals exact rational rounding."""
    sf = float(oracle.f16_to_f32(scale_bits))
    allh = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    win = allh[allh <= 8.6 * sf]
    win = np.concatenate([win, -win])
    got = [oracle.quantize_value(float(v), sf, 0, -8, 7) for v in win.tolist()]
    assert got == _nearest_grid_codes(win, sf, 0, -8, 7)


# ------------------------------------------------------- scale / zero rule

@pytest.mark.parametrize("g", [32, 64, 128])
def test_symmetric_scale_is_amax_over_7(g):
    W = _f16(wl.student_t_weight(64, 1024, 5).float().numpy())
    q, s, _ = oracle.quantize_pack(W, g, True)
    sf = oracle.f16_bits_to_f32_array(s).astype(np.float64)
    amax = np.abs(W.reshape(64, -1, g)).max(-1).astype(np.float64)
    # stored fp16 scale within fp16 rounding (2^-11 relative) of amax / 7
    assert np.all(np.abs(sf * 7 - amax) <= amax * 2.0 ** -11 * 1.0001)
    # the group maximum gets code +-7; -8 is never produced
    codes = np.array([[oracle.code_at(q, 1024, r, k, True) for k in range(1024)] for r in range(64)])
    assert codes.min() >= -7 and codes.max() <= 7
    grp_codes = np.abs(codes.reshape(64, -1, g)).max(-1)
    assert np.all(grp_codes == 7)


@pytest.mark.parametrize("g", [32, 64, 128])
def test_asymmetric_scale_and_zero_point(g):
    W = _f16(wl.normal_weight(64, 1024, 6).float().numpy() + 0.004)
    q, s, z = oracle.quantize_pack(W, g, False)
    sf = oracle.f16_bits_to_f32_array(s).astype(np.float64)
    zf = oracle.f16_bits_to_f32_array(z).astype(np.float64)
    grp = W.reshape(64, -1, g).astype(np.float64)
    mn, mx = grp.min(-1), grp.max(-1)
    rng_ = mx - mn
    assert np.all(np.abs(sf * 15 - rng_) <= rng_ * 2.0 ** -11 * 1.0001)
    assert np.all((zf >= 0) & (zf <= 15) & (zf == np.round(zf)))
    # z is the code of real zero: -z*s is the grid point nearest the minimum
    inside = mn <= 0
    assert np.all(np.abs(-zf * sf - mn)[inside] <= sf[inside] / 2 * 1.0001)
    codes = np.array([[oracle.code_at(q, 1024, r, k, False) for k in range(1024)]
                      for r in range(64)]).reshape(64, -1, g)
    assert codes.min() >= 0 and codes.max() <= 15
    # min maps to code 0, max to 15 (or 14 by rounding of s and z)
    assert np.all(codes.min(-1) == 0)
    assert np.all(codes.max(-1) >= 14)


def test_degenerate_groups():
    W = np.zeros((2, 64), dtype=np.float32)
    W[1, :32] = _f16(np.full(32, 0.5))          # constant group
    for sym in (True, False):
        q, s, z = oracle.quantize_pack(W, 32, sym)
        assert s[0].tolist() == [0, 0] and not q[0].any()
        W_hat = oracle.dequant(q, s, z, 2, 64, 32, sym)
        assert not W_hat[0].any()
    q, s, _ = oracle.quantize_pack(W, 32, True)
    assert [oracle.code_at(q, 64, 1, k, True) for k in range(32)] == [7] * 32
    assert np.allclose(oracle.dequant(q, s, None, 2, 64, 32, True)[1, :32], 0.5, rtol=2.0 ** -11)


# -------------------------------------------------- dequant: grid + error

@pytest.mark.parametrize("symmetric", [True, False])
@pytest.mark.parametrize("g", [32, 128])
def test_dequant_is_grid_point_within_half_step(symmetric, g):
    W = _f16(wl.normal_weight(128, 2048, 7).float().numpy())
    q, s, z = oracle.quantize_pack(W, g, symmetric)
    W_hat = oracle.dequant(q, s, z, 128, 2048, g, symmetric).astype(np.float64)
    sf = np.repeat(oracle.f16_bits_to_f32_array(s).astype(np.float64), g, axis=1)
    zf = 0.0 if symmetric else np.repeat(oracle.f16_bits_to_f32_array(z).astype(np.float64), g, axis=1)
    idx = W_hat / sf + zf
    assert np.all(idx == np.round(idx))
    lo, hi = (-8, 7) if symmetric else (0, 15)
    assert idx.min() >= lo and idx.max() <= hi
    err = np.abs(W_hat - W.astype(np.float64))
    # interior codes: nearest grid point, error <= s/2.  Codes at the ends of
    # the range may be clipped: asymmetric groups round z, which shifts the
    # grid by up to s/2, so the min / max can sit up to s beyond it.
    interior = (idx > lo) & (idx < hi)
    assert np.all(err[interior] <= (sf / 2 * (1 + 2.0 ** -10))[interior])
    assert np.all(err <= sf * (1 + 2.0 ** -10))
    if symmetric:
        assert np.all(err <= sf / 2 * (1 + 2.0 ** -10))


# ----------------------------------------------- uniform-noise statistics

@pytest.mark.parametrize("dist", ["normal", "uniform"])
@pytest.mark.parametrize("g", [32, 64, 128, 512])
def test_noise_law_delta_squared_over_12(dist, g):
    """E[e^2] = Delta^2/12 per group (arganzheng.life, section 三.1).

    Symmetric groups hold one exact element (the max maps to +-7 exactly), so
    the expected MSE is (1 - 1/g) * mean(s^2)/12."""
    gen = wl.normal_weight if dist == "normal" else wl.uniform_weight
    W = _f16(gen(1024, 4096, 11).float().numpy())
    for sym in (True, False):
        q, s, z = oracle.quantize_pack(W, g, sym)
        W_hat = oracle.dequant(q, s, z, 1024, 4096, g, sym)
        mse = float(np.mean((W_hat.astype(np.float64) - W) ** 2))
        pred = float(np.mean(oracle.f16_bits_to_f32_array(s).astype(np.float64) ** 2) / 12)
        if sym:
            assert abs(mse / (pred * (1 - 1 / g)) - 1) < 0.01, (sym, g)
        else:
            assert abs(mse / pred - 1) < 0.04, (sym, g)


def test_noise_law_heavy_tail_bound():
    W = _f16(wl.student_t_weight(1024, 4096, 12).float().numpy())
    for g in (32, 64, 128):
        q, s, _ = oracle.quantize_pack(W, g, True)
        W_hat = oracle.dequant(q, s, None, 1024, 4096, g, True)
        mse = float(np.mean((W_hat.astype(np.float64) - W) ** 2))
        pred = float(np.mean(oracle.f16_bits_to_f32_array(s).astype(np.float64) ** 2) / 12)
        assert 0.75 <= mse / pred <= 1.02


def test_mse_decreases_with_group_size():
    """Ordering of the MSE-vs-group-size table of "LLM 后训练量化深度实战",
    section 二 (the printed values themselves do not reproduce)."""
    W = _f16(wl.normal_weight(4096, 4096, 0).float().numpy())
    mses = []
    for g in (4096, 512, 128, 32):
        q, s, _ = oracle.quantize_pack(W, g, True)
        W_hat = oracle.dequant(q, s, None, 4096, 4096, g, True)
        mses.append(float(np.mean((W_hat.astype(np.float64) - W) ** 2)))
    assert mses[0] > mses[1] > mses[2] > mses[3]


# --------------------------------------------------------------- products

def _tiny_case(symmetric, g=8, out=6, inn=32, seed=3):
    W = _f16(wl.normal_weight(out, inn, seed).float().numpy())
    q, s, z = oracle.quantize_pack(W, g, symmetric)
    return W, q, s, z


@pytest.mark.parametrize("symmetric", [True, False])
def test_gemv_exact_rational_tiny(symmetric):
    out, inn, g = 6, 32, 8
    _, q, s, z = _tiny_case(symmetric)
    x = wl.activations(3, inn, 9, dtype=torch.bfloat16).float().numpy().astype(np.float64)
    y = oracle.gemv(q, s, z, out, inn, g, symmetric, x)
    W_hat = oracle.dequant(q, s, z, out, inn, g, symmetric)
    for b in range(3):
        for r in range(out):
            exact = sum(Fraction(float(W_hat[r, k])) * Fraction(float(x[b, k])) for k in range(inn))
            mag = sum(abs(float(W_hat[r, k]) * x[b, k]) for k in range(inn))
            assert abs(float(exact) - y[b, r]) <= 1e-15 * mag + 1e-300


@pytest.mark.parametrize("symmetric", [True, False])
def test_gemv_special_cases(symmetric):
    out, inn, g = 16, 256, 32
    W = _f16(wl.normal_weight(out, inn, 4).float().numpy())
    q, s, z = oracle.quantize_pack(W, g, symmetric)
    W_hat = oracle.dequant(q, s, z, out, inn, g, symmetric).astype(np.float64)
    # one-hot x returns a column of W_hat exactly
    for k in (0, 37, 255):
        x = np.zeros((1, inn))
        x[0, k] = 1.0
        assert np.array_equal(oracle.gemv(q, s, z, out, inn, g, symmetric, x)[0], W_hat[:, k])
    # x = 1 on one group returns s * sum(q - z) over that group
    x = np.zeros((1, inn))
    x[0, 64:96] = 1.0
    y = oracle.gemv(q, s, z, out, inn, g, symmetric, x)[0]
    assert np.allclose(y, W_hat[:, 64:96].sum(1), rtol=1e-15, atol=0)
    # scaling x by 2^p scales y by exactly 2^p; rows are independent of batch
    xr = wl.activations(4, inn, 8, dtype=torch.bfloat16).float().numpy().astype(np.float64)
    y1 = oracle.gemv(q, s, z, out, inn, g, symmetric, xr)
    assert np.array_equal(oracle.gemv(q, s, z, out, inn, g, symmetric, xr * 8.0), y1 * 8.0)
    assert np.array_equal(oracle.gemv(q, s, z, out, inn, g, symmetric, xr[2:3])[0], y1[2])
    # a second route: numpy matmul of the dequantised weights
    assert np.allclose(y1, xr @ W_hat.T, rtol=1e-12, atol=1e-12)
    rows = np.array([3, 0, 15])
    assert np.array_equal(oracle.gemv(q, s, z, out, inn, g, symmetric, xr, rows=rows), y1[:, rows])


def test_dense_reference():
    W = wl.normal_weight(8, 64, 2).to(torch.bfloat16).float().numpy()
    x = wl.activations(2, 64, 3).float().numpy().astype(np.float64)
    y = oracle.dense(W, x)
    assert np.allclose(y, x @ W.astype(np.float64).T, rtol=1e-13, atol=1e-15)


def test_bits_per_weight_accounting():
    """Buffer sizes give b + (b_scale + b_zero)/g bits per weight."""
    g = _golden("bits_per_weight.json")
    for row in g["rows"]:
        gs = row["group_size"]
        W = _f16(wl.normal_weight(2, 4096, 1).float().numpy())
        q, s, z = oracle.quantize_pack(W, gs, False)
        n = W.size
        bits_codes_scales = (q.nbytes + s.nbytes) * 8 / n
        # the page counts a 4-bit zero point; ours is stored as fp16 (16 bits)
        assert abs(bits_codes_scales + 4 / gs - row["bits_per_weight"]) < 1e-3 + 1e-9
        assert abs((q.nbytes + s.nbytes + z.nbytes) * 8 / n - (4 + 32 / gs)) < 1e-12
    assert abs((4 + 32 / 128) - g["fp16_scale_fp16_zero_g128"]) < 1e-12


# ---------------------------------------------- range (clipping) search
# arganzheng.life post-training-quantization-gptq-awq-and-rotation, section
# 三.2: scan ranges alpha from 0.8 to 1.0 of max|w|, keep the smallest error.

def _clip_reference(w, n):
    """Independent numpy restatement of one group's search: candidate fp16
    scales, codes rint(w / s) clamped to +-7, fp64 squared error, ties to
    the wider range."""
    w = np.asarray(w, dtype=np.float32)
    a = np.float32(np.max(np.abs(w)))
    K = 5 * (n - 1)
    errs, scales = [], []
    for j in range(n):
        num = a if n == 1 else np.float32(a * np.float32(K - j))
        den = np.float32(7.0) if n == 1 else np.float32(7 * K)
        s = np.float32(np.float16(np.float32(num) / den))
        q = np.zeros_like(w) if s == 0 else np.clip(np.rint(w / s), -7, 7)
        d = w.astype(np.float64) - np.float64(s) * q.astype(np.float64)
        errs.append(float(np.sum(d * d)))
        scales.append(s)
    best = 0
    for j in range(1, n):
        if scales[j] != 0 and errs[j] < errs[best] * (1 - 1e-12):
            best = j
    return best, np.array(errs), np.array(scales)


def test_clip_search_single_candidate_is_rtn():
    W = wl.normal_weight(48, 1024, 41).float().numpy()
    q1, s1, idx = oracle.quantize_pack_clip(W, 128, 1)
    qr, sr, _ = oracle.quantize_pack(W, 128, True)
    assert np.array_equal(q1, qr) and np.array_equal(s1, sr) and not idx.any()


@pytest.mark.parametrize("kind", ["normal", "t3", "uniform"])
def test_clip_search_matches_independent_restatement(kind):
    gen = {"normal": wl.normal_weight, "t3": wl.student_t_weight, "uniform": wl.uniform_weight}[kind]
    W = gen(16, 512, 42).float().numpy()
    for r in range(16):
        for j in range(4):
            w = W[r, j * 128:(j + 1) * 128]
            best, err, s16 = oracle.clip_errors(w, 21)
            rbest, rerr, rs = _clip_reference(w, 21)
            assert best == rbest
            assert np.allclose(err, rerr, rtol=1e-12, atol=0)
            assert np.array_equal(s16.view(np.float16).astype(np.float32), rs)


def test_clip_search_never_worse_than_rtn_and_grid_refinement():
    W = wl.student_t_weight(64, 1024, 43).float().numpy()
    for n_small, n_big in [(21, 41), (5, 9)]:
        _, _, _ = oracle.quantize_pack_clip(W, 128, n_small)
        for r in range(0, 64, 7):
            for j in range(8):
                w = W[r, j * 128:(j + 1) * 128]
                b1, e1, _ = oracle.clip_errors(w, 1)
                bs, es, _ = oracle.clip_errors(w, n_small)
                bb, eb, _ = oracle.clip_errors(w, n_big)
                assert es[bs] <= e1[0]                      # candidate 0 is RTN
                assert eb[bb] <= es[bs] * (1 + 1e-12)        # the small grid is a subset


def test_clip_search_gaussian_optimum_below_max():
    """For large Gaussian groups the best range lies well below max|w| (the
    section puts the 4-bit optimum at 2.5-3 sigma against a max of 4-5
    sigma): every group of 4096 picks the grid's floor, 0.8 max."""
    W = wl.normal_weight(32, 4096, 44).float().numpy()
    _, _, idx = oracle.quantize_pack_clip(W, 4096, 21)
    assert np.all(idx == 20)
    sigma = 0.02
    amax = np.abs(W).max(axis=1) / sigma
    # the floor 0.8 max lies at or above 2.5 sigma: the optimum is below it
    assert np.all(0.8 * amax > 2.5) and np.median(amax) > 3.5


# ------------------------------------------------------------- act-order
# arganzheng.life post-training-quantization-gptq-awq-and-rotation, section
# 五.3 (desc_act, g_idx) and 九.2 (the reorder is a gather).

@pytest.mark.parametrize("sym", [True, False])
def test_act_order_identity_is_plain_quantization(sym):
    W = wl.normal_weight(24, 512, 61).float().numpy()
    a = oracle.quantize_pack_perm(W, 64, sym, np.arange(512, dtype=np.int32))
    b = oracle.quantize_pack(W, 64, sym)
    for x, y in zip(a, b):
        assert (x is None and y is None) or np.array_equal(x, y)


@pytest.mark.parametrize("sym", [True, False])
def test_act_order_groups_follow_g_idx(sym):
    """Column k's code and scale are those of group g_idx[k]: each group's
    scale is the statistic of exactly the columns g_idx assigns to it
    (checked column by column, without building the permuted matrix)."""
    rng = np.random.default_rng(62)
    out, inn, g = 16, 512, 128
    W = wl.student_t_weight(out, inn, 63).float().numpy()
    perm = rng.permutation(inn).astype(np.int32)
    q, s, z = oracle.quantize_pack_perm(W, g, sym, perm)
    gi = oracle.g_idx(perm, g)
    assert np.array_equal(np.bincount(gi), np.full(inn // g, g))
    pos = np.empty(inn, dtype=np.int64)
    pos[perm] = np.arange(inn)
    for r in range(out):
        for t in range(inn // g):
            cols = np.nonzero(gi == t)[0]
            wv = W[r, cols]
            if sym:
                want = np.float16(np.float32(np.max(np.abs(wv))) / np.float32(7.0))
            else:
                want = np.float16(np.float32(np.float32(wv.max()) - np.float32(wv.min())) / np.float32(15.0))
            assert np.uint16(s[r, t]) == want.view(np.uint16)
        # dequantised value of every original column from its own position
        Wh = oracle.dequant(q, s, z, out, inn, g, sym)[r]
        sf = np.asarray(s[r]).view(np.float16).astype(np.float32)
        for k in rng.choice(inn, 16, replace=False):
            j = pos[k]
            code = oracle.code_at(q, inn, r, int(j), sym)
            zz = 0.0 if sym else float(np.asarray(z[r, j // g]).view(np.float16))
            assert Wh[j] == np.float32(sf[j // g] * np.float32(code - zz))


def test_act_order_product_is_a_gather():
    """y = x W_hat^T over original columns equals the product of the stored
    (permuted) weights with the gathered activations x[:, perm]."""
    rng = np.random.default_rng(64)
    out, inn, g = 40, 1024, 128
    W = wl.normal_weight(out, inn, 65).float().numpy()
    perm = rng.permutation(inn).astype(np.int32)
    q, s, _ = oracle.quantize_pack_perm(W, g, True, perm)
    x = wl.activations(3, inn, 66).float().numpy().astype(np.float64)
    y_gather = oracle.gemv(q, s, None, out, inn, g, True, x[:, perm])
    Wp = oracle.dequant(q, s, None, out, inn, g, True).astype(np.float64)
    W_orig = np.empty_like(Wp)
    W_orig[:, perm] = Wp
    assert np.allclose(y_gather, x @ W_orig.T, rtol=1e-12, atol=1e-12)
