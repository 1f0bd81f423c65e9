"""CPU model of the quantizers' division-free rounding.

The CUDA quantizers round w / s without dividing: t = w * r with r the
correctly rounded reciprocal of s, and rint(t) is taken when |t| < 178 and
|t - rint(t)| < 0.5 - 3.2e-5; otherwise the IEEE quotient is rounded.  The
bound |t - fl(w/s)| <= |t| (3u + u^2) < 3.2e-5 (u = 2^-24) makes both give
the same integer.  This test replays that rule in numpy's IEEE binary32
arithmetic (no code shared with the kernels) against rint(fl(w / s)) on
16-bit scales and weights, including constructed exact and near ties, and
checks that the shortcut is taken for almost every ordinary value."""
import numpy as np
import pytest
import torch

f32 = np.float32


def _shortcut(w, s):
    r = (np.float64(1.0) / s.astype(np.float64)).astype(f32)      # correctly rounded 1/s
    r = np.where(np.abs(r) >= f32(1.17549435e-38), r, f32(np.nan))
    with np.errstate(all="ignore"):
        t = (w * r).astype(f32)
        q = np.rint(t)
        fast = (np.abs((t - q).astype(f32)) < f32(0.4999679)) & (np.abs(t) < f32(178))
        exact = np.rint((w / s).astype(f32))
    return np.where(fast, q, exact), exact, fast


def _to16(a, bf16):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16 if bf16 else torch.float16).float().numpy()


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("kind", ["random", "exact_ties", "near_ties"])
def test_shortcut_equals_ieee_rounding(bf16, kind):
    rng = np.random.default_rng(7 + bf16)
    n = 400_000
    s = _to16(rng.uniform(0.5, 1.0, n) * 2.0 ** rng.integers(-14, 8, n), bf16)
    if kind == "random":
        # quotients in the codes' range (|w/s| up to ~130, as the quantizers produce)
        w = _to16(rng.standard_normal(n) * s * rng.choice([3.0, 10.0, 40.0], n), bf16)
    else:
        k = rng.integers(-130, 130, n) + 0.5
        w = (k * s.astype(np.float64)).astype(f32)
        if kind == "near_ties":
            w = np.nextafter(w, np.where(rng.random(n) < 0.5, np.inf, -np.inf).astype(f32)).astype(f32)
        w = _to16(w, bf16)
    ok = np.isfinite(w) & np.isfinite(s) & (s != 0)
    got, exact, fast = _shortcut(w[ok], s[ok])
    assert np.array_equal(got, exact)
    if kind == "random":
        assert fast.mean() > 0.99   # bf16 quotients hit exact ties more often


def test_int8_form_with_stored_cache_scale():
    """The KV-cache form: s = cache_type(amax / 127) of the row, codes clamped
    to [-128, 127]; the float-to-int rounding is the same rule."""
    rng = np.random.default_rng(11)
    rows = 20_000
    mag = 2.0 ** rng.uniform(-12, 12, (rows, 1))
    v = _to16(rng.standard_normal((rows, 128)) * mag, True)
    s = _to16(np.abs(v).max(1, keepdims=True) / f32(127), True)
    got, exact, _ = _shortcut(v, np.broadcast_to(s, v.shape).astype(f32))
    assert np.array_equal(np.clip(got, -128, 127), np.clip(exact, -128, 127))
