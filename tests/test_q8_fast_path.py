"""The fused decode kernel's Q8_0 of x takes q = round(v * RN(1/d)) unless that
product lies within 1e-4 of a half-integer (or is out of range), where it divides.
This checks, in fp32 on the host, that the shortcut gives the same integer as
rounding the correctly rounded quotient RN(v / d) (the Q8_0 definition: d =
max|v| / 127, q = round half away from zero, clamp to +-127) on random blocks
over a wide range of scales and on blocks built to land on exact ties."""
import numpy as np


def _round_away(x):
    return np.where(x >= 0, np.floor(x + 0.5), -np.floor(-x + 0.5))


def _codes(v):
    v = v.astype(np.float32)
    d = (np.max(np.abs(v), axis=1, keepdims=True) / np.float32(127)).astype(np.float32)
    keep = d[:, 0] != 0
    v, d = v[keep], d[keep]
    exact = np.clip(_round_away((v / d).astype(np.float32).astype(np.float64)), -127, 127)
    with np.errstate(over="ignore", invalid="ignore"):  # 1/d may overflow: t is then inf and divides
        r = (np.float32(1) / d).astype(np.float32)
        t = (v * r).astype(np.float32)
        a = np.abs(t)
        fast_ok = (a <= 128) & (np.abs(a - np.floor(a) - np.float32(0.5)) >= np.float32(1e-4))
    fast = np.clip(_round_away(np.where(fast_ok, t, 0).astype(np.float64)), -127, 127)
    shortcut = np.where(fast_ok, fast, exact)
    return exact, shortcut, fast_ok


def test_reciprocal_shortcut_matches_division_on_random_blocks():
    rng = np.random.default_rng(11)
    v = rng.standard_normal((100_000, 32)) * np.exp(rng.uniform(-30, 30, (100_000, 1)))
    exact, shortcut, fast_ok = _codes(v)
    assert np.array_equal(exact, shortcut)
    assert fast_ok.mean() > 0.99  # the division is the rare path


def test_reciprocal_shortcut_matches_division_on_ties():
    # max |v| = 254 * 2^s makes d = 2^(s+1) and every odd multiple of 2^s an exact tie
    rng = np.random.default_rng(12)
    n = 50_000
    blk = (rng.integers(-126, 127, (n, 32)) * 2 + 1).astype(np.float64)
    blk[:, 0] = np.where(rng.random(n) < 0.5, 254.0, -254.0)
    v = blk * np.exp2(rng.integers(-120, 100, (n, 1)).astype(np.float64))
    exact, shortcut, fast_ok = _codes(v)
    assert np.array_equal(exact, shortcut)
    assert not fast_ok[:, 1:].any()  # every tie goes to the division
    # ties under scales whose reciprocal rounds either way: d = m 2^e with m odd
    # and below 2^15, max |v| = 127 d, v = (2 k + 1) d / 2 (all exact in fp32)
    m = (rng.integers(0, 2**14, (n, 1)) * 2 + 1).astype(np.float64)
    dd = m * np.exp2(rng.integers(-40, 40, (n, 1)).astype(np.float64))
    u = (rng.integers(-127, 127, (n, 32)) * 2 + 1) * dd / 2
    u[:, 0] = 127 * dd[:, 0]
    exact, shortcut, fast_ok = _codes(u)
    assert np.array_equal(exact, shortcut)
    # values a few ulps off a tie, on both sides (d = 2)
    k = rng.integers(-126, 126, (n, 31)) + 0.5
    off = rng.integers(-8, 9, (n, 31)) * np.float64(np.spacing(np.float32(100.0)))
    w = np.concatenate([np.full((n, 1), 254.0), (k * 2.0 + off)], axis=1)
    exact, shortcut, _ = _codes(w)
    assert np.array_equal(exact, shortcut)


def test_reciprocal_shortcut_near_fp32_limits():
    # tiny blocks (1/d overflows below d = 2^-128) and large ones
    rng = np.random.default_rng(13)
    for s in (-149, -140, -130, -127, -126, 100, 120):
        v = rng.standard_normal((20_000, 32)) * np.exp2(float(s))
        exact, shortcut, _ = _codes(v)
        assert np.array_equal(exact, shortcut), s
