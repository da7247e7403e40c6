"""The NVFP4 encoders take a block's E4M3 scale byte from one product, ta = amax * c6 with
c6 = 1/(6g), instead of the two divisions (amax/6)/g that define it. They do so only where
ta is a normal E4M3 value (>= 2^-6), finite, and more than 32 binary32 units away from an
E4M3 rounding midpoint (mantissa bits 19..0 = 0x80000); everywhere else they take the two
divisions. The argument: ta and the quotient differ by fewer than 6 units. This test replays
the rule in binary32 with numpy, on random and adversarial (amax, g) pairs, and checks that
every case it takes gives the byte of the definition. It also checks that the margin matters:
near the midpoints the product alone would round to another byte.
"""
import ml_dtypes
import numpy as np

F32 = np.float32


def e4m3(x):
    """E4M3 byte, round to nearest even, saturating at +-448."""
    x = np.asarray(x, np.float32)
    r = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8).copy()
    big = np.abs(x) > 448.0
    r[big] = np.where(np.signbit(x[big]), 0xFE, 0x7E)
    return r


def shortcut(amax, g):
    """(taken, byte of ta, byte of the definition) for float32 arrays amax, g."""
    with np.errstate(over="ignore", invalid="ignore", divide="ignore"):
        c6 = F32(1) / (F32(6) * g)
        ta = amax * c6
        t = (amax / F32(6)) / g
    off = (ta.view(np.uint32) & 0xFFFFF).astype(np.int64) - 0x80000
    taken = (ta >= F32(2.0 ** -6)) & np.isfinite(ta) & (np.abs(off) > 32)
    return taken, e4m3(ta), e4m3(t)


def random_pairs(rng, n):
    g = (rng.uniform(1, 2, n) * 2.0 ** rng.integers(-30, 31, n)).astype(F32)
    t = 2.0 ** rng.uniform(-14, np.log2(448.0), n)  # the block's scale before rounding
    amax = (t * 6.0 * g.astype(np.float64)).astype(F32)
    return amax, g


def test_random_pairs_match_the_definition():
    rng = np.random.default_rng(11)
    amax, g = random_pairs(rng, 4_000_000)
    taken, fast, exact = shortcut(amax, g)
    # above the smallest normal E4M3 value (quotients just under 2^-6 that round up to it
    # are left to the divisions) only the midpoint neighbourhoods, 65 in 2^20, take them
    normal = exact > 0x08
    assert taken[normal].mean() > 0.9995
    bad = np.nonzero(taken & (fast != exact))[0]
    assert bad.size == 0, (amax[bad[:5]], g[bad[:5]])


def test_near_every_midpoint_the_rule_is_exact_and_the_margin_is_needed():
    rng = np.random.default_rng(12)
    amax_l, g_l = [], []
    for e in range(-6, 9):  # every binade of normal E4M3 values
        for k in range(8):  # every midpoint in it: (1 + (2k+1)/16) * 2^e
            mid = (1.0 + (2 * k + 1) / 16.0) * 2.0 ** e
            for d in range(-48, 49):  # binary32 units from the midpoint
                g = (rng.uniform(1, 2, 24) * 2.0 ** rng.integers(-12, 13, 24)).astype(F32)
                amax_l.append((mid * (1.0 + d * 2.0 ** -23) * 6.0 * g.astype(np.float64)).astype(F32))
                g_l.append(g)
    amax, g = np.concatenate(amax_l), np.concatenate(g_l)
    taken, fast, exact = shortcut(amax, g)
    bad = np.nonzero(taken & (fast != exact))[0]
    assert bad.size == 0, (amax[bad[:5]], g[bad[:5]])
    # the product alone would be wrong on some of the cases the rule sends to the divisions
    assert np.count_nonzero(~taken & (fast != exact)) > 0
    assert taken.mean() > 0.2  # and the cases further out do take the product


def test_special_values_take_the_divisions_or_match():
    amax = np.array([0.0, 1e-45, 3e38, np.inf, np.nan, 1.0, 1.0], F32)
    g = np.array([1.0, 1.0, 1e-30, 1.0, 1.0, 0.0, np.inf], F32)
    taken, fast, exact = shortcut(amax, g)
    assert not taken[3] and not taken[4]  # non-finite inputs
    assert not taken[5] and not taken[6]  # g = 0 or inf: c6 is inf or 0
    assert np.array_equal(fast[taken], exact[taken])
