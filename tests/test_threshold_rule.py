"""The weight-code threshold rule, checked against IEEE float32 division.

BitNet b1.58 (dmarx anthology record LIT-380, Key takeaways bullet 1) maps a weight to
RoundClip(w / (gamma + eps), -1, 1). For d = gamma + eps > 0 the code is +1 exactly when the
correctly rounded quotient fl(w / d) exceeds 0.5. The GPU kernel never divides: it uses the
fact that fl(t / d) > 0.5 holds exactly when t > d * (0.5 + 2^-25) (the midpoint between 0.5
and the next float; the tie rounds to the even 0.5), a product that is exact in float64, and
takes the smallest float strictly above it as the threshold T. This test checks both claims
with numpy's float32 division (IEEE round-to-nearest-even), including the floats right next
to every threshold, over normal and subnormal d.
"""
import numpy as np


def threshold(d: np.float32) -> np.float32:
    m = np.float64(d) * (0.5 + 2.0 ** -25)  # exact: 24 x 26 significant bits
    t = np.float32(m)
    if np.float64(t) < m:
        t = np.nextafter(t, np.float32(np.inf))
    if np.float64(t) == m:
        t = np.nextafter(t, np.float32(np.inf))
    return t


def qualifies(t: np.float32, d: np.float32) -> bool:
    with np.errstate(over="ignore", under="ignore"):
        return bool(np.float32(t) / np.float32(d) > np.float32(0.5))


def test_threshold_rule_random_and_neighbours():
    rng = np.random.default_rng(1234)
    ds = np.concatenate([
        rng.uniform(1e-4, 1.0, 3000).astype(np.float32),
        (rng.uniform(1.0, 2.0, 1000) * 2.0 ** rng.integers(-120, 120, 1000)).astype(np.float32),
        np.array([1.0, 0.5, 2.0, 3.0, 0.1, 0.0125, 1e-38, 1.5e-39, 1e-45, 3e38], np.float32),
        rng.integers(1, 2 ** 23, 300).astype(np.uint32).view(np.float32),  # subnormal d
    ])
    for d in ds:
        d = np.float32(d)
        if not (d > 0 and np.isfinite(d)):
            continue
        t = threshold(d)
        if not np.isfinite(t):
            continue
        assert qualifies(t, d), (d, t)
        below = np.nextafter(t, np.float32(0))
        assert not qualifies(below, d), (d, t, below)
        # the rule itself on a few floats around the threshold
        tb = int(t.view(np.uint32))
        for k in range(-3, 4):
            if not 0 < tb + k < 0x7f800000:  # positive finite floats only
                continue
            x = np.uint32(tb + k).view(np.float32)
            rule = np.float64(x) > np.float64(d) * (0.5 + 2.0 ** -25)
            assert rule == qualifies(x, d), (d, x)


def test_midpoint_is_never_a_float():
    # d (0.5 + 2^-25) = d (2^24 + 1) 2^-25: d's odd significand times the odd 2^24 + 1 needs at
    # least 25 significant bits, so no float t sits exactly on the midpoint and the
    # round-half-to-even tie never decides a code (the kernel's "step once more" branch is
    # a guard that does not fire).
    rng = np.random.default_rng(99)
    ds = rng.integers(1, 0x7f7fffff, 20000).astype(np.uint32).view(np.float32)
    for d in ds:
        m = np.float64(d) * (0.5 + 2.0 ** -25)
        assert np.float64(np.float32(m)) != m or m == 0.0
