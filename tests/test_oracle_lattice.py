"""Pins for the oracle's E8 quantiser (paper page abstract: E8 lattice quantisation of row-normalised weights).

The quantiser is pinned by facts that do not depend on it:
- brute-force enumeration of every nearby point of D8 and D8+½;
- the defining invariants of E8: membership, a covering radius of 1, and invariance under lattice translation;
- the closed-form normalised second moment G(E8) = 929/12960 (Conway & Sloane, SPLAG, ch. 21).
"""
import itertools

import numpy as np
import pytest

pytestmark = pytest.mark.filterwarnings("ignore")


def brute_force_e8(x):
    """Nearest E8 point by enumeration. Within the covering radius (1) every
    coordinate of the answer lies within 1 of x, so these candidates suffice."""
    best, best_d = None, np.inf
    for half in (0.0, 0.5):
        ranges = []
        for xi in x:
            lo = int(np.ceil(xi - 1.0 - half))
            hi = int(np.floor(xi + 1.0 - half))
            ranges.append(range(lo, hi + 1))
        cand = np.array(list(itertools.product(*ranges)), dtype=np.int64)
        cand = cand[(cand.sum(axis=1) % 2) == 0]
        pts = cand + half
        d = ((pts - x) ** 2).sum(axis=1)
        k = int(np.argmin(d))
        if d[k] < best_d:
            best_d, best = d[k], pts[k]
    return best


def as_point(b, u):
    return np.asarray(u, dtype=np.float64) + 0.5 * b


def in_e8(p):
    two = 2 * p
    if not np.all(two == np.round(two)):
        return False
    frac = p - np.floor(p)
    if not (np.all(frac == 0) or np.all(frac == 0.5)):
        return False
    return int(round(p.sum())) % 2 == 0


def test_nearest_matches_brute_force(orc):
    rng = np.random.default_rng(1234)
    for scale in (0.3, 1.0, 4.0, 40.0):
        for _ in range(300):
            x = rng.normal(size=8) * scale
            b, u = orc.e8_nearest(x)
            p = as_point(b, u)
            q = brute_force_e8(x)
            assert np.allclose(((p - x) ** 2).sum(), ((q - x) ** 2).sum(), rtol=0, atol=1e-12), (x, p, q)
            assert np.array_equal(p, q), (x, p, q)


def test_invariants_membership_covering_translation(orc):
    rng = np.random.default_rng(7)
    for _ in range(3000):
        x = rng.uniform(-6, 6, size=8)
        b, u = orc.e8_nearest(x)
        p = as_point(b, u)
        assert in_e8(p)
        assert int(np.sum(u)) % 2 == 0  # u ∈ D8 in both cosets
        assert ((x - p) ** 2).sum() <= 1.0 + 1e-12  # covering radius of E8 is 1
        # translation by a lattice vector λ: Q(x + λ) = Q(x) + λ
        lam = rng.integers(-5, 6, size=8).astype(np.float64)
        if int(lam.sum()) % 2:
            lam[0] += 1
        if rng.random() < 0.5:
            lam = lam + 0.5
            if int(round((lam - 0.5).sum())) % 2:
                lam[1] += 1
        assert in_e8(lam)
        b2, u2 = orc.e8_nearest(x + lam)
        assert np.array_equal(as_point(b2, u2), p + lam)


def test_hand_worked_points(orc):
    # Each case can be checked by hand against the two cosets.
    cases = [
        (np.full(8, 0.6), np.full(8, 0.5)),     # D8 gives 1^8 at d²=1.28; D8+½ gives (½)^8 at 0.08
        (np.zeros(8), np.zeros(8)),
        (np.array([0.9, 0.1, 0, 0, 0, 0, 0, 0]), np.array([1.0, 1.0, 0, 0, 0, 0, 0, 0])),
        (np.array([1.2, 0, 0, 0, 0, 0, 0, 0]), np.array([2.0, 0, 0, 0, 0, 0, 0, 0])),  # d² 0.64 < 1.04 of (1,1,0..)
        (np.array([-0.7, -0.7, 0.1, 0, 0, 0, 0, 0]), np.array([-1.0, -1.0, 0, 0, 0, 0, 0, 0])),
    ]
    for x, want in cases:
        b, u = orc.e8_nearest(x)
        got = as_point(b, u)
        if not np.array_equal(got, want):
            # (0.9,0.1,0..) is a tie: (0,..) and (1,1,0..) are both at d² = 0.82. Only the distance is pinned.
            assert np.isclose(((got - x) ** 2).sum(), ((want - x) ** 2).sum()), (x, got, want)
            assert in_e8(got)


def test_second_moment_closed_form(orc):
    """Mean of ||x - Q(x)||²/8 over uniform x → G(E8) = 929/12960 ≈ 0.0716821.
    Z^8 would give 1/12 ≈ 0.0833 and D8 0.0766, so this also pins the coset choice."""
    rng = np.random.default_rng(99)
    n = 40000
    vals = np.empty(n)
    for i in range(n):
        x = rng.uniform(0, 64, size=8)
        b, u = orc.e8_nearest(x)
        vals[i] = ((x - as_point(b, u)) ** 2).sum() / 8.0
    g = 929.0 / 12960.0
    sem = vals.std() / np.sqrt(n)
    assert abs(vals.mean() - g) < 4 * sem, (vals.mean(), g, sem)
