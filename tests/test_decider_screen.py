"""The fp32 screen of the [ART] 2.2 stability test used by the tensor-core decode's decider.

The kernel first evaluates the test's two quantities in fp32 on the probe values and decides
only when a value lies farther from its threshold than a proven bound on the distance to the
defining fp64 evaluation (``oracle.probe_step``): 8u(|x| + |x'| + ds) for the norm difference,
32u for the direction term, u = 2^-24, both squared norms in [2^-60, 2^60]. Otherwise it runs
the fp64 evaluation. This file restates that fp32 arithmetic step by step in numpy (products
rounded to fp32, the warp's xor-butterfly sums, rounded root and divide) and checks, over
random and adversarial probe pairs with thresholds placed within a few ulps of the computed
values, that the screen never decides differently from the fp64 test. It pins the bound, not
the CUDA code (whose decisions the GPU tests compare with the oracle)."""
import math

import numpy as np
import pytest

from oracle import bsa_oracle as O

U = np.float32(2.0 ** -24)
F = np.float32


def _lane_terms(a, b):
    """Per-lane fp32 terms a_i b_i + a_{i+32} b_{i+32} of 64 padded coordinates."""
    pa = np.zeros(64, np.float32)
    pb = np.zeros(64, np.float32)
    pa[:a.size] = a
    pb[:b.size] = b
    return (pa[:32] * pb[:32]).astype(np.float32) + (pa[32:] * pb[32:]).astype(np.float32)


def _warp_sum(v):
    """Lane i adds lane i ^ off for off = 16, 8, 4, 2, 1 (fp32 each); every lane ends equal."""
    v = v.astype(np.float32)
    idx = np.arange(32)
    for off in (16, 8, 4, 2, 1):
        v = (v + v[idx ^ off]).astype(np.float32)
    assert np.all(v == v[0])
    return v[0]


def screen(x, xp, tau, phi):
    """1 / 0 when the fp32 screen decides stable / unstable, -1 when it leaves it to fp64."""
    x = np.asarray(x, np.float32)
    xp = np.asarray(xp, np.float32)
    tau, phi = F(tau), F(phi)
    if not tau > 0:
        return 0
    s32 = _warp_sum(_lane_terms(x, x))
    sp32 = _warp_sum(_lane_terms(xp, xp))
    d32 = _warp_sum(_lane_terms(x, xp))
    lo, hi = F(2.0 ** -60), F(2.0 ** 60)
    if not (lo <= s32 <= hi and lo <= sp32 <= hi and np.isfinite(d32)):
        return -1
    n32, np32 = np.sqrt(s32), np.sqrt(sp32)
    ds32 = F(abs(F(n32 - np32)))
    e1 = F(F(8) * U) * F(F(n32 + np32) + ds32)
    if F(ds32 - e1) >= tau:
        return 0
    if not F(ds32 + e1) < tau:
        return -1
    dd32 = F(F(1) - F(d32 / F(n32 * np32)))
    e2 = F(32) * U
    if F(dd32 + e2) < phi:
        return 1
    if F(dd32 - e2) >= phi:
        return 0
    return -1


def fp64_decision(x, xp, tau, phi):
    ds, dd = O.probe_step(xp, x)
    return int(ds < float(F(tau)) and dd < float(F(phi)))


def _cases(rng, n_cases):
    for _ in range(n_cases):
        n = int(rng.integers(1, 65))
        scale = 2.0 ** float(rng.uniform(-25, 25))
        xp = (rng.standard_normal(n) * scale).astype(np.float32)
        # consecutive probes of a converging stream: a relative change from 1e-1 down to 1e-8
        eps = 10.0 ** float(rng.uniform(-8, -1))
        x = (xp * (1 + eps * rng.standard_normal(n))).astype(np.float32)
        yield x, xp


def test_screen_matches_fp64_near_the_thresholds():
    rng = np.random.default_rng(2024)
    decided = undecided = 0
    for x, xp in _cases(rng, 3000):
        ds, dd = O.probe_step(xp, x)
        # thresholds at the computed values, a few ulps either side, and far away
        taus = [ds * (1 + k * 1e-7) for k in (-40, -3, -1, 0, 1, 3, 40)] + [1e30]
        phis = [dd * (1 + k * 1e-7) for k in (-40, -3, -1, 0, 1, 3, 40)] + [dd + 1e-7, 2.0]
        for tau in taus:
            for phi in phis:
                if not (np.isfinite(F(tau)) and np.isfinite(F(phi))):
                    continue
                v = screen(x, xp, tau, phi)
                if v < 0:
                    undecided += 1
                    continue
                decided += 1
                assert v == fp64_decision(x, xp, tau, phi), (x, xp, tau, phi, ds, dd)
    # the screen settles most cases away from the threshold and leaves the band to fp64
    assert decided > 0 and undecided > 0


def test_screen_decides_far_from_the_thresholds():
    """Away from both thresholds the screen must decide (or the fp64 path would run on
    every block)."""
    rng = np.random.default_rng(7)
    for x, xp in _cases(rng, 500):
        ds, dd = O.probe_step(xp, x)
        if not (math.isfinite(ds) and math.isfinite(dd)):
            continue
        n = float(np.linalg.norm(x.astype(np.float64))) + float(np.linalg.norm(xp.astype(np.float64)))
        if n < 2.0 ** -29 or n > 2.0 ** 29:
            continue
        far_tau = ds + 1e-3 * n + 1e-30
        assert screen(x, xp, far_tau, max(dd, 0.0) + 1e-3) == 1
        assert screen(x, xp, ds / 2 if ds > 1e-3 * n else 0.0, 2.0) in (0, -1)
        if ds > 1e-4 * n:
            assert screen(x, xp, ds / 2, 2.0) == 0


@pytest.mark.parametrize("tau", [0.0, -1.0, float("nan")])
def test_screen_non_positive_tau_is_never_stable(tau):
    x = np.ones(8, np.float32)
    assert screen(x, x, tau, 2.0) == 0
    assert fp64_decision(x, x, tau, 2.0) == 0


def test_screen_leaves_extreme_scales_to_fp64():
    x = np.full(4, 2.0 ** -40, np.float32)     # squared norm below 2^-60
    assert screen(x, x, 1.0, 2.0) == -1
    y = np.full(4, 2.0 ** 40, np.float32)      # squared norm above 2^60
    assert screen(y, y, 1.0, 2.0) == -1
    z = np.zeros(4, np.float32)
    assert screen(z, x, 1.0, 2.0) == -1
