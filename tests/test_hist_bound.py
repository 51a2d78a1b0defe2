"""The forward kernel filters histogram-pass candidates with a closed-form lower
bound of tau_h (the root of the reduced histogram problem, AdaSplash-2 zh
§2.1): for each bin b, the C_b scores of bins b..top, whose lower edges
average mean_b, give sum c [x - tau]_+^k >= C_b (mean_b - tau)^k for
tau <= x_b, so tau_h >= min(x_b, mean_b - C_b^(-1/k)).  These CPU checks pin
that inequality (and equality at alpha = 2) against the oracle's tau_h."""

import numpy as np
import pytest

import oracle as O


def moment_bound(s, alpha, n_bins):
    """max over b of min(x_b, mean_b - C_b^(-1/k)) on the max-anchored grid."""
    k = 1.0 / (alpha - 1.0)
    gtop = int(np.floor(n_bins * s.max()))
    g = np.floor(n_bins * s).astype(np.int64)
    best, c_tot, a_tot = -np.inf, 0, 0.0
    for b in range(n_bins, -1, -1):
        x_b = (gtop - n_bins + b) / n_bins
        c_b = int(np.sum(g == gtop - n_bins + b))
        c_tot += c_b
        a_tot += c_b * x_b
        if c_tot:
            best = max(best, min(x_b, a_tot / c_tot - c_tot ** (-1.0 / k)))
    return best


@pytest.mark.parametrize("alpha", [1.5, 2.0])
@pytest.mark.parametrize("temp", [0.5, 1.0, 4.0])
def test_moment_bound_below_tau_h(alpha, temp):
    rng = np.random.default_rng(int(10 * temp + 100 * alpha))
    for _ in range(40):
        n = int(rng.integers(1, 3000))
        s = (alpha - 1.0) * temp * rng.standard_normal(n)
        tau_h = O.histogram_threshold(s, alpha, 8, anchor="grid")
        lb = moment_bound(s, alpha, 8)
        assert lb <= tau_h + 1e-12
        if alpha == 2.0:   # the bound is tau_h itself
            assert lb == pytest.approx(tau_h, abs=1e-9)
        else:              # and close to it: within one bin
            assert tau_h - lb <= 1.0 / 8 + 1e-12


def test_moment_bound_single_score():
    # one score: the bound and tau_h both equal its bin edge minus 1
    s = np.array([0.3])
    assert moment_bound(s, 1.5, 8) == pytest.approx(O.histogram_threshold(s, 1.5, 8), abs=1e-12)
