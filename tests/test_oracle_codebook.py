"""Pins for the oracle's NF4 codebook (CPU only).

What the pages fix ("从LoRA到QLoRA" §2.3; "QLoRA 原理精讲" §2.1): 16 values,
quantiles of N(0,1) sampled uniformly in probability, normalized to [-1, 1],
bins of (near) equal probability mass.  The checks below use scipy's normal
CDF, which the oracle does not use, so a wrong quantile, offset, sort or
normalization in the oracle fails here.
"""
import numpy as np
import pytest
from scipy.special import ndtr, ndtri

import oracle

DELTA = 0.5 * ((1 - 1 / 30) + (1 - 1 / 32))


@pytest.fixture(scope="module")
def codes():
    return oracle.codebook().astype(np.float64)


def test_shape_order_endpoints(codes):
    assert codes.shape == (16,)
    assert np.all(np.diff(codes) > 0), "codes must ascend strictly"
    assert codes[0] == -1.0 and codes[15] == 1.0
    assert codes[7] == 0.0, "exact zero at index 7"
    assert np.sum(codes > 0) == 8 and np.sum(codes < 0) == 7


def test_codes_are_normal_quantiles_uniform_in_probability(codes):
    # c = Phi^-1(p) / Phi^-1(delta): mapping back through an independent CDF
    # must give probabilities in arithmetic progression from delta toward 1/2.
    zstar = ndtri(DELTA)
    pos = codes[8:][::-1]               # 1, 0.72, ..., 0.08
    neg = -codes[:7]                    # 1, 0.70, ..., 0.09
    p_pos = ndtr(pos * zstar)
    p_neg = ndtr(neg * zstar)
    want_pos = DELTA + (0.5 - DELTA) * np.arange(8) / 8
    want_neg = DELTA + (0.5 - DELTA) * np.arange(7) / 7
    # fp32 rounding of a code moves p by at most phi(z)*z*2^-24 < 1e-7
    assert np.max(np.abs(p_pos - want_pos)) < 2e-7
    assert np.max(np.abs(p_neg - want_neg)) < 2e-7


def _bin_masses(codes):
    zstar = ndtri(DELTA)
    mids = (codes[:-1] + codes[1:]) / 2 * zstar
    edges = np.concatenate([[-np.inf], mids, [np.inf]])
    return np.diff(ndtr(edges))


def test_bins_near_equiprobable(codes):
    m = _bin_masses(codes) * 16
    assert abs(m.sum() - 16) < 1e-12
    assert m.min() > 0.85 and m.max() < 1.15, m


def test_sampled_histogram_matches_masses(codes):
    rng = np.random.default_rng(1234)
    z = rng.standard_normal(10_000_000)
    x = np.clip(z / ndtri(DELTA), -1, 1).astype(np.float32)
    q = oracle.nearest_code(x, np.float32(1.0))
    frac = np.bincount(q, minlength=16) / z.size
    want = _bin_masses(codes)
    assert np.max(np.abs(frac / want - 1)) < 0.005
