"""The seeded synthetic inputs follow their stated recipes (CPU only).

Checked against closed forms with a fixed seed:
  - normal weights: standard deviation;
  - the robustness weight, Student-t with 3 degrees of freedom scaled to
    standard deviation 0.02 with 0.1% of entries multiplied by 20: the median
    of |w| and the two-sided tail mass of the mixture above a threshold, both
    from the t distribution's quantile and survival functions;
  - the same seed gives the same bits.
"""
import math

import numpy as np
import torch
from scipy import stats

from bit_nf4_quantized_12_b200 import workloads


def _f64(t):
    return t.float().numpy().astype(np.float64).reshape(-1)


def test_normal_weight_scale():
    w = _f64(workloads.weight(1024, 2048, 0.02, seed=5))
    assert abs(w.std() / 0.02 - 1) < 0.01          # 2M samples: standard error ~0.05%
    assert abs(w.mean()) < 1e-4


def test_student_t_outlier_weight_recipe():
    rows, cols = 2048, 2048
    w = np.abs(_f64(workloads.weight(rows, cols, 0.02, seed=3, kind="student_t_outliers")))
    sigma = 0.02 / math.sqrt(3.0)                   # scale of t(3) with standard deviation 0.02
    # median of |w|: the mixture is 99.9% unscaled t, so its median moves only slightly
    p_out = 0.001
    med = stats.t.ppf(0.75, 3) * sigma
    # exact median of the mixture |w|: solve (1-p) F(m/s) + p F(m/20s) = 1/2 for the |t| CDF
    f = lambda m: (1 - p_out) * (2 * stats.t.cdf(m / sigma, 3) - 1) + p_out * (2 * stats.t.cdf(m / (20 * sigma), 3) - 1) - 0.5
    lo, hi = 0.5 * med, 2 * med
    for _ in range(100):
        mid = (lo + hi) / 2
        lo, hi = (mid, hi) if f(mid) < 0 else (lo, mid)
    assert abs(np.median(w) / lo - 1) < 0.01
    # tail mass above 40 sigma: far beyond the unscaled t, well inside the x20 part
    tau = 40 * sigma
    expect = (1 - p_out) * 2 * stats.t.sf(tau / sigma, 3) + p_out * 2 * stats.t.sf(tau / (20 * sigma), 3)
    got = np.mean(w > tau)
    se = math.sqrt(expect * (1 - expect) / w.size)
    assert abs(got - expect) < 5 * se, (got, expect, se)


def test_inputs_are_reproducible():
    a = workloads.weight(64, 128, 0.02, seed=9, kind="student_t_outliers")
    b = workloads.weight(64, 128, 0.02, seed=9, kind="student_t_outliers")
    assert torch.equal(a, b)
    io1 = workloads.layer_inputs(8, 64, 128, 16, seed=2)
    io2 = workloads.layer_inputs(8, 64, 128, 16, seed=2)
    assert all(torch.equal(io1[k], io2[k]) for k in io1)
    x = _f64(workloads.layer_inputs(256, 64, 4096, 16, seed=4)["X"])
    assert abs(x.std() - 1) < 0.01
