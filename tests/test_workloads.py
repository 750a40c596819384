"""The seeded input generators draw what their recipes state (CPU).

The calibration stand-ins (Student-t(4) and half-normal activations with
outlier channels, correlated Z L activations, Gaussian weights) are checked
against closed-form quantiles and moments of those distributions, with
order statistics where the tails are heavy (a Student-t(4) variable has no
finite fourth moment, so its sample variance converges too slowly to pin).
Bounds are several standard errors wide for the sample sizes used.
"""
import math

import numpy as np
import pytest
import torch
from scipy import stats

import workloads


def _plain_channels(x: torch.Tensor, idx) -> np.ndarray:
    keep = np.setdiff1d(np.arange(x.shape[1]), np.asarray(idx))
    return x.to(torch.float64).numpy()[:, keep]


def test_generators_are_pure_functions_of_their_seed():
    a = workloads.student_t_activations(300, 40, seed=9)
    b = workloads.student_t_activations(300, 40, seed=9)
    c = workloads.student_t_activations(300, 40, seed=10)
    assert a.dtype == torch.bfloat16 and a.shape == (300, 40)
    assert torch.equal(a, b) and not torch.equal(a, c)
    wl = workloads.WORKLOADS["tiny"]
    assert torch.equal(workloads.weights(wl), workloads.weights(wl))
    # replicas draw distinct layers
    assert not torch.equal(workloads.weights(wl, seed_offset=1), workloads.weights(wl))
    assert not torch.equal(workloads.activations(wl, n_tokens=64, seed_offset=1),
                           workloads.activations(wl, n_tokens=64))


def test_gaussian_weights_have_the_stated_spread():
    w = workloads.gaussian_weights(512, 512, 0.02, seed=3).double().numpy().ravel()
    n = w.size
    assert abs(w.mean()) < 5 * 0.02 / math.sqrt(n)
    assert abs(w.std() / 0.02 - 1.0) < 5 / math.sqrt(2 * n)


def test_student_t_activations_follow_t4_with_outlier_channels():
    n, d, frac, scale = 32768, 200, 0.01, 50.0
    x = workloads.student_t_activations(n, d, seed=5, outlier_frac=frac, outlier_scale=scale)
    idx = workloads.outlier_channels(d, frac, 5).numpy()
    assert len(idx) == round(frac * d) == 2
    v = np.abs(_plain_channels(x, idx)).ravel()
    # |T| quantiles of Student-t with 4 degrees of freedom
    for p in (0.5, 0.9, 0.99):
        q = stats.t.ppf(0.5 + p / 2, df=4)
        emp = float(np.mean(v <= q))
        se = math.sqrt(p * (1 - p) / v.size)
        assert abs(emp - p) < 6 * se, (p, emp)
    # the outlier channels carry the same law, 50 times wider
    med_out = np.median(np.abs(x[:, idx].to(torch.float64).numpy()))
    assert abs(med_out / (scale * stats.t.ppf(0.75, df=4)) - 1.0) < 0.03


def test_half_normal_activations_are_nonnegative_with_the_half_normal_law():
    n, d, frac, scale = 32768, 400, 0.005, 30.0
    x = workloads.half_normal_activations(n, d, seed=6, outlier_frac=frac, outlier_scale=scale)
    idx = workloads.outlier_channels(d, frac, 6).numpy()
    assert len(idx) == 2
    v = _plain_channels(x, idx).ravel()
    assert v.min() >= 0.0
    mean = math.sqrt(2 / math.pi)
    sd = math.sqrt(1 - 2 / math.pi)
    assert abs(v.mean() - mean) < 6 * sd / math.sqrt(v.size)
    assert abs(np.median(v) - stats.norm.ppf(0.75)) < 0.01
    assert abs(np.mean(x[:, idx].to(torch.float64).numpy()) / (scale * mean) - 1.0) < 0.02


def test_correlated_activations_span_the_stated_condition():
    """X = Z L: channel j's variance is the squared norm of column j of L, so
    the last channel (only L's diagonal entry 10^-3) has standard deviation
    10^-3 and the first about sqrt(1 + (d - 1) 0.01 / d)."""
    n, d = 20000, 64
    x = workloads.correlated_activations(n, d, seed=8, n_outliers=0).to(torch.float64).numpy()
    sd = x.std(axis=0)
    se = 1 / math.sqrt(2 * n)
    assert abs(sd[-1] / 1e-3 - 1.0) < 6 * se + 4e-3      # bf16 keeps 8 bits
    assert abs(sd[0] / math.sqrt(1 + (d - 1) * 0.01 / d) - 1.0) < 6 * se + 4e-3
    x4 = workloads.correlated_activations(n, d, seed=8, n_outliers=4, outlier_scale=20.0)
    idx = workloads.outlier_channels(d, 0.0, 8, count=4).numpy()
    sd4 = x4.to(torch.float64).numpy().std(axis=0)
    assert np.allclose(sd4[idx] / sd[idx], 20.0, rtol=1e-2)


@pytest.mark.parametrize("name", sorted(workloads.WORKLOADS))
def test_workload_table_matches_its_description(name):
    wl = workloads.WORKLOADS[name]
    assert wl.block_size == 128 and wl.bits in (2, 3, 4, 8)
    if name != "tiny":
        assert wl.n_tokens == 128 * 2048      # 128 sequences of 2048 tokens
        assert wl.damp == 0.01
    x = workloads.activations(wl, n_tokens=8)
    assert x.shape == (8, wl.d_col) and x.dtype == torch.bfloat16
